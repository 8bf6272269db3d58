// fh_api.cu — the C ABI declared in include/flashhead.h: argument checks, workspace layout and the
// launch sequence of each call.  All device work is done by the kernels in fh_kernels.cu.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <new>

#include "../../include/flashhead.h"
#include "fh_device.cuh"
#include "fh_kernels.cuh"
#include "fh_nvtx.cuh"

struct fh_index {
  fh_index_desc desc;
  int num_sms;
  int device;
};

namespace {

thread_local char g_err[512] = "";

fh_status fail(fh_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

fh_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FH_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr size_t kHeaderBytes = 1024 + 4096;  // control words, then the score histogram
constexpr size_t kGenOffset = 536;             // batch-1 head: tag of the last completed call
constexpr size_t kTcTicketOffset = 544;        // tensor-core head: arrival ticket (zero between calls)
constexpr size_t kKeysReadyOffset = 552;       // batch-1 head: arrivals before its full selection
constexpr size_t kArriveOffset = 556;          // batch-1 head: blocks done (zero between calls)
constexpr size_t kUnionTicketOffset = 560;     // batched union Stage 2: arrival ticket (zero between calls)
constexpr size_t kBestOffset = 568;            // batch-1 head: the call's packed maximum (zero between calls)
constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace regions of one call; offsets from the workspace base.
struct Layout {
  size_t keys = 0, sel = 0, part = 0, bucket = 0, qmask = 0, best = 0, tiles = 0, z = 0, s = 0,
         zmax = 0, Z = 0,
         cluster_of = 0, per_draw = 0;
  size_t total = 0;
};

// The query masks (c words), the flags of the 128-row tiles of the cluster-major copy and the count of
// the list that follows them: one region, zeroed before each batched Stage 2.
int64_t tile_count_of(const fh_index_desc& D) { return (D.v + 127) / 128; }
size_t qmask_region_bytes(const fh_index_desc& D) { return (size_t)D.c * 8 + (size_t)(tile_count_of(D) + 1) * 4; }

Layout layout_for(const fh_index* idx, int op, int B, int p, int T, int64_t N) {
  const fh_index_desc& D = idx->desc;
  Layout L;
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up(off + bytes);
    return at;
  };
  if (op == FH_OP_GREEDY || op == FH_OP_SAMPLE) {
    const int64_t P = (int64_t)p * D.b;
    const int G = fh::stage2_blocks(P, B, idx->num_sms);
    L.keys = take((size_t)B * D.c * 4);
    L.sel = take((size_t)B * p * 4);
    L.part = take((size_t)G * B * 8);
    if (B > 1) {  // batched Stage 2: per-cluster query masks, then per-tile flags and the list's count
      // (cleared together by each call's selection kernel), the arg-maxima, the listed clusters or tiles
      L.qmask = take(qmask_region_bytes(D));
      L.best = take((size_t)B * 8);
      L.tiles = take((size_t)std::max<int64_t>(D.c, (D.v + 127) / 128) * 4);
    }
    if (B == 1 && fh::head1_threads(D.c) != 0) {  // the persistent batch-1 kernel's word table
      L.bucket = take((size_t)fh::kHead1Bins * fh::kHead1BucketCap * 8);
    }
  } else if (op == FH_OP_DENSE) {
    const int G = fh::stage2_blocks(D.v, B, idx->num_sms);
    L.part = take((size_t)G * B * 8);
    L.best = take((size_t)B * 8);
  } else if (op == FH_OP_MC) {
    const int G = fh::stage2_blocks(D.v, B, idx->num_sms);
    L.part = take((size_t)G * B * 8);
    L.z = take((size_t)B * D.v * 4);
    L.s = take((size_t)B * D.c * 4);
    L.zmax = take((size_t)B * 4);
    L.Z = take((size_t)B * D.c * 8);
    L.cluster_of = take((size_t)D.v * 4);
    L.per_draw = take((size_t)B * N * T * 8);
    L.best = take((size_t)B * 8);
  }
  L.total = off;
  return L;
}

fh_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(FH_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % kAlign)
    return fail(FH_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(FH_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  return FH_OK;
}

// Workspace header (first kHeaderBytes): status word at 0, per-query tickets at 16 (64 x 4 bytes),
// the persistent head's call generation at 536 (the tag of the last completed call), the tensor-core
// head's ticket at 544, the persistent head's key-arrival count at 552 and its count of finished
// blocks at 556, the union Stage 2's ticket at 560, the persistent head's packed arg-max at 568; bytes
// [1024, 5120) hold its 1024-bin score histogram in every layout, so no other call ever writes there.
// The per-query tickets, the key-arrival count and the generation only grow; the other tickets, the
// finished-block count, the arg-max and the histogram return to zero at the end of every call, and
// the word table is tagged with the call generation.
// A new workspace must start zeroed (fh_ws_status re-zeroes the header after a device-side error,
// keeping the generation moving; a workspace whose call failed must pass through it before reuse).
uint32_t* status_of(void* ws) { return reinterpret_cast<uint32_t*>(ws); }
uint32_t* tickets_of(void* ws) { return reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 16); }
uint32_t* word_at(void* ws, size_t off) { return reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + off); }

// The tensor-core path: BF16 E (and, for FlashHead, its cluster-major copy), batches up to 64.  The
// dense head and FlashHead's Stage-1 keys take it from 2 queries on (measured at the Llama-3.2-1B
// shape: Stage-1 keys 16 µs at 16 queries, the CUDA-core kernel 24.5 µs at 4); FlashHead's Stage 2
// above kUnionMaxBatch (the union kernel 70 / 103 / 124 µs a call at 4 / 12 / 16 queries against
// 73 / 145 / 148 µs before it; at 24 and 32 queries its 8-warp form, all that fits beside the query
// vectors, took 237 and 290 µs against the tensor cores' 155 and 158 µs).
constexpr int kTcMinBatchDense = 2;
#ifndef FH_TC_MIN_BATCH_STAGE1
#define FH_TC_MIN_BATCH_STAGE1 2
#endif
constexpr int kTcMinBatchStage1 = FH_TC_MIN_BATCH_STAGE1;
#ifndef FH_UNION_MAX_BATCH
#define FH_UNION_MAX_BATCH 16
#endif
constexpr int kUnionMaxBatch = FH_UNION_MAX_BATCH;
bool tc_eligible(const fh_index* idx, int B, int min_batch) {
  const fh_index_desc& D = idx->desc;
  return B >= min_batch && D.dtype == FH_BF16 && fh::tc_supported(fh::kBF16, D.d, B);
}

fh_status check_batch(const fh_index* idx, const void* H, int B) {
  if (!idx) return fail(FH_ERR_ARG, "index handle is NULL");
  if (!H) return fail(FH_ERR_ARG, "H is NULL");
  if (!aligned16(H)) return fail(FH_ERR_ARG, "H must be 16-byte aligned");
  if (B < 1 || B > FH_MAX_BATCH) return fail(FH_ERR_ARG, "B=%d outside [1, %d]", B, FH_MAX_BATCH);
  return FH_OK;
}

fh_stage1_fmt s1fmt(const fh_index* idx) { return (fh_stage1_fmt)idx->desc.s1_fmt; }

// INT4 Stage 1 on the tensor cores from this many queries on (measured at the Gemma-3-1B shape: the
// CUDA-core kernels take 51 µs for 2 queries and 56 µs for 8, the tensor-core kernel 18.3–18.5 µs
// for 4 to 8; one query is the same 19 µs either way).
#ifndef FH_TC_MIN_BATCH_INT4
#define FH_TC_MIN_BATCH_INT4 2
#endif
constexpr int kTcMinBatchInt4 = FH_TC_MIN_BATCH_INT4;

// Stage 1 (scores or Gumbel keys) of s1.B queries: the dequantising tensor-core kernel for INT4
// centroids at batch, the CUDA-core kernels otherwise.
cudaError_t launch_stage1_for(const fh_index* idx, const fh::Stage1Params& s1, cudaStream_t st) {
  const fh_index_desc& D = idx->desc;
  if (s1fmt(idx) == FH_STAGE1_INT4_G32 && s1.B >= kTcMinBatchInt4 &&
      fh::tc_int4_supported(D.d, s1.B, D.C_scales))
    return fh::launch_tc_keys_int4(D.C_q4, D.C_scales, D.c, D.d, s1.H, s1.B, s1.sample, s1.tau,
                                   s1.seed, s1.step, s1.out, s1.status, s1.tickets_to_clear,
                                   s1.n_tickets, idx->num_sms, st);
  return fh::launch_stage1(s1, D.dtype, s1fmt(idx) == FH_STAGE1_INT4_G32, idx->num_sms, st, false);
}

fh::Stage1Params stage1_params(const fh_index* idx, const void* H, int B, float* out, void* ws) {
  const fh_index_desc& D = idx->desc;
  fh::Stage1Params s = {};
  s.C = D.C;
  s.q4 = D.C_q4;
  s.scales = D.C_scales;
  s.H = H;
  s.out = out;
  s.c = D.c;
  s.d = D.d;
  s.B = B;
  s.status = status_of(ws);
  return s;
}

// The greedy/sampling head: Stage 1 (scores or Gumbel keys) → selection → Stage 2 + decision.
fh_status run_head(const fh_index* idx, const void* H, int B, int p, int sample, float tau,
                   uint64_t seed, uint64_t step, int32_t* out_tok, void* ws, size_t ws_bytes,
                   cudaStream_t st, const fh_debug_out* dbg) {
  fh_status r = check_batch(idx, H, B);
  if (r != FH_OK) return r;
  const fh_index_desc& D = idx->desc;
  if (!out_tok) return fail(FH_ERR_ARG, "out_tok is NULL");
  if (p < 1 || p > D.c) return fail(FH_ERR_ARG, "p=%d outside [1, c=%lld]", p, (long long)D.c);
  if (sample && !(tau > 0.0f)) return fail(FH_ERR_ARG, "tau must be > 0");
  const Layout L = layout_for(idx, sample ? FH_OP_SAMPLE : FH_OP_GREEDY, B, p, 0, 0);
  if ((r = check_ws(ws, ws_bytes, L.total)) != FH_OK) return r;
  char* base = static_cast<char*>(ws);
  float* keys = reinterpret_cast<float*>(base + L.keys);
  int32_t* sel = reinterpret_cast<int32_t*>(base + L.sel);

  cudaError_t e;
  // The persistent batch-1 kernel copies 16-byte C2T chunks next to each row, so it needs C2T
  // 16-byte aligned and v % 4 == 0 (no chunk runs past the end of C2T).
  // It also splits rows with 32-bit arithmetic: v * num_sms < 2^31.
  if (B == 1 && fh::head1_threads(D.c) != 0 && D.v % 4 == 0 && aligned16(D.C2T) &&
      D.v * (int64_t)idx->num_sms < (int64_t{1} << 31)) {
    fh::Head1Params h = {};
    h.C = D.C;
    h.q4 = D.C_q4;
    h.scales = D.C_scales;
    h.H = H;
    h.E = D.E;
    h.E_perm = D.E_perm;
    h.C2T = D.C2T;
    h.keys = keys;
    h.c = D.c;
    h.d = D.d;
    h.b = D.b;
    h.p = p;
    h.sample = sample;
    h.tau = tau;
    h.seed = seed;
    h.step = step;
    h.arrive = word_at(ws, kArriveOffset);
    h.best = reinterpret_cast<unsigned long long*>(base + kBestOffset);
    h.hist = word_at(ws, 1024);
    h.gen = word_at(ws, kGenOffset);
    h.keys_ready = word_at(ws, kKeysReadyOffset);
    h.bucket = reinterpret_cast<unsigned long long*>(base + L.bucket);
    h.out_tok = out_tok;
    h.dbg_sel = dbg ? dbg->sel : nullptr;
    h.dbg_tok = dbg ? dbg->cand_tok : nullptr;
    h.dbg_logit = dbg ? dbg->cand_logit : nullptr;
    h.status = status_of(ws);
    e = fh::launch_head1(h, D.dtype, s1fmt(idx) == FH_STAGE1_INT4_G32, idx->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "persistent head launch");
    return FH_OK;
  }
  const bool fused = false;
  // Stage 2 of a batch: the union of the probe sets streamed once on the CUDA cores (up to
  // kUnionMaxBatch queries, while all query vectors fit shared memory), the tensor-core tiles above;
  // neither produces per-candidate outputs, so asking for them takes the per-query Stage 2 instead
  // (the probe sets alone can come from any of them).
  const bool per_cand = dbg && (dbg->cand_tok || dbg->cand_logit);
  const int elem = D.dtype == FH_BF16 ? fh::kBF16 : fh::kF32;
  const bool uni = B > 1 && B <= kUnionMaxBatch && !per_cand && D.E_perm != nullptr &&
                   fh::union_supported(elem, D.d, D.v, D.b, B, idx->num_sms);
  const bool tc = !uni && tc_eligible(idx, B, kTcMinBatchDense) && !per_cand && D.E_perm != nullptr;
  // the query masks, the list's count and the tile flags of a batched Stage 2 are cleared by the
  // selection kernel that precedes their builder
  void* mask_region = (uni || tc) ? static_cast<void*>(base + L.qmask) : nullptr;
  const size_t mask_bytes = (uni || tc) ? qmask_region_bytes(D) : 0;
  // the mask builder may overlap the selection kernel's tail unless a copy of the probe sets sits
  // between them on the stream
  const bool overlap = !(dbg && dbg->sel);
  if ((tc || uni) && tc_eligible(idx, B, kTcMinBatchStage1) && s1fmt(idx) == FH_STAGE1_DENSE) {
    // Stage 1 on the tensor cores too: keys[q][k] = C[k]·h_q (+ the Gumbel term when sampling)
    fh::TcParams tp = {};
    tp.rows = D.c;
    tp.d = D.d;
    tp.B = B;
    tp.b = 1;
    tp.sample = sample;
    tp.tau = tau;
    tp.seed = seed;
    tp.step = step;
    tp.out_keys = keys;
    tp.status = status_of(ws);
    if ((e = fh::launch_tc_head(D.C, H, tp, idx->num_sms, st)) != cudaSuccess)
      return cuda_fail(e, "tensor-core stage-1 launch");
    if ((e = fh::launch_select(keys, sel, B, D.c, p, st, mask_region, mask_bytes)) != cudaSuccess)
      return cuda_fail(e, "select launch");
    if (dbg && dbg->sel &&
        (e = cudaMemcpyAsync(dbg->sel, sel, (size_t)B * p * 4, cudaMemcpyDeviceToDevice, st)) !=
            cudaSuccess)
      return cuda_fail(e, "debug copy");
  } else {
    fh::Stage1Params s1 = stage1_params(idx, H, B, keys, ws);
    s1.sample = sample;
    s1.tau = tau;
    s1.seed = seed;
    s1.step = step;
    s1.rng_stream = FH_RNG_STAGE1;
    s1.tickets_to_clear = tickets_of(ws);
    s1.n_tickets = B;
    e = launch_stage1_for(idx, s1, st);
    if (e != cudaSuccess) return cuda_fail(e, "stage-1 launch");
    if (!fused) {
      if ((e = fh::launch_select(keys, sel, B, D.c, p, st, mask_region, mask_bytes)) != cudaSuccess)
        return cuda_fail(e, "select launch");
      if (dbg && dbg->sel &&
          (e = cudaMemcpyAsync(dbg->sel, sel, (size_t)B * p * 4, cudaMemcpyDeviceToDevice, st)) !=
              cudaSuccess)
        return cuda_fail(e, "debug copy");
    }
  }
  if (uni) {
    unsigned long long* qmask = reinterpret_cast<unsigned long long*>(base + L.qmask);
    int32_t* count = reinterpret_cast<int32_t*>(qmask + D.c) + tile_count_of(D);
    int32_t* list = reinterpret_cast<int32_t*>(base + L.tiles);
    if ((e = fh::launch_build_qmask(sel, B, p, qmask, st, list, count, nullptr, 0, 0, 128, overlap)) !=
        cudaSuccess)
      return cuda_fail(e, "mask launch");
    fh::UnionParams up = {};
    up.E_perm = D.E_perm;
    up.C2T = D.C2T;
    up.H = H;
    up.v = D.v;
    up.d = D.d;
    up.c = D.c;
    up.b = D.b;
    up.B = B;
    up.qmask = qmask;
    up.cl_list = list;
    up.cl_count = count;
    up.sample = sample;
    up.tau = tau;
    up.seed = seed;
    up.step = step;
    up.best = reinterpret_cast<unsigned long long*>(base + L.best);
    up.ticket = word_at(ws, kUnionTicketOffset);
    up.out_tok = out_tok;
    up.status = status_of(ws);
    if ((e = fh::launch_union_rows(up, elem, idx->num_sms, st)) != cudaSuccess)
      return cuda_fail(e, "union stage-2 launch");
    return FH_OK;
  }
  if (tc) {
    // Stage 2 on the tensor cores: every tile of the cluster-major copy that some query selected,
    // masked per (cluster, query), the arg-max of each query fused in.
    unsigned long long* qmask = reinterpret_cast<unsigned long long*>(base + L.qmask);
    uint32_t* flags = reinterpret_cast<uint32_t*>(qmask + D.c);
    int32_t* count = reinterpret_cast<int32_t*>(flags + tile_count_of(D));
    int32_t* list = reinterpret_cast<int32_t*>(base + L.tiles);
    // the query masks and, as their clusters are first selected, the 128-row tiles that hold them
    if ((e = fh::launch_build_qmask(sel, B, p, qmask, st, list, count, flags, D.b, D.v, 128, overlap)) !=
        cudaSuccess)
      return cuda_fail(e, "mask launch");
    fh::TcParams tp = {};
    tp.rows = D.v;
    tp.d = D.d;
    tp.B = B;
    tp.b = D.b;
    tp.qmask = qmask;
    tp.row_tok = D.C2T;  // row e of the cluster-major copy is token C2T[e]
    tp.sample = sample;
    tp.tau = tau;
    tp.seed = seed;
    tp.step = step;
    tp.best = reinterpret_cast<unsigned long long*>(base + L.best);
    tp.ticket = reinterpret_cast<unsigned long long*>(word_at(ws, kTcTicketOffset));
    tp.out_tok = out_tok;
    // the 128-row tiles that hold a cluster some query takes
    tp.tile_list = list;
    tp.tile_count = count;
    tp.status = status_of(ws);
    if ((e = fh::launch_tc_head(D.E_perm, H, tp, idx->num_sms, st)) != cudaSuccess)
      return cuda_fail(e, "tensor-core stage-2 launch");
    return FH_OK;
  }
  fh::Stage2Params s2 = {};
  s2.E = D.E;
  s2.E_perm = D.E_perm;
  s2.C2T = D.C2T;
  s2.H = H;
  s2.keys = nullptr;
  s2.sel = sel;
  s2.v = D.v;
  s2.d = D.d;
  s2.c = D.c;
  s2.b = D.b;
  s2.B = B;
  s2.p = p;
  s2.sample = sample;
  s2.tau = tau;
  s2.seed = seed;
  s2.step = step;
  s2.part = reinterpret_cast<unsigned long long*>(base + L.part);
  s2.tickets = tickets_of(ws);
  s2.out_tok = out_tok;
  s2.dbg_sel = nullptr;
  s2.dbg_tok = dbg ? dbg->cand_tok : nullptr;
  s2.dbg_logit = dbg ? dbg->cand_logit : nullptr;
  s2.status = status_of(ws);
  if ((e = fh::launch_stage2(s2, D.dtype, idx->num_sms, st)) != cudaSuccess)
    return cuda_fail(e, "stage-2 launch");
  return FH_OK;
}

}  // namespace

namespace fh {
// The error reporter of the other C ABI files (the k-means builder): sets fh_last_error().
fh_status report(fh_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}
}  // namespace fh

// Used by fh_static.cu to report its own errors through fh_last_error().
fh_status fh_internal_set_error(fh_status st, const char* msg) { return fail(st, "%s", msg); }

// Used by fh_static.cu: the host-side argument checks of a head call (nothing is launched).
fh_status fh_internal_check_head(const fh_index* idx, const void* H, int B, int p, const int32_t* out_tok) {
  fh_status r = check_batch(idx, H, B);
  if (r != FH_OK) return r;
  if (!out_tok) return fail(FH_ERR_ARG, "out_tok is NULL");
  if (p < 1 || p > idx->desc.c) return fail(FH_ERR_ARG, "p=%d outside [1, c=%lld]", p, (long long)idx->desc.c);
  return FH_OK;
}

extern "C" {

const char* fh_last_error(void) { return g_err; }

size_t fh_index_load_ws_bytes(const fh_index_desc* desc) {
  if (!desc || desc->v <= 0) return 0;
  return kHeaderBytes + up((size_t)((desc->v + 31) / 32) * 4);
}

fh_status fh_index_load(const fh_index_desc* desc, void* ws, size_t ws_bytes, fh_stream stream,
                        fh_index** out) {
  FH_NVTX_RANGE("fh_index_load");
  if (out) *out = nullptr;
  if (!desc || !out) return fail(FH_ERR_ARG, "desc or out is NULL");
  const fh_index_desc& D = *desc;
  if (D.v <= 0 || D.d <= 0 || D.c <= 0 || D.b <= 0) return fail(FH_ERR_SHAPE, "non-positive size");
  if (D.v != D.c * D.b) return fail(FH_ERR_SHAPE, "v=%lld != c*b=%lld", (long long)D.v,
                                    (long long)(D.c * D.b));
  if (D.v > 0x7FFFFFFFLL) return fail(FH_ERR_SHAPE, "v too large for int32 token ids");
  if (D.c > FH_MAX_C) return fail(FH_ERR_SHAPE, "c=%lld exceeds %d", (long long)D.c, FH_MAX_C);
  if (D.d > FH_MAX_D) return fail(FH_ERR_SHAPE, "d=%lld exceeds %d", (long long)D.d, FH_MAX_D);
  if (D.d % 8) return fail(FH_ERR_SHAPE, "d must be a multiple of 8");
  if (D.dtype != FH_F32 && D.dtype != FH_BF16) return fail(FH_ERR_ARG, "unknown dtype");
  if (D.s1_fmt != FH_STAGE1_DENSE && D.s1_fmt != FH_STAGE1_INT4_G32)
    return fail(FH_ERR_ARG, "unknown stage-1 format");
  if (!D.E || !D.C2T) return fail(FH_ERR_ARG, "E and C2T are required");
  if (!aligned16(D.E) || !aligned16(D.C) || !aligned16(D.E_perm) || !aligned16(D.C_q4))
    return fail(FH_ERR_ARG, "E, C, E_perm and C_q4 must be 16-byte aligned");
  if (D.s1_fmt == FH_STAGE1_DENSE && !D.C) return fail(FH_ERR_ARG, "C is required");
  if (D.s1_fmt == FH_STAGE1_INT4_G32) {
    if (D.dtype != FH_BF16) return fail(FH_ERR_ARG, "INT4 Stage 1 needs BF16 E and H");
    if (!D.C_q4 || !D.C_scales) return fail(FH_ERR_ARG, "C_q4 and C_scales are required");
    if (D.d % 32) return fail(FH_ERR_SHAPE, "INT4 groups need d % 32 == 0");
    if (D.d > 4096) return fail(FH_ERR_UNSUPPORTED, "INT4 Stage 1 supports d <= 4096");
  }
  fh_status r = check_ws(ws, ws_bytes, fh_index_load_ws_bytes(desc));
  if (r != FH_OK) return r;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query");

  // C2T must list every token id exactly once (equal-size clusters, a dense c x b table).
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + kHeaderBytes);
  if ((e = cudaMemsetAsync(ws, 0, fh_index_load_ws_bytes(desc), st)) != cudaSuccess)
    return cuda_fail(e, "memset");
  if ((e = fh::launch_validate_c2t(D.C2T, D.v, bitmap, status_of(ws), st)) != cudaSuccess)
    return cuda_fail(e, "C2T validation launch");
  uint32_t status = 0;
  if ((e = cudaMemcpyAsync(&status, ws, 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(e, "status copy");
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "C2T validation");
  if (status != 0) return fail(FH_ERR_INDEX, "C2T is not a permutation of 0..v-1");
  if (D.E_perm) {
    if ((e = fh::launch_build_perm(D.E, D.C2T, D.v, D.d, D.dtype, D.E_perm, st)) != cudaSuccess)
      return cuda_fail(e, "E_perm build launch");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "E_perm build");
  }
  fh_index* idx = new (std::nothrow) fh_index;
  if (!idx) return fail(FH_ERR_ARG, "out of host memory");
  idx->desc = D;
  idx->num_sms = sms;
  idx->device = dev;
  *out = idx;
  return FH_OK;
}

void fh_index_free(fh_index* idx) { delete idx; }

size_t fh_workspace_bytes(const fh_index* idx, int op, int B, int p, int T, int64_t N) {
  if (!idx || B < 1 || B > FH_MAX_BATCH) return 0;
  if ((op == FH_OP_GREEDY || op == FH_OP_SAMPLE || op == FH_OP_MC) && (p < 1 || p > idx->desc.c))
    return 0;
  if (op == FH_OP_MC && (T < 1 || T > 64 || N < 1)) return 0;
  if (op < FH_OP_GREEDY || op > FH_OP_DENSE) return 0;
  return layout_for(idx, op, B, p, T, N).total;
}

fh_status fh_ws_status(void* ws, fh_stream stream) {
  FH_NVTX_RANGE("fh_ws_status");
  if (!ws) return fail(FH_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t status = 0;
  cudaError_t e = cudaMemcpyAsync(&status, ws, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (status != 0) {
    // Zero the control block, but move the call generation past every tag the failed call may have
    // written, so that no entry it left behind is taken for a later call's.
    uint32_t gen = 0;
    e = cudaMemcpyAsync(&gen, static_cast<char*>(ws) + kGenOffset, 4, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    gen += 1u;
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, kHeaderBytes, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(ws) + kGenOffset, &gen, 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    if (status == FH_ERR_TIMEOUT) return fail(FH_ERR_TIMEOUT, "a device-side wait timed out");
    if (status == FH_ERR_INDEX) return fail(FH_ERR_INDEX, "a kernel met an index out of range");
    return fail((fh_status)status, "device error %u", status);
  }
  return FH_OK;
}

fh_status fh_head_greedy(const fh_index* idx, const void* H, int B, int p, int32_t* out_tok,
                         void* ws, size_t ws_bytes, fh_stream stream, const fh_debug_out* dbg) {
  FH_NVTX_RANGE("fh_head_greedy");
  return run_head(idx, H, B, p, 0, 1.0f, 0, 0, out_tok, ws, ws_bytes,
                  static_cast<cudaStream_t>(stream), dbg);
}

fh_status fh_head_greedy_host(const fh_index* idx, const void* H_host, int B, int p, int32_t* tok_host,
                              void* h_dev, int32_t* tok_dev, void* ws, size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_head_greedy_host");
  fh_status s = check_batch(idx, h_dev, B);
  if (s != FH_OK) return s;
  if (!H_host || !tok_host || !tok_dev) return fail(FH_ERR_ARG, "H_host, tok_host or tok_dev is NULL");
  if (p < 1 || p > idx->desc.c) return fail(FH_ERR_ARG, "p=%d outside [1, c=%lld]", p, (long long)idx->desc.c);
  if ((s = check_ws(ws, ws_bytes, layout_for(idx, FH_OP_GREEDY, B, p, 0, 0).total)) != FH_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t h_bytes = (size_t)B * (size_t)idx->desc.d * (idx->desc.dtype == FH_BF16 ? 2u : 4u);
  cudaError_t e = cudaMemcpyAsync(h_dev, H_host, h_bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "query copy");
  if ((s = run_head(idx, h_dev, B, p, 0, 1.0f, 0, 0, tok_dev, ws, ws_bytes, st, nullptr)) != FH_OK) return s;
  if ((e = cudaMemcpyAsync(tok_host, tok_dev, (size_t)B * 4u, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(e, "token copy");
  return FH_OK;
}

fh_status fh_head_sample(const fh_index* idx, const void* H, int B, int p, float tau, uint64_t seed,
                         uint64_t step, int32_t* out_tok, void* ws, size_t ws_bytes,
                         fh_stream stream, const fh_debug_out* dbg) {
  FH_NVTX_RANGE("fh_head_sample");
  return run_head(idx, H, B, p, 1, tau, seed, step, out_tok, ws, ws_bytes,
                  static_cast<cudaStream_t>(stream), dbg);
}

fh_status fh_dense_head(const fh_index* idx, const void* H, int B, int sample, float tau,
                        uint64_t seed, uint64_t step, int32_t* out_tok, float* out_logits,
                        void* ws, size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_dense_head");
  fh_status r = check_batch(idx, H, B);
  if (r != FH_OK) return r;
  if (!out_tok && !out_logits) return fail(FH_ERR_ARG, "out_tok and out_logits are both NULL");
  if (sample && !(tau > 0.0f)) return fail(FH_ERR_ARG, "tau must be > 0");
  const Layout L = layout_for(idx, FH_OP_DENSE, B, 1, 0, 0);
  if ((r = check_ws(ws, ws_bytes, L.total)) != FH_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const fh_index_desc& D = idx->desc;
  cudaError_t e;
  if (tc_eligible(idx, B, kTcMinBatchDense)) {
    fh::TcParams tp = {};
    tp.rows = D.v;
    tp.d = D.d;
    tp.B = B;
    tp.b = 1;
    tp.sample = sample;
    tp.tau = tau;
    tp.seed = seed;
    tp.step = step;
    tp.best = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.best);
    tp.ticket = reinterpret_cast<unsigned long long*>(word_at(ws, kTcTicketOffset));
    tp.out_tok = out_tok;
    tp.out_logits = out_logits;
    tp.status = status_of(ws);
    if ((e = fh::launch_tc_head(D.E, H, tp, idx->num_sms, st)) != cudaSuccess)
      return cuda_fail(e, "tensor-core dense launch");
    return FH_OK;
  }
  e = cudaMemsetAsync(tickets_of(ws), 0, (size_t)B * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  fh::DenseParams dp = {};
  dp.E = D.E;
  dp.H = H;
  dp.v = D.v;
  dp.d = D.d;
  dp.B = B;
  dp.sample = sample;
  dp.tau = tau;
  dp.seed = seed;
  dp.step = step;
  dp.part = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.part);
  dp.tickets = tickets_of(ws);
  dp.out_tok = out_tok;
  dp.out_logits = out_logits;
  dp.status = status_of(ws);
  if ((e = fh::launch_dense(dp, D.dtype, idx->num_sms, st)) != cudaSuccess)
    return cuda_fail(e, "dense launch");
  return FH_OK;
}

fh_status fh_mc_token_prob(const fh_index* idx, const void* H, int B, const int32_t* targets, int T,
                           int p, float tau, int64_t N, uint64_t seed, double* out_mean,
                           double* out_se, void* ws, size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_mc_token_prob");
  return fh_mc_token_prob_range(idx, H, B, targets, T, p, tau, 0, N, seed, out_mean, out_se, ws,
                                ws_bytes, stream);
}

fh_status fh_mc_token_prob_range(const fh_index* idx, const void* H, int B, const int32_t* targets,
                                 int T, int p, float tau, int64_t i0, int64_t N, uint64_t seed,
                                 double* out_mean, double* out_se, void* ws, size_t ws_bytes,
                                 fh_stream stream) {
  FH_NVTX_RANGE("fh_mc_token_prob_range");
  if (i0 < 0 || i0 > (int64_t{1} << 40)) return fail(FH_ERR_ARG, "i0 outside [0, 2^40]");
  fh_status r = check_batch(idx, H, B);
  if (r != FH_OK) return r;
  const fh_index_desc& D = idx->desc;
  if (!targets || !out_mean || !out_se) return fail(FH_ERR_ARG, "targets/out_mean/out_se NULL");
  if (T < 1 || T > 64) return fail(FH_ERR_ARG, "T=%d outside [1, 64]", T);
  if (N < 1 || N > (1LL << 24)) return fail(FH_ERR_ARG, "N outside [1, 2^24]");
  if (p < 1 || p > D.c) return fail(FH_ERR_ARG, "p outside [1, c]");
  if (!(tau > 0.0f)) return fail(FH_ERR_ARG, "tau must be > 0");
  if (D.c > 256 * 64) return fail(FH_ERR_UNSUPPORTED, "Monte Carlo supports c <= 16384");
  const Layout L = layout_for(idx, FH_OP_MC, B, p, T, N);
  if ((r = check_ws(ws, ws_bytes, L.total)) != FH_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  cudaError_t e = cudaMemsetAsync(tickets_of(ws), 0, (size_t)B * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "memset");
  // exact logits over the vocabulary, once per query (S-independent)
  if (tc_eligible(idx, B, kTcMinBatchDense)) {  // all v logits of every query, on the tensor cores
    fh::TcParams tp = {};
    tp.rows = D.v;
    tp.d = D.d;
    tp.B = B;
    tp.b = 1;
    tp.best = reinterpret_cast<unsigned long long*>(base + L.best);
    tp.ticket = reinterpret_cast<unsigned long long*>(word_at(ws, kTcTicketOffset));
    tp.out_logits = reinterpret_cast<float*>(base + L.z);
    tp.status = status_of(ws);
    if ((e = fh::launch_tc_head(D.E, H, tp, idx->num_sms, st)) != cudaSuccess)
      return cuda_fail(e, "tensor-core logits launch");
  } else {
    fh::DenseParams dp = {};
    dp.E = D.E;
    dp.H = H;
    dp.v = D.v;
    dp.d = D.d;
    dp.B = B;
    dp.tau = 1.0f;
    dp.part = reinterpret_cast<unsigned long long*>(base + L.part);
    dp.tickets = tickets_of(ws);
    dp.out_logits = reinterpret_cast<float*>(base + L.z);
    dp.status = status_of(ws);
    if ((e = fh::launch_dense(dp, D.dtype, idx->num_sms, st)) != cudaSuccess)
      return cuda_fail(e, "MC logits launch");
  }
  // Stage-1 scores
  fh::Stage1Params s1 = stage1_params(idx, H, B, reinterpret_cast<float*>(base + L.s), ws);
  if ((e = launch_stage1_for(idx, s1, st)) != cudaSuccess) return cuda_fail(e, "MC stage-1 launch");
  fh::McParams mp = {};
  mp.s = reinterpret_cast<float*>(base + L.s);
  mp.z = reinterpret_cast<float*>(base + L.z);
  mp.C2T = D.C2T;
  mp.cluster_of = reinterpret_cast<int32_t*>(base + L.cluster_of);
  mp.targets = targets;
  mp.zmax = reinterpret_cast<float*>(base + L.zmax);
  mp.Z = reinterpret_cast<double*>(base + L.Z);
  mp.per_draw = reinterpret_cast<double*>(base + L.per_draw);
  mp.out_mean = out_mean;
  mp.out_se = out_se;
  mp.v = D.v;
  mp.c = D.c;
  mp.b = D.b;
  mp.N = N;
  mp.i0 = i0;
  mp.B = B;
  mp.T = T;
  mp.p = p;
  mp.tau = tau;
  mp.seed = seed;
  mp.status = status_of(ws);
  if ((e = fh::launch_mc(mp, idx->num_sms, st)) != cudaSuccess) return cuda_fail(e, "MC launch");
  return FH_OK;
}

fh_status fh_stage1_scores(const fh_index* idx, const void* H, int B, float* out_s, void* ws,
                           size_t ws_bytes, fh_stream stream) {
  FH_NVTX_RANGE("fh_stage1_scores");
  fh_status r = check_batch(idx, H, B);
  if (r != FH_OK) return r;
  if (!out_s) return fail(FH_ERR_ARG, "out_s is NULL");
  if ((r = check_ws(ws, ws_bytes, kHeaderBytes)) != FH_OK) return r;
  cudaError_t e;
  if (tc_eligible(idx, B, kTcMinBatchStage1) && s1fmt(idx) == FH_STAGE1_DENSE) {
    // the kernel the fused head runs at these batches: keys mode of the tensor-core head
    fh::TcParams tp = {};
    tp.rows = idx->desc.c;
    tp.d = idx->desc.d;
    tp.B = B;
    tp.b = 1;
    tp.out_keys = out_s;
    tp.status = status_of(ws);
    if ((e = fh::launch_tc_head(idx->desc.C, H, tp, idx->num_sms, static_cast<cudaStream_t>(stream))) !=
        cudaSuccess)
      return cuda_fail(e, "tensor-core stage-1 launch");
    return FH_OK;
  }
  fh::Stage1Params s1 = stage1_params(idx, H, B, out_s, ws);
  e = launch_stage1_for(idx, s1, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stage-1 launch");
  return FH_OK;
}

fh_status fh_gumbel_keys(const float* s, int B, int64_t c, float tau, uint64_t seed, uint64_t step,
                         uint32_t rng_stream, float* out_keys, fh_stream stream) {
  FH_NVTX_RANGE("fh_gumbel_keys");
  if (!s || !out_keys) return fail(FH_ERR_ARG, "s or out_keys is NULL");
  if (B < 1 || c < 1) return fail(FH_ERR_ARG, "empty input");
  if (!(tau > 0.0f)) return fail(FH_ERR_ARG, "tau must be > 0");
  cudaError_t e = fh::launch_gumbel_keys(s, out_keys, B, c, tau, seed, step, rng_stream,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gumbel launch");
  return FH_OK;
}

fh_status fh_select_topp(const float* keys, int B, int64_t c, int p, int32_t* out_sel,
                         fh_stream stream) {
  FH_NVTX_RANGE("fh_select_topp");
  if (!keys || !out_sel) return fail(FH_ERR_ARG, "keys or out_sel is NULL");
  if (B < 1 || B > 65535) return fail(FH_ERR_ARG, "B outside [1, 65535]");
  if (c < 1 || c > FH_MAX_C) return fail(FH_ERR_SHAPE, "c outside [1, %d]", FH_MAX_C);
  if (p < 1 || p > c) return fail(FH_ERR_ARG, "p outside [1, c]");
  cudaError_t e = fh::launch_select(keys, out_sel, B, c, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  return FH_OK;
}

fh_status fh_gather_candidates(const fh_index* idx, const int32_t* sel, int B, int p,
                               int32_t* out_cand, fh_stream stream) {
  FH_NVTX_RANGE("fh_gather_candidates");
  if (!idx || !sel || !out_cand) return fail(FH_ERR_ARG, "NULL argument");
  if (B < 1 || p < 1 || p > idx->desc.c) return fail(FH_ERR_ARG, "bad B or p");
  cudaError_t e = fh::launch_gather(idx->desc.C2T, idx->desc.b, sel, B, p, out_cand,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return FH_OK;
}

fh_status fh_candidate_logits(const fh_index* idx, const void* H, int B, const int32_t* cand,
                              int64_t P, float* out_z, fh_stream stream) {
  FH_NVTX_RANGE("fh_candidate_logits");
  fh_status r = check_batch(idx, H, B);
  if (r != FH_OK) return r;
  if (!cand || !out_z) return fail(FH_ERR_ARG, "cand or out_z is NULL");
  if (P < 1) return fail(FH_ERR_ARG, "P must be >= 1");
  cudaError_t e = fh::launch_cand_logits(idx->desc.E, idx->desc.dtype, idx->desc.d, H, B, cand, P,
                                         out_z, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "logits launch");
  return FH_OK;
}

fh_status fh_philox_u32(uint64_t seed, uint64_t step, uint32_t row, uint32_t rng_stream, int64_t n,
                        uint32_t* out, fh_stream stream) {
  FH_NVTX_RANGE("fh_philox_u32");
  if (!out || n < 1) return fail(FH_ERR_ARG, "out is NULL or n < 1");
  if (n > (1LL << 32)) return fail(FH_ERR_ARG, "n > 2^32");
  cudaError_t e = fh::launch_philox(seed, step, row, rng_stream, n, out,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "philox launch");
  return FH_OK;
}

}  // extern "C"
