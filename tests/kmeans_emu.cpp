// Host build of the index builder's steps (clustered_retrieval_classification_b200/csrc/
// fh_kmeans_core.cuh) for the CPU tests: the same per-item functions and the same iteration loop as
// the device build, run sequentially.  Only the similarity product differs: here it is a plain
// sequential fp32 dot product, on the device it is the tensor-core kernel.  Test infrastructure.
#include <stdint.h>

#include <vector>

#include "../clustered_retrieval_classification_b200/csrc/fh_kmeans_core.cuh"

using namespace fhkm;

namespace {

struct HostBackend {
  const uint16_t* E = nullptr;
  int64_t v = 0, d = 0, b = 0;
  int c = 0;
  const int32_t* init = nullptr;
  const uint16_t* C_score = nullptr;
  const int32_t* labels_in = nullptr;
  int32_t* labels = nullptr;
  int32_t* C2T = nullptr;
  float* C = nullptr;
  uint16_t* Cb = nullptr;
  double* objective = nullptr;
  std::vector<float> S, inv, norms, price, slot_bid, bid_beta;
  std::vector<int32_t> prev, slot_tok, fill, cnt, off, inbox, U0, U1, bid_k, pos;
  int32_t n_next = 0;
  int cur = 0;
  Auction a{};

  int32_t* U(int i) { return i == 0 ? U0.data() : U1.data(); }

  void alloc() {
    S.assign((size_t)v * c, 0.f);
    inv.assign(v, 0.f);
    norms.assign(c, 0.f);
    price.assign(c, 0.f);
    slot_bid.assign(v, 0.f);
    bid_beta.assign(v, 0.f);
    prev.assign(v, -1);
    slot_tok.assign(v, 0);
    fill.assign(c, 0);
    cnt.assign(c, 0);
    off.assign(c, 0);
    inbox.assign(v, 0);
    U0.assign(v, 0);
    U1.assign(v, 0);
    bid_k.assign(v, 0);
    pos.assign(v, 0);
    a.v = v;
    a.c = c;
    a.b = b;
    a.price = price.data();
    a.slot_bid = slot_bid.data();
    a.slot_tok = slot_tok.data();
    a.fill = fill.data();
    a.cnt = cnt.data();
    a.off = off.data();
    a.inbox = inbox.data();
    a.bid_k = bid_k.data();
    a.bid_beta = bid_beta.data();
    a.pos = pos.data();
    a.n_next = &n_next;
  }

  bool row_norms(int64_t* bad) {
    *bad = 0;
    for (int64_t i = 0; i < v; ++i) {
      inv[i] = row_inv_norm(E + i * d, d);
      if (inv[i] == 0.f) ++*bad;
    }
    return true;
  }

  bool init_centres(int64_t* bad) {
    *bad = 0;
    for (int k = 0; k < c; ++k) {
      const int32_t tok = claim_init_token(init, k, v, prev.data());
      if (tok < 0) ++*bad;
      for (int64_t j = 0; j < d; ++j) {
        const float x = tok >= 0 ? unit_value(E, inv.data(), tok, d, j) : 0.f;
        C[(int64_t)k * d + j] = x;
        Cb[(int64_t)k * d + j] = f32_to_bf16(x);
      }
    }
    return true;
  }

  bool similarities() {
    for (int64_t i = 0; i < v; ++i)
      for (int k = 0; k < c; ++k) {
        float acc = 0.f;
        for (int64_t j = 0; j < d; ++j)
          acc = fma_rn(bf16_to_f32(C_score[(int64_t)k * d + j]), bf16_to_f32(E[i * d + j]), acc);
        S[(size_t)i * c + k] = acc;
      }
    return true;
  }

  bool zero_prices() {
    for (auto& p : price) p = 0.f;
    return true;
  }

  bool reset_phase() {
    for (auto& f : fill) f = 0;
    cur = 0;
    for (int64_t i = 0; i < v; ++i) U0[i] = (int32_t)i;
    return true;
  }

  bool one_cluster() {
    for (int64_t i = 0; i < v; ++i) slot_tok[i] = (int32_t)i;
    fill[0] = (int32_t)v;
    return true;
  }

  bool round(int64_t n, float eps) {
    Auction s = a;
    s.U = U(cur);
    s.U_next = U(cur ^ 1);
    for (int64_t w = 0; w < n; ++w) {  // k_km_bid: 32 lanes, then their merge
      const int32_t i = s.U[w];
      Top2 t = top2_init();
      for (int lane = 0; lane < 32; ++lane)
        t = top2_merge(t, lane_top2(S.data() + (size_t)i * c, inv[i], s.price, c, lane, 32));
      const int k1 = (t.k1 >= 0 && t.k1 < c) ? t.k1 : 0;
      s.bid_k[w] = k1;
      s.bid_beta[w] = bid_value(t, eps);
      s.pos[w] = fetch_add(&s.cnt[k1], 1);
    }
    int32_t run = 0;  // k_km_scan
    for (int k = 0; k < c; ++k) {
      s.off[k] = run;
      run += s.cnt[k];
    }
    for (int64_t t = 0; t < n; ++t) scatter_bid(s, t);
    for (int k = 0; k < c; ++k) resolve_cluster(k, s);
    return true;
  }

  bool next_count(int64_t* left) {
    *left = n_next;
    n_next = 0;
    cur ^= 1;
    return true;
  }

  bool slots_from_labels(int64_t* bad) {
    *bad = 0;
    for (auto& f : fill) f = 0;
    for (int64_t i = 0; i < v; ++i)
      if (!slot_from_label(i, labels_in, c, b, fill.data(), slot_tok.data())) ++*bad;
    return true;
  }

  bool finish_labels(bool first, int64_t* changed) {
    for (int k = 0; k < c; ++k) write_cluster(k, slot_tok.data(), b, labels, C2T);
    *changed = 0;
    for (int64_t i = 0; i < v; ++i) {
      if (!first && labels[i] != prev[i]) ++*changed;
      prev[i] = labels[i];
    }
    return true;
  }

  bool update_centres(int t, int64_t* degenerate) {
    *degenerate = 0;
    std::vector<float> acc(d);
    for (int k = 0; k < c; ++k) {
      const int32_t* members = C2T + (int64_t)k * b;
      for (int64_t j = 0; j < d; ++j) acc[j] = member_sum(E, inv.data(), members, b, d, j);
      const float n = column_norm(acc.data(), d);
      norms[k] = n;
      if (!(n > 0.f)) ++*degenerate;
      for (int64_t j = 0; j < d; ++j) {
        const float x = centre_value(acc[j], n);
        C[(int64_t)k * d + j] = x;
        Cb[(int64_t)k * d + j] = f32_to_bf16(x);
      }
    }
    if (objective) {
      double parts[kObjectiveParts];
      for (int p = 0; p < kObjectiveParts; ++p) parts[p] = objective_part(norms.data(), c, p, kObjectiveParts);
      objective[t] = objective_total(parts, kObjectiveParts);
    }
    return true;
  }
};

}  // namespace

// op: 0 build, 1 assign, 2 update.  Returns the loop's outcome code (0 = done).
extern "C" int emu_kmeans(int op, const uint16_t* E, int64_t v, int64_t d, int64_t c, int iters,
                          float eps, int64_t max_rounds, const int32_t* init, const uint16_t* C_in,
                          const int32_t* labels_in, int32_t* labels, int32_t* C2T, float* C,
                          uint16_t* C_bf16, double* objective, float* prices, int32_t* iters_done,
                          int64_t* rounds) {
  HostBackend be;
  be.E = E;
  be.v = v;
  be.d = d;
  be.c = (int)c;
  be.b = v / c;
  be.init = init;
  be.labels_in = labels_in;
  std::vector<int32_t> scratch_labels(v);
  std::vector<float> scratch_C((size_t)c * d);
  std::vector<uint16_t> Cb((size_t)c * d);
  be.labels = labels ? labels : scratch_labels.data();
  be.C2T = C2T;
  be.C = C ? C : scratch_C.data();
  be.Cb = Cb.data();
  be.C_score = op == 1 ? C_in : Cb.data();
  be.objective = objective;
  be.alloc();
  const Config cfg = make_config(v, d, c, op == 0 ? iters : 1, eps, max_rounds);
  Progress pr;
  const Outcome o = op == 0 ? run(be, cfg, pr) : op == 1 ? assign_only(be, cfg, pr) : update_only(be, cfg);
  *rounds = pr.rounds;
  *iters_done = op == 0 ? pr.iters_done : (op == 2 && o == kDone ? 1 : 0);
  if (o == kDone && C_bf16 && op != 1)
    for (size_t i = 0; i < Cb.size(); ++i) C_bf16[i] = Cb[i];
  if (o == kDone && prices && op != 2)
    for (int k = 0; k < c; ++k) prices[k] = be.price[k];
  return (int)o;
}
