"""ctypes binding of libflashhead.so (C ABI in include/flashhead.h).

Argument marshalling only: every step of the head runs in the library's CUDA kernels.  PyTorch
provides device memory and streams.  The binding raises FlashHeadError when the library is missing
or a call fails; there is no other code path.

BF16 tensors are torch.bfloat16 on the device; fp32 tensors are torch.float32.  Functions take the
current torch CUDA stream unless `stream` is given.
"""

from __future__ import annotations

import ctypes as ct
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libflashhead.so")

FH_F32, FH_BF16 = 0, 1
FH_STAGE1_DENSE, FH_STAGE1_INT4_G32 = 0, 1
FH_OP_GREEDY, FH_OP_SAMPLE, FH_OP_MC, FH_OP_DENSE = 0, 1, 2, 3
FH_RNG_STAGE1, FH_RNG_STAGE2, FH_RNG_MC = 0, 1, 2
STATUS_NAMES = {0: "FH_OK", 1: "FH_ERR_ARG", 2: "FH_ERR_SHAPE", 3: "FH_ERR_INDEX",
                4: "FH_ERR_WORKSPACE", 5: "FH_ERR_CUDA", 6: "FH_ERR_TIMEOUT",
                7: "FH_ERR_UNSUPPORTED"}


class FlashHeadError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class IndexDesc(ct.Structure):
    _fields_ = [("v", ct.c_int64), ("d", ct.c_int64), ("c", ct.c_int64), ("b", ct.c_int64),
                ("dtype", ct.c_int32), ("s1_fmt", ct.c_int32),
                ("E", ct.c_void_p), ("C", ct.c_void_p), ("C2T", ct.c_void_p),
                ("C_q4", ct.c_void_p), ("C_scales", ct.c_void_p), ("E_perm", ct.c_void_p)]


class DebugOut(ct.Structure):
    _fields_ = [("sel", ct.c_void_p), ("cand_tok", ct.c_void_p), ("cand_logit", ct.c_void_p)]


class CfDesc(ct.Structure):
    """fh_cf_desc (include/fh_cfhead.h)."""
    _fields_ = [("v", ct.c_int64), ("d", ct.c_int64), ("w", ct.c_int32), ("K", ct.c_int32),
                ("E", ct.c_void_p), ("codebooks", ct.c_void_p), ("codes", ct.c_void_p)]


class KmeansArgs(ct.Structure):
    """fh_kmeans_args (include/fh_kmeans.h)."""
    _fields_ = [("E", ct.c_void_p), ("dtype", ct.c_int32), ("v", ct.c_int64), ("d", ct.c_int64),
                ("c", ct.c_int64), ("iters", ct.c_int32), ("eps", ct.c_float),
                ("max_rounds", ct.c_int64), ("init_tokens", ct.c_void_p), ("C_in", ct.c_void_p),
                ("labels_in", ct.c_void_p), ("labels", ct.c_void_p), ("C2T", ct.c_void_p),
                ("C", ct.c_void_p), ("C_bf16", ct.c_void_p), ("objective", ct.c_void_p),
                ("prices", ct.c_void_p), ("iters_done", ct.c_int32), ("rounds", ct.c_int64)]


_lib = None
_p, _i, _i64, _u32, _u64, _f, _sz = (ct.c_void_p, ct.c_int, ct.c_int64, ct.c_uint32, ct.c_uint64,
                                      ct.c_float, ct.c_size_t)

SIGNATURES = {
    "fh_index_load_ws_bytes": (_sz, [_p]),
    "fh_index_load": (_i, [_p, _p, _sz, _p, _p]),
    "fh_index_free": (None, [_p]),
    "fh_workspace_bytes": (_sz, [_p, _i, _i, _i, _i, _i64]),
    "fh_ws_status": (_i, [_p, _p]),
    "fh_last_error": (ct.c_char_p, []),
    "fh_head_greedy": (_i, [_p, _p, _i, _i, _p, _p, _sz, _p, _p]),
    "fh_head_greedy_host": (_i, [_p, _p, _i, _i, _p, _p, _p, _p, _sz, _p]),
    "fh_head_sample": (_i, [_p, _p, _i, _i, _f, _u64, _u64, _p, _p, _sz, _p, _p]),
    "fh_mc_token_prob": (_i, [_p, _p, _i, _p, _i, _i, _f, _i64, _u64, _p, _p, _p, _sz, _p]),
    "fh_mc_token_prob_range": (_i, [_p, _p, _i, _p, _i, _i, _f, _i64, _i64, _u64, _p, _p, _p, _sz, _p]),
    "fh_dense_head": (_i, [_p, _p, _i, _i, _f, _u64, _u64, _p, _p, _p, _sz, _p]),
    "fh_stage1_scores": (_i, [_p, _p, _i, _p, _p, _sz, _p]),
    "fh_gumbel_keys": (_i, [_p, _i, _i64, _f, _u64, _u64, _u32, _p, _p]),
    "fh_select_topp": (_i, [_p, _i, _i64, _i, _p, _p]),
    "fh_gather_candidates": (_i, [_p, _p, _i, _i, _p, _p]),
    "fh_candidate_logits": (_i, [_p, _p, _i, _p, _i64, _p, _p]),
    "fh_philox_u32": (_i, [_u64, _u64, _u32, _u32, _i64, _p, _p]),
    "fh_head_greedy_static": (_i, [_p, _p, _i, _p, _p]),
    "fh_static_status": (_i, [_p]),
    "fh_static_scratch": (_i, [_p, _p]),
    "fh_cf_load": (_i, [_p, _p]),
    "fh_cf_free": (None, [_p]),
    "fh_cf_workspace_bytes": (_sz, [_p, _i, _i]),
    "fh_cf_head": (_i, [_p, _p, _i, _i, _i, _f, _u64, _u64, _p, _p, _sz, _p, _p, _p]),
    "fh_cf_coarse_scores": (_i, [_p, _p, _i, _p, _p, _sz, _p]),
    "fh_kmeans_ws_bytes": (_sz, [_i64, _i64, _i64]),
    "fh_kmeans_build": (_i, [_p, _p, _sz, _p]),
    "fh_kmeans_assign": (_i, [_p, _p, _sz, _p]),
    "fh_kmeans_update": (_i, [_p, _p, _sz, _p]),
}


def load():
    """Load libflashhead.so; raises FlashHeadError if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FlashHeadError(5, f"{LIB_PATH} is missing; build it with "
                                    "clustered_retrieval_classification_b200._build.build()")
        L = ct.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise FlashHeadError(status, load().fh_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ct.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ct.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FH_BF16
    if t.dtype == torch.float32:
        return FH_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


class Index:
    """A loaded FlashHead index.  Keeps the device tensors alive while the handle lives.

    E: [v, d], C: [c, d] (bf16 or fp32), C2T: [c, b] int32.  For INT4 Stage 1 pass C_q4 ([c, d/2]
    uint8) and C_scales ([c, d/32] bf16) and int4=True.  cluster_major=True gives the library a
    v x d buffer for its cluster-major copy of E."""

    def __init__(self, E, C, C2T, C_q4=None, C_scales=None, int4=False, cluster_major=True,
                 stream=None):
        L = load()
        for t, n in ((E, "E"), (C2T, "C2T")):
            _need(t, n)
        if C is not None:
            _need(C, "C")
        self.E, self.C, self.C2T, self.C_q4, self.C_scales = E, C, C2T, C_q4, C_scales
        self.v, self.d = E.shape
        self.c, self.b = C2T.shape
        self.dtype = E.dtype
        self.int4 = bool(int4)
        self.E_perm = torch.empty_like(E) if cluster_major else None
        self.desc = IndexDesc(self.v, self.d, self.c, self.b, _dtype_code(E),
                              FH_STAGE1_INT4_G32 if int4 else FH_STAGE1_DENSE,
                              E.data_ptr(), C.data_ptr() if C is not None else None,
                              C2T.data_ptr(),
                              C_q4.data_ptr() if C_q4 is not None else None,
                              C_scales.data_ptr() if C_scales is not None else None,
                              self.E_perm.data_ptr() if self.E_perm is not None else None)
        nbytes = L.fh_index_load_ws_bytes(ct.byref(self.desc))
        ws = torch.empty(nbytes, dtype=torch.uint8, device=E.device)
        handle = ct.c_void_p()
        _check(L.fh_index_load(ct.byref(self.desc), _ptr(ws), nbytes, _stream(stream),
                               ct.byref(handle)))
        self.handle = handle
        self._ws = {}

    def workspace_bytes(self, op, B, p=1, T=1, N=1) -> int:
        n = load().fh_workspace_bytes(self.handle, op, B, p, T, N)
        if n == 0:
            raise FlashHeadError(1, "invalid workspace request")
        return n

    def workspace(self, op, B, p=1, T=1, N=1) -> torch.Tensor:
        """A cached device workspace large enough for (op, B, p, T, N)."""
        n = self.workspace_bytes(op, B, p, T, N)
        key = (op,)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < n:
            ws = torch.zeros(n, dtype=torch.uint8, device=self.E.device)
            self._ws[key] = ws
        return ws

    def close(self):
        if getattr(self, "handle", None):
            load().fh_index_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _debug(debug):
    if debug is None:
        return None
    return ct.byref(DebugOut(*(debug.get(k).data_ptr() if debug.get(k) is not None else None
                                for k in ("sel", "cand_tok", "cand_logit"))))


def head_greedy(index: Index, H, p, out=None, ws=None, stream=None, debug=None):
    """Greedy FlashHead head: returns int32 token ids [B] (FlashHead notes, Module 2, Eq. 2)."""
    _need(H, "H")
    B = H.shape[0]
    out = out if out is not None else torch.empty(B, dtype=torch.int32, device=H.device)
    ws = ws if ws is not None else index.workspace(FH_OP_GREEDY, B, p)
    _check(load().fh_head_greedy(index.handle, _ptr(H), B, p, _ptr(out), _ptr(ws), ws.numel(),
                                 _stream(stream), _debug(debug)))
    return out


def head_greedy_host(index: Index, H_host, p, tok_host, h_dev, tok_dev, ws=None, stream=None):
    """head_greedy with host buffers: H_host (CPU, [B, d], pinned for an asynchronous copy) is copied
    to h_dev, the head runs into tok_dev, and the tokens are copied to tok_host (CPU int32 [B]), all
    queued on the stream in one library call; tok_host is valid once the stream has synchronised."""
    _need(h_dev, "h_dev")
    _need(tok_dev, "tok_dev")
    if H_host.is_cuda or tok_host.is_cuda or not H_host.is_contiguous() or not tok_host.is_contiguous():
        raise ValueError("H_host and tok_host must be contiguous host tensors")
    B = H_host.shape[0]
    if h_dev.shape != H_host.shape or h_dev.dtype != H_host.dtype or tok_dev.numel() < B or tok_host.numel() < B:
        raise ValueError("staging buffers do not match the queries")
    ws = ws if ws is not None else index.workspace(FH_OP_GREEDY, B, p)
    _check(load().fh_head_greedy_host(index.handle, _ptr(H_host), B, p, _ptr(tok_host), _ptr(h_dev),
                                      _ptr(tok_dev), _ptr(ws), ws.numel(), _stream(stream)))
    return tok_host


def head_sample(index: Index, H, p, tau, seed, step, out=None, ws=None, stream=None, debug=None):
    """Sampling FlashHead head (Gumbel-top-p, then Gumbel-max): int32 token ids [B]."""
    _need(H, "H")
    B = H.shape[0]
    out = out if out is not None else torch.empty(B, dtype=torch.int32, device=H.device)
    ws = ws if ws is not None else index.workspace(FH_OP_SAMPLE, B, p)
    _check(load().fh_head_sample(index.handle, _ptr(H), B, p, float(tau), seed, step, _ptr(out),
                                 _ptr(ws), ws.numel(), _stream(stream), _debug(debug)))
    return out


def dense_head(index: Index, H, sample=False, tau=1.0, seed=0, step=0, out=None, logits=None,
               ws=None, stream=None):
    """Dense head over all v tokens: int32 token ids [B] (and fp32 logits [B, v] if given)."""
    _need(H, "H")
    B = H.shape[0]
    out = out if out is not None else torch.empty(B, dtype=torch.int32, device=H.device)
    ws = ws if ws is not None else index.workspace(FH_OP_DENSE, B)
    _check(load().fh_dense_head(index.handle, _ptr(H), B, 1 if sample else 0, float(tau), seed,
                                step, _ptr(out), _ptr(logits), _ptr(ws), ws.numel(),
                                _stream(stream)))
    return out


def mc_token_prob(index: Index, H, targets, p, tau, N, seed, ws=None, stream=None, i0=None):
    """Monte Carlo marginal probabilities: (mean [B, T] fp64, se [B, T] fp64) over draws
    [0, N), or [i0, i0 + N) when i0 is given."""
    _need(H, "H")
    _need(targets, "targets")
    B, T = targets.shape
    mean = torch.empty((B, T), dtype=torch.float64, device=H.device)
    se = torch.empty((B, T), dtype=torch.float64, device=H.device)
    ws = ws if ws is not None else index.workspace(FH_OP_MC, B, p, T, N)
    if i0 is None:
        _check(load().fh_mc_token_prob(index.handle, _ptr(H), B, _ptr(targets), T, p, float(tau), N,
                                       seed, _ptr(mean), _ptr(se), _ptr(ws), ws.numel(),
                                       _stream(stream)))
    else:
        _check(load().fh_mc_token_prob_range(index.handle, _ptr(H), B, _ptr(targets), T, p, float(tau),
                                             i0, N, seed, _ptr(mean), _ptr(se), _ptr(ws), ws.numel(),
                                             _stream(stream)))
    return mean, se


def stage1_scores(index: Index, H, out=None, ws=None, stream=None):
    _need(H, "H")
    B = H.shape[0]
    out = out if out is not None else torch.empty((B, index.c), dtype=torch.float32, device=H.device)
    ws = ws if ws is not None else index.workspace(FH_OP_DENSE, B)
    _check(load().fh_stage1_scores(index.handle, _ptr(H), B, _ptr(out), _ptr(ws), ws.numel(),
                                   _stream(stream)))
    return out


def gumbel_keys(s, tau, seed, step, rng_stream=FH_RNG_STAGE1, out=None, stream=None):
    _need(s, "s")
    B, c = s.shape
    out = out if out is not None else torch.empty_like(s)
    _check(load().fh_gumbel_keys(_ptr(s), B, c, float(tau), seed, step, rng_stream, _ptr(out),
                                 _stream(stream)))
    return out


def select_topp(keys, p, out=None, stream=None):
    _need(keys, "keys")
    B, c = keys.shape
    out = out if out is not None else torch.empty((B, p), dtype=torch.int32, device=keys.device)
    _check(load().fh_select_topp(_ptr(keys), B, c, p, _ptr(out), _stream(stream)))
    return out


def gather_candidates(index: Index, sel, out=None, stream=None):
    _need(sel, "sel")
    B, p = sel.shape
    out = out if out is not None else torch.empty((B, p * index.b), dtype=torch.int32,
                                                  device=sel.device)
    _check(load().fh_gather_candidates(index.handle, _ptr(sel), B, p, _ptr(out), _stream(stream)))
    return out


def candidate_logits(index: Index, H, cand, out=None, stream=None):
    _need(H, "H")
    _need(cand, "cand")
    B, P = cand.shape
    out = out if out is not None else torch.empty((B, P), dtype=torch.float32, device=H.device)
    _check(load().fh_candidate_logits(index.handle, _ptr(H), B, _ptr(cand), P, _ptr(out),
                                      _stream(stream)))
    return out


def philox_u32(seed, step, row, rng_stream, n, device="cuda", stream=None):
    out = torch.empty(n, dtype=torch.int32, device=device)
    _check(load().fh_philox_u32(seed, step, row, rng_stream, n, _ptr(out), _stream(stream)))
    return out


def head_greedy_static(index: Index, H, p, out=None, stream=None):
    """Batch-1 greedy head that uses the library's static device scratch instead of a workspace."""
    _need(H, "H")
    if H.shape[0] != 1:
        raise ValueError("head_greedy_static takes one query")
    out = out if out is not None else torch.empty(1, dtype=torch.int32, device=H.device)
    _check(load().fh_head_greedy_static(index.handle, _ptr(H), p, _ptr(out), _stream(stream)))
    return out


def static_status(stream=None):
    """Raise if an allocation-free call recorded a device-side error in the static scratch (and zero
    its control block, so that the next call starts clean)."""
    _check(load().fh_static_status(_stream(stream)))


def static_scratch():
    """(device address, bytes) of the static scratch on the current device."""
    ptr, n = ct.c_void_p(), ct.c_size_t()
    _check(load().fh_static_scratch(ct.byref(ptr), ct.byref(n)))
    return ptr.value, n.value


def ws_status(ws, stream=None):
    """Raise if a previous call recorded a device-side error in this workspace."""
    _check(load().fh_ws_status(_ptr(ws), _stream(stream)))


def device_array(a, kind: str, device="cuda") -> torch.Tensor:
    """Copy a host array to the device: kind "f32" (float32), "bf16" (uint16 BF16 patterns),
    "i32", "u8"."""
    import numpy as np
    a = np.ascontiguousarray(a)
    if kind == "bf16":
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    elif kind == "f32":
        t = torch.from_numpy(a.astype(np.float32, copy=False))
    elif kind == "i32":
        t = torch.from_numpy(a.astype(np.int32, copy=False))
    elif kind == "u8":
        t = torch.from_numpy(a.astype(np.uint8, copy=False))
    else:
        raise ValueError(kind)
    return t.to(device)


def index_from_host(E, C, C2T, dtype: str, C_q4=None, C_scales=None, int4=False,
                    cluster_major=True, device="cuda") -> Index:
    """Upload host arrays (as produced by the synthetic generator) and load them as an Index."""
    Ed = device_array(E, dtype, device)
    Cd = device_array(C, dtype, device) if C is not None else None
    C2Td = device_array(C2T, "i32", device)
    q4 = device_array(C_q4, "u8", device) if C_q4 is not None else None
    sc = device_array(C_scales, "bf16", device) if C_scales is not None else None
    return Index(Ed, Cd, C2Td, q4, sc, int4=int4, cluster_major=cluster_major)


# ----------------------------------------------------------------------------- coarse-fine head


class CfIndex:
    """A coarse-fine head index (include/fh_cfhead.h): E [v, d] bf16, codebooks [T, K, w] float32,
    codes [T/8, v] int32 (the packed 4-bit index map, uint32 bit patterns).  Keeps them alive."""

    def __init__(self, E, codebooks, codes):
        for t, n in ((E, "E"), (codebooks, "codebooks"), (codes, "codes")):
            _need(t, n)
        if E.dtype != torch.bfloat16 or codebooks.dtype != torch.float32:
            raise TypeError("E must be bfloat16 and codebooks float32")
        self.E, self.codebooks, self.codes = E, codebooks, codes
        self.v, self.d = E.shape
        T, self.K, self.w = codebooks.shape
        self.desc = CfDesc(self.v, self.d, self.w, self.K, E.data_ptr(), codebooks.data_ptr(),
                           codes.data_ptr())
        h = ct.c_void_p()
        _check(load().fh_cf_load(ct.byref(self.desc), ct.byref(h)))
        self.handle = h

    def workspace_bytes(self, B, k) -> int:
        n = load().fh_cf_workspace_bytes(self.handle, B, k)
        if n == 0:
            raise FlashHeadError(1, "invalid workspace request")
        return n

    def close(self):
        if getattr(self, "handle", None):
            load().fh_cf_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def cf_index_from_host(E, codebooks, codes, device="cuda") -> CfIndex:
    """Upload a bf16 E (uint16 patterns), float32 codebooks and the packed uint32 index map."""
    import numpy as np
    cw = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint32).view(np.int32)).to(device)
    return CfIndex(device_array(E, "bf16", device), device_array(codebooks, "f32", device), cw)


def cf_head(index: CfIndex, H, k, sample=False, tau=1.0, seed=0, step=0, out=None, ws=None,
            stream=None, debug=None):
    """Coarse-fine head: int32 token ids [B].  debug: dict with optional "cand" (int32 [B, k]) and
    "coarse" (float32 [B, v]) device tensors to fill."""
    _need(H, "H")
    B = H.shape[0]
    out = out if out is not None else torch.empty(B, dtype=torch.int32, device=H.device)
    if ws is None:
        ws = torch.zeros(index.workspace_bytes(B, k), dtype=torch.uint8, device=H.device)
    debug = debug or {}
    _check(load().fh_cf_head(index.handle, _ptr(H), B, k, 1 if sample else 0, float(tau), seed, step,
                             _ptr(out), _ptr(ws), ws.numel(), _stream(stream), _ptr(debug.get("cand")),
                             _ptr(debug.get("coarse"))))
    return out


def cf_coarse_scores(index: CfIndex, H, ws=None, stream=None):
    """Coarse scores float32 [B, v] (the first step of cf_head)."""
    _need(H, "H")
    B = H.shape[0]
    if ws is None:
        ws = torch.zeros(index.workspace_bytes(B, 1), dtype=torch.uint8, device=H.device)
    out = torch.empty((B, index.v), dtype=torch.float32, device=H.device)
    _check(load().fh_cf_coarse_scores(index.handle, _ptr(H), B, _ptr(out), _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return out


# ----------------------------------------------------------------------------- index builder


def _kmeans_call(fn_name, E, c, stream, **fields):
    _need(E, "E")
    if E.dtype != torch.bfloat16 or E.dim() != 2:
        raise TypeError("E must be a v x d torch.bfloat16 matrix")
    v, d = E.shape
    L = load()
    nbytes = L.fh_kmeans_ws_bytes(v, d, c)
    if nbytes == 0:
        raise FlashHeadError(2, f"invalid builder sizes v={v} d={d} c={c}")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=E.device)
    keep = []
    args = KmeansArgs()
    args.E = E.data_ptr()
    args.dtype = FH_BF16
    args.v, args.d, args.c = v, d, c
    for name, value in fields.items():
        if isinstance(value, torch.Tensor):
            _need(value, name)
            keep.append(value)
            setattr(args, name, value.data_ptr())
        elif value is not None:
            setattr(args, name, value)
    _check(getattr(L, fn_name)(ct.byref(args), _ptr(ws), nbytes, _stream(stream)))
    return args


def kmeans_build(E, c, init_tokens, iters, eps=1e-4, max_rounds=0, stream=None):
    """Equal-size spherical k-means of the rows of E (v x d BF16) into c clusters, starting from
    the unit rows of init_tokens (c distinct ids, int32 on the device).  Returns a dict with labels
    (v), C2T (c x v/c), C (c x d fp32), C_bf16, objective (one Eq.4 value per update), prices
    (last auction), iters and rounds.  Synchronises the stream."""
    v, d = E.shape
    dev = E.device
    out = dict(labels=torch.empty(v, dtype=torch.int32, device=dev),
               C2T=torch.empty((c, v // c), dtype=torch.int32, device=dev),
               C=torch.empty((c, d), dtype=torch.float32, device=dev),
               C_bf16=torch.empty((c, d), dtype=torch.bfloat16, device=dev),
               objective=torch.zeros(iters, dtype=torch.float64, device=dev),
               prices=torch.empty(c, dtype=torch.float32, device=dev))
    a = _kmeans_call("fh_kmeans_build", E, c, stream, iters=iters, eps=eps, max_rounds=max_rounds,
                     init_tokens=init_tokens, **out)
    out["objective"] = out["objective"][:a.iters_done]
    out["iters"], out["rounds"] = a.iters_done, a.rounds
    return out


def kmeans_assign(E, C_bf16, eps=1e-4, max_rounds=0, stream=None):
    """The equal-size assignment of the rows of E to the BF16 centres C_bf16 (c x d), within
    v * eps of the optimum.  Returns labels, C2T, prices and rounds.  Synchronises the stream."""
    v, d = E.shape
    c = C_bf16.shape[0]
    dev = E.device
    out = dict(labels=torch.empty(v, dtype=torch.int32, device=dev),
               C2T=torch.empty((c, v // c), dtype=torch.int32, device=dev),
               prices=torch.empty(c, dtype=torch.float32, device=dev))
    a = _kmeans_call("fh_kmeans_assign", E, c, stream, eps=eps, max_rounds=max_rounds,
                     C_in=C_bf16, **out)
    out["rounds"] = a.rounds
    return out


def kmeans_update(E, labels, c, stream=None):
    """Eq.5 for an equal-size labeling: returns C2T, C (fp32 unit rows), C_bf16 and the objective
    of Eq.4 (one value).  Synchronises the stream."""
    v, d = E.shape
    dev = E.device
    out = dict(C2T=torch.empty((c, v // c), dtype=torch.int32, device=dev),
               C=torch.empty((c, d), dtype=torch.float32, device=dev),
               C_bf16=torch.empty((c, d), dtype=torch.bfloat16, device=dev),
               objective=torch.zeros(1, dtype=torch.float64, device=dev))
    _kmeans_call("fh_kmeans_update", E, c, stream, eps=1e-4, labels_in=labels, **out)
    return out
