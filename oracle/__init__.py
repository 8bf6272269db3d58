"""CPU oracle of the FlashHead head — TEST INFRASTRUCTURE ONLY.

Thin numpy/ctypes wrapper around flashhead_oracle.c (float64 restatement of the method; see the
header comment of that file for the steps and their sources).  Only tests/, the smoke check and the
benchmark's CPU-baseline leg may import this package; the product path never does, and this package
imports nothing from the product package.

Arrays are passed as stored: float32 values for dtype "f32", uint16 BF16 bit patterns for "bf16".
"""

from __future__ import annotations

import ctypes as ct

import numpy as np

from . import build as _build

_lib = None

F32, BF16 = 0, 1
_DT = {"f32": F32, "bf16": BF16}

_p = ct.c_void_p
_i64 = ct.c_int64
_i32 = ct.c_int
_u32 = ct.c_uint32
_u64 = ct.c_uint64
_f64 = ct.c_double


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ct.CDLL(path)
        L.orc_philox4x32_10.argtypes = [_p, _p, _p]
        L.orc_draw_u32.argtypes = [_u64, _u64, _u32, _u32, _u64]
        L.orc_draw_u32.restype = _u32
        L.orc_philox_words.argtypes = [_u64, _u64, _u32, _u32, _i64, _p]
        L.orc_uniform.argtypes = [_u32]
        L.orc_uniform.restype = _f64
        L.orc_gumbel.argtypes = [_u32]
        L.orc_gumbel.restype = _f64
        L.orc_stage1_scores.argtypes = [_p, _i32, _p, _p, _i32, _i64, _i64, _p, _i32, _p]
        L.orc_gumbel_keys.argtypes = [_p, _i32, _i64, _f64, _u64, _u64, _u32, _p]
        L.orc_select_topp.argtypes = [_p, _i32, _i64, _i32, _p, _p]
        L.orc_gather.argtypes = [_p, _i64, _p, _i32, _i32, _p]
        L.orc_logits.argtypes = [_p, _i32, _i64, _p, _i32, _p, _i64, _p]
        L.orc_head.argtypes = [_p, _p, _i32, _p, _p, _i32, _p, _i64, _i64, _i64, _i64, _p, _i32,
                               _i32, _i32, _f64, _u64, _u64, _p, _p, _p, _p, _p, _p, _p]
        L.orc_dense.argtypes = [_p, _i32, _i64, _i64, _p, _i32, _i32, _f64, _u64, _u64, _p, _p, _p]
        L.orc_mc.argtypes = [_p, _p, _i32, _p, _p, _i32, _p, _i64, _i64, _i64, _i64, _p, _i32, _p,
                             _i32, _i32, _f64, _i64, _i64, _u64, _p, _p, _p]
        L.orc_num_threads.restype = _i32
        L.orc_set_num_threads.argtypes = [_i32]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ct.c_void_p)


def _c(a, dtype=None):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Threads the oracle's parallel loops use from now on (timing only; results do not change)."""
    lib().orc_set_num_threads(int(n))


# ----------------------------------------------------------------------------- Philox


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def draw_u32(seed, step, row, stream, elem) -> int:
    return int(lib().orc_draw_u32(seed, step, row, stream, elem))


def philox_words(seed, step, row, stream, n) -> np.ndarray:
    out = np.zeros(n, dtype=np.uint32)
    lib().orc_philox_words(seed, step, row, stream, n, _ptr(out))
    return out


def uniform(x: int) -> float:
    return float(lib().orc_uniform(x))


def gumbel(x: int) -> float:
    return float(lib().orc_gumbel(x))


# ----------------------------------------------------------------------------- steps


def stage1_scores(C, dtype, H, c, d, q4=None, scales=None) -> np.ndarray:
    """s = C·h for every row of H, float64 [B, c]."""
    H = _c(H)
    B = H.shape[0]
    s = np.zeros((B, c), dtype=np.float64)
    fmt = 1 if q4 is not None else 0
    C = _c(C)
    q4 = _c(q4, np.uint8)
    scales = _c(scales, np.uint16)
    lib().orc_stage1_scores(_ptr(C), _DT[dtype], _ptr(q4), _ptr(scales), fmt, c, d, _ptr(H), B,
                            _ptr(s))
    return s


def gumbel_keys(s, tau, seed, step, stream) -> np.ndarray:
    s = _c(s, np.float64)
    B, c = s.shape
    keys = np.zeros_like(s)
    lib().orc_gumbel_keys(_ptr(s), B, c, tau, seed, step, stream, _ptr(keys))
    return keys


def select_topp(keys, p):
    """Returns (sel [B, p] ascending ids, margin [B])."""
    keys = _c(keys, np.float64)
    B, c = keys.shape
    sel = np.zeros((B, p), dtype=np.int32)
    margin = np.zeros(B, dtype=np.float64)
    lib().orc_select_topp(_ptr(keys), B, c, p, _ptr(sel), _ptr(margin))
    return sel, margin


def gather(C2T, sel) -> np.ndarray:
    C2T = _c(C2T, np.int32)
    sel = _c(sel, np.int32)
    B, p = sel.shape
    b = C2T.shape[1]
    cand = np.zeros((B, p * b), dtype=np.int32)
    lib().orc_gather(_ptr(C2T), b, _ptr(sel), B, p, _ptr(cand))
    return cand


def logits(E, dtype, H, cand) -> np.ndarray:
    E = _c(E)
    H = _c(H)
    cand = _c(cand, np.int32)
    B, P = cand.shape
    z = np.zeros((B, P), dtype=np.float64)
    lib().orc_logits(_ptr(E), _DT[dtype], E.shape[1], _ptr(H), B, _ptr(cand), P, _ptr(z))
    return z


# ----------------------------------------------------------------------------- whole calls


def head(index, H, p, sample=False, tau=1.0, seed=0, step=0, use_int4=None):
    """Greedy (sample=False) or sampling FlashHead on every row of H.

    index: an object with E, C, C2T, cfg (dtype, v, d, c, b) and optionally C_q4/C_scales.
    Returns a dict of numpy arrays: tok, sel, cand, z, dec, set_margin, tok_margin."""
    cfg = index.cfg
    H = _c(H)
    B = H.shape[0]
    b = cfg.v // cfg.c
    P = p * b
    if use_int4 is None:
        use_int4 = getattr(index, "C_q4", None) is not None and cfg.int4
    q4 = _c(index.C_q4, np.uint8) if use_int4 else None
    sc = _c(index.C_scales, np.uint16) if use_int4 else None
    out = dict(tok=np.zeros(B, np.int32), sel=np.zeros((B, p), np.int32),
               cand=np.zeros((B, P), np.int32), z=np.zeros((B, P)), dec=np.zeros((B, P)),
               set_margin=np.zeros(B), tok_margin=np.zeros(B))
    E = _c(index.E)
    C = _c(index.C)
    C2T = _c(index.C2T, np.int32)
    lib().orc_head(_ptr(E), _ptr(C), _DT[cfg.dtype], _ptr(q4), _ptr(sc), 1 if use_int4 else 0,
                   _ptr(C2T), cfg.v, cfg.d, cfg.c, b, _ptr(H), B, p, 1 if sample else 0,
                   float(tau), seed, step, _ptr(out["tok"]), _ptr(out["sel"]), _ptr(out["cand"]),
                   _ptr(out["z"]), _ptr(out["dec"]), _ptr(out["set_margin"]),
                   _ptr(out["tok_margin"]))
    return out


def dense(index, H, sample=False, tau=1.0, seed=0, step=0, want_z=False):
    """Dense head over all v tokens.  Returns dict(tok, tok_margin[, z])."""
    cfg = index.cfg
    H = _c(H)
    B = H.shape[0]
    tok = np.zeros(B, np.int32)
    margin = np.zeros(B)
    z = np.zeros((B, cfg.v)) if want_z else None
    E = _c(index.E)
    lib().orc_dense(_ptr(E), _DT[cfg.dtype], cfg.v, cfg.d, _ptr(H), B, 1 if sample else 0,
                    float(tau), seed, step, _ptr(tok), _ptr(z), _ptr(margin))
    out = dict(tok=tok, tok_margin=margin)
    if want_z:
        out["z"] = z
    return out


def mc(index, H, targets, p, tau, seed, n_draws=None, i0=0, i1=None, use_int4=None,
       per_draw=False):
    """Monte Carlo marginal over draws [i0, i1).  Returns dict(mean, se[, per_draw])."""
    cfg = index.cfg
    H = _c(H)
    targets = _c(targets, np.int32)
    B, T = targets.shape
    if i1 is None:
        i1 = i0 + n_draws
    n = i1 - i0
    if use_int4 is None:
        use_int4 = getattr(index, "C_q4", None) is not None and cfg.int4
    q4 = _c(index.C_q4, np.uint8) if use_int4 else None
    sc = _c(index.C_scales, np.uint16) if use_int4 else None
    pd = np.zeros((B, n, T)) if per_draw else None
    mean = np.zeros((B, T))
    se = np.zeros((B, T))
    E = _c(index.E)
    C = _c(index.C)
    C2T = _c(index.C2T, np.int32)
    b = cfg.v // cfg.c
    lib().orc_mc(_ptr(E), _ptr(C), _DT[cfg.dtype], _ptr(q4), _ptr(sc), 1 if use_int4 else 0,
                 _ptr(C2T), cfg.v, cfg.d, cfg.c, b, _ptr(H), B, _ptr(targets), T, p, float(tau),
                 i0, i1, seed, _ptr(pd), _ptr(mean), _ptr(se))
    out = dict(mean=mean, se=se)
    if per_draw:
        out["per_draw"] = pd
    return out
