"""Offline study: Stage-1 top-p recall of INT4 centroids against BF16 ones, as a function of the
centroid shift t in C' = C - t·mean(C) applied before quantisation (FlashHead notes, INT4 centroids;
the shift is the reparameterisation listed among the follow-ups).

The GPU path is unchanged by the shift: it scores whatever INT4 bytes the index holds.  This module
only prepares shifted, quantised centroids and measures, in float64 on the host, how many of the p
clusters chosen from the INT4 scores are among the p chosen from the BF16 scores.

    python -m clustered_retrieval_classification_b200.int4_shift_study

The synthetic centroids are isotropic (their mean is ~0, so a shift changes little); the study also
runs a variant whose unit centroids share a common direction (weight `common`), the situation the
shift targets: real head centroids have a dominant mean component.
"""

from __future__ import annotations

import math

import numpy as np

from . import synth


def dequantize_int4_g32(packed: np.ndarray, scales_bits: np.ndarray) -> np.ndarray:
    """float64 values q·scale of an INT4 g32 packing (low nibble = even column)."""
    rows = packed.shape[0]
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    q = np.empty((rows, packed.shape[1] * 2), dtype=np.int16)
    q[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    q[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    scale = synth.f32_from_bf16(scales_bits).astype(np.float64)
    return q.reshape(rows, -1, 32).astype(np.float64) * scale[:, :, None]


def topp_sets(scores: np.ndarray, p: int) -> np.ndarray:
    """Per row, the ids of the p largest scores (ties by lower id), as a boolean mask."""
    order = np.lexsort((np.broadcast_to(np.arange(scores.shape[1]), scores.shape), -scores), axis=1)
    mask = np.zeros(scores.shape, dtype=bool)
    np.put_along_axis(mask, order[:, :p], True, axis=1)
    return mask


def recall(C_ref: np.ndarray, C_int4: np.ndarray, H: np.ndarray, p: int) -> float:
    """Mean over queries of |top-p(C_int4·h) ∩ top-p(C_ref·h)| / p."""
    a = topp_sets(H @ C_ref.T, p)
    b = topp_sets(H @ C_int4.reshape(C_ref.shape).T, p)
    return float(np.mean(np.sum(a & b, axis=1) / p))


def anisotropic_centroids(c: int, d: int, common: float, seed: int) -> np.ndarray:
    """Unit centroids normalise(u + common·m·sqrt(d)) with u ~ N(0, I) and one fixed unit m."""
    rng = np.random.Generator(np.random.PCG64(seed))
    m = rng.standard_normal(d)
    m /= np.linalg.norm(m)
    u = rng.standard_normal((c, d)) + common * math.sqrt(d) * m[None, :]
    return u / np.linalg.norm(u, axis=1, keepdims=True)


def study(C: np.ndarray, H: np.ndarray, p: int, ts) -> dict:
    """Recall of INT4(shift(C, t)) against the BF16-rounded C, for each t."""
    C_ref = synth.stored_to_f64(synth.store(C.astype(np.float32), "bf16"), "bf16")
    out = {}
    for t in ts:
        Cs = synth.shift_centroids(C_ref, t)
        q, sc = synth.quantize_int4_g32(Cs)
        out[float(t)] = recall(C_ref, dequantize_int4_g32(q, sc), H, p)
    return out


def main(n_queries: int = 64, ts=(-2.0, -1.0, 0.0, 0.5, 1.0, 2.0, 4.0, 8.0)) -> dict:
    cfg = synth.CONFIGS["gemma"]
    idx = synth.make_index(cfg)
    H = synth.stored_to_f64(synth.make_queries(cfg, n_queries), "bf16")
    res = {"synthetic (isotropic)": study(synth.stored_to_f64(idx.C, "bf16"), H, cfg.p, ts)}
    for common in (0.5, 1.0):
        C = anisotropic_centroids(cfg.c, cfg.d, common, cfg.data_seed + 7)
        res[f"common direction {common}"] = study(C, H, cfg.p, ts)
    for name, r in res.items():
        print(f"{name:24s} " + "  ".join(f"t={t:+.1f}: {v:.4f}" for t, v in r.items()))
    return res


if __name__ == "__main__":
    main()
