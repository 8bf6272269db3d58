"""The offline centroid shift C' = C - t·mean(C) before INT4 quantisation (host only; the GPU run of
the shifted bytes is in test_gpu_fullsize.py).  Pins: the top-p set of exact scores does not move
with t (every score of a query shifts by the same amount); the shift removes the mean at t = 1; the
packing that quantize_int4_g32 writes decodes to the oracle's INT4 scores; the set recall used by
the benchmark is 1 for a set against itself."""

import numpy as np

from clustered_retrieval_classification_b200 import synth


def dequantize_int4_g32(packed, scales_bits):
    """float64 values q·scale of an INT4 g32 packing (low nibble = even column)."""
    rows = packed.shape[0]
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    q = np.empty((rows, packed.shape[1] * 2), dtype=np.int16)
    q[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    q[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    scale = synth.f32_from_bf16(scales_bits).astype(np.float64)
    return (q.reshape(rows, -1, 32).astype(np.float64) * scale[:, :, None]).reshape(rows, -1)


def topp_sets(scores, p):
    """Per row, the ids of the p largest scores (ties by lower id), as a boolean mask."""
    order = np.lexsort((np.broadcast_to(np.arange(scores.shape[1]), scores.shape), -scores), axis=1)
    mask = np.zeros(scores.shape, dtype=bool)
    np.put_along_axis(mask, order[:, :p], True, axis=1)
    return mask


def recall(C_ref, C_other, H, p):
    """Mean over queries of |top-p(C_other·h) ∩ top-p(C_ref·h)| / p."""
    a = topp_sets(H @ C_ref.T, p)
    b = topp_sets(H @ C_other.T, p)
    return float(np.mean(np.sum(a & b, axis=1) / p))


def test_shift_leaves_exact_top_p_unchanged():
    rng = np.random.default_rng(11)
    C = rng.standard_normal((300, 64))
    C /= np.linalg.norm(C, axis=1, keepdims=True)
    C += 0.8 * rng.standard_normal(64)[None, :] / 8.0   # a common direction, as in real heads
    H = rng.standard_normal((12, 64))
    ref = topp_sets(H @ C.T, 25)
    for t in (-2.0, 0.5, 1.0, 8.0):
        assert np.array_equal(topp_sets(H @ synth.shift_centroids(C, t).T, 25), ref)


def test_shift_removes_the_mean_at_t_one():
    rng = np.random.default_rng(3)
    C = rng.standard_normal((50, 32)) + 2.0
    assert np.allclose(synth.shift_centroids(C, 1.0).mean(axis=0), 0.0, atol=1e-12)


def test_packing_decodes_to_the_oracle_int4_scores(orc):
    rng = np.random.default_rng(5)
    c, d = 40, 96
    C = rng.standard_normal((c, d)) / np.sqrt(d)
    q, sc = synth.quantize_int4_g32(C)
    H = synth.store(rng.standard_normal((3, d)).astype(np.float32), "bf16")
    Hf = synth.stored_to_f64(H, "bf16")
    mine = Hf @ dequantize_int4_g32(q, sc).T
    theirs = orc.stage1_scores(None, "bf16", H, c, d, q4=q, scales=sc)
    assert np.abs(mine - theirs).max() <= 1e-12


def test_recall_of_a_set_against_itself_is_one_and_drops_with_noise():
    rng = np.random.default_rng(8)
    C = rng.standard_normal((200, 32))
    H = rng.standard_normal((10, 32))
    assert recall(C, C, H, 20) == 1.0
    assert recall(C, C + 0.5 * rng.standard_normal(C.shape), H, 20) < 1.0


def test_anisotropic_centroids_share_a_direction():
    C = synth.anisotropic_centroids(400, 64, 1.0, seed=4)
    assert np.allclose(np.linalg.norm(C, axis=1), 1.0)
    m = C.mean(axis=0)
    assert np.linalg.norm(m) > 0.5                       # a dominant common component
    assert np.linalg.norm(synth.shift_centroids(C, 1.0).mean(axis=0)) < 1e-12
