"""The offline centroid shift C' = C - t·mean(C) before INT4 quantisation, and the helpers of its
recall study (host only).  Pins: the top-p set of exact scores does not move with t (every score of a
query shifts by the same amount); the study's dequantiser agrees with the oracle's INT4 scores; the
recall of a set against itself is 1."""

import numpy as np

from clustered_retrieval_classification_b200 import int4_shift_study as S
from clustered_retrieval_classification_b200 import synth


def test_shift_leaves_exact_top_p_unchanged():
    rng = np.random.default_rng(11)
    C = rng.standard_normal((300, 64))
    C /= np.linalg.norm(C, axis=1, keepdims=True)
    C += 0.8 * rng.standard_normal(64)[None, :] / 8.0   # a common direction, as in real heads
    H = rng.standard_normal((12, 64))
    ref = S.topp_sets(H @ C.T, 25)
    for t in (-2.0, 0.5, 1.0, 8.0):
        assert np.array_equal(S.topp_sets(H @ synth.shift_centroids(C, t).T, 25), ref)


def test_shift_removes_the_mean_at_t_one():
    rng = np.random.default_rng(3)
    C = rng.standard_normal((50, 32)) + 2.0
    assert np.allclose(synth.shift_centroids(C, 1.0).mean(axis=0), 0.0, atol=1e-12)


def test_dequantiser_matches_the_oracle_int4_scores(orc):
    rng = np.random.default_rng(5)
    c, d = 40, 96
    C = rng.standard_normal((c, d)) / np.sqrt(d)
    q, sc = synth.quantize_int4_g32(C)
    H = synth.store(rng.standard_normal((3, d)).astype(np.float32), "bf16")
    Hf = synth.stored_to_f64(H, "bf16")
    mine = Hf @ S.dequantize_int4_g32(q, sc).reshape(c, d).T
    theirs = orc.stage1_scores(None, "bf16", H, c, d, q4=q, scales=sc)
    assert np.abs(mine - theirs).max() <= 1e-12


def test_recall_of_a_set_against_itself_is_one_and_drops_with_noise():
    rng = np.random.default_rng(8)
    C = rng.standard_normal((200, 32))
    H = rng.standard_normal((10, 32))
    assert S.recall(C, C, H, 20) == 1.0
    assert S.recall(C, C + 0.5 * rng.standard_normal(C.shape), H, 20) < 1.0
