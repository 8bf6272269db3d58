"""Checks of the index builder's results against the equal-size k-means oracle, shared by the CPU
tests of the builder's host build and the GPU tests of the device build.

Several labelings can be equally good, so what is compared is what the definitions fix:
  * assignment: equal-size, C2T consistent with the labels, the returned prices certify
    eps-complementary slackness on the oracle's float64 similarities, and the value is within
    v * (eps + tol) of the exact optimum (linear assignment);
  * update (Eq.5): centres and objective element by element against the oracle's float64 update
    of the same labels, BF16 centres = the fp32 centres rounded to nearest even;
  * a whole run: the final centres are Eq.5 of the final labels, and the objective of Eq.4 falls
    from one iteration to the next up to the auction's v * eps and the BF16 scoring of the centres.
"""

import numpy as np

from clustered_retrieval_classification_b200 import synth
from oracle import kmeans_oracle as K

SIM_TOL = 2e-5      # |fp32 similarity (fp32 dot, fp32 1/|e|) - float64 similarity| for |cos| <= 1
CENTRE_TOL = 2e-5   # fp32 member sums over b rows of unit vectors, then normalised
BF16_SCORING = 8e-3 # per-token change of a cosine when the centre is rounded to BF16 (2^-8 relative)


def check_assignment(E, C_in, c, eps, labels, C2T, prices):
    X = K.unit_rows(E)
    Cs = K.stored_to_f64(C_in)
    A = X @ Cs.T
    v = X.shape[0]
    b = v // c
    assert K.is_equal_size(labels, c, b)
    assert np.array_equal(C2T, K.c2t_from_labels(labels, c, b))
    gap = K.eps_cs_gap(A, labels, prices.astype(np.float64))
    assert gap <= eps + 2 * SIM_TOL, gap
    best = K.assignment_value(A, K.assign_equal_size(X, Cs, b))
    got = K.assignment_value(A, labels)
    assert got >= best - v * (eps + 2 * SIM_TOL), (got, best)
    return got, best


def check_update(E, labels, c, C, C_bf16, objective0):
    X = K.unit_rows(E)
    Co = K.update_centres(X, np.asarray(labels, dtype=np.int64), c)
    assert np.abs(C.astype(np.float64) - Co).max() <= CENTRE_TOL
    assert np.array_equal(C_bf16, synth.bf16_from_f32(C.astype(np.float32)))
    J = K.objective(X, Co, np.asarray(labels, dtype=np.int64))
    assert abs(objective0 - J) <= 1e-5 * abs(J) + 1e-6
    return Co


def check_run(E, c, labels, C2T, C, C_bf16, history, eps):
    X = K.unit_rows(E)
    v = X.shape[0]
    b = v // c
    assert K.is_equal_size(labels, c, b)
    assert np.array_equal(C2T, K.c2t_from_labels(labels, c, b))
    Co = K.update_centres(X, np.asarray(labels, dtype=np.int64), c)
    assert np.abs(C.astype(np.float64) - Co).max() <= CENTRE_TOL
    assert np.array_equal(C_bf16, synth.bf16_from_f32(C.astype(np.float32)))
    slack = v * (eps + 2 * SIM_TOL + 2 * BF16_SCORING)
    for a, bb in zip(history, history[1:]):
        assert bb <= a + slack, (a, bb)
    assert abs(history[-1] - K.objective(X, Co, np.asarray(labels, dtype=np.int64))) <= 1e-5 * v
