"""Comparison rules between the CUDA path and the oracle.

Tolerances (fp32 accumulation of BF16 products against float64):
  * logits and Stage-1 scores: |Δ| <= 2e-3 absolute (the error bound of an fp32 sum of d = 2048
    products of size up to |e||h| ~ 24 is d·2^-24·Σ|e_j h_j| ≈ 3e-3 in the worst case; observed errors
    are ~1e-5);
  * an index set must be identical whenever the oracle's p-th-cluster margin exceeds 4e-3; below it,
    the clusters that differ must lie within 4e-3 of the threshold;
  * a token id must be identical whenever the sets agree and the oracle's top-1 margin exceeds 4e-3;
    otherwise the token must be a near-maximum (within 4e-3) of the oracle's decision keys over the
    candidates the GPU used;
  * Monte Carlo means (same Philox draws on both sides) within max(1e-9, 1e-3·mean, 0.1·se) and
    standard errors within max(1e-12, 1e-2·se): relative bounds, so that a target of probability
    ~1/v is checked as closely as a likely one.  The slack covers draws whose probe sets differ
    because the GPU forms the keys in fp32 (a near-tie at the p-th key).
"""

import numpy as np

LOGIT_TOL = 2e-3
MARGIN = 4e-3


def check_sets(gpu_sel, orc_sel, orc_keys, set_margin, tol=MARGIN):
    """Returns the number of queries whose sets differ (all of them within the margin rule)."""
    differ = 0
    for q in range(gpu_sel.shape[0]):
        g, o = set(gpu_sel[q].tolist()), set(orc_sel[q].tolist())
        assert len(g) == len(o) == gpu_sel.shape[1]
        assert np.all(np.diff(gpu_sel[q]) > 0), "probe set must be ascending"
        if g == o:
            continue
        differ += 1
        assert set_margin[q] <= tol, f"query {q}: sets differ with margin {set_margin[q]}"
        k = np.sort(orc_keys[q])[::-1]
        p = gpu_sel.shape[1]
        thr = 0.5 * (k[p - 1] + k[p])
        for cl in g ^ o:
            assert abs(orc_keys[q][cl] - thr) <= tol, f"query {q}: cluster {cl} far from threshold"
    return differ


def check_tokens(gpu_tok, orc_tok, tok_margin, same_set, valid_fn, tol=MARGIN):
    """valid_fn(q, tok) -> (best decision key, decision key of tok) over the GPU's candidates."""
    differ = 0
    for q in range(len(gpu_tok)):
        if gpu_tok[q] == orc_tok[q]:
            continue
        differ += 1
        assert (not same_set[q]) or tok_margin[q] <= tol, (
            f"query {q}: token {gpu_tok[q]} != {orc_tok[q]} with margin {tok_margin[q]}")
        best, mine = valid_fn(q, int(gpu_tok[q]))
        assert mine >= best - tol, f"query {q}: GPU token is not a near-maximum"
    return differ


def check_mc(mean, se, o):
    """GPU Monte Carlo estimates against the oracle's on the same draws (see the module docstring)."""
    tol = np.maximum(np.maximum(1e-9, 1e-3 * np.abs(o["mean"])), 0.1 * o["se"])
    assert np.all(np.abs(mean - o["mean"]) <= tol), (mean, o["mean"], tol)
    assert np.all(np.abs(se - o["se"]) <= np.maximum(1e-12, 1e-2 * o["se"])), (se, o["se"])
