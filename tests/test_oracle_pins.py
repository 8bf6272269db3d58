"""Pins of the CPU oracle against facts fixed outside it.

Each test checks the oracle against something it does not compute itself: published known-answer
vectors, closed forms, a library routine for a special case, exhaustive enumeration on tiny inputs,
or exact distributions.  Sources: "FlashHead notes" (reading-notes page of "FlashHead: Efficient
Drop-In Replacement for the Classification Head in Language Model Inference": overall architecture,
Modules 1–4, Eq. 1–7) and the SC'11 Philox paper.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy import stats

from clustered_retrieval_classification_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
EULER_GAMMA = 0.5772156649015329


def widen(a, dtype):
    """Exact float64 values of stored data, computed with torch (independent of the oracle)."""
    if dtype == "f32":
        return torch.from_numpy(np.asarray(a, np.float32)).double().numpy()
    return torch.from_numpy(np.asarray(a, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def top_p_reference(keys, p):
    """Top-p by the definition: the unique set S with |S| = p such that every member beats every
    non-member under (key desc, id asc).  Found by enumerating all subsets (tiny c only)."""
    c = len(keys)
    found = []
    for S in itertools.combinations(range(c), p):
        inside = set(S)
        ok = all((keys[i] > keys[j]) or (keys[i] == keys[j] and i < j)
                 for i in inside for j in range(c) if j not in inside)
        if ok:
            found.append(S)
    assert len(found) == 1
    return list(found[0])


# ----------------------------------------------------------------------------- Philox


def test_philox_known_answers(orc):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        vals = [int(x, 16) for x in r]
        out = orc.philox4x32_10(vals[0:4], vals[4:6])
        assert out.tolist() == vals[6:10]


def test_counter_layout(orc):
    seed, step, row, stream = 0x0123456789ABCDEF, (7 << 32) | 99, 5, 2
    for elem in [0, 1, 2, 3, 4, 5, 1023, 123457]:
        ctr = [elem >> 2, row, step & 0xFFFFFFFF, (stream << 24) | ((step >> 32) & 0xFFFFFF)]
        key = [seed & 0xFFFFFFFF, seed >> 32]
        assert orc.draw_u32(seed, step, row, stream, elem) == int(orc.philox4x32_10(ctr, key)[elem & 3])
    words = orc.philox_words(seed, step, row, stream, 64)
    assert [orc.draw_u32(seed, step, row, stream, e) for e in range(64)] == words.tolist()


def test_uniform_endpoints(orc):
    assert orc.uniform(0) == 0.5 * 2.0 ** -23
    assert orc.uniform(0xFFFFFFFF) == (2.0 ** 23 - 0.5) * 2.0 ** -23
    # every value is exactly representable in fp32 (at most 24 significant bits)
    for x in (0, 1 << 9, 0x7FFFFFFF, 0xFFFFFE00, 0xFFFFFFFF):
        assert float(np.float32(orc.uniform(x))) == orc.uniform(x)
    assert 0.0 < orc.uniform(0) < orc.uniform(0xFFFFFFFF) < 1.0
    # G = -log(-log u) at the middle of the range
    x = 0x80000000
    u = ((x >> 9) + 0.5) / 2 ** 23
    assert orc.gumbel(x) == pytest.approx(-math.log(-math.log(u)), rel=0, abs=1e-15)


def test_gumbel_distribution(orc):
    """Standard Gumbel: mean = Euler's gamma, variance = pi^2/6, CDF exp(-exp(-x))."""
    n = 200_000
    words = orc.philox_words(12345, 3, 1, 0, n)
    g = np.array([orc.gumbel(int(x)) for x in words[:20000]])
    u = (((words.astype(np.float64) // 512) + 0.5) / 2 ** 23)
    gall = -np.log(-np.log(u))
    np.testing.assert_allclose(g, gall[:20000], rtol=0, atol=1e-15)
    se_mean = math.pi / math.sqrt(6) / math.sqrt(n)
    assert abs(gall.mean() - EULER_GAMMA) < 5 * se_mean
    assert abs(gall.var() - math.pi ** 2 / 6) < 0.03
    ks = stats.kstest(gall, lambda x: np.exp(-np.exp(-x)))
    assert ks.pvalue > 1e-3


# ----------------------------------------------------------------------------- Stage 1


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_stage1_scores_equal_matmul(orc, dtype):
    rng = np.random.default_rng(7)
    c, d, B = 37, 96, 3
    C = synth.store(rng.standard_normal((c, d)).astype(np.float32), dtype)
    H = synth.store(rng.standard_normal((B, d)).astype(np.float32), dtype)
    s = orc.stage1_scores(C, dtype, H, c, d)
    ref = widen(H, dtype) @ widen(C, dtype).T
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-13)


def test_int4_packing_and_closed_form(orc):
    # packing of known values: low nibble = even column, two's complement
    x = np.array([[-7, 7, -1, 0, 3, -3] + [0] * 26], dtype=np.float64) * 0.5
    packed, scales = synth.quantize_int4_g32(x)
    assert synth.f32_from_bf16(scales)[0, 0] == np.float32(0.5)        # max|x| / 7
    assert packed[0, :3].tolist() == [0x79, 0x0F, 0xD3]                 # (-7, 7), (-1, 0), (3, -3)
    assert packed[0, 3:].tolist() == [0] * 13
    rng = np.random.default_rng(3)
    c, d = 9, 64
    C = rng.standard_normal((c, d))
    C /= np.linalg.norm(C, axis=1, keepdims=True)
    q4, sc = synth.quantize_int4_g32(C)
    # unpack with independent code
    lo = (q4 & 0xF).astype(np.int16)
    hi = (q4 >> 4).astype(np.int16)
    q = np.empty((c, d), np.int16)
    q[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    q[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    assert q.min() >= -8 and q.max() <= 7
    scale = widen(sc, "bf16")
    H = synth.store(rng.standard_normal((2, d)).astype(np.float32), "bf16")
    h = widen(H, "bf16")
    # closed form: s_k = Σ_g scale_g Σ_{j in g} q_j h_j
    ref = np.zeros((2, c))
    for qi in range(2):
        for k in range(c):
            ref[qi, k] = sum(scale[k, g] * float(np.dot(q[k, 32 * g:32 * g + 32], h[qi, 32 * g:32 * g + 32]))
                             for g in range(d // 32))
    s = orc.stage1_scores(None, "bf16", H, c, d, q4=q4, scales=sc)
    np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-14)
    # the quantiser reconstructs within half a step per element
    recon = q * np.repeat(scale, 32, axis=1)
    assert np.all(np.abs(recon - C) <= np.repeat(scale, 32, axis=1) * 0.5 + 1e-12)


# ----------------------------------------------------------------------------- selection


def test_select_against_definition(orc):
    rng = np.random.default_rng(11)
    for trial in range(60):
        c = int(rng.integers(1, 9))
        p = int(rng.integers(1, c + 1))
        keys = rng.integers(-3, 4, size=c).astype(np.float64)   # many ties
        if trial % 3 == 0:
            keys = rng.standard_normal(c)
        if trial % 7 == 0:
            keys[:] = -0.0
            keys[::2] = 0.0
        sel, margin = orc.select_topp(keys[None, :], p)
        assert sel[0].tolist() == top_p_reference(keys.tolist(), p)
        srt = sorted(keys, reverse=True)
        exp_margin = srt[p - 1] - srt[p] if p < c else math.inf
        assert margin[0] == exp_margin


def test_select_large_invariants(orc):
    rng = np.random.default_rng(5)
    c, p = 8016, 512
    keys = np.round(rng.standard_normal((2, c)), 2)   # rounded: ties at the boundary
    sel, _ = orc.select_topp(keys, p)
    for q in range(2):
        S = sel[q]
        assert len(S) == p and np.all(np.diff(S) > 0)
        mask = np.zeros(c, bool)
        mask[S] = True
        kin, kout = keys[q][mask], keys[q][~mask]
        assert kin.min() >= kout.max()
        tie = kin.min()
        if tie == kout.max():
            assert np.flatnonzero(mask & (keys[q] == tie)).max() < np.flatnonzero(~mask & (keys[q] == tie)).min()


# ----------------------------------------------------------------------------- Stage 2


def test_gather_and_logits(orc):
    idx = synth.random_index(v=48, d=16, c=6, seed=21, dtype="bf16")
    sel = np.array([[0, 2, 5], [1, 3, 4]], np.int32)
    cand = orc.gather(idx.C2T, sel)
    for q in range(2):
        for r in range(3):
            for j in range(8):
                assert cand[q, r * 8 + j] == idx.C2T[sel[q, r], j]
    H = synth.store(np.random.default_rng(2).standard_normal((2, 16)).astype(np.float32), "bf16")
    z = orc.logits(idx.E, "bf16", H, cand)
    Ew, hw = widen(idx.E, "bf16"), widen(H, "bf16")
    for q in range(2):
        np.testing.assert_allclose(z[q], Ew[cand[q]] @ hw[q], rtol=1e-13, atol=1e-13)


def _tiny_greedy_by_hand(E, C, C2T, h, p):
    """Pure-Python restatement on a tiny head: scores, sort, candidates, argmax."""
    c, b = C2T.shape
    s = [sum(C[k][j] * h[j] for j in range(len(h))) for k in range(c)]
    order = sorted(range(c), key=lambda k: (-s[k], k))
    S = sorted(order[:p])
    best_t, best_z = None, None
    for k in S:
        for j in range(b):
            t = int(C2T[k][j])
            z = sum(E[t][i] * h[i] for i in range(len(h)))
            if best_t is None or z > best_z or (z == best_z and t < best_t):
                best_t, best_z = t, z
    return best_t, S


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_greedy_brute_force_tiny(orc, seed):
    idx = synth.random_index(v=24, d=8, c=6, seed=100 + seed, dtype="f32")
    H = np.random.default_rng(seed).standard_normal((3, 8)).astype(np.float32)
    out = orc.head(idx, H, p=2)
    E, C, hh = widen(idx.E, "f32"), widen(idx.C, "f32"), widen(H, "f32")
    for q in range(3):
        t, S = _tiny_greedy_by_hand(E.tolist(), C.tolist(), idx.C2T, hh[q].tolist(), 2)
        assert out["tok"][q] == t
        assert out["sel"][q].tolist() == S


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_p_equals_c_greedy_is_dense_argmax(orc, dtype):
    """With p = c every cluster is probed, so the candidates are the whole vocabulary and FlashHead
    greedy must equal the dense head's argmax (FlashHead notes, Eq. 1 and Eq. 2)."""
    cfg = synth.scaled(synth.CONFIGS["tiny"], v=2048, c=32, d=64)
    cfg = synth.dataclasses.replace(cfg, dtype=dtype)
    idx = synth.make_index(cfg)
    H = synth.make_queries(cfg, 6)
    out = orc.head(idx, H, p=cfg.c)
    z = widen(H, dtype) @ widen(idx.E, dtype).T          # textbook matvec
    ref = np.argmax(z, axis=1)                            # first index among equal maxima
    assert out["tok"].tolist() == ref.tolist()
    assert orc.dense(idx, H)["tok"].tolist() == ref.tolist()


def test_p_equals_c_sampling_is_dense_sampling(orc):
    """With p = c FlashHead sampling and dense sampling draw the same token: the Stage-2 noise is keyed
    by token id on the same stream."""
    idx = synth.random_index(v=96, d=16, c=8, seed=7, dtype="bf16")
    H = synth.store(np.random.default_rng(9).standard_normal((4, 16)).astype(np.float32), "bf16")
    for step in range(5):
        a = orc.head(idx, H, p=8, sample=True, tau=0.8, seed=42, step=step)["tok"]
        bd = orc.dense(idx, H, sample=True, tau=0.8, seed=42, step=step)["tok"]
        assert a.tolist() == bd.tolist()


# ----------------------------------------------------------------------------- distributions


def _pair_probs(w):
    """Exact distribution of the unordered pair drawn by sequential sampling without replacement
    with weights w (successive draws proportional to the remaining weights)."""
    W = w.sum()
    probs = {}
    for a, b_ in itertools.combinations(range(len(w)), 2):
        probs[(a, b_)] = w[a] / W * w[b_] / (W - w[a]) + w[b_] / W * w[a] / (W - w[b_])
    return probs


def test_gumbel_top_p_is_sampling_without_replacement(orc):
    """FlashHead notes, Module 2: sampling mode draws p clusters without replacement from the
    softmax of the centroid logits.  Pair frequencies of Gumbel-top-2 over c = 6 must follow the
    exact successive-sampling probabilities."""
    s = np.array([[0.3, -0.2, 1.1, 0.0, 0.7, -1.0]])
    tau = 0.9
    n = 30000
    counts = {}
    for step in range(n):
        keys = orc.gumbel_keys(s, tau, seed=77, step=step, stream=0)
        sel, _ = orc.select_topp(keys, 2)
        key = tuple(sel[0].tolist())
        counts[key] = counts.get(key, 0) + 1
    probs = _pair_probs(np.exp(s[0] / tau))
    obs = np.array([counts.get(k, 0) for k in probs])
    exp = np.array([probs[k] * n for k in probs])
    assert stats.chisquare(obs, exp).pvalue > 1e-3


def _exact_token_dist(z, s, C2T, p, tau):
    """Exact token distribution of the two-stage sampler: S ~ successive sampling without
    replacement from softmax(s/τ), then a token from softmax(z/τ) over the tokens of S."""
    c, b = C2T.shape
    w = np.exp(s / tau)
    out = np.zeros(len(z))
    for order in itertools.permutations(range(c), p):
        pr, rem = 1.0, w.sum()
        for k in order:
            pr *= w[k] / rem
            rem -= w[k]
        toks = C2T[list(order)].reshape(-1)
        ez = np.exp(z[toks] / tau)
        out[toks] += pr * ez / ez.sum()
    return out


def test_two_stage_sampling_distribution(orc):
    """Token frequencies of the sampler equal the exact two-stage distribution (Module 2 sampling
    mode followed by Eq. 3 over the candidates); with p = c this is the dense softmax(z/τ)."""
    idx = synth.random_index(v=12, d=8, c=4, seed=3, dtype="f32")
    h = (np.random.default_rng(4).standard_normal((1, 8)) * 1.5).astype(np.float32)
    z = widen(idx.E, "f32") @ widen(h, "f32")[0]
    s = widen(idx.C, "f32") @ widen(h, "f32")[0]
    tau, n = 0.7, 20000
    for p in (2, 4):
        toks = np.array([orc.head(idx, h, p=p, sample=True, tau=tau, seed=5, step=st)["tok"][0]
                         for st in range(n)])
        obs = np.bincount(toks, minlength=12)
        exact = _exact_token_dist(z, s, idx.C2T, p, tau)
        if p == 4:
            soft = np.exp(z / tau) / np.exp(z / tau).sum()
            np.testing.assert_allclose(exact, soft, rtol=1e-12)
        keep = exact * n > 5
        obs_k = np.append(obs[keep], obs[~keep].sum())
        exp_k = np.append(exact[keep] * n, exact[~keep].sum() * n)
        if exp_k[-1] == 0:
            obs_k, exp_k = obs_k[:-1], exp_k[:-1]
        assert stats.chisquare(obs_k, exp_k * obs_k.sum() / exp_k.sum()).pvalue > 1e-3


# ----------------------------------------------------------------------------- Monte Carlo


def test_mc_p_equals_c_is_dense_softmax(orc):
    """With p = c every draw probes every cluster, so each p_i(t) is the dense softmax(z/τ)_t and the
    standard error is zero (FlashHead notes, Eq. 7)."""
    idx = synth.random_index(v=64, d=16, c=8, seed=31, dtype="bf16")
    H = synth.store((np.random.default_rng(1).standard_normal((2, 16)) * 2).astype(np.float32), "bf16")
    targets = np.array([[0, 5, 17, 63], [1, 2, 3, 40]], np.int32)
    tau = 0.9
    out = orc.mc(idx, H, targets, p=8, tau=tau, seed=9, n_draws=50)
    z = widen(H, "bf16") @ widen(idx.E, "bf16").T
    for q in range(2):
        soft = np.exp(z[q] / tau - (z[q] / tau).max())
        soft /= soft.sum()
        np.testing.assert_allclose(out["mean"][q], soft[targets[q]], rtol=1e-12, atol=1e-15)
        assert np.all(out["se"][q] < 1e-15)


def test_mc_converges_to_enumerated_marginal(orc):
    """The estimator's mean matches E_S[p(t|h,S)] computed exactly by enumerating every ordered draw
    of successive sampling without replacement (c = 5, p = 2), within 4.5 standard errors."""
    idx = synth.random_index(v=15, d=8, c=5, seed=44, dtype="f32")
    h = (np.random.default_rng(8).standard_normal((1, 8)) * 2).astype(np.float32)
    tau = 0.8
    z = widen(idx.E, "f32") @ widen(h, "f32")[0]
    s = widen(idx.C, "f32") @ widen(h, "f32")[0]
    w = np.exp(s / tau)
    exact = np.zeros(15)
    for order in itertools.permutations(range(5), 2):
        pr = w[order[0]] / w.sum() * w[order[1]] / (w.sum() - w[order[0]])
        toks = idx.C2T[list(order)].reshape(-1)
        ez = np.exp(z[toks] / tau)
        exact[toks] += pr * ez / ez.sum()
    targets = np.arange(15, dtype=np.int32)[None, :]
    out = orc.mc(idx, h, targets, p=2, tau=tau, seed=1234, n_draws=20000)
    err = np.abs(out["mean"][0] - exact)
    assert np.all(err <= 4.5 * out["se"][0] + 1e-12), (err, out["se"][0])
    assert abs(exact.sum() - 1.0) < 1e-12


# ----------------------------------------------------------------------------- cost model


def test_cost_model_matches_printed_head_sizes():
    """The pages print the Llama-3.2-1B head as 263M parameters and the FlashHead head as 33M active
    parameters (-87.4%); the roofline's work model must reproduce them."""
    from clustered_retrieval_classification_b200 import costmodel
    kv = {}
    for line in open(os.path.join(GOLDEN, "flashhead_head_sizes.txt")):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            kv[k] = float(v)
    v, d, c, p = int(kv["v"]), int(kv["d"]), int(kv["c"]), int(kv["p"])
    assert v % c == 0
    b = v // c
    dense = costmodel.dense_params(v, d)
    active = costmodel.active_params(c, d, p, b)
    assert round(dense / 1e6) == kv["dense_head_params_millions"]
    assert round(active / 1e6) == kv["active_head_params_millions"]
    assert round(100 * (1 - active / dense), 1) == kv["param_reduction_percent"]
