"""The coarse-fine head (include/fh_cfhead.h) against its fp64 oracle (oracle/cfhead_oracle.py).

Page "Fast LM Head via Coarse-Fine Decomposition and Tile-Wise Weight Clustering", abstract: coarse
scores over the whole vocabulary from per-tile look-up tables and the streamed index map, then exact
logits on the top-k candidates.  Rules (parity.py): coarse scores and logits within 2e-3; the
candidate set identical unless the oracle's k-th-score margin is within 4e-3 (then the tokens that
differ lie within 4e-3 of the threshold); tokens identical where the sets agree and the top-1 margin
exceeds 4e-3, otherwise a near-maximum over the GPU's candidates."""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth
from oracle import cfhead_oracle as CF
from parity import LOGIT_TOL, MARGIN, check_sets, check_tokens

pytestmark = pytest.mark.gpu

MID = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="cf-mid")


@pytest.fixture(scope="module")
def mid(fh):
    idx = synth.make_index(MID)
    cb, words = synth.cf_index(idx.E, "bf16")
    I = fh.cf_index_from_host(idx.E, cb, words)
    return idx, cb, words, I, synth.make_queries(MID, 16)


def _check(fh, orc, idx, cb, words, I, H, k, sample=False, tau=0.8, seed=3, step=5):
    B = H.shape[0]
    Hd = fh.device_array(H, "bf16")
    cand = torch.empty((B, k), dtype=torch.int32, device="cuda")
    coarse = torch.empty((B, idx.cfg.v), dtype=torch.float32, device="cuda")
    tok = fh.cf_head(I, Hd, k, sample=sample, tau=tau, seed=seed, step=step,
                     debug=dict(cand=cand, coarse=coarse)).cpu().numpy()
    torch.cuda.synchronize()
    o = CF.head(idx.E, "bf16", cb, words, H, k, sample=sample, tau=tau, seed=seed, step=step)
    assert np.abs(coarse.cpu().numpy() - o["coarse"]).max() <= LOGIT_TOL
    gsel = np.sort(cand.cpu().numpy(), axis=1)
    check_sets(gsel, o["cand"], o["coarse"], o["set_margin"])
    same = [np.array_equal(gsel[q], o["cand"][q]) for q in range(B)]

    def valid(q, t):
        z = orc.logits(idx.E, "bf16", H[q:q + 1], gsel[q:q + 1])[0]
        if sample:
            z = z / tau + np.array([orc.gumbel(orc.draw_u32(seed, step, q, 1, int(u))) for u in gsel[q]])
        return z.max(), z[list(gsel[q]).index(t)]

    check_tokens(tok, o["tok"], o["tok_margin"], same, valid)
    decided = np.array([same[q] and o["tok_margin"][q] > MARGIN for q in range(B)])
    return tok, o, decided


def test_coarse_scores_element_by_element(fh, mid):
    idx, cb, words, I, H = mid
    g = fh.cf_coarse_scores(I, fh.device_array(H[:3], "bf16")).cpu().numpy()
    assert np.abs(g - CF.coarse_scores(cb, words, H[:3])).max() <= LOGIT_TOL


@pytest.mark.parametrize("B,k", [(1, 256), (3, 256), (16, 64), (2, 1), (1, 4097)])
def test_greedy_mid(fh, orc, mid, B, k):
    idx, cb, words, I, H = mid
    _, _, dec = _check(fh, orc, idx, cb, words, I, H[:B], k)
    if k > 1:
        assert dec.sum() >= max(1, B // 2)


def test_sampling_mid(fh, orc, mid):
    idx, cb, words, I, H = mid
    _check(fh, orc, idx, cb, words, I, H[:4], 256, sample=True)


def test_k_equals_v_is_the_dense_head(fh, mid):
    idx, cb, words, I, H = mid
    Hd = fh.device_array(H[:3], "bf16")
    FI = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16", cluster_major=False)
    assert np.array_equal(fh.cf_head(I, Hd, idx.cfg.v).cpu().numpy(), fh.dense_head(FI, Hd).cpu().numpy())
    s = fh.cf_head(I, Hd, idx.cfg.v, sample=True, tau=0.8, seed=4, step=9).cpu().numpy()
    ds = fh.dense_head(FI, Hd, sample=True, tau=0.8, seed=4, step=9).cpu().numpy()
    assert np.array_equal(s, ds)


def test_all_equal_coarse_scores_take_the_lowest_ids(fh, orc, mid):
    """Every token gets the same codes, so every coarse score is equal: the k candidates are the k
    smallest token ids (the tie rule), found by the exact id passes of the boundary ranking."""
    idx, cb, words, I, H = mid
    zero = np.zeros_like(words)
    J = fh.cf_index_from_host(idx.E, cb, zero)
    k = 300
    cand = torch.empty((2, k), dtype=torch.int32, device="cuda")
    tok = fh.cf_head(J, fh.device_array(H[:2], "bf16"), k, debug=dict(cand=cand)).cpu().numpy()
    assert np.array_equal(np.sort(cand.cpu().numpy(), axis=1), np.tile(np.arange(k), (2, 1)))
    o = CF.head(idx.E, "bf16", cb, zero, H[:2], k)
    decided = o["tok_margin"] > MARGIN
    assert np.array_equal(tok[decided], o["tok"][decided])


def test_consecutive_calls_reuse_one_workspace(fh, mid):
    idx, cb, words, I, H = mid
    ws = torch.zeros(I.workspace_bytes(4, 256), dtype=torch.uint8, device="cuda")
    Hd = fh.device_array(H[:4], "bf16")
    ref = [fh.cf_head(I, Hd[q:q + 1], 256).item() for q in range(4)]
    for _ in range(2):
        got = [fh.cf_head(I, Hd[q:q + 1], 256, ws=ws).item() for q in range(4)]
        assert got == ref
    assert fh.cf_head(I, Hd, 256, ws=ws).cpu().numpy().tolist() == ref
    fh.ws_status(ws)


def test_llama_full_size(fh, orc, llama_host):
    """The Llama-3.2-1B-shaped vocabulary (v=128256, d=2048: 256 tiles of 8 columns, 16 codes each)
    with k = 1024 candidates, two queries greedy and one sampled."""
    idx, H = llama_host
    cb, words = synth.cf_index(idx.E, "bf16")
    I = fh.cf_index_from_host(idx.E, cb, words)
    _, _, dec = _check(fh, orc, idx, cb, words, I, H[:2], synth.CF_TOPK)
    _check(fh, orc, idx, cb, words, I, H[2:3], synth.CF_TOPK, sample=True)
    assert dec.sum() >= 1
