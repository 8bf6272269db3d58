"""Parity of the tensor-core (tcgen05) path with the fp64 oracle.

Batches of 2..64 queries on a BF16 index take the tensor-core kernel for the dense head; FlashHead
takes it for its Stage-1 keys from 12 queries on and for its Stage 2 above 16 queries (below, the
union of the probe sets is streamed on the CUDA cores) when no per-candidate outputs are requested.  Sizes span several 128-row tiles with a
ragged tail (v = 32064), batches that are not a multiple of the 16-query MMA width, and a d that is
not a multiple of the 64-element K-block.  Logits are compared element by element (|Δ| <= 2e-3);
token ids must be identical wherever the oracle's margins decide them (parity.MARGIN)."""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth
from parity import LOGIT_TOL, MARGIN

pytestmark = pytest.mark.gpu

DEV = "cuda"
MID = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="llama-mid")


def dev(a, kind):
    from clustered_retrieval_classification_b200 import flashhead as F
    return F.device_array(a, kind, DEV)


@pytest.fixture(scope="module")
def mid():
    return synth.make_index(MID), synth.make_queries(MID, 64)


@pytest.fixture(scope="module")
def mid_index(fh, mid):
    idx, _ = mid
    return fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")


@pytest.mark.parametrize("B", [2, 16, 17, 64])
@pytest.mark.parametrize("sample", [False, True])
def test_dense_batched(fh, orc, mid, mid_index, B, sample):
    idx, H = mid
    cfg = idx.cfg
    logits = torch.empty((B, cfg.v), dtype=torch.float32, device=DEV)
    tok = fh.dense_head(mid_index, dev(H[:B], "bf16"), sample=sample, tau=0.8, seed=7, step=B,
                        logits=logits).cpu().numpy()
    o = orc.dense(idx, H[:B], sample=sample, tau=0.8, seed=7, step=B, want_z=True)
    assert np.abs(logits.cpu().numpy() - o["z"]).max() <= LOGIT_TOL
    decided = o["tok_margin"] > MARGIN
    assert np.array_equal(tok[decided], o["tok"][decided])
    assert decided.sum() >= B // 2


def test_dense_d_not_multiple_of_k_block(fh, orc):
    """d = 200: the last 64-wide K-block runs past the row and must read zeros."""
    idx = synth.random_index(v=1000, d=200, c=50, seed=23, dtype="bf16")
    rng = np.random.default_rng(5)
    H = synth.store((rng.standard_normal((5, 200)) * 2).astype(np.float32), "bf16")
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    logits = torch.empty((5, 1000), dtype=torch.float32, device=DEV)
    tok = fh.dense_head(I, dev(H, "bf16"), logits=logits).cpu().numpy()
    o = orc.dense(idx, H, want_z=True)
    assert np.abs(logits.cpu().numpy() - o["z"]).max() <= LOGIT_TOL
    decided = o["tok_margin"] > MARGIN
    assert np.array_equal(tok[decided], o["tok"][decided])


SMALL = synth.scaled(synth.CONFIGS["llama"], v=16384, c=512, d=256, p=16, name="llama-small")


@pytest.fixture(scope="module")
def small(fh):
    idx = synth.make_index(SMALL)
    return idx, synth.make_queries(SMALL, 64), fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")


@pytest.mark.parametrize("B", [4, 8, 12, 16, 33, 64])
@pytest.mark.parametrize("sample", [False, True])
def test_flashhead_batched_without_debug(fh, orc, small, B, sample):
    """Tokens equal the oracle's wherever its set and token margins decide them; every other token
    comes from a cluster the oracle selected or one within the margin of its threshold.  B = 4 … 16
    stream the union of the probe sets on the CUDA cores (tensor-core Stage-1 keys from 12 on),
    B = 33 and 64 stream the tensor-core tiles that hold a selected cluster."""
    idx, H, I = small
    cfg = idx.cfg
    Hd = dev(H[:B], "bf16")
    if sample:
        tok = fh.head_sample(I, Hd, cfg.p, 0.8, synth.SAMPLE_SEED, 5).cpu().numpy()
    else:
        tok = fh.head_greedy(I, Hd, cfg.p).cpu().numpy()
    o = orc.head(idx, H[:B], cfg.p, sample=sample, tau=0.8, seed=synth.SAMPLE_SEED, step=5)
    decided = (o["set_margin"] > MARGIN) & (o["tok_margin"] > MARGIN)
    assert np.array_equal(tok[decided], o["tok"][decided]), np.nonzero(tok != o["tok"])
    assert decided.sum() >= max(1, B // 4)
    s = orc.stage1_scores(idx.C, cfg.dtype, H[:B], cfg.c, cfg.d)
    keys = orc.gumbel_keys(s, 0.8, synth.SAMPLE_SEED, 5, 0) if sample else s
    for q in range(B):
        k = np.sort(keys[q])[::-1]
        thr = 0.5 * (k[cfg.p - 1] + k[cfg.p])
        allowed = set(np.asarray(o["sel"][q]).tolist()) | set(np.nonzero(np.abs(keys[q] - thr) <= MARGIN)[0].tolist())
        assert any(int(tok[q]) in idx.C2T[cl] for cl in allowed), q


def test_flashhead_batched_matches_cuda_core_path(fh, mid, mid_index):
    """The tensor-core Stage 2 (no debug outputs, 40 queries) and the per-query CUDA-core Stage 2
    (taken when debug outputs are requested) select the same sets and agree on every token whose
    logit margin exceeds the fp32 accumulation-order difference."""
    idx, H = mid
    cfg = idx.cfg
    B = 40
    Hd = dev(H[:B], "bf16")
    tc = fh.head_greedy(mid_index, Hd, cfg.p).cpu().numpy()
    P = cfg.p * cfg.b
    dbg = dict(sel=torch.empty((B, cfg.p), dtype=torch.int32, device=DEV),
               cand_tok=torch.empty((B, P), dtype=torch.int32, device=DEV),
               cand_logit=torch.empty((B, P), dtype=torch.float32, device=DEV))
    cc = fh.head_greedy(mid_index, Hd, cfg.p, debug=dbg).cpu().numpy()
    z = dbg["cand_logit"].cpu().numpy()
    zs = np.sort(z, axis=1)
    gap = zs[:, -1] - zs[:, -2]
    close = gap <= 1e-4
    assert np.array_equal(tc[~close], cc[~close])


def test_workspace_reuse_across_batch_sizes(fh, orc, mid, mid_index):
    """One workspace, consecutive tensor-core calls with different batch sizes and grids."""
    idx, H = mid
    cfg = idx.cfg
    ws = mid_index.workspace(fh.FH_OP_DENSE, 64)
    for B in (16, 3, 64, 2):
        tok = fh.dense_head(mid_index, dev(H[:B], "bf16"), ws=ws).cpu().numpy()
        o = orc.dense(idx, H[:B])
        decided = o["tok_margin"] > MARGIN
        assert np.array_equal(tok[decided], o["tok"][decided])
    fh.ws_status(ws)


STRADDLE = synth.scaled(synth.CONFIGS["llama"], v=12000, c=500, d=256, p=40, name="llama-b24")


@pytest.mark.parametrize("B", [20, 33])
@pytest.mark.parametrize("sample", [False, True])
def test_flashhead_batched_clusters_straddle_tiles(fh, orc, B, sample):
    """b = 24 rows a cluster: clusters straddle the 128-row tiles of the cluster-major copy, so the
    tile list must hold every tile a selected cluster overlaps (the last tile is partial, v = 12000);
    the tensor-core Stage 2 against the oracle."""
    idx = synth.make_index(STRADDLE)
    H = synth.make_queries(STRADDLE, B)
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    cfg = idx.cfg
    Hd = dev(H, "bf16")
    if sample:
        tok = fh.head_sample(I, Hd, cfg.p, 0.8, synth.SAMPLE_SEED, 7).cpu().numpy()
    else:
        tok = fh.head_greedy(I, Hd, cfg.p).cpu().numpy()
    o = orc.head(idx, H, cfg.p, sample=sample, tau=0.8, seed=synth.SAMPLE_SEED, step=7)
    decided = (o["set_margin"] > MARGIN) & (o["tok_margin"] > MARGIN)
    assert np.array_equal(tok[decided], o["tok"][decided]), np.nonzero(tok != o["tok"])
    assert decided.sum() >= max(1, B // 4)
    # every token is a candidate of its query: from a cluster the oracle selected, or one within the
    # margin of the threshold
    s = orc.stage1_scores(idx.C, cfg.dtype, H, cfg.c, cfg.d)
    keys = orc.gumbel_keys(s, 0.8, synth.SAMPLE_SEED, 7, 0) if sample else s
    for q in range(B):
        k = np.sort(keys[q])[::-1]
        thr = 0.5 * (k[cfg.p - 1] + k[cfg.p])
        allowed = set(np.asarray(o["sel"][q]).tolist()) | set(np.nonzero(np.abs(keys[q] - thr) <= MARGIN)[0].tolist())
        assert any(int(tok[q]) in idx.C2T[cl] for cl in allowed), q


@pytest.mark.parametrize("d", [200, 320])
@pytest.mark.parametrize("B", [2, 40])
def test_stage1_keys_partial_stage(fh, orc, d, B):
    """Tensor-core Stage-1 keys stream several consecutive K-blocks per pipeline stage; d = 320 (five
    64-column K-blocks: a stage of four, then one of one) and d = 200 (a partial last K-block) check
    the partial stages element by element."""
    idx = synth.random_index(v=4000, d=d, c=500, seed=41, dtype="bf16")
    rng = np.random.default_rng(43)
    H = synth.store((rng.standard_normal((B, d)) * 0.5).astype(np.float32), "bf16")
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    g = fh.stage1_scores(I, dev(H, "bf16")).cpu().numpy()
    o = orc.stage1_scores(idx.C, "bf16", H, idx.c, d)
    assert np.abs(g - o).max() <= LOGIT_TOL
