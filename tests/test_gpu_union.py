"""Batched Stage 2 over the union of the probe sets (FlashHead notes, Figure 1 Stage 2, for a batch)
against the fp64 oracle.

From 2 to 16 queries, when no per-candidate outputs are asked for, the clusters some query selected
are streamed once and every row is dotted with the queries whose probe set holds its cluster.  Sizes
here: c = 2004 clusters of b = 16 rows (the union's rows do not divide evenly over the blocks),
batches that are not a multiple of 8, the 16-query maximum, p = 1 (a sparse union) and p = c
(every query takes every cluster), identical queries (every cluster mask full), sampling, and a
workspace reused across calls.  Tokens must equal the oracle's wherever its set and token margins
decide them (parity.MARGIN); the probe sets are compared as in every other head test."""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth
from headcheck import check_head, dev, load
from parity import MARGIN

pytestmark = pytest.mark.gpu

MID = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="llama-mid")


@pytest.fixture(scope="module")
def mid():
    return synth.make_index(MID), synth.make_queries(MID, 64)


@pytest.fixture(scope="module")
def mid_index(fh, mid):
    idx, _ = mid
    return load(fh, idx)


@pytest.mark.parametrize("B", [2, 5, 11, 16])
def test_union_greedy(fh, orc, mid, mid_index, B):
    idx, H = mid
    check_head(fh, orc, idx, H, idx.cfg.p, batch=B, debug="sel", I=mid_index)


@pytest.mark.parametrize("B", [3, 16])
def test_union_sampling(fh, orc, mid, mid_index, B):
    idx, H = mid
    check_head(fh, orc, idx, H, idx.cfg.p, sample=True, tau=0.8, seed=synth.SAMPLE_SEED, step=B,
               batch=B, debug="sel", I=mid_index)


@pytest.mark.parametrize("p", [1, 2004])
def test_union_edge_p(fh, orc, mid, mid_index, p):
    """p = 1: a handful of clusters for the whole grid; p = c: every row, every mask full."""
    idx, H = mid
    check_head(fh, orc, idx, H, p, batch=6, debug="sel", I=mid_index)


def test_union_identical_queries(fh, orc, mid, mid_index):
    """Twelve copies of one query: every listed cluster carries all twelve mask bits, and every query
    gets the token of the single query."""
    idx, H = mid
    Hq = np.repeat(H[:1], 12, axis=0)
    tok = fh.head_greedy(mid_index, dev(Hq, "bf16"), idx.cfg.p).cpu().numpy()
    assert (tok == tok[0]).all()
    o = orc.head(idx, H[:1], idx.cfg.p)
    if o["set_margin"][0] > MARGIN and o["tok_margin"][0] > MARGIN:
        assert tok[0] == o["tok"][0]


def test_union_matches_per_query_path(fh, mid, mid_index):
    """The union Stage 2 (no debug outputs) and the per-query Stage 2 (taken when per-candidate outputs
    are requested) select the same sets and agree on every token whose logit margin exceeds the fp32
    accumulation-order difference."""
    idx, H = mid
    cfg = idx.cfg
    B = 14
    Hd = dev(H[:B], "bf16")
    uni = fh.head_greedy(mid_index, Hd, cfg.p).cpu().numpy()
    P = cfg.p * cfg.b
    dbg = dict(sel=torch.empty((B, cfg.p), dtype=torch.int32, device="cuda"),
               cand_tok=torch.empty((B, P), dtype=torch.int32, device="cuda"),
               cand_logit=torch.empty((B, P), dtype=torch.float32, device="cuda"))
    pq = fh.head_greedy(mid_index, Hd, cfg.p, debug=dbg).cpu().numpy()
    zs = np.sort(dbg["cand_logit"].cpu().numpy(), axis=1)
    clear = zs[:, -1] - zs[:, -2] > 1e-4
    assert clear.sum() >= B // 2
    assert np.array_equal(uni[clear], pq[clear])


def test_union_reuses_one_workspace(fh, mid, mid_index):
    """The arg-maxima and the arrival ticket return to zero at the end of every call: repeated calls
    on one workspace give the same tokens, and the status word stays clean."""
    idx, H = mid
    B = 9
    ws = torch.zeros(mid_index.workspace_bytes(fh.FH_OP_GREEDY, B, idx.cfg.p), dtype=torch.uint8,
                     device="cuda")
    Hd = dev(H[:B], "bf16")
    ref = fh.head_greedy(mid_index, Hd, idx.cfg.p, ws=ws).cpu().numpy()
    for _ in range(3):
        assert np.array_equal(fh.head_greedy(mid_index, Hd, idx.cfg.p, ws=ws).cpu().numpy(), ref)
    fh.ws_status(ws)


@pytest.mark.parametrize("dtype,d,B,sample", [
    ("bf16", 3072, 16, False),   # 6 KB rows: read from the ring in place, 8 warps (16 x 6 KB of queries)
    ("bf16", 3072, 16, True),
    ("bf16", 3072, 5, False),    # 12 warps with two slots each beside five query vectors
    ("f32", 1536, 16, False),    # fp32 rows over 4 KB, 8 warps
    ("f32", 768, 12, False),     # fp32 rows held in registers, 16 warps x 3 slots
])
def test_union_row_sizes_and_warp_splits(fh, orc, dtype, d, B, sample):
    """The union kernel's other forms: rows too long to hold in registers (over 4 KB) and the warp
    counts left when the query vectors crowd the ring, in BF16 and fp32 (the pair-wise dot products
    and the early slot refill of register-held rows in fp32 too)."""
    cfg = synth.dataclasses.replace(synth.scaled(synth.CONFIGS["llama"], v=8000, c=500, d=d, p=40,
                                                 name=f"union-{dtype}-d{d}"), dtype=dtype)
    idx = synth.make_index(cfg)
    H = synth.make_queries(cfg, B)
    check_head(fh, orc, idx, H, cfg.p, sample=sample, tau=0.8, seed=synth.SAMPLE_SEED, step=B,
               batch=B, debug="sel")
