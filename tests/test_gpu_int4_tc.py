"""INT4 Stage 1 on the tensor cores (FlashHead notes, Module 3) against the fp64 oracle.

From 2 queries on, INT4 centroid scores are computed by a kernel that dequantises the nibbles and
their BF16 group scales to fp16 in shared memory (q·scale is exact in fp16), converts the queries
from BF16 to fp16 and contracts them with fp16 MMAs accumulating in FP32.  Shapes here cover a
ragged last tile of centroid rows (c % 128 != 0), a half K-block (d % 64 == 32), scales whose tile
does not end on a 16-byte boundary, partial 16-query blocks and the 64-query maximum; the keys are
compared element by element (2e-3, the logit tolerance), the Gumbel keys of the sampling mode too,
and whole greedy and sampling heads through the INT4 path."""

import numpy as np
import pytest

from clustered_retrieval_classification_b200 import synth
from headcheck import check_head, dev, load
from parity import LOGIT_TOL

pytestmark = pytest.mark.gpu

# c = 2004 centroid rows (15 full tiles and one of 84 rows), d = 1120 (35 scale groups: 17 full
# K-blocks of 64 columns and one of 32; 70 scale bytes per row, so the last tile's scales end 8 bytes
# past a 16-byte boundary)
RAGGED = synth.dataclasses.replace(synth.scaled(synth.CONFIGS["gemma"], v=32064, c=2004, d=1120, p=96),
                                   name="gemma-ragged")


@pytest.fixture(scope="module")
def ragged():
    return synth.make_index(RAGGED), synth.make_queries(RAGGED, 64)


@pytest.fixture(scope="module")
def ragged_index(fh, ragged):
    idx, _ = ragged
    return load(fh, idx, int4=True)


def _oracle_scores(orc, idx, H):
    return orc.stage1_scores(None, "bf16", H, idx.c, idx.d, q4=idx.C_q4, scales=idx.C_scales)


@pytest.mark.parametrize("B", [2, 5, 16, 17, 64])
def test_int4_scores_element_by_element(fh, orc, ragged, ragged_index, B):
    idx, H = ragged
    g = fh.stage1_scores(ragged_index, dev(H[:B], "bf16")).cpu().numpy()
    o = _oracle_scores(orc, idx, H[:B])
    assert g.shape == o.shape
    assert np.abs(g - o).max() <= LOGIT_TOL


def test_int4_scores_do_not_depend_on_the_batch(fh, ragged, ragged_index):
    """Row q of a 64-query call equals the same query's row in a 4-query call: each accumulator is
    one query's own dot product, whatever else shares the MMA."""
    _, H = ragged
    g64 = fh.stage1_scores(ragged_index, dev(H[:64], "bf16")).cpu().numpy()
    for q0 in (0, 20, 60):
        g4 = fh.stage1_scores(ragged_index, dev(H[q0:q0 + 4], "bf16")).cpu().numpy()
        assert np.array_equal(g4, g64[q0:q0 + 4])


@pytest.mark.parametrize("B", [8, 17])
def test_int4_greedy_head(fh, orc, ragged, ragged_index, B):
    idx, H = ragged
    check_head(fh, orc, idx, H, idx.cfg.p, batch=B, int4=True, debug="sel", I=ragged_index)


def test_int4_sampling_head(fh, orc, ragged, ragged_index):
    """The sampling keys s/τ + G (stream FH_RNG_STAGE1, elem = cluster id) from the MMA epilogue."""
    idx, H = ragged
    check_head(fh, orc, idx, H, idx.cfg.p, sample=True, tau=0.7, seed=11, step=3, batch=9, int4=True,
               debug="sel", I=ragged_index)


@pytest.mark.parametrize("B", [16, 64])
def test_gemma_int4_scores_full_size(fh, orc, gemma_host, B):
    """The Gemma-3-1B-shaped centroids (c=16384, d=1152: 128 tiles of 128 rows, 18 K-blocks)."""
    idx, H = gemma_host
    I = load(fh, idx, int4=True)
    Hq = np.concatenate([H] * (B // len(H) + 1))[:B]
    g = fh.stage1_scores(I, dev(Hq, "bf16")).cpu().numpy()
    o = _oracle_scores(orc, idx, Hq)
    assert np.abs(g - o).max() <= LOGIT_TOL
