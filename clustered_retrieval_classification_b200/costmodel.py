"""Algorithmic work of one head call: the element, byte and flop counts the roofline divides by.

FlashHead replaces the O(v·d) dense head by O(c·d + p·b·d) work per query, b = v/c
(FlashHead notes, Eq. 6): Stage 1 reads the c centroids once, Stage 2 reads the p·b candidate rows.
For a batch the candidate rows of clusters chosen by several queries need to be read once, so the
Stage-2 byte count uses the number of distinct clusters probed by the batch (U).
"""

from __future__ import annotations


def active_params(c: int, d: int, p: int, b: int) -> int:
    """Head weights touched per query: c·d centroid entries plus p·b·d candidate-row entries."""
    return c * d + p * b * d


def dense_params(v: int, d: int) -> int:
    return v * d


def stage1_bytes(c: int, d: int, elem_bytes: int, int4: bool = False) -> int:
    """Centroid bytes: BF16/fp32 rows, or INT4 nibbles plus one BF16 scale per 32 columns."""
    if int4:
        return c * d // 2 + c * (d // 32) * 2
    return c * d * elem_bytes


def head_bytes(v: int, d: int, c: int, p: int, B: int, unique_clusters: int, elem_bytes: int,
               int4: bool = False) -> int:
    """Bytes one fused head call must move: centroids once, the U distinct probed clusters' rows
    once, the C2T entries of every query's candidates, the B hidden vectors and the B token ids."""
    b = v // c
    return (stage1_bytes(c, d, elem_bytes, int4)
            + unique_clusters * b * d * elem_bytes
            + B * p * b * 4
            + B * d * elem_bytes
            + B * 4)


def dense_bytes(v: int, d: int, B: int, elem_bytes: int) -> int:
    """Dense head: every row of E once, plus the hidden vectors and the token ids."""
    return v * d * elem_bytes + B * d * elem_bytes + B * 4


def head_flops(d: int, c: int, p: int, b: int, B: int) -> int:
    """Multiply-adds ×2 of the method proper: B·(c + p·b)·d."""
    return 2 * B * (c + p * b) * d


def cf_bytes(v: int, d: int, w: int, K: int, k: int, B: int, unique_candidates: int) -> int:
    """Coarse-fine head (page "Fast LM Head via Coarse-Fine Decomposition and Tile-Wise Weight
    Clustering"): the 4-bit index map once (d/w codes per token, half a byte each), the fp32
    codebooks once, the E rows of the distinct candidates of the batch once (BF16), the B hidden
    vectors and the B token ids."""
    T = d // w
    return v * T // 2 + T * K * w * 4 + unique_candidates * d * 2 + B * d * 2 + B * 4
