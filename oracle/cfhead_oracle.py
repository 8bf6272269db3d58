"""CPU oracle of the coarse-fine head — TEST INFRASTRUCTURE ONLY.

Plain float64 numpy restatement of the coarse-fine LM head of the page "Fast LM Head via Coarse-Fine
Decomposition and Tile-Wise Weight Clustering" (abstract): the head weights E are represented by a
per-tile codebook and an index map built offline by tile-wise k-means; at decode time coarse scores
over the whole vocabulary come from per-tile look-up tables and the streamed indices, and the exact
product with the original weights runs only on the top-k candidates.  Only tests/, the smoke check
and the benchmark's CPU-baseline leg import this module; it imports nothing from the product
package.

Readings (the abstract fixes no parameter, layout or tie rule):
  * tiles are w consecutive columns of E, T = d / w of them; tile t has its own codebook of K entries
    Cb[t] ∈ R^{K×w} (float32 values), and token u's index map row holds one code I[u, t] < K per tile;
  * the look-up table of a query h is LUT[t, j] = Cb[t, j]·h[t·w : (t+1)·w];
  * the coarse score of token u is ŝ_u = Σ_t LUT[t, I[u, t]];
  * the candidates are the k tokens with the largest coarse scores, ordered (score desc, id asc);
  * their exact logits are z_u = E[u]·h, and the token is the arg-max of z (greedy) or of
    z/τ + G(seed, step, q, 1, u) (sampling: a softmax(z/τ) draw over the candidates by Gumbel-max,
    with the Stage-2 Philox stream of the FlashHead calls), ties by the smaller token id;
  * the index map is stored as 4-bit codes packed eight tiles to a 32-bit word: word (g, u) of a
    [T/8, v] array holds tile 8g + j of token u in bits 4j..4j+3.
Every step is computed here as written, in float64 on the exactly widened stored values; the top-k
uses the FlashHead oracle's full-sort selection and its Philox stream (both pinned separately).
"""

from __future__ import annotations

import numpy as np

from . import _c, draw_u32, gumbel, logits, select_topp

BF16_OR_F32 = ("bf16", "f32")


def _widen(a, dtype):
    a = np.ascontiguousarray(a)
    if dtype == "f32":
        return a.astype(np.float32).astype(np.float64)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def unpack_codes(words: np.ndarray) -> np.ndarray:
    """[T/8, v] packed words -> (v, T) integer codes (tile 8g + j in bits 4j..4j+3 of word (g, u))."""
    words = np.asarray(words, dtype=np.uint64)
    G, v = words.shape
    codes = np.empty((v, 8 * G), dtype=np.int64)
    for g in range(G):
        for j in range(8):
            codes[:, 8 * g + j] = (words[g] >> np.uint64(4 * j)) & np.uint64(0xF)
    return codes


def lut(codebooks: np.ndarray, h: np.ndarray) -> np.ndarray:
    """LUT[t, j] = Cb[t, j]·h_t for one query h (float64 [d]); returns float64 [T, K]."""
    cb = np.asarray(codebooks, dtype=np.float32).astype(np.float64)
    T, K, w = cb.shape
    out = np.empty((T, K))
    for t in range(T):
        out[t] = cb[t] @ h[t * w:(t + 1) * w]
    return out


def coarse_scores(codebooks, words, H, dtype="bf16") -> np.ndarray:
    """ŝ[q, u] = Σ_t LUT_q[t, I[u, t]] for every query row of H; float64 [B, v]."""
    Hf = _widen(H, dtype)
    codes = unpack_codes(words)
    v, T = codes.shape
    out = np.empty((Hf.shape[0], v))
    cols = np.arange(T)[None, :]
    for q in range(Hf.shape[0]):
        L = lut(codebooks, Hf[q])
        out[q] = L[cols, codes].sum(axis=1)
    return out


def head(E, dtype, codebooks, words, H, k, sample=False, tau=1.0, seed=0, step=0):
    """The coarse-fine head for every query row of H.  Returns a dict of numpy arrays:
    tok [B]; cand [B, k] (ascending ids); z [B, k] exact logits of cand; coarse [B, v];
    set_margin [B] (k-th minus (k+1)-th coarse score); tok_margin [B] (best minus runner-up of the
    decision keys over the candidates)."""
    H = _c(H)
    B = H.shape[0]
    s = coarse_scores(codebooks, words, H, dtype)
    cand, set_margin = select_topp(s, k)
    z = logits(E, dtype, H, cand)
    tok = np.zeros(B, dtype=np.int32)
    tok_margin = np.zeros(B)
    for q in range(B):
        dec = z[q].copy()
        if sample:
            dec = np.array([z[q, i] / tau + gumbel(draw_u32(seed, step, q, 1, int(u)))
                            for i, u in enumerate(cand[q])])
        best = 0
        for i in range(1, k):
            if dec[i] > dec[best] or (dec[i] == dec[best] and cand[q, i] < cand[q, best]):
                best = i
        tok[q] = cand[q, best]
        rest = np.delete(dec, best)
        tok_margin[q] = dec[best] - rest.max() if rest.size else np.inf
    return dict(tok=tok, cand=cand, z=z, coarse=s, set_margin=set_margin, tok_margin=tok_margin)
