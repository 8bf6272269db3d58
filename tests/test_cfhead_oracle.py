"""Pins of the coarse-fine head's oracle (oracle/cfhead_oracle.py) against what the definitions fix,
none of them a retyping of its formulas:

* packing: a hand-packed word decodes to the codes it was built from (nibble order), and the
  generator's packing round-trips;
* exact codebooks: when every tile sub-row of E is one of its tile's codebook entries, the coarse
  score of every token is its exact logit E[u]·h (a numpy matmul of the widened values);
* the coarse score equals the logit of the dequantised row (the concatenated codebook entries of
  the token's codes), a matmul that shares nothing with the look-up-table gather;
* k = v: the candidates are the whole vocabulary, so the head is the dense head (greedy arg-max and
  the same Gumbel-max sample, by the FlashHead oracle's dense routine);
* brute force on a tiny head: pure-Python loops over every token, sorted() for the top-k;
* a planted mistake in the nibble order, the tile width or the sign of the look-up table fails one
  of the above (checked on the oracle's own functions with the mistake put in)."""

import numpy as np
import pytest

import oracle
from clustered_retrieval_classification_b200 import synth
from oracle import cfhead_oracle as CF


def _tiny(v=48, d=32, w=4, K=5, seed=3):
    rng = np.random.default_rng(seed)
    T = d // w
    cb = rng.standard_normal((T, K, w)).astype(np.float32)
    codes = rng.integers(0, K, size=(v, T))
    E = synth.store(rng.standard_normal((v, d)).astype(np.float32) / np.sqrt(d), "bf16")
    H = synth.store(rng.standard_normal((3, d)).astype(np.float32), "bf16")
    return E, cb, codes, H


def test_packing_nibble_order_and_round_trip():
    codes = np.zeros((2, 16), dtype=np.int64)
    codes[0, :8] = [1, 2, 3, 4, 5, 6, 7, 8]
    codes[1, 8:] = [15, 0, 0, 0, 0, 0, 0, 9]
    words = synth.cf_pack_codes(codes)
    assert words.shape == (2, 2) and words.dtype == np.uint32
    assert words[0, 0] == 0x87654321 and words[1, 1] == 0x9000000F and words[1, 0] == 0 and words[0, 1] == 0
    rng = np.random.default_rng(1)
    big = rng.integers(0, 16, size=(37, 24))
    assert np.array_equal(CF.unpack_codes(synth.cf_pack_codes(big)), big)


def test_exact_codebooks_give_exact_logits():
    rng = np.random.default_rng(5)
    v, d, w, K = 200, 64, 8, 16
    T = d // w
    cb = synth.stored_to_f64(synth.store(rng.standard_normal((T, K, w)).astype(np.float32), "bf16"),
                             "bf16").astype(np.float32)
    codes = rng.integers(0, K, size=(v, T))
    rows = cb[np.arange(T)[None, :], codes].reshape(v, d)          # each sub-row is a codebook entry
    E = synth.store(rows, "bf16")                                   # exact: the entries are BF16 values
    H = synth.store(rng.standard_normal((4, d)).astype(np.float32), "bf16")
    s = CF.coarse_scores(cb, synth.cf_pack_codes(codes), H)
    z = synth.stored_to_f64(H, "bf16") @ synth.stored_to_f64(E, "bf16").T
    assert np.abs(s - z).max() <= 1e-12


def test_coarse_score_is_the_logit_of_the_dequantised_row():
    E, cb, codes, H = _tiny(v=300, d=64, w=8, K=16)
    T, K, w = cb.shape
    deq = cb.astype(np.float64)[np.arange(T)[None, :], codes].reshape(codes.shape[0], T * w)
    s = CF.coarse_scores(cb, synth.cf_pack_codes(codes), H)
    assert np.abs(s - synth.stored_to_f64(H, "bf16") @ deq.T).max() <= 1e-12


@pytest.mark.parametrize("sample", [False, True])
def test_k_equals_v_is_the_dense_head(sample):
    cfg = synth.scaled(synth.CONFIGS["llama"], v=2048, c=128, d=64, p=8, name="cf-pin")
    idx = synth.make_index(cfg)
    cb, words = synth.cf_index(idx.E, "bf16")
    H = synth.make_queries(cfg, 3)
    o = CF.head(idx.E, "bf16", cb, words, H, cfg.v, sample=sample, tau=0.8, seed=9, step=4)
    d = oracle.dense(idx, H, sample=sample, tau=0.8, seed=9, step=4)
    assert np.array_equal(o["tok"], d["tok"])
    assert np.all(o["cand"] == np.arange(cfg.v)[None, :])


def test_brute_force_tiny_head():
    E, cb, codes, H = _tiny()
    v, T = codes.shape
    w = cb.shape[2]
    Ef = synth.stored_to_f64(E, "bf16")
    Hf = synth.stored_to_f64(H, "bf16")
    k = 7
    o = CF.head(E, "bf16", cb, synth.cf_pack_codes(codes), H, k)
    for q in range(H.shape[0]):
        coarse = []
        for u in range(v):
            acc = 0.0
            for t in range(T):
                for i in range(w):
                    acc += float(cb[t, codes[u, t], i]) * Hf[q, t * w + i]
            coarse.append((acc, u))
        top = sorted(coarse, key=lambda x: (-x[0], x[1]))[:k]
        cand = sorted(u for _, u in top)
        assert list(o["cand"][q]) == cand
        best = max(cand, key=lambda u: (sum(Ef[u, j] * Hf[q, j] for j in range(Ef.shape[1])), -u))
        assert o["tok"][q] == best


def test_planted_mistakes_are_caught(monkeypatch):
    E, cb, codes, H = _tiny(v=120, d=64, w=8, K=16, seed=11)
    words = synth.cf_pack_codes(codes)
    T = cb.shape[0]
    deq = cb.astype(np.float64)[np.arange(T)[None, :], codes].reshape(codes.shape[0], -1)
    want = synth.stored_to_f64(H, "bf16") @ deq.T

    def reversed_nibbles(words):
        w64 = np.asarray(words, dtype=np.uint64)
        G, v = w64.shape
        out = np.empty((v, 8 * G), dtype=np.int64)
        for g in range(G):
            for j in range(8):
                out[:, 8 * g + j] = (w64[g] >> np.uint64(4 * (7 - j))) & np.uint64(0xF)
        return out

    good = CF.unpack_codes
    monkeypatch.setattr(CF, "unpack_codes", reversed_nibbles)
    assert np.abs(CF.coarse_scores(cb, words, H) - want).max() > 1e-3
    monkeypatch.setattr(CF, "unpack_codes", good)
    good_lut = CF.lut
    monkeypatch.setattr(CF, "lut", lambda cbk, h: -good_lut(cbk, h))
    assert np.abs(CF.coarse_scores(cb, words, H) - want).max() > 1e-3

    def shifted_tiles(cbk, h):                     # every tile reads its columns one place late
        c64 = np.asarray(cbk, dtype=np.float32).astype(np.float64)
        Tn, Kn, wn = c64.shape
        hp = np.concatenate([h[1:], h[:1]])
        return np.stack([c64[t] @ hp[t * wn:(t + 1) * wn] for t in range(Tn)])

    monkeypatch.setattr(CF, "lut", shifted_tiles)
    assert np.abs(CF.coarse_scores(cb, words, H) - want).max() > 1e-3
    monkeypatch.setattr(CF, "lut", good_lut)
    assert np.abs(CF.coarse_scores(cb, words, H) - want).max() <= 1e-12
