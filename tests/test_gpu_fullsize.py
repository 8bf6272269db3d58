"""Parity with the oracle at the full sizes the benchmark runs, in the kernels those sizes select.

* Gemma-3-1B-shaped INT4 Stage 1 (v=262144, d=1152, c=16384, p=1024): batch 1 runs the persistent
  kernel with 512 threads (more than 8192 clusters), batches 8 and 32 the INT4 tensor-core Stage 1
  with the union Stage 2 (8) or the tensor-core Stage 2 (32).
* The crowded boundary bin at c > 8192 (the 512-thread full-selection branch).
* Llama-3.2-1B-shaped batches of 16, 32 and 64 queries (d=2048: 32 K-blocks per tile) on the
  tensor-core Stage 1 with the union Stage 2 (16) or the tensor-core Stage 2 (32, 64), greedy and
  sampling; the tensor-core Stage-1 keys element by element.
* The Qwen-3-0.6B-shaped Monte Carlo marginal (c=9496, p=512), which selects with 20 keys per
  thread, on likely targets (each query's dense top 8) with relative tolerances.

FlashHead notes: Module 2 (greedy and sampling selection), Module 3 (INT4 Stage 1), Module 4 and
Eq. 7 (Monte Carlo)."""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth
from headcheck import check_head, decided, dev, load, run_head
from parity import LOGIT_TOL, check_mc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gemma_index(fh, gemma_host):
    idx, _ = gemma_host
    return load(fh, idx, int4=True)


@pytest.fixture(scope="module")
def llama_index(fh, llama_host):
    idx, _ = llama_host
    return load(fh, idx)


# ----------------------------------------------------------------------------- Gemma INT4


def test_gemma_int4_batch1_full_size(fh, orc, gemma_host, gemma_index):
    idx, H = gemma_host
    n_dec = 0
    for q in range(4):
        check_head(fh, orc, idx, H[q:q + 1], idx.cfg.p, int4=True, I=gemma_index)
    # the decided count: set equal to the oracle's and top-1 margin above 4e-3
    P = idx.cfg.p * idx.cfg.b
    for q in range(4):
        tok, dbg = run_head(fh, gemma_index, dev(H[q:q + 1], "bf16"), idx.cfg.p, False, 1.0, 0, 0, P, 1)
        o = orc.head(idx, H[q:q + 1], idx.cfg.p, use_int4=True)
        d = decided(o, dbg["sel"])
        n_dec += int(d.sum())
        if d[0]:
            assert tok[0] == o["tok"][0]
    assert n_dec >= 2


@pytest.mark.parametrize("B", [8, 32])
def test_gemma_int4_batched_full_size(fh, orc, gemma_host, gemma_index, B):
    idx, H = gemma_host
    check_head(fh, orc, idx, H, idx.cfg.p, batch=B, int4=True, debug="sel", I=gemma_index)


@pytest.mark.parametrize("perturb", [0.0, 1e-3])
def test_crowded_boundary_bin_512_threads(fh, orc, perturb):
    """16384 clusters (the 512-thread persistent kernel) whose centroids are (nearly) one direction:
    far more keys than the distributed selection ranks share the boundary bin."""
    v, d, c = 32768, 64, 16384
    idx = synth.random_index(v=v, d=d, c=c, seed=29, dtype="bf16")
    rng = np.random.default_rng(31)
    base = rng.standard_normal(d)
    rows = base[None, :] + perturb * rng.standard_normal((c, d))
    rows /= np.linalg.norm(rows, axis=1, keepdims=True)
    idx.C = synth.store(rows.astype(np.float32), "bf16")
    H = synth.store((rng.standard_normal((2, d)) * 2).astype(np.float32), "bf16")
    for q in range(2):
        check_head(fh, orc, idx, H[q:q + 1], 1000)


# ----------------------------------------------------------------------------- Llama batches


@pytest.mark.parametrize("B", [2, 16, 64])
def test_llama_stage1_keys_tensor_core(fh, orc, llama_host, llama_index, B):
    idx, H = llama_host
    g = fh.stage1_scores(llama_index, dev(H[:B], "bf16")).cpu().numpy()
    o = orc.stage1_scores(idx.C, "bf16", H[:B], idx.c, idx.d)
    assert np.abs(g - o).max() <= LOGIT_TOL


@pytest.mark.parametrize("B", [16, 32, 64])
def test_llama_batched_greedy(fh, orc, llama_host, llama_index, B):
    idx, H = llama_host
    n_set, n_tok = check_head(fh, orc, idx, H, idx.cfg.p, batch=B, debug="sel", I=llama_index)
    # most queries must be decided (same set as the oracle, top-1 margin > 4e-3)
    P = idx.cfg.p * idx.cfg.b
    tok, dbg = run_head(fh, llama_index, dev(H[:B], "bf16"), idx.cfg.p, False, 1.0, 0, 0, P, B, "sel")
    o = orc.head(idx, H[:B], idx.cfg.p)
    d = decided(o, dbg["sel"])
    assert d.sum() >= B // 2, d.sum()
    assert np.array_equal(tok[d], o["tok"][d])


@pytest.mark.parametrize("B", [16, 32, 64])
def test_llama_batched_sampling(fh, orc, llama_host, llama_index, B):
    idx, H = llama_host
    check_head(fh, orc, idx, H, idx.cfg.p, batch=B, sample=True, tau=0.8, seed=synth.SAMPLE_SEED,
               step=B, debug="sel", I=llama_index)


def test_llama_batch_tokens_match_batch1(fh, llama_host, llama_index):
    """The union Stage 2 of a 16-query batch and the persistent batch-1 kernel sum the same logits
    in different orders; their tokens agree wherever fp32 rounding cannot decide between two
    candidates."""
    idx, H = llama_host
    Hd = dev(H[:16], "bf16")
    tb = fh.head_greedy(llama_index, Hd, idx.cfg.p).cpu().numpy()
    t1 = np.array([fh.head_greedy(llama_index, Hd[q:q + 1], idx.cfg.p).item() for q in range(16)])
    assert np.mean(tb == t1) >= 0.9


# ----------------------------------------------------------------------------- Qwen Monte Carlo


def test_mc_qwen_shape_likely_targets(fh, orc):
    """c = 9496 > 16 keys per thread of the 512-thread draw block: the 20-key instantiation."""
    cfg = synth.scaled(synth.CONFIGS["qwen"], v=151936, c=9496, d=64, p=512, name="qwen-c9496-d64")
    idx = synth.make_index(cfg)
    H = synth.make_queries(cfg, 2)
    z = synth.stored_to_f64(H, "bf16") @ synth.stored_to_f64(idx.E, "bf16").T
    targets = np.argsort(-z, axis=1)[:, :8].astype(np.int32)   # each query's dense top 8
    I = load(fh, idx, cluster_major=False)
    N = 500
    mean, se = fh.mc_token_prob(I, dev(H, "bf16"), dev(targets, "i32"), cfg.p, 1.0, N, synth.MC_SEED)
    torch.cuda.synchronize()
    mean, se = mean.cpu().numpy(), se.cpu().numpy()
    o = orc.mc(idx, H, targets, cfg.p, 1.0, synth.MC_SEED, n_draws=N)
    assert np.all(o["mean"] > 0)                  # likely targets: every estimate is informative
    check_mc(mean, se, o)


# ----------------------------------------------------------------------------- shifted INT4 centroids


def test_shifted_int4_centroids_parity_and_recall(fh, orc):
    """The reparameterised INT4 Stage 1 (Softmax Reparameterization pages; FlashHead notes, Module 3):
    centroids that share a common direction, shifted by C' = C - t·mean(C) before quantisation.  The
    GPU path scores whatever INT4 bytes the index holds, so the shifted bytes are checked against the
    oracle like any others; and removing the mean (t = 1) raises the recall of the INT4 probe sets
    against the BF16 ones (the GPU's own sets on both sides)."""
    cfg = synth.dataclasses.replace(synth.scaled(synth.CONFIGS["gemma"], v=32768, c=2048, d=1152, p=128),
                                    name="gemma-mid-aniso")
    base = synth.make_index(cfg)
    Cf = synth.anisotropic_centroids(cfg.c, cfg.d, 1.0, 77)
    C = synth.store(Cf.astype(np.float32), "bf16")
    Cb = synth.stored_to_f64(C, "bf16")
    H = synth.make_queries(cfg, 32)
    B = 32

    def sets(idx, int4):
        I = load(fh, idx, int4=int4)
        sel = torch.empty((B, cfg.p), dtype=torch.int32, device="cuda")
        fh.head_greedy(I, dev(H, "bf16"), cfg.p, debug=dict(sel=sel))
        return sel.cpu().numpy()

    bf16 = synth.Index(cfg, base.E, C, base.C2T)
    ref = sets(bf16, False)
    rec = {}
    for t in (0.0, 1.0):
        q, sc = synth.quantize_int4_g32(synth.shift_centroids(Cb, t))
        idx = synth.Index(cfg, base.E, C, base.C2T, q, sc)
        check_head(fh, orc, idx, H[:1], cfg.p, int4=True)
        check_head(fh, orc, idx, H, cfg.p, batch=4, int4=True)
        got = sets(idx, True)
        rec[t] = np.mean([len(set(got[i]) & set(ref[i])) / cfg.p for i in range(B)])
    assert rec[1.0] > rec[0.0] + 0.01, rec


def test_mc_draw_ranges_recompose(fh, orc):
    """Draws [i0, i0 + N) through the start-draw call equal the oracle's over the same draws, and two
    consecutive ranges recompose the whole run's mean."""
    cfg = synth.scaled(synth.CONFIGS["qwen"], v=16384, c=1024, d=256, p=64, name="qwen-small")
    idx = synth.make_index(cfg)
    H = synth.make_queries(cfg, 2)
    z = synth.stored_to_f64(H, "bf16") @ synth.stored_to_f64(idx.E, "bf16").T
    targets = np.argsort(-z, axis=1)[:, :4].astype(np.int32)
    I = load(fh, idx, cluster_major=False)
    Hd, td = dev(H, "bf16"), dev(targets, "i32")
    m_all, _ = fh.mc_token_prob(I, Hd, td, cfg.p, 1.0, 600, synth.MC_SEED)
    m_a, _ = fh.mc_token_prob(I, Hd, td, cfg.p, 1.0, 200, synth.MC_SEED, i0=0)
    m_b, se_b = fh.mc_token_prob(I, Hd, td, cfg.p, 1.0, 400, synth.MC_SEED, i0=200)
    torch.cuda.synchronize()
    recomposed = (200 * m_a.cpu().numpy() + 400 * m_b.cpu().numpy()) / 600
    assert np.abs(recomposed - m_all.cpu().numpy()).max() <= 1e-12
    o = orc.mc(idx, H, targets, cfg.p, 1.0, synth.MC_SEED, i0=200, i1=600)
    check_mc(m_b.cpu().numpy(), se_b.cpu().numpy(), o)
