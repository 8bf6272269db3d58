"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle on the same seeded inputs.

Sizes span several blocks per kernel with ragged tails; the full Llama-shaped head is checked on
sampled queries in the launch configuration the benchmark times (batch 1, fused selection)."""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth
from headcheck import check_head as _check_head, dev, load
from parity import LOGIT_TOL, MARGIN, check_mc

pytestmark = pytest.mark.gpu

DEV = "cuda"


def widen(a, dtype):
    return synth.stored_to_f64(a, dtype)


# ----------------------------------------------------------------------------- fixtures

MID = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="llama-mid")
MID_INT4 = synth.dataclasses.replace(synth.scaled(synth.CONFIGS["gemma"], v=32768, c=2048, d=1152,
                                                  p=128), name="gemma-mid")


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.CONFIGS["tiny"]
    return synth.make_index(cfg), synth.make_queries(cfg, 256)


@pytest.fixture(scope="module")
def mid():
    return synth.make_index(MID), synth.make_queries(MID, 24)


@pytest.fixture(scope="module")
def mid_int4():
    return synth.make_index(MID_INT4), synth.make_queries(MID_INT4, 8)


# ----------------------------------------------------------------------------- Philox / Gumbel


@pytest.mark.parametrize("seed,step,row,stream", [(0, 0, 0, 0), (0xF1A54EAD, 12345, 3, 1),
                                                  (2 ** 64 - 1, 2 ** 40 + 7, 63, 2)])
def test_philox_bit_exact(fh, orc, seed, step, row, stream):
    n = 100_003
    g = fh.philox_u32(seed, step, row, stream, n).cpu().numpy().view(np.uint32)
    o = orc.philox_words(seed, step, row, stream, n)
    assert np.array_equal(g, o)


def test_gumbel_keys(fh, orc):
    rng = np.random.default_rng(1)
    s = (rng.standard_normal((3, 5000)) * 0.3).astype(np.float32)
    for tau in (0.8, 1.0):
        g = fh.gumbel_keys(dev(s, "f32"), tau, seed=99, step=7).cpu().numpy()
        o = orc.gumbel_keys(s.astype(np.float64), tau, 99, 7, 0)
        np.testing.assert_allclose(g, o, rtol=2e-6, atol=2e-5)


# ----------------------------------------------------------------------------- selection


def _select_cases():
    rng = np.random.default_rng(2)
    cases = []
    for c, p in [(1, 1), (7, 3), (64, 8), (100, 100), (2004, 128), (8016, 512), (8016, 1),
                 (9496, 512), (16384, 1024), (32768, 4000)]:
        cases.append((f"normal-{c}-{p}", rng.standard_normal((2, c)).astype(np.float32), p))
    cases.append(("ties", rng.integers(-3, 4, size=(3, 5000)).astype(np.float32), 700))
    cases.append(("all-equal", np.full((2, 3000), 0.25, np.float32), 1000))
    z = np.zeros((2, 999), np.float32)
    z[:, ::2] = -0.0
    cases.append(("signed-zero", z, 500))
    big = rng.standard_normal((2, 4000)).astype(np.float32)
    big[:, 0], big[:, 1] = 3e38, -3e38
    cases.append(("huge-range", big, 300))
    dense_bin = np.round(rng.standard_normal((2, 8016)) * 0.001, 6).astype(np.float32)
    dense_bin[:, :10] = 50.0
    cases.append(("crowded-bin", dense_bin, 2000))
    return cases


@pytest.mark.parametrize("name,keys,p", _select_cases(), ids=lambda x: x if isinstance(x, str) else "")
def test_select_bit_exact(fh, orc, name, keys, p):
    g = fh.select_topp(dev(keys, "f32"), p).cpu().numpy()
    o, _ = orc.select_topp(keys.astype(np.float64), p)
    assert np.array_equal(g, o), name


# ----------------------------------------------------------------------------- single steps


def test_stage1_scores(fh, orc, tiny, mid):
    """fp32 (tiny): the CUDA-core kernel at every batch; BF16 (mid): the CUDA-core kernel at B = 1,
    the tensor cores from B = 2 (partial 16-query blocks at 2 and 5)."""
    for idx, H in (tiny, mid):
        cfg = idx.cfg
        I = load(fh, idx)
        for B in (1, 2, 5):
            Hq = H[:B]
            g = fh.stage1_scores(I, dev(Hq, cfg.dtype)).cpu().numpy()
            o = orc.stage1_scores(idx.C, cfg.dtype, Hq, cfg.c, cfg.d)
            assert np.abs(g - o).max() <= LOGIT_TOL


@pytest.mark.parametrize("B", [1, 3, 8])
def test_stage1_scores_int4(fh, orc, mid_int4, B):
    """The CUDA-core kernel at B = 1 (one query per block); the dequantising tensor-core kernel at
    B = 3 (a partial 16-query block) and B = 8."""
    idx, H = mid_int4
    I = load(fh, idx, int4=True)
    g = fh.stage1_scores(I, dev(H[:B], "bf16")).cpu().numpy()
    o = orc.stage1_scores(None, "bf16", H[:B], idx.c, idx.d, q4=idx.C_q4, scales=idx.C_scales)
    assert np.abs(g - o).max() <= LOGIT_TOL


def test_gather_and_candidate_logits(fh, orc, mid):
    idx, H = mid
    cfg = idx.cfg
    I = load(fh, idx)
    rng = np.random.default_rng(5)
    sel = np.sort(np.stack([rng.choice(cfg.c, cfg.p, replace=False) for _ in range(3)]), axis=1)
    sel = sel.astype(np.int32)
    g = fh.gather_candidates(I, dev(sel, "i32")).cpu().numpy()
    o = orc.gather(idx.C2T, sel)
    assert np.array_equal(g, o)
    z = fh.candidate_logits(I, dev(H[:3], cfg.dtype), dev(o, "i32")).cpu().numpy()
    assert np.abs(z - orc.logits(idx.E, cfg.dtype, H[:3], o)).max() <= LOGIT_TOL


# ----------------------------------------------------------------------------- fused head


def test_greedy_tiny_fp32_batch1(fh, orc, tiny):
    idx, H = tiny
    for q in range(0, 64, 3):
        _check_head(fh, orc, idx, H[q:q + 1], idx.cfg.p)


def test_greedy_tiny_batched(fh, orc, tiny):
    idx, H = tiny
    _check_head(fh, orc, idx, H[:64], idx.cfg.p)
    _check_head(fh, orc, idx, H[:5], idx.cfg.p)


@pytest.mark.parametrize("cluster_major", [True, False])
def test_greedy_mid_batch1(fh, orc, mid, cluster_major):
    idx, H = mid
    for q in range(6):
        _check_head(fh, orc, idx, H[q:q + 1], idx.cfg.p, cluster_major=cluster_major)


@pytest.mark.parametrize("B", [3, 16])
def test_greedy_mid_batched(fh, orc, mid, B):
    idx, H = mid
    _check_head(fh, orc, idx, H, idx.cfg.p, batch=B)


@pytest.mark.parametrize("p", [1, 2004])
def test_greedy_mid_edge_p(fh, orc, mid, p):
    idx, H = mid
    _check_head(fh, orc, idx, H[:1], p)
    _check_head(fh, orc, idx, H[:2], p)


def test_sample_mid(fh, orc, mid):
    idx, H = mid
    for step in range(4):
        _check_head(fh, orc, idx, H[step:step + 1], idx.cfg.p, sample=True, tau=0.8,
                    seed=synth.SAMPLE_SEED, step=step)
    _check_head(fh, orc, idx, H[:6], idx.cfg.p, sample=True, tau=0.8, seed=synth.SAMPLE_SEED,
                step=99)


def test_int4_mid(fh, orc, mid_int4):
    idx, H = mid_int4
    _check_head(fh, orc, idx, H[:1], idx.cfg.p, int4=True)
    _check_head(fh, orc, idx, H[:4], idx.cfg.p, int4=True)


def test_p_equals_c_matches_dense(fh, mid):
    """With p = c the candidates are the vocabulary: the greedy head must return the dense argmax and
    the sampling head the dense sample (same Stage-2 noise keyed by token id)."""
    idx, H = mid
    I = load(fh, idx)
    Hd = dev(H[:4], "bf16")
    for B in (1, 4):
        g = fh.head_greedy(I, Hd[:B], idx.c).cpu().numpy()
        d = fh.dense_head(I, Hd[:B]).cpu().numpy()
        assert np.array_equal(g, d)
        gs = fh.head_sample(I, Hd[:B], idx.c, 0.8, 5, 3).cpu().numpy()
        ds = fh.dense_head(I, Hd[:B], sample=True, tau=0.8, seed=5, step=3).cpu().numpy()
        assert np.array_equal(gs, ds)


# ----------------------------------------------------------------------------- dense head


@pytest.mark.parametrize("sample", [False, True])
def test_dense_head(fh, orc, mid, sample):
    idx, H = mid
    cfg = idx.cfg
    I = load(fh, idx)
    B = 3
    logits = torch.empty((B, cfg.v), dtype=torch.float32, device=DEV)
    tok = fh.dense_head(I, dev(H[:B], "bf16"), sample=sample, tau=0.8, seed=11, step=2,
                        logits=logits).cpu().numpy()
    o = orc.dense(idx, H[:B], sample=sample, tau=0.8, seed=11, step=2, want_z=True)
    assert np.abs(logits.cpu().numpy() - o["z"]).max() <= LOGIT_TOL
    for q in range(B):
        if tok[q] != o["tok"][q]:
            assert o["tok_margin"][q] <= MARGIN


# ----------------------------------------------------------------------------- Monte Carlo


def test_mc_matches_oracle(fh, orc):
    cfg = synth.scaled(synth.CONFIGS["qwen"], v=16384, c=1024, d=256, p=64, name="qwen-small")
    idx = synth.make_index(cfg)
    H = synth.make_queries(cfg, 3)
    targets = synth.make_targets(cfg.v, 3, 8)
    # make some targets likely: include each query's dense argmax
    z = widen(H, "bf16") @ widen(idx.E, "bf16").T
    targets[:, 0] = np.argmax(z, axis=1)
    I = load(fh, idx)
    N = 2000
    mean, se = fh.mc_token_prob(I, dev(H, "bf16"), dev(targets, "i32"), cfg.p, 1.0, N, synth.MC_SEED)
    mean, se = mean.cpu().numpy(), se.cpu().numpy()
    o = orc.mc(idx, H, targets, cfg.p, 1.0, synth.MC_SEED, n_draws=N)
    check_mc(mean, se, o)


def test_mc_p_equals_c_is_dense_softmax(fh):
    cfg = synth.scaled(synth.CONFIGS["qwen"], v=4096, c=256, d=128, p=256, name="qwen-pc")
    idx = synth.make_index(cfg)
    H = synth.make_queries(cfg, 2)
    targets = np.array([[0, 1, 2, 3], [4000, 17, 256, 4095]], np.int32)
    I = load(fh, idx)
    mean, se = fh.mc_token_prob(I, dev(H, "bf16"), dev(targets, "i32"), cfg.c, 0.7, 50, 1)
    logits = torch.empty((2, cfg.v), dtype=torch.float32, device=DEV)
    fh.dense_head(I, dev(H, "bf16"), logits=logits)
    soft = torch.softmax(logits.double() / 0.7, dim=1).cpu().numpy()
    np.testing.assert_allclose(mean.cpu().numpy(), np.take_along_axis(soft, targets, 1), rtol=1e-5)
    assert np.all(se.cpu().numpy() < 1e-9)


# ----------------------------------------------------------------------------- robustness


def test_determinism(fh, mid):
    idx, H = mid
    I = load(fh, idx)
    Hd = dev(H[:1], "bf16")
    runs = [fh.head_sample(I, Hd, idx.cfg.p, 0.8, 1, 2).item() for _ in range(3)]
    assert len(set(runs)) == 1
    a = [fh.head_greedy(I, dev(H[:8], "bf16"), idx.cfg.p).cpu().numpy() for _ in range(2)]
    assert np.array_equal(a[0], a[1])


def test_bad_c2t_rejected(fh):
    idx = synth.random_index(v=256, d=64, c=16, seed=3, dtype="bf16")
    bad = idx.C2T.copy()
    bad[3, 2] = bad[5, 1]                       # duplicate id
    with pytest.raises(fh.FlashHeadError) as e:
        fh.index_from_host(idx.E, idx.C, bad, "bf16")
    assert e.value.status == 3
    bad = idx.C2T.copy()
    bad[0, 0] = 256                             # out of range
    with pytest.raises(fh.FlashHeadError):
        fh.index_from_host(idx.E, idx.C, bad, "bf16")


def test_batch1_without_debug_outputs_on_one_workspace(fh, orc, mid):
    """The timed configuration: batch 1, no debug outputs, one workspace reused by consecutive calls
    whose p and mode change (each call must ignore what the earlier ones left behind).  Every token
    must equal that of a call on a fresh zeroed workspace with debug outputs (the same selection and
    the same fp32 dot products), and the oracle's wherever its margins decide it."""
    idx, H = mid
    cfg = idx.cfg
    I = load(fh, idx)
    ws = I.workspace(fh.FH_OP_GREEDY, 1, cfg.c)
    plan = [(0, cfg.p, False), (1, 37, False), (2, cfg.p, True), (3, 1, False), (4, cfg.c, False),
            (5, cfg.p, False), (6, 500, True), (7, cfg.p, False), (7, 37, False), (8, 2, True)]
    checked = 0
    for q, p, sample in plan:
        Hd = dev(H[q:q + 1], cfg.dtype)
        fresh = torch.zeros_like(ws)
        dbg = dict(sel=torch.empty((1, p), dtype=torch.int32, device=DEV),
                   cand_tok=torch.empty((1, p * cfg.b), dtype=torch.int32, device=DEV),
                   cand_logit=torch.empty((1, p * cfg.b), dtype=torch.float32, device=DEV))
        if sample:
            args = (I, Hd, p, 0.8, synth.SAMPLE_SEED, q)
            tok = fh.head_sample(*args, ws=ws).item()
            ref = fh.head_sample(*args, ws=fresh, debug=dbg).item()
        else:
            tok = fh.head_greedy(I, Hd, p, ws=ws).item()
            ref = fh.head_greedy(I, Hd, p, ws=fresh, debug=dbg).item()
        assert tok == ref, (q, p, sample)
        o = orc.head(idx, H[q:q + 1], p, sample=sample, tau=0.8, seed=synth.SAMPLE_SEED, step=q)
        if (p == cfg.c or o["set_margin"][0] > MARGIN) and o["tok_margin"][0] > MARGIN:
            assert tok == o["tok"][0], (q, p, sample)
            checked += 1
    fh.ws_status(ws)
    assert checked >= 2


@pytest.mark.parametrize("B", [1, 5])
def test_head_greedy_host_buffers(fh, mid, B):
    """fh_head_greedy_host (host query and token buffers, both copies queued by the library) gives
    the tokens of fh_head_greedy on the same queries, call after call on one workspace."""
    idx, H = mid
    cfg = idx.cfg
    I = load(fh, idx)
    ws = I.workspace(fh.FH_OP_GREEDY, B, cfg.p)
    h_dev = torch.empty((B, cfg.d), dtype=dev(H[:1], cfg.dtype).dtype, device=DEV)
    tok_dev = torch.empty(B, dtype=torch.int32, device=DEV)
    tok_host = torch.empty(B, dtype=torch.int32).pin_memory()
    for k in range(3):
        Hd = dev(H[k:k + B], cfg.dtype)
        ref = fh.head_greedy(I, Hd, cfg.p).cpu().numpy()
        fh.head_greedy_host(I, Hd.cpu().pin_memory(), cfg.p, tok_host, h_dev, tok_dev, ws=ws)
        torch.cuda.synchronize()
        assert np.array_equal(tok_host.numpy(), ref), k
    fh.ws_status(ws)


def test_bounded_wait_times_out_and_workspace_recovers(fh, mid):
    """Failure detection without a fault: one histogram bin of the workspace is pre-set so that the
    batch-1 kernel's grid barrier (a bounded poll of the histogram until its counts reach c) can never
    complete.  Every block gives up after 0.5 s with no copy in flight; the call records
    FH_ERR_TIMEOUT, fh_ws_status reports it once and resets the control block, and the same workspace
    then gives the right token again."""
    idx, H = mid
    cfg = idx.cfg
    I = load(fh, idx)
    Hd = dev(H[:1], cfg.dtype)
    ws = torch.zeros(I.workspace_bytes(fh.FH_OP_GREEDY, 1, cfg.p), dtype=torch.uint8, device=DEV)
    ref = fh.head_greedy(I, Hd, cfg.p, ws=torch.zeros_like(ws)).item()
    ws[1024:1028] = 0xFF                       # bin 0 = 2^32 - 1: the counts now sum to c - 1
    fh.head_greedy(I, Hd, cfg.p, ws=ws)
    torch.cuda.synchronize()
    with pytest.raises(fh.FlashHeadError) as e:
        fh.ws_status(ws)
    assert e.value.status == 6                 # FH_ERR_TIMEOUT
    fh.ws_status(ws)                           # reported once, then clear
    assert fh.head_greedy(I, Hd, cfg.p, ws=ws).item() == ref
    fh.ws_status(ws)


def test_workspace_status_clean(fh, mid):
    idx, H = mid
    I = load(fh, idx)
    ws = I.workspace(fh.FH_OP_GREEDY, 1, idx.cfg.p)
    fh.head_greedy(I, dev(H[:1], "bf16"), idx.cfg.p, ws=ws)
    fh.ws_status(ws)
    with pytest.raises(fh.FlashHeadError) as e:
        fh.head_greedy(I, dev(H[:1], "bf16"), idx.cfg.p, ws=ws[:100])
    assert e.value.status == 4


# ----------------------------------------------------------------------------- full size


@pytest.fixture(scope="module")
def llama(llama_host):
    idx, H = llama_host
    return idx, H[:4]


def test_llama_full_size_batch1_sampled(fh, orc, llama):
    """The Llama-shaped head (v=128256, d=2048, c=8016, p=512) at batch 1 with the fused selection,
    the configuration the benchmark times; four queries greedy and two sampled."""
    idx, H = llama
    for q in range(4):
        _check_head(fh, orc, idx, H[q:q + 1], idx.cfg.p)
    for q in range(2):
        _check_head(fh, orc, idx, H[q:q + 1], idx.cfg.p, sample=True, tau=0.8,
                    seed=synth.SAMPLE_SEED, step=q)


@pytest.mark.parametrize("perturb", [0.0, 1e-3])
def test_crowded_boundary_bin_batch1(fh, orc, perturb):
    """More keys than the fast path ranks share the boundary bin (identical or nearly identical
    centroids), so the batch-1 kernel takes its full-selection branch; ties break by cluster id."""
    v, d, c = 8192, 64, 1024
    idx = synth.random_index(v=v, d=d, c=c, seed=17, dtype="bf16")
    rng = np.random.default_rng(3)
    base = rng.standard_normal(d)
    rows = base[None, :] + perturb * rng.standard_normal((c, d))
    rows /= np.linalg.norm(rows, axis=1, keepdims=True)
    idx.C = synth.store(rows.astype(np.float32), "bf16")
    H = synth.store((rng.standard_normal((3, d)) * 2).astype(np.float32), "bf16")
    for q in range(3):
        _check_head(fh, orc, idx, H[q:q + 1], 100)
