"""The allocation-free greedy head (fh_head_greedy_static).

For callers that can neither allocate device memory nor lend a workspace, the library keeps the
scratch of one batch-1 greedy call in a static device array.  These checks call it through the C ABI
and compare it with the workspace-based fh_head_greedy on the same inputs, on consecutive calls (the
array keeps the previous call's contents, so later calls check that each call leaves it ready), on
both batch-1 code paths (the persistent kernel up to 16384 clusters, the separate Stage-1 / selection
/ Stage-2 kernels above), and check that a call that fails on the device reports it: -1 in its output
and the error in fh_static_status.  Token ids are integers, so the comparison is exact.  This file is
collected last on purpose.
"""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth

pytestmark = pytest.mark.gpu


class _Raw:
    """A byte view of raw device memory for torch.as_tensor (the static scratch, for the fault test)."""

    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3}


def _compare(fh, I, H, p, ws, queries):
    for q in queries:
        got = fh.head_greedy_static(I, H[q:q + 1], p)
        ref = fh.head_greedy(I, H[q:q + 1], p, ws=ws)
        torch.cuda.synchronize()
        assert got.item() == ref.item(), (q, p)
    fh.static_status()


def test_static_scratch_matches_workspace_calls(fh):
    cfg = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="static-mid")
    idx = synth.make_index(cfg)
    H = fh.device_array(synth.make_queries(cfg, 4), "bf16")
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    _compare(fh, I, H, cfg.p, I.workspace(fh.FH_OP_GREEDY, 1, cfg.p), (0, 1, 1, 2))
    # p = c (every cluster) and p = 1 through the same array
    for p in (1, cfg.c):
        _compare(fh, I, H, p, I.workspace(fh.FH_OP_GREEDY, 1, p), (3,))


def test_static_scratch_above_the_persistent_kernel(fh):
    """20000 clusters: the batch-1 call runs the separate Stage-1, selection and Stage-2 kernels, whose
    per-query tickets live in the shared array too."""
    cfg = synth.scaled(synth.CONFIGS["llama"], v=20000 * 4, c=20000, d=64, p=512, name="static-c20000")
    idx = synth.make_index(cfg)
    H = fh.device_array(synth.make_queries(cfg, 3), "bf16")
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    _compare(fh, I, H, cfg.p, I.workspace(fh.FH_OP_GREEDY, 1, cfg.p), (0, 1, 2, 0))


def test_static_scratch_reports_a_device_side_failure(fh):
    """Failure detection without a fault: one histogram bin of the static array is pre-set so that the
    persistent kernel's grid barrier (a bounded poll of the histogram until its counts reach c) can
    never complete.  The call gives up after 0.5 s with no copy in flight and leaves -1 in its output;
    fh_static_status reports FH_ERR_TIMEOUT once and zeroes the control block; the next call gives
    the workspace call's token again."""
    cfg = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="static-mid")
    idx = synth.make_index(cfg)
    H = fh.device_array(synth.make_queries(cfg, 1), "bf16")
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    ref = fh.head_greedy(I, H, cfg.p, ws=I.workspace(fh.FH_OP_GREEDY, 1, cfg.p)).item()
    fh.head_greedy_static(I, H, cfg.p)
    torch.cuda.synchronize()
    fh.static_status()
    ptr, n = fh.static_scratch()
    assert n > 5120
    scratch = torch.as_tensor(_Raw(ptr, n), device="cuda")
    scratch[1024:1028] = 0xFF                    # bin 0 = 2^32 - 1: the counts now sum to c - 1
    torch.cuda.synchronize()
    out = fh.head_greedy_static(I, H, cfg.p)
    torch.cuda.synchronize()
    assert out.item() == -1
    with pytest.raises(fh.FlashHeadError) as e:
        fh.static_status()
    assert e.value.status == 6                   # FH_ERR_TIMEOUT
    fh.static_status()                           # reported once, then clear
    for _ in range(2):
        assert fh.head_greedy_static(I, H, cfg.p).item() == ref
    fh.static_status()


def test_static_scratch_rejects_indices_that_do_not_fit(fh):
    c = 16384                                    # the persistent kernel's word table plus p = c
    rng = np.random.default_rng(0)
    E = synth.store(rng.standard_normal((c, 8)).astype(np.float32), "bf16")
    C2T = rng.permutation(c).astype(np.int32).reshape(c, 1)
    I = fh.index_from_host(E, E[C2T[:, 0]], C2T, "bf16", cluster_major=False)
    H = fh.device_array(synth.store(rng.standard_normal((1, 8)).astype(np.float32), "bf16"), "bf16")
    with pytest.raises(fh.FlashHeadError) as e:
        fh.head_greedy_static(I, H, c)
    assert e.value.status == 4 and "static scratch" in str(e.value)
    with pytest.raises(fh.FlashHeadError) as e:  # argument errors are reported before any launch
        fh.head_greedy_static(I, H, 0)
    assert e.value.status == 1
