"""The allocation-free greedy head (fh_head_greedy_static).

For callers that can neither allocate device memory nor lend a workspace, the library keeps the
scratch of one batch-1 greedy call in a static device array.  These checks call it through the C ABI
and compare it with the workspace-based fh_head_greedy on the same inputs, on consecutive calls (the
array keeps the previous call's contents, so the second call checks that the call clears what it
must).  Token ids are integers, so the comparison is exact.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_calls(fh):
    cfg = synth.scaled(synth.CONFIGS["llama"], v=32064, c=2004, d=512, p=128, name="static-mid")
    idx = synth.make_index(cfg)
    H = fh.device_array(synth.make_queries(cfg, 4), "bf16")
    I = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    ws = I.workspace(fh.FH_OP_GREEDY, 1, cfg.p)
    for q in (0, 1, 1, 2):                       # consecutive calls, one repeated query
        got = fh.head_greedy_static(I, H[q:q + 1], cfg.p)
        ref = fh.head_greedy(I, H[q:q + 1], cfg.p, ws=ws)
        torch.cuda.synchronize()
        assert got.item() == ref.item()
    # p = c (every cluster) and p = 1 through the same array
    for p in (1, cfg.c):
        got = fh.head_greedy_static(I, H[3:4], p)
        ref = fh.head_greedy(I, H[3:4], p, ws=I.workspace(fh.FH_OP_GREEDY, 1, p))
        assert got.item() == ref.item()


def test_static_scratch_rejects_indices_that_do_not_fit(fh):
    c = 32768                                    # keys and probe set of p = c fill the array
    rng = np.random.default_rng(0)
    E = synth.store(rng.standard_normal((c, 8)).astype(np.float32), "bf16")
    C2T = rng.permutation(c).astype(np.int32).reshape(c, 1)
    I = fh.index_from_host(E, E[C2T[:, 0]], C2T, "bf16", cluster_major=False)
    H = fh.device_array(synth.store(rng.standard_normal((1, 8)).astype(np.float32), "bf16"), "bf16")
    with pytest.raises(fh.FlashHeadError) as e:
        fh.head_greedy_static(I, H, c)
    assert e.value.status == 4 and "static scratch" in str(e.value)
