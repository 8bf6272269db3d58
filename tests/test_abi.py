"""The C ABI library: it loads without a GPU, exports every function include/flashhead.h declares,
the binding declares a signature for each, and host-side argument checks reject bad calls before
any device work."""

import ctypes as ct
import os
import re

import pytest

from clustered_retrieval_classification_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashhead.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fh_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    path = _build.build()
    return ct.CDLL(path)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["fh_index_load", "fh_index_free", "fh_workspace_bytes", "fh_head_greedy",
                     "fh_head_sample", "fh_mc_token_prob", "fh_dense_head", "fh_last_error",
                     "fh_ws_status", "fh_stage1_scores", "fh_select_topp",
                     "fh_gather_candidates", "fh_candidate_logits", "fh_philox_u32"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_symbol():
    from clustered_retrieval_classification_b200 import flashhead
    assert sorted(flashhead.SIGNATURES) == declared_functions()


def test_host_side_argument_checks(lib):
    from clustered_retrieval_classification_b200 import flashhead as F
    L = F.load()
    # a shape error is reported before any CUDA call: v != c*b
    desc = F.IndexDesc(100, 64, 7, 16, F.FH_BF16, F.FH_STAGE1_DENSE, 16, 16, 16, None, None, None)
    out = ct.c_void_p()
    assert L.fh_index_load(ct.byref(desc), None, 0, None, ct.byref(out)) == 2   # FH_ERR_SHAPE
    assert b"c*b" in L.fh_last_error()
    desc = F.IndexDesc(112, 60, 7, 16, F.FH_BF16, F.FH_STAGE1_DENSE, 16, 16, 16, None, None, None)
    assert L.fh_index_load(ct.byref(desc), None, 0, None, ct.byref(out)) == 2   # d % 8
    desc = F.IndexDesc(112, 64, 7, 16, F.FH_BF16, F.FH_STAGE1_INT4_G32, 16, 16, 16, None, None, None)
    assert L.fh_index_load(ct.byref(desc), None, 0, None, ct.byref(out)) == 1   # INT4 arrays missing
    desc = F.IndexDesc(112, 64, 7, 16, F.FH_BF16, F.FH_STAGE1_DENSE, 16, 16, 16, None, None, None)
    assert L.fh_index_load(ct.byref(desc), None, 0, None, ct.byref(out)) == 4   # no workspace
    assert L.fh_index_load_ws_bytes(ct.byref(desc)) >= 1024 + 16
    # calls on a NULL handle
    assert L.fh_head_greedy(None, None, 1, 1, None, None, 0, None, None) == 1
    assert L.fh_workspace_bytes(None, 0, 1, 1, 1, 1) == 0
    assert L.fh_select_topp(None, 1, 8, 2, None, None) == 1
    assert L.fh_philox_u32(0, 0, 0, 0, 0, None, None) == 1
