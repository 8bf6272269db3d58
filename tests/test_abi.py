"""The C ABI library: it loads without a GPU, exports every function include/*.h declares,
the binding declares a signature for each, and host-side argument checks reject bad calls before
any device work."""

import ctypes as ct
import glob
import os
import re

import pytest

from clustered_retrieval_classification_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"\b(fh_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    path = _build.build()
    return ct.CDLL(path)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["fh_index_load", "fh_index_free", "fh_workspace_bytes", "fh_head_greedy",
                     "fh_head_sample", "fh_mc_token_prob", "fh_dense_head", "fh_last_error",
                     "fh_ws_status", "fh_stage1_scores", "fh_select_topp",
                     "fh_gather_candidates", "fh_candidate_logits", "fh_philox_u32",
                     "fh_kmeans_ws_bytes", "fh_kmeans_build", "fh_kmeans_assign", "fh_kmeans_update"]:
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
    assert L.fh_head_greedy_host(None, None, 1, 1, None, None, None, None, 0, None) == 1
    assert L.fh_workspace_bytes(None, 0, 1, 1, 1, 1) == 0
    assert L.fh_select_topp(None, 1, 8, 2, None, None) == 1
    assert L.fh_philox_u32(0, 0, 0, 0, 0, None, None) == 1


def test_cfhead_host_side_argument_checks(lib):
    """Coarse-fine head (include/fh_cfhead.h): shapes and arguments are checked before any CUDA call."""
    from clustered_retrieval_classification_b200 import flashhead as F
    L = F.load()
    out = ct.c_void_p()
    d = F.CfDesc(1000, 72, 8, 16, 16, 16, 16)
    assert L.fh_cf_load(ct.byref(d), ct.byref(out)) == 2        # d not a multiple of 8 tiles
    d = F.CfDesc(1000, 64, 8, 17, 16, 16, 16)
    assert L.fh_cf_load(ct.byref(d), ct.byref(out)) == 2        # K > 16: codes are 4 bits
    d = F.CfDesc(1000, 64, 8, 16, 16, None, 16)
    assert L.fh_cf_load(ct.byref(d), ct.byref(out)) == 1        # codebooks missing
    assert b"codebooks" in L.fh_last_error()
    assert L.fh_cf_workspace_bytes(None, 1, 1) == 0
    assert L.fh_cf_head(None, None, 1, 1, 0, 1.0, 0, 0, None, None, 0, None, None, None) == 1


def test_builder_host_side_argument_checks(lib):
    """Index builder (include/fh_kmeans.h): sizes and arguments are checked before any CUDA call."""
    from clustered_retrieval_classification_b200 import flashhead as F
    L = F.load()
    assert L.fh_kmeans_ws_bytes(100, 64, 7) == 0          # c does not divide v
    assert L.fh_kmeans_ws_bytes(112, 64, 7) >= 112 * 7 * 4
    assert L.fh_kmeans_build(None, None, 0, None) == 1    # FH_ERR_ARG
    a = F.KmeansArgs()
    a.E, a.dtype, a.v, a.d, a.c, a.iters, a.eps = 16, F.FH_F32, 112, 64, 7, 1, 1e-4
    assert L.fh_kmeans_build(ct.byref(a), None, 0, None) == 7   # FP32 E: FH_ERR_UNSUPPORTED
    a.dtype = F.FH_BF16
    a.v = 100
    assert L.fh_kmeans_build(ct.byref(a), None, 0, None) == 2   # v % c
    a.v, a.d = 112, 60
    assert L.fh_kmeans_build(ct.byref(a), None, 0, None) == 2   # d % 8
    a.d = 64
    assert L.fh_kmeans_build(ct.byref(a), None, 0, None) == 1   # init_tokens NULL
    assert b"init_tokens" in L.fh_last_error()
    assert L.fh_kmeans_assign(ct.byref(a), None, 0, None) == 1  # C_in NULL
    assert L.fh_kmeans_update(ct.byref(a), None, 0, None) == 1  # labels_in NULL


@pytest.mark.parametrize("struct,pyname", [("fh_index_desc", "IndexDesc"), ("fh_debug_out", "DebugOut"),
                                           ("fh_kmeans_args", "KmeansArgs"), ("fh_cf_desc", "CfDesc")])
def test_binding_structs_match_the_headers(tmp_path, struct, pyname):
    """Every field of the binding's ctypes structures sits at the offset the C compiler gives it."""
    import subprocess
    from clustered_retrieval_classification_b200 import flashhead as F
    py = getattr(F, pyname)
    fields = [f[0] for f in py._fields_]
    src = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "fh_kmeans.h"', '#include "fh_cfhead.h"',
             "int main(void) {",
             f'  printf("%zu\\n", sizeof({struct}));']
    lines += [f'  printf("%zu\\n", offsetof({struct}, {f}));' for f in fields]
    lines += ["  return 0;", "}"]
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    out = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert out[0] == ct.sizeof(py)
    assert out[1:] == [getattr(py, f).offset for f in fields]
