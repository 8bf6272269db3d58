"""Index directories (clustered_retrieval_classification_b200/index_io.py): round trips are exact,
a changed byte or a broken invariant is refused before anything reaches the device."""

import json
import os

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import index_io, synth


def small_index():
    idx = synth.random_index(v=512, d=64, c=32, seed=5, dtype="bf16")
    rows = synth.f32_from_bf16(idx.C)
    q4, sc = synth.quantize_int4_g32(rows)
    return idx, q4, sc


def test_round_trip_is_exact(tmp_path):
    idx, q4, sc = small_index()
    hdr = index_io.save_index(str(tmp_path), idx.E, idx.C, idx.C2T, "bf16", C_q4=q4, C_scales=sc,
                              meta={"source": "random_index", "seed": 5})
    assert (hdr["v"], hdr["d"], hdr["c"], hdr["b"]) == (512, 64, 32, 16)
    h2, a = index_io.load_index(str(tmp_path))
    assert h2 == hdr
    for name, ref in (("E", idx.E), ("C", idx.C), ("C2T", idx.C2T), ("C_q4", q4), ("C_scales", sc)):
        assert a[name].dtype == ref.dtype and np.array_equal(a[name], ref), name


def test_torch_tensors_are_stored_as_their_bits(tmp_path):
    idx, _, _ = small_index()
    E = torch.from_numpy(idx.E.view(np.int16)).view(torch.bfloat16)
    C = torch.from_numpy(idx.C.view(np.int16)).view(torch.bfloat16)
    index_io.save_index(str(tmp_path), E, C, torch.from_numpy(idx.C2T), "bf16")
    _, a = index_io.load_index(str(tmp_path))
    assert np.array_equal(a["E"], idx.E) and np.array_equal(a["C"], idx.C)
    assert "C_q4" not in a


def test_changed_bytes_are_refused(tmp_path):
    idx, _, _ = small_index()
    index_io.save_index(str(tmp_path), idx.E, idx.C, idx.C2T, "bf16")
    path = os.path.join(str(tmp_path), "C.npy")
    C = np.load(path)
    C[3, 7] ^= 1
    np.save(path, C)
    with pytest.raises(ValueError, match="SHA-256"):
        index_io.load_index(str(tmp_path))
    index_io.load_index(str(tmp_path), verify=False)  # the caller may opt out


def test_broken_invariants_are_refused(tmp_path):
    idx, _, _ = small_index()
    bad = idx.C2T.copy()
    bad[0, 0] = bad[1, 0]
    with pytest.raises(ValueError, match="permutation"):
        index_io.save_index(str(tmp_path / "a"), idx.E, idx.C, bad, "bf16")
    with pytest.raises(ValueError, match="c\\*b"):
        index_io.save_index(str(tmp_path / "b"), idx.E[:500], idx.C, idx.C2T, "bf16")
    with pytest.raises(TypeError):
        index_io.save_index(str(tmp_path / "c"), idx.E.astype(np.float32), idx.C, idx.C2T, "bf16")
    index_io.save_index(str(tmp_path / "d"), idx.E, idx.C, idx.C2T, "bf16")
    hp = tmp_path / "d" / "index.json"
    h = json.loads(hp.read_text())
    h["version"] = 99
    hp.write_text(json.dumps(h))
    with pytest.raises(ValueError, match="not a flashhead-index"):
        index_io.load_index(str(tmp_path / "d"))


@pytest.mark.gpu
def test_saved_index_serves_the_same_tokens(fh, tmp_path):
    """An index written to disk and loaded back onto the device gives the same tokens as the
    index uploaded directly."""
    from clustered_retrieval_classification_b200 import index_io
    idx = synth.random_index(v=8192, d=64, c=1024, seed=17, dtype="bf16")
    index_io.save_index(str(tmp_path), idx.E, idx.C, idx.C2T, "bf16")
    I1 = fh.index_from_host(idx.E, idx.C, idx.C2T, "bf16")
    I2 = index_io.to_device(str(tmp_path))
    rng = np.random.default_rng(2)
    H = fh.device_array(synth.store((rng.standard_normal((4, 64)) * 2).astype(np.float32), "bf16"), "bf16")
    for q in range(4):
        assert int(fh.head_greedy(I1, H[q:q + 1], 64).item()) == int(fh.head_greedy(I2, H[q:q + 1], 64).item())
