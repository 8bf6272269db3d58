"""Saving and loading a FlashHead index on disk.

An index is built once, offline (the equal-size k-means builder, or the synthetic generator) and
served many times, so it is kept as a directory:

    index.json    header: format and version, v, d, c, b, storage dtype, and for every array its
                  file, shape, numpy dtype and SHA-256 digest, plus free-form metadata
    E.npy         v x d token embeddings
    C.npy         c x d centroids (unit rows)
    C2T.npy       c x b int32 cluster-to-token table (row k = the tokens of cluster k)
    C_q4.npy      optional: c x d/2 uint8 INT4 centroids (two per byte, low nibble = even column)
    C_scales.npy  optional: c x d/32 BF16 group scales

BF16 arrays are stored as their uint16 bit patterns (dtype "bf16" in the header), fp32 as float32.
Loading checks every digest and the index invariants (v = c*b, C2T a permutation of 0..v-1, shapes
consistent) before anything reaches the device.  This module does host I/O only; `to_device`
hands the arrays to the CUDA library through the binding.
"""

from __future__ import annotations

import hashlib
import json
import os

import numpy as np

FORMAT = "flashhead-index"
VERSION = 1
_HEADER = "index.json"
_OPTIONAL = ("C_q4", "C_scales")


def _as_host(a, kind: str) -> np.ndarray:
    """A numpy array in storage form: uint16 patterns for "bf16", float32, int32 or uint8."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            t = a.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            a = t.numpy()
    except ImportError:  # the module works on numpy arrays alone
        pass
    a = np.ascontiguousarray(a)
    want = {"bf16": np.uint16, "f32": np.float32, "i32": np.int32, "u8": np.uint8}[kind]
    if a.dtype != want:
        raise TypeError(f"expected {np.dtype(want).name} storage for {kind}, got {a.dtype}")
    return a


def _sha256(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def check_invariants(E: np.ndarray, C: np.ndarray, C2T: np.ndarray, C_q4=None, C_scales=None):
    """Shapes consistent, v = c*b, and C2T a permutation of 0..v-1 (each cluster exactly b tokens)."""
    v, d = E.shape
    c, b = C2T.shape
    if v != c * b:
        raise ValueError(f"v = {v} is not c*b = {c}*{b}")
    if C.shape != (c, d):
        raise ValueError(f"C has shape {C.shape}, expected {(c, d)}")
    flat = C2T.ravel()
    if flat.min(initial=0) < 0 or flat.max(initial=0) >= v or np.bincount(flat, minlength=v).max(initial=0) != 1:
        raise ValueError("C2T is not a permutation of 0..v-1")
    if C_q4 is not None and C_q4.shape != (c, d // 2):
        raise ValueError(f"C_q4 has shape {C_q4.shape}, expected {(c, d // 2)}")
    if C_scales is not None and C_scales.shape != (c, d // 32):
        raise ValueError(f"C_scales has shape {C_scales.shape}, expected {(c, d // 32)}")


def save_index(path: str, E, C, C2T, dtype: str = "bf16", C_q4=None, C_scales=None,
               meta: dict | None = None) -> dict:
    """Write an index directory (created if missing).  E and C in `dtype` ("bf16" or "f32") as numpy
    storage arrays or torch tensors; C2T int32.  Returns the header that was written."""
    if dtype not in ("bf16", "f32"):
        raise ValueError("dtype must be 'bf16' or 'f32'")
    arrays = {"E": _as_host(E, dtype), "C": _as_host(C, dtype), "C2T": _as_host(C2T, "i32")}
    if C_q4 is not None:
        arrays["C_q4"] = _as_host(C_q4, "u8")
    if C_scales is not None:
        arrays["C_scales"] = _as_host(C_scales, "bf16")
    check_invariants(arrays["E"], arrays["C"], arrays["C2T"], arrays.get("C_q4"), arrays.get("C_scales"))
    os.makedirs(path, exist_ok=True)
    v, d = arrays["E"].shape
    c, b = arrays["C2T"].shape
    header = {"format": FORMAT, "version": VERSION, "v": int(v), "d": int(d), "c": int(c),
              "b": int(b), "dtype": dtype, "meta": meta or {}, "arrays": {}}
    for name, a in arrays.items():
        fname = f"{name}.npy"
        np.save(os.path.join(path, fname), a, allow_pickle=False)
        header["arrays"][name] = {"file": fname, "shape": list(a.shape), "numpy_dtype": a.dtype.name,
                                  "sha256": _sha256(a)}
    tmp = os.path.join(path, _HEADER + ".tmp")
    with open(tmp, "w") as f:
        json.dump(header, f, indent=1, sort_keys=True)
    os.replace(tmp, os.path.join(path, _HEADER))  # the header appears last, complete
    return header


def load_index(path: str, verify: bool = True) -> tuple[dict, dict]:
    """Read an index directory.  Returns (header, arrays) with arrays E, C, C2T and the optional
    INT4 pair.  With verify (default) every digest and invariant is checked; a mismatch raises
    ValueError naming the array."""
    with open(os.path.join(path, _HEADER)) as f:
        header = json.load(f)
    if header.get("format") != FORMAT or header.get("version") != VERSION:
        raise ValueError(f"not a {FORMAT} v{VERSION} directory: {path}")
    arrays = {}
    for name, info in header["arrays"].items():
        a = np.load(os.path.join(path, info["file"]), allow_pickle=False)
        if list(a.shape) != info["shape"] or a.dtype.name != info["numpy_dtype"]:
            raise ValueError(f"{name}: shape or dtype differs from the header")
        if verify and _sha256(a) != info["sha256"]:
            raise ValueError(f"{name}: SHA-256 digest differs from the header")
        arrays[name] = a
    for name in ("E", "C", "C2T"):
        if name not in arrays:
            raise ValueError(f"{name} is missing")
    if verify:
        check_invariants(arrays["E"], arrays["C"], arrays["C2T"], arrays.get("C_q4"),
                         arrays.get("C_scales"))
    return header, arrays


def to_device(path: str, int4: bool = False, cluster_major: bool = True, device="cuda"):
    """Load an index directory onto the GPU as a served index (clustered_retrieval_classification_b200
    .flashhead.Index); int4 selects the INT4 Stage 1 stored with it."""
    from . import flashhead as F
    header, a = load_index(path)
    if int4 and ("C_q4" not in a or "C_scales" not in a):
        raise ValueError("this index holds no INT4 centroids")
    return F.index_from_host(a["E"], a["C"], a["C2T"], header["dtype"],
                             C_q4=a.get("C_q4") if int4 else None,
                             C_scales=a.get("C_scales") if int4 else None, int4=int4,
                             cluster_major=cluster_major, device=device)
