"""Checks of the seeded input generator: equal-size clusters, a permutation C2T, unit centroids that
are the normalised means of their stored rows (FlashHead notes, Module 1 and Eq. 5), BF16 rounding,
and determinism."""

import math

import numpy as np
import pytest
import torch

from clustered_retrieval_classification_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 1e-30],
                                 np.float32)])
    ours = synth.bf16_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.f32_from_bf16(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("name", ["tiny"])
def test_index_invariants(name):
    cfg = synth.CONFIGS[name]
    idx = synth.make_index(cfg)
    v, c, b, d = cfg.v, cfg.c, cfg.b, cfg.d
    assert idx.C2T.shape == (c, b) and idx.C2T.dtype == np.int32
    flat = np.sort(idx.C2T.reshape(-1))
    assert np.array_equal(flat, np.arange(v))                       # permutation of 0..v-1
    assert np.all(np.diff(idx.C2T, axis=1) > 0)                      # rows ascending
    Cw = synth.stored_to_f64(idx.C, cfg.dtype)
    assert np.allclose(np.linalg.norm(Cw, axis=1), 1.0, atol=1e-6)
    Ew = synth.stored_to_f64(idx.E, cfg.dtype)
    means = Ew[idx.C2T].mean(axis=1)
    means /= np.linalg.norm(means, axis=1, keepdims=True)
    assert np.allclose(Cw, means, atol=1e-7)
    norms = np.linalg.norm(Ew, axis=1)
    assert norms.min() > 0.8 - 1e-5 and norms.max() < 1.2 + 1e-5
    # each token is closest (cosine) to its own centroid for this noise level
    own = np.einsum("kbd,kd->kb", Ew[idx.C2T], Cw)
    assert own.mean() > 0.9 * norms.mean()


def test_heavy_tokens_and_bf16_scaled():
    cfg = synth.scaled(synth.CONFIGS["llama"], v=8192, c=512, d=128)
    idx = synth.make_index(cfg)
    Ew = synth.stored_to_f64(idx.E, "bf16")
    norms = np.linalg.norm(Ew, axis=1)
    heavy = norms > 2.0
    assert heavy.sum() == math.floor(0.02 * cfg.v)
    assert norms[heavy].min() > 3 * 0.8 - 0.05 and norms[~heavy].max() < 1.2 + 0.01
    assert np.array_equal(np.sort(idx.C2T.reshape(-1)), np.arange(cfg.v))


def test_determinism():
    cfg = synth.scaled(synth.CONFIGS["llama"], v=4096, c=256, d=64)
    a, b = synth.make_index(cfg), synth.make_index(cfg)
    assert np.array_equal(a.E, b.E) and np.array_equal(a.C, b.C) and np.array_equal(a.C2T, b.C2T)
    assert np.array_equal(synth.make_queries(cfg, 4), synth.make_queries(cfg, 4))


def test_queries_scale():
    cfg = synth.scaled(synth.CONFIGS["llama"], v=4096, c=256, d=2048)
    h = synth.stored_to_f64(synth.make_queries(cfg, 64), "bf16")
    assert abs(np.linalg.norm(h, axis=1).mean() - 8.0) < 0.2


def test_int4_index():
    cfg = synth.scaled(synth.CONFIGS["gemma"], v=4096, c=256, d=128)
    idx = synth.make_index(cfg)
    assert idx.C_q4.shape == (256, 64) and idx.C_scales.shape == (256, 4)
