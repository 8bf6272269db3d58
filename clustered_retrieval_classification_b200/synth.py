"""Seeded synthetic FlashHead indices and queries.

This module only builds inputs: embedding matrices E, the equal-size cluster-to-token table C2T,
the centroids C (and their INT4 packing), hidden vectors h and target ids.  It performs none of
the head's own arithmetic (scoring, selection, gathering, logits, sampling, Monte Carlo), so both
the CUDA path and the CPU oracle can take their inputs from here.

Recipe (the pages give no data; these shapes follow the heads the FlashHead pages evaluate —
Llama-3.2-1B with hidden size 2048 and a 128,256-token vocabulary, c = 8016 clusters and p = 512
probes as the default configuration, plus Gemma-3-1B and Qwen-3-0.6B shapes):

* c unit centroids uniform on the sphere S^{d-1}.
* b = v/c tokens per centroid: token = centroid + N(0, sigma^2 I) noise, L2-normalised, then scaled
  by a norm drawn from U(0.8, 1.2).  A fraction ``heavy_frac`` of the token ids (chosen by a seeded
  permutation) has its norm multiplied by ``heavy_mult`` to mimic frequent tokens.
* Token ids are a seeded random permutation of the generation order; cluster k's row of C2T lists
  the ids of the tokens generated from centroid k, sorted ascending, so every cluster holds exactly
  b tokens (the equal-size constraint of FlashHead notes, Module 1) and C2T flattened is a
  permutation of 0..v-1.
* The stored centroid C[k] is the L2-normalised mean of the *stored* rows of cluster k (the centroid
  update of FlashHead notes, Eq. 5), computed in float64 and rounded to the storage dtype.  This is
  the offline index construction of the synthetic workload; no k-means iterations are run.
* Queries h ~ N(0, I/d) * scale, rounded to the storage dtype.

BF16 values are stored as uint16 bit patterns rounded to nearest even from float32.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

# ----------------------------------------------------------------------------- bf16 helpers


def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bit patterns.

    Inputs are finite by construction here; NaN handling is not needed."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def f32_from_bf16(u: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32)


def stored_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a stored array (float32 values or bf16 bit patterns)."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    return f32_from_bf16(a).astype(np.float64)


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float values to the storage dtype ("f32" -> float32, "bf16" -> uint16 patterns)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    return bf16_from_f32(np.asarray(x, dtype=np.float32))


# ----------------------------------------------------------------------------- configurations


@dataclasses.dataclass(frozen=True)
class HeadConfig:
    """Shapes and generator parameters of one synthetic head."""

    name: str
    v: int
    d: int
    c: int
    p: int
    dtype: str                 # "f32" or "bf16"
    noise: float               # sigma * sqrt(d) of the token noise
    heavy_frac: float          # fraction of tokens with norm * heavy_mult
    heavy_mult: float
    h_scale: float             # h ~ N(0, I/d) * h_scale
    data_seed: int
    query_seed: int
    tau: float = 1.0
    int4: bool = False

    @property
    def b(self) -> int:
        return self.v // self.c


CONFIGS = {
    # tiny greedy case: fp32, v=4096, d=256, 64 clusters of 64, 8 probes
    "tiny": HeadConfig("tiny", v=4096, d=256, c=64, p=8, dtype="f32", noise=0.3,
                       heavy_frac=0.0, heavy_mult=1.0, h_scale=1.0,
                       data_seed=1000, query_seed=1001),
    # Llama-3.2-1B-shaped head (greedy and sampling, tau = 0.8 for sampling)
    "llama": HeadConfig("llama", v=128256, d=2048, c=8016, p=512, dtype="bf16", noise=0.5,
                        heavy_frac=0.02, heavy_mult=3.0, h_scale=8.0,
                        data_seed=2000, query_seed=2001, tau=0.8),
    # Gemma-3-1B-shaped head with INT4 Stage-1 centroids
    "gemma": HeadConfig("gemma", v=262144, d=1152, c=16384, p=1024, dtype="bf16", noise=0.5,
                        heavy_frac=0.02, heavy_mult=3.0, h_scale=8.0,
                        data_seed=4000, query_seed=4001, int4=True),
    # Qwen-3-0.6B-shaped head for the Monte Carlo marginal, tau = 1.0
    "qwen": HeadConfig("qwen", v=151936, d=1024, c=9496, p=512, dtype="bf16", noise=0.5,
                       heavy_frac=0.02, heavy_mult=3.0, h_scale=8.0,
                       data_seed=5000, query_seed=5001, tau=1.0),
}

SAMPLE_SEED = 0xF1A54EAD      # Philox seed of the sampling workload
MC_SEED = 5000                 # Philox seed of the Monte Carlo workload
MC_TARGET_SEED = 5002


def scaled(cfg: HeadConfig, v: int, c: int, d: int | None = None, p: int | None = None,
           name: str | None = None) -> HeadConfig:
    """A smaller head with the same generator recipe (used for fast checks)."""
    return dataclasses.replace(cfg, v=v, c=c, d=d if d is not None else cfg.d,
                               p=p if p is not None else cfg.p,
                               name=name or f"{cfg.name}-v{v}-c{c}")


# ----------------------------------------------------------------------------- index


@dataclasses.dataclass
class Index:
    cfg: HeadConfig
    E: np.ndarray          # v x d, float32 or uint16 (bf16 patterns)
    C: np.ndarray          # c x d, same dtype
    C2T: np.ndarray        # c x b, int32
    C_q4: np.ndarray | None = None      # c x d/2 uint8
    C_scales: np.ndarray | None = None  # c x d/32 uint16 (bf16 patterns)

    @property
    def v(self):
        return self.cfg.v

    @property
    def d(self):
        return self.cfg.d

    @property
    def c(self):
        return self.cfg.c

    @property
    def b(self):
        return self.cfg.b


def make_index(cfg: HeadConfig, chunk_clusters: int = 2048) -> Index:
    """Build E, C, C2T (and the INT4 packing of C when cfg.int4) for one configuration."""
    v, d, c = cfg.v, cfg.d, cfg.c
    if v % c:
        raise ValueError("v must be a multiple of c (equal-size clusters)")
    b = v // c
    rng = np.random.Generator(np.random.PCG64(cfg.data_seed))

    # 1. unit centroids uniform on the sphere
    cent = rng.standard_normal((c, d), dtype=np.float32)
    cent /= np.linalg.norm(cent, axis=1, keepdims=True)

    # 2. token ids: generation index g = k*b + j receives id perm[g]
    perm = rng.permutation(v).astype(np.int64)
    # 3. norms and the heavy-token subset (chosen among token ids)
    norms = rng.uniform(0.8, 1.2, size=v).astype(np.float32)   # indexed by token id
    n_heavy = int(math.floor(cfg.heavy_frac * v))
    if n_heavy:
        heavy_ids = rng.permutation(v)[:n_heavy]
        norms[heavy_ids] *= np.float32(cfg.heavy_mult)

    sigma = np.float32(cfg.noise / math.sqrt(d))
    E = np.empty((v, d), dtype=np.float32 if cfg.dtype == "f32" else np.uint16)
    for k0 in range(0, c, chunk_clusters):
        k1 = min(c, k0 + chunk_clusters)
        n = (k1 - k0) * b
        tok = np.repeat(cent[k0:k1], b, axis=0)
        tok += rng.standard_normal((n, d), dtype=np.float32) * sigma
        tok /= np.linalg.norm(tok, axis=1, keepdims=True)
        ids = perm[k0 * b:k1 * b]
        tok *= norms[ids][:, None]
        E[ids] = store(tok, cfg.dtype)

    C2T = np.sort(perm.reshape(c, b), axis=1).astype(np.int32)

    # 4. centroids: normalised mean of the stored rows of each cluster, in float64
    C = np.empty((c, d), dtype=E.dtype)
    for k0 in range(0, c, chunk_clusters):
        k1 = min(c, k0 + chunk_clusters)
        rows = stored_to_f64(E[C2T[k0:k1].reshape(-1)], cfg.dtype).reshape(k1 - k0, b, d)
        mean = rows.mean(axis=1)
        mean /= np.linalg.norm(mean, axis=1, keepdims=True)
        C[k0:k1] = store(mean.astype(np.float32) if cfg.dtype == "bf16" else mean, cfg.dtype)

    idx = Index(cfg, E, C, C2T)
    if cfg.int4:
        idx.C_q4, idx.C_scales = quantize_int4_g32(stored_to_f64(C, cfg.dtype))
    return idx


def quantize_int4_g32(x: np.ndarray):
    """Symmetric 4-bit quantisation with one BF16 scale per group of 32 columns.

    scale = bf16(float32(max|x| / 7)); q = clamp(round_half_even(x / scale), -8, 7), q = 0 where
    scale == 0.  Packing: two values per byte, the low nibble holds the even column, two's complement.
    Returns (packed uint8 [rows, d/2], scales uint16 bf16 patterns [rows, d/32])."""
    rows, d = x.shape
    if d % 32:
        raise ValueError("d must be a multiple of 32 for INT4 groups")
    g = x.reshape(rows, d // 32, 32)
    amax = np.abs(g).max(axis=2)
    scales_bits = bf16_from_f32((amax / 7.0).astype(np.float32))
    scale = f32_from_bf16(scales_bits).astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(scale[:, :, None] > 0, np.rint(g / scale[:, :, None]), 0.0)
    q = np.clip(q, -8, 7).astype(np.int8).reshape(rows, d)
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return np.ascontiguousarray(packed), np.ascontiguousarray(scales_bits)


def shift_centroids(C: np.ndarray, t: float) -> np.ndarray:
    """C - t * mean(C) (rows), in float64: the offline reparameterisation of the centroids before
    INT4 quantisation.  Every Stage-1 score of a query moves by the same t * mean(C)·h, so the top-p
    set and softmax(s/τ) are unchanged in exact arithmetic; only the quantisation error changes."""
    C = np.asarray(C, dtype=np.float64)
    return C - t * C.mean(axis=0, keepdims=True)


def anisotropic_centroids(c: int, d: int, common: float, seed: int) -> np.ndarray:
    """Unit centroids normalise(u + common·sqrt(d)·m) with u ~ N(0, I) and one fixed unit direction m
    (float64): stand-ins for real head centroids, which share a dominant mean component, for the
    centroid-shift study of INT4 Stage 1."""
    rng = np.random.Generator(np.random.PCG64(seed))
    m = rng.standard_normal(d)
    m /= np.linalg.norm(m)
    u = rng.standard_normal((c, d)) + common * math.sqrt(d) * m[None, :]
    return u / np.linalg.norm(u, axis=1, keepdims=True)


# ----------------------------------------------------------------------------- coarse-fine head inputs
# The coarse-fine head (page "Fast LM Head via Coarse-Fine Decomposition and Tile-Wise Weight
# Clustering", abstract) reads E through a per-tile codebook and an index map.  These helpers build
# that offline index for a synthetic E; the head's own arithmetic (look-up tables, coarse scores,
# selection, exact logits) is not here.

CF_TILE_W = 2        # columns per tile
CF_CODES = 16        # codebook entries per tile (4-bit codes)
CF_TOPK = 1024       # candidates that get exact logits
CF_FIT_TOKENS = 16384  # tokens the codebooks are fitted on


def cf_pack_codes(codes: np.ndarray) -> np.ndarray:
    """Pack a (v, T) array of 4-bit codes (T % 8 == 0) into the index-map layout the library reads:
    uint32 words [T/8, v], word (g, u) holding the codes of tiles 8g..8g+7 of token u, tile 8g+j in
    bits 4j..4j+3."""
    codes = np.asarray(codes, dtype=np.uint32)
    v, T = codes.shape
    if T % 8:
        raise ValueError("the number of tiles must be a multiple of 8")
    g = codes.reshape(v, T // 8, 8)
    words = np.zeros((v, T // 8), dtype=np.uint32)
    for j in range(8):
        words |= (g[:, :, j] & 0xF) << np.uint32(4 * j)
    return np.ascontiguousarray(words.T)


def cf_index(E: np.ndarray, dtype: str, w: int = CF_TILE_W, K: int = CF_CODES, iters: int = 4,
             seed: int = 7000, fit_tokens: int = CF_FIT_TOKENS, chunk: int = 8192, device=None):
    """Offline tile-wise k-means of the embedding rows: E's columns are cut into T = d/w tiles; per
    tile, K centres are fitted by `iters` Lloyd iterations (float32) on the sub-rows of `fit_tokens`
    tokens drawn by a seeded permutation (all tokens when v is smaller), starting from K distinct
    ones of them; an empty centre keeps its old value.  Every token then gets the code of its nearest
    centre.  Returns (codebooks float32 [T, K, w], packed codes uint32 [T/8, v]).  The arithmetic runs
    in torch on `device` (default: the GPU when there is one); the index it returns is an input, read
    as stored by the library and by the oracle alike."""
    import torch
    if device is None:
        device = "cuda" if torch.cuda.is_available() else "cpu"
    X = torch.from_numpy(stored_to_f64(E, dtype).astype(np.float32)).to(device)
    v, d = X.shape
    if d % (8 * w):
        raise ValueError("d must be a multiple of 8 tiles")
    T = d // w
    rng = np.random.Generator(np.random.PCG64(seed))
    Xt = X.reshape(v, T, w).permute(1, 0, 2).contiguous()                # (T, v, w)
    fit = torch.from_numpy(rng.permutation(v)[:min(v, fit_tokens)].astype(np.int64)).to(device)
    Xf = Xt[:, fit, :].contiguous()
    cb = Xf[:, :K, :].clone()                                            # (T, K, w)

    def assign(Xs, cb):
        n = Xs.shape[1]
        codes = torch.empty((T, n), dtype=torch.int64, device=device)
        for u0 in range(0, n, chunk):
            x = Xs[:, u0:u0 + chunk, :]
            dist = torch.zeros((T, x.shape[1], K), device=device)
            for i in range(w):
                dist += (x[:, :, None, i] - cb[:, None, :, i]) ** 2
            codes[:, u0:u0 + chunk] = dist.argmin(-1)
        return codes

    for _ in range(iters):
        codes = assign(Xf, cb)
        sums = torch.zeros((T, K, w), device=device).scatter_add_(1, codes[:, :, None].expand(-1, -1, w), Xf)
        cnt = torch.zeros((T, K), device=device).scatter_add_(1, codes, torch.ones(codes.shape, device=device))
        nz = cnt > 0
        cb = torch.where(nz[:, :, None], sums / cnt.clamp(min=1)[:, :, None], cb)
    codes = assign(Xt, cb)
    return (np.ascontiguousarray(cb.cpu().numpy().astype(np.float32)),
            cf_pack_codes(codes.T.cpu().numpy()))


# ----------------------------------------------------------------------------- queries


def make_queries(cfg: HeadConfig, n: int, seed: int | None = None) -> np.ndarray:
    """n hidden vectors h ~ N(0, I/d) * h_scale, rounded to the storage dtype."""
    rng = np.random.Generator(np.random.PCG64(cfg.query_seed if seed is None else seed))
    h = rng.standard_normal((n, cfg.d)) / math.sqrt(cfg.d) * cfg.h_scale
    return store(h.astype(np.float32), cfg.dtype)


def make_targets(v: int, n: int, t: int, seed: int = MC_TARGET_SEED) -> np.ndarray:
    """n x t token ids drawn uniformly from [0, v)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, v, size=(n, t)).astype(np.int32)


def random_index(v: int, d: int, c: int, seed: int, dtype: str = "f32") -> Index:
    """A small unstructured index: E ~ N(0, 1/d) rows, random equal-size C2T, C = unit means.
    Used for edge cases where clustered structure is not wanted."""
    b = v // c
    rng = np.random.Generator(np.random.PCG64(seed))
    E = store(rng.standard_normal((v, d)).astype(np.float32) / np.float32(math.sqrt(d)), dtype)
    C2T = np.sort(rng.permutation(v).reshape(c, b), axis=1).astype(np.int32)
    rows = stored_to_f64(E[C2T.reshape(-1)], dtype).reshape(c, b, d).mean(axis=1)
    rows /= np.linalg.norm(rows, axis=1, keepdims=True)
    C = store(rows.astype(np.float32), dtype)
    cfg = HeadConfig(f"random-{v}-{d}-{c}", v=v, d=d, c=c, p=min(c, 4), dtype=dtype, noise=0.0,
                     heavy_frac=0.0, heavy_mult=1.0, h_scale=1.0, data_seed=seed,
                     query_seed=seed + 1)
    return Index(cfg, E, C, C2T)


# ----------------------------------------------------------------------------- index-builder inputs

KMEANS_SEED = 6000


def planted_embeddings(c: int, b: int, d: int, spread: float, seed: int = KMEANS_SEED):
    """Inputs for the equal-size k-means builder: v = c*b BF16 rows around c random directions,
    exactly b per direction (noise N(0, spread^2/d) per column, norms from U(0.5, 2)), token ids
    shuffled.  Returns (E as BF16 patterns [v, d], the generating direction of each token [v])."""
    rng = np.random.Generator(np.random.PCG64(seed))
    dirs = rng.standard_normal((c, d))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    lab = np.repeat(np.arange(c), b)
    X = dirs[lab] + spread * rng.standard_normal((c * b, d)) / math.sqrt(d)
    X *= rng.uniform(0.5, 2.0, size=(c * b, 1))
    perm = rng.permutation(c * b)
    return bf16_from_f32(X[perm].astype(np.float32)), lab[perm].astype(np.int32)


def init_tokens(v: int, c: int, seed: int = KMEANS_SEED + 1) -> np.ndarray:
    """c distinct token ids drawn by a seeded permutation: the builder's initial centres."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.permutation(v)[:c].astype(np.int32)
