"""Seeded synthetic inputs for the QuaRot hot path.

This module holds random numbers and shapes only -- none of the method's
arithmetic.  The same arrays feed the CUDA library and the CPU oracle.

The pages measure on LLaMA-2 layers fed with real text (WikiText-2 and
zero-shot suites); neither the weights nor the data are available here, so
these generators stand in for them with the shapes of LLaMA-2-7B and -70B
linear layers and heavy-tailed activations with a few outlier channels (the
QuaRot summary: outliers are individual channels much larger than the rest;
DuQuant Knowl 4: massive outliers reach 100-1400 in magnitude).

Every array is drawn in fp64 from numpy's default_rng, scaled, then rounded to
fp16 (asserted finite).  Seeds: inputs use seed = 1000 + workload id, signs
use seed + 1, weights seed + 2, sampled rows seed + 3.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

_CHUNK_ELEMS = 1 << 25  # generate big tensors in row chunks of ~32M values


@dataclasses.dataclass(frozen=True)
class Linear:
    wid: int
    name: str
    M: int                  # tokens
    K: int                  # input channels
    Ns: tuple               # output channels of the linears that read this activation
    had_block: int          # 0 = full Hadamard of size K, 128 = I (x) H_128
    group: int              # 0 = per-token / per-channel scale, 128 = group-wise
    dist: str               # activation distribution
    outlier_channels: Optional[tuple] = None
    outlier_frac: float = 0.0
    outlier_count: int = 0
    outlier_scale: float = 1.0
    w_std: float = 0.02

    @property
    def seed(self) -> int:
        return 1000 + self.wid


@dataclasses.dataclass(frozen=True)
class KVCache:
    wid: int
    name: str
    B: int
    T: int
    Hkv: int
    D: int
    Hq: int
    k_outliers_per_head: int
    k_outlier_scale: float

    @property
    def seed(self) -> int:
        return 1000 + self.wid


TINY = Linear(1, "tiny linear 16x256 -> 256", 16, 256, (256,), 0, 0, "normal",
              outlier_channels=(3, 77, 140, 201), outlier_scale=50.0, w_std=0.02)
LLAMA2_7B = Linear(2, "llama2-7b prefill 2048 tok, K 4096 -> N 4096 / 11008", 2048, 4096,
                   (4096, 11008), 0, 0, "student_t3", outlier_frac=0.01, outlier_scale=20.0,
                   w_std=0.02)
DOWN_PROJ = Linear(3, "llama2-7b down-proj 2048 tok, K 11008 (I_86 x H_128, g128) -> N 4096",
                   2048, 11008, (4096,), 128, 128, "laplace", outlier_count=4,
                   outlier_scale=500.0, w_std=0.02)
LLAMA2_70B = Linear(4, "llama2-70b prefill 32768 tok, K 8192 (H_8192) -> N 28672", 32768, 8192,
                    (28672,), 0, 0, "student_t3", outlier_frac=0.005, outlier_scale=30.0,
                    w_std=0.015)
KV_70B = KVCache(5, "llama2-70b GQA INT4 KV cache B64 T2048 Hkv8 D128, decode 64 q-heads",
                 64, 2048, 8, 128, 64, 2, 15.0)

LINEARS = {w.wid: w for w in (TINY, LLAMA2_7B, DOWN_PROJ, LLAMA2_70B)}


def _to_f16(a: np.ndarray) -> np.ndarray:
    h = a.astype(np.float16)
    if not np.all(np.isfinite(h)):
        raise ValueError("synthetic input overflowed fp16")
    return h


def _draw(rng: np.random.Generator, dist: str, shape) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(shape)
    if dist == "student_t3":
        return rng.standard_t(3.0, shape)
    if dist == "laplace":
        return rng.laplace(0.0, 1.0, shape)
    raise ValueError(dist)


def outlier_channels(w: Linear) -> np.ndarray:
    if w.outlier_channels is not None:
        return np.asarray(w.outlier_channels, np.int64)
    count = w.outlier_count if w.outlier_count else int(round(w.outlier_frac * w.K))
    rng = np.random.default_rng(w.seed + 4)
    return np.sort(rng.choice(w.K, size=count, replace=False))


def activations(w: Linear, rows: Optional[int] = None) -> np.ndarray:
    """fp16 [rows or M, K]; the first `rows` rows of the full workload's stream."""
    M = w.M if rows is None else rows
    rng = np.random.default_rng(w.seed)
    ch = outlier_channels(w)
    out = np.empty((M, w.K), np.float16)
    step = max(1, _CHUNK_ELEMS // w.K)
    for r0 in range(0, M, step):
        r1 = min(M, r0 + step)
        x = _draw(rng, w.dist, (r1 - r0, w.K))
        x[:, ch] *= w.outlier_scale
        out[r0:r1] = _to_f16(x)
    return out


def weights(w: Linear, N: int, rows: Optional[int] = None) -> np.ndarray:
    """fp16 [N or rows, K] drawn N(0, w_std)."""
    R = N if rows is None else rows
    rng = np.random.default_rng(w.seed + 2 + 7919 * N)
    out = np.empty((R, w.K), np.float16)
    step = max(1, _CHUNK_ELEMS // w.K)
    for r0 in range(0, R, step):
        r1 = min(R, r0 + step)
        out[r0:r1] = _to_f16(rng.normal(0.0, w.w_std, (r1 - r0, w.K)))
    return out


def signs(K: int, seed: int) -> np.ndarray:
    """Random +-1 vector (int8) for the randomized Hadamard."""
    rng = np.random.default_rng(seed + 1)
    return rng.choice(np.array([-1, 1], np.int8), size=K)


def sample_rows(n_total: int, n_sample: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed + 3)
    n = min(n_total, n_sample)
    return np.sort(rng.choice(n_total, size=n, replace=False))


def kv_inputs(c: KVCache, batch: Optional[int] = None):
    """(k, v, q, signs): k, v fp16 [B, T, Hkv, D]; q fp16 [B, Hq, D]; signs int8 [Hkv, D]."""
    B = c.B if batch is None else batch
    rng = np.random.default_rng(c.seed)
    k = np.empty((B, c.T, c.Hkv, c.D), np.float16)
    v = np.empty((B, c.T, c.Hkv, c.D), np.float16)
    ch = np.stack([np.sort(np.random.default_rng(c.seed + 4 + h).choice(
        c.D, size=c.k_outliers_per_head, replace=False)) for h in range(c.Hkv)])
    for b in range(B):
        kb = rng.standard_normal((c.T, c.Hkv, c.D))
        for h in range(c.Hkv):
            kb[:, h, ch[h]] *= c.k_outlier_scale
        k[b] = _to_f16(kb)
        v[b] = _to_f16(rng.standard_normal((c.T, c.Hkv, c.D)))
    q = _to_f16(np.random.default_rng(c.seed + 5).standard_normal((B, c.Hq, c.D)))
    s = np.stack([signs(c.D, c.seed + 10 * h) for h in range(c.Hkv)])
    return k, v, q, s


def random_f16(shape, seed: int, scale: float = 1.0, dist: str = "normal") -> np.ndarray:
    """Generic seeded fp16 tensor for edge-case tests."""
    rng = np.random.default_rng(seed)
    return _to_f16(_draw(rng, dist, shape) * scale)


def random_codes(shape, seed: int) -> np.ndarray:
    """Uniform INT4 codes in [-8, 7] (int8 container)."""
    rng = np.random.default_rng(seed)
    return rng.integers(-8, 8, size=shape, dtype=np.int8)


def names() -> List[str]:
    return [w.name for w in LINEARS.values()] + [KV_70B.name]
