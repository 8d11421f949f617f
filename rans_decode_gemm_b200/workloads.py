"""Seeded synthetic workloads shaped like the pages' layers.

This module only draws random numbers and lays them out in the weights'
storage formats (packed int4 nibbles, bf16 bits, e4m3 codes, bf16/fp32
scales, bf16 activations).  It holds none of the coding method's arithmetic,
so both the CUDA path and the CPU oracle may take their inputs from it.

The pages measure on real Llama-3 / Qwen / Mixtral checkpoints, which are not
available here; these distributions stand in for them:

  tiny_int4    512x512 int4 codes clip(rint(N(0, 1.5)), -8, 7), per-row bf16
               scale U[0.005, 0.02], 128x32 tiles, X 1x512 N(0,1), seed 0
  bf16_4096    4096x4096 bf16(N(0, 0.02)), 128x64 tiles, X Mx4096, M in
               {1, 16, 128}, seed 1
  llama8b_mlp  gate/up 14336x4096 and down 4096x14336, bf16 N(0, 0.02) with a
               uniform 0.1% of entries (drawn without replacement) multiplied
               by 20 before rounding to bf16, 128x64 tiles, seed 2
  int4_70b     28672x8192 int4 codes clip(rint(Laplace(0, 0.9)), -8, 7),
               group-128 bf16 scales U[0.003, 0.03], 256x64 tiles, seed 3
  fp8_405b     53248x16384 e4m3 codes of w / (amax_n / 448), w ~ N(0, 0.02),
               per-row fp32 scale amax_n / 448, 128x128 tiles, seed 4
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

INT4, BF16_SPLIT, FP8_E4M3, INT4_PAIRS, INT8, FP4_E2M1, FP4_PAIRS, BF16_WHOLE = 0, 1, 2, 3, 4, 5, 6, 7
SCALE_NONE, SCALE_ROW_BF16, SCALE_ROW_F32, SCALE_GROUP_BF16 = 0, 1, 2, 3


@dataclass
class Config:
    name: str
    dtype: int
    N: int
    K: int
    tile_n: int
    tile_k: int
    scale_kind: int
    group_k: int
    Ms: list
    seed: int
    matrices: list = field(default_factory=lambda: [("w", None, None)])


CONFIGS = {
    "tiny_int4": Config("tiny_int4", INT4, 512, 512, 128, 32, SCALE_ROW_BF16, 0, [1], 0),
    "bf16_4096": Config("bf16_4096", BF16_SPLIT, 4096, 4096, 128, 64, SCALE_NONE, 0,
                        [1, 16, 128], 1),
    "llama8b_mlp": Config("llama8b_mlp", BF16_SPLIT, 14336, 4096, 128, 64, SCALE_NONE, 0,
                          [1, 8, 32, 128, 512], 2,
                          [("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336)]),
    "int4_70b": Config("int4_70b", INT4, 28672, 8192, 256, 64, SCALE_GROUP_BF16, 128,
                       [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024], 3),
    "fp8_405b": Config("fp8_405b", FP8_E4M3, 53248, 16384, 128, 128, SCALE_ROW_F32, 0,
                       [1, 4, 16, 64, 256, 2048], 4),
    # int8 (absmax per row) of a Llama-8B-shaped MLP projection
    "int8_8b": Config("int8_8b", INT8, 14336, 4096, 128, 64, SCALE_ROW_F32, 0, [1, 16, 128], 5),
    # fp4 e2m1 (absmax per row, nearest grid value) of the same shape
    "fp4_8b": Config("fp4_8b", FP4_E2M1, 14336, 4096, 128, 64, SCALE_ROW_F32, 0, [1, 16, 128], 6),
}

# e2m1 codes 0..7 in increasing value: 0, 0.5, 1, 1.5, 2, 3, 4, 6 (the sign is bit 3)
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """int8 codes in [-8, 7] (row-major, even count per row) -> packed nibbles,
    element k even in the low nibble."""
    c = np.ascontiguousarray(codes, dtype=np.int8).reshape(-1).view(np.uint8) & 0xF
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def _rows_chunks(N: int, K: int, budget: int = 1 << 24):
    step = max(1, budget // max(1, K))
    for r0 in range(0, N, step):
        yield r0, min(N, r0 + step)


def make_weights(cfg: Config, matrix: int = 0, N: int | None = None, K: int | None = None):
    """Weights of one matrix of `cfg` (optionally at a smaller N x K with the same
    distribution).  Returns dict(w=packed storage ndarray, scales=ndarray|None,
    N=, K=)."""
    name, mN, mK = cfg.matrices[matrix]
    N = N if N is not None else (mN or cfg.N)
    K = K if K is not None else (mK or cfg.K)
    rng = np.random.default_rng([cfg.seed, matrix])
    scales = None
    if cfg.dtype == INT4:
        w = np.empty(N * K // 2, np.uint8)
        for r0, r1 in _rows_chunks(N, K):
            if cfg.name == "int4_70b":
                v = rng.laplace(0.0, 0.9, size=(r1 - r0, K))
            else:
                v = rng.standard_normal((r1 - r0, K)) * 1.5
            codes = np.clip(np.rint(v), -8, 7).astype(np.int8)
            w[r0 * K // 2:r1 * K // 2] = pack_int4(codes)
        if cfg.scale_kind == SCALE_ROW_BF16:
            scales = to_bf16_bits(rng.uniform(0.005, 0.02, size=N))
        elif cfg.scale_kind == SCALE_GROUP_BF16:
            scales = to_bf16_bits(rng.uniform(0.003, 0.03, size=(N, K // cfg.group_k)))
    elif cfg.dtype == BF16_SPLIT:
        w = np.empty(N * K, np.uint16)
        n_out = int(round(0.001 * N * K)) if cfg.name == "llama8b_mlp" else 0
        outliers = np.sort(rng.choice(N * K, size=n_out, replace=False)) if n_out else None
        for r0, r1 in _rows_chunks(N, K):
            v = (rng.standard_normal((r1 - r0, K)) * 0.02).astype(np.float32).reshape(-1)
            if outliers is not None:
                lo, hi = np.searchsorted(outliers, [r0 * K, r1 * K])
                v[outliers[lo:hi] - r0 * K] *= 20.0
            w[r0 * K:r1 * K] = to_bf16_bits(v)
    elif cfg.dtype == FP4_E2M1:
        w = np.empty(N * K // 2, np.uint8)
        scales = np.empty(N, np.float32)
        for r0, r1 in _rows_chunks(N, K):
            v = (rng.standard_normal((r1 - r0, K)) * 0.02).astype(np.float32)
            s = (np.abs(v).max(axis=1) / 6.0).astype(np.float32)
            scales[r0:r1] = s
            a = np.abs(v / s[:, None])
            mag = np.abs(a[..., None] - _E2M1_GRID).argmin(axis=-1).astype(np.uint8)
            codes = mag | (np.signbit(v).astype(np.uint8) << 3)
            codes[mag == 0] = 0                       # +0 for values that round to zero
            c = codes.reshape(-1)
            w[r0 * K // 2:r1 * K // 2] = c[0::2] | (c[1::2] << 4)
    elif cfg.dtype == INT8:
        w = np.empty(N * K, np.uint8)
        scales = np.empty(N, np.float32)
        for r0, r1 in _rows_chunks(N, K):
            v = (rng.standard_normal((r1 - r0, K)) * 0.02).astype(np.float32)
            s = (np.abs(v).max(axis=1) / 127.0).astype(np.float32)
            scales[r0:r1] = s
            q = np.clip(np.rint(v / s[:, None]), -127, 127).astype(np.int8)
            w[r0 * K:r1 * K] = q.view(np.uint8).reshape(-1)
    else:
        w = np.empty(N * K, np.uint8)
        scales = np.empty(N, np.float32)
        for r0, r1 in _rows_chunks(N, K):
            v = (rng.standard_normal((r1 - r0, K)) * 0.02).astype(np.float32)
            amax = np.abs(v).max(axis=1)
            s = (amax / 448.0).astype(np.float32)
            scales[r0:r1] = s
            q = torch.from_numpy(v / s[:, None]).to(torch.float8_e4m3fn)
            w[r0 * K:r1 * K] = q.view(torch.uint8).numpy().reshape(-1)
    return {"w": w, "scales": scales, "N": N, "K": K}


def make_x(cfg: Config, M: int, K: int | None = None, stream: int = 0) -> np.ndarray:
    """Activations X (M x K) as bf16 bits, N(0, 1)."""
    K = K if K is not None else cfg.K
    rng = np.random.default_rng([cfg.seed, 1000 + stream, M])
    return to_bf16_bits(rng.standard_normal((M, K))).reshape(M, K)
