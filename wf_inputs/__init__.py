"""Seeded synthetic inputs for the Wave Forcing round-attention path.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark. It holds workload shapes and random draws only: no attention, no
rotary embedding, no paging arithmetic. Every random value is drawn in float64
from ``numpy.random.default_rng(SeedSequence([...]))`` and then rounded once
(round-to-nearest-even) to the working dtype, so both sides of a parity test see
the same bits.

Workload shapes follow "Wave Forcing: Towards Speed-of-Light Streaming Video
Generation":
  * chunk = 3 latent frames of a 30x52 patch grid = 4680 tokens (the 832x480
    Wan2.1 setting, and the 95,846,400-byte one-layer K+V copy of Table 8,
    which is 4680 tokens x 5120 hidden x 2 tensors x 2 bytes);
  * 1.3B: 12 heads x 128, 30 layers; 14B: 40 heads x 128 (Table 11);
  * S = 4 or 5 denoising stages plus the store stage (Figure 1, Table 3).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = ["WorkloadConfig", "CONFIGS", "draw_normal", "draw_round_inputs",
           "draw_page_order", "draw_k_outlier_mask"]

# Tensor ids mixed into the seed sequence.
_T_Q, _T_K, _T_V, _T_KMASK = 0, 1, 2, 3


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    num_stages: int          # S denoising stages; the store is slot S
    chunk_tokens: int        # C
    num_heads: int
    head_dim: int
    anchor_chunks: int       # 0 or 1
    history_chunks: int      # H
    page_tokens: int         # P
    num_layers: int
    dtype: str               # "bf16" or "f32"
    rope: int                # 0 off, 1 3D rotary
    frames_per_chunk: int
    grid_h: int
    grid_w: int
    rope_split: tuple = (44, 42, 42)
    rope_base: float = 10000.0
    k_outlier_frac: float = 0.0   # fraction of K rows scaled
    k_outlier_scale: float = 1.0  # by this power of two
    rounds: int = 1               # rounds run by the workload
    seed: int = 0
    mask: str = "wf"              # "wf" (M_WF) or "rf" (bidirectional live window)

    @property
    def pages_per_chunk(self) -> int:
        return -(-self.chunk_tokens // self.page_tokens)

    @property
    def num_slots(self) -> int:
        return self.num_stages + 1

    def steady_round(self) -> int:
        """First round in which every slot is live and the history is full."""
        return self.num_stages + self.anchor_chunks + self.history_chunks

    def replace(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, WorkloadConfig] = {
    # S=2 + store, chunk 128, 2 heads x 64, anchor 1, history 1, page 64,
    # fp32, attention only (no rotary); steady at round 4.
    "tiny_f32": WorkloadConfig(
        name="tiny_f32", num_stages=2, chunk_tokens=128, num_heads=2, head_dim=64,
        anchor_chunks=1, history_chunks=1, page_tokens=64, num_layers=1, dtype="f32",
        rope=0, frames_per_chunk=1, grid_h=8, grid_w=16, rounds=5, seed=0),
    # Wan2.1-1.3B-shaped layer: S=4 + store, 4680 tokens, 12 x 128, history 2.
    "wan13b_bf16": WorkloadConfig(
        name="wan13b_bf16", num_stages=4, chunk_tokens=4680, num_heads=12, head_dim=128,
        anchor_chunks=1, history_chunks=2, page_tokens=128, num_layers=1, dtype="bf16",
        rope=1, frames_per_chunk=3, grid_h=30, grid_w=52, rounds=8, seed=0),
    # 5-step variant: S=5 + store, history 3, 5% of K rows scaled x8.
    "wan13b_5step_bf16": WorkloadConfig(
        name="wan13b_5step_bf16", num_stages=5, chunk_tokens=4680, num_heads=12,
        head_dim=128, anchor_chunks=1, history_chunks=3, page_tokens=128, num_layers=1,
        dtype="bf16", rope=1, frames_per_chunk=3, grid_h=30, grid_w=52,
        k_outlier_frac=0.05, k_outlier_scale=8.0, rounds=10, seed=0),
    # 14B-scale layer: 40 heads x 128.
    "wan14b_bf16": WorkloadConfig(
        name="wan14b_bf16", num_stages=4, chunk_tokens=4680, num_heads=40, head_dim=128,
        anchor_chunks=1, history_chunks=2, page_tokens=128, num_layers=1, dtype="bf16",
        rope=1, frames_per_chunk=3, grid_h=30, grid_w=52, rounds=8, seed=0),
    # Streaming rollout: 30 layers x 200 rounds, sliding 2-chunk history.
    "stream_13b_bf16": WorkloadConfig(
        name="stream_13b_bf16", num_stages=4, chunk_tokens=4680, num_heads=12,
        head_dim=128, anchor_chunks=1, history_chunks=2, page_tokens=128, num_layers=30,
        dtype="bf16", rope=1, frames_per_chunk=3, grid_h=30, grid_w=52, rounds=200,
        seed=0),
}


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(x) for x in key]))


def _round_to(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values once, to nearest-even, to the working dtype.

    Returns float32 for "f32" and a uint16 array of bf16 bit patterns for "bf16".
    """
    if dtype == "f32":
        return x64.astype(np.float32)
    if dtype == "bf16":
        f = x64.astype(np.float32)            # fp64 -> fp32 is exact for N(0,1)
        u = f.view(np.uint32).astype(np.uint64)  # draws up to 2^-24 relative;
        # round-to-nearest-even on the upper 16 bits of the fp32 pattern.
        lsb = (u >> 16) & 1
        u = (u + 0x7FFF + lsb) >> 16
        return u.astype(np.uint16)
    raise ValueError(dtype)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def draw_normal(shape, dtype: str, *key: int) -> np.ndarray:
    x = _rng(*key).standard_normal(size=shape)
    return _round_to(x, dtype)


def draw_k_outlier_mask(cfg: WorkloadConfig, rnd: int, layer: int, slot: int) -> Optional[np.ndarray]:
    """Bernoulli(k_outlier_frac) per (token, head) of one slot's K, or None."""
    if cfg.k_outlier_frac <= 0.0:
        return None
    u = _rng(cfg.seed, rnd, layer, slot, _T_KMASK).random(size=(cfg.chunk_tokens, cfg.num_heads))
    return u < cfg.k_outlier_frac


def draw_round_inputs(cfg: WorkloadConfig, rnd: int, layer: int, slots=None,
                      seed: Optional[int] = None):
    """Pre-rotary q, k, v of every slot for one (round, layer).

    Returns three arrays shaped [S+1][C][heads][head_dim] in the working dtype
    (float32, or uint16 bf16 bit patterns). Rows of slots not listed in
    ``slots`` are zero. Slot s of round k holds chunk k - s (the store is slot S).
    For configurations with K outliers, the selected K rows are multiplied by
    ``k_outlier_scale`` (a power of two, so exact) after rounding.
    """
    seed = cfg.seed if seed is None else seed
    S1, C, Hh, D = cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim
    if slots is None:
        slots = range(S1)
    np_dtype = np.float32 if cfg.dtype == "f32" else np.uint16
    out = [np.zeros((S1, C, Hh, D), dtype=np_dtype) for _ in range(3)]
    for s in slots:
        for t, arr in zip((_T_Q, _T_K, _T_V), out):
            x = _rng(seed, rnd, layer, s, t).standard_normal(size=(C, Hh, D))
            if t == _T_K and cfg.k_outlier_frac > 0.0:
                m = draw_k_outlier_mask(cfg, rnd, layer, s)
                x = np.where(m[:, :, None], x * cfg.k_outlier_scale, x)
            arr[s] = _round_to(x, cfg.dtype)
    return tuple(out)


def draw_page_order(num_pages: int, seed: int) -> np.ndarray:
    """A seeded permutation of physical page ids (int32)."""
    return _rng(seed, 0x9A6E).permutation(num_pages).astype(np.int32)
