"""FP8 (E4M3) storage of published Q, K and V: CPU oracle.

TEST INFRASTRUCTURE ONLY, like ``wf_oracle``: only ``tests/`` (and the smoke
check and the CPU-baseline leg of the benchmark) may import it. It shares no
code with the CUDA library. Quantisation decisions are taken in float32 exactly
as the pages' storage format would take them (see below), so the FP8 codes and
scales are predicted bit for bit; attention over them is the exact float64
definition of ``wf_oracle.attention_slot_prefix`` applied to the dequantised
values.

Source: "Wave Forcing: Towards Speed-of-Light Streaming Video Generation",
Appendix Table 8: K/V can travel as FP8 with scale factors ("payload and scale
transfer, excluding conversion"), about half the BF16 transfer time; Tables
4-6 run the model with SageAttention (8-bit attention operands). The pages fix
neither the 8-bit format, nor the granularity of the scales, nor the rounding.
Readings taken here (each listed in the design notes of the repository):
  * format E4M3, the OCP 8-bit float with 1 sign bit, 4 exponent bits (bias 7)
    and 3 mantissa bits, no infinities, largest finite value 448, NaN at
    S.1111.111;
  * one scale per block: per (page of 128 tokens, head) for K and for V, and per
    (128-row query tile, head) for Q. The scale is a power of two 2^e, with e
    the smallest integer such that amax * 2^-e <= 448 (amax = the largest |x|
    in the block), clamped below at -100 (an all-zero block gets e = -100);
  * codes are round-to-nearest-even of x * 2^-e (an exact product), so every
    block's largest magnitude lands in [224, 448];
  * Q and K are rotated (3D rotary) in float32 before quantisation: each
    product and each sum rounded once to float32 (no fused multiply-add), with
    the (cos, sin) tables computed in float64 by the C library's pow, cos and
    sin and rounded to float32. V is quantised from its bf16 value;
  * rows of a chunk's last page past C are zero codes; query tiles cover rows
    [128 t, 128 t + 128) clipped at C.

Pins (tests/test_oracle_fp8.py): decoding of all 256 codes and encoding
(including every tie) against PyTorch's float8_e4m3fn conversion (a library
routine); the smallest-exponent property of the scale rule by exhaustive checks;
float32 rotation against the float64 rotation within float32 rounding and
against a correctly rounded single-operation reference; quantisation error
within half a unit in the last place of the format; zero tails.
"""
from __future__ import annotations

import math
from typing import Dict, Sequence

import numpy as np

__all__ = ["E4M3_MAX", "SCALE_EXP_MIN", "e4m3_decode", "e4m3_encode", "scale_exponent",
           "quantize_block", "rope_tables_f32", "rope_3d_f32", "publish_fp8_slot",
           "dequantize_rows"]

E4M3_MAX = 448.0
SCALE_EXP_MIN = -100


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Float64 value of E4M3 codes (uint8): exponent field E, mantissa field m;
    E = 0 is subnormal, m * 2^-9; otherwise 2^(E-7) * (1 + m/8); S.1111.111 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(E == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(E - 7.0))
    mag = np.where((E == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """Round finite values to the nearest E4M3 value, ties to even mantissa,
    saturating at +-448; returns uint8 codes. The sign of zero is kept."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    codes = np.zeros(y.shape, dtype=np.int64)
    # Subnormal range [0, 2^-6): a grid of step 2^-9; a result of 8 steps is
    # the smallest normal 2^-6, whose code is also 8.
    sub = a < 2.0 ** -6
    codes[sub] = np.rint(a[sub] * 2.0 ** 9).astype(np.int64)
    # Normal range: a = f * 2^E with f in [1, 2); 8 * f rounded to an integer
    # q in [8, 16]; q = 16 carries into the next binade.
    nor = ~sub
    mant, ex = np.frexp(a[nor])             # a = mant * 2^ex, mant in [0.5, 1)
    E = ex.astype(np.int64) - 1
    q = np.rint(mant * 16.0).astype(np.int64)   # = rint(8 * f)
    carry = q == 16
    E = np.where(carry, E + 1, E)
    q = np.where(carry, 8, q)
    field = E + 7
    cn = (field << 3) | (q - 8)
    cn = np.where((field > 15) | ((field == 15) & (q - 8 == 7)), 0x7E, cn)   # saturate
    codes[nor] = cn
    codes = codes | np.where(np.signbit(y), 0x80, 0)
    return codes.astype(np.uint8)


def scale_exponent(amax: float) -> int:
    """Smallest integer e with amax * 2^-e <= 448, clamped below at -100."""
    amax = float(amax)
    if amax == 0.0:
        return SCALE_EXP_MIN
    mant, ex = math.frexp(amax)             # amax = (2 mant) * 2^(ex - 1), 2 mant in [1, 2)
    f, E = 2.0 * mant, ex - 1
    e = E - 8 if f <= 1.75 else E - 7       # 448 = 1.75 * 2^8
    return max(e, SCALE_EXP_MIN)


def quantize_block(x32: np.ndarray):
    """Codes and scale exponent of one block of float32 values."""
    x32 = np.asarray(x32, dtype=np.float32)
    amax = float(np.max(np.abs(x32))) if x32.size else 0.0
    e = scale_exponent(amax)
    y = x32 * np.float32(2.0 ** -e)           # float32 product by a power of two
    return e4m3_encode(y), e


def rope_tables_f32(n_pos: int, width: int, base: float):
    """(cos, sin) [n_pos][width/2] of pos * base^(-2m/width), float64 rounded to float32.

    The float64 values come from the C library's pow, cos and sin (Python's
    math module), the double-precision routines a host program calls: NumPy's
    vectorised pow may differ from them in the last bit, which can move a
    float32-rounded table entry and, through it, an E4M3 code."""
    half = width // 2
    cos_t = np.empty((n_pos, half), dtype=np.float32)
    sin_t = np.empty((n_pos, half), dtype=np.float32)
    for m in range(half):
        inv = math.pow(float(base), -2.0 * m / float(width))
        for pos in range(n_pos):
            ang = float(pos) * inv
            cos_t[pos, m] = math.cos(ang)
            sin_t[pos, m] = math.sin(ang)
    return cos_t, sin_t


def rope_3d_f32(x32: np.ndarray, chunk: int, F: int, gh: int, gw: int,
                split: Sequence[int] = (44, 42, 42), base: float = 10000.0) -> np.ndarray:
    """3D rotary of x [C][heads][d] in float32 arithmetic: for each pair (a, b)
    of a band, (a c - b s, a s + b c) with every product and sum rounded to
    float32. Positions as in ``wf_oracle.rope_positions``."""
    x32 = np.asarray(x32, dtype=np.float32)
    C = x32.shape[0]
    n = np.arange(C, dtype=np.int64)
    pos = (F * chunk + n // (gh * gw), (n // gw) % gh, n % gw)
    out = x32.copy()
    off = 0
    for p, width in zip(pos, split):
        cos_t, sin_t = rope_tables_f32(int(p.max()) + 1, width, base)
        c = cos_t[p][:, None, :]
        s = sin_t[p][:, None, :]
        a = x32[:, :, off:off + width:2]
        b = x32[:, :, off + 1:off + width:2]
        out[:, :, off:off + width:2] = (a * c) - (b * s)
        out[:, :, off + 1:off + width:2] = (a * s) + (b * c)
        off += width
    return out


def _blocks(x32: np.ndarray, rows: int, n_blocks: int):
    """Codes [n_blocks * rows][heads][d] (zero past the data) and exponents [n_blocks][heads]."""
    N, Hh, d = x32.shape
    codes = np.zeros((n_blocks * rows, Hh, d), dtype=np.uint8)
    exps = np.zeros((n_blocks, Hh), dtype=np.int64)
    for j in range(n_blocks):
        lo, hi = j * rows, min(N, (j + 1) * rows)
        for h in range(Hh):
            c, e = quantize_block(x32[lo:hi, h])
            codes[lo:hi, h] = c
            exps[j, h] = e
    return codes, exps


def publish_fp8_slot(q: np.ndarray, k: np.ndarray, v: np.ndarray, chunk: int, P: int,
                     rope: bool, F: int = 1, gh: int = 1, gw: int = 1,
                     split: Sequence[int] = (44, 42, 42), base: float = 10000.0
                     ) -> Dict[str, np.ndarray]:
    """Predicted FP8 publication of one slot's chunk.

    q, k, v: [C][heads][d] bf16 values as float32 (exact). Returns q_codes
    [C][heads][d] with q_exp [ceil(C/128)][heads], and K/V page rows
    k_codes, v_codes [npc * P][heads][d] (zero past C) with k_exp, v_exp
    [npc][heads], npc = ceil(C / P).
    """
    C = q.shape[0]
    q32 = np.asarray(q, dtype=np.float32)
    k32 = np.asarray(k, dtype=np.float32)
    v32 = np.asarray(v, dtype=np.float32)
    if rope:
        q32 = rope_3d_f32(q32, chunk, F, gh, gw, split, base)
        k32 = rope_3d_f32(k32, chunk, F, gh, gw, split, base)
    qc, qe = _blocks(q32, 128, -(-C // 128))
    npc = -(-C // P)
    kc, ke = _blocks(k32, P, npc)
    vc, ve = _blocks(v32, P, npc)
    return {"q_codes": qc[:C], "q_exp": qe, "k_codes": kc, "k_exp": ke,
            "v_codes": vc, "v_exp": ve}


def dequantize_rows(codes: np.ndarray, exps: np.ndarray, rows: int) -> np.ndarray:
    """Float64 values code * 2^e of rows [N][heads][d], block b = row // rows."""
    vals = e4m3_decode(codes)
    N = codes.shape[0]
    blk = np.arange(N) // rows
    return vals * np.exp2(exps[blk].astype(np.float64))[:, :, None]
