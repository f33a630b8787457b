"""Pins of the FP8 (E4M3) oracle, on the CPU.

Each check ties oracle/wf_fp8.py to something other than itself: PyTorch's
float8_e4m3fn conversion (a library routine) for the format, exhaustive
properties for the scale rule, correctly rounded single operations for the
float32 rotation, and the float64 rotation of wf_oracle within float32 error.
"""
import math

import numpy as np
import pytest
import torch

import wf_inputs
from oracle import wf_fp8 as F8
from oracle import wf_oracle as O


def _torch_decode(codes):
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.float().double().numpy()


def _torch_encode(y32):
    t = torch.from_numpy(np.asarray(y32, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours, ref = F8.e4m3_decode(codes), _torch_decode(codes)
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert (ours[~nan] == ref[~nan]).all()
    assert np.nanmax(ours) == F8.E4M3_MAX and ours[1] == 2.0 ** -9 and ours[8] == 2.0 ** -6


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F8.e4m3_decode(codes)
    assert (F8.e4m3_encode(vals) == codes).all()


def test_encode_ties_and_midpoints_match_torch():
    pos = np.array([c for c in range(0x7F)], dtype=np.uint8)       # +0 .. 448, increasing
    v = F8.e4m3_decode(pos)
    assert (np.diff(v) > 0).all()
    mids = (v[:-1] + v[1:]) / 2.0                # exact in float32 (4 significant bits)
    y = np.concatenate([mids, -mids]).astype(np.float32)
    got = F8.e4m3_encode(y)
    assert (got == _torch_encode(y)).all()
    # ties go to the even mantissa: the code of each midpoint is even
    assert (got[: mids.size] % 2 == 0).all()


def test_encode_random_values_match_torch():
    rng = np.random.default_rng(7)
    y = []
    for e in range(-12, 9):
        y.append(rng.uniform(-1, 1, 4000) * 2.0 ** e)
    y = np.clip(np.concatenate(y), -448, 448).astype(np.float32)
    y = np.concatenate([y, np.float32([0.0, -0.0, 448.0, -448.0, 2.0 ** -10, 2.0 ** -6])])
    got = F8.e4m3_encode(y)
    assert (got == _torch_encode(y)).all()
    assert got[-6 + 1] == 0x80                    # -0.0 keeps its sign


def test_scale_exponent_is_smallest():
    rng = np.random.default_rng(11)
    amaxes = list(np.float32(rng.lognormal(0, 3, 5000)))
    amaxes += [448.0, float(np.nextafter(np.float32(448), np.float32(1e9))), 224.0, 1.0, 1.75,
               float(np.nextafter(np.float32(1.75), np.float32(2))), 2.0 ** -60, 3.0e20]
    for a in amaxes:
        e = F8.scale_exponent(a)
        assert a * 2.0 ** -e <= 448.0, a
        assert a * 2.0 ** -(e - 1) > 448.0, a          # e - 1 would overflow the format
        assert 224.0 < a * 2.0 ** -e or a == 224.0, a  # largest value lands in (224, 448]
    assert F8.scale_exponent(448.0) == 0
    assert F8.scale_exponent(1.0) == -8              # 1 * 2^8 = 256 <= 448 < 512
    assert F8.scale_exponent(0.0) == F8.SCALE_EXP_MIN
    assert F8.scale_exponent(2.0 ** -120) == F8.SCALE_EXP_MIN


def test_quantize_block_error_within_half_ulp():
    rng = np.random.default_rng(3)
    for scale in (1e-3, 1.0, 37.0):
        x = (rng.standard_normal((128, 128)) * scale).astype(np.float32)
        codes, e = F8.quantize_block(x)
        deq = F8.e4m3_decode(codes) * 2.0 ** e
        y = np.abs(x.astype(np.float64)) * 2.0 ** -e
        assert y.max() <= 448.0 and y.max() > 224.0
        # half a unit in the last place: 2^-4 relative in the normal range,
        # 2^-10 absolute (before scaling) in the subnormal range
        bound = np.where(y >= 2.0 ** -6, 2.0 ** -4 * y, 2.0 ** -10) * 2.0 ** e
        assert (np.abs(deq - x) <= bound * (1 + 1e-12)).all()


def test_rope_f32_operations_are_correctly_rounded_float32():
    rng = np.random.default_rng(5)
    a = rng.standard_normal(1000).astype(np.float32)
    c = rng.standard_normal(1000).astype(np.float32)
    # a float32 product or sum equals the exact float64 result rounded once
    assert ((a * c) == (a.astype(np.float64) * c.astype(np.float64)).astype(np.float32)).all()
    assert ((a + c) == (a.astype(np.float64) + c.astype(np.float64)).astype(np.float32)).all()


def test_rope_f32_close_to_float64_rotation():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    x = wf_inputs.bf16_bits_to_f64(wf_inputs.draw_normal((cfg.chunk_tokens, 2, 128), "bf16", 9))
    for chunk in (0, 7, 150):
        r32 = F8.rope_3d_f32(x.astype(np.float32), chunk, cfg.frames_per_chunk, cfg.grid_h,
                             cfg.grid_w, cfg.rope_split, cfg.rope_base)
        r64 = O.rope_3d(x, chunk, cfg.frames_per_chunk, cfg.grid_h, cfg.grid_w,
                        cfg.rope_split, cfg.rope_base)
        # table rounding (2^-24 relative each) + two products + one sum, float32
        pair = np.abs(x[..., 0::2]) + np.abs(x[..., 1::2])
        bound = np.repeat(pair, 2, axis=-1) * 2.0 ** -21
        assert (np.abs(r32 - r64) <= bound).all()


def test_publish_fp8_slot_blocks_and_tails():
    C, Hh, d, P = 300, 2, 128, 128
    rng = np.random.default_rng(1)
    q, k, v = (wf_inputs.bf16_bits_to_f64(wf_inputs.draw_normal((C, Hh, d), "bf16", 1, t))
               .astype(np.float32) for t in range(3))
    k[:, 1] *= 16.0                                   # a second head with larger keys
    out = F8.publish_fp8_slot(q, k, v, chunk=2, P=P, rope=True, F=1, gh=10, gw=30)
    npc = 3
    assert out["k_codes"].shape == (npc * P, Hh, d) and out["k_exp"].shape == (npc, Hh)
    assert out["q_codes"].shape == (C, Hh, d) and out["q_exp"].shape == (npc, Hh)
    assert (out["k_codes"][C:] == 0).all() and (out["v_codes"][C:] == 0).all()
    assert (out["k_exp"][:, 1] == out["k_exp"][:, 0] + 4).sum() >= 2   # x16 moves e by 4
    kr = O.rope_3d(k.astype(np.float64), 2, 1, 10, 30)
    deq = F8.dequantize_rows(out["k_codes"][:C], out["k_exp"], P)
    rel = np.abs(deq - kr) / (np.abs(kr) + 2.0 ** (out["k_exp"].max() - 6))
    assert rel.max() <= 2.0 ** -4 + 1e-5
    dv = F8.dequantize_rows(out["v_codes"][:C], out["v_exp"], P)
    assert np.abs(dv - v).max() <= 2.0 ** -4 * np.abs(v).max()


def test_dequantize_then_attention_reduces_to_exact_when_values_representable():
    """Values already on the E4M3 grid (times a power of two) survive
    quantisation exactly, so attention over the dequantised operands equals
    attention over the originals."""
    rng = np.random.default_rng(2)
    grid = F8.e4m3_decode(np.arange(0x00, 0x70, dtype=np.uint8))   # 0 .. 240
    x = rng.choice(np.concatenate([grid, -grid]), size=(128, 1, 16)) * 2.0 ** -5
    x[0, 0, 0] = 448.0 * 2.0 ** -5                  # pins the block's exponent at -5
    codes, e = F8.quantize_block(x[:, 0].astype(np.float32))
    assert e == -5
    assert (F8.e4m3_decode(codes) * 2.0 ** e == x[:, 0]).all()
