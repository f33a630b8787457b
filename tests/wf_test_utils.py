"""Helpers that drive libwf and the float64 oracle side by side.

Inputs come from wf_inputs (seeded, rounded once to the working dtype); the
oracle side widens exactly those bits to float64 and applies its own rotary
embedding and attention. Nothing here computes the method on the GPU side: the
library does, through its C ABI.
"""
from __future__ import annotations

import json
import math
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

import wf_inputs
from wf_inputs import WorkloadConfig, bf16_bits_to_f64
from oracle import wf_oracle as O
from oracle import wf_fp8 as F8


def pool_config(cfg: WorkloadConfig, **over):
    from chunk_causal_wavefront_b200 import make_config
    kw = dict(num_stages=cfg.num_stages, chunk_tokens=cfg.chunk_tokens, num_heads=cfg.num_heads,
              head_dim=cfg.head_dim, anchor_chunks=cfg.anchor_chunks,
              history_chunks=cfg.history_chunks, page_tokens=cfg.page_tokens,
              num_layers=cfg.num_layers, dtype=cfg.dtype, rope=cfg.rope,
              frames_per_chunk=cfg.frames_per_chunk, grid_h=cfg.grid_h, grid_w=cfg.grid_w,
              rope_split=cfg.rope_split if cfg.rope else (0, 0, 0), rope_base=cfg.rope_base,
              max_rounds=max(cfg.rounds, cfg.steady_round()) + 8, num_pages=0, mask=cfg.mask)
    kw.update(over)
    return make_config(**kw)


def min_pages(cfg: WorkloadConfig) -> int:
    return (cfg.num_stages + 1 + cfg.anchor_chunks + cfg.history_chunks) * cfg.pages_per_chunk


def to_f64(arr: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits_to_f64(arr) if dtype == "bf16" else arr.astype(np.float64)


def to_device(arr: np.ndarray, dtype: str, device) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(arr).to(device)


def tensor_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


class Rollout:
    """One pool on one GPU plus the oracle's view of the same rounds."""

    def __init__(self, cfg: WorkloadConfig, device="cuda", page_seed: Optional[int] = 7,
                 num_pages: int = 0, layers: Optional[int] = None):
        from chunk_causal_wavefront_b200 import KVPool
        self.cfg = cfg
        self.device = torch.device(device)
        self.layers = cfg.num_layers if layers is None else layers
        n_pages = num_pages or min_pages(cfg)
        self.page_order = (None if page_seed is None
                           else wf_inputs.draw_page_order(n_pages, page_seed))
        self.pool = KVPool(pool_config(cfg, num_layers=self.layers, num_pages=num_pages),
                           device=self.device, page_order=self.page_order)
        shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
        tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        self.q_rot = torch.zeros(shape, dtype=tdt, device=self.device)
        self.out = torch.zeros(shape, dtype=tdt, device=self.device)
        # per layer: chunk -> (k bits, v bits) the store published; slot -> (q, k, v, chunk)
        self.stored: Dict[int, Dict[int, tuple]] = {l: {} for l in range(self.layers)}
        self.live: Dict[int, Dict[int, tuple]] = {l: {} for l in range(self.layers)}

    @property
    def round(self) -> int:
        return self.pool.round

    def layout(self):
        c = self.cfg
        return O.round_layout(c.num_stages, c.anchor_chunks, c.history_chunks, self.round)

    def publish(self, layer: int = 0, inputs=None, real_slots: Optional[Sequence[int]] = None):
        """Draw (or take) this round's inputs and run wf_publish_kv."""
        c = self.cfg
        lay = self.layout()
        live = [p.slot for p in lay if p.slot is not None]
        if inputs is None:
            slots = live if real_slots is None else [s for s in live if s in real_slots]
            inputs = wf_inputs.draw_round_inputs(c, self.round, layer, slots=slots)
        q, k, v = inputs
        self.inputs = inputs
        tq, tk, tv = (to_device(x, c.dtype, self.device) for x in (q, k, v))
        self.pool.publish(layer, tq, tk, tv, self.q_rot)
        self.live[layer] = {}
        for p in lay:
            if p.slot is None:
                continue
            self.live[layer][p.slot] = (q[p.slot], k[p.slot], v[p.slot], p.chunk)
            if p.kind == "store":
                self.stored[layer][p.chunk] = (k[p.slot], v[p.slot])
        return inputs

    def attention(self, layer: int = 0, fill: float = float("nan")):
        self.out.fill_(fill)
        self.pool.attention(layer, self.q_rot, self.out)

    def advance(self):
        self.pool.advance()

    # ---- oracle side ----------------------------------------------------------------
    def _rope(self, x64: np.ndarray, chunk: int) -> np.ndarray:
        c = self.cfg
        if not c.rope:
            return x64
        return O.rope_3d(x64, chunk, c.frames_per_chunk, c.grid_h, c.grid_w,
                         split=c.rope_split, base=c.rope_base)

    def oracle_tensors(self, heads: Sequence[int], layer: int = 0):
        """fp64 rotated q per live slot, rotated K and V per context chunk."""
        c, hs = self.cfg, list(heads)
        q_rot, keys, vals = {}, {}, {}
        for s, (q, k, v, chunk) in self.live[layer].items():
            q_rot[s] = self._rope(to_f64(q, c.dtype)[:, hs], chunk)
        for p in self.layout():
            if p.slot is None:
                kb, vb = self.stored[layer][p.chunk]
            else:
                _, kb, vb, _ = self.live[layer][p.slot]
            keys[p.chunk] = self._rope(to_f64(kb, c.dtype)[:, hs], p.chunk)
            vals[p.chunk] = to_f64(vb, c.dtype)[:, hs]
        return q_rot, keys, vals

    def oracle_out(self, heads: Sequence[int], rows: Optional[np.ndarray] = None, layer: int = 0):
        q_rot, keys, vals = self.oracle_tensors(heads, layer)
        return O.attention_slot_prefix(q_rot, keys, vals, self.layout(), rows=rows,
                                       mask=self.cfg.mask)

    def oracle_out_bf16_operands(self, heads: Sequence[int], rows=None, layer: int = 0):
        """Oracle attention on the operands the pool publishes: q and k rotated
        in float32 with each product and sum rounded once (rope_3d_f32, the
        oracle's rule for published rotations), then rounded to bf16 by the
        oracle itself (round_bf16), the storage format of q_rot and the K pages.
        Nothing here is read back from the GPU."""
        c, hs = self.cfg, list(heads)
        if c.dtype != "bf16":
            raise ValueError("bf16 pools only")

        def pub(bits, chunk):
            x = to_f64(bits, c.dtype)[:, hs]
            if c.rope:
                x = F8.rope_3d_f32(x.astype(np.float32), chunk, c.frames_per_chunk, c.grid_h,
                                   c.grid_w, c.rope_split, c.rope_base).astype(np.float64)
            return O.round_bf16(x)

        q_rot, keys, vals = {}, {}, {}
        for s, (q, k, v, chunk) in self.live[layer].items():
            q_rot[s] = pub(q, chunk)
        for p in self.layout():
            kb, vb = (self.stored[layer][p.chunk] if p.slot is None
                      else self.live[layer][p.slot][1:3])
            keys[p.chunk] = pub(kb, p.chunk)
            vals[p.chunk] = to_f64(vb, c.dtype)[:, hs]
        return O.attention_slot_prefix(q_rot, keys, vals, self.layout(), rows=rows,
                                       mask=c.mask)

    def close(self):
        self.pool.close()


# ---- parity checks shared by the GPU tests -------------------------------------------

BF16_ABS, BF16_REL = 2e-2, 1e-2
F32_ABS = 1e-5
# Every bf16 case is checked twice.
#  * Against the oracle run on the published operands (q and k rotated in
#    float32 and rounded to bf16 by the oracle, the values the publish tests
#    find bit for bit in q_rot and the K pages): this is the kernel's own
#    error. Per element, |O - O_pub| <= 2e-2 + u |O_pub|, and rel-L2 <= 1e-2.
#    u = 2^-8 is bf16's unit roundoff (8-bit significand): the output is
#    stored in bf16 (the pages run BF16), and at |O| in [4, 8), where the x8
#    outlier keys put some outputs, rounding alone moves it by up to 2^-6.
#  * Against the exact float64 oracle: rel-L2 <= 1e-2, and per element
#    max-abs 2e-2 on top of the rounding effect |O_exact - O_pub| that the
#    oracle itself computes. With 5% of K rows scaled x8 the softmax is sharply
#    peaked and rounding q and k to bf16 moves each dominant logit by about
#    8 * 2^-9; near-tied dominant keys then shift outputs of size ~3 by a few
#    1e-2 against the exact result, whatever the kernel does.
BF16_U = 2.0 ** -8


def log_parity(name, **kw):
    path = os.environ.get("WF_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(test=name, **kw)) + "\n")


def compare_with_oracle(ro: "Rollout", heads, rows=None, gpu_operands=True, name="", layer=0):
    """Check ro.out (live slots; idle slots must still be NaN) against the
    float64 oracle for the given heads and rows, at the tolerances above."""
    c = ro.cfg
    want = ro.oracle_out(heads, rows, layer)
    want_g = (ro.oracle_out_bf16_operands(heads, rows, layer)
              if gpu_operands and c.dtype == "bf16" else None)
    out = tensor_f64(ro.out)
    live = {p.slot for p in ro.layout() if p.slot is not None}
    for s in range(c.num_slots):
        got_s = out[s][:, list(heads)] if rows is None else out[s][rows][:, list(heads)]
        if s not in live:
            assert np.isnan(got_s).all(), f"idle slot {s} was written"
            continue
        assert np.isfinite(got_s).all(), s
        err = float(np.abs(got_s - want[s]).max())
        if c.dtype == "f32":
            log_parity(name, round=ro.round, slot=s, max_abs=err)
            assert err <= F32_ABS, (s, err)
            continue
        r = rel_l2(got_s, want[s])
        rec = dict(round=ro.round, slot=s, max_abs=err, rel_l2=r)
        if want_g is not None:
            rec.update(max_abs_bf16_operands=float(np.abs(got_s - want_g[s]).max()),
                       rel_l2_bf16_operands=rel_l2(got_s, want_g[s]),
                       rounding_effect=float(np.abs(want_g[s] - want[s]).max()),
                       max_abs_out=float(np.abs(want_g[s]).max()))
        log_parity(name, **rec)
        assert r <= BF16_REL, (s, rec)
        if want_g is None:
            assert err <= BF16_ABS, (s, rec)
        else:
            assert (np.abs(got_s - want[s]) <= BF16_ABS + np.abs(want_g[s] - want[s])).all(), (s, rec)
            dev = np.abs(got_s - want_g[s])
            assert (dev <= BF16_ABS + BF16_U * np.abs(want_g[s])).all(), (s, rec)
            assert rec["rel_l2_bf16_operands"] <= BF16_REL, (s, rec)
            if c.k_outlier_frac == 0:
                assert err <= BF16_ABS, (s, rec)
