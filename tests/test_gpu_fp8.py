"""GPU parity of the FP8 (E4M3) pool: wf_publish_kv and wf_round_attention
against the oracle of oracle/wf_fp8.py (codes and scales) and oracle/wf_oracle.py
(attention over the dequantised operands).

Publication is checked bit for bit: every E4M3 code of q_rot and of the K/V
pages, every block scale, the zero tails and the ready tags. That holds while
the library and the oracle build their rotary (cos, sin) tables with the same
host C library: both evaluate pow, cos and sin in float64 through the system
libm (libwf's pool set-up in C++, the oracle through Python's math module) and
round once to float32. A libm whose results differ in the last bit could move
a float32 table entry and, through it, an occasional E4M3 code; the attention
checks below would still pass, the bit-for-bit code check would not.

Attention tolerances (derived, E4M3 P operand): the kernel rounds each
probability, scaled by a power of two, to E4M3. In the normal range that is a
relative error of at most 2^-4 (half a unit in the last of 3 mantissa bits), so
|out - oracle| <= 2^-4 * sum_i p_i |v_i| / sum_i p_i per element; the bound
used is twice that, for probabilities in E4M3's subnormal range, plus bf16
output rounding (2^-8 |out|). The rounding errors are unbiased, and over
thousands of keys the relative L2 error per slot is about 2^-4 / sqrt(3) times
a factor below 1 (measured 0.014-0.026 on CPU models of these workloads); the
bound used is 0.04. Against the exact oracle (unquantised bf16 inputs), the
FP8 storage of q, k and v adds about 4-5 % relative L2 (12 % with the x8 key
outliers): checked at 0.10 and 0.20.
"""
import numpy as np
import pytest
import torch

import wf_inputs
from oracle import wf_fp8 as F8
from oracle import wf_oracle as O
from wf_test_utils import min_pages, pool_config, rel_l2, tensor_f64

import chunk_causal_wavefront_b200 as wfb

pytestmark = pytest.mark.gpu

REL_DEQ = 0.04
REL_EXACT = 0.10
REL_EXACT_OUTLIERS = 0.20


class Fp8Rollout:
    """An FP8 pool on the GPU plus the oracle's prediction of every byte."""

    def __init__(self, cfg, page_seed=7, layers=1):
        self.cfg = cfg
        self.layers = layers
        order = wf_inputs.draw_page_order(min_pages(cfg), page_seed) if page_seed is not None else None
        self.pool = wfb.KVPool(pool_config(cfg, dtype="fp8", num_layers=layers), device="cuda",
                               page_order=order)
        shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
        self.q_rot = torch.zeros(shape, dtype=torch.uint8, device="cuda")
        self.out = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        self.stored = {l: {} for l in range(layers)}   # chunk -> (pub, k bits, v bits)
        self.live = {l: {} for l in range(layers)}     # slot -> (pub, chunk, q, k, v bits)

    @property
    def round(self):
        return self.pool.round

    def layout(self):
        c = self.cfg
        return O.round_layout(c.num_stages, c.anchor_chunks, c.history_chunks, self.round)

    def publish(self, layer=0, inputs=None):
        c = self.cfg
        lay = self.layout()
        live = [p.slot for p in lay if p.slot is not None]
        if inputs is None:
            inputs = wf_inputs.draw_round_inputs(c, self.round, layer, slots=live)
        q, k, v = inputs
        dev = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (q, k, v)]
        self.pool.publish(layer, dev[0], dev[1], dev[2], self.q_rot)
        self.live[layer] = {}
        for p in lay:
            if p.slot is None:
                continue
            f32 = [wf_inputs.bf16_bits_to_f64(x[p.slot]).astype(np.float32) for x in (q, k, v)]
            pub = F8.publish_fp8_slot(*f32, chunk=p.chunk, P=c.page_tokens, rope=bool(c.rope),
                                      F=c.frames_per_chunk, gh=c.grid_h, gw=c.grid_w,
                                      split=c.rope_split, base=c.rope_base)
            self.live[layer][p.slot] = (pub, p.chunk, q[p.slot], k[p.slot], v[p.slot])
            if p.kind == "store":
                self.stored[layer][p.chunk] = (pub, k[p.slot], v[p.slot])
        return inputs

    def attention(self, layer=0):
        self.out.fill_(float("nan"))
        self.pool.attention(layer, self.q_rot, self.out)

    # ---- checks -----------------------------------------------------------------
    def check_publish(self, layer=0, heads=None):
        c = self.cfg
        hs = list(range(c.num_heads)) if heads is None else list(heads)
        P = c.page_tokens
        qrot = self.q_rot.cpu().numpy()
        qsc = self.pool.q_scales_view()[layer].cpu().numpy()
        pages = self.pool.pages_view()[layer]
        ksc = self.pool.kv_scales_view()[layer].cpu().numpy()
        tags = self.pool.tags_view()[layer].cpu().numpy()
        for kind, chunk, slot, tag, pgs in self.pool.layout():
            if slot is None:
                continue
            pub = self.live[layer][slot][0]
            assert (qrot[slot][:, hs] == pub["q_codes"][:, hs]).all(), ("q codes", slot)
            assert (qsc[slot][:, hs] == np.exp2(pub["q_exp"][:, hs])).all(), ("q scales", slot)
            got = pages[torch.tensor(pgs, device="cuda")].cpu().numpy()   # [npc][2][Hh][P][d]
            for kv, name in ((0, "k"), (1, "v")):
                want = pub[name + "_codes"].reshape(len(pgs), P, c.num_heads, c.head_dim)
                want = np.transpose(want, (0, 2, 1, 3))                      # [npc][Hh][P][d]
                assert (got[:, kv][:, hs] == want[:, hs]).all(), (name, "codes", slot)
                assert (ksc[pgs][:, kv][:, hs] == np.exp2(pub[name + "_exp"][:, hs])).all(), \
                    (name, "scales", slot)
            assert all(tags[g] == tag for g in pgs), ("tags", slot)

    def _deq_operands(self, layer, heads):
        c = self.cfg
        P = c.page_tokens
        q, keys, vals, kx, vx = {}, {}, {}, {}, {}
        for s, (pub, chunk, qb, kb, vb) in self.live[layer].items():
            q[s] = F8.dequantize_rows(pub["q_codes"], pub["q_exp"], 128)[:, heads]
        for p in self.layout():
            if p.slot is None:
                pub, kb, vb = self.stored[layer][p.chunk]
            else:
                pub, _, _, kb, vb = self.live[layer][p.slot]
            keys[p.chunk] = F8.dequantize_rows(pub["k_codes"][:c.chunk_tokens], pub["k_exp"], P)[:, heads]
            vals[p.chunk] = F8.dequantize_rows(pub["v_codes"][:c.chunk_tokens], pub["v_exp"], P)[:, heads]
            kx[p.chunk] = (kb, vb)
        return q, keys, vals, kx

    def check_attention(self, layer=0, heads=None, rows=None, exact=True, record=None):
        c = self.cfg
        hs = list(range(c.num_heads)) if heads is None else list(heads)
        q, keys, vals, kx = self._deq_operands(layer, hs)
        lay = self.layout()
        want = O.attention_slot_prefix(q, keys, vals, lay, rows=rows, mask=c.mask)
        # sum_i p_i |v_i| / sum_i p_i: the same attention with |V|
        wabs = O.attention_slot_prefix(q, keys, {k: np.abs(v) for k, v in vals.items()}, lay,
                                       rows=rows, mask=c.mask)
        if exact:
            qe, ke, ve = {}, {}, {}
            for s, (pub, chunk, qb, kb, vb) in self.live[layer].items():
                qe[s] = self._rope(wf_inputs.bf16_bits_to_f64(qb)[:, hs], chunk)
            for p in lay:
                kb, vb = kx[p.chunk]
                ke[p.chunk] = self._rope(wf_inputs.bf16_bits_to_f64(kb)[:, hs], p.chunk)
                ve[p.chunk] = wf_inputs.bf16_bits_to_f64(vb)[:, hs]
            want_x = O.attention_slot_prefix(qe, ke, ve, lay, rows=rows, mask=c.mask)
        out = tensor_f64(self.out)
        live = {p.slot for p in lay if p.slot is not None}
        for s in range(c.num_slots):
            got = out[s][:, hs] if rows is None else out[s][rows][:, hs]
            if s not in live:
                assert np.isnan(got).all(), f"idle slot {s} was written"
                continue
            assert np.isfinite(got).all(), s
            err = np.abs(got - want[s])
            bound = 2.0 ** -3 * wabs[s] + 2.0 ** -8 * np.abs(want[s]) + 1e-5
            r = rel_l2(got, want[s])
            rec = dict(slot=s, rel_l2_deq=r, max_err_over_bound=float((err / bound).max()))
            if exact:
                rec["rel_l2_exact"] = rel_l2(got, want_x[s])
            if record is not None:
                record.append(rec)
            assert (err <= bound).all(), rec
            assert r <= REL_DEQ, rec
            if exact:
                lim = REL_EXACT_OUTLIERS if c.k_outlier_frac > 0 else REL_EXACT
                assert rec["rel_l2_exact"] <= lim, rec

    def _rope(self, x64, chunk):
        c = self.cfg
        if not c.rope:
            return x64
        return O.rope_3d(x64, chunk, c.frames_per_chunk, c.grid_h, c.grid_w, c.rope_split,
                         c.rope_base)

    def close(self):
        self.pool.close()


SMALL = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    num_stages=3, chunk_tokens=300, num_heads=2, history_chunks=2, frames_per_chunk=1,
    grid_h=10, grid_w=30, rounds=10)


# The largest stage count the ABI accepts (WF_MAX_STAGES = 16: 17 live query
# slots, every per-slot array of the launch parameters full), with a ragged
# two-tile chunk (130 = 128 + 2 rows).
MAX_STAGES = SMALL.replace(num_stages=16, chunk_tokens=130, grid_h=10, grid_w=13, history_chunks=3,
                          rounds=24)


@pytest.mark.parametrize("cfg", [SMALL, SMALL.replace(mask="rf"), MAX_STAGES],
                         ids=["wf", "rf", "max_stages"])
def test_fp8_small_every_round(cfg):
    ro = Fp8Rollout(cfg, page_seed=3)
    for k in range(cfg.steady_round() + 3):
        ro.publish()
        ro.attention()
        assert ro.pool.check_status() == 0
        ro.check_publish()
        ro.check_attention()
        ro.pool.advance()
    ro.close()


def test_fp8_outliers_small():
    cfg = wf_inputs.CONFIGS["wan13b_5step_bf16"].replace(
        chunk_tokens=300, num_heads=2, frames_per_chunk=1, grid_h=10, grid_w=30)
    ro = Fp8Rollout(cfg, page_seed=4)
    for k in range(cfg.steady_round() + 1):
        ro.publish()
        if k == cfg.steady_round():
            ro.attention()
            assert ro.pool.check_status() == 0
            ro.check_publish()
            ro.check_attention()
        ro.pool.advance()
    ro.close()


@pytest.mark.parametrize("name", ["wan13b_bf16", "wan13b_5step_bf16"])
def test_fp8_full_size_sampled(name):
    cfg = wf_inputs.CONFIGS[name]
    ro = Fp8Rollout(cfg, page_seed=5)
    heads = [0, 7]
    rows = np.array([0, 1, 127, 128, 1000, 2345, 4607, 4608, 4679])
    rec = []
    for k in range(cfg.steady_round() + 1):
        ro.publish()
        if k == cfg.steady_round():
            ro.attention()
            assert ro.pool.check_status() == 0
            ro.check_publish(heads=heads)
            ro.check_attention(heads=heads, rows=rows, record=rec)
        ro.pool.advance()
    ro.close()
    assert rec


def test_fp8_full_size_all_rows():
    # Every query row of every live slot of one head at full size (19 tile
    # pairs per slot in the launch configuration bench.py times).
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    ro = Fp8Rollout(cfg, page_seed=8)
    rec = []
    for k in range(cfg.steady_round() + 1):
        ro.publish()
        if k == cfg.steady_round():
            ro.attention()
            assert ro.pool.check_status() == 0
            ro.check_publish(heads=[4])
            ro.check_attention(heads=[4], rows=None, record=rec)
        ro.pool.advance()
    ro.close()
    assert len(rec) == cfg.num_slots


def test_fp8_long_context_past_page_cache():
    # 29 chunks x 37 pages = 1073 key tiles: page ids and K/V scale exponents
    # past the 1024 cached in shared memory are read through the page table.
    cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(
        name="long_context_bf16", num_stages=1, num_heads=1, history_chunks=26, rounds=30)
    positions = cfg.anchor_chunks + cfg.history_chunks + cfg.num_stages + 1
    assert positions * cfg.pages_per_chunk > 1024
    ro = Fp8Rollout(cfg, page_seed=6)
    rows = np.array([0, 1, 127, 128, 777, 2345, 3000, 4607, 4608, 4679])
    rec = []
    for k in range(cfg.steady_round() + 1):
        ro.publish()
        if k == cfg.steady_round():
            ro.attention()
            assert ro.pool.check_status() == 0
            ro.check_publish()
            ro.check_attention(rows=rows, record=rec)
        ro.pool.advance()
    ro.close()
    assert rec


def test_fp8_value_ones_and_mask_perturbation():
    """V = 1 everywhere gives out = 1 up to the P rounding bound; changing the
    K/V of a noisier slot leaves every cleaner slot's output bit-identical."""
    cfg = SMALL
    ro = Fp8Rollout(cfg, page_seed=1)
    for k in range(cfg.steady_round() + 1):                # V = 1 in every round
        q, kk, v = wf_inputs.draw_round_inputs(cfg, ro.round, 0)
        ones = np.full_like(v, 0x3F80)                     # bf16 1.0
        ro.publish(inputs=(q, kk, ones))
        if k < cfg.steady_round():
            ro.pool.advance()
    k = kk
    ro.attention()
    assert ro.pool.check_status() == 0
    live = [p.slot for p in ro.layout() if p.slot is not None]
    out = tensor_f64(ro.out)
    for s in live:
        # V blocks of 1.0 quantise exactly (code 0x78 with scale 2^-8)
        assert np.abs(out[s] - 1.0).max() <= 2.0 ** -3 + 2.0 ** -8, s
    # perturbation: rewrite slot 0's K and V; slots 1.. must not change
    ro.publish(inputs=(q, k, v))
    ro.attention()
    base = ro.out.clone()
    k2, v2 = k.copy(), v.copy()
    k2[0] = wf_inputs.draw_normal(k2[0].shape, "bf16", 99, 1)
    v2[0] = wf_inputs.draw_normal(v2[0].shape, "bf16", 99, 2)
    ro.publish(inputs=(q, k2, v2))
    ro.attention()
    assert ro.pool.check_status() == 0
    for s in live:
        if s == 0:
            continue
        assert torch.equal(ro.out[s], base[s]), s
    ro.close()


def test_fp8_page_permutation_invariance():
    cfg = SMALL
    outs = []
    for seed in (11, 12):
        ro = Fp8Rollout(cfg, page_seed=seed)
        for k in range(cfg.steady_round() + 1):
            ro.publish()
            if k == cfg.steady_round():
                ro.attention()
                assert ro.pool.check_status() == 0
                outs.append(ro.out.clone())
            ro.pool.advance()
        ro.close()
    assert torch.equal(outs[0], outs[1])


def test_fp8_not_ready_and_unsupported():
    cfg = SMALL
    ro = Fp8Rollout(cfg, page_seed=2)
    ro.publish()
    ro.pool.advance()
    ro.out.fill_(7.0)
    ro.pool.attention(0, ro.q_rot, ro.out)                 # round 1 never published
    assert ro.pool.check_status() == wfb.WF_ERR_NOT_READY
    assert (ro.out.float() == 7.0).all()
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wfb.WfError) as e:
        ro.pool.project_publish(0, x, x, ro.q_rot)
    assert e.value.status == wfb.WF_ERR_UNSUPPORTED
    ro.close()
