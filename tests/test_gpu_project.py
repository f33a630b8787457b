"""GPU parity of wf_project_publish: fused QKV projection + 3D rotary + paged
publication, then round attention on what it published, against the float64
oracle (project_qkv, rope_3d, attention_slot_prefix) on the same bf16 x and w.

Tolerances: the projection accumulates in fp32 and rounds once to bf16, so
q_rot and the K/V pages must lie within one bf16 ulp of the exact value plus
1e-3 (fp32 accumulation over 256-1536 terms); attention after it follows the
bf16 bounds of the attention tests (max-abs 2e-2 and rel-L2 1e-2 against the
oracle on bf16-rounded operands, rel-L2 1e-2 against the exact oracle)."""
import numpy as np
import pytest
import torch

import wf_inputs
from oracle import wf_oracle as O
from wf_test_utils import bf16_ulp, min_pages, pool_config, rel_l2, tensor_f64

import chunk_causal_wavefront_b200 as wfb

pytestmark = pytest.mark.gpu


def _weights(cfg, seed, scale_pow2):
    hidden = cfg.num_heads * cfg.head_dim
    bits = wf_inputs.draw_normal((3 * hidden, hidden), "bf16", seed, 4242)
    w = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16) * (2.0 ** -scale_pow2)
    return w.contiguous(), w.double().numpy()            # power-of-two scale: exact


def _x(cfg, rnd, layer):
    hidden = cfg.num_heads * cfg.head_dim
    bits = wf_inputs.draw_normal((cfg.num_slots, cfg.chunk_tokens, hidden), "bf16",
                                 cfg.seed, rnd, layer, 777)
    return bits, wf_inputs.bf16_bits_to_f64(bits)


class ProjRollout:
    def __init__(self, cfg, page_seed, w_pow2):
        self.cfg = cfg
        self.order = wf_inputs.draw_page_order(min_pages(cfg), page_seed)
        self.pool = wfb.KVPool(pool_config(cfg), device="cuda", page_order=self.order)
        shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
        self.q_rot = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        self.out = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        self.w_dev, self.w64 = _weights(cfg, 1, w_pow2)
        self.w_dev = self.w_dev.cuda()
        self.stored = {}       # chunk -> (k_rot64, v64) on the heads kept by the oracle
        self.heads = list(range(cfg.num_heads))

    def layout(self):
        c = self.cfg
        return O.round_layout(c.num_stages, c.anchor_chunks, c.history_chunks, self.pool.round)

    def step(self, heads=None):
        c = self.cfg
        hs = self.heads if heads is None else heads
        bits, x64 = _x(c, self.pool.round, 0)
        self.pool.project_publish(0, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda(),
                                  self.w_dev, self.q_rot)
        # oracle side: projection of the live slots on the kept heads
        hidden = c.num_heads * c.head_dim
        rows = np.concatenate([np.arange(sec * hidden + h * c.head_dim,
                                         sec * hidden + (h + 1) * c.head_dim)
                               for sec in range(3) for h in hs])
        w_sel = self.w64[rows]
        self.q, self.k, self.v = {}, {}, {}
        for p in self.layout():
            if p.slot is None:
                continue
            q, k, v = O.project_qkv(x64[p.slot], w_sel, len(hs), c.head_dim)
            rope = lambda a: O.rope_3d(a, p.chunk, c.frames_per_chunk, c.grid_h, c.grid_w,
                                       c.rope_split, c.rope_base)
            self.q[p.slot] = rope(q)
            self.k[p.chunk] = rope(k)
            self.v[p.chunk] = v
            if p.kind == "store":
                self.stored[p.chunk] = (self.k[p.chunk], v)
        for p in self.layout():
            if p.slot is None:
                self.k[p.chunk], self.v[p.chunk] = self.stored[p.chunk]

    def check_publish(self, heads, rows=None):
        c = self.cfg
        pages = self.pool.pages_view()[0]
        lay_gpu = self.pool.layout()
        tags = self.pool.tags_view()[0].cpu().numpy()
        for (kind, chunk, slot, tag, pgs), p in zip(lay_gpu, self.layout()):
            if slot is None:
                continue
            idx = torch.tensor(pgs, device="cuda")
            got = pages[idx].permute(1, 0, 3, 2, 4).reshape(2, -1, c.num_heads, c.head_dim)
            gk = tensor_f64(got[0, :c.chunk_tokens][:, heads])
            gv = tensor_f64(got[1, :c.chunk_tokens][:, heads])
            gq = tensor_f64(self.q_rot[slot][:, heads])
            for g, want in ((gq, self.q[slot]), (gk, self.k[chunk]), (gv, self.v[chunk])):
                if rows is not None:
                    g, want = g[rows], want[rows]
                assert (np.abs(g - want) <= bf16_ulp(want) + 1e-3).all(), (kind, slot)
            assert (got[:, c.chunk_tokens:].float() == 0).all()
            assert all(tags[g] == tag for g in pgs)

    def check_attention(self, heads, rows=None):
        lay = self.layout()
        q = {s: v for s, v in self.q.items()}
        want = O.attention_slot_prefix(q, self.k, self.v, lay, rows=rows)
        want_b = O.attention_slot_prefix({s: O.round_bf16(v) for s, v in q.items()},
                                         {c: O.round_bf16(v) for c, v in self.k.items()},
                                         {c: O.round_bf16(v) for c, v in self.v.items()},
                                         lay, rows=rows)
        out = tensor_f64(self.out)
        for s in want:
            g = out[s][:, heads] if rows is None else out[s][rows][:, heads]
            assert rel_l2(g, want[s]) <= 1e-2, s
            assert np.abs(g - want_b[s]).max() <= 2e-2 and rel_l2(g, want_b[s]) <= 1e-2, s


SMALL = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    num_stages=3, chunk_tokens=300, num_heads=2, history_chunks=2, frames_per_chunk=1,
    grid_h=10, grid_w=30)


def test_project_publish_small_every_round():
    ro = ProjRollout(SMALL, page_seed=3, w_pow2=4)      # hidden 256: w ~ N(0, 1/256)
    for k in range(SMALL.steady_round() + 2):
        ro.step()
        ro.pool.attention(0, ro.q_rot, ro.out)
        torch.cuda.synchronize()
        assert ro.pool.check_status() == 0
        ro.check_publish(list(range(SMALL.num_heads)))
        ro.check_attention(list(range(SMALL.num_heads)))
        ro.pool.advance()
    ro.pool.close()


def test_project_publish_full_size_sampled():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    ro = ProjRollout(cfg, page_seed=5, w_pow2=5)        # hidden 1536: w ~ N(0, 2^-10)
    heads = [0, 7]
    ro.heads = heads
    rows = np.array([0, 1, 127, 128, 1000, 4607, 4608, 4679])
    for k in range(cfg.steady_round() + 1):
        ro.step(heads)
        if k == cfg.steady_round():
            ro.pool.attention(0, ro.q_rot, ro.out)
            torch.cuda.synchronize()
            assert ro.pool.check_status() == 0
            ro.check_publish(heads, rows)
            ro.check_attention(heads, rows)
        else:
            ro.pool.advance()
    ro.pool.close()


def test_project_publish_rejects_fp32_pool():
    cfg = wf_inputs.CONFIGS["tiny_f32"]
    pool = wfb.KVPool(pool_config(cfg), device="cuda")
    x = torch.zeros(16, device="cuda")
    with pytest.raises(wfb.WfError) as e:
        pool.project_publish(0, x, x, x.clone())
    assert e.value.status == wfb.WF_ERR_UNSUPPORTED
    pool.close()
