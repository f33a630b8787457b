"""GPU parity of wf_publish_kv: rotary embedding and paged scatter.

Page placement and V contents are checked bit-exactly against the oracle's
page-table model; rotated K and q_rot bit for bit against the oracle's float32
rotation rounded once to the pool's dtype, and within one bf16 ulp (fp32: 1e-5
absolute) of the float64 rotation, at the full 1.3B-shaped size."""
import numpy as np
import pytest
import torch

import wf_inputs
from oracle import wf_oracle as O
from oracle import wf_fp8 as F8
from wf_test_utils import Rollout, bf16_ulp, min_pages, tensor_f64, to_f64

pytestmark = pytest.mark.gpu


def _model(ro: Rollout):
    c = ro.cfg
    m = O.PoolModel(c.num_stages, c.anchor_chunks, c.history_chunks, c.pages_per_chunk,
                    min_pages(c), ro.page_order)
    for _ in range(ro.round):
        m.advance()
    return m


def _check_round(ro: Rollout, layer: int = 0, full_rope_check: bool = True):
    c = ro.cfg
    pages = ro.pool.pages_view()[layer]                   # [num_pages][2][Hh][P][d]
    tags = ro.pool.tags_view()[layer].cpu().numpy()
    model = _model(ro)
    P, C = c.page_tokens, c.chunk_tokens
    npc = c.pages_per_chunk
    for p, pgs, tag in model.table():
        if p.slot is None:
            continue
        q, k, v, chunk = ro.live[layer][p.slot]
        assert chunk == p.chunk
        idx = torch.tensor(pgs, device=ro.device)
        got = pages[idx]                                  # [npc][2][Hh][P][d]
        flat = got.permute(1, 0, 3, 2, 4).reshape(2, npc * P, c.num_heads, c.head_dim)
        # V: bit-exact copy into the slot's pages, in page-table order
        vw = torch.from_numpy(v.view(np.int16) if c.dtype == "bf16" else v.view(np.int32))
        gv = flat[1, :C].contiguous().view(torch.int16 if c.dtype == "bf16" else torch.int32)
        assert torch.equal(gv.cpu(), vw), p
        # rows past the end of the chunk are zero (K and V)
        assert (flat[:, C:].float() == 0).all(), p
        # ready tags of every page of this slot
        assert all(tags[g] == tag for g in pgs), p
        if full_rope_check:
            k64 = to_f64(k, c.dtype)
            q64 = to_f64(q, c.dtype)
            if c.rope:
                k64 = O.rope_3d(k64, chunk, c.frames_per_chunk, c.grid_h, c.grid_w, c.rope_split,
                                c.rope_base)
                q64 = O.rope_3d(q64, chunk, c.frames_per_chunk, c.grid_h, c.grid_w, c.rope_split,
                                c.rope_base)
            gk = tensor_f64(flat[0, :C])
            gq = tensor_f64(ro.q_rot[p.slot])
            if c.dtype == "bf16":
                # fp32 math + one rounding: within one bf16 ulp of the exact value
                assert (np.abs(gk - k64) <= bf16_ulp(k64) + 1e-6).all(), p
                assert (np.abs(gq - q64) <= bf16_ulp(q64) + 1e-6).all(), p
            else:
                assert np.abs(gk - k64).max() <= 1e-5, p
                assert np.abs(gq - q64).max() <= 1e-5, p
            if c.rope:
                # bit for bit: the oracle's float32 rotation (each product and
                # sum rounded once), then one rounding to the pool's dtype
                for got, x in ((gk, k), (gq, q)):
                    r32 = F8.rope_3d_f32(to_f64(x, c.dtype).astype(np.float32), chunk,
                                         c.frames_per_chunk, c.grid_h, c.grid_w, c.rope_split,
                                         c.rope_base).astype(np.float64)
                    want = O.round_bf16(r32) if c.dtype == "bf16" else r32
                    assert np.array_equal(got, want), (p, int((got != want).sum()))
            if not c.rope:
                assert np.array_equal(gk, k64) and np.array_equal(gq, q64)


def test_publish_full_size_steady_round():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    ro = Rollout(cfg, page_seed=11)
    for _ in range(cfg.steady_round()):
        ro.advance()
    ro.publish(0)
    torch.cuda.synchronize()
    assert ro.pool.check_status() == 0
    _check_round(ro)
    ro.close()


def test_publish_fill_round_leaves_idle_rows():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(chunk_tokens=3 * 10 * 13, grid_h=10, grid_w=13)
    ro = Rollout(cfg, page_seed=5)
    ro.advance()                                          # round 1: slots 0 and 1 live
    ro.q_rot.fill_(float("nan"))
    ro.publish(0)
    torch.cuda.synchronize()
    _check_round(ro)
    assert torch.isnan(ro.q_rot[2:].float()).all()        # idle slots untouched
    assert not torch.isnan(ro.q_rot[:2].float()).any()
    ro.close()


@pytest.mark.parametrize("rope", [0, 1])
def test_publish_f32(rope):
    cfg = wf_inputs.CONFIGS["tiny_f32"].replace(
        rope=rope, chunk_tokens=2 * 6 * 10, frames_per_chunk=2, grid_h=6, grid_w=10,
        rope_split=(24, 20, 20), page_tokens=48)
    ro = Rollout(cfg, page_seed=2)
    for _ in range(cfg.steady_round()):
        ro.advance()
    ro.publish(0)
    torch.cuda.synchronize()
    _check_round(ro)
    ro.close()


def test_publish_rope_off_bf16_is_bitwise_copy():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(rope=0, chunk_tokens=300, grid_h=10, grid_w=30,
                                                   frames_per_chunk=1, num_heads=3)
    ro = Rollout(cfg, page_seed=1)
    for _ in range(5):
        ro.advance()
    ro.publish(0)
    torch.cuda.synchronize()
    _check_round(ro)
    ro.close()


def test_publish_second_layer_independent():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(chunk_tokens=3 * 10 * 13, grid_h=10, grid_w=13,
                                                   num_layers=3)
    ro = Rollout(cfg, page_seed=9)
    for _ in range(cfg.steady_round()):
        ro.advance()
    ro.publish(2)
    torch.cuda.synchronize()
    _check_round(ro, layer=2)
    # layers 0 and 1 were never written: their tags are still zero
    tags = ro.pool.tags_view().cpu().numpy()
    assert (tags[0] == 0).all() and (tags[1] == 0).all()
    ro.close()


# The bf16 publish for 128-token pages moves half pages (64 rows) through TMA:
# chunks that end exactly on or inside either half of a page, or below one
# half, and one that fills its pages exactly.
@pytest.mark.parametrize("C,gh,gw", [(40, 5, 8), (64, 8, 8), (100, 10, 10), (192, 12, 16),
                                     (256, 16, 16)])
def test_publish_half_page_boundaries(C, gh, gw):
    cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(
        num_stages=3, chunk_tokens=C, num_heads=3, history_chunks=1, frames_per_chunk=1,
        grid_h=gh, grid_w=gw)
    ro = Rollout(cfg, page_seed=C)
    for _ in range(cfg.steady_round()):
        ro.advance()
    ro.publish(0)
    torch.cuda.synchronize()
    assert ro.pool.check_status() == 0
    _check_round(ro)
    ro.close()

