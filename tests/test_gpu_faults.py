"""Failure detection on the GPU without faulting it.

The readiness check of the Method section (K/V must be published before
attention reads them) and the page bounds checks are exercised by planting the
error on the host side: a skipped publish leaves stale ready tags, and a test
hook writes an out-of-range id into the device page table. The kernels record
the error in the pool's status word and write nothing; no kernel traps or
faults.

The bounded waits of the tensor-core attention kernel are exercised the same
way: a test hook makes the next launch skip one K load, so the waits for that
tile can only run out, and shortens their limit to about 0.1 ms. Every CTA
whose context reaches that tile must record WF_ERR_TIMEOUT, drain its
in-flight copies and MMAs, free its tensor memory and write no output; CTAs
with shorter contexts finish normally; and the next launch on the same pool
must produce the same output as a launch before the stall."""
import numpy as np
import pytest
import torch

import wf_inputs
import chunk_causal_wavefront_b200 as wfb
from test_gpu_fp8 import Fp8Rollout
from wf_test_utils import Rollout

pytestmark = pytest.mark.gpu

CFG = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    num_stages=3, chunk_tokens=300, num_heads=2, frames_per_chunk=1, grid_h=10, grid_w=30)


@pytest.mark.parametrize("cfg", [CFG, wf_inputs.CONFIGS["tiny_f32"]], ids=["bf16", "f32"])
def test_attention_before_publish_is_not_ready(cfg):
    ro = Rollout(cfg, page_seed=1)
    for _ in range(cfg.steady_round()):
        ro.publish(0)
        ro.advance()
    # this round's publish is skipped: the pages hold last round's tags
    ro.attention(0, fill=7.0)
    assert ro.pool.check_status() == wfb.WF_ERR_NOT_READY
    assert (ro.out.float() == 7.0).all()
    assert ro.pool.check_status() == wfb.WF_OK            # status cleared after reading
    # publishing then attending works again
    ro.publish(0)
    ro.attention(0)
    assert ro.pool.check_status() == wfb.WF_OK
    assert torch.isfinite(ro.out.float()).all()
    ro.close()


def test_store_pages_recycled_without_publish_are_not_ready():
    # In steady state the store reuses the pages of the chunk that left the
    # history window; those pages carry that chunk's tag until republished.
    cfg = CFG
    ro = Rollout(cfg, page_seed=2)
    for _ in range(cfg.steady_round() + 1):
        ro.publish(0)
        ro.advance()
    q, k, v = wf_inputs.draw_round_inputs(cfg, ro.round, 0)
    # publish, then overwrite the store's tags with the recycled chunk's value
    ro.publish(0, inputs=(q, k, v))
    lay = ro.pool.layout()
    store = [r for r in lay if r[0] == "store"][0]
    tags = ro.pool.tags_view()
    tags[0, store[4][0]] = store[3] - (cfg.num_stages + 1)   # the previous round's tag
    ro.attention(0, fill=3.0)
    assert ro.pool.check_status() == wfb.WF_ERR_NOT_READY
    assert (ro.out.float() == 3.0).all()
    ro.close()


@pytest.mark.parametrize("cfg", [CFG, wf_inputs.CONFIGS["tiny_f32"]], ids=["bf16", "f32"])
def test_bad_page_id_is_caught(cfg):
    ro = Rollout(cfg, page_seed=1)
    for _ in range(cfg.steady_round()):
        ro.publish(0)
        ro.advance()
    ro.publish(0)
    ro.attention(0)
    assert ro.pool.check_status() == wfb.WF_OK
    ro.pool.poke_page(0, 0, 1 << 30)                     # anchor's first page -> out of range
    ro.attention(0, fill=5.0)
    assert ro.pool.check_status() == wfb.WF_ERR_BAD_PAGE
    assert (ro.out.float() == 5.0).all()
    last = len(ro.pool.layout()) - 1                     # slot 0, which publish writes
    ro.pool.poke_page(last, 0, -1)
    ro.publish(0)                                        # publish skips the bad page, flags it
    assert ro.pool.check_status() == wfb.WF_ERR_BAD_PAGE
    ro.advance()                                         # the next round rewrites the table
    ro.publish(0)
    ro.attention(0)
    assert ro.pool.check_status() == wfb.WF_OK
    ro.close()


def test_host_argument_errors():
    ro = Rollout(CFG, page_seed=1)
    p = ro.pool
    q = ro.q_rot
    from chunk_causal_wavefront_b200 import wf as W
    s = torch.cuda.current_stream().cuda_stream
    base = q.data_ptr()
    assert W.wf_publish_kv(p.handle, 1, base, base, base, ro.out.data_ptr(), s) == W.WF_ERR_INVALID_ARG
    assert W.wf_publish_kv(p.handle, -1, base, base, base, ro.out.data_ptr(), s) == W.WF_ERR_INVALID_ARG
    assert W.wf_publish_kv(p.handle, 0, base + 2, base, base, ro.out.data_ptr(), s) == W.WF_ERR_INVALID_ARG
    assert W.wf_publish_kv(p.handle, 0, base, base, base, base, s) == W.WF_ERR_INVALID_ARG
    assert W.wf_round_attention(p.handle, 0, base, base, s) == W.WF_ERR_INVALID_ARG
    assert W.wf_round_attention(p.handle, 0, base, ro.out.data_ptr() + 8, s) == W.WF_ERR_INVALID_ARG
    assert W.wf_round_attention(p.handle, 0, 0, ro.out.data_ptr(), s) == W.WF_ERR_INVALID_ARG
    assert p.check_status() == wfb.WF_OK
    ro.close()


def test_pool_memory_too_small_or_misaligned():
    from chunk_causal_wavefront_b200 import wf as W
    from wf_test_utils import pool_config
    c = pool_config(CFG)
    n = W.wf_kv_pool_bytes(c)
    mem = torch.empty(n + 512, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    with pytest.raises(W.WfError) as e:
        W.wf_kv_pool_create(c, mem.data_ptr(), n - 1, None, s)
    assert e.value.status == W.WF_ERR_INVALID_ARG
    with pytest.raises(W.WfError) as e:
        W.wf_kv_pool_create(c, mem.data_ptr() + 16, n, None, s)
    assert e.value.status == W.WF_ERR_INVALID_ARG


STALL_LIMIT = 200_000   # SM cycles: ~0.1 ms at 1.9 GHz


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("key_tile", [0, 5, 13])
def test_bounded_wait_runs_out(dtype, key_tile):
    # CFG: 3 pages per chunk; in a steady round the store reads 4 chunks (12
    # key tiles) and the denoising slots 5..7 chunks (15..21 tiles). Tile 0
    # stalls every CTA before its first MMA, tile 5 every CTA mid-stream with
    # copies and MMAs in flight, tile 13 every CTA except the store's.
    cfg = CFG.replace(rounds=8)
    ro = Fp8Rollout(cfg, page_seed=3) if dtype == "fp8" else Rollout(cfg, page_seed=3)
    for _ in range(cfg.steady_round()):
        ro.publish(0)
        ro.pool.advance()
    ro.publish(0)
    ro.attention(0)
    assert ro.pool.check_status() == wfb.WF_OK
    clean = ro.out.clone()
    lay = ro.pool.layout()
    tiles = {slot: (i + 1) * 3 for i, (kind, chunk, slot, tag, pgs) in enumerate(lay)
             if slot is not None}
    assert min(tiles.values()) == 12 and max(tiles.values()) == 21

    ro.pool.stall_next_attention(key_tile, STALL_LIMIT)
    ro.attention(0)                                       # fills out with NaN first
    assert ro.pool.check_status() == wfb.WF_ERR_TIMEOUT
    out = ro.out.float()
    for slot, n in tiles.items():
        if n > key_tile:
            assert torch.isnan(out[slot]).all(), (slot, n)   # gave up: nothing written
        else:
            assert torch.equal(ro.out[slot].view(torch.int16), clean[slot].view(torch.int16))
    assert ro.pool.check_status() == wfb.WF_OK            # status cleared after reading

    ro.attention(0)                                       # the hook lasted one launch
    assert ro.pool.check_status() == wfb.WF_OK
    for slot in tiles:
        assert torch.equal(ro.out[slot].view(torch.int16), clean[slot].view(torch.int16)), slot
    ro.close()


def test_stall_hook_arguments():
    ro = Rollout(CFG, page_seed=1)
    with pytest.raises(wfb.WfError) as e:
        ro.pool.stall_next_attention(-1, STALL_LIMIT)
    assert e.value.status == wfb.WF_ERR_INVALID_ARG
    with pytest.raises(wfb.WfError) as e:
        ro.pool.stall_next_attention(0, 10)               # below the minimum limit
    assert e.value.status == wfb.WF_ERR_INVALID_ARG
    ro.close()
    f32 = Rollout(wf_inputs.CONFIGS["tiny_f32"], page_seed=1)
    with pytest.raises(wfb.WfError) as e:
        f32.pool.stall_next_attention(0, STALL_LIMIT)
    assert e.value.status == wfb.WF_ERR_UNSUPPORTED
    f32.close()
