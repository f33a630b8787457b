"""Failure detection on the GPU without faulting it.

The readiness check of the Method section (K/V must be published before
attention reads them) and the page bounds checks are exercised by planting the
error on the host side: a skipped publish leaves stale ready tags, and a test
hook writes an out-of-range id into the device page table. The kernels record
the error in the pool's status word and write nothing; no kernel traps,
faults or waits on a flag that is never set."""
import numpy as np
import pytest
import torch

import wf_inputs
import chunk_causal_wavefront_b200 as wfb
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
