"""Wave Parallelism on one GPU: one pool per rank, every rank publishing and
attending its own slot and delivering its pages to the ranks that read them
(wf_publish_kv_slot, wf_deliver_kv, wf_round_attention_slot, following
wave_plan). The ranks' pools live on the same device here (the delivery
kernel stores through a plain device pointer either way; on several GPUs the
pointer is a peer's buffer, and test_gpu_wave_ipc.py delivers across process
boundaries).

Every round, each rank's output of its slot is compared with the float64
oracle (bf16 tolerances, or the derived E4M3 bounds for FP8 pools), and must
also equal, bit for bit, the single-pool path's output of that slot, for both
masks and for bf16 and FP8 pools.

A skipped delivery must surface as WF_ERR_NOT_READY on the receiving rank,
delivering a slot that was not published in this round as WF_ERR_NOT_READY on
the sender with nothing written to the receiver (pages, tags and, for FP8
pools, block scales), and a receiver with another config or page order as
WF_ERR_INVALID_ARG on the sender, again with the receiver untouched."""
import pytest
import torch

import wf_inputs
from chunk_causal_wavefront_b200 import KVPool
from chunk_causal_wavefront_b200 import wf as W
from chunk_causal_wavefront_b200.wave import live_slots, wave_plan
from test_gpu_fp8 import Fp8Rollout
from wf_test_utils import Rollout, compare_with_oracle, min_pages, pool_config, to_device

pytestmark = pytest.mark.gpu

SMALL = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    num_stages=3, chunk_tokens=300, num_heads=2, history_chunks=2, frames_per_chunk=1,
    grid_h=10, grid_w=30, rounds=9)
PAGE_SEED = 5


class Wave:
    """S + 1 rank pools plus one single-pool rollout (with the oracle's view of
    the same rounds), all on cuda:0."""

    def __init__(self, cfg, dtype, mask):
        self.cfg, self.S, self.dtype, self.mask = cfg.replace(mask=mask), cfg.num_stages, dtype, mask
        self.ro = (Fp8Rollout(self.cfg, page_seed=PAGE_SEED) if dtype == "fp8"
                   else Rollout(self.cfg, page_seed=PAGE_SEED))
        order = wf_inputs.draw_page_order(min_pages(self.cfg), PAGE_SEED)
        pc = pool_config(self.cfg, dtype=dtype)
        self.ranks = [KVPool(pc, device="cuda", page_order=order) for _ in range(self.S + 1)]
        shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
        qdt = torch.uint8 if dtype == "fp8" else torch.bfloat16
        self.q = [torch.zeros(shape, dtype=qdt, device="cuda") for _ in self.ranks]
        self.out = [torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
                    for _ in self.ranks]

    def round(self, k, skip=None):
        inputs = wf_inputs.draw_round_inputs(self.cfg, k, 0, slots=live_slots(self.S, k))
        self.ro.publish(0, inputs=inputs)
        self.ro.attention(0)
        tq, tk, tv = (to_device(x, "bf16", torch.device("cuda")) for x in inputs)
        for r in live_slots(self.S, k):
            self.ranks[r].publish_slot(0, r, tq, tk, tv, self.q[r])
        for j, dsts in wave_plan(self.S, k, self.mask).items():
            for r in dsts:
                if skip != (j, r):
                    self.ranks[j].deliver(0, j, self.ranks[r])
        for r in live_slots(self.S, k):
            self.out[r].fill_(float("nan"))
            self.ranks[r].attention_slot(0, r, self.q[r], self.out[r])
        torch.cuda.synchronize()

    def check_against_oracle(self, k):
        """Each live rank's rows of its own slot, gathered into the rollout's
        output tensor, against the float64 oracle."""
        gathered = torch.full_like(self.ro.out, float("nan"))
        for r in live_slots(self.S, k):
            gathered[r] = self.out[r][r]
        self.ro.out = gathered
        heads = range(self.cfg.num_heads)
        if self.dtype == "fp8":
            self.ro.check_attention(heads=heads)
        else:
            compare_with_oracle(self.ro, heads, name=f"wave_{self.mask}")

    def advance(self):
        self.ro.pool.advance()
        for p in self.ranks:
            p.advance()

    def close(self):
        self.ro.close()
        for p in self.ranks:
            p.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("mask", ["wf", "rf"])
def test_wave_ranks_match_oracle_and_single_pool(dtype, mask):
    w = Wave(SMALL, dtype, mask)
    for k in range(SMALL.steady_round() + 3):
        w.round(k)
        assert w.ro.pool.check_status() == 0
        for r in range(w.S + 1):
            assert w.ranks[r].check_status() == 0, (k, r)
        ref_out = w.ro.out.clone()
        for r in live_slots(w.S, k):
            assert torch.equal(w.out[r][r].view(torch.int16), ref_out[r].view(torch.int16)), (k, r)
            if dtype == "bf16":
                assert torch.equal(w.q[r][r].view(torch.int16), w.ro.q_rot[r].view(torch.int16))
            else:
                assert torch.equal(w.q[r][r], w.ro.q_rot[r])
        w.check_against_oracle(k)
        w.advance()
    w.close()


def _receiver_state(pool, dtype):
    state = [pool.pages_view()[0].view(torch.uint8).clone(), pool.tags_view()[0].clone()]
    if dtype == "fp8":
        state.append(pool.kv_scales_view()[0].clone())
    return state


def _same_state(a, b):
    return all(torch.equal(x, y) for x, y in zip(a, b))


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("mask", ["wf", "rf"])
def test_wave_missing_delivery_is_not_ready(dtype, mask):
    w = Wave(SMALL, dtype, mask)
    k_steady = SMALL.steady_round()
    for k in range(k_steady):
        w.round(k)
        w.advance()
    # round k_steady: the store's pages never reach rank 0 (which reads the
    # store under both masks)
    w.round(k_steady, skip=(w.S, 0))
    assert w.ranks[0].check_status() == W.WF_ERR_NOT_READY
    for r in range(1, w.S + 1):
        assert w.ranks[r].check_status() == 0
    assert torch.isnan(w.out[0][0].float()).all()           # no output written
    w.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("mask", ["wf", "rf"])
def test_wave_deliver_of_unpublished_slot_is_not_ready(dtype, mask):
    w = Wave(SMALL, dtype, mask)
    for k in range(3):
        w.round(k)
        w.advance()
    # round 3: slot 1 is live but not yet published in this round
    before = _receiver_state(w.ranks[0], dtype)
    w.ranks[1].deliver(0, 1, w.ranks[0])
    torch.cuda.synchronize()
    assert w.ranks[1].check_status() == W.WF_ERR_NOT_READY
    assert _same_state(_receiver_state(w.ranks[0], dtype), before)
    # argument checks on the host
    with pytest.raises(W.WfError):
        w.ranks[1].deliver(0, 1, w.ranks[1])                # receiver is the sender
    with pytest.raises(W.WfError):
        w.ranks[1].deliver(0, w.S + 1, w.ranks[0])          # no such slot
    with pytest.raises(W.WfError) as e:                     # receiver of another size
        w.ranks[1].deliver_to(0, 1, w.ranks[0].mem.data_ptr(), w.ranks[0].nbytes - 256)
    assert e.value.status == W.WF_ERR_INVALID_ARG
    w.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_wave_deliver_into_foreign_pool_is_refused(dtype):
    # Same size, different page order: the receiver's signature does not match,
    # so the sender records WF_ERR_INVALID_ARG and writes nothing.
    cfg = SMALL
    pc = pool_config(cfg, dtype=dtype)
    order = wf_inputs.draw_page_order(min_pages(cfg), PAGE_SEED)
    sender = KVPool(pc, device="cuda", page_order=order)
    other = KVPool(pc, device="cuda", page_order=order[::-1].copy())
    assert sender.nbytes == other.nbytes
    inputs = wf_inputs.draw_round_inputs(cfg, 0, 0, slots=[0])
    tq, tk, tv = (to_device(x, "bf16", torch.device("cuda")) for x in inputs)
    q_rot = torch.zeros((cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim),
                        dtype=torch.uint8 if dtype == "fp8" else torch.bfloat16, device="cuda")
    sender.publish_slot(0, 0, tq, tk, tv, q_rot)
    before = _receiver_state(other, dtype)
    sender.deliver(0, 0, other)
    torch.cuda.synchronize()
    assert sender.check_status() == W.WF_ERR_INVALID_ARG
    assert other.check_status() == 0
    assert _same_state(_receiver_state(other, dtype), before)
    sender.close()
    other.close()
