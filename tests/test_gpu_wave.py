"""Wave Parallelism on one GPU: one pool per rank, every rank publishing and
attending its own slot and delivering its pages to the ranks that read them
(wf_publish_kv_slot, wf_deliver_kv, wf_round_attention_slot, following
wave_plan). The ranks' pools live on the same device here (the delivery
kernel stores through a plain device pointer either way; on several GPUs the
pointer is a peer's buffer). Each rank's output of its slot must equal,
bit for bit, the single-pool path's output of that slot, every round, for both
masks and for bf16 and FP8 pools; the single-pool path is itself checked
against the float64 oracle in test_gpu_attention.py and test_gpu_fp8.py.

A skipped delivery must surface as WF_ERR_NOT_READY on the receiving rank,
and delivering a slot that was not published in this round as
WF_ERR_NOT_READY on the sender, with nothing written to the receiver."""
import pytest
import torch

import wf_inputs
from chunk_causal_wavefront_b200 import KVPool
from chunk_causal_wavefront_b200 import wf as W
from chunk_causal_wavefront_b200.wave import live_slots, wave_plan
from wf_test_utils import min_pages, pool_config, to_device

pytestmark = pytest.mark.gpu

SMALL = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    num_stages=3, chunk_tokens=300, num_heads=2, history_chunks=2, frames_per_chunk=1,
    grid_h=10, grid_w=30, rounds=9)


class Wave:
    """S + 1 rank pools plus one single-pool reference, all on cuda:0."""

    def __init__(self, cfg, dtype, mask):
        self.cfg, self.S = cfg, cfg.num_stages
        order = wf_inputs.draw_page_order(min_pages(cfg), 5)
        pc = pool_config(cfg, dtype=dtype, mask=mask)
        self.ref = KVPool(pc, device="cuda", page_order=order)
        self.ranks = [KVPool(pc, device="cuda", page_order=order) for _ in range(self.S + 1)]
        shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
        qdt = torch.uint8 if dtype == "fp8" else torch.bfloat16
        self.ref_q, self.ref_out = torch.zeros(shape, dtype=qdt, device="cuda"), \
            torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        self.q = [torch.zeros(shape, dtype=qdt, device="cuda") for _ in self.ranks]
        self.out = [torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
                    for _ in self.ranks]
        self.mask = mask

    def inputs(self, k):
        q, kk, v = wf_inputs.draw_round_inputs(self.cfg, k, 0, slots=live_slots(self.S, k))
        return [to_device(x, "bf16", torch.device("cuda")) for x in (q, kk, v)]

    def round(self, k, skip=None):
        tq, tk, tv = self.inputs(k)
        self.ref.publish(0, tq, tk, tv, self.ref_q)
        self.ref.attention(0, self.ref_q, self.ref_out)
        for r in live_slots(self.S, k):
            self.ranks[r].publish_slot(0, r, tq, tk, tv, self.q[r])
        for j, dsts in wave_plan(self.S, k, self.mask).items():
            for r in dsts:
                if skip != (j, r):
                    self.ranks[j].deliver(0, j, self.ranks[r])
        for r in live_slots(self.S, k):
            self.ranks[r].attention_slot(0, r, self.q[r], self.out[r])
        torch.cuda.synchronize()

    def advance(self):
        self.ref.advance()
        for p in self.ranks:
            p.advance()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("mask", ["wf", "rf"])
def test_wave_ranks_match_single_pool(dtype, mask):
    w = Wave(SMALL, dtype, mask)
    for k in range(SMALL.steady_round() + 3):
        w.round(k)
        assert w.ref.check_status() == 0
        for r in range(w.S + 1):
            assert w.ranks[r].check_status() == 0, (k, r)
        for r in live_slots(w.S, k):
            got = w.out[r][r].view(torch.int16)
            want = w.ref_out[r].view(torch.int16)
            assert torch.equal(got, want), (k, r)
            if dtype == "bf16":
                assert torch.equal(w.q[r][r].view(torch.int16), w.ref_q[r].view(torch.int16))
            else:
                assert torch.equal(w.q[r][r], w.ref_q[r])
        w.advance()


def test_wave_missing_delivery_is_not_ready():
    w = Wave(SMALL, "bf16", "wf")
    k_steady = SMALL.steady_round()
    for k in range(k_steady):
        w.round(k)
        w.advance()
    # round k_steady: the store's pages never reach rank 0
    w.out[0].fill_(float("nan"))
    w.round(k_steady, skip=(w.S, 0))
    assert w.ranks[0].check_status() == W.WF_ERR_NOT_READY
    for r in range(1, w.S + 1):
        assert w.ranks[r].check_status() == 0
    assert torch.isnan(w.out[0][0].float()).all()           # no output written


def test_wave_deliver_of_unpublished_slot_is_not_ready():
    w = Wave(SMALL, "bf16", "wf")
    for k in range(3):
        w.round(k)
        w.advance()
    # round 3: slot 1 is live but not yet published in this round
    before = w.ranks[0].pages_view()[0].view(torch.int16).clone()      # bit patterns
    tags0 = w.ranks[0].tags_view()[0].clone()
    w.ranks[1].deliver(0, 1, w.ranks[0])
    torch.cuda.synchronize()
    assert w.ranks[1].check_status() == W.WF_ERR_NOT_READY
    assert torch.equal(w.ranks[0].pages_view()[0].view(torch.int16), before)
    assert torch.equal(w.ranks[0].tags_view()[0], tags0)
    # argument checks on the host
    with pytest.raises(W.WfError):
        w.ranks[1].deliver(0, 1, w.ranks[1])                # receiver is the sender
    with pytest.raises(W.WfError):
        w.ranks[1].deliver(0, w.S + 1, w.ranks[0])          # no such slot
