"""Wave Parallelism delivery plan (host logic, CPU).

The plan is checked against the oracle's own definition of what each query
slot reads (round_layout + visible_positions): over a rollout, every rank holds
every chunk its slot attends to, either because it published it (its own
slot), or because the owner delivered it in this round (live slots), or because
the store delivered it to every rank in its store round (anchor and history).
No rank receives a slot it does not read (except the store's chunk, which
every rank keeps for later rounds). The multi-process test runs the plan on
gloo ranks (one per slot), each computing its own sends, and checks that the
gathered sends are exactly what every rank needs."""
import ctypes
import os
import sys

import pytest
import torch.multiprocessing as mp

from oracle import wf_oracle as O
from chunk_causal_wavefront_b200.wave import live_slots, readers, wave_plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCHEDULES = [(1, 1, 0), (2, 1, 1), (3, 1, 2), (4, 1, 2), (5, 1, 3), (3, 0, 1), (4, 0, 0)]


def _needs(S, A, H, k, s, mask):
    """Chunks query slot s reads in round k, with the producing slot (None for stored)."""
    lay = O.round_layout(S, A, H, k)
    return [(lay[i].chunk, lay[i].slot, lay[i].kind) for i in O.visible_positions(lay, s, mask)]


@pytest.mark.parametrize("S,A,H", SCHEDULES)
@pytest.mark.parametrize("mask", ["wf", "rf"])
def test_every_rank_holds_what_its_slot_reads(S, A, H, mask):
    held = {r: set() for r in range(S + 1)}          # chunks in each rank's pool
    for k in range(S + H + 6):
        plan = wave_plan(S, k, mask)
        assert sorted(plan) == live_slots(S, k)
        lay = O.round_layout(S, A, H, k)
        chunk_of = {p.slot: p.chunk for p in lay if p.slot is not None}
        # this round's publications and deliveries
        for j, dsts in plan.items():
            held[j].add(chunk_of[j])
            assert j not in dsts
            for r in dsts:
                held[r].add(chunk_of[j])
        for s in live_slots(S, k):
            for chunk, producer, kind in _needs(S, A, H, k, s, mask):
                assert chunk in held[s], (k, s, chunk, kind)
                if producer is not None and producer != s:
                    # a live slot's chunk reaches s only through this round's plan
                    assert s in plan[producer], (k, s, producer)


@pytest.mark.parametrize("S,A,H", SCHEDULES)
def test_no_delivery_to_a_rank_that_does_not_read_it(S, A, H):
    for k in range(S + H + 6):
        for j, dsts in wave_plan(S, k, "wf").items():
            if j == S:
                assert sorted(dsts) == list(range(S))     # the store goes everywhere
                continue
            for r in dsts:
                seen = [p for _, p, _ in _needs(S, A, H, k, r, "wf")]
                assert j in seen, (k, j, r)


def test_plan_small_cases_by_hand():
    # S = 2: round 0 only slot 0 is live; round 1 slots 0, 1; round 2 adds the store
    assert wave_plan(2, 0) == {0: []}
    assert wave_plan(2, 1) == {0: [], 1: [0]}
    assert wave_plan(2, 2) == {0: [], 1: [0], 2: [0, 1]}
    assert wave_plan(2, 2, "rf") == {0: [1, 2], 1: [0, 2], 2: [0, 1]}   # the store reads all
    assert readers(2, 0, 1) == []                         # slot 1 not live yet
    with pytest.raises(ValueError):
        readers(2, 3, 1, "bogus")


def _rank(rank, world, port, rounds, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from chunk_causal_wavefront_b200.wave import wave_plan as plan
    S = world - 1
    sends = [(k, rank, r) for k in range(rounds) for r in plan(S, k).get(rank, [])]
    allsends = [None] * world
    dist.all_gather_object(allsends, sends)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, allsends))


@pytest.mark.parametrize("world", [2, 4])
def test_plan_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + world) % 1000
    rounds = 12
    procs = [ctx.Process(target=_rank, args=(r, world, port, rounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    S = world - 1
    gathered = [sorted(sum(res[r], [])) for r in range(world)]
    assert all(g == gathered[0] for g in gathered)        # every rank sees the same sends
    received = {r: {(k, src) for k, src, dst in gathered[0] if dst == r} for r in range(world)}
    for k in range(rounds):
        for s in live_slots(S, k):
            lay = O.round_layout(S, 1, 2, k)
            for i in O.visible_positions(lay, s):
                j = lay[i].slot
                if j is not None and j != s:
                    assert (k, j) in received[s], (k, s, j)


# Delivery writes a slot's pages at the same physical ids in the receiver's
# pool, which holds only because every rank's bookkeeping is the same
# function of (config, page order, round). Host-only pools (no device memory)
# run that bookkeeping here.
def _layouts(cfg, order, rounds):
    import chunk_causal_wavefront_b200 as wfb
    from wf_test_utils import pool_config
    pool = wfb.KVPool(pool_config(cfg, max_rounds=rounds + 2), page_order=order)
    out = []
    for _ in range(rounds):
        out.append(pool.layout())
        pool.advance()
    pool.close()
    return out


def test_rank_pools_keep_identical_page_tables():
    import wf_inputs
    from wf_test_utils import min_pages
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    order = wf_inputs.draw_page_order(min_pages(cfg), 5)
    ranks = [_layouts(cfg, order, 60) for _ in range(cfg.num_stages + 1)]
    assert all(r == ranks[0] for r in ranks)
    # and the pages the plan hands over in a steady round are the slot's own pages
    lay = ranks[0][cfg.steady_round()]
    pages = {slot: pg for kind, chunk, slot, tag, pg in lay if slot is not None and slot >= 0}
    assert sorted(pages) == live_slots(cfg.num_stages, cfg.steady_round())
    flat = [p for pg in pages.values() for p in pg]
    assert len(flat) == len(set(flat))                    # no page shared between slots


def test_wave_calls_on_host_only_pools():
    import wf_inputs
    import chunk_causal_wavefront_b200 as wfb
    from chunk_causal_wavefront_b200 import wf as W
    from wf_test_utils import pool_config
    cfg = wf_inputs.CONFIGS["tiny_f32"]
    pool = wfb.KVPool(pool_config(cfg))
    assert W.wf_publish_kv_slot(pool.handle, 0, 0, 16, 16, 16, 32, 0) == W.WF_ERR_CALL_ORDER
    assert W.wf_publish_kv_slot(pool.handle, 0, -1, 16, 16, 16, 32, 0) == W.WF_ERR_INVALID_ARG
    assert W.wf_round_attention_slot(pool.handle, 0, 0, 16, 32, 0) == W.WF_ERR_CALL_ORDER
    assert W.wf_round_attention_slot(pool.handle, 0, -1, 16, 32, 0) == W.WF_ERR_INVALID_ARG
    assert W.wf_deliver_kv(pool.handle, 0, 0, 256, pool.nbytes, 0) == W.WF_ERR_CALL_ORDER
    assert W.wf_deliver_kv(pool.handle, 0, 0, None, pool.nbytes, 0) == W.WF_ERR_INVALID_ARG
    assert W.lib().wf_deliver_kv(None, 0, 0, None, 0, None) == W.WF_ERR_INVALID_ARG
    # the stall hook needs a device pool with a tensor-core attention path
    assert W.wf_pool_debug_stall_next_attention(pool.handle, 0, 10**6) == W.WF_ERR_CALL_ORDER
    assert W.lib().wf_pool_debug_stall_next_attention(None, 0, 10**6) == W.WF_ERR_INVALID_ARG
    pool.close()


def test_ipc_calls_reject_bad_arguments():
    # Argument checks only: no CUDA context is needed to refuse these.
    from chunk_causal_wavefront_b200 import wf as W
    h = W.WfIpcHandle()
    off = ctypes.c_size_t(0)
    ptr = ctypes.c_void_p(0)
    assert W.lib().wf_ipc_get_mem_handle(None, ctypes.byref(h), ctypes.byref(off)) == W.WF_ERR_INVALID_ARG
    assert W.lib().wf_ipc_get_mem_handle(256, None, ctypes.byref(off)) == W.WF_ERR_INVALID_ARG
    assert W.lib().wf_ipc_open_mem(None, 0, ctypes.byref(ptr)) == W.WF_ERR_INVALID_ARG
    assert W.lib().wf_ipc_open_mem(ctypes.byref(h), 0, None) == W.WF_ERR_INVALID_ARG
    assert W.lib().wf_ipc_close_mem(None, 0) == W.WF_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        W.wf_ipc_open_mem(b"short", 0)


def _rank_tables(rank, world, port, q):
    import hashlib
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import wf_inputs
    from wf_test_utils import min_pages
    cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(num_stages=world - 1)
    order = wf_inputs.draw_page_order(min_pages(cfg), 11)
    digest = [hashlib.sha256(repr(l).encode()).hexdigest() for l in _layouts(cfg, order, 40)]
    got = [None] * world
    dist.all_gather_object(got, digest)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got))


def test_page_tables_agree_across_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = 3
    port = 29700 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_tables, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert all(d == res[r][0] for d in res[r])         # all ranks: same tables, every round
