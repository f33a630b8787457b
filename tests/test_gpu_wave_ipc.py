"""Wave Parallelism across process boundaries: one process per rank (S + 1 = 3
ranks), as the pages' runtime runs one process per stage GPU (Method section
and Figure 3c of "Wave Forcing"; thelatestinai listing, Table 10).

Each process creates its own pool on cuda:0, exports the pool buffer with
wf_ipc_get_mem_handle, gathers the other ranks' handles over a gloo process
group and maps them with wf_ipc_open_mem. Every round, each live rank publishes
its slot, delivers it with wf_deliver_kv straight into the mapped pools of the
ranks that read it (wave_plan), synchronises its stream and meets the others
at a barrier; then each live rank runs wf_round_attention_slot, and a second
barrier keeps round k + 1's deliveries from overwriting pages that a round-k
attention is still reading. Rank 0 gathers every rank's output of its own
slot and checks it against the float64 oracle and, bit for bit, against a
single-pool run of the same rounds.

All ranks share one GPU here, so the copies stay in one device's memory; on
several GPUs the same calls store over NVLink. No kernel waits on another
process: ordering is done on the host (stream synchronisation + barriers)."""
import os
import sys
import traceback

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _rank_main(rank, world, port, dtype, mask, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path[:0] = [ROOT, os.path.join(ROOT, "tests")]
        import datetime

        import numpy as np
        import torch
        import torch.distributed as dist

        import wf_inputs
        from chunk_causal_wavefront_b200 import KVPool
        from chunk_causal_wavefront_b200 import wf as W
        from chunk_causal_wavefront_b200.wave import live_slots, wave_plan
        from test_gpu_fp8 import Fp8Rollout
        from wf_test_utils import Rollout, compare_with_oracle, min_pages, pool_config, to_device

        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        torch.cuda.set_device(0)
        S = world - 1
        cfg = wf_inputs.CONFIGS["wan13b_bf16"].replace(
            num_stages=S, chunk_tokens=300, num_heads=2, history_chunks=2, frames_per_chunk=1,
            grid_h=10, grid_w=30, rounds=9, mask=mask)
        order = wf_inputs.draw_page_order(min_pages(cfg), 5)
        pool = KVPool(pool_config(cfg, dtype=dtype), device="cuda", page_order=order)
        handles = [None] * world
        dist.all_gather_object(handles, pool.ipc_handle())
        peers = {r: (W.wf_ipc_open_mem(h, off), off) for r, (h, off) in enumerate(handles)
                 if r != rank}
        ref = None
        if rank == 0:   # single-pool run of the same rounds, with the oracle's view
            ref = (Fp8Rollout(cfg, page_seed=5) if dtype == "fp8" else Rollout(cfg, page_seed=5))
        shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
        q_rot = torch.zeros(shape, dtype=torch.uint8 if dtype == "fp8" else torch.bfloat16,
                            device="cuda")
        out = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        checked = 0
        for k in range(cfg.steady_round() + 3):
            live = live_slots(S, k)
            inputs = wf_inputs.draw_round_inputs(cfg, k, 0, slots=live)
            if rank in live:
                tq, tk, tv = (to_device(x, "bf16", torch.device("cuda")) for x in inputs)
                pool.publish_slot(0, rank, tq, tk, tv, q_rot)
                for r in wave_plan(S, k, mask).get(rank, []):
                    pool.deliver_to(0, rank, peers[r][0], pool.nbytes)
            torch.cuda.synchronize()
            dist.barrier()                       # every delivery of round k has landed
            mine = None
            if rank in live:
                out.fill_(float("nan"))
                pool.attention_slot(0, rank, q_rot, out)
                torch.cuda.synchronize()
                mine = out[rank].view(torch.int16).cpu().numpy()
            st = pool.check_status()
            dist.barrier()                       # round k's attention is done everywhere
            gathered = [None] * world
            dist.all_gather_object(gathered, (st, mine))
            if rank == 0:
                assert all(s == W.WF_OK for s, _ in gathered), (k, [s for s, _ in gathered])
                ref.publish(0, inputs=inputs)
                ref.attention(0)
                assert ref.pool.check_status() == 0
                single = ref.out.clone()
                ref.out = torch.full_like(single, float("nan"))
                for r in live:
                    got = torch.from_numpy(gathered[r][1]).view(torch.bfloat16).cuda()
                    assert torch.equal(got.view(torch.int16), single[r].view(torch.int16)), (k, r)
                    ref.out[r] = got
                if dtype == "fp8":
                    ref.check_attention()
                else:
                    compare_with_oracle(ref, range(cfg.num_heads), name=f"wave_ipc_{mask}")
                ref.pool.advance()
                checked += len(live)
            pool.advance()
        for ptr, off in peers.values():
            assert W.wf_ipc_close_mem(ptr, off) == W.WF_OK
        dist.barrier()                           # no rank frees its pool while mapped elsewhere
        pool.close()
        if ref is not None:
            ref.close()
        dist.destroy_process_group()
        q.put((rank, "ok", checked))
    except Exception:
        q.put((rank, "error", traceback.format_exc()))
        raise


@pytest.mark.parametrize("dtype,mask", [("bf16", "wf"), ("fp8", "rf")])
def test_wave_delivery_across_processes(dtype, mask):
    world = 3
    os.environ["PYTORCH_CUDA_ALLOC_CONF"] = "expandable_segments:False"   # IPC-exportable segments
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + (os.getpid() + (0 if dtype == "bf16" else 7)) % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, dtype, mask, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in procs:
            rank, status, info = q.get(timeout=300)
            res[rank] = (status, info)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.exitcode is None:
                p.kill()
    errors = {r: info for r, (status, info) in res.items() if status != "ok"}
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs)
    assert res[0][1] > 0                         # rank 0 checked some slots
