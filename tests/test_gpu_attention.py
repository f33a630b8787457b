"""GPU parity of wf_round_attention against the float64 oracle.

Tolerances: fp32 max-abs 1e-5; bf16 max-abs 2e-2 and relative L2 1e-2, against
the oracle fed the exact inputs and, separately, against the oracle run on q_rot
and K rounded to bf16 by the oracle itself (which isolates the attention
kernel's error from the rounding of the published format). Small cases cover
every round of fill and steady state with several key tiles and ragged tails.
Full-size cases run the launch configuration that bench.py times: every row of
two heads of the 1.3B-shaped layer and of one head of the 14B-shaped layer,
sampled rows of the other configs, and a context longer than the kernel's
1024-entry page-id cache (its uncached path)."""
import numpy as np
import pytest
import torch

import wf_inputs
from oracle import wf_oracle as O
from wf_test_utils import Rollout, rel_l2, tensor_f64
from wf_test_utils import compare_with_oracle as _compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [
    wf_inputs.CONFIGS["tiny_f32"],
    wf_inputs.CONFIGS["tiny_f32"].replace(mask="rf"),
    # the largest stage count the ABI accepts: 17 live query slots
    wf_inputs.CONFIGS["tiny_f32"].replace(num_stages=16, rounds=24),
], ids=["wf", "rf", "S16"])
def test_tiny_f32_every_round(cfg):
    ro = Rollout(cfg, page_seed=0)
    for k in range(cfg.rounds + 3):
        ro.publish(0)
        ro.attention(0)
        torch.cuda.synchronize()
        assert ro.pool.check_status() == 0
        _compare(ro, range(cfg.num_heads), gpu_operands=False, name="tiny_f32")
        ro.advance()
    ro.close()


SMALL_BF16 = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    num_stages=3, chunk_tokens=300, num_heads=2, history_chunks=2, frames_per_chunk=1,
    grid_h=10, grid_w=30, rounds=9)


@pytest.mark.parametrize("cfg", [
    SMALL_BF16,
    SMALL_BF16.replace(anchor_chunks=0, history_chunks=1, chunk_tokens=3 * 4 * 11,
                       frames_per_chunk=3, grid_h=4, grid_w=11),
    SMALL_BF16.replace(num_stages=1, history_chunks=0, chunk_tokens=128, grid_h=8, grid_w=16),
    SMALL_BF16.replace(chunk_tokens=1, grid_h=1, grid_w=1),
    SMALL_BF16.replace(mask="rf"),
    SMALL_BF16.replace(mask="rf", anchor_chunks=0, history_chunks=1, chunk_tokens=3 * 4 * 11,
                       frames_per_chunk=3, grid_h=4, grid_w=11),
    # the largest stage count the ABI accepts: 17 live query slots
    SMALL_BF16.replace(num_stages=16, chunk_tokens=130, grid_h=10, grid_w=13, history_chunks=3,
                       rounds=24),
    SMALL_BF16.replace(num_stages=16, chunk_tokens=130, grid_h=10, grid_w=13, history_chunks=3,
                       rounds=24, mask="rf"),
], ids=["S3_C300", "noanchor_C132", "S1_C128", "C1", "rf_S3_C300", "rf_noanchor_C132",
        "S16_C130", "rf_S16_C130"])
def test_bf16_every_round_small(cfg):
    ro = Rollout(cfg, page_seed=4)
    for k in range(cfg.steady_round() + 3):
        ro.publish(0)
        ro.attention(0)
        torch.cuda.synchronize()
        assert ro.pool.check_status() == 0
        _compare(ro, range(cfg.num_heads), name="small_bf16")
        ro.advance()
    ro.close()


def _steady(cfg, page_seed=7, real_only_store=True):
    """Run a full-size rollout to its first steady round (publishing only the
    store before it, since denoising slots re-publish every round)."""
    ro = Rollout(cfg, page_seed=page_seed)
    S = cfg.num_stages
    for k in range(cfg.steady_round()):
        if k >= S:
            ro.publish(0, real_slots=[S] if real_only_store else None)
        ro.advance()
    ro.publish(0)
    ro.attention(0)
    torch.cuda.synchronize()
    assert ro.pool.check_status() == 0
    return ro


def _sample_rows(C, n, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(C, size=n - 6, replace=False).tolist())
    rows |= {0, 127, 128, C - 73, C - 72, C - 1}        # tile edges and the ragged tail
    return np.array(sorted(rows))


@pytest.mark.parametrize("name,heads", [("wan13b_bf16", (0, 11)), ("wan14b_bf16", (17,)),
                                        ("wan13b_5step_bf16", (3,)), ("wan13b_bf16_rf", (5,))])
def test_full_size_all_rows(name, heads):
    # Every query row of every live slot of the listed heads: 19 tile pairs
    # per (slot, head) in the full grid's launch order, against the oracle.
    cfg = (wf_inputs.CONFIGS["wan13b_bf16"].replace(mask="rf") if name.endswith("_rf")
           else wf_inputs.CONFIGS[name])
    ro = _steady(cfg)
    _compare(ro, heads, rows=None, name=name + "_all_rows")
    ro.close()


# A context of 29 chunks x 37 pages = 1073 key tiles: past the 1024 page ids
# (and FP8 scale exponents) the attention kernel caches in shared memory, so
# the tiles after the first 1024 take the uncached path through the page table.
LONG_CONTEXT = wf_inputs.CONFIGS["wan13b_bf16"].replace(
    name="long_context_bf16", num_stages=1, num_heads=1, history_chunks=26, rounds=30)


def test_long_context_past_page_cache():
    cfg = LONG_CONTEXT
    positions = cfg.anchor_chunks + cfg.history_chunks + cfg.num_stages + 1
    assert positions * cfg.pages_per_chunk > 1024
    ro = _steady(cfg)
    rows = _sample_rows(cfg.chunk_tokens, 48, 3)
    _compare(ro, [0], rows, name="long_context")
    ro.close()


@pytest.mark.parametrize("name", ["wan13b_bf16", "wan13b_5step_bf16", "wan14b_bf16", "wan13b_bf16_rf"])
def test_full_size_sampled(name):
    cfg = (wf_inputs.CONFIGS["wan13b_bf16"].replace(mask="rf") if name.endswith("_rf")
           else wf_inputs.CONFIGS[name])
    ro = _steady(cfg)
    heads = sorted({0, cfg.num_heads // 2, cfg.num_heads - 1})
    rows = _sample_rows(cfg.chunk_tokens, 40, 1)
    _compare(ro, heads, rows, name=name)
    ro.close()


def test_mask_perturbation_is_bit_exact():
    # M_WF(s, j) = 1[j >= s]: changing the K/V of slot j must leave every
    # cleaner slot s > j (and the store) bit-identical, because their CTAs never
    # read slot j's pages; noisier slots s <= j must change.
    cfg = SMALL_BF16
    ro = Rollout(cfg, page_seed=3)
    for _ in range(cfg.steady_round()):
        ro.publish(0)
        ro.advance()
    q, k, v = ro.publish(0)
    ro.attention(0)
    base = ro.out.clone()
    j = 1
    k2, v2 = k.copy(), v.copy()
    k2[j] = wf_inputs.draw_normal(k[j].shape, cfg.dtype, 99, 1)
    v2[j] = wf_inputs.draw_normal(v[j].shape, cfg.dtype, 99, 2)
    ro.publish(0, inputs=(q, k2, v2))
    ro.attention(0)
    torch.cuda.synchronize()
    for s in range(cfg.num_slots):
        same = torch.equal(ro.out[s].view(torch.int16), base[s].view(torch.int16))
        assert same == (s > j), s
    ro.close()


def test_page_permutation_invariance():
    cfg = SMALL_BF16
    outs = []
    for seed in (None, 21, 22):
        ro = Rollout(cfg, page_seed=seed)
        for _ in range(cfg.steady_round() + 1):
            ro.publish(0)
            ro.advance()
        ro.publish(0)
        ro.attention(0)
        torch.cuda.synchronize()
        outs.append(ro.out.view(torch.int16).clone())
        ro.close()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_value_ones_give_ones():
    cfg = SMALL_BF16
    ro = Rollout(cfg, page_seed=8)
    for _ in range(cfg.steady_round()):
        q, k, v = wf_inputs.draw_round_inputs(cfg, ro.round, 0)
        one = np.full_like(v, 0x3F80)                 # bf16 1.0
        ro.publish(0, inputs=(q, k, one))
        ro.advance()
    q, k, v = wf_inputs.draw_round_inputs(cfg, ro.round, 0)
    ro.publish(0, inputs=(q, k, np.full_like(v, 0x3F80)))
    ro.attention(0)
    torch.cuda.synchronize()
    assert torch.equal(ro.out.float(), torch.ones_like(ro.out.float()))
    ro.close()


def test_identical_keys_give_mean_of_values():
    cfg = SMALL_BF16
    ro = Rollout(cfg, page_seed=8)
    krow = wf_inputs.draw_normal((1, cfg.num_heads, cfg.head_dim), "bf16", 5, 5)
    for _ in range(cfg.steady_round() + 1):
        q, k, v = wf_inputs.draw_round_inputs(cfg, ro.round, 0)
        k[:] = krow[None]
        ro.publish(0, inputs=(q, k, v))
        if ro.round < cfg.steady_round():
            ro.advance()
    ro.attention(0)
    torch.cuda.synchronize()
    # with rotary on, keys differ by position; compare against the oracle instead
    _compare(ro, range(cfg.num_heads))
    ro.close()
    # rotary off: every key is the same vector, so the output is the plain mean of V
    cfg2 = cfg.replace(rope=0)
    ro = Rollout(cfg2, page_seed=8)
    for _ in range(cfg2.steady_round() + 1):
        q, k, v = wf_inputs.draw_round_inputs(cfg2, ro.round, 0)
        k[:] = krow[None]
        ro.publish(0, inputs=(q, k, v))
        if ro.round < cfg2.steady_round():
            ro.advance()
    ro.attention(0)
    torch.cuda.synchronize()
    out = tensor_f64(ro.out)
    lay = ro.layout()
    _, keys, vals = ro.oracle_tensors(range(cfg2.num_heads))
    for p in lay:
        if p.slot is None:
            continue
        vis = O.visible_positions(lay, p.slot)
        mean = np.mean(np.concatenate([vals[lay[i].chunk] for i in vis]), axis=0)
        assert np.abs(out[p.slot] - mean[None]).max() <= 2e-2
        assert rel_l2(out[p.slot], np.broadcast_to(mean, out[p.slot].shape)) <= 1e-2
    ro.close()
