"""Streaming rollout on the GPU: many consecutive rounds over several layers,
through pipeline fill into steady state, with the store's pages recycled from
the chunk that leaves the history window every round (the pool holds exactly
the minimum number of pages). Every round's device page table is checked
against the oracle's pool model, and outputs against the float64 oracle."""
import numpy as np
import pytest
import torch

import wf_inputs
from oracle import wf_oracle as O
from test_gpu_attention import _compare
from wf_test_utils import Rollout, min_pages

pytestmark = pytest.mark.gpu


def _check_layout(ro: Rollout, model: O.PoolModel):
    got = ro.pool.layout()
    want = model.table()
    assert [(g[0], g[1], g[2], g[3], g[4]) for g in got] == \
        [(p.kind, p.chunk, p.slot, t, pg) for p, pg, t in want]


def test_streaming_small_every_round_every_layer():
    cfg = wf_inputs.CONFIGS["stream_13b_bf16"].replace(
        num_layers=3, chunk_tokens=3 * 4 * 10, grid_h=4, grid_w=10, num_heads=2, rounds=24)
    ro = Rollout(cfg, page_seed=13)
    model = O.PoolModel(cfg.num_stages, cfg.anchor_chunks, cfg.history_chunks,
                        cfg.pages_per_chunk, min_pages(cfg), ro.page_order)
    for k in range(cfg.rounds):
        _check_layout(ro, model)
        for layer in range(cfg.num_layers):
            ro.publish(layer)
            ro.attention(layer)
            torch.cuda.synchronize()
            assert ro.pool.check_status() == 0, (k, layer)
            if layer != 1 or k % 4 == 0:
                _compare(ro, range(cfg.num_heads), name="stream_small", layer=layer)
        ro.advance()
        model.advance()
    ro.close()


def test_streaming_full_shape_sampled():
    # Full 1.3B shape (C = 4680, 12 heads) for two layers, rounds 0..9: fill
    # rounds 0..6, then steady rounds with page recycling.
    cfg = wf_inputs.CONFIGS["stream_13b_bf16"].replace(num_layers=2, rounds=10)
    ro = Rollout(cfg, page_seed=17)
    model = O.PoolModel(cfg.num_stages, cfg.anchor_chunks, cfg.history_chunks,
                        cfg.pages_per_chunk, min_pages(cfg), ro.page_order)
    S = cfg.num_stages
    rows = np.array([0, 1, 127, 128, 2000, 4607, 4608, 4679])
    for k in range(cfg.rounds):
        _check_layout(ro, model)
        last = k == cfg.rounds - 1
        for layer in range(cfg.num_layers):
            ro.publish(layer, real_slots=None if last else [S])
            ro.attention(layer)
            torch.cuda.synchronize()
            assert ro.pool.check_status() == 0, (k, layer)
            if last:
                _compare(ro, [0, 5, 11], rows, name="stream_full", layer=layer)
        ro.advance()
        model.advance()
    ro.close()
