"""C-ABI checks that need no GPU: the library loads, exports what include/wf.h
declares, validates configs, and its host-side round bookkeeping (page table,
free list, ordered context, ready tags) matches the oracle's pool model
bit-exactly over long rollouts."""
import os
import re

import numpy as np
import pytest

import wf_inputs
from oracle import wf_oracle as O
from wf_test_utils import min_pages, pool_config

import chunk_causal_wavefront_b200 as wfb
from chunk_causal_wavefront_b200 import wf as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "wf.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wf_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    declared = header_functions()
    assert len(declared) >= 12
    lib = W.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(W.EXPORTS) == declared


def test_status_strings():
    for s in range(9):
        assert W.wf_status_string(s).startswith("WF_")
    assert "unknown" in W.wf_status_string(99)


def test_pool_bytes_and_geometry():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    c = pool_config(cfg)
    nbytes = W.wf_kv_pool_bytes(c)
    pool = wfb.KVPool(c)          # host-only
    g = pool.geometry
    assert g.total_bytes == nbytes
    assert g.pages_per_chunk == 37 and g.num_pages == 8 * 37
    assert g.page_bytes == 2 * 12 * 128 * 128 * 2
    assert g.pages_offset % 1024 == 0
    assert nbytes >= g.pages_offset + g.num_pages * g.page_bytes
    # one 1.3B layer's pool: 296 pages x 786432 B = 232.8 MB, more than the 126 MB L2
    assert g.num_pages * g.page_bytes == 232783872
    pool.close()


def test_fp8_pool_geometry():
    """FP8 pools: 1-byte pages (half of bf16) plus fp32 block scales for every
    (layer, page, K|V, head) and every (layer, slot, query tile, head)."""
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    c = pool_config(cfg, dtype="fp8", num_layers=3)
    pool = wfb.KVPool(c)
    g = pool.geometry
    assert g.page_bytes == 2 * 12 * 128 * 128
    assert g.pages_offset % 1024 == 0 and g.kv_scale_offset % 256 == 0
    assert g.tags_offset < g.kv_scale_offset < g.q_scale_offset < g.pages_offset
    assert g.q_scale_offset - g.kv_scale_offset >= 3 * g.num_pages * 2 * 12 * 4
    assert g.pages_offset - g.q_scale_offset >= 3 * 5 * 37 * 12 * 4
    assert g.total_bytes >= g.pages_offset + 3 * g.num_pages * g.page_bytes
    bf = wfb.KVPool(pool_config(cfg, num_layers=3)).geometry
    assert bf.kv_scale_offset == 0 and bf.q_scale_offset == 0
    assert bf.page_bytes == 2 * g.page_bytes
    pool.close()
    for over in (dict(head_dim=64), dict(page_tokens=64)):
        with pytest.raises(W.WfError) as e:
            W.wf_kv_pool_bytes(pool_config(cfg, dtype="fp8", **over))
        assert e.value.status == W.WF_ERR_UNSUPPORTED


@pytest.mark.parametrize("over,err", [
    (dict(num_stages=0), W.WF_ERR_INVALID_ARG),
    (dict(num_stages=17), W.WF_ERR_INVALID_ARG),
    (dict(anchor_chunks=2), W.WF_ERR_INVALID_ARG),
    (dict(history_chunks=65), W.WF_ERR_INVALID_ARG),
    (dict(head_dim=64), W.WF_ERR_UNSUPPORTED),
    (dict(page_tokens=64), W.WF_ERR_UNSUPPORTED),
    (dict(grid_w=51), W.WF_ERR_INVALID_ARG),             # C != F * gh * gw
    (dict(rope_split=(44, 42, 40)), W.WF_ERR_INVALID_ARG),  # bands do not sum to head_dim
    (dict(rope_split=(43, 43, 42)), W.WF_ERR_INVALID_ARG),
    (dict(num_pages=8 * 37 - 1), W.WF_ERR_OUT_OF_PAGES),
])
def test_config_validation(over, err):
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    c = pool_config(cfg, **over)
    with pytest.raises(W.WfError) as e:
        W.wf_kv_pool_bytes(c)
    assert e.value.status == err


def test_page_order_validation():
    cfg = wf_inputs.CONFIGS["tiny_f32"]
    c = pool_config(cfg)
    n = min_pages(cfg)
    bad = list(range(n))
    bad[3] = bad[4]
    with pytest.raises(W.WfError) as e:
        wfb.KVPool(c, page_order=bad)
    assert e.value.status == W.WF_ERR_INVALID_ARG
    with pytest.raises(W.WfError):
        wfb.KVPool(c, page_order=list(range(n - 1)) + [n])


def _compare_with_model(cfg, rounds, extra_pages=0, seed=3):
    npg = min_pages(cfg) + extra_pages * cfg.pages_per_chunk
    order = wf_inputs.draw_page_order(npg, seed)
    pool = wfb.KVPool(pool_config(cfg, num_pages=npg, max_rounds=rounds + 1), page_order=order)
    model = O.PoolModel(cfg.num_stages, cfg.anchor_chunks, cfg.history_chunks,
                        cfg.pages_per_chunk, npg, order)
    for k in range(rounds):
        assert pool.round == k == model.k
        got = pool.layout()
        want = model.table()
        assert len(got) == len(want), k
        for (kind, chunk, slot, tag, pages), (p, mpages, mtag) in zip(got, want):
            assert (kind, chunk, slot) == (p.kind, p.chunk, p.slot), k
            assert tag == mtag, k
            assert pages == mpages, k
        if k + 1 < rounds:
            pool.advance()
            model.advance()
    pool.close()


@pytest.mark.parametrize("name", ["tiny_f32", "wan13b_bf16", "wan13b_5step_bf16", "stream_13b_bf16"])
def test_host_bookkeeping_matches_oracle_model(name):
    cfg = wf_inputs.CONFIGS[name]
    _compare_with_model(cfg, 200)


@pytest.mark.parametrize("S,A,H,extra", [(2, 0, 0, 0), (3, 0, 2, 1), (1, 1, 0, 0), (6, 1, 5, 2)])
def test_host_bookkeeping_edge_schedules(S, A, H, extra):
    cfg = wf_inputs.CONFIGS["tiny_f32"].replace(num_stages=S, anchor_chunks=A, history_chunks=H)
    _compare_with_model(cfg, 60, extra_pages=extra)


def test_max_rounds_enforced():
    cfg = wf_inputs.CONFIGS["tiny_f32"]
    pool = wfb.KVPool(pool_config(cfg, max_rounds=3))
    pool.advance()
    pool.advance()
    with pytest.raises(W.WfError) as e:
        pool.advance()
    assert e.value.status == W.WF_ERR_CALL_ORDER
    assert pool.round == 2
    pool.close()


def test_host_only_pool_refuses_device_calls():
    cfg = wf_inputs.CONFIGS["tiny_f32"]
    pool = wfb.KVPool(pool_config(cfg))
    st = W.wf_publish_kv(pool.handle, 0, 16, 16, 16, 32, 0)
    assert st == W.WF_ERR_CALL_ORDER
    st = W.wf_round_attention(pool.handle, 0, 16, 32, 0)
    assert st == W.WF_ERR_CALL_ORDER
    assert W.wf_pool_check_status(pool.handle, 0) == W.WF_OK
    pool.close()


def test_null_pool_arguments():
    lib = W.lib()
    assert lib.wf_pool_round(None) == -1
    assert lib.wf_advance_round(None, None) == W.WF_ERR_INVALID_ARG
    assert lib.wf_pool_destroy(None) == W.WF_ERR_INVALID_ARG
    assert lib.wf_kv_pool_bytes(None, None) == W.WF_ERR_INVALID_ARG


def test_mask_mode_validation():
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    c = pool_config(cfg)
    c.mask_mode = 2
    with pytest.raises(W.WfError) as e:
        W.wf_kv_pool_bytes(c)
    assert e.value.status == W.WF_ERR_INVALID_ARG
    # the page table does not depend on the mask
    a = wfb.KVPool(pool_config(cfg, mask="wf"))
    b = wfb.KVPool(pool_config(cfg, mask="rf"))
    for _ in range(9):
        assert a.layout() == b.layout()
        a.advance()
        b.advance()


def test_bench_traffic_record_follows_kernel_code(tmp_path):
    # bench.py reports a kernel's recorded ncu traffic only while the hash of
    # its code matches; comment and blank-line edits keep the hash.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "bench_mod", os.path.join(os.path.dirname(os.path.dirname(__file__)), "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    src = tmp_path / "k.cu"
    src.write_text("// header\nint f(int x) {\n  return x + 1;   // add\n}\n")
    h0 = b.source_sha(str(src))
    src.write_text("// another header\n\nint f(int x) {\n  return x + 1;\n}\n")
    assert b.source_sha(str(src)) == h0
    src.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert b.source_sha(str(src)) != h0
    # every committed record matches the kernel source it names
    import json
    root = os.path.dirname(os.path.dirname(__file__))
    rec = json.load(open(os.path.join(root, "profiles", "ncu_traffic.json")))
    for key, e in rec.items():
        path = os.path.join(root, "chunk_causal_wavefront_b200", "csrc", key.split(":")[0])
        assert e["source_sha"] == b.source_sha(path), key
        assert e["dram_bytes_per_launch"] > 0
