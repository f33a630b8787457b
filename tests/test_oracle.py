"""Pins for the float64 oracle, checked against facts fixed outside the oracle.

Runs on the CPU. Each test names the property of the method it relies on; a
plausible slip in the oracle (a dropped term, a wrong sign or index, a swapped
operand, an off-by-one in the window) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import wf_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _run_rounds(S, A, H, C, Hh, d, rounds, seed=0, rope=False):
    """Drive the oracle through rounds 0..rounds-1 like a streaming rollout.

    Returns per round: (layout, q_rot, keys, vals) where keys/vals map chunk ->
    [C][Hh][d] for every chunk in that round's context; stored chunks keep the
    K/V their store round published (the clean-history cache convention).
    """
    stored = {}
    out = []
    for k in range(rounds):
        layout = O.round_layout(S, A, H, k)
        q_rot, keys, vals = {}, {}, {}
        for p in layout:
            if p.slot is None:
                keys[p.chunk], vals[p.chunk] = stored[p.chunk]
                continue
            q = _rand((C, Hh, d), (seed, k, p.slot, 0))
            kk = _rand((C, Hh, d), (seed, k, p.slot, 1))
            v = _rand((C, Hh, d), (seed, k, p.slot, 2))
            if rope:
                q = O.rope_3d(q, p.chunk, 1, 2, C // 2, split=(2, 2, d - 4))
                kk = O.rope_3d(kk, p.chunk, 1, 2, C // 2, split=(2, 2, d - 4))
            q_rot[p.slot], keys[p.chunk], vals[p.chunk] = q, kk, v
            if p.kind == "store":
                stored[p.chunk] = (kk, v)
        out.append((layout, q_rot, keys, vals))
    return out


# --- schedule ---------------------------------------------------------------

def test_schedule_matches_figure1_table3():
    rows = []
    with open(os.path.join(GOLDEN, "wavefront_schedule_S4.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append(line.split())
    assert len(rows) == 9
    for r in rows:
        k = int(r[0])
        layout = O.round_layout(4, 1, 2, k)
        held = {p.slot: p.chunk for p in layout if p.slot is not None}
        for s in range(5):
            want = r[1 + s]
            assert (str(held[s]) if s in held else "-") == want, (k, s)


def test_one_chunk_per_round_after_fill():
    # Figure 1(c): over five rounds after fill, five chunks complete (1F1C).
    S = 4
    done = [p.chunk for k in range(S, S + 5) for p in O.round_layout(S, 1, 2, k)
            if p.kind == "store"]
    assert done == [0, 1, 2, 3, 4]
    assert all(p.kind != "store" for k in range(S) for p in O.round_layout(S, 1, 2, k))


def test_context_order_and_window():
    # e-cogni "Como funciona": anchor || bounded clean history || store || denoising.
    lay = O.round_layout(4, 1, 2, 9)
    assert [p.kind for p in lay] == ["anchor", "history", "history", "store",
                                     "slot", "slot", "slot", "slot"]
    assert [p.chunk for p in lay] == [0, 3, 4, 5, 6, 7, 8, 9]
    assert [p.slot for p in lay][3:] == [4, 3, 2, 1, 0]
    # the anchor appears only once chunk 0 has been stored (round S), i.e. from S+1
    assert all(p.kind != "anchor" for p in O.round_layout(4, 1, 2, 4))
    assert O.round_layout(4, 1, 2, 5)[0] == O.Position("anchor", 0, None)
    # no anchor kept: history may include chunk 0
    assert [p.chunk for p in O.round_layout(2, 0, 1, 3) if p.kind == "history"] == [0]
    assert [p.chunk for p in O.round_layout(2, 0, 1, 4) if p.kind == "history"] == [1]


def test_visible_sets_are_lower_triangular_prefixes():
    # M_WF(s, j) = 1[j >= s]: each slot reads a prefix of the ordered context,
    # and a slot's context contains only chunks no newer than its own.
    for S, A, H in [(4, 1, 2), (5, 1, 3), (2, 1, 1), (3, 0, 2)]:
        for k in range(S + A + H + 3):
            lay = O.round_layout(S, A, H, k)
            for idx, p in enumerate(lay):
                if p.slot is None:
                    continue
                vis = O.visible_positions(lay, p.slot)
                assert vis == list(range(idx + 1))
                assert all(lay[i].chunk <= p.chunk for i in vis)
                assert all(lay[i].chunk > p.chunk for i in range(idx + 1, len(lay)))


def test_unmasked_pair_count_closed_form():
    # Steady state: slot s < S reads A + H + 1 + (S - s) chunks; the store A + H + 1.
    # Sum = (S+1)(A+H) + (S+1)(S+2)/2.
    for S, A, H in [(4, 1, 2), (5, 1, 3), (2, 1, 1)]:
        k = S + A + H + 1
        lay = O.round_layout(S, A, H, k)
        pairs = sum(len(O.visible_positions(lay, p.slot)) for p in lay if p.slot is not None)
        assert pairs == (S + 1) * (A + H) + (S + 1) * (S + 2) // 2
        assert O.unmasked_flops(S, A, H, k, 10, 3, 8) == 4 * 10 * 10 * 8 * 3 * pairs


def test_chunk_shape_matches_table8_copy():
    with open(os.path.join(GOLDEN, "table8_kv_copy_bytes.txt")) as f:
        nbytes, hidden, ntens, elt = [int(x) for x in
                                      [l for l in f if not l.startswith("#")][0].split()]
    C = 3 * 30 * 52          # 3 latent frames x 30 x 52 patches
    assert C * hidden * ntens * elt == nbytes
    assert hidden == 40 * 128


# --- attention ---------------------------------------------------------------

@pytest.mark.parametrize("S,A,H", [(2, 1, 1), (3, 0, 2)])
def test_three_formulations_agree(S, A, H):
    C, Hh, d = 3, 2, 4
    for layout, q, kk, vv in _run_rounds(S, A, H, C, Hh, d, S + A + H + 3, rope=True):
        o1 = O.attention_slot_prefix(q, kk, vv, layout)
        o2 = O.attention_dense_mask(q, kk, vv, layout)
        o3 = O.attention_bruteforce(q, kk, vv, layout)
        assert set(o1) == set(o2) == set(o3)
        for s in o1:
            np.testing.assert_allclose(o1[s], o2[s], rtol=0, atol=1e-12)
            np.testing.assert_allclose(o1[s], o3[s], rtol=0, atol=1e-12)


def test_mask_perturbation_no_reverse_edge():
    S, A, H, C, Hh, d = 4, 1, 2, 5, 2, 8
    layout, q, kk, vv = _run_rounds(S, A, H, C, Hh, d, 9)[-1]
    base = O.attention_dense_mask(q, kk, vv, layout)
    for p in layout:
        if p.kind != "slot":
            continue
        kk2 = dict(kk)
        vv2 = dict(vv)
        kk2[p.chunk] = kk[p.chunk] + 3.0 * _rand(kk[p.chunk].shape, 77)
        vv2[p.chunk] = vv[p.chunk] - 2.0
        pert = O.attention_dense_mask(q, kk2, vv2, layout)
        for s in base:
            if s < p.slot:
                continue
            if s == p.slot:
                assert np.abs(pert[s] - base[s]).max() > 1e-3   # own chunk is read
            else:
                # slot s > j is cleaner: it must not see the noisier slot j
                assert np.array_equal(pert[s], base[s]), (s, p.slot)
        # noisier slots s < j do read slot j
        for s in base:
            if s < p.slot:
                assert np.abs(pert[s] - base[s]).max() > 1e-3


def test_single_live_slot_is_plain_attention():
    # Round 0: only slot 0 is live, no anchor, history or store -> plain
    # bidirectional attention over its own chunk (library routine).
    C, Hh, d = 37, 3, 16
    layout, q, kk, vv = _run_rounds(4, 1, 2, C, Hh, d, 1)[0]
    assert [p.slot for p in layout] == [0]
    o = O.attention_slot_prefix(q, kk, vv, layout)[0]
    tq = torch.from_numpy(q[0]).permute(1, 0, 2)[None]
    tk = torch.from_numpy(kk[0]).permute(1, 0, 2)[None]
    tv = torch.from_numpy(vv[0]).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-13)


def test_softmax_rows_sum_to_one():
    S, A, H, C, Hh, d = 2, 1, 1, 6, 2, 8
    for layout, q, kk, vv in _run_rounds(S, A, H, C, Hh, d, 5):
        ones = {c: np.ones_like(v) for c, v in vv.items()}
        o = O.attention_slot_prefix(q, kk, ones, layout)
        for s in o:
            np.testing.assert_allclose(o[s], 1.0, rtol=0, atol=1e-14)


def test_identical_keys_give_mean_of_visible_values():
    S, A, H, C, Hh, d = 3, 1, 2, 4, 2, 8
    layout, q, kk, vv = _run_rounds(S, A, H, C, Hh, d, 7)[-1]
    same = {c: np.broadcast_to(_rand((1, Hh, d), 5), x.shape).copy() for c, x in kk.items()}
    o = O.attention_slot_prefix(q, same, vv, layout)
    for p in layout:
        if p.slot is None:
            continue
        vis = O.visible_positions(layout, p.slot)
        mean = np.mean(np.concatenate([vv[layout[i].chunk] for i in vis]), axis=0)
        np.testing.assert_allclose(o[p.slot], np.broadcast_to(mean, o[p.slot].shape),
                                   rtol=0, atol=1e-13)


# --- rotary -------------------------------------------------------------------

def test_rope_matches_complex_rotation():
    C, Hh, d, F, gh, gw = 24, 2, 16, 2, 3, 4
    split = (4, 6, 6)
    x = _rand((C, Hh, d), 3)
    chunk = 5
    got = O.rope_3d(x, chunk, F, gh, gw, split=split, base=100.0)
    n = np.arange(C)
    pos = [F * chunk + n // (gh * gw), (n // gw) % gh, n % gw]
    off = 0
    for p, da in zip(pos, split):
        z = x[:, :, off:off + da:2] + 1j * x[:, :, off + 1:off + da:2]
        freq = 100.0 ** (-np.arange(0, da, 2) / da)
        zr = z * np.exp(1j * p[:, None, None] * freq[None, None, :])
        np.testing.assert_allclose(got[:, :, off:off + da:2], zr.real, atol=1e-12)
        np.testing.assert_allclose(got[:, :, off + 1:off + da:2], zr.imag, atol=1e-12)
        off += da


def test_rope_closed_form_values():
    # token n = gh*gw of chunk 0 sits at t = 1, y = 0, x = 0: the first pair of
    # the t band turns by exactly 1 radian, the h and w bands do not move.
    C, F, gh, gw = 2 * 6, 2, 2, 3
    x = np.zeros((C, 1, 128))
    x[:, :, 0] = 1.0
    x[:, :, 44] = 1.0
    x[:, :, 86] = 1.0
    r = O.rope_3d(x, 0, F, gh, gw)
    n = gh * gw
    assert r[n, 0, 0] == pytest.approx(math.cos(1.0), abs=1e-15)
    assert r[n, 0, 1] == pytest.approx(math.sin(1.0), abs=1e-15)
    assert r[n, 0, 44] == 1.0 and r[n, 0, 45] == 0.0
    assert r[n, 0, 86] == 1.0 and r[n, 0, 87] == 0.0
    # position (0,0,0) is the identity
    y = _rand((C, 2, 128), 9)
    np.testing.assert_array_equal(O.rope_3d(y, 0, F, gh, gw)[0], y[0])
    # last pair of the w band turns by x * base^(-40/42) at token (y=0, x=2)
    x2 = np.zeros((C, 1, 128))
    x2[:, :, 126] = 1.0
    r2 = O.rope_3d(x2, 0, F, gh, gw)
    ang = 2 * 10000.0 ** (-40.0 / 42.0)
    assert r2[2, 0, 126] == pytest.approx(math.cos(ang), abs=1e-15)
    assert r2[2, 0, 127] == pytest.approx(math.sin(ang), abs=1e-15)


def test_rope_norm_and_relative_position():
    C, Hh, F, gh, gw = 30, 2, 1, 5, 6
    q = _rand((C, Hh, 128), 1)
    k = _rand((C, Hh, 128), 2)
    rq = O.rope_3d(q, 4, F, gh, gw)
    np.testing.assert_allclose(np.hypot(rq[..., 0::2], rq[..., 1::2]),
                               np.hypot(q[..., 0::2], q[..., 1::2]), atol=1e-12)
    # q.k after rotation depends on the position difference only
    a = np.einsum("chd,chd->ch", O.rope_3d(q, 4, F, gh, gw), O.rope_3d(k, 2, F, gh, gw))
    b = np.einsum("chd,chd->ch", O.rope_3d(q, 9, F, gh, gw), O.rope_3d(k, 7, F, gh, gw))
    np.testing.assert_allclose(a, b, atol=1e-10)
    c = np.einsum("chd,chd->ch", O.rope_3d(q, 9, F, gh, gw), O.rope_3d(k, 6, F, gh, gw))
    assert np.abs(a - c).max() > 1e-3


# --- page pool model ------------------------------------------------------------

@pytest.mark.parametrize("S,A,H,npc,extra", [(4, 1, 2, 37, 0), (5, 1, 3, 3, 2), (2, 1, 1, 2, 1),
                                             (3, 0, 2, 2, 0), (2, 0, 0, 1, 0)])
def test_pool_model_partition_and_recycling(S, A, H, npc, extra):
    num_pages = (S + 1 + A + H + extra) * npc
    order = np.random.default_rng(1).permutation(num_pages)
    pm = O.PoolModel(S, A, H, npc, num_pages, order)
    assert pm.slot_pages[0] == [int(x) for x in order[:npc]]
    for k in range(60):
        assert pm.k == k
        tab = pm.table()
        assert [r[0] for r in tab] == O.round_layout(S, A, H, k)
        used = [pg for _, pages, _ in tab for pg in pages]
        idle = [pg for s in range(S) if k - s < 0 for pg in pm.slot_pages[s]]
        assert len(set(used)) == len(used)
        assert sorted(used + idle + list(pm.free)) == list(range(num_pages))
        tags = [t for _, _, t in tab]
        assert len(set(tags)) == len(tags)
        before_free = list(pm.free)
        evicted = None
        if k >= S and len(pm.history) == H and not (A == 1 and k - S == 0):
            evicted = pm.history[0][1] if H > 0 else pm.store_pages
        pm.advance()
        if evicted is not None and extra == 0:
            # the pool is exactly full: the new store reuses the evicted pages
            assert pm.store_pages == list(evicted)
        if k + 1 >= S and extra == 0 and evicted is None:
            assert not before_free or pm.store_pages == before_free[:npc]


def test_pool_model_rejects_small_pool():
    with pytest.raises(ValueError):
        O.PoolModel(4, 1, 2, 3, (4 + 1 + 1 + 2) * 3 - 1)


def test_publish_pages_layout():
    C, Hh, d, P = 10, 2, 4, 4
    k = _rand((C, Hh, d), 1)
    v = _rand((C, Hh, d), 2)
    pk, pv = O.publish_pages(k, v, [5, 0, 3], P, 6)
    np.testing.assert_array_equal(pk[5, 1, 2], k[2, 1])
    np.testing.assert_array_equal(pv[3, 0, 1], v[9, 0])
    assert (pk[3, :, 2:] == 0).all() and (pv[3, :, 2:] == 0).all()
    assert np.isnan(pk[1]).all()


def test_round_bf16_matches_library_cast():
    # the library's float32 -> bfloat16 cast rounds to nearest even too
    x = np.concatenate([_rand(20000, 4) * 10.0 ** np.random.default_rng(5).integers(-3, 4, 20000),
                        [1.0, -2.5, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.0 * 2 ** -9]])
    x32 = x.astype(np.float32).astype(np.float64)      # exactly representable in fp32
    ref = torch.from_numpy(x32).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_bf16(x32), ref)
    # ties: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> even (1.0)
    assert O.round_bf16(np.array([1.0 + 2 ** -8]))[0] == 1.0
    assert O.round_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6


# --- Rolling Forcing mask variant ------------------------------------------------

@pytest.mark.parametrize("S,A,H", [(2, 1, 1), (3, 0, 2)])
def test_rf_three_formulations_agree(S, A, H):
    C, Hh, d = 3, 2, 4
    for layout, q, kk, vv in _run_rounds(S, A, H, C, Hh, d, S + A + H + 3, rope=True):
        o1 = O.attention_slot_prefix(q, kk, vv, layout, mask="rf")
        o2 = O.attention_dense_mask(q, kk, vv, layout, mask="rf")
        o3 = O.attention_bruteforce(q, kk, vv, layout, mask="rf")
        for s in o1:
            np.testing.assert_allclose(o1[s], o2[s], rtol=0, atol=1e-12)
            np.testing.assert_allclose(o1[s], o3[s], rtol=0, atol=1e-12)


def test_rf_has_reverse_edges_and_wf_does_not():
    # Under RF a cleaner slot reads noisier live slots; under WF it never does.
    S, A, H, C, Hh, d = 4, 1, 2, 5, 2, 8
    layout, q, kk, vv = _run_rounds(S, A, H, C, Hh, d, 9)[-1]
    j = 1
    chunk_j = [p.chunk for p in layout if p.slot == j][0]
    kk2 = dict(kk)
    kk2[chunk_j] = kk[chunk_j] + 2.0 * _rand(kk[chunk_j].shape, 3)
    for mask, cleaner_changes in (("rf", True), ("wf", False)):
        base = O.attention_slot_prefix(q, kk, vv, layout, mask=mask)
        pert = O.attention_slot_prefix(q, kk2, vv, layout, mask=mask)
        for s in base:
            if s > j:
                assert (np.abs(pert[s] - base[s]).max() > 1e-3) == cleaner_changes, (mask, s)
    # with one live slot the two graphs coincide
    layout0, q0, k0, v0 = _run_rounds(S, A, H, C, Hh, d, 1)[0]
    a = O.attention_slot_prefix(q0, k0, v0, layout0, mask="rf")[0]
    b = O.attention_slot_prefix(q0, k0, v0, layout0, mask="wf")[0]
    np.testing.assert_array_equal(a, b)


def test_rf_work_closed_form():
    # RF: every live slot reads the whole context of A + H + S + 1 chunks.
    S, A, H = 4, 1, 2
    k = S + A + H + 1
    assert O.unmasked_flops(S, A, H, k, 7, 2, 8, "rf") == 4 * 7 * 7 * 8 * 2 * (S + 1) * (A + H + S + 1)


# --- QKV projection -----------------------------------------------------------

def test_project_qkv_against_elementwise_sums():
    rng = np.random.default_rng(11)
    C, heads, d = 5, 2, 4
    hidden = heads * d
    x = rng.standard_normal((C, hidden))
    w = rng.standard_normal((3 * hidden, hidden))
    q, k, v = O.project_qkv(x, w, heads, d)
    for which, out in enumerate((q, k, v)):
        for n in range(C):
            for h in range(heads):
                for c in range(d):
                    f = which * hidden + h * d + c        # output feature index
                    want = sum(x[n, i] * w[f, i] for i in range(hidden))
                    assert out[n, h, c] == pytest.approx(want, abs=1e-12)
