"""Float64 CPU oracle for one Wave Forcing round of chunk-wise causal attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, links or calls
this module: it is used by ``tests/``, by ``__graft_entry__.smoke()`` (to check
its one GPU call) and by the CPU-baseline leg of ``bench.py``. It shares no code
with the CUDA library: it is written from the method's definition, in plain
NumPy float64, slow on purpose, so that a reader can check it by eye.

Source: "Wave Forcing: Towards Speed-of-Light Streaming Video Generation"
(arXiv 2611.00859), as summarised on five web pages:
  * Method section of the hyper.ai summary: the wavefront round k = i + s; full
    attention inside each chunk, chunk-wise causal attention across chunks; the
    mask M_WF(s, j) = 1[j >= s] over the query slot s and key slot j, lower
    triangular over itself and all cleaner predecessors, with no reverse edge;
    K/V are published right after the QKV projection and RoPE and delivered as
    direct writes into ordered attention slots, followed by a readiness signal.
  * "Como funciona" section of the e-cogni article: the ordered context of each
    layer is anchor (from the initial chunk) || bounded clean history || live
    store || denoising K/V; newer chunks are never read by older ones.
  * Appendix Table 3 (notation): chunk i, stage s (0 <= s < S), store is stage S,
    round k, clean endpoint B_i = Z_i(S).

Readings where the pages are silent (each one is listed with its reason in the
design notes of the repository):
  * softmax scale 1/sqrt(d);
  * the history window is the H most recently stored chunks, excluding chunk 0
    when an anchor is kept; the anchor is visible from the round after chunk 0's
    store round;
  * the store slot (s = S) attends to anchor + history + itself;
  * 3D rotary: head_dim split into t/h/w bands of widths (44, 42, 42); inside a
    band of width d_a, adjacent pairs (x[2m], x[2m+1]) rotate by the angle
    pos * base^(-2m/d_a), the standard (x cos - y sin, x sin + y cos) rotation;
    token n of chunk i sits at t = F*i + n // (gh*gw), y = (n // gw) % gh,
    x = n % gw (absolute positions);
  * paging (page ids, free list) is this build's own design, not the pages'.

Pins (tests/test_oracle.py, CPU): mask structure by perturbation; reduction to
library scaled-dot-product attention when one slot is live; softmax rows sum to
one; identical keys give the mean of V; two independent formulations (slot
prefix here vs a dense token mask built from chunk indices) agree; a pure-Python
brute force on tiny inputs; rotary against complex multiplication and its norm
and relative-position properties; the round schedule against Figure 1 / Table 3;
the chunk shape against Table 8's one-layer K+V copy size; page-pool invariants.
"""
from __future__ import annotations

import collections
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "Position", "round_layout", "visible_positions", "rope_positions", "rope_3d",
    "attention_slot_prefix", "attention_dense_mask", "attention_bruteforce",
    "PoolModel", "expected_tag", "publish_pages", "unmasked_flops", "round_bf16",
    "project_qkv",
]


# ---------------------------------------------------------------------------
# Round schedule: which chunk each slot holds, and the ordered context.
# ---------------------------------------------------------------------------

Position = collections.namedtuple("Position", "kind chunk slot")
"""One entry of the ordered context: kind in {"anchor", "history", "store",
"slot"}, the chunk index i it holds, and the producing slot (S for the store,
s for a denoising slot, None for anchor/history)."""


def round_layout(S: int, A: int, H: int, k: int) -> List[Position]:
    """Ordered context of round k (Method section; e-cogni "Como funciona").

    Slot s (0 <= s < S) holds chunk i = k - s and is live iff i >= 0 (round
    k = i + s, Table 3). The store (slot S) holds chunk k - S, live iff k >= S.
    Chunks 0 .. k-S-1 were stored in earlier rounds: chunk 0 is the anchor when
    A = 1, and the history is the H newest of the remaining stored chunks.
    Order: anchor, history oldest -> newest, store, slots S-1 down to 0, so that
    the keys a slot may read form a prefix of this list.
    """
    pos: List[Position] = []
    last_stored = k - S - 1
    if A == 1 and last_stored >= 0:
        pos.append(Position("anchor", 0, None))
    lo = max(A, k - S - H)
    for c in range(lo, last_stored + 1):
        pos.append(Position("history", c, None))
    if k >= S:
        pos.append(Position("store", k - S, S))
    for s in range(S - 1, -1, -1):
        if k - s >= 0:
            pos.append(Position("slot", k - s, s))
    return pos


def visible_positions(layout: Sequence[Position], s: int, mask: str = "wf") -> List[int]:
    """Indices of the context entries query slot s attends to.

    mask="wf": M_WF(s, j) = 1[j >= s] over live slots j (the store counts as
    j = S), plus the anchor and history, which every query slot sees (Method
    section). mask="rf": the Rolling Forcing graph the pages contrast WF with
    (e-cogni "Contexto"; Method section: WF removes RF's reverse refinement),
    read here as bidirectional attention among all live slots: every query
    slot sees the whole context.
    """
    out = []
    for idx, p in enumerate(layout):
        if mask == "rf" or p.kind in ("anchor", "history"):
            out.append(idx)
        elif p.slot >= s:
            out.append(idx)
    return out


def unmasked_flops(S: int, A: int, H: int, k: int, C: int, heads: int, d: int,
                   mask: str = "wf") -> int:
    """Multiply-add FLOPs of QK^T and PV over visible (query, key) pairs."""
    layout = round_layout(S, A, H, k)
    total = 0
    for p in layout:
        if p.slot is None:
            continue
        nvis = len(visible_positions(layout, p.slot, mask))
        total += 4 * C * (nvis * C) * d * heads
    return total


# ---------------------------------------------------------------------------
# 3D rotary embedding (applied after QKV, before publication).
# ---------------------------------------------------------------------------

def rope_positions(chunk: int, C: int, F: int, gh: int, gw: int):
    """(t, y, x) of each token of chunk ``chunk`` (absolute positions)."""
    n = np.arange(C, dtype=np.int64)
    t = F * chunk + n // (gh * gw)
    y = (n // gw) % gh
    x = n % gw
    return t, y, x


def rope_3d(x: np.ndarray, chunk: int, F: int, gh: int, gw: int,
            split: Sequence[int] = (44, 42, 42), base: float = 10000.0) -> np.ndarray:
    """Rotate x [C][heads][d] (float64) by the 3D rotary embedding of its chunk."""
    x = np.asarray(x, dtype=np.float64)
    C, _, d = x.shape
    assert sum(split) == d and all(w % 2 == 0 for w in split)
    t, y, w = rope_positions(chunk, C, F, gh, gw)
    out = x.copy()
    off = 0
    for pos, da in zip((t, y, w), split):
        m = np.arange(da // 2, dtype=np.float64)
        inv_freq = base ** (-2.0 * m / da)
        ang = pos.astype(np.float64)[:, None] * inv_freq[None, :]      # [C][da/2]
        c = np.cos(ang)[:, None, :]
        s = np.sin(ang)[:, None, :]
        a = x[:, :, off:off + da:2]
        b = x[:, :, off + 1:off + da:2]
        out[:, :, off:off + da:2] = a * c - b * s
        out[:, :, off + 1:off + da:2] = a * s + b * c
        off += da
    return out


# ---------------------------------------------------------------------------
# QKV projection (the local step before publication).
# ---------------------------------------------------------------------------

def project_qkv(x: np.ndarray, w_qkv: np.ndarray, heads: int, d: int):
    """q, k, v = x W_q^T, x W_k^T, x W_v^T for one chunk, in float64.

    x: [C][hidden] activations; w_qkv: [3 * hidden][hidden] with the q, k and v
    output features stacked (the per-rank QKV projection that runs before
    RoPE and publication, Method section). Returns three [C][heads][d] arrays.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    hidden = heads * d
    y = x @ w.T                                   # library matmul as one step
    return tuple(y[:, i * hidden:(i + 1) * hidden].reshape(x.shape[0], heads, d)
                 for i in range(3))


# ---------------------------------------------------------------------------
# Storage format of published K/V.
# ---------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits, ties
    to even), returned as float64.

    The pages run the model in BF16 (Table 1's BF16/FA3 backend), so published
    rotated queries and keys are bf16 values; this models that storage format.
    Written from the definition: scale each value so its 8 significant bits are
    the integer part, round half to even, scale back. Normal range only (the
    inputs here are O(1)); zeros stay zero.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    scale = np.exp2(7.0 - e)
    out[nz] = np.rint(x[nz] * scale) / scale          # np.rint rounds half to even
    return out


# ---------------------------------------------------------------------------
# Round attention, three independent formulations.
# ---------------------------------------------------------------------------

def _softmax_attend(q: np.ndarray, kk: np.ndarray, vv: np.ndarray, scale: float,
                    mask: Optional[np.ndarray] = None, block: int = 256) -> np.ndarray:
    """Exact two-pass softmax attention for one head, in blocks of query rows.

    q [Nq][d], kk [Nk][d], vv [Nk][dv]; mask [Nq][Nk] bool (True = visible).
    """
    out = np.empty((q.shape[0], vv.shape[1]), dtype=np.float64)
    for r0 in range(0, q.shape[0], block):
        sc = (q[r0:r0 + block] @ kk.T) * scale
        if mask is not None:
            sc = np.where(mask[r0:r0 + block], sc, -np.inf)
        m = sc.max(axis=1, keepdims=True)
        e = np.exp(sc - m)
        l = e.sum(axis=1, keepdims=True)
        out[r0:r0 + block] = (e @ vv) / l
    return out


def attention_slot_prefix(q_rot: Dict[int, np.ndarray], keys: Dict[int, np.ndarray],
                          vals: Dict[int, np.ndarray], layout: Sequence[Position],
                          scale: Optional[float] = None,
                          heads: Optional[Sequence[int]] = None,
                          rows: Optional[np.ndarray] = None,
                          mask: str = "wf") -> Dict[int, np.ndarray]:
    """O_s = softmax(Q_s K^T / sqrt(d)) V over the keys slot s may read.

    q_rot[s]: [C][heads][d] rotated queries of live slot s (store = S).
    keys[chunk], vals[chunk]: [C][heads][d] rotated K and V of every chunk in
    the layout. Returns {s: [C or len(rows)][heads][d]} for live slots (heads not
    in ``heads`` are left at zero). ``rows`` restricts the query rows.
    """
    out = {}
    for p in layout:
        if p.slot is None:
            continue
        s = p.slot
        vis = visible_positions(layout, s, mask)
        K = np.concatenate([keys[layout[i].chunk] for i in vis], axis=0)
        V = np.concatenate([vals[layout[i].chunk] for i in vis], axis=0)
        Q = q_rot[s] if rows is None else q_rot[s][rows]
        d = Q.shape[-1]
        sc = (1.0 / math.sqrt(d)) if scale is None else scale
        o = np.zeros(Q.shape[:2] + (V.shape[-1],), dtype=np.float64)
        for h in (range(Q.shape[1]) if heads is None else heads):
            o[:, h] = _softmax_attend(Q[:, h].astype(np.float64), K[:, h].astype(np.float64),
                                      V[:, h].astype(np.float64), sc)
        out[s] = o
    return out


def attention_dense_mask(q_rot: Dict[int, np.ndarray], keys: Dict[int, np.ndarray],
                         vals: Dict[int, np.ndarray], layout: Sequence[Position],
                         scale: Optional[float] = None, mask: str = "wf") -> Dict[int, np.ndarray]:
    """Second formulation: one dense token x token mask for the whole round.

    All context tokens form one key sequence and all live query tokens one query
    sequence. A query token of chunk i_q sees a key token of chunk i_k iff
    i_k <= i_q: itself (full attention inside the chunk) and every cleaner,
    older chunk in the context, never a newer one (no reverse edge). With
    mask="rf" every query token sees every context token.
    """
    q_slots = [p for p in layout if p.slot is not None]
    Q = np.concatenate([q_rot[p.slot] for p in q_slots], axis=0)
    q_chunk = np.concatenate([np.full(q_rot[p.slot].shape[0], p.chunk) for p in q_slots])
    K = np.concatenate([keys[p.chunk] for p in layout], axis=0)
    V = np.concatenate([vals[p.chunk] for p in layout], axis=0)
    k_chunk = np.concatenate([np.full(keys[p.chunk].shape[0], p.chunk) for p in layout])
    if mask == "rf":
        visible = np.ones((q_chunk.size, k_chunk.size), dtype=bool)
    else:
        visible = k_chunk[None, :] <= q_chunk[:, None]
    d = Q.shape[-1]
    sc = (1.0 / math.sqrt(d)) if scale is None else scale
    O = np.zeros(Q.shape[:2] + (V.shape[-1],), dtype=np.float64)
    for h in range(Q.shape[1]):
        O[:, h] = _softmax_attend(Q[:, h], K[:, h], V[:, h], sc, mask=visible)
    out, r = {}, 0
    for p in q_slots:
        n = q_rot[p.slot].shape[0]
        out[p.slot] = O[r:r + n]
        r += n
    return out


def attention_bruteforce(q_rot, keys, vals, layout, scale=None, mask="wf"):
    """Third formulation, pure Python loops (tiny inputs only).

    For every live query slot s, head h and query token, walk the context and
    accumulate exp(q.k * scale) and exp(q.k * scale) * v over keys of slots
    j >= s (M_WF) plus anchor and history, then divide.
    """
    out = {}
    for p in layout:
        if p.slot is None:
            continue
        s = p.slot
        Q = q_rot[s]
        C, Hh, d = Q.shape
        sc = (1.0 / math.sqrt(d)) if scale is None else scale
        o = np.zeros((C, Hh, vals[p.chunk].shape[-1]))
        for h in range(Hh):
            for n in range(C):
                logits, vs = [], []
                for e in layout:
                    if mask == "wf" and e.slot is not None and e.slot < s:
                        continue                      # M_WF(s, j) = 0 for j < s
                    for m in range(keys[e.chunk].shape[0]):
                        logits.append(sum(float(Q[n, h, c]) * float(keys[e.chunk][m, h, c])
                                          for c in range(d)) * sc)
                        vs.append(vals[e.chunk][m, h])
                mx = max(logits)
                w = [math.exp(z - mx) for z in logits]
                tot = sum(w)
                o[n, h] = sum(wi * vi for wi, vi in zip(w, vs)) / tot
        out[s] = o
    return out


# ---------------------------------------------------------------------------
# Paged K/V pool: host model of the page table (this build's own policy).
# ---------------------------------------------------------------------------

def expected_tag(S: int, rnd: int, slot: int) -> int:
    """Readiness tag written with the K/V that slot ``slot`` publishes in round rnd."""
    return rnd * (S + 1) + slot + 1


class PoolModel:
    """Page allocation policy, modelled independently of the C++ pool.

    * Physical pages are handed out from a FIFO free list initialised to
      ``page_order``.
    * At creation, denoising slots 0..S-1 take npc pages each, slot 0 first;
      they keep them for good (a slot re-publishes its chunk every round).
    * When round k >= S begins, the store takes npc pages from the free list.
    * On advance from round k (k >= S), the store's chunk c = k - S keeps its
      pages and becomes the anchor (A = 1 and c = 0) or the newest history
      entry; if the history then holds more than H chunks, the oldest one's
      pages go to the tail of the free list in page-index order.
    """

    def __init__(self, S: int, A: int, H: int, npc: int, num_pages: int,
                 page_order: Optional[Sequence[int]] = None):
        self.S, self.A, self.H, self.npc = S, A, H, npc
        need = (S + 1 + A + H) * npc
        if num_pages < need:
            raise ValueError("pool too small")
        order = list(range(num_pages)) if page_order is None else [int(x) for x in page_order]
        assert sorted(order) == list(range(num_pages))
        self.free = collections.deque(order)
        self.slot_pages = [[self.free.popleft() for _ in range(npc)] for _ in range(S)]
        self.store_pages: Optional[List[int]] = None
        self.anchor: Optional[Tuple[int, List[int]]] = None
        self.history: "collections.deque[Tuple[int, List[int]]]" = collections.deque()
        self.k = 0
        if self.k >= S:
            self.store_pages = self._take()

    def _take(self) -> List[int]:
        return [self.free.popleft() for _ in range(self.npc)]

    def advance(self) -> None:
        S = self.S
        if self.k >= S:
            c = self.k - S
            if self.A == 1 and c == 0:
                self.anchor = (0, self.store_pages)
            else:
                self.history.append((c, self.store_pages))
                if len(self.history) > self.H:
                    _, old = self.history.popleft()
                    self.free.extend(old)
            self.store_pages = None
        self.k += 1
        if self.k >= S:
            self.store_pages = self._take()

    def layout(self) -> List[Position]:
        return round_layout(self.S, self.A, self.H, self.k)

    def pages_of(self, p: Position) -> List[int]:
        if p.kind == "anchor":
            return self.anchor[1]
        if p.kind == "history":
            for c, pg in self.history:
                if c == p.chunk:
                    return pg
            raise KeyError(p)
        if p.kind == "store":
            return self.store_pages
        return self.slot_pages[p.slot]

    def table(self) -> List[Tuple[Position, List[int], int]]:
        """[(position, physical pages, expected readiness tag)] in context order."""
        rows = []
        for p in self.layout():
            if p.kind in ("anchor", "history"):
                tag = expected_tag(self.S, p.chunk + self.S, self.S)
            else:
                tag = expected_tag(self.S, self.k, p.slot)
            rows.append((p, list(self.pages_of(p)), tag))
        return rows


def publish_pages(k_rot: np.ndarray, v: np.ndarray, pages: Sequence[int], P: int,
                  num_pages: int) -> Tuple[np.ndarray, np.ndarray]:
    """Predicted pool contents after publishing one slot's K/V into ``pages``.

    Returns (pool_k, pool_v) shaped [num_pages][heads][P][d]; rows past the end
    of the chunk in its last page are zero, other pages are NaN (untouched).
    """
    C, Hh, d = k_rot.shape
    pk = np.full((num_pages, Hh, P, d), np.nan)
    pv = np.full((num_pages, Hh, P, d), np.nan)
    for j, pg in enumerate(pages):
        pk[pg] = 0.0
        pv[pg] = 0.0
        lo, hi = j * P, min(C, (j + 1) * P)
        pk[pg, :, :hi - lo] = np.transpose(k_rot[lo:hi], (1, 0, 2))
        pv[pg, :, :hi - lo] = np.transpose(v[lo:hi], (1, 0, 2))
    return pk, pv
