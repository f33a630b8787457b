"""Torch-facing wrapper of the libwf pool: tensors in, C-ABI calls out.

PyTorch provides the device memory (one uint8 tensor that the pool lives in)
and the stream; every computation runs in libwf's kernels.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import wf as _wf
from .wf import WfError, WfPoolConfig

# pool dtype -> (C enum, element type of the pages and of q_rot)
_DTYPES = {"bf16": (_wf.WF_DTYPE_BF16, torch.bfloat16), "f32": (_wf.WF_DTYPE_F32, torch.float32),
           "fp8": (_wf.WF_DTYPE_FP8_E4M3, torch.uint8)}
_ELEMENT = {code: t for code, t in _DTYPES.values()}


def make_config(*, num_stages: int, chunk_tokens: int, num_heads: int, head_dim: int,
                anchor_chunks: int, history_chunks: int, page_tokens: int, num_layers: int = 1,
                dtype: str = "bf16", rope: int = 0, frames_per_chunk: int = 1, grid_h: int = 1,
                grid_w: int = 1, rope_split: Sequence[int] = (0, 0, 0),
                rope_base: float = 10000.0, max_rounds: int = 1024,
                num_pages: int = 0, mask: str = "wf") -> WfPoolConfig:
    c = WfPoolConfig()
    c.num_stages, c.chunk_tokens, c.num_heads, c.head_dim = num_stages, chunk_tokens, num_heads, head_dim
    c.anchor_chunks, c.history_chunks, c.page_tokens = anchor_chunks, history_chunks, page_tokens
    c.num_layers = num_layers
    c.dtype = _DTYPES[dtype][0]
    c.rope = rope
    c.frames_per_chunk, c.grid_h, c.grid_w = frames_per_chunk, grid_h, grid_w
    for i in range(3):
        c.rope_split[i] = int(rope_split[i])
    c.rope_base = rope_base
    c.max_rounds = max_rounds
    c.num_pages = num_pages
    c.mask_mode = {"wf": _wf.WF_MASK_WF, "rf": _wf.WF_MASK_RF}[mask]
    return c


def _ptr(t: torch.Tensor) -> int:
    if not t.is_contiguous():
        raise ValueError("tensors passed to libwf must be contiguous")
    return t.data_ptr()


def _stream(device, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


class KVPool:
    """A paged K/V pool on one GPU (or host-only bookkeeping when device=None)."""

    def __init__(self, cfg: WfPoolConfig, device: Optional[torch.device] = None,
                 page_order: Optional[Sequence[int]] = None, stream=None,
                 mem: Optional[torch.Tensor] = None):
        """``mem`` reuses an existing uint8 device buffer of at least
        wf_kv_pool_bytes(cfg) bytes (the pool restarts at round 0 in it)."""
        self.cfg = cfg
        self.nbytes = _wf.wf_kv_pool_bytes(cfg)
        self.device = None if device is None else torch.device(device)
        # element type of the pages and of q_rot (E4M3 codes as uint8 for FP8
        # pools); q, k, v inputs and out are bf16 for bf16 and FP8 pools
        self.dtype = _ELEMENT[cfg.dtype]
        self.io_dtype = torch.float32 if cfg.dtype == _wf.WF_DTYPE_F32 else torch.bfloat16
        self.mem = None
        if self.device is not None:
            if mem is not None:
                if mem.dtype != torch.uint8 or mem.numel() < self.nbytes or not mem.is_cuda:
                    raise ValueError("mem must be a CUDA uint8 tensor of at least wf_kv_pool_bytes")
                self.mem = mem
            else:
                self.mem = torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)
            with torch.cuda.device(self.device):
                self.handle = _wf.wf_kv_pool_create(cfg, self.mem.data_ptr(), self.nbytes,
                                                    page_order, _stream(self.device, stream))
        else:
            self.handle = _wf.wf_kv_pool_create(cfg, 0, 0, page_order, 0)
        self.geometry = _wf.wf_pool_get_geometry(self.handle)

    # -- round calls -----------------------------------------------------------------
    def publish(self, layer: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                q_rot: torch.Tensor, stream=None) -> None:
        st = _wf.wf_publish_kv(self.handle, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(q_rot),
                               _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_publish_kv")

    def project_publish(self, layer: int, x: torch.Tensor, w_qkv: torch.Tensor,
                        q_rot: torch.Tensor, stream=None) -> None:
        st = _wf.wf_project_publish(self.handle, layer, _ptr(x), _ptr(w_qkv), _ptr(q_rot),
                                    _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_project_publish")

    def attention(self, layer: int, q_rot: torch.Tensor, out: torch.Tensor, stream=None) -> None:
        st = _wf.wf_round_attention(self.handle, layer, _ptr(q_rot), _ptr(out),
                                    _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_round_attention")

    # -- Wave Parallelism: one slot per rank ------------------------------------------
    def publish_slot(self, layer: int, slot: int, q: torch.Tensor, k: torch.Tensor,
                     v: torch.Tensor, q_rot: torch.Tensor, stream=None) -> None:
        st = _wf.wf_publish_kv_slot(self.handle, layer, slot, _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(q_rot), _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_publish_kv_slot")

    def attention_slot(self, layer: int, slot: int, q_rot: torch.Tensor, out: torch.Tensor,
                       stream=None) -> None:
        st = _wf.wf_round_attention_slot(self.handle, layer, slot, _ptr(q_rot), _ptr(out),
                                         _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_round_attention_slot")

    def deliver(self, layer: int, slot: int, dst: "KVPool", stream=None) -> None:
        """Copy this pool's pages of `slot` (published in this round) into the
        receiver pool `dst` (same config, page order and round) and stamp its
        ready tags. `dst.mem` must be addressable from this pool's device."""
        self.deliver_to(layer, slot, dst.mem.data_ptr(), dst.nbytes, stream)

    def deliver_to(self, layer: int, slot: int, dst_pool_mem: int, dst_pool_bytes: int,
                   stream=None) -> None:
        """wf_deliver_kv into a receiver given by its raw device pointer and size,
        e.g. another process's pool buffer mapped with wf_ipc_open_mem."""
        st = _wf.wf_deliver_kv(self.handle, layer, slot, dst_pool_mem, dst_pool_bytes,
                               _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_deliver_kv")

    def ipc_handle(self):
        """(handle bytes, offset) exporting this pool's buffer to other processes."""
        return _wf.wf_ipc_get_mem_handle(self.mem.data_ptr())

    def stall_next_attention(self, key_tile: int, wait_limit_cycles: int) -> None:
        """Test hook: the next attention launch skips one K load and gives up on
        its waits after wait_limit_cycles (wf_pool_debug_stall_next_attention)."""
        st = _wf.wf_pool_debug_stall_next_attention(self.handle, key_tile, wait_limit_cycles)
        if st != _wf.WF_OK:
            raise WfError(st, "wf_pool_debug_stall_next_attention")

    def advance(self, stream=None) -> None:
        s = 0 if self.device is None else _stream(self.device, stream)
        st = _wf.wf_advance_round(self.handle, s)
        if st != _wf.WF_OK:
            raise WfError(st, "wf_advance_round")

    def check_status(self, stream=None) -> int:
        s = 0 if self.device is None else _stream(self.device, stream)
        return _wf.wf_pool_check_status(self.handle, s)

    # -- queries -------------------------------------------------------------------
    @property
    def round(self) -> int:
        return _wf.wf_pool_round(self.handle)

    def layout(self):
        """[(kind, chunk, slot, expected_tag, [physical pages])] in context order."""
        g = self.geometry
        return _wf.wf_pool_get_layout(self.handle, g.max_positions, g.pages_per_chunk)

    def pages_view(self) -> torch.Tensor:
        """The page region as [layers][num_pages][2][heads][P][d] (K = 0, V = 1)."""
        g, c = self.geometry, self.cfg
        n = c.num_layers * g.num_pages * g.page_bytes
        raw = self.mem[g.pages_offset:g.pages_offset + n]
        return raw.view(self.dtype).view(c.num_layers, g.num_pages, 2, c.num_heads,
                                         c.page_tokens, c.head_dim)

    def kv_scales_view(self) -> torch.Tensor:
        """FP8 pools: the block scales as [layers][num_pages][2][heads] fp32."""
        g, c = self.geometry, self.cfg
        if c.dtype != _wf.WF_DTYPE_FP8_E4M3:
            raise ValueError("only FP8 pools carry scales")
        n = c.num_layers * g.num_pages * 2 * c.num_heads * 4
        raw = self.mem[g.kv_scale_offset:g.kv_scale_offset + n]
        return raw.view(torch.float32).view(c.num_layers, g.num_pages, 2, c.num_heads)

    def q_scales_view(self) -> torch.Tensor:
        """FP8 pools: q_rot's tile scales as [layers][S+1][pages_per_chunk][heads] fp32."""
        g, c = self.geometry, self.cfg
        if c.dtype != _wf.WF_DTYPE_FP8_E4M3:
            raise ValueError("only FP8 pools carry scales")
        n = c.num_layers * (c.num_stages + 1) * g.pages_per_chunk * c.num_heads * 4
        raw = self.mem[g.q_scale_offset:g.q_scale_offset + n]
        return raw.view(torch.float32).view(c.num_layers, c.num_stages + 1, g.pages_per_chunk,
                                            c.num_heads)

    def tags_view(self) -> torch.Tensor:
        g, c = self.geometry, self.cfg
        raw = self.mem[g.tags_offset:g.tags_offset + c.num_layers * g.num_pages * 4]
        return raw.view(torch.int32).view(c.num_layers, g.num_pages)

    def poke_page(self, position: int, j: int, physical: int, stream=None) -> None:
        st = _wf.wf_pool_debug_poke_page(self.handle, position, j, physical,
                                         _stream(self.device, stream))
        if st != _wf.WF_OK:
            raise WfError(st, "wf_pool_debug_poke_page")

    def close(self) -> None:
        if getattr(self, "handle", None):
            _wf.wf_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
