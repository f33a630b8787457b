"""ctypes binding of libwf (include/wf.h): argument marshalling only.

Every step of the round runs in libwf's CUDA kernels; PyTorch is used here only
for device memory and streams. Importing this module fails loudly if libwf.so
has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwf.so")

WF_OK = 0
WF_ERR_INVALID_ARG = 1
WF_ERR_OUT_OF_PAGES = 2
WF_ERR_NOT_READY = 3
WF_ERR_BAD_PAGE = 4
WF_ERR_CALL_ORDER = 5
WF_ERR_CUDA = 6
WF_ERR_UNSUPPORTED = 7
WF_ERR_TIMEOUT = 8
WF_DTYPE_BF16 = 0
WF_DTYPE_F32 = 1
WF_DTYPE_FP8_E4M3 = 2
WF_ROPE_OFF = 0
WF_ROPE_3D = 1
WF_MASK_WF = 0
WF_MASK_RF = 1
KIND_NAMES = {0: "anchor", 1: "history", 2: "store", 3: "slot"}

EXPORTS = (
    "wf_kv_pool_bytes", "wf_kv_pool_create", "wf_publish_kv", "wf_round_attention",
    "wf_advance_round", "wf_pool_check_status", "wf_pool_destroy", "wf_status_string",
    "wf_pool_round", "wf_pool_get_geometry", "wf_pool_get_layout", "wf_pool_debug_poke_page",
    "wf_project_publish", "wf_publish_kv_slot", "wf_round_attention_slot", "wf_deliver_kv",
    "wf_pool_debug_stall_next_attention", "wf_ipc_get_mem_handle", "wf_ipc_open_mem",
    "wf_ipc_close_mem",
)


class WfPoolConfig(ctypes.Structure):
    _fields_ = [
        ("num_stages", ctypes.c_int32), ("chunk_tokens", ctypes.c_int32),
        ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("anchor_chunks", ctypes.c_int32), ("history_chunks", ctypes.c_int32),
        ("page_tokens", ctypes.c_int32), ("num_layers", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("rope", ctypes.c_int32),
        ("frames_per_chunk", ctypes.c_int32), ("grid_h", ctypes.c_int32),
        ("grid_w", ctypes.c_int32), ("rope_split", ctypes.c_int32 * 3),
        ("rope_base", ctypes.c_float), ("max_rounds", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("mask_mode", ctypes.c_int32),
    ]


class WfPoolGeometry(ctypes.Structure):
    _fields_ = [
        ("num_pages", ctypes.c_int64), ("pages_per_chunk", ctypes.c_int32),
        ("max_positions", ctypes.c_int32), ("status_offset", ctypes.c_size_t),
        ("tags_offset", ctypes.c_size_t), ("pages_offset", ctypes.c_size_t),
        ("page_bytes", ctypes.c_size_t), ("total_bytes", ctypes.c_size_t),
        ("kv_scale_offset", ctypes.c_size_t), ("q_scale_offset", ctypes.c_size_t),
    ]


class WfIpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


class WfError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {wf_status_string(self.status)}" if what else
                         wf_status_string(self.status))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python chunk_causal_wavefront_b200/build.py` "
            "(the CUDA library is required; there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(WfPoolConfig)
    i32p = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "wf_kv_pool_bytes": (I32, [cfgp, ctypes.POINTER(SZ)]),
        "wf_kv_pool_create": (I32, [cfgp, P, SZ, i32p, P, ctypes.POINTER(P)]),
        "wf_publish_kv": (I32, [P, I32, P, P, P, P, P]),
        "wf_round_attention": (I32, [P, I32, P, P, P]),
        "wf_advance_round": (I32, [P, P]),
        "wf_pool_check_status": (I32, [P, P]),
        "wf_pool_destroy": (I32, [P]),
        "wf_status_string": (ctypes.c_char_p, [I32]),
        "wf_pool_round": (I64, [P]),
        "wf_pool_get_geometry": (I32, [P, ctypes.POINTER(WfPoolGeometry)]),
        "wf_pool_get_layout": (I32, [P, i32p, i32p, i32p, i32p, i32p, i32p, I32]),
        "wf_pool_debug_poke_page": (I32, [P, I32, I32, I32, P]),
        "wf_project_publish": (I32, [P, I32, P, P, P, P]),
        "wf_publish_kv_slot": (I32, [P, I32, I32, P, P, P, P, P]),
        "wf_round_attention_slot": (I32, [P, I32, I32, P, P, P]),
        "wf_deliver_kv": (I32, [P, I32, I32, P, SZ, P]),
        "wf_pool_debug_stall_next_attention": (I32, [P, I32, I64]),
        "wf_ipc_get_mem_handle": (I32, [P, ctypes.POINTER(WfIpcHandle), ctypes.POINTER(SZ)]),
        "wf_ipc_open_mem": (I32, [ctypes.POINTER(WfIpcHandle), SZ, ctypes.POINTER(P)]),
        "wf_ipc_close_mem": (I32, [P, SZ]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


# --- same-named thin wrappers ---------------------------------------------------

def wf_status_string(status: int) -> str:
    return _lib.wf_status_string(int(status)).decode()


def wf_kv_pool_bytes(cfg: WfPoolConfig) -> int:
    n = ctypes.c_size_t(0)
    st = _lib.wf_kv_pool_bytes(ctypes.byref(cfg), ctypes.byref(n))
    if st != WF_OK:
        raise WfError(st, "wf_kv_pool_bytes")
    return n.value


def wf_kv_pool_create(cfg: WfPoolConfig, dev_mem: int, nbytes: int,
                      page_order: Optional[Sequence[int]], stream: int) -> int:
    arr = None
    if page_order is not None:
        arr = (ctypes.c_int32 * len(page_order))(*[int(x) for x in page_order])
    out = ctypes.c_void_p(0)
    st = _lib.wf_kv_pool_create(ctypes.byref(cfg), ctypes.c_void_p(dev_mem or None), nbytes,
                                arr, ctypes.c_void_p(stream or None), ctypes.byref(out))
    if st != WF_OK:
        raise WfError(st, "wf_kv_pool_create")
    return out.value


def wf_publish_kv(pool: int, layer: int, q: int, k: int, v: int, q_rot: int, stream: int) -> int:
    return _lib.wf_publish_kv(pool, layer, q, k, v, q_rot, ctypes.c_void_p(stream or None))


def wf_round_attention(pool: int, layer: int, q_rot: int, out: int, stream: int) -> int:
    return _lib.wf_round_attention(pool, layer, q_rot, out, ctypes.c_void_p(stream or None))


def wf_publish_kv_slot(pool: int, layer: int, slot: int, q: int, k: int, v: int, q_rot: int,
                       stream: int) -> int:
    return _lib.wf_publish_kv_slot(pool, layer, slot, q, k, v, q_rot,
                                   ctypes.c_void_p(stream or None))


def wf_round_attention_slot(pool: int, layer: int, slot: int, q_rot: int, out: int,
                            stream: int) -> int:
    return _lib.wf_round_attention_slot(pool, layer, slot, q_rot, out,
                                        ctypes.c_void_p(stream or None))


def wf_deliver_kv(pool: int, layer: int, slot: int, dst_pool_mem: int, dst_pool_bytes: int,
                  stream: int) -> int:
    return _lib.wf_deliver_kv(pool, layer, slot, dst_pool_mem, dst_pool_bytes,
                              ctypes.c_void_p(stream or None))


def wf_pool_debug_stall_next_attention(pool: int, key_tile: int, wait_limit_cycles: int) -> int:
    return _lib.wf_pool_debug_stall_next_attention(pool, key_tile, wait_limit_cycles)


def wf_ipc_get_mem_handle(dev_ptr: int):
    """(64 handle bytes, offset of dev_ptr inside its allocation)."""
    h = WfIpcHandle()
    off = ctypes.c_size_t(0)
    st = _lib.wf_ipc_get_mem_handle(dev_ptr, ctypes.byref(h), ctypes.byref(off))
    if st != WF_OK:
        raise WfError(st, "wf_ipc_get_mem_handle")
    return bytes(h.bytes), off.value


def wf_ipc_open_mem(handle: bytes, offset: int) -> int:
    """Device pointer of another process's exported buffer, mapped here."""
    if len(handle) != 64:
        raise ValueError("an IPC handle is 64 bytes")
    h = WfIpcHandle()
    ctypes.memmove(h.bytes, handle, 64)
    ptr = ctypes.c_void_p(0)
    st = _lib.wf_ipc_open_mem(ctypes.byref(h), offset, ctypes.byref(ptr))
    if st != WF_OK:
        raise WfError(st, "wf_ipc_open_mem")
    return ptr.value


def wf_ipc_close_mem(dev_ptr: int, offset: int) -> int:
    return _lib.wf_ipc_close_mem(dev_ptr, offset)


def wf_advance_round(pool: int, stream: int) -> int:
    return _lib.wf_advance_round(pool, ctypes.c_void_p(stream or None))


def wf_pool_check_status(pool: int, stream: int) -> int:
    return _lib.wf_pool_check_status(pool, ctypes.c_void_p(stream or None))


def wf_pool_destroy(pool: int) -> int:
    return _lib.wf_pool_destroy(pool)


def wf_pool_round(pool: int) -> int:
    return _lib.wf_pool_round(pool)


def wf_pool_get_geometry(pool: int) -> WfPoolGeometry:
    g = WfPoolGeometry()
    st = _lib.wf_pool_get_geometry(pool, ctypes.byref(g))
    if st != WF_OK:
        raise WfError(st, "wf_pool_get_geometry")
    return g


def wf_pool_get_layout(pool: int, max_positions: int, pages_per_chunk: int):
    n = ctypes.c_int32(0)
    cap = max_positions
    kinds = (ctypes.c_int32 * cap)()
    chunks = (ctypes.c_int32 * cap)()
    slots = (ctypes.c_int32 * cap)()
    tags = (ctypes.c_int32 * cap)()
    pages = (ctypes.c_int32 * (cap * pages_per_chunk))()
    st = _lib.wf_pool_get_layout(pool, ctypes.byref(n), kinds, chunks, slots, tags, pages, cap)
    if st != WF_OK:
        raise WfError(st, "wf_pool_get_layout")
    rows = []
    for i in range(n.value):
        rows.append((KIND_NAMES[kinds[i]], chunks[i], None if slots[i] < 0 else slots[i],
                     tags[i], list(pages[i * pages_per_chunk:(i + 1) * pages_per_chunk])))
    return rows


def wf_pool_debug_poke_page(pool: int, position: int, j: int, physical: int, stream: int) -> int:
    return _lib.wf_pool_debug_poke_page(pool, position, j, physical,
                                        ctypes.c_void_p(stream or None))



def wf_project_publish(pool: int, layer: int, x: int, w_qkv: int, q_rot: int, stream: int) -> int:
    return _lib.wf_project_publish(pool, layer, x, w_qkv, q_rot, ctypes.c_void_p(stream or None))
