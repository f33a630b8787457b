"""Wave Forcing round attention on NVIDIA B200 (sm_100a).

One causal-wavefront round of chunk-wise causal attention ("Wave Forcing:
Towards Speed-of-Light Streaming Video Generation"): early K/V publication
with 3D rotary embedding into a paged pool, then M_WF-masked round attention on
the 5th-generation tensor cores. The C ABI is include/wf.h (libwf.so); this
package is its Python binding.
"""
from .wf import (LIB_PATH, WF_DTYPE_BF16, WF_DTYPE_F32, WF_DTYPE_FP8_E4M3, WF_ERR_BAD_PAGE, WF_ERR_CALL_ORDER,
                 WF_ERR_CUDA, WF_ERR_INVALID_ARG, WF_ERR_NOT_READY, WF_ERR_OUT_OF_PAGES,
                 WF_ERR_TIMEOUT, WF_ERR_UNSUPPORTED, WF_MASK_RF, WF_MASK_WF, WF_OK, WF_ROPE_3D,
                 WF_ROPE_OFF, WfError,
                 WfPoolConfig, wf_status_string)
from .pool import KVPool, make_config

__all__ = [
    "KVPool", "make_config", "WfError", "WfPoolConfig", "wf_status_string", "LIB_PATH",
    "WF_OK", "WF_ERR_INVALID_ARG", "WF_ERR_OUT_OF_PAGES", "WF_ERR_NOT_READY", "WF_ERR_BAD_PAGE",
    "WF_ERR_CALL_ORDER", "WF_ERR_CUDA", "WF_ERR_UNSUPPORTED", "WF_ERR_TIMEOUT",
    "WF_DTYPE_BF16", "WF_DTYPE_F32", "WF_DTYPE_FP8_E4M3", "WF_ROPE_OFF", "WF_ROPE_3D", "WF_MASK_WF", "WF_MASK_RF",
]
