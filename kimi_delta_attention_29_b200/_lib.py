"""ctypes binding of libkda.so (the C ABI declared in include/kda.h).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
Loading fails loudly if the library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")

# Status codes (include/kda.h)
KDA_OK = 0
KDA_ERR_NULL_ARG = -1
KDA_ERR_BAD_SHAPE = -2
KDA_ERR_BAD_DTYPE = -3
KDA_ERR_MISALIGNED = -4
KDA_ERR_UNSUPPORTED = -5
KDA_ERR_BAD_SEQLENS = -6
KDA_ERR_WORKSPACE_TOO_SMALL = -7
KDA_ERR_CUDA = -8
KDA_ERR_TIMEOUT = -9
KDA_ERR_ALIASING = -10
KDA_ERR_BAD_SLOT = -11
KDA_ERR_BAD_VALUE = -12

KDA_F32 = 0
KDA_BF16 = 1

# Prologue flags of the _ex entry points
KDA_PROLOGUE_L2NORM_QK = 1
KDA_PROLOGUE_GATE = 2

# Every entry point include/kda.h declares.
EXPORTED = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_chunk_fwd_noalloc", "kda_chunk_fwd_ex", "kda_decode_step",
            "kda_decode_multi", "kda_decode_multi_ex", "kda_output_gate_norm", "kda_chunk_bwd_workspace_size",
            "kda_chunk_bwd", "kda_state_compose", "kda_segment_map", "kda_get_status",
            "kda_status_string", "kda_version", "kda_trace_begin", "kda_trace_end")

KERNEL_NAMES = {0: "kda_chunk_table_kernel", 1: "kda_tc_prep_kernel", 2: "kda_tc_state_kernel",
                3: "kda_prefill_simt_kernel", 4: "kda_decode_kernel", 5: "kda_decode_multi_kernel",
                6: "kda_output_gate_norm_kernel", 7: "kda_bwd_state_kernel", 8: "kda_bwd_chunk_kernel",
                9: "kda_bwd_prep_kernel", 10: "kda_state_compose_kernel",
                11: "kda_tc_prefill (state kernel and intra-chunk kernel, concurrent)", 12: "kda_bwd_pair_kernel"}

_lib = None


def load() -> ctypes.CDLL:
    """Load libkda.so once and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m kimi_delta_attention_29_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    i, sz = ctypes.c_int, ctypes.c_size_t
    lib.kda_chunk_fwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.kda_chunk_fwd_workspace_size.restype = sz
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, ip, i, i, i, i, i, i, i, i, vp, fp, vp, sz, vp]
    lib.kda_chunk_fwd.restype = i
    lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, ip, i, i, i, i, i, i, i, i, vp, fp, vp]
    lib.kda_chunk_fwd_noalloc.restype = i
    lib.kda_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, i, i, i, i, i, vp, vp]
    lib.kda_decode_step.restype = i
    lib.kda_decode_multi.argtypes = [vp, vp, vp, fp, fp, fp, i, ip, ip, i, i, i, i, i, i, vp, ip, vp]
    lib.kda_decode_multi.restype = i
    u = ctypes.c_uint
    lib.kda_chunk_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, ip, i, i, i, i, i, i, i, i, vp, fp, vp, sz, u, fp, fp, vp]
    lib.kda_chunk_fwd_ex.restype = i
    lib.kda_decode_multi_ex.argtypes = [vp, vp, vp, fp, fp, fp, i, ip, ip, i, i, i, i, i, i, vp, ip, u, fp, fp, vp]
    lib.kda_decode_multi_ex.restype = i
    lib.kda_chunk_bwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.kda_chunk_bwd_workspace_size.restype = sz
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, ip, i, i, i, i, i, i, i, i, vp, fp, vp, vp, vp, fp, fp, fp,
                                  vp, sz, vp]
    lib.kda_chunk_bwd.restype = i
    lib.kda_state_compose.argtypes = [fp, fp, i, i, i, i, fp, fp, vp]
    lib.kda_state_compose.restype = i
    lib.kda_segment_map.argtypes = [vp, vp, vp, fp, fp, i, i, i, i, i, i, vp, fp, vp, sz, vp]
    lib.kda_segment_map.restype = i
    lib.kda_output_gate_norm.argtypes = [vp, vp, fp, ctypes.c_float, i, i, i, i, vp, vp]
    lib.kda_output_gate_norm.restype = i
    lib.kda_get_status.argtypes = [vp, vp]
    lib.kda_get_status.restype = i
    lib.kda_status_string.argtypes = [i]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_trace_begin.argtypes = [i]
    lib.kda_trace_begin.restype = i
    lib.kda_trace_end.argtypes = [ctypes.c_void_p, ctypes.c_void_p, i]
    lib.kda_trace_end.restype = i
    lib.kda_version.argtypes = []
    lib.kda_version.restype = i
    _lib = lib
    return lib


class KdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


def status_string(code: int) -> str:
    return load().kda_status_string(int(code)).decode()
