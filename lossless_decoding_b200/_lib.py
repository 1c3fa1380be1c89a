"""ctypes loader for libuno.so and the declarations of its C ABI (include/uno.h).

The library is required: if it is missing or cannot be loaded, importing this
module raises, and nothing falls back to another implementation.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libuno.so")

UNO_BF16 = 0
UNO_F32 = 1

STATUS = {
    0: "UNO_OK",
    -1: "UNO_ERR_NULL",
    -2: "UNO_ERR_SIZE",
    -3: "UNO_ERR_ALIGN",
    -4: "UNO_ERR_DTYPE",
    -5: "UNO_ERR_WORKSPACE",
    -6: "UNO_ERR_CUDA",
    -7: "UNO_ERR_DEVICE",
}


class UnoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {lib.uno_status_string(status).decode()}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m lossless_decoding_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
    L.uno_status_string.argtypes = [i32]
    L.uno_status_string.restype = ctypes.c_char_p
    L.uno_version.argtypes = []
    L.uno_version.restype = i32
    L.uno_verify_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.uno_verify_workspace_bytes.restype = sz
    L.uno_verify_block.argtypes = [vp, vp, vp, i32, i32, i32, i32, u64, u64, vp, vp, vp, vp, vp,
                                   vp, sz, vp]
    L.uno_verify_block.restype = i32
    L.uno_verify_block_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, u64, u64, vp, vp, vp,
                                           vp, vp, vp]
    L.uno_verify_block_noalloc.restype = i32
    L.uno_dualpath_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.uno_dualpath_workspace_bytes.restype = sz
    L.uno_dualpath_linear.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp, vp, i32, i32, i32, i32,
                                      i32, vp, sz, vp]
    L.uno_dualpath_linear.restype = i32
    L.uno_dualpath_grouped_workspace_bytes.argtypes = [i32, i32, i32, vp, i32, i32]
    L.uno_dualpath_grouped_workspace_bytes.restype = sz
    L.uno_dualpath_linear_grouped.argtypes = [i32, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp,
                                              i32, i32, vp, sz, vp]
    L.uno_dualpath_linear_gated.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, i32, i32,
                                            i32, i32, i32, vp, sz, vp]
    L.uno_dualpath_linear_gated.restype = i32
    L.uno_dualpath_linear_grouped.restype = i32
    L.uno_sample_drafts.argtypes = [vp, i32, i32, i32, i32, u64, u64, vp, vp]
    L.uno_sample_drafts.restype = i32
    L.uno_sample_drafts_blocks.argtypes = [vp, i32, i32, i32, i32, i32, u64, u64, vp, vp]
    L.uno_sample_drafts_blocks.restype = i32
    L.uno_dualpath_stats_tiles.argtypes = [i32, i32]
    L.uno_dualpath_stats_tiles.restype = i32
    L.uno_dualpath_linear_stats.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, vp,
                                            i32, i32, i32, i32, i32, vp, sz, vp]
    L.uno_dualpath_linear_stats.restype = i32
    L.uno_verify_block_head.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, u64, u64,
                                        vp, vp, vp, vp, vp, vp, sz, vp]
    L.uno_verify_block_head.restype = i32
    L.uno_tree_nodes.argtypes = [i32, i32]
    L.uno_tree_nodes.restype = i32
    L.uno_tree_draft_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.uno_tree_draft_workspace_bytes.restype = sz
    L.uno_tree_draft.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                 sz, vp]
    L.uno_tree_draft.restype = i32
    L.uno_tree_verify.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, u64, u64, vp, vp,
                                  vp, vp]
    L.uno_tree_verify.restype = i32
    L.uno_device_fault_flags.argtypes = [i32, ctypes.POINTER(ctypes.c_uint)]
    L.uno_device_fault_flags.restype = i32
    L.uno_dualpath_test_hooks.argtypes = [u64, ctypes.c_uint32]
    L.uno_dualpath_test_hooks.restype = i32
    return L


lib = _load()
