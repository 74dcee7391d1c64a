"""ctypes declarations of libssd_bidir.so (see include/ssd_bidir.h).

Loading fails loudly: there is no Python or CPU implementation behind these
names, so a missing or stale library is an ImportError, not a fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssd_bidir.so")

# Values of include/ssd_bidir.h.
SSD_F32, SSD_BF16 = 0, 1
SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED = 0, -1, -2
SSD_ERR_CUDA, SSD_ERR_WORKSPACE, SSD_ERR_TIMEOUT = -3, -4, -5
SSD_OP_BIDIR_FWD, SSD_OP_PREFIX_STATE, SSD_OP_BLOCK_STEP, SSD_OP_BIDIR_BWD = 0, 1, 2, 3
SSD_OP_BIDIR_FWD_X2, SSD_OP_MIXER_BLOCK = 4, 5
SSD_PATH_AUTO, SSD_PATH_SIMT, SSD_PATH_CHUNKED, SSD_PATH_FUSED, SSD_PATH_SEGMENTED, SSD_PATH_PAIR = 0, 1, 2, 3, 4, 5
SSD_PATH_BLOCK = 6
SSD_PATH_ONETILE = 7

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

# name -> (restype, argtypes); the C-ABI surface the header declares.
SIGNATURES = {
    "ssd_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "ssd_select_path": (_i, [_i] * 8),
    "ssd_workspace_init": (_i, [_vp, _sz, _vp]),
    "ssd_bidir_fwd": (_i, [_vp] * 7 + [_i] * 8 + [_vp, _sz, _vp]),
    "ssd_bidir_fwd_path": (_i, [_vp] * 7 + [_i] * 9 + [_vp, _sz, _vp]),
    "ssd_prefix_state": (_i, [_vp] * 6 + [_i] * 8 + [_vp, _sz, _vp]),
    "ssd_block_step": (_i, [_vp] * 8 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_prefix_state_path": (_i, [_vp] * 6 + [_i] * 9 + [_vp, _sz, _vp]),
    "ssd_block_step_path": (_i, [_vp] * 8 + [_i] * 8 + [_vp, _sz, _vp]),
    "ssd_bidir_fwd_noalloc": (_i, [_vp] * 7 + [_i] * 8 + [_vp]),
    "ssd_noalloc_get_status": (_i, [_vp]),
    "ssd_segment_states": (_i, [_vp] * 8 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_segment_carry": (_i, [_vp] * 4 + [_i] * 2 + [_vp] * 2 + [_i] * 4 + [_vp]),
    "ssd_bidir_fwd_seeded": (_i, [_vp] * 9 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_bidir_fwd_dtraw": (_i, [_vp] * 3 + [ctypes.c_float] * 2 + [_vp] * 5 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_bidir_bwd": (_i, [_vp] * 13 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_bidir_bwd_seeded": (_i, [_vp] * 17 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_prefix_state_layers": (_i, [_vp] * 6 + [_i] * 9 + [_vp, _sz, _vp]),
    "ssd_bidir_fwd_x2": (_i, [_vp] * 7 + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_mixer_block_fwd": (_i, [_vp] * 5 + [_i, _vp] + [ctypes.c_float] * 2 + [_vp] * 3 + [ctypes.c_float, _vp]
                            + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_get_device_status": (_i, [_vp, _vp]),
    "ssd_selftest_wait_timeout": (_i, [_vp, _sz, _i, _vp]),
    "ssd_error_string": (ctypes.c_char_p, [_i]),
    "ssd_version": (_i, []),
}

_lib = None


def load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is not built; run `python -c 'import __graft_entry__ as g; g.build()'` "
                "(nvcc, sm_100a). There is no fallback implementation.")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib
