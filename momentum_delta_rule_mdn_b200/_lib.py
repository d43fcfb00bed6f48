"""ctypes declarations of libmdn's C ABI (include/mdn.h).  No fallback: if the
library is missing or fails to load, importing the binding raises."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libmdn.so")

MDN_OK, MDN_ERR_INVALID_ARG, MDN_ERR_UNSUPPORTED, MDN_ERR_CUDA, MDN_ERR_NONFINITE, \
    MDN_ERR_TIMEOUT = range(6)
MDN_F32, MDN_BF16 = 0, 1
MDN_CHECK_FINITE = 0x1
MDN_FORCE_SIMT = 0x2
MDN_SLICE32 = 0x4
MDN_SLICE64 = 0x8
MDN_SLICE128 = 0x10
MDN_TEST_NO_INTRA = 0x100
MDN_ETA_TANH = 0
MDN_ETA_2SIGMOID = 1

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

# name -> (restype, argtypes); every function include/mdn.h declares.
SIGNATURES = {
    "mdn_abi_version": (_i, []),
    "mdn_status_string": (ctypes.c_char_p, [_i]),
    "mdn_last_cuda_error": (ctypes.c_char_p, []),
    "mdn_chunk_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "mdn_chunk_fwd_workspace_size_flags": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "mdn_chunk_fwd_status": (_i, [_vp, _vp]),
    "mdn_chunk_fwd": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                           _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _i, _vp]),
    "mdn_step": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                      _i, _i, _i, _i, _vp, _vp, _i, _vp]),
    "mdn_step_delta_norm": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                                 _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp]),
    "mdn_gate_params": (_i, [_vp, _vp, _vp, _vp, ctypes.c_longlong, _f, _f, _i,
                             _vp, _vp, _vp, _vp, _vp]),
    "mdn_chunk_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "mdn_chunk_bwd": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp,
                           _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp,
                           _vp, _vp, _vp, _vp, _sz, _i, _vp]),
    "mdn_chunk_fwd_varlen_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "mdn_chunk_fwd_varlen_workspace_size_flags": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "mdn_chunk_fwd_varlen": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _i, _i,
                                  _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _i,
                                  _vp]),
    "mdn_chunk_fwd_preact": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _f, _i, _f, _vp,
                                  _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _i,
                                  _vp]),
    "mdn_chunk_gate_prep": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                 _vp, _vp, _vp, _vp, _vp, _vp]),
    "mdn_chunk_fwd_noalloc": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _f, _vp, _vp,
                                   _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp]),
    "mdn_profile_enable": (_i, [_i]),
    "mdn_profile_read": (_i, [_i, ctypes.POINTER(ctypes.c_char_p),
                              ctypes.POINTER(ctypes.c_double),
                              ctypes.POINTER(ctypes.c_longlong), _i]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(
            f"libmdn.so not found at {path}; build it with "
            "`python -m momentum_delta_rule_mdn_b200.build_lib`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib
