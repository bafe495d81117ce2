"""ctypes binding of libh2o.so: the C ABI of include/h2o.h, names unchanged.

Argument marshalling only -- every step of the chunk runs in the library's CUDA
kernels.  Importing this module loads the in-tree libh2o.so and fails loudly if
it has not been built (``python h2o_kv_cache_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

# H2O_LIBRARY names another build of the same library to load instead (the
# stamps build of stamps.py); unset, the in-tree libh2o.so
LIB_PATH = os.environ.get("H2O_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                         "libh2o.so")

H2O_OK, H2O_EINVAL, H2O_ESHAPE, H2O_ESTATE, H2O_ENOMEM, H2O_ECUDA, H2O_ETIMEOUT = 0, -1, -2, -3, -4, -5, -6
H2O_F32, H2O_BF16 = 0, 1
H2O_POLICY_H2O, H2O_POLICY_LR = 0, 1
STATUS_NAMES = {0: "H2O_OK", -1: "H2O_EINVAL", -2: "H2O_ESHAPE", -3: "H2O_ESTATE",
                -4: "H2O_ENOMEM", -5: "H2O_ECUDA", -6: "H2O_ETIMEOUT"}

_i64, _i32, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p

# name -> (restype, argtypes), exactly the declarations of include/h2o.h
SIGNATURES = {
    "h2o_create": (_i32, [_i64, _i64, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp)]),
    "h2o_create_policy": (_i32, [_i64, _i64, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp)]),
    "h2o_prefill": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _vp]),
    "h2o_step": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _vp]),
    "h2o_step_layers": (_i32, [ctypes.POINTER(_vp), _i32, ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                               ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i64, _vp]),
    "h2o_read_state": (_i32, [_vp, _vp, _vp, _vp, _vp]),
    "h2o_read_kv": (_i32, [_vp, _vp, _vp, _vp]),
    "h2o_read_delta": (_i32, [_vp, _vp, _vp, _vp]),
    "h2o_info": (_i32, [_vp, ctypes.POINTER(_i64)]),
    "h2o_set_profiling": (_i32, [_vp, _i32]),
    "h2o_step_timings": (_i32, [_vp, _i32, ctypes.POINTER(ctypes.c_float), _i32]),
    "h2o_last_timings": (_i32, [_vp, ctypes.POINTER(ctypes.c_float), _i32]),
    "h2o_destroy": (_i32, [_vp]),
    "h2o_last_error": (ctypes.c_char_p, [_vp]),
    "h2o_select": (_i32, [_vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _vp]),
    "h2o_attend_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i64,
                                  _i64, _i64, _vp, _vp, _vp]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python h2o_kv_cache_b200/build.py` "
                          "(the library has no fallback path)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    for extra in ("h2o_stamps_read", "h2o_tail_stamps_read", "h2o_unit_stamps_read"):   # stamps build only
        if hasattr(lib, extra):
            getattr(lib, extra).restype = _i32
            getattr(lib, extra).argtypes = [_vp]
    if hasattr(lib, "h2o_tail_empty_launch"):   # stamps build only
        lib.h2o_tail_empty_launch.restype = _i32
        lib.h2o_tail_empty_launch.argtypes = [_i32, _i32, _i32, _i32, _vp]
    return lib


lib = load()
