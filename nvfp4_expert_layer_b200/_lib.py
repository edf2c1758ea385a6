"""ctypes declarations of libmoe_fp4.so (the C ABI in include/moe_fp4.h).

Loading fails loudly: there is no fallback implementation of the layer."""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_fp4.so")

STATUS = {
    0: "MOE_FP4_OK", 1: "MOE_FP4_ERR_INVALID_ARG", 2: "MOE_FP4_ERR_UNSUPPORTED",
    3: "MOE_FP4_ERR_NOT_LOADED", 4: "MOE_FP4_ERR_CUDA", 5: "MOE_FP4_ERR_OOM",
    6: "MOE_FP4_ERR_DEVICE_TIMEOUT", 7: "MOE_FP4_ERR_NUMERIC", 8: "MOE_FP4_ERR_CAPTURE",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

_vp = ctypes.c_void_p
_i = ctypes.c_int


class Experts(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("gate_q", "gate_sf", "gate_gs", "up_q", "up_sf", "up_gs",
                                   "down_q", "down_sf", "down_gs")]


class Routing(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("logits", "topk_ids", "topk_w", "counts", "offsets", "perm", "inv")]


class Debug(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("logits", "topk_ids", "topk_w", "counts", "offsets", "perm",
                                   "h", "partial")]


# name -> (restype, argtypes); must match every MOE_FP4_API declaration of the header
SIGNATURES = {
    "moe_fp4_create": (_i, [_i, _i, _i, _i, ctypes.POINTER(_vp)]),
    "moe_fp4_load_experts": (_i, [_vp, ctypes.POINTER(Experts)]),
    "moe_fp4_reserve": (_i, [_vp, _i]),
    "moe_fp4_forward": (_i, [_vp, _vp, _i, _vp, _vp, _vp]),
    "moe_fp4_forward_ex": (_i, [_vp, _vp, _i, _vp, _vp, _vp, ctypes.POINTER(Debug)]),
    "moe_fp4_forward_host": (_i, [_vp, _vp, _i, _vp, _vp, _vp]),
    "moe_fp4_set_dense_threshold": (_i, [_vp, _i]),
    "moe_fp4_set_expert_norm": (_i, [_vp, _i, ctypes.c_float]),
    "moe_fp4_set_act_scale": (_i, [_vp, _i]),
    "moe_fp4_set_residual": (_i, [_vp, _i]),
    "moe_fp4_forward_layers": (_i, [ctypes.POINTER(_vp), _i, _vp, _i, ctypes.POINTER(_vp), _vp, _vp]),
    "moe_fp4_route": (_i, [_vp, _vp, _i, _vp, ctypes.POINTER(Routing), _vp]),
    "moe_fp4_gather_rows": (_i, [_vp, _i, _i, _vp, _i, _i, _vp, _vp]),
    "moe_fp4_forward_routed": (_i, [_vp, _vp, _i, _vp, _vp, _vp]),
    "moe_fp4_combine_rows": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_fp4_set_resident_classes": (_i, [_vp, _i, _i]),
    "moe_fp4_device_bytes": (_i, [_vp, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "moe_fp4_set_wait_timeout_ms": (_i, [_vp, _i]),
    "moe_fp4_set_unreachable_wait": (_i, [_vp, _i]),
    "moe_fp4_get_device_error": (_i, [_vp, ctypes.POINTER(_i)]),
    "moe_fp4_set_stage_events": (_i, [_vp, ctypes.POINTER(_vp), _i]),
    "moe_fp4_route_topk_static": (_i, [_vp, _i, _i, _vp, _i, _i, _vp, _vp, _vp]),
    "moe_fp4_status_string": (ctypes.c_char_p, [_i]),
    "moe_fp4_last_error_detail": (ctypes.c_char_p, []),
    "moe_fp4_destroy": (None, [_vp]),
}

_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libmoe_fp4.so (built in-tree by nvfp4_expert_layer_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or os.environ.get("MOE_FP4_LIB", LIB_PATH)
    if not os.path.exists(p):
        raise RuntimeError(f"libmoe_fp4.so not found at {p}; build it with "
                           "`python -m nvfp4_expert_layer_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


class MoeFp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def check(status: int, where: str) -> None:
    if status != 0:
        if status == STATUS_CODE["MOE_FP4_ERR_CUDA"] and _lib is not None:
            where = f"{where} [{_lib.moe_fp4_last_error_detail().decode()}]"
        raise MoeFp4Error(status, where)
