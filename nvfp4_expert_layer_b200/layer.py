"""Python binding of the NVFP4 sparse-MoE layer (argument marshalling only).

PyTorch supplies device memory and the stream; every step of the forward runs
in libmoe_fp4.so's CUDA kernels."""
from __future__ import annotations

import ctypes

import torch

from . import _lib

EXPERT_FIELDS = ("gate_q", "gate_sf", "gate_gs", "up_q", "up_sf", "up_gs",
                 "down_q", "down_sf", "down_gs")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class MoeFp4Layer:
    """Handle of one layer: MoeFp4Layer(E, top_k, d, f) on the current device."""

    def __init__(self, E: int, top_k: int, d: int, f: int):
        self.lib = _lib.load()
        self.E, self.k, self.d, self.f = E, top_k, d, f
        h = ctypes.c_void_p()
        _lib.check(self.lib.moe_fp4_create(E, top_k, d, f, ctypes.byref(h)), "moe_fp4_create")
        self._h = h

    # ------------------------------------------------------------------ setup
    def load_experts(self, experts: dict) -> None:
        """experts: canonical device tensors (uint8 q/sf, float32 gs), see moe_fp4.h."""
        s = _lib.Experts()
        for n in EXPERT_FIELDS:
            t = experts[n]
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous CUDA tensor")
            setattr(s, n, t.data_ptr())
        _lib.check(self.lib.moe_fp4_load_experts(self._h, ctypes.byref(s)), "moe_fp4_load_experts")

    def reserve(self, max_T: int) -> None:
        _lib.check(self.lib.moe_fp4_reserve(self._h, max_T), "moe_fp4_reserve")

    def set_dense_threshold(self, thr: int) -> None:
        _lib.check(self.lib.moe_fp4_set_dense_threshold(self._h, thr), "moe_fp4_set_dense_threshold")

    def set_resident_classes(self, light: bool = True, dense: bool = True) -> None:
        """Weight copies the next load_experts keeps (see moe_fp4.h)."""
        _lib.check(self.lib.moe_fp4_set_resident_classes(self._h, int(light), int(dense)),
                   "moe_fp4_set_resident_classes")

    def device_bytes(self) -> tuple:
        """(weight bytes, workspace bytes) the handle holds on the device."""
        wb, sb = ctypes.c_size_t(0), ctypes.c_size_t(0)
        _lib.check(self.lib.moe_fp4_device_bytes(self._h, ctypes.byref(wb), ctypes.byref(sb)),
                   "moe_fp4_device_bytes")
        return wb.value, sb.value

    def set_expert_norm(self, enable: bool, eps: float = 1e-6) -> None:
        """RMS-normalise each expert's output before the weighted sum (see moe_fp4.h)."""
        _lib.check(self.lib.moe_fp4_set_expert_norm(self._h, 1 if enable else 0, eps),
                   "moe_fp4_set_expert_norm")

    def set_act_scale(self, dynamic: bool) -> None:
        """Dense class: power-of-two activation tensor scales per call (see moe_fp4.h)."""
        _lib.check(self.lib.moe_fp4_set_act_scale(self._h, 1 if dynamic else 0), "moe_fp4_set_act_scale")

    def set_residual(self, enable: bool) -> None:
        """out = bf16(x + MoE(x)) (see moe_fp4.h)."""
        _lib.check(self.lib.moe_fp4_set_residual(self._h, 1 if enable else 0), "moe_fp4_set_residual")

    def set_wait_timeout_ms(self, ms: int) -> None:
        _lib.check(self.lib.moe_fp4_set_wait_timeout_ms(self._h, ms), "moe_fp4_set_wait_timeout_ms")

    def set_unreachable_wait(self, enable: bool) -> None:
        """Test hook: light-class down tiles wait for a count that is never reached."""
        _lib.check(self.lib.moe_fp4_set_unreachable_wait(self._h, 1 if enable else 0),
                   "moe_fp4_set_unreachable_wait")

    STAGES = ("router", "topk", "permute", "dense_quant", "dense_gate_up", "dense_down", "light", "combine")

    def set_stage_events(self, events) -> None:
        """events: list of len(STAGES) + 1 torch.cuda.Event(enable_timing=True), or None to turn off."""
        if events is None:
            _lib.check(self.lib.moe_fp4_set_stage_events(self._h, None, 0), "moe_fp4_set_stage_events")
            self._stage_events = None
            return
        for e in events:            # torch creates the CUDA event at its first record
            if not e.cuda_event:
                e.record()
        n = len(self.STAGES) + 1
        if len(events) != n:
            raise ValueError(f"set_stage_events needs {n} events")
        arr = (ctypes.c_void_p * n)(*[ctypes.c_void_p(e.cuda_event) for e in events])
        _lib.check(self.lib.moe_fp4_set_stage_events(self._h, arr, n), "moe_fp4_set_stage_events")
        self._stage_events = (events, arr)

    def device_error(self) -> int:
        code = ctypes.c_int(0)
        _lib.check(self.lib.moe_fp4_get_device_error(self._h, ctypes.byref(code)),
                   "moe_fp4_get_device_error")
        return code.value

    # ---------------------------------------------------------------- forward
    def _out(self, x, out):
        if out is None:
            out = torch.empty_like(x)
        return out

    def forward(self, x: torch.Tensor, router_w: torch.Tensor, out=None, stream=None):
        out = self._out(x, out)
        T = x.shape[0] if x.dim() == 2 else 0
        _lib.check(self.lib.moe_fp4_forward(self._h, _ptr(x), T, _ptr(router_w), _ptr(out),
                                            _stream_ptr(stream)), "moe_fp4_forward")
        return out

    __call__ = forward

    def forward_ex(self, x: torch.Tensor, router_w: torch.Tensor, out=None, stream=None,
                   want=("logits", "topk_ids", "topk_w", "counts", "offsets", "perm", "h",
                         "partial")):
        out = self._out(x, out)
        T = x.shape[0]
        P = T * self.k
        dev = x.device
        shapes = {"logits": ((T, self.E), torch.float32), "topk_ids": ((T, self.k), torch.int32),
                  "topk_w": ((T, self.k), torch.float32), "counts": ((self.E,), torch.int32),
                  "offsets": ((self.E + 1,), torch.int32), "perm": ((P,), torch.int32),
                  "h": ((P, self.f), torch.float32), "partial": ((P, self.d), torch.float32)}
        bufs = {n: torch.full(shapes[n][0], float("nan") if shapes[n][1] == torch.float32 else -1,
                              dtype=shapes[n][1], device=dev) for n in want}
        dbg = _lib.Debug()
        for n, t in bufs.items():
            setattr(dbg, n, t.data_ptr())
        _lib.check(self.lib.moe_fp4_forward_ex(self._h, _ptr(x), T, _ptr(router_w), _ptr(out),
                                               _stream_ptr(stream), ctypes.byref(dbg)),
                   "moe_fp4_forward_ex")
        return out, bufs

    def forward_host(self, x_host: torch.Tensor, router_w: torch.Tensor, out_host=None,
                     stream=None):
        """x_host / out_host: CPU bf16 tensors (pinned for asynchronous copies)."""
        if out_host is None:
            out_host = torch.empty_like(x_host, pin_memory=x_host.is_pinned())
        _lib.check(self.lib.moe_fp4_forward_host(self._h, _ptr(x_host), x_host.shape[0],
                                                 _ptr(router_w), _ptr(out_host),
                                                 _stream_ptr(stream)), "moe_fp4_forward_host")
        return out_host

    # -------------------------------------------------------------- lifetime
    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            self.lib.moe_fp4_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def experts_to_device(ex, device="cuda") -> dict:
    """Upload workloads.ExpertWeights (numpy) as canonical device tensors."""
    out = {}
    for n in EXPERT_FIELDS:
        a = getattr(ex, n)
        out[n] = torch.from_numpy(a).to(device)
    return out


def forward_layers(layers, x: torch.Tensor, router_ws, out=None, stream=None) -> torch.Tensor:
    """A stack of MoeFp4Layer handles applied in order on one stream (see
    moe_fp4_forward_layers): x_{l+1} = layers[l](x_l, router_ws[l])."""
    lib = _lib.load()
    L = len(layers)
    if out is None:
        out = torch.empty_like(x)
    hs = (ctypes.c_void_p * L)(*[l._h.value for l in layers])
    rws = (ctypes.c_void_p * L)(*[r.data_ptr() for r in router_ws])
    T = x.shape[0] if x.dim() == 2 else 0
    _lib.check(lib.moe_fp4_forward_layers(hs, L, _ptr(x), T, rws, _ptr(out), _stream_ptr(stream)),
               "moe_fp4_forward_layers")
    return out
