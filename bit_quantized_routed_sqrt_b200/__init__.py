"""Thin ctypes binding of ``libds4moe.so``: the routed Q2_K mixture-of-experts layer.

Every function mirrors one ``extern "C"`` entry point of ``include/ds4moe.h`` under
the same name and only marshals arguments (torch tensors become device pointers,
torch's current stream becomes the ``cuda_stream`` argument).  All arithmetic runs
in the library's CUDA kernels; there is no fallback: importing this package fails
if the library has not been built, and every call raises on a non-OK status.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libds4moe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "ds4moe.h")

FLAG_FORCE_DECODE = 0x1
FLAG_FORCE_PREFILL = 0x2
FLAG_PROFILE = 0x4
FLAG_TRACE = 0x8
FLAG_TEST_TIMEOUT = 0x10
ROUTE_STATIC_MAX_TOKENS = 256

STATUS = {0: "DS4MOE_OK", 1: "DS4MOE_EINVAL", 2: "DS4MOE_ENOMEM", 3: "DS4MOE_ECUDA",
          4: "DS4MOE_ESTATE", 5: "DS4MOE_ETIMEOUT", 6: "DS4MOE_EDEVICE"}

if not os.path.exists(LIB_PATH):
    raise ImportError("libds4moe.so is not built (run __graft_entry__.build()); "
                      "this package has no CPU fallback")


class ds4moe_config(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("inter", C.c_int32), ("shared_inter", C.c_int32), ("max_tokens", C.c_int32),
                ("flags", C.c_uint32)]


class ds4moe_stats(C.Structure):
    _fields_ = [("router_fallback_tokens", C.c_int64), ("last_path", C.c_int32),
                ("last_tokens", C.c_int32), ("n_stages", C.c_int32), ("stage_ms", C.c_float * 8)]


lib = C.CDLL(LIB_PATH)
_vp, _i32 = C.c_void_p, C.c_int32
lib.ds4moe_create.argtypes = [C.POINTER(ds4moe_config), C.c_int, C.POINTER(_vp)]
lib.ds4moe_destroy.argtypes = [_vp]
lib.ds4moe_destroy.restype = None
lib.ds4moe_load_q2k_experts.argtypes = [_vp] * 10
lib.ds4moe_route.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.ds4moe_route_static.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.ds4moe_forward.argtypes = [_vp, _vp, _i32, _vp, _vp]
lib.ds4moe_forward_host.argtypes = [_vp, _vp, _i32, _vp, _vp]
lib.ds4moe_rms_renorm.argtypes = [_vp, _i32, _i32, _vp, _vp]
lib.ds4moe_score_eval.argtypes = [_vp, _i32, _vp, _i32, _vp]
lib.ds4moe_export_q2k.argtypes = [_vp, _i32, _i32, _vp]
lib.ds4moe_sync_status.argtypes = [_vp]
lib.ds4moe_get_stats.argtypes = [_vp, C.POINTER(ds4moe_stats)]
lib.ds4moe_get_trace.argtypes = [_vp, _vp, _i32, C.POINTER(_i32), _vp]
lib.ds4moe_status_string.argtypes = [C.c_int]
lib.ds4moe_status_string.restype = C.c_char_p
lib.ds4moe_last_error.argtypes = [_vp]
lib.ds4moe_last_error.restype = C.c_char_p
for _n in ("ds4moe_create", "ds4moe_load_q2k_experts", "ds4moe_route", "ds4moe_route_static", "ds4moe_forward", "ds4moe_forward_host",
           "ds4moe_rms_renorm", "ds4moe_score_eval", "ds4moe_export_q2k", "ds4moe_sync_status", "ds4moe_get_stats",
           "ds4moe_get_trace"):
    getattr(lib, _n).restype = C.c_int


class Ds4MoeError(RuntimeError):
    pass


def _check(rc: int, handle=None, what: str = ""):
    if rc != 0:
        detail = lib.ds4moe_last_error(handle).decode() if handle else ""
        raise Ds4MoeError("%s failed: %s (%s) %s" % (what, STATUS.get(rc, rc),
                                                   lib.ds4moe_status_string(rc).decode(), detail))


def _ptr(t) -> Optional[int]:
    """Device/host address of a torch tensor or numpy array (None stays None)."""
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return int(stream)
    import torch
    return torch.cuda.current_stream().cuda_stream


def ds4moe_status_string(status: int) -> str:
    return lib.ds4moe_status_string(status).decode()


def ds4moe_rms_renorm(y, T: int, H: int, x_out, stream=None):
    _check(lib.ds4moe_rms_renorm(_ptr(y), T, H, _ptr(x_out), _stream(stream)), None, "ds4moe_rms_renorm")


def ds4moe_score_eval(logits, n: int, scores, variant: int = 0, stream=None):
    _check(lib.ds4moe_score_eval(_ptr(logits), n, _ptr(scores), variant, _stream(stream)), None, "ds4moe_score_eval")


class Ds4Moe:
    """One layer on one device (the ``ds4moe`` handle)."""

    def __init__(self, hidden: int, n_experts: int, top_k: int, inter: int, shared_inter: int,
                 max_tokens: int, flags: int = 0, device: int = 0):
        self.cfg = ds4moe_config(hidden, n_experts, top_k, inter, shared_inter, max_tokens, flags)
        self.hidden, self.n_experts, self.top_k = hidden, n_experts, top_k
        self.inter, self.shared_inter, self.max_tokens = inter, shared_inter, max_tokens
        self.device = device
        h = _vp()
        _check(lib.ds4moe_create(C.byref(self.cfg), device, C.byref(h)), None, "ds4moe_create")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            lib.ds4moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- calls with the C names -------------------------------------------------
    def ds4moe_load_q2k_experts(self, gate, up, down, router, bias=None, shared_gate=None, shared_up=None,
                                shared_down=None, stream=None):
        """Host arrays (numpy) in the layouts of include/ds4moe.h."""
        import numpy as np
        keep = [np.ascontiguousarray(a) if a is not None else None
                for a in (gate, up, down, router, bias, shared_gate, shared_up, shared_down)]
        _check(lib.ds4moe_load_q2k_experts(self.h, *[_ptr(a) for a in keep], _stream(stream)), self.h,
               "ds4moe_load_q2k_experts")

    def load(self, lw, stream=None):
        """Load a ``synth.LayerWeights``-like object (fields gate, up, down, router, bias, shared_*)."""
        self.ds4moe_load_q2k_experts(lw.gate, lw.up, lw.down, lw.router, lw.bias, lw.shared_gate, lw.shared_up,
                                     lw.shared_down, stream)

    def ds4moe_route(self, x, T, topk_idx, topk_w, offsets=None, sorted_token=None, sorted_slot=None,
                     inv_pos=None, stream=None):
        _check(lib.ds4moe_route(self.h, _ptr(x), T, _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
                                _ptr(sorted_token), _ptr(sorted_slot), _ptr(inv_pos), _stream(stream)),
               self.h, "ds4moe_route")

    def ds4moe_route_static(self, x, T, topk_idx, topk_w, offsets, sorted_token, sorted_slot, inv_pos,
                            stream=None):
        _check(lib.ds4moe_route_static(self.h, _ptr(x), T, _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
                                       _ptr(sorted_token), _ptr(sorted_slot), _ptr(inv_pos), _stream(stream)),
               self.h, "ds4moe_route_static")

    def ds4moe_forward(self, x, T, y, stream=None):
        _check(lib.ds4moe_forward(self.h, _ptr(x), T, _ptr(y), _stream(stream)), self.h, "ds4moe_forward")

    def ds4moe_forward_host(self, x_host, T, y_host, stream=None):
        _check(lib.ds4moe_forward_host(self.h, _ptr(x_host), T, _ptr(y_host), _stream(stream)), self.h,
               "ds4moe_forward_host")

    def ds4moe_export_q2k(self, which: int, expert: int, out):
        _check(lib.ds4moe_export_q2k(self.h, which, expert, _ptr(out)), self.h, "ds4moe_export_q2k")

    def ds4moe_sync_status(self):
        _check(lib.ds4moe_sync_status(self.h), self.h, "ds4moe_sync_status")

    def ds4moe_get_stats(self) -> ds4moe_stats:
        s = ds4moe_stats()
        _check(lib.ds4moe_get_stats(self.h, C.byref(s)), self.h, "ds4moe_get_stats")
        return s

    def ds4moe_get_trace(self, max_records: int = 1 << 20):
        """Returns (records int64 [n, 4], unit_bounds int32 [7]) of the last batched-GEMV launch
        (record layout in include/ds4moe.h)."""
        import numpy as np
        out = np.zeros((max_records, 4), dtype=np.int64)
        n = C.c_int32()
        bounds = np.zeros(7, dtype=np.int32)
        _check(lib.ds4moe_get_trace(self.h, out.ctypes.data, max_records, C.byref(n), bounds.ctypes.data), self.h,
               "ds4moe_get_trace")
        return out[:n.value], bounds

    # -- torch conveniences (marshalling only) -----------------------------------
    def route(self, x):
        import torch
        T = x.shape[0]
        k = self.top_k
        dev = x.device
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        off = torch.empty(self.n_experts + 1, dtype=torch.int32, device=dev)
        st = torch.empty(T * k, dtype=torch.int32, device=dev)
        ss = torch.empty(T * k, dtype=torch.int32, device=dev)
        inv = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.ds4moe_route(x, T, idx, w, off, st, ss, inv)
        return idx, w, off, st, ss, inv

    def forward(self, x, y=None):
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.hidden), dtype=torch.float32, device=x.device)
        self.ds4moe_forward(x, T, y)
        return y


def exported_symbols():
    """Names of the ``ds4moe_*`` functions declared in include/ds4moe.h."""
    import re
    src = open(HEADER).read()
    return sorted(set(re.findall(r"\b(ds4moe_[a-z_0-9]+)\s*\(", src)))
