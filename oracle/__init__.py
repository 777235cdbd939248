"""fp64 oracle of the routed Q2_K mixture-of-experts FFN layer (TEST INFRASTRUCTURE).

A ctypes wrapper over ``ds4moe_oracle.c``: a plain, slow, single-threaded C99
restatement of the layer in double precision.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library under ``bit_quantized_routed_sqrt_b200/`` never does, and the
two share no code.

Every function names the passage it follows in the C source's header; the
readings taken where the sources are silent are listed there too.

Parity pinning: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (hand-worked golden blocks, closed forms,
invariants, special cases and a brute-force dense evaluation), except that the
Q2_K byte layout itself is a reading (GGUF order) that no file in this
repository can confirm against the real model files: that one point is
"parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ds4moe_oracle.c")
_LIB = os.path.join(_HERE, "libds4moe_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (no CUDA); returns the .so path."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


class OraLayer(C.Structure):
    _fields_ = [
        ("hidden", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int),
        ("inter", C.c_int), ("shared_inter", C.c_int),
        ("gate", C.c_void_p), ("up", C.c_void_p), ("down", C.c_void_p),
        ("router", C.c_void_p), ("bias", C.c_void_p),
        ("sg", C.c_void_p), ("su", C.c_void_p), ("sd", C.c_void_p),
    ]


def _declare(lib):
    vp, i, d = C.c_void_p, C.c_int, C.c_double
    lib.ora_bf16_to_double.argtypes = [C.c_uint16]; lib.ora_bf16_to_double.restype = d
    lib.ora_f16_to_double.argtypes = [C.c_uint16]; lib.ora_f16_to_double.restype = d
    lib.ora_double_to_bf16.argtypes = [d]; lib.ora_double_to_bf16.restype = C.c_uint16
    lib.ora_q2k_dequant.argtypes = [vp, vp]; lib.ora_q2k_dequant.restype = None
    lib.ora_softplus.argtypes = [d]; lib.ora_softplus.restype = d
    lib.ora_score.argtypes = [d]; lib.ora_score.restype = d
    lib.ora_logit.argtypes = [vp, vp, i, vp]; lib.ora_logit.restype = d
    lib.ora_route.argtypes = [vp, i, i, vp, vp, i, i, vp, vp, vp]; lib.ora_route.restype = None
    lib.ora_permute.argtypes = [vp, i, i, i, vp, vp, vp, vp]; lib.ora_permute.restype = None
    lib.ora_expert.argtypes = [vp, vp, vp, i, i, vp, vp, vp, vp, vp]; lib.ora_expert.restype = None
    lib.ora_shared.argtypes = [vp, vp, vp, i, i, vp, vp, vp]; lib.ora_shared.restype = None
    lib.ora_layer_forward.argtypes = [C.POINTER(OraLayer), vp, i, vp, i, vp, vp, vp]
    lib.ora_layer_forward.restype = None
    lib.ora_dense_forward.argtypes = [C.POINTER(OraLayer), vp, i, vp]; lib.ora_dense_forward.restype = i
    lib.ora_rms_renorm.argtypes = [vp, i, i, vp]; lib.ora_rms_renorm.restype = None


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library; ``path`` loads another build (mutants)."""
    global _lib
    if path is not None:
        lib = C.CDLL(path)
        _declare(lib)
        return lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            _declare(lib)
            _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """Handle over one build of the oracle library (the default build unless ``lib`` is given)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    # --- formats -------------------------------------------------------------
    def bf16_to_double(self, b: int) -> float:
        return self.lib.ora_bf16_to_double(int(b))

    def f16_to_double(self, h: int) -> float:
        return self.lib.ora_f16_to_double(int(h))

    def double_to_bf16(self, v: float) -> int:
        return int(self.lib.ora_double_to_bf16(float(v)))

    # --- Q2_K ----------------------------------------------------------------
    def dequant_block(self, blk) -> np.ndarray:
        b = np.ascontiguousarray(np.frombuffer(bytes(blk), dtype=np.uint8) if isinstance(blk, (bytes, bytearray))
                                 else blk, dtype=np.uint8)
        assert b.size == 84
        out = np.empty(256, dtype=np.float64)
        self.lib.ora_q2k_dequant(_p(b), _p(out))
        return out

    def dequant_matrix(self, q: np.ndarray) -> np.ndarray:
        """Dequantise a [rows, K/256, 84] Q2_K matrix to a dense fp64 [rows, K] array."""
        q = np.ascontiguousarray(q, dtype=np.uint8)
        rows, nb = q.shape[0], q.shape[1]
        out = np.empty((rows, nb * 256), dtype=np.float64)
        for r in range(rows):
            for b in range(nb):
                o = out[r, b * 256:(b + 1) * 256]
                self.lib.ora_q2k_dequant(_p(q[r, b]), o.ctypes.data_as(C.c_void_p))
        return out

    # --- router --------------------------------------------------------------
    def softplus(self, l: float) -> float:
        return self.lib.ora_softplus(float(l))

    def score(self, l: float) -> float:
        return self.lib.ora_score(float(l))

    def route(self, x: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray], k: int):
        """Returns (idx int32 [T,k], weights fp64 [T,k], logits fp64 [T,E])."""
        x = _c(x, np.uint16); wr = _c(wr, np.uint16); bias = _c(bias, np.float32)
        T, H = x.shape
        E = wr.shape[0]
        assert 1 <= k <= min(E, 64)
        idx = np.empty((T, k), dtype=np.int32)
        w = np.empty((T, k), dtype=np.float64)
        lg = np.empty((T, E), dtype=np.float64)
        self.lib.ora_route(_p(x), T, H, _p(wr), _p(bias), E, k, _p(idx), _p(w), _p(lg))
        return idx, w, lg

    def permute(self, idx: np.ndarray, E: int):
        """Returns (offsets [E+1], sorted_token [T*k], sorted_slot [T*k], inv_pos [T*k]), int32."""
        idx = _c(idx, np.int32)
        T, k = idx.shape
        off = np.empty(E + 1, dtype=np.int32)
        st = np.empty(T * k, dtype=np.int32)
        ss = np.empty(T * k, dtype=np.int32)
        inv = np.empty(T * k, dtype=np.int32)
        self.lib.ora_permute(_p(idx), T, k, E, _p(off), _p(st), _p(ss), _p(inv))
        return off, st, ss, inv

    # --- experts -------------------------------------------------------------
    def expert(self, gate_e, up_e, down_e, x: np.ndarray):
        """One routed expert on one fp64 token vector; returns (g, u, h, o)."""
        gate_e = _c(gate_e, np.uint8); up_e = _c(up_e, np.uint8); down_e = _c(down_e, np.uint8)
        I, nbh = gate_e.shape[0], gate_e.shape[1]
        H = nbh * 256
        x = _c(x, np.float64)
        g = np.empty(I); u = np.empty(I); h = np.empty(I); o = np.empty(H)
        self.lib.ora_expert(_p(gate_e), _p(up_e), _p(down_e), H, I, _p(x), _p(g), _p(u), _p(h), _p(o))
        return g, u, h, o

    def shared(self, sg, su, sd, x: np.ndarray):
        """Shared bf16 expert on one fp64 token vector; returns (h, S)."""
        sg = _c(sg, np.uint16); su = _c(su, np.uint16); sd = _c(sd, np.uint16)
        Is, H = sg.shape
        x = _c(x, np.float64)
        h = np.empty(Is); s = np.empty(H)
        self.lib.ora_shared(_p(sg), _p(su), _p(sd), H, Is, _p(x), _p(h), _p(s))
        return h, s

    # --- layer ---------------------------------------------------------------
    def _layer(self, lw, k: int):
        gate = _c(lw.gate, np.uint8); up = _c(lw.up, np.uint8); down = _c(lw.down, np.uint8)
        router = _c(lw.router, np.uint16); bias = _c(lw.bias, np.float32)
        sg = _c(lw.shared_gate, np.uint16); su = _c(lw.shared_up, np.uint16); sd = _c(lw.shared_down, np.uint16)
        E, I, nbh = gate.shape[0], gate.shape[1], gate.shape[2]
        H = nbh * 256
        Is = 0 if sg is None else sg.shape[0]
        assert 1 <= k <= min(E, 64)
        L = OraLayer(H, E, k, I, Is, _p(gate), _p(up), _p(down), _p(router), _p(bias), _p(sg), _p(su), _p(sd))
        keep = (gate, up, down, router, bias, sg, su, sd)
        return L, keep, H

    def layer_forward(self, lw, x: np.ndarray, k: int, tokens: Optional[Sequence[int]] = None,
                      threads: int = 1):
        """Layer output y fp64 [n, H] for the listed tokens (all when None), with their routing.

        ``threads`` > 1 runs disjoint token subsets concurrently in separate calls of the
        same single-threaded routine (ctypes releases the GIL); the arithmetic is unchanged.
        """
        L, keep, H = self._layer(lw, k)
        x = _c(x, np.uint16)
        T = x.shape[0]
        tok = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, dtype=np.int32)
        n = tok.size
        y = np.empty((n, H), dtype=np.float64)
        idx = np.empty((n, k), dtype=np.int32)
        w = np.empty((n, k), dtype=np.float64)

        def run(lo, hi):
            if hi <= lo:
                return
            t = np.ascontiguousarray(tok[lo:hi])
            yy = np.empty((hi - lo, H)); ii = np.empty((hi - lo, k), dtype=np.int32); ww = np.empty((hi - lo, k))
            self.lib.ora_layer_forward(C.byref(L), _p(x), T, _p(t), hi - lo, _p(yy), _p(ii), _p(ww))
            y[lo:hi] = yy; idx[lo:hi] = ii; w[lo:hi] = ww

        if threads <= 1 or n <= 1:
            run(0, n)
        else:
            cuts = np.linspace(0, n, min(threads, n) + 1).astype(int)
            with ThreadPoolExecutor(len(cuts) - 1) as ex:
                list(ex.map(lambda i: run(cuts[i], cuts[i + 1]), range(len(cuts) - 1)))
        del keep
        return y, idx, w

    def dense_forward(self, lw, x: np.ndarray, k: int) -> np.ndarray:
        """Brute-force all-experts masked evaluation (tiny shapes only)."""
        L, keep, H = self._layer(lw, k)
        x = _c(x, np.uint16)
        T = x.shape[0]
        y = np.empty((T, H), dtype=np.float64)
        rc = self.lib.ora_dense_forward(C.byref(L), _p(x), T, _p(y))
        assert rc == 0, "out of memory in the dense evaluation"
        del keep
        return y

    def rms_renorm(self, y: np.ndarray) -> np.ndarray:
        y = _c(y, np.float64)
        T, H = y.shape
        out = np.empty((T, H), dtype=np.uint16)
        self.lib.ora_rms_renorm(_p(y), T, H, _p(out))
        return out


_default = None


def oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
