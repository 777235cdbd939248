"""Seeded synthetic workloads for the routed Q2_K mixture-of-experts layer.

This module is shared by the fp64 oracle (``oracle/``) and the CUDA path: it
draws every input both sides consume, and it holds none of the layer's own
arithmetic (no routing, no dequantisation, no projection).  What it does:

* a counter-based 64-bit generator: the SplitMix64 output function (Steele,
  Lea and Flood, "Fast splittable pseudorandom number generators", OOPSLA
  2014) applied to ``key + (counter + 1) * 0x9E3779B97F4A7C15``, so any slice
  of any tensor can be drawn on its own, in any order, with the same result;
* uniform doubles from the top 53 bits; normals by Box-Muller (one cosine
  branch per pair of uniforms);
* round-to-nearest-even narrowing to bf16 (through fp32) and to fp16;
* random Q2_K super-blocks in the GGUF byte order: 16 scale bytes (low nibble
  = scale, high nibble = min), 64 bytes of 2-bit quants, then fp16 ``d`` and
  fp16 ``dmin`` (little-endian), 84 bytes per 256 weights.  Scale and min
  nibbles and the quants are uniform; ``d`` and ``dmin`` are U(1e-3, 4e-3).

The workloads (``WORKLOADS``) follow the layer shapes of the routed-MoE FFN of
DeepSeek-V4-style models run by the DwarfStar (ds4) engine: "antirez/ds4"
README (molayo1419.me translation), section on the 2-bit quantisation mix,
which quantises only the routed experts and keeps the shared expert, the
projections and the router unquantised.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "LayerWeights",
    "bits64", "uniform01", "normal", "bf16_bits", "f16_bits",
    "q2k_blocks", "make_layer", "make_tokens", "tensor_key", "Q2K_BLOCK_BYTES",
]

Q2K_BLOCK_BYTES = 84
Q2K_BLOCK_WEIGHTS = 256

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK_BLOCKS = 1 << 20


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def _mix_scalar(v: int) -> int:
    return int(_mix64(np.array([v & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0])


_TAGS = {
    "gate": 1, "up": 2, "down": 3, "router": 4, "bias": 5,
    "shared_gate": 6, "shared_up": 7, "shared_down": 8, "x": 9, "zipf_rank": 10,
}


def tensor_key(seed: int, tag: str, stream: int = 0) -> int:
    """64-bit key of one tensor: mixes the seed, the tensor's tag and a stream index."""
    k = _mix_scalar(seed * 0x9E3779B97F4A7C15 + 0x632BE59BD9B4E019)
    k = _mix_scalar(k ^ (_TAGS[tag] * 0xD1B54A32D192ED03))
    return _mix_scalar(k ^ (stream * 0xA0761D6478BD642F + 0x8EBC6AF09C88C6E3))


def bits64(key: int, start: int, n: int) -> np.ndarray:
    """Counter-based draws: element i is SplitMix64(key + (start + i + 1) * gamma)."""
    ctr = np.arange(start + 1, start + 1 + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + ctr * _GAMMA
    return _mix64(z)


def uniform01(key: int, start: int, n: int) -> np.ndarray:
    """Uniform doubles in [0, 1) from the top 53 bits of each draw."""
    return (bits64(key, start, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(key: int, n: int, sigma: float = 1.0, start: int = 0) -> np.ndarray:
    """N(0, sigma) doubles by Box-Muller: normal i uses draws 2(start+i) and 2(start+i)+1."""
    u = uniform01(key, 2 * start, 2 * n).reshape(n, 2)
    r = np.sqrt(-2.0 * np.log1p(-u[:, 0]))          # 1 - u in (0, 1]
    return sigma * r * np.cos(2.0 * math.pi * u[:, 1])


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of doubles: RNE to fp32, then RNE to bf16 (finite inputs)."""
    f = np.ascontiguousarray(a, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def f16_bits(a: np.ndarray) -> np.ndarray:
    """IEEE fp16 bit patterns of doubles, round to nearest even."""
    return np.ascontiguousarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


def q2k_blocks(key: int, first_block: int, n_blocks: int, out: Optional[np.ndarray] = None) -> np.ndarray:
    """Random Q2_K super-blocks ``[n_blocks, 84]`` uint8; block b draws counters 12b .. 12b+11.

    Draws 0..9 give the 80 bytes of scales (16) and quants (64); draw 10 gives d and
    draw 11 gives dmin, both U(1e-3, 4e-3) rounded to fp16.
    """
    if out is None:
        out = np.empty((n_blocks, Q2K_BLOCK_BYTES), dtype=np.uint8)
    raw = bits64(key, 12 * first_block, 12 * n_blocks).reshape(n_blocks, 12)
    out[:, :80] = raw[:, :10].copy().view(np.uint8).reshape(n_blocks, 80)
    u = (raw[:, 10:12] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    dm = f16_bits(1e-3 + 3e-3 * u)                       # [n, 2] fp16 bits: d, dmin
    out[:, 80:84] = dm.copy().view(np.uint8).reshape(n_blocks, 4)
    return out


def _workers() -> int:
    import os
    return max(1, min(16, os.cpu_count() or 1))


def _q2k_tensor(key: int, n_blocks: int) -> np.ndarray:
    """Chunks are independent (counter-based draws), so they are filled by a thread pool;
    numpy releases the GIL inside the array operations."""
    from concurrent.futures import ThreadPoolExecutor
    out = np.empty((n_blocks, Q2K_BLOCK_BYTES), dtype=np.uint8)
    starts = list(range(0, n_blocks, _CHUNK_BLOCKS))

    def fill(b0):
        nb = min(_CHUNK_BLOCKS, n_blocks - b0)
        q2k_blocks(key, b0, nb, out[b0:b0 + nb])

    if len(starts) == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_workers()) as ex:
            list(ex.map(fill, starts))
    return out


def _normal_bf16(key: int, n: int, sigma: float) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    step = 1 << 22
    for s in range(0, n, step):
        m = min(step, n - s)
        out[s:s + m] = bf16_bits(normal(key, m, sigma, start=s))
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and value distributions of one synthetic routed-MoE workload."""
    name: str
    tokens: int           # T
    hidden: int           # H
    n_experts: int        # E
    top_k: int            # k
    inter: int            # I (routed expert intermediate)
    shared_inter: int     # I_s (0 = no shared expert)
    router_sigma: float   # Wr ~ N(0, router_sigma), bf16
    bias: str             # "none" | "normal" (N(0, bias_sigma)) | "zipf" (-s ln rank)
    bias_sigma: float
    zipf_s: float
    layer_seeds: tuple    # one seed per chained layer
    token_seed: int
    shared_sigma: float = 0.02
    description: str = ""

    @property
    def layers(self) -> int:
        return len(self.layer_seeds)

    def q2k_bytes_per_matrix(self) -> int:
        return self.inter * self.hidden // Q2K_BLOCK_WEIGHTS * Q2K_BLOCK_BYTES


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_t4_h256_e8_k2", 4, 256, 8, 2, 256, 256, 0.05, "none", 0.0, 0.0, (0,), 0,
                 description="tiny layer: 4 tokens, H=256, 8 experts, top-2, I=256, shared I=256"),
        Workload("decode_t1_h4096_e256_k8", 1, 4096, 256, 8, 2048, 2048, 0.02, "none", 0.0, 0.0, (1,), 1,
                 description="single-token decode: H=4096, 256 experts, top-8, I=2048, shared I=2048"),
        Workload("decode_t16_h4096_e256_k8", 16, 4096, 256, 8, 2048, 2048, 0.02, "none", 0.0, 0.0, (1,), 2,
                 description="16-session micro-batched decode, same layer as the single-token decode"),
        Workload("prefill_t2048_h4096_e256_k8_bias", 2048, 4096, 256, 8, 2048, 2048, 0.02, "normal", 0.5, 0.0,
                 (3,), 3, description="2048-token prefill chunk, per-expert logit bias N(0, 0.5)"),
        Workload("prefill4_t8192_h7168_e256_k8_zipf", 8192, 7168, 256, 8, 2048, 2048, 0.02, "zipf", 0.0, 1.1,
                 (40, 41, 42, 43), 4,
                 description="4 chained layers, 8192 tokens, H=7168, Zipf(1.1)-shaped logit bias, "
                             "RMS renormalisation between layers"),
    ]
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


@dataclasses.dataclass
class LayerWeights:
    """Host-side weights of one layer, in the layouts the C ABI loads.

    gate/up: uint8 [E, I, H/256, 84]; down: uint8 [E, H, I/256, 84] (Q2_K, AoS blocks,
    each row contiguous along its input dimension); router: uint16 bf16 bits [E, H];
    bias: float32 [E] or None; shared_gate/shared_up: uint16 [I_s, H];
    shared_down: uint16 [H, I_s] (row-major bf16 bits).
    """
    gate: np.ndarray
    up: np.ndarray
    down: np.ndarray
    router: np.ndarray
    bias: Optional[np.ndarray]
    shared_gate: Optional[np.ndarray]
    shared_up: Optional[np.ndarray]
    shared_down: Optional[np.ndarray]


def make_bias(w: Workload, seed: int) -> Optional[np.ndarray]:
    E = w.n_experts
    if w.bias == "none":
        return None
    if w.bias == "normal":
        return normal(tensor_key(seed, "bias"), E, w.bias_sigma).astype(np.float32)
    if w.bias == "zipf":
        # rank_e = 1 + a seeded random permutation of 0..E-1; bias = -s * ln(rank_e)
        u = uniform01(tensor_key(seed, "zipf_rank"), 0, E)
        rank = np.empty(E, dtype=np.int64)
        rank[np.argsort(u, kind="stable")] = np.arange(1, E + 1)
        return (-w.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32)
    raise ValueError(w.bias)


def make_layer(w: Workload, layer: int = 0, experts: Optional[int] = None) -> LayerWeights:
    """Draw the weights of layer ``layer`` of workload ``w`` (all experts unless ``experts``)."""
    seed = w.layer_seeds[layer]
    E = w.n_experts if experts is None else experts
    H, I, Is = w.hidden, w.inter, w.shared_inter
    gate = _q2k_tensor(tensor_key(seed, "gate"), E * I * H // 256).reshape(E, I, H // 256, 84)
    up = _q2k_tensor(tensor_key(seed, "up"), E * I * H // 256).reshape(E, I, H // 256, 84)
    down = _q2k_tensor(tensor_key(seed, "down"), E * H * I // 256).reshape(E, H, I // 256, 84)
    router = _normal_bf16(tensor_key(seed, "router"), w.n_experts * H, w.router_sigma).reshape(w.n_experts, H)
    bias = make_bias(w, seed)
    if Is > 0:
        sg = _normal_bf16(tensor_key(seed, "shared_gate"), Is * H, w.shared_sigma).reshape(Is, H)
        su = _normal_bf16(tensor_key(seed, "shared_up"), Is * H, w.shared_sigma).reshape(Is, H)
        sd = _normal_bf16(tensor_key(seed, "shared_down"), H * Is, w.shared_sigma).reshape(H, Is)
    else:
        sg = su = sd = None
    return LayerWeights(gate, up, down, router, bias, sg, su, sd)


def make_tokens(w: Workload, tokens: Optional[int] = None, stream: int = 0) -> np.ndarray:
    """Token activations x: uint16 bf16 bits [T, H], N(0, 1); ``stream`` selects an independent batch."""
    T = w.tokens if tokens is None else tokens
    return _normal_bf16(tensor_key(w.token_seed, "x", stream), T * w.hidden, 1.0).reshape(T, w.hidden)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact); a format conversion, used by tests for display."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
