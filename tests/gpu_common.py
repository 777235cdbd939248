"""Shared helpers of the GPU parity tests: seeded workloads, the CUDA layer, oracle checks."""
from __future__ import annotations

import functools
import os

import numpy as np

import synth

# Output tolerance of the layer (fp32 output against the fp64 oracle):
# relative L2 error <= 5e-3 and max |error| <= 2e-2 * RMS(output).
REL_L2 = 5e-3
MAX_ABS_RMS = 2e-2
ORACLE_THREADS = max(1, min(32, os.cpu_count() or 1))


@functools.lru_cache(maxsize=2)
def layer_weights(name: str, layer: int = 0):
    return synth.make_layer(synth.workload(name), layer)


def tokens(name: str, T=None, stream: int = 0):
    return synth.make_tokens(synth.workload(name), T, stream)


def make_layer(ds4, w, flags=0, max_tokens=None):
    return ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter,
                      max_tokens=max_tokens or w.tokens, flags=flags)


def to_dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()


def check_output(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = ""):
    y = y_gpu.astype(np.float64)
    err = y - y_ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300)
    rms = np.sqrt((y_ref ** 2).mean())
    mx = np.abs(err).max() / max(rms, 1e-300)
    assert rel <= REL_L2 and mx <= MAX_ABS_RMS, "%s: rel_l2=%.3e max_abs/rms=%.3e" % (what, rel, mx)
    return rel, mx


def check_permutation(ora, idx_ref, E, off, st, ss, inv):
    o_off, o_st, o_ss, o_inv = ora.permute(idx_ref, E)
    assert np.array_equal(off, o_off)
    assert np.array_equal(st, o_st)
    assert np.array_equal(ss, o_ss)
    assert np.array_equal(inv, o_inv)


def oracle_route_all(ora, x, lw, k, threads=ORACLE_THREADS):
    """Oracle routing of every token, split over threads (each call single-threaded)."""
    from concurrent.futures import ThreadPoolExecutor
    T = x.shape[0]
    cuts = np.linspace(0, T, min(threads, T) + 1).astype(int)
    parts = [None] * (len(cuts) - 1)

    def run(i):
        parts[i] = ora.route(x[cuts[i]:cuts[i + 1]], lw.router, lw.bias, k)

    with ThreadPoolExecutor(len(parts)) as ex:
        list(ex.map(run, range(len(parts))))
    idx = np.concatenate([p[0] for p in parts])
    w = np.concatenate([p[1] for p in parts])
    lg = np.concatenate([p[2] for p in parts])
    return idx, w, lg


def sample_tokens(T: int, n: int, seed: int, idx=None, E=None, n_heavy: int = 4, n_light: int = 4, cap=None):
    """A seeded sample of n tokens plus, when the routing is given, every token of the
    n_heavy heaviest and the n_light lightest non-empty experts (at most `cap` tokens of
    each of those experts when a cap is given, drawn with the same seed)."""
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=min(n, T), replace=False).tolist())
    if idx is not None:
        counts = np.bincount(idx.reshape(-1), minlength=E)
        nz = np.nonzero(counts)[0]
        order = nz[np.argsort(counts[nz], kind="stable")]
        for e in list(order[:n_light]) + list(order[::-1][:n_heavy]):
            toks = np.nonzero((idx == e).any(axis=1))[0]
            if cap is not None and len(toks) > cap:
                toks = rng.choice(toks, size=cap, replace=False)
            s.update(toks.tolist())
    return np.array(sorted(s), dtype=np.int64)
