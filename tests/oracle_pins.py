"""Pins of the fp64 oracle: checks against what the sources and mathematics fix.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when it is
wrong.  ``tests/test_oracle_pins.py`` runs them on the real oracle, and
``tests/test_oracle_mutants.py`` runs them on copies of the oracle with a
planted mistake, to show that each plausible mistake fails at least one pin.

What pins what:
* Q2_K dequantisation: three hand-worked blocks (tests/golden/q2k_blocks.txt).
* fp16/bf16 decoding and bf16 rounding: exact values and library conversions.
* softplus / score: closed forms (softplus(0) = ln 2, softplus(l) - softplus(-l)
  = l), and agreement with numpy's logaddexp and math.log1p.
* routing: invariants (k distinct experts, descending logits, weights sum to
  1, ties to the lower index on planted exact ties), k = 1 and k = E cases,
  and the logits against numpy's float64 dot of the exact bf16 values.
* permutation: numpy's stable argsort gives the same order; bijection.
* expert / shared / layer: numpy matmuls over the dequantised matrices,
  special cases (zero quants and mins give a zero routed output; zero shared
  weights leave only the routed part), and the brute-force dense evaluation.
"""
from __future__ import annotations

import math
import os
import re

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden_blocks():
    """Parse tests/golden/q2k_blocks.txt into [(name, bytes84, expected256)]."""
    out = []
    name = None
    blk = None
    exp = None
    for line in open(os.path.join(GOLDEN, "q2k_blocks.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("block "):
            if name is not None:
                out.append((name, blk, exp))
            name = line.split()[1]
            exp = np.zeros(256)
            blk = None
        elif line.startswith("bytes "):
            blk = bytes(int(v, 16) for v in line.split()[1:])
            assert len(blk) == 84
        elif line.startswith("value "):
            _, a, b, v = line.split()
            exp[int(a):int(b) + 1] = float(v)
    out.append((name, blk, exp))
    return out


# ----------------------------------------------------------------- formats

def pin_formats(o):
    assert o.bf16_to_double(0x3F80) == 1.0
    assert o.bf16_to_double(0xC040) == -3.0
    assert o.bf16_to_double(0x3E80) == 0.25
    assert o.f16_to_double(0x3C00) == 1.0
    assert o.f16_to_double(0x1800) == 2.0 ** -9
    assert o.f16_to_double(0x1C00) == 2.0 ** -8
    assert o.f16_to_double(0x0001) == 2.0 ** -24          # smallest subnormal
    assert o.f16_to_double(0xC500) == -5.0
    rng = np.random.default_rng(5)
    h = rng.integers(0, 0x7C00, 2000).astype(np.uint16)    # finite positive halves
    ref = h.view(np.float16).astype(np.float64)
    got = np.array([o.f16_to_double(int(v)) for v in h])
    assert np.array_equal(got, ref)
    b = rng.integers(0, 0x7F80, 2000).astype(np.uint32)
    refb = (b << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    gotb = np.array([o.bf16_to_double(int(v)) for v in b])
    assert np.array_equal(gotb, refb)
    # rounding to bf16: exact values, a tie to even, and above/below a tie
    assert o.double_to_bf16(1.0) == 0x3F80
    assert o.double_to_bf16(1.0 + 2 ** -8) == 0x3F80          # tie -> even (mantissa 0)
    assert o.double_to_bf16(1.0 + 3 * 2 ** -8) == 0x3F82      # tie -> even (mantissa 2)
    assert o.double_to_bf16(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert o.double_to_bf16(-2.5) == 0xC020


# ------------------------------------------------------------------- Q2_K

def pin_q2k_golden(o):
    for name, blk, exp in load_golden_blocks():
        got = o.dequant_block(blk)
        assert np.array_equal(got, exp), (name, np.nonzero(got != exp)[0][:8])


# ----------------------------------------------------------------- softplus

def pin_softplus(o):
    assert o.softplus(0.0) == math.log(2.0)
    for l in [0.5, 1.0, 3.0, 12.0, 40.0, 700.0]:
        assert abs((o.softplus(l) - o.softplus(-l)) - l) <= 4e-16 * max(1.0, l)
    for l in np.linspace(-700, 700, 4001):
        ref = np.logaddexp(0.0, l)
        assert abs(o.softplus(l) - ref) <= 4e-16 * max(ref, 1e-300) + 1e-320, l
    for l in [-12.0, -20.0, -50.0, -300.0]:
        ref = math.log1p(math.exp(l))
        assert abs(o.softplus(l) - ref) <= 2e-16 * ref
    for l in [-3.0, 0.0, 0.7, 5.0]:
        assert o.score(l) == math.sqrt(o.softplus(l))
    # the score is strictly increasing in the logit: needed for ranking by logit
    ls = np.linspace(-30, 30, 6001)
    s = np.array([o.score(l) for l in ls])
    assert np.all(np.diff(s) > 0)


# ----------------------------------------------------------------- routing

def _tiny_layer(E=8, H=256, I=256, Is=256, seed=7, bias=False):
    w = synth.Workload("pin", 4, H, E, 2, I, Is, 0.05, "normal" if bias else "none", 0.5, 0.0, (seed,), seed)
    return w, synth.make_layer(w)


def pin_route_invariants(o):
    for E, k, bias in [(8, 2, False), (8, 8, False), (8, 1, True), (16, 4, True), (256, 8, False)]:
        w, lw = _tiny_layer(E=E, bias=bias, seed=11 + E + k)
        x = synth.make_tokens(w, tokens=6)
        idx, wts, lg = o.route(x, lw.router, lw.bias, k)
        xr = synth.bf16_to_f32(x).astype(np.float64)
        wr = synth.bf16_to_f32(lw.router).astype(np.float64)
        ref_lg = xr @ wr.T + (0.0 if lw.bias is None else lw.bias.astype(np.float64))
        assert np.allclose(lg, ref_lg, rtol=0, atol=1e-12)
        for t in range(x.shape[0]):
            assert len(set(idx[t])) == k
            assert np.all(np.diff(lg[t, idx[t]]) <= 0)
            kth = lg[t, idx[t, -1]]
            others = np.setdiff1d(np.arange(E), idx[t])
            assert np.all(lg[t, others] <= kth)
            assert abs(wts[t].sum() - 1.0) <= 1e-12
            s = np.sqrt(np.logaddexp(0.0, lg[t, idx[t]]))
            assert np.allclose(wts[t], s / s.sum(), rtol=1e-13, atol=0)
            if k == 1:
                assert wts[t, 0] == 1.0
            if k == E:
                assert sorted(idx[t]) == list(range(E))


def pin_route_ties(o):
    # experts 1, 3 and 6 get identical router rows: their logits tie exactly, so the
    # lower index must come first and the selection must take the lower ones
    w, lw = _tiny_layer(E=8)
    wr = lw.router.copy()
    wr[1] = wr[3] = wr[6] = synth.bf16_bits(np.full(256, 0.25))
    x = synth.bf16_bits(np.full((1, 256), 1.0))             # logit 64 for the three, largest
    wr[[0, 2, 4, 5, 7]] = synth.bf16_bits(np.full((5, 256), -0.01))
    idx, wts, lg = o.route(x, wr, None, 2)
    assert list(idx[0]) == [1, 3]
    assert wts[0, 0] == wts[0, 1] == 0.5
    idx, _, _ = o.route(x, wr, None, 3)
    assert list(idx[0]) == [1, 3, 6]


def pin_permutation(o):
    rng = np.random.default_rng(3)
    for T, E, k in [(1, 8, 2), (5, 8, 3), (64, 256, 8), (33, 16, 16)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        off, st, ss, inv = o.permute(idx, E)
        flat = idx.reshape(-1)
        order = np.argsort(flat, kind="stable")              # by expert, then pair order
        assert np.array_equal(st, order // k)
        assert np.array_equal(ss, order % k)
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        assert np.array_equal(inv[order], np.arange(T * k))
        assert np.array_equal(idx[st, ss], np.repeat(np.arange(E), np.diff(off)))


# ------------------------------------------------------------------ experts

def _silu(g):
    return g / (1.0 + np.exp(-g))


def pin_expert_matmul(o):
    w, lw = _tiny_layer(E=2, H=512, I=256, Is=256, seed=21)
    x = synth.bf16_to_f32(synth.make_tokens(w, tokens=1))[0].astype(np.float64)
    for e in range(2):
        Wg = o.dequant_matrix(lw.gate[e]); Wu = o.dequant_matrix(lw.up[e]); Wd = o.dequant_matrix(lw.down[e])
        g, u, h, out = o.expert(lw.gate[e], lw.up[e], lw.down[e], x)
        assert np.allclose(g, Wg @ x, rtol=1e-12, atol=1e-12)
        assert np.allclose(u, Wu @ x, rtol=1e-12, atol=1e-12)
        assert np.allclose(h, _silu(Wg @ x) * (Wu @ x), rtol=1e-12, atol=1e-12)
        assert np.allclose(out, Wd @ (_silu(Wg @ x) * (Wu @ x)), rtol=1e-11, atol=1e-12)
    sg = synth.bf16_to_f32(lw.shared_gate).astype(np.float64)
    su = synth.bf16_to_f32(lw.shared_up).astype(np.float64)
    sd = synth.bf16_to_f32(lw.shared_down).astype(np.float64)
    h, s = o.shared(lw.shared_gate, lw.shared_up, lw.shared_down, x)
    assert np.allclose(h, _silu(sg @ x) * (su @ x), rtol=1e-12, atol=1e-14)
    assert np.allclose(s, sd @ h, rtol=1e-11, atol=1e-14)
    # silu closed forms
    assert abs(_silu(0.0)) == 0.0


def pin_layer_dense(o):
    cases = [(8, 2, 4, False), (4, 1, 3, False), (8, 4, 1, True), (4, 4, 3, True), (8, 2, 3, True)]
    for E, k, T, bias in cases:
        w, lw = _tiny_layer(E=E, bias=bias, seed=31 + E * k + T)
        x = synth.make_tokens(w, tokens=T)
        y, idx, wts = o.layer_forward(lw, x, k)
        yd = o.dense_forward(lw, x, k)
        scale = np.abs(yd).max()
        assert np.abs(y - yd).max() <= 1e-12 * scale, (E, k, T)


def pin_layer_special(o):
    w, lw = _tiny_layer(E=8, seed=41)
    x = synth.make_tokens(w, tokens=3)
    xd = synth.bf16_to_f32(x).astype(np.float64)
    # zero quants and zero mins: every routed weight is 0, so y is the shared output alone
    z = synth.LayerWeights(**{**lw.__dict__})
    for name in ("gate", "up", "down"):
        a = getattr(lw, name).copy()
        a[..., :80] = 0
        setattr(z, name, a)
    y, _, _ = o.layer_forward(z, x, 2)
    for t in range(3):
        _, s = o.shared(lw.shared_gate, lw.shared_up, lw.shared_down, xd[t])
        assert np.array_equal(y[t], s)
    # zero shared weights: y is the weighted routed sum
    z2 = synth.LayerWeights(**{**lw.__dict__})
    z2.shared_gate = np.zeros_like(lw.shared_gate)
    z2.shared_up = np.zeros_like(lw.shared_up)
    z2.shared_down = np.zeros_like(lw.shared_down)
    y2, idx, wts = o.layer_forward(z2, x, 2)
    for t in range(3):
        acc = np.zeros(w.hidden)
        for j in range(2):
            e = idx[t, j]
            acc += wts[t, j] * o.expert(lw.gate[e], lw.up[e], lw.down[e], xd[t])[3]
        assert np.allclose(y2[t], acc, rtol=1e-13, atol=1e-15)


def pin_rms_renorm(o):
    rng = np.random.default_rng(9)
    y = rng.normal(0, 3.0, (5, 512))
    x = o.rms_renorm(y)
    ref = y / np.sqrt((y ** 2).mean(axis=1, keepdims=True) + 1e-6)
    got = synth.bf16_to_f32(x).astype(np.float64)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8)      # half an ulp of 8 significant bits
    # exact case: y = 2 everywhere -> 2 / sqrt(4 + 1e-6) rounds to bf16 1.0
    x1 = o.rms_renorm(np.full((1, 256), 2.0))
    assert np.all(x1 == 0x3F80)


ALL_PINS = [pin_formats, pin_q2k_golden, pin_softplus, pin_route_invariants, pin_route_ties,
            pin_permutation, pin_expert_matmul, pin_layer_dense, pin_layer_special, pin_rms_renorm]
