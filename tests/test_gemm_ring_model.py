"""CPU model of the grouped GEMM's barrier protocol (pf_gemm_kernel in csrc/prefill.cuh).

The kernel's roles synchronise through mbarriers waited on by parity.  A parity wait only
tells two consecutive phases apart, so a role that skipped a phase could pass a wait one
phase early and touch a stage still in use.  This model replays the roles' waits and
arrivals, in the kernel's order, under random interleavings, with the ring depths read from
the kernel source.  It checks that
  * every wait that passes does so on the phase it was meant for (no aliasing),
  * no stage is refilled while the MMAs still read it, and no MMA reads a stage before all
    of its data has landed,
  * every interleaving runs to the end (no deadlock).
A mutant of the protocol (a role that skips a wait) must fail the same checks.

The model mirrors these waits and arrivals of the kernel, per 64-wide K step `it`:
  producer  raw column every 4 quantised steps: wait raw_empty, expect_tx raw_full, copies;
            wait empty[s], expect_tx full_b[s], activation TMA
  loader    wait empty[s]; dense step: expect_tx full_at[s], weight TMA;
            wait full_b[s]; dense step: wait full_at[s]; arrive full[s]
  dequant   (8 warps) quantised step: wait raw_full at a column start; wait empty[s];
            write the weight stage; arrive full[s]; arrive raw_empty after a column
  MMA       per tile: wait acc_empty; per step: wait full[s], MMAs, commit empty[s];
            per tile: commit acc_full
  epilogue  (4 warps) per tile: wait acc_full, arrive acc_empty
"""
import os
import random
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PREFILL = os.path.join(ROOT, "bit_quantized_routed_sqrt_b200", "csrc", "prefill.cuh")
DEQUANT_WARPS, EPILOGUE_WARPS = 8, 4


def kernel_rings():
    """(STAGES of GEMM1, STAGES of GEMM2, RAWS) as the kernel source declares them."""
    src = open(PREFILL).read()
    m = re.search(r"static constexpr int STAGES = G == 1 \? (\d+) : (\d+);", src)
    r = re.search(r"static constexpr int RAWS = (\d+);", src)
    assert m and r, "ring depths not found in prefill.cuh"
    return int(m.group(1)), int(m.group(2)), int(r.group(1))


class Bar:
    """An mbarrier: `count` arrivals plus the expected transaction bytes complete a phase."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, ("too many arrivals", self.name)
        self._check()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0, ("bytes beyond expect_tx", self.name)
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passes(self, parity):
        # try_wait.parity(P) succeeds once the phase with parity P has completed
        return (self.phase & 1) != parity


def run(tiles, stages, raws, nmat, seed, mutant=None):
    rnd = random.Random(seed)
    S, R = stages, raws
    full = [Bar("full%d" % i, DEQUANT_WARPS + 1) for i in range(S)]
    empty = [Bar("empty%d" % i, 1) for i in range(S)]
    full_b = [Bar("full_b%d" % i, 1) for i in range(S)]
    full_at = [Bar("full_at%d" % i, 1) for i in range(S)]
    raw_full = [Bar("raw_full%d" % i, 1) for i in range(R)]
    raw_empty = [Bar("raw_empty%d" % i, DEQUANT_WARPS) for i in range(R)]
    acc_full = [Bar("acc_full%d" % i, 1) for i in range(2)]
    acc_empty = [Bar("acc_empty%d" % i, EPILOGUE_WARPS) for i in range(2)]
    copies = []      # in-flight async copies: (barrier, bytes, what landed)
    tensor = []      # in-flight MMA groups: list of completions
    b_state, a_state, r_state = ["free"] * S, ["free"] * S, ["free"] * R
    dq_done = {}

    def wait(bar, parity, phase_index):
        """Wait meant for phase `phase_index` (-1: the initial, already complete one)."""
        while not bar.passes(parity):
            yield
        assert bar.phase >= phase_index + 1, ("wait passed a phase early", bar.name, bar.phase, phase_index)

    def producer():
        it = rit = 0
        for quant, nk in tiles:
            for ks in range(nk):
                if quant and ks % 4 == 0:
                    r = rit % R
                    yield from wait(raw_empty[r], ((rit // R) & 1) ^ 1, rit // R - 1)
                    assert r_state[r] == "free", r_state
                    r_state[r] = "loading"
                    raw_full[r].expect_tx(nmat * 4)
                    copies.extend((raw_full[r], 1, ("raw", r)) for _ in range(nmat * 4))
                    rit += 1
                s = it % S
                if mutant != "producer_skips_empty" or it % 3:
                    yield from wait(empty[s], ((it // S) & 1) ^ 1, it // S - 1)
                assert b_state[s] == "free", ("activation stage refilled while in use", b_state)
                b_state[s] = "loading"
                full_b[s].expect_tx(16)
                copies.append((full_b[s], 16, ("b", s)))
                it += 1

    def loader():
        it = 0
        dense_fills = [0] * S
        for quant, nk in tiles:
            for ks in range(nk):
                s, ph = it % S, (it // S) & 1
                yield from wait(empty[s], ph ^ 1, it // S - 1)
                fill = None
                if not quant:
                    assert a_state[s] == "free", ("weight stage refilled while in use", a_state)
                    a_state[s] = "loading"
                    full_at[s].expect_tx(nmat * 16)
                    copies.extend((full_at[s], 16, ("a", s)) for _ in range(nmat))
                    fill = dense_fills[s]
                    dense_fills[s] += 1
                yield from wait(full_b[s], ph, it // S)
                if fill is not None:
                    yield from wait(full_at[s], fill & 1, fill)
                full[s].arrive()
                it += 1

    def dequant(w):
        it = rit = 0
        for quant, nk in tiles:
            for ks in range(nk):
                r = rit % R
                if quant and ks % 4 == 0:
                    yield from wait(raw_full[r], (rit // R) & 1, rit // R)
                s = it % S
                if mutant != "dequant_skips_empty" or it % 2:
                    yield from wait(empty[s], ((it // S) & 1) ^ 1, it // S - 1)
                if quant:
                    assert r_state[r] == "landed", ("raw column read before it landed", r_state)
                    assert a_state[s] in ("free", "writing"), ("weight stage rewritten while in use", a_state)
                    a_state[s] = "writing"
                    dq_done.setdefault(it, set()).add(w)
                    if len(dq_done[it]) == DEQUANT_WARPS:
                        a_state[s] = "ready"
                for _ in range(rnd.randint(0, 2)):
                    yield
                full[s].arrive()
                if quant and ks % 4 == 3:
                    raw_empty[r].arrive()
                    if raw_empty[r].pending == raw_empty[r].count:
                        r_state[r] = "free"
                    rit += 1
                it += 1

    def mma():
        it = tc = 0
        for quant, nk in tiles:
            b = tc & 1
            yield from wait(acc_empty[b], ((tc >> 1) & 1) ^ 1, (tc >> 1) - 1)
            for ks in range(nk):
                s = it % S
                yield from wait(full[s], (it // S) & 1, it // S)
                assert b_state[s] == "landed", ("MMA before the activation tile landed", b_state)
                assert a_state[s] == "ready", ("MMA before the weight tile was complete", a_state)
                b_state[s] = a_state[s] = "mma"
                tensor.append([("release", s), empty[s]])
                it += 1
            tensor.append([acc_full[b]])
            tc += 1

    def epilogue(q):
        tc = 0
        for _ in tiles:
            b = tc & 1
            yield from wait(acc_full[b], (tc >> 1) & 1, tc >> 1)
            for _ in range(rnd.randint(0, 3)):
                yield
            acc_empty[b].arrive()
            tc += 1

    roles = [producer(), loader(), mma()] + [epilogue(q) for q in range(EPILOGUE_WARPS)] + \
            [dequant(w) for w in range(DEQUANT_WARPS)]
    alive, steps = list(roles), 0
    while alive or copies or tensor:
        steps += 1
        assert steps < 2_000_000, "deadlock"
        c = rnd.random()
        if copies and c < 0.2:   # an async copy lands
            bar, nbytes, (kind, i) = copies.pop(rnd.randrange(len(copies)))
            bar.complete_tx(nbytes)
            if bar.pending == bar.count and bar.tx == 0:
                if kind == "b":
                    b_state[i] = "landed"
                elif kind == "a":
                    a_state[i] = "ready"
                else:
                    r_state[i] = "landed"
            continue
        if tensor and c < 0.35:   # the tensor core finishes the oldest MMA group (in order)
            for ev in tensor.pop(0):
                if isinstance(ev, tuple):
                    b_state[ev[1]] = a_state[ev[1]] = "free"
                else:
                    ev.arrive()
            continue
        if alive:
            g = rnd.choice(alive)
            try:
                next(g)
            except StopIteration:
                alive.remove(g)
    assert all(v == "free" for v in b_state + a_state), (b_state, a_state)


# tile lists: (quantised, K steps); K steps are whole 256-wide columns (multiples of 4)
TILE_LISTS = [
    [(1, 16)] * 3 + [(0, 16)],
    [(1, 4)] * 3 + [(0, 4)] * 2,
    [(0, 8), (1, 8), (0, 4), (1, 4)],
    [(0, 4), (0, 4), (1, 4), (0, 8)],
]


@pytest.mark.parametrize("gemm", [1, 2])
def test_ring_protocol_under_random_interleavings(gemm):
    s1, s2, raws = kernel_rings()
    stages, nmat = (s1, 2) if gemm == 1 else (s2, 1)
    for li, tiles in enumerate(TILE_LISTS):
        for seed in range(6):
            run(tiles, stages, raws, nmat, seed=1000 * gemm + 10 * li + seed)


@pytest.mark.parametrize("mutant", ["producer_skips_empty", "dequant_skips_empty"])
def test_ring_model_catches_a_skipped_wait(mutant):
    s1, _, raws = kernel_rings()
    caught = 0
    for seed in range(12):
        try:
            run(TILE_LISTS[0], s1, raws, 2, seed=seed, mutant=mutant)
        except AssertionError:
            caught += 1
    assert caught > 0, "the model did not notice a role skipping its stage wait"
