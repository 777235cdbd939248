"""CPU models of the batched-GEMV kernel (decode_kernel in csrc/decode.cuh), run before it
ever touches a GPU and kept as regression checks.

1. Index model.  The kernel's unit -> piece -> address arithmetic is restated here, with its
   constants read from the kernel source, and every address the kernel forms is checked
   against the buffer it points into, on the five workload shapes and on ragged ones:
     * each bulk copy: source inside its weight array, 16-byte aligned, a multiple of 16
       bytes, at most one ring slot;
     * each consumer warp's shared-memory reads inside the bytes its piece brought;
     * each activation read (x, int16 x, sub-block sums, scales, h) inside its buffer;
     * each epilogue write (shared h, routed h, outputs, y) inside its buffer, and every
       output element written exactly once.
2. Protocol model.  The producer, the consumer warps and the epilogue synchronise through
   mbarriers waited on by parity (ring slots full/empty, partial buffers full/empty).  The
   roles' waits and arrivals are replayed in the kernel's order under random interleavings
   and random copy completion; every wait must pass on the phase it was meant for, every
   consumer must read the piece the producer put in the slot for it, the epilogue must
   read each unit's partials once (one epilogue warp per partial buffer, each in order),
   and every interleaving must reach the end.  A mutant
   that skips a wait must be caught.
"""
import os
import random
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DECODE = os.path.join(ROOT, "bit_quantized_routed_sqrt_b200", "csrc", "decode.cuh")
COMMON = os.path.join(ROOT, "bit_quantized_routed_sqrt_b200", "csrc", "common.cuh")


def constants():
    src = open(DECODE).read() + open(COMMON).read()

    def c(name):
        m = re.search(r"constexpr int %s = ([^;]+);" % name, src)
        assert m, name
        return m.group(1).strip()

    tile_bytes = 32 * 84
    K = {
        "CW": int(c("DK_CW")), "NSLOT": int(c("DK_NSLOT")), "TU": int(c("DK_TU")), "TR": int(c("DK_TR")),
        "RANGE": int(c("DK_RANGE")), "DENSE": int(c("DK_DENSE_ELEMS")), "TILE": tile_bytes,
        "MAXT": int(c("MAX_DECODE_T")), "PBUF": int(c("DK_PBUF")),
    }
    K["XA"] = int(c("DK_XA"))
    slot = c("DK_SLOT")
    m = re.match(r"DK_XA \+ (\d+) \* TILE_BYTES", slot)
    assert m, slot
    K["WSLOT"] = int(m.group(1)) * tile_bytes          # the weight area of a slot
    K["SLOT"] = K["XA"] + K["WSLOT"]
    return K


KC = constants()


def dense_rows(K):
    r = 16
    while r > 1 and r * K > KC["DENSE"]:
        r >>= 1
    return r


def plan(T, H, E, k, I, Is):
    p = dict(nbH=H // 256, nbI=I // 256, RSG=dense_rows(H))
    p["SSG"] = 16 // p["RSG"]
    p["RSD"] = dense_rows(Is) if Is > 0 else 16
    p["SSD"] = 16 // p["RSD"]
    p["nSG"] = Is // p["RSG"] if Is > 0 else 0
    p["nSD"] = H // (2 * p["RSD"]) if Is > 0 else 0
    p["RGI"] = I // 32
    p["RPH"] = H // KC["RANGE"]
    p["ppGm"] = (p["nbH"] + 15) // 16
    p["ppD"] = (2 * p["nbI"] + 15) // 16
    p["nTR"] = (T + KC["TR"] - 1) // KC["TR"]
    p["n_route_items"] = E * p["nTR"] + T * p["nbH"]
    p["sd_per_range"] = KC["RANGE"] // (2 * p["RSD"]) if Is > 0 else 0
    p["nB"] = 0
    p["nA"] = p["nSG"] - p["nB"]
    p["nC1"] = 0
    p["nC0"] = p["nSD"] - p["nC1"]
    p["xs_off"] = 2 * H
    p["xc_off"] = p["xs_off"] + H // 4
    p["xrec"] = (p["xc_off"] + H // 64 + 15) // 16 * 16
    p["stage_g"] = KC["TU"] * p["xrec"] <= KC["XA"]
    p["stage_sg"] = T * 2 * H <= KC["XA"]
    p["hs_off"] = 2 * I
    p["hc_off"] = p["hs_off"] + I // 4
    p["hrec"] = (p["hc_off"] + I // 8 + 15) // 16 * 16
    p["stage_d"] = KC["TU"] * p["hrec"] <= KC["XA"]
    p["stage_sd"] = Is > 0 and T * 4 * Is <= KC["XA"]
    return p


def table(topi, T, k, E, pl):
    """build_table: expert token masks, pair offsets, expert groups of <= TU tokens,
    the pair order (by expert, then token) and the unit bounds."""
    TU = KC["TU"]
    mask = [0] * E
    for p, e in enumerate(topi):
        mask[e] |= 1 << (p // k)
    off, grp, base = [0] * (E + 1), [], 0
    for e in range(E):
        off[e] = base
        cnt = bin(mask[e]).count("1")
        for q in range((cnt + TU - 1) // TU):
            grp.append((e, base + q * TU, min(TU, cnt - q * TU)))
        base += cnt
    off[E] = base
    P = T * k
    pair_tok, pair_slot, inv = [None] * P, [None] * P, [None] * P
    for p, e in enumerate(topi):
        t, j = divmod(p, k)
        pos = off[e] + bin(mask[e] & ((1 << t) - 1)).count("1")
        pair_tok[pos], pair_slot[pos], inv[p] = t, j, pos
    NG = len(grp)
    nG, nD = NG * pl["RGI"], NG * pl["RPH"]
    uC = pl["nA"] + nG + pl["nB"]
    uC1 = uC + pl["nC0"]
    uEnd = uC1 + nD + pl["nC1"]
    return dict(mask=mask, off=off, grp=grp, pair_tok=pair_tok, pair_slot=pair_slot, inv=inv, NG=NG, nG=nG,
                nD=nD, uC=uC, uC1=uC1, uEnd=uEnd)


def decode_unit(pl, tb, u):
    """The kernel's unit order: phase A (SG), B (G with one SG after every two G), C0 (SD),
    C1 (D with one SD after every two D)."""
    sg = g = sd = d = None
    if u < pl["nA"]:
        sg = u
    elif u < tb["uC"]:
        p = u - pl["nA"]
        if p % 3 == 2 and p // 3 < pl["nB"]:
            sg = pl["nA"] + p // 3
        else:
            g = p - min(pl["nB"], p // 3)
    elif u < tb["uC1"]:
        sd = u - tb["uC"]
    else:
        p = u - tb["uC1"]
        if p % 3 == 2 and p // 3 < pl["nC1"]:
            sd = pl["nC0"] + p // 3
        else:
            d = p - min(pl["nC1"], p // 3)
    if sg is not None:
        return ("SG", sg * pl["RSG"], 0)
    if g is not None:
        return ("G", g // pl["RGI"], g % pl["RGI"])
    if sd is not None:
        return ("SD", sd * 2 * pl["RSD"], 0)
    return ("D", d // pl["RPH"], d % pl["RPH"])


def unit_pieces(pl, kind):
    return 2 * pl["ppGm"] if kind == "G" else pl["ppD"] if kind == "D" else 2


def piece_src(cfg, pl, tb, un, pi):
    """(array name, byte offset, bytes) of piece pi of unit un."""
    H, I, Is = cfg["H"], cfg["I"], cfg["Is"]
    kind, a, b = un
    gu = I // 32 * (H // 256) * KC["TILE"]
    db = H // 32 * (I // 256) * KC["TILE"]
    if kind == "SG":
        return ("sg" if pi == 0 else "su", a * H * 2, pl["RSG"] * H * 2)
    if kind == "SD":
        return ("sd", (a + pi * pl["RSD"]) * Is * 2, pl["RSD"] * Is * 2)
    e = tb["grp"][a][0]
    if kind == "G":
        mat, b0 = divmod(pi, pl["ppGm"])
        b0 *= 16
        nt = min(16, pl["nbH"] - b0)
        return ("gate" if mat == 0 else "up", e * gu + (b * pl["nbH"] + b0) * KC["TILE"], nt * KC["TILE"])
    t0 = pi * 16
    nt = min(16, 2 * pl["nbI"] - t0)
    return ("down", e * db + (b * 2 * pl["nbI"] + t0) * KC["TILE"], nt * KC["TILE"])


def buffers(cfg):
    T, H, E, k, I, Is = (cfg[n] for n in ("T", "H", "E", "k", "I", "Is"))
    Td = min(cfg.get("max_tokens", T), KC["MAXT"])
    Pd = Td * k
    gu = I // 32 * (H // 256) * KC["TILE"]
    db = H // 32 * (I // 256) * KC["TILE"]
    return dict(gate=E * gu, up=E * gu, down=E * db, sg=Is * H * 2, su=Is * H * 2, sd=H * Is * 2,
                x=T * H, xrec=Td * plan(T, H, E, k, I, Is)["xrec"], hs=Td * max(Is, 1),
                hrec=Pd * plan(1, H, E, k, I, Is)["hrec"], o=Pd * H, s=Td * H, y=T * H)


def check_indices(cfg, topi):
    T, H, E, k, I, Is = (cfg[n] for n in ("T", "H", "E", "k", "I", "Is"))
    pl = plan(T, H, E, k, I, Is)
    tb = table(topi, T, k, E, pl)
    buf = buffers(cfg)
    CW, WSLOT, TILE = KC["CW"], KC["WSLOT"], KC["TILE"]
    XR = pl["xrec"]

    def rd(name, lo, n=1):
        assert 0 <= lo and lo + n <= buf[name], (name, lo, n, buf[name])

    writes = {n: np.zeros(buf[n], np.int32) for n in ("hs", "hrec", "o", "s", "y")}
    HR = pl["hrec"]
    assert HR % 16 == 0 and pl["hc_off"] + 4 * (I // 32) <= HR
    # routing items
    assert pl["n_route_items"] == E * pl["nTR"] + T * pl["nbH"]
    assert XR % 16 == 0 and pl["xc_off"] + 4 * pl["nbH"] <= XR
    for v in range(T * pl["nbH"]):
        t, blk = divmod(v, pl["nbH"])
        rd("xrec", t * XR + blk * 512, 512)
        rd("xrec", t * XR + pl["xs_off"] + blk * 64, 64)
        rd("xrec", t * XR + pl["xc_off"] + blk * 4, 4)
    for u in range(tb["uEnd"]):
        un = decode_unit(pl, tb, u)
        kind, a, b = un
        for pi in range(unit_pieces(pl, kind)):
            name, off, nbytes = piece_src(cfg, pl, tb, un, pi)
            assert off % 16 == 0 and nbytes % 16 == 0 and 0 < nbytes <= WSLOT, (un, pi, off, nbytes)
            rd(name, off, nbytes)
            # activations copied to the front of the slot with the piece
            if kind == "G" and pl["stage_g"]:
                e, p0, nt = tb["grp"][a]
                assert nt * XR <= KC["XA"]
                for t in range(nt):
                    rd("xrec", tb["pair_tok"][p0 + t] * XR, XR)
            if kind == "SG" and pl["stage_sg"]:
                assert T * 2 * H <= KC["XA"] and (T * 2 * H) % 16 == 0
                rd("x", 0, T * H)
            # SD and D inputs, when the producer stages them (the kernel decides at run time;
            # both paths are checked)
            if kind == "D" and pl["stage_d"]:
                e, p0, nt = tb["grp"][a]
                assert nt * HR <= KC["XA"]
                for t in range(nt):
                    rd("hrec", (p0 + t) * HR, HR)
            if kind == "SD" and pl["stage_sd"]:
                assert T * 4 * Is <= KC["XA"] and (T * 4 * Is) % 16 == 0
                rd("hs", 0, T * Is)
            for w in range(CW):
                if kind in ("SG", "SD"):
                    R = pl["RSG"] if kind == "SG" else pl["RSD"]
                    K = H if kind == "SG" else Is
                    S = 16 // R
                    row, seg = divmod(w, S)
                    ln, k0 = K // S, (w % S) * (K // S)
                    assert ln % 8 == 0 and ln <= 1024
                    for it in range(4):
                        kk = it * 256
                        if kk < ln:   # lane 0 .. the last lane with k < len
                            last = min(ln - 8, kk + 31 * 8)
                            assert row * K * 2 + (k0 + last) * 2 + 16 <= nbytes
                            for t in range(T):
                                if kind == "SG":
                                    rd("x", t * H + k0 + last, 8)
                                else:
                                    rd("hs", t * Is + k0 + last, 8)
                                    if pl["stage_sd"]:   # the staged copy in the slot
                                        assert (t * Is + k0 + last + 8) * 4 <= KC["XA"]
                elif kind == "G":
                    mat, b0 = divmod(pi, pl["ppGm"])
                    bb = b0 * 16 + w
                    if bb >= pl["nbH"]:
                        continue
                    assert (w + 1) * TILE <= nbytes
                    e, p0, nt = tb["grp"][a]
                    for t in range(nt):
                        tok = tb["pair_tok"][p0 + t]
                        assert tb["mask"][e] >> tok & 1
                        # staged: the slot's record t; otherwise the global record of tok
                        base = t * XR if pl["stage_g"] else tok * XR
                        lim = KC["XA"] if pl["stage_g"] else buf["xrec"]
                        for lo, n in ((bb * 512, 512), (pl["xs_off"] + bb * 64, 64), (pl["xc_off"] + bb * 4, 4)):
                            assert 0 <= base + lo and base + lo + n <= lim
                else:
                    tq = pi * 16 + w
                    if tq >= 2 * pl["nbI"]:
                        continue
                    assert (w + 1) * TILE <= nbytes
                    bb = tq % pl["nbI"]
                    e, p0, nt = tb["grp"][a]
                    for t in range(nt):
                        p = p0 + t
                        # global record p, and (when staged) the slot's record t
                        for base, lim in ((p * HR, buf["hrec"]),) + (((t * HR, KC["XA"]),) if pl["stage_d"] else ()):
                            for lo, n in ((bb * 512, 512), (pl["hs_off"] + bb * 64, 64), (pl["hc_off"] + bb * 32, 32)):
                                assert 0 <= base + lo and base + lo + n <= lim
        # epilogue writes
        if kind == "SG":
            for r in range(pl["RSG"]):
                for t in range(T):
                    writes["hs"][t * Is + a + r] += 1
        elif kind == "SD":
            for st in range(2):
                for r in range(pl["RSD"]):
                    for t in range(T):
                        writes["s"][t * H + a + st * pl["RSD"] + r] += 1
            assert (a + 2 * pl["RSD"] - 1) // KC["RANGE"] == a // KC["RANGE"]
        elif kind == "G":
            e, p0, nt = tb["grp"][a]
            for t in range(nt):
                r0 = (p0 + t) * HR
                writes["hrec"][r0 + b * 64: r0 + b * 64 + 64] += 1                                  # 32 int16
                writes["hrec"][r0 + pl["hs_off"] + b * 8: r0 + pl["hs_off"] + b * 8 + 8] += 1      # 2 sums
                writes["hrec"][r0 + pl["hc_off"] + b * 4: r0 + pl["hc_off"] + b * 4 + 4] += 1      # 1 scale
        else:
            e, p0, nt = tb["grp"][a]
            assert b < H // KC["RANGE"] <= 256
            for t in range(nt):
                p = p0 + t
                assert 0 <= tb["pair_slot"][p] < k and tb["pair_tok"][p] < T
                writes["o"][p * H + b * KC["RANGE"]: p * H + (b + 1) * KC["RANGE"]] += 1
    for rg in range(H // KC["RANGE"]):
        for t in range(T):
            for h in range(2):
                writes["y"][t * H + rg * KC["RANGE"] + h * 32: t * H + rg * KC["RANGE"] + h * 32 + 32] += 1
            for j in range(k):
                pos = tb["inv"][t * k + j]
                assert 0 <= pos < T * k
    P = T * k
    # every element of the outputs this call defines is written exactly once
    if Is:
        assert np.all(writes["hs"].reshape(-1, Is)[:T] == 1)
        assert np.all(writes["s"].reshape(-1, H)[:T] == 1)
    recs = writes["hrec"].reshape(-1, HR)[:P]
    assert np.all(recs[:, :pl["hc_off"] + 4 * (I // 32)] == 1) and np.all(recs[:, pl["hc_off"] + 4 * (I // 32):] == 0)
    assert np.all(writes["o"].reshape(-1, H)[:P] == 1)
    assert np.all(writes["y"] == 1)
    # every unit index decodes to a distinct unit, each kind exactly covered; the
    # dependencies point backwards: every SG before any SD, every G before any D
    seen = {}
    for u in range(tb["uEnd"]):
        seen.setdefault(decode_unit(pl, tb, u)[0], []).append(u)
    assert len(seen.get("SG", [])) == pl["nSG"] and len(seen.get("SD", [])) == pl["nSD"]
    assert len(seen.get("G", [])) == tb["nG"] and len(seen.get("D", [])) == tb["nD"]
    assert len(set(decode_unit(pl, tb, u) for u in range(tb["uEnd"]))) == tb["uEnd"]
    if pl["nSD"]:
        assert max(seen["SG"]) < min(seen["SD"])
    assert max(seen["G"]) < min(seen["D"])
    # a D unit waits only for its own group's G units: all of them come before it
    g_before = {}
    for u in range(tb["uEnd"]):
        kind, ga, _ = decode_unit(pl, tb, u)
        if kind == "G":
            g_before[ga] = g_before.get(ga, 0) + 1
        elif kind == "D":
            assert g_before.get(ga, 0) == pl["RGI"], ("D unit before its group's G units", u, ga)
    assert all(u < pl["nA"] for u in range(pl["nA"]) if decode_unit(pl, tb, u)[0] == "SG")
    # the combine of a 64-row range of H runs when its count reaches sd_per_range + NG: its
    # down units are exactly that many (each SD unit inside one range, one D unit per group)
    RANGE = KC["RANGE"]
    per_range = [0] * pl["RPH"]
    for u in range(tb["uEnd"]):
        kind, ua, ub = decode_unit(pl, tb, u)
        if kind == "SD":
            r0, r1 = ua // RANGE, (ua + 2 * pl["RSD"] - 1) // RANGE
            assert r0 == r1 and r1 < pl["RPH"], ("SD unit across ranges", u, ua)
            per_range[r0] += 1
        elif kind == "D":
            per_range[ub] += 1
    assert per_range == [pl["sd_per_range"] + tb["NG"]] * pl["RPH"], per_range
    # the permutation is the (expert, token) order and inv is its inverse
    order = sorted(range(P), key=lambda p: (topi[p], p // k))
    assert [tb["inv"][p] for p in order] == list(range(P))
    return pl, tb


SHAPES = [
    # T, H, E, k, I, Is
    (4, 256, 8, 2, 256, 256),
    (1, 4096, 256, 8, 2048, 2048),
    (16, 4096, 256, 8, 2048, 2048),
    (32, 7168, 256, 8, 2048, 2048),
    (5, 256, 4, 4, 256, 0),
    (3, 512, 8, 1, 512, 256),
    (6, 512, 16, 4, 256, 256),
    (32, 768, 32, 16, 768, 512),
    (7, 16384, 64, 6, 1280, 16384),
    (2, 10752, 16, 3, 4864, 2816),
]


@pytest.mark.parametrize("shape", SHAPES, ids=["T%d_H%d_E%d_k%d_I%d_Is%d" % s for s in SHAPES])
def test_decode_indices_in_bounds(shape):
    T, H, E, k, I, Is = shape
    cfg = dict(T=T, H=H, E=E, k=k, I=I, Is=Is)
    rng = np.random.default_rng(T * 1000 + E)
    for trial in range(3):
        if trial == 2 and E >= k:   # crowd the tokens onto few experts (groups of several tokens)
            pool = rng.choice(E, size=max(k, 2), replace=False) if E > k else np.arange(E)
            topi = [int(v) for t in range(T) for v in rng.permutation(pool)[:k]]
        else:
            topi = [int(v) for t in range(T) for v in rng.choice(E, size=k, replace=False)]
        check_indices(cfg, topi)


# ------------------------------------------------------------------ protocol model

class Bar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        self._check()

    def expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        assert self.tx >= 0
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.phase & 1) != parity


def run_protocol(units, n_cons, seed, mutant=None):
    """units: list of piece counts per unit, in claim order of one CTA.  Returns True when
    every role finished; raises AssertionError on a protocol violation."""
    rnd = random.Random(seed)
    NS = KC["NSLOT"]
    full = [Bar(1) for _ in range(NS)]
    empty = [Bar(n_cons) for _ in range(NS)]
    NB = KC["PBUF"]
    pfull = [Bar(n_cons) for _ in range(NB)]
    pempty = [Bar(1) for _ in range(NB)]
    slot_meta = [None] * NS         # what the producer put in each slot
    slot_data = [None] * NS         # what the landed copy holds
    inflight = []                   # (slot, payload)
    part_unit = [None] * NB
    part_data = [[None] * n_cons for _ in range(NB)]
    seq = [(u, pi) for u, np_ in enumerate(units) for pi in range(np_)]
    done = {"epi": []}

    def producer():
        for i, (u, pi) in enumerate(seq):
            s = i % NS
            if i >= NS:
                par = (i // NS - 1) & 1
                if mutant != "producer_skips_empty":
                    while not empty[s].passes(par):
                        yield
            # nothing still reads the slot: every consumer has released position i - NS
            assert all(c >= i - NS + 1 for c in cons_released), ("slot refilled under a reader", i)
            slot_meta[s] = (u, pi, i)
            full[s].expect_tx(1)
            inflight.append((s, (u, pi, i)))
            yield
        i = len(seq)
        s = i % NS
        if i >= NS:
            while not empty[s].passes((i // NS - 1) & 1):
                yield
        slot_meta[s] = (-1, 0, i)
        slot_data[s] = (-1, 0, i)
        full[s].arrive()

    cons_released = [0] * n_cons

    def consumer(c):
        i, n = 0, 0
        while True:
            s = i % NS
            while not full[s].passes((i // NS) & 1):
                yield
            meta = slot_meta[s]
            assert meta[2] == i, ("consumer read another position's slot", c, i, meta)
            if meta[0] < 0:
                break
            assert slot_data[s] == meta, ("data not landed", c, i)
            u, pi, _ = meta
            yield
            empty[s].arrive()
            cons_released[c] = i + 1
            if pi == units[u] - 1:
                b, use = n % NB, n // NB
                if use > 0 and mutant != "consumer_skips_pempty":
                    while not pempty[b].passes((use - 1) & 1):
                        yield
                assert part_data[b][c] is None, ("partials overwritten before the epilogue read them", c, n)
                part_data[b][c] = u
                if c == 0:
                    part_unit[b] = u
                pfull[b].arrive()
                n += 1
            i += 1
        # an end marker in every buffer (one epilogue warp per buffer)
        for m in range(n, n + NB):
            b, use = m % NB, m // NB
            if use > 0:
                while not pempty[b].passes((use - 1) & 1):
                    yield
            assert part_data[b][c] is None
            part_data[b][c] = -1
            if c == 0:
                part_unit[b] = -1
            pfull[b].arrive()

    def epilogue(which):
        # epilogue warp `which` takes the units of buffer `which`, in order
        n = which
        while True:
            b = which
            while not pfull[b].passes((n // NB) & 1):
                yield
            u = part_unit[b]
            assert all(v == u for v in part_data[b]), ("partials of different units", n, part_data[b])
            for c in range(n_cons):
                part_data[b][c] = None
            if u < 0:
                break
            done["epi"].append(u)
            assert u % NB == which
            yield
            pempty[b].arrive()
            n += NB

    roles = [producer()] + [consumer(c) for c in range(n_cons)] + [epilogue(b) for b in range(NB)]
    alive = list(range(len(roles)))
    steps = 0
    while alive:
        steps += 1
        assert steps < 200000, "no progress (deadlock)"
        if inflight and rnd.random() < 0.4:
            s, payload = inflight.pop(rnd.randrange(len(inflight)))
            slot_data[s] = payload
            full[s].complete_tx(1)
            continue
        r = rnd.choice(alive)
        try:
            next(roles[r])
        except StopIteration:
            alive.remove(r)
    assert sorted(done["epi"]) == list(range(len(units))), done["epi"]
    for b in range(NB):
        mine = [u for u in done["epi"] if u % NB == b]
        assert mine == sorted(mine), mine
    return True


@pytest.mark.parametrize("seed", range(40))
def test_decode_protocol_random_interleavings(seed):
    rnd = random.Random(seed)
    units = [rnd.choice([1, 2, 2, 2, 4]) for _ in range(rnd.randint(0, 14))]
    assert run_protocol(units, n_cons=rnd.choice([1, 2, 3]), seed=seed)


@pytest.mark.parametrize("mutant", ["producer_skips_empty", "consumer_skips_pempty"])
def test_decode_protocol_mutants_are_caught(mutant):
    caught = 0
    for seed in range(60):
        rnd = random.Random(seed)
        units = [rnd.choice([1, 2]) for _ in range(12)]
        try:
            run_protocol(units, n_cons=2, seed=seed, mutant=mutant)
        except AssertionError:
            caught += 1
    assert caught > 0, mutant


# ------------------------------------------------------------------ grid protocol model
# Several CTAs claiming units from one counter.  Per CTA: the producer (claims units in
# order; before a shared-down or routed-down unit it waits until the unit's inputs are
# published, then issues its pieces into a ring of NSLOT pieces), the consumers (one agent:
# pieces in ring order), the epilogue (one agent: finished units in order through PBUF
# buffers).  Gate/up epilogues publish their counts (shared: one count; routed: a count per
# expert group); a down epilogue writes its rows and adds one to its 64-row range's count,
# and the one that brings the count to sd_per_range + NG combines the range.

def run_grid_protocol(pl, tb, n_cta, seed, mutant=None):
    rnd = random.Random(seed)
    NS, NB, RANGE = KC["NSLOT"], KC["PBUF"], KC["RANGE"]
    units = [decode_unit(pl, tb, u) for u in range(tb["uEnd"])]
    pieces = [unit_pieces(pl, kind) for kind, _, _ in units]
    nxt = {"u": 0}
    sg_done, grp_done = [0], [0] * tb["NG"]
    rng_done = [0] * pl["RPH"]
    target = pl["sd_per_range"] + tb["NG"] - (1 if mutant == "range_target_short" else 0)
    s_rows = set()                      # (row of H) written by SD units
    o_rows = set()                      # (group, range) written by D units
    combined = []
    ring = [[] for _ in range(n_cta)]   # pieces issued, not yet consumed
    fin = [[] for _ in range(n_cta)]    # units computed, not yet through the epilogue

    def inputs_ready(kind, a):
        if kind == "SD":
            return sg_done[0] == pl["nSG"]
        if kind == "D":
            return grp_done[a] == pl["RGI"]
        return True

    def producer(c):
        while True:
            u = nxt["u"]
            nxt["u"] += 1
            if u >= tb["uEnd"]:
                break
            kind, a, _ = units[u]
            if mutant != "producer_skips_input_wait":
                while not inputs_ready(kind, a):
                    yield
            for pi in range(pieces[u]):
                while len(ring[c]) >= NS:
                    yield
                ring[c].append((u, pi))
                yield
        ring[c].append(None)

    def consumer(c):
        while True:
            while not ring[c]:
                yield
            item = ring[c][0]
            if item is None:
                ring[c].pop(0)
                break
            u, pi = item
            kind, a, _ = units[u]
            # the piece carries its inputs: they must be complete when it is computed
            assert inputs_ready(kind, a), ("inputs not ready", kind, a, u)
            yield
            ring[c].pop(0)
            if pi == pieces[u] - 1:
                while len(fin[c]) >= NB:
                    yield
                fin[c].append(u)
        fin[c].append(None)

    def epilogue(c):
        while True:
            while not fin[c]:
                yield
            u = fin[c].pop(0)
            if u is None:
                break
            kind, a, b = units[u]
            yield
            if kind == "SG":
                sg_done[0] += 1
            elif kind == "G":
                grp_done[a] += 1
            else:
                if kind == "SD":
                    r = a // RANGE
                    s_rows.update(range(a, a + 2 * pl["RSD"]))
                else:
                    r = b
                    o_rows.add((a, b))
                yield
                rng_done[r] += 1
                if rng_done[r] == target:
                    # the combine reads every row of the range: S and each group's w*o
                    assert all(row in s_rows for row in range(r * RANGE, (r + 1) * RANGE)) or pl["nSD"] == 0, \
                        ("combine before the shared down rows", r)
                    assert all((g, r) in o_rows for g in range(tb["NG"])), ("combine before the routed rows", r)
                    combined.append(r)

    roles = []
    for c in range(n_cta):
        roles += [producer(c), consumer(c), epilogue(c)]
    alive = list(range(len(roles)))
    steps = 0
    while alive:
        steps += 1
        assert steps < 400000, "no progress (deadlock)"
        r = rnd.choice(alive)
        try:
            next(roles[r])
        except StopIteration:
            alive.remove(r)
    assert sorted(combined) == list(range(pl["RPH"])), combined
    return True


GRID_SHAPES = [
    # T, H, E, k, I, Is
    (1, 512, 16, 4, 256, 256),
    (3, 256, 8, 2, 256, 256),
    (2, 512, 8, 3, 512, 0),
    (5, 256, 4, 4, 256, 512),
]


@pytest.mark.parametrize("shape", GRID_SHAPES, ids=["T%d_H%d_E%d_k%d_I%d_Is%d" % s for s in GRID_SHAPES])
def test_decode_grid_protocol(shape):
    T, H, E, k, I, Is = shape
    for seed in range(6):
        rnd = np.random.default_rng(seed)
        topi = [int(v) for t in range(T) for v in rnd.choice(E, size=k, replace=False)]
        pl = plan(T, H, E, k, I, Is)
        tb = table(topi, T, k, E, pl)
        assert run_grid_protocol(pl, tb, n_cta=1 + seed % 4, seed=seed)


@pytest.mark.parametrize("mutant", ["producer_skips_input_wait", "range_target_short"])
def test_decode_grid_protocol_mutants_are_caught(mutant):
    T, H, E, k, I, Is = GRID_SHAPES[1]
    caught = 0
    for seed in range(40):
        rnd = np.random.default_rng(seed)
        topi = [int(v) for t in range(T) for v in rnd.choice(E, size=k, replace=False)]
        pl = plan(T, H, E, k, I, Is)
        tb = table(topi, T, k, E, pl)
        try:
            run_grid_protocol(pl, tb, n_cta=8, seed=seed, mutant=mutant)
        except AssertionError:
            caught += 1
    assert caught > 0, mutant
