"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on seeded inputs.

Indices and the permutation must be bit-exact; the fp32 layer output must be within
relative L2 5e-3 and max |err| 2e-2 x RMS of the oracle; router scores within 3e-6.
"""
import numpy as np
import pytest

import synth
from gpu_common import (check_output, check_permutation, layer_weights, make_layer, oracle_route_all,
                        sample_tokens, to_dev, tokens, ORACLE_THREADS)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ds4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build_library()
    import bit_quantized_routed_sqrt_b200 as m
    return m


# ------------------------------------------------------------------ repack

def test_repack_round_trip_is_byte_exact(ds4):
    w = synth.Workload("rt", 3, 512, 3, 2, 768, 0, 0.02, "none", 0, 0, (77,), 77)
    lw = synth.make_layer(w)
    layer = make_layer(ds4, w)
    layer.load(lw)
    for which, src in enumerate((lw.gate, lw.up, lw.down)):
        for e in range(w.n_experts):
            out = np.empty_like(src[e])
            layer.ds4moe_export_q2k(which, e, out)
            assert np.array_equal(out, src[e]), (which, e)
    layer.close()


# ------------------------------------------------------------------ router score

def test_router_score_within_3e6_and_naive_form_fails(ds4, ora):
    ls = np.concatenate([np.arange(-80.0, 80.0, 0.01), [-12.0, -12.5, -11.7, -13.3]]).astype(np.float32)
    l_dev = torch.from_numpy(ls).cuda()
    s_dev = torch.empty_like(l_dev)
    ds4.ds4moe_score_eval(l_dev, ls.size, s_dev, 0)
    s = s_dev.cpu().numpy().astype(np.float64)
    ref = np.array([ora.score(float(v)) for v in ls])
    rel = np.abs(s - ref) / ref
    assert rel.max() <= 3e-6, (rel.max(), ls[rel.argmax()])
    ds4.ds4moe_score_eval(l_dev, ls.size, s_dev, 1)
    sn = s_dev.cpu().numpy().astype(np.float64)
    near = (ls > -13.5) & (ls < -11.5)
    reln = np.abs(sn[near] - ref[near]) / ref[near]
    assert reln.max() > 3e-6   # the naive fp32 log(1 + exp(l)) fails the same check near -12


# ------------------------------------------------------------------ routing

ROUTE_CASES = ["tiny_t4_h256_e8_k2", "decode_t1_h4096_e256_k8", "decode_t16_h4096_e256_k8",
               "prefill_t2048_h4096_e256_k8_bias", "prefill4_t8192_h7168_e256_k8_zipf"]


@pytest.mark.parametrize("name", ROUTE_CASES)
def test_route_matches_oracle(ds4, ora, name):
    w = synth.workload(name)
    lw = synth.make_layer(w, 0) if name.startswith("prefill4") else layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w)
    layer.load(lw)
    idx, wt, off, st, ss, inv = layer.route(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    idx_ref, w_ref, _ = oracle_route_all(ora, x, lw, w.top_k)
    idx = idx.cpu().numpy()
    assert np.array_equal(idx, idx_ref), np.argwhere(idx != idx_ref)[:5]
    assert np.allclose(wt.cpu().numpy(), w_ref, rtol=2e-6, atol=1e-7)
    check_permutation(ora, idx_ref, w.n_experts, off.cpu().numpy(), st.cpu().numpy(), ss.cpu().numpy(),
                      inv.cpu().numpy())
    layer.close()


@pytest.mark.parametrize("T", [6, 2], ids=["top-k-per-token-claims", "top-k-in-every-cta"])
def test_planted_ties_go_to_lower_index_via_fp64_rerank(ds4, ora, T):
    """Exact logit ties defeat the bounds: the token falls back to the exact selection (the
    batched-GEMV kernel's two top-k arrangements: tokens claimed from a counter for T > 2,
    every CTA selecting every token for T <= 2)."""
    w = synth.Workload("ties", T, 512, 16, 4, 256, 256, 0.05, "none", 0, 0, (5,), 5)
    lw = synth.make_layer(w)
    wr = lw.router.copy()
    wr[3] = wr[9] = wr[12] = wr[5]            # four experts with identical rows: exact logit ties
    lw.router = wr
    x = synth.make_tokens(w)
    x[0] = synth.bf16_bits(synth.bf16_to_f32(wr[5]) * 20.0)   # token 0 strongly prefers the tied experts
    layer = make_layer(ds4, w)
    layer.load(lw)
    idx, wt, off, st, ss, inv = layer.route(to_dev(x))
    stats = layer.ds4moe_get_stats()
    idx_ref, w_ref, _ = ora.route(x, lw.router, None, w.top_k)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert list(idx_ref[0]) == [3, 5, 9, 12]
    assert stats.router_fallback_tokens >= 1
    layer.close()


# ------------------------------------------------------------------ forward

FORWARD_FULL = ["tiny_t4_h256_e8_k2", "decode_t1_h4096_e256_k8", "decode_t16_h4096_e256_k8"]


@pytest.mark.parametrize("name", FORWARD_FULL)
def test_forward_matches_oracle_every_token(ds4, ora, name):
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w)
    layer.load(lw)
    y = layer.forward(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    y_ref, idx_ref, _ = ora.layer_forward(lw, x, w.top_k, threads=ORACLE_THREADS)
    check_output(y.cpu().numpy(), y_ref, name)
    layer.close()


def test_forward_prefill_sampled_tokens(ds4, ora):
    name = "prefill_t2048_h4096_e256_k8_bias"
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w)
    layer.load(lw)
    xd = to_dev(x)
    y = layer.forward(xd)
    idx, *_ = layer.route(xd)
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    idx = idx.cpu().numpy()
    # 256 seeded tokens plus every token of the 4 heaviest and the 4 lightest experts
    sel = sample_tokens(w.tokens, 256, seed=3, idx=idx, E=w.n_experts)
    y_ref, idx_ref, _ = ora.layer_forward(lw, x, w.top_k, tokens=sel, threads=ORACLE_THREADS)
    assert np.array_equal(idx[sel], idx_ref)
    check_output(y.cpu().numpy()[sel], y_ref, name)
    layer.close()


def test_forward_paths_agree(ds4, ora):
    name = "decode_t16_h4096_e256_k8"
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    xd = to_dev(x)
    ys = []
    for flags in (ds4.FLAG_FORCE_DECODE, ds4.FLAG_FORCE_PREFILL):
        layer = make_layer(ds4, w, flags=flags)
        layer.load(lw)
        ys.append(layer.forward(xd).cpu().numpy())
        layer.ds4moe_sync_status()
        layer.close()
    y_ref, _, _ = ora.layer_forward(lw, x, w.top_k, threads=ORACLE_THREADS)
    for y in ys:
        check_output(y, y_ref)


def test_chained_layers_teacher_forced(ds4, ora):
    """Four chained layers with RMS renormalisation: each layer is checked on the GPU's own
    bf16 input to it (a chained comparison would let near-tied routing flip).  Per layer,
    the routing of every token and the permutation are compared bit for bit, and the
    output on 256 seeded tokens plus tokens of the 4 heaviest and 4 lightest experts (at
    most 32 tokens of each: the heaviest Zipf experts hold thousands)."""
    name = "prefill4_t8192_h7168_e256_k8_zipf"
    w = synth.workload(name)
    T = w.tokens
    x = tokens(name, T)
    xd = to_dev(x)
    for layer_i in range(w.layers):
        lw = synth.make_layer(w, layer_i)
        layer = make_layer(ds4, w, max_tokens=T)
        layer.load(lw)
        y = layer.forward(xd)
        idx, wt, off, st, ss, inv = layer.route(xd)
        torch.cuda.synchronize()
        layer.ds4moe_sync_status()
        x_in = xd.cpu().numpy().view(np.uint16)
        idx = idx.cpu().numpy()
        idx_all, w_all, _ = oracle_route_all(ora, x_in, lw, w.top_k)
        assert np.array_equal(idx, idx_all), ("layer %d" % layer_i, np.argwhere(idx != idx_all)[:5])
        assert np.allclose(wt.cpu().numpy(), w_all, rtol=2e-6, atol=1e-7)
        check_permutation(ora, idx_all, w.n_experts, off.cpu().numpy(), st.cpu().numpy(), ss.cpu().numpy(),
                          inv.cpu().numpy())
        sel = sample_tokens(T, 256, seed=40 + layer_i, idx=idx, E=w.n_experts, cap=32)
        y_ref, idx_ref, _ = ora.layer_forward(lw, x_in, w.top_k, tokens=sel, threads=ORACLE_THREADS)
        assert np.array_equal(idx[sel], idx_ref)
        check_output(y.cpu().numpy()[sel], y_ref, "layer %d" % layer_i)
        # renormalise on the GPU; compare with the oracle's renorm of the GPU output
        x_next = torch.empty_like(xd)
        ds4.ds4moe_rms_renorm(y, T, w.hidden, x_next)
        torch.cuda.synchronize()
        ref_next = ora.rms_renorm(y.cpu().numpy().astype(np.float64))
        got = synth.bf16_to_f32(x_next.cpu().numpy().view(np.uint16)).astype(np.float64)
        exp = synth.bf16_to_f32(ref_next).astype(np.float64)
        assert np.all(np.abs(got - exp) <= np.abs(exp) * 2.0 ** -7 + 1e-30)   # at most one bf16 ulp
        xd = x_next
        layer.close()
        del lw


GROUPED_CASES = [
    # (T, H, E, k, I, Is, bias): ragged token counts, several tiles, no shared expert, I != Is
    (300, 512, 16, 4, 512, 256, "normal"),
    (257, 256, 8, 2, 768, 0, "none"),
    (130, 768, 32, 8, 256, 512, "normal"),
]


@pytest.mark.parametrize("case", GROUPED_CASES, ids=["T%d_H%d_E%d_k%d_I%d_Is%d" % c[:6] for c in GROUPED_CASES])
def test_grouped_path_every_token(ds4, ora, case):
    T, H, E, k, I, Is, bias = case
    w = synth.Workload("grouped", T, H, E, k, I, Is, 0.05, bias, 0.5, 0.0, (61 + T,), 61 + T)
    lw = synth.make_layer(w)
    x = synth.make_tokens(w)
    layer = make_layer(ds4, w, flags=ds4.FLAG_FORCE_PREFILL)
    layer.load(lw)
    y = layer.forward(to_dev(x))
    idx, *_ = layer.route(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    assert layer.ds4moe_get_stats().last_path == 2
    y_ref, idx_ref, _ = ora.layer_forward(lw, x, k, threads=ORACLE_THREADS)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_output(y.cpu().numpy(), y_ref, "grouped T=%d" % T)
    layer.close()


# ------------------------------------------------------------------ edge cases

def test_edge_cases(ds4, ora):
    # k = E (every expert), ragged T, no shared expert
    w = synth.Workload("edge", 5, 256, 4, 4, 256, 0, 0.05, "normal", 0.5, 0, (9,), 9)
    lw = synth.make_layer(w)
    x = synth.make_tokens(w)
    layer = make_layer(ds4, w)
    layer.load(lw)
    y = layer.forward(to_dev(x))
    y_ref, idx_ref, _ = ora.layer_forward(lw, x, w.top_k)
    check_output(y.cpu().numpy(), y_ref, "k=E")
    # T = 0 is a no-op; T > max_tokens and misaligned pointers are rejected
    layer.ds4moe_forward(to_dev(x), 0, torch.empty(1, device="cuda"))
    with pytest.raises(ds4.Ds4MoeError):
        layer.ds4moe_forward(to_dev(x), 6, torch.empty((6, 256), device="cuda"))
    xd = to_dev(np.concatenate([x.reshape(-1), np.zeros(8, np.uint16)]))
    with pytest.raises(ds4.Ds4MoeError):
        layer.ds4moe_forward(xd[1:], 1, torch.empty((1, 256), device="cuda"))
    layer.close()
    # k = 1
    w1 = synth.Workload("k1", 3, 512, 8, 1, 512, 256, 0.05, "none", 0, 0, (10,), 10)
    lw1 = synth.make_layer(w1)
    x1 = synth.make_tokens(w1)
    l1 = make_layer(ds4, w1)
    l1.load(lw1)
    idx, wt, *_ = l1.route(to_dev(x1))
    assert np.all(wt.cpu().numpy() == 1.0)
    y1 = l1.forward(to_dev(x1))
    y1_ref, _, _ = ora.layer_forward(lw1, x1, 1)
    check_output(y1.cpu().numpy(), y1_ref, "k=1")
    l1.close()


def test_decode_down_inputs_too_large_for_the_slot(ds4, ora):
    # I = 4096: two tokens' int16 h records (2 x 9,728 B) exceed a slot's activation area,
    # so the routed down units read h from global memory after waiting for their group
    w = synth.Workload("wide_i", 3, 512, 8, 2, 4096, 256, 0.05, "none", 0.0, 0.0, (17,), 17)
    lw = synth.make_layer(w)
    x = synth.make_tokens(w)
    layer = make_layer(ds4, w)
    layer.load(lw)
    y = layer.forward(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    assert layer.ds4moe_get_stats().last_path == 1
    y_ref, idx_ref, _ = ora.layer_forward(lw, x, w.top_k)
    check_output(y.cpu().numpy(), y_ref, "decode I=4096")
    layer.close()


def test_forward_host_matches_device(ds4):
    name = "tiny_t4_h256_e8_k2"
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w)
    layer.load(lw)
    y_dev = layer.forward(to_dev(x)).cpu().numpy()
    y_host = np.empty((w.tokens, w.hidden), dtype=np.float32)
    layer.ds4moe_forward_host(np.ascontiguousarray(x), w.tokens, y_host)
    assert np.array_equal(y_dev, y_host)
    layer.close()


# ------------------------------------------------------------------ special cases of the method

def _zero_routed(lw):
    """Every routed weight 0: quants 0 and min nibbles 0 (scale nibbles and d, dmin kept)."""
    out = []
    for m in (lw.gate, lw.up, lw.down):
        m = m.copy()
        m[..., 16:80] = 0            # the 64 quant bytes
        m[..., 0:16] &= 0x0F         # min nibbles (high) to 0
        out.append(m)
    return out


@pytest.mark.parametrize("flags", [0, 2], ids=["decode", "grouped"])
def test_zero_routed_experts_leave_the_shared_expert(ds4, ora, flags):
    """All quants and mins zero: every routed weight is 0, so y is the shared expert alone
    (the oracle's special-case pin, here through both CUDA paths)."""
    w = synth.Workload("zero", 6, 512, 16, 4, 512, 256, 0.05, "normal", 0.5, 0.0, (21,), 21)
    lw = synth.make_layer(w)
    lw.gate, lw.up, lw.down = _zero_routed(lw)
    x = synth.make_tokens(w)
    layer = make_layer(ds4, w, flags=flags)
    layer.load(lw)
    y = layer.forward(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    y_ref, _, _ = ora.layer_forward(lw, x, w.top_k)
    check_output(y.cpu().numpy(), y_ref, "zero routed")
    # and that reference is the shared expert alone
    xd64 = synth.bf16_to_f32(x).astype(np.float64)
    y_sh = np.stack([ora.shared(lw.shared_gate, lw.shared_up, lw.shared_down, xd64[t])[1] for t in range(w.tokens)])
    check_output(y.cpu().numpy(), y_sh, "shared only")
    layer.close()


def test_decode_path_handles_large_activations(ds4, ora):
    """The batched-GEMV path quantises activations with a per-block scale, so their
    magnitude does not matter: tokens scaled far beyond the fp16 range still match."""
    w = synth.Workload("big", 3, 512, 16, 4, 512, 256, 0.05, "none", 0.0, 0.0, (23,), 23)
    lw = synth.make_layer(w)
    x = synth.bf16_bits(synth.bf16_to_f32(synth.make_tokens(w)) * 3.0e5)
    layer = make_layer(ds4, w)
    layer.load(lw)
    y = layer.forward(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    y_ref, _, _ = ora.layer_forward(lw, x, w.top_k)
    check_output(y.cpu().numpy(), y_ref, "large activations")
    layer.close()


def test_grouped_path_reports_activations_beyond_fp16(ds4):
    """The grouped path computes in fp16: an activation beyond its range is reported as a
    device-side check failure instead of silently becoming an infinity."""
    w = synth.Workload("big", 40, 512, 16, 4, 512, 256, 0.05, "none", 0.0, 0.0, (23,), 23)
    lw = synth.make_layer(w)
    x = synth.make_tokens(w)
    x[7, 100] = synth.bf16_bits(np.array([1.0e5], np.float32))[0]
    layer = make_layer(ds4, w, flags=ds4.FLAG_FORCE_PREFILL)
    layer.load(lw)
    layer.forward(to_dev(x))
    with pytest.raises(ds4.Ds4MoeError, match="EDEVICE"):
        layer.ds4moe_sync_status()
    # the handle stays usable: in-range tokens run clean afterwards
    x[7, 100] = synth.bf16_bits(np.array([1.0], np.float32))[0]
    layer.forward(to_dev(x))
    layer.ds4moe_sync_status()
    layer.close()


# ------------------------------------------------------------------ failure paths

def test_timed_out_wait_reports_and_the_handle_recovers(ds4, ora):
    """The test hook makes the first forward's routed-down wait run out (a count nothing
    reaches, about 2 ms): the call ends with ETIMEOUT through ds4moe_sync_status, every
    role of the kernel exits, and the next forward on the same handle matches the oracle."""
    name = "tiny_t4_h256_e8_k2"
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w, flags=ds4.FLAG_TEST_TIMEOUT)
    layer.load(lw)
    y = torch.empty((w.tokens, w.hidden), dtype=torch.float32, device="cuda")
    layer.ds4moe_forward(to_dev(x), w.tokens, y)
    with pytest.raises(ds4.Ds4MoeError, match="ETIMEOUT"):
        layer.ds4moe_sync_status()
    y = layer.forward(to_dev(x))
    torch.cuda.synchronize()
    layer.ds4moe_sync_status()
    y_ref, _, _ = ora.layer_forward(lw, x, w.top_k)
    check_output(y.cpu().numpy(), y_ref, "after a timeout")
    layer.close()


def test_injected_host_failures_return_status(ds4, monkeypatch):
    """DS4MOE_FAULT makes a host-side step fail without touching the GPU; the handle is
    usable again once the variable is gone."""
    name = "tiny_t4_h256_e8_k2"
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w)
    monkeypatch.setenv("DS4MOE_FAULT", "h2d")
    with pytest.raises(ds4.Ds4MoeError, match="ECUDA.*injected"):
        layer.load(lw)
    monkeypatch.delenv("DS4MOE_FAULT")
    layer.load(lw)
    monkeypatch.setenv("DS4MOE_FAULT", "launch")
    with pytest.raises(ds4.Ds4MoeError, match="ECUDA.*injected"):
        layer.forward(to_dev(x))
    monkeypatch.delenv("DS4MOE_FAULT")
    layer.forward(to_dev(x))
    layer.ds4moe_sync_status()
    layer.close()


def test_decode_trace_records_every_unit(ds4):
    """The timeline of one batched-GEMV launch: every unit was issued, started and finished
    in that order, the unit kinds are in their documented order, and every CTA recorded
    its start, routing and exit."""
    name = "decode_t1_h4096_e256_k8"
    w = synth.workload(name)
    lw = layer_weights(name)
    x = tokens(name)
    layer = make_layer(ds4, w, flags=ds4.FLAG_TRACE)
    layer.load(lw)
    layer.forward(to_dev(x))
    rec, b = layer.ds4moe_get_trace()
    n_units, n_cta = int(b[5]), int(b[6])
    assert 0 == b[0] <= b[1] <= b[2] <= b[3] <= b[4] <= n_units
    units = rec[:b[4]]
    assert np.array_equal(units[:, 0] & 0xFFFFFFFF, np.arange(b[4]))
    assert np.all(units[:, 1] > 0) and np.all(units[:, 2] >= units[:, 1]) and np.all(units[:, 3] >= units[:, 2])
    ctas = rec[n_units:n_units + 2 * n_cta].reshape(n_cta, 8)
    start, items, seen, topk, table, done = (ctas[:, i] for i in range(6))
    assert np.all(items >= start) and np.all(seen >= start) and np.all(topk >= seen) and np.all(table >= topk)
    assert np.all(done >= table)
    tail = rec[n_units + 2 * n_cta:n_units + 2 * n_cta + 4].reshape(-1)
    assert list(tail[:4]) == list(b[1:5])
    assert np.all(np.diff(tail[8:14]) >= 0) and tail[8] >= seen[0]
    ext = rec[n_units + 2 * n_cta + 4:n_units + 2 * n_cta + 4 + 2 * n_units].reshape(n_units, 8)[:b[4]]
    assert len(ext) == b[4]
    assert np.all(((ext[:, 2] & 0xFFFF) >= 0) & ((ext[:, 2] & 0xFFFF) < n_cta))
    # a piece is seen landed after it was issued, computed after it was seen
    assert np.all(ext[:, 3] >= units[:, 1]) and np.all(ext[:, 6] >= ext[:, 3])
    # partials written after the unit started, epilogue started after that, ended after that
    assert np.all(ext[:, 0] >= units[:, 2]) and np.all(ext[:, 1] >= ext[:, 0]) and np.all(units[:, 3] >= ext[:, 1])
    layer.close()
