"""ds4moe_route_static (routing with scratch in a static device array, no allocation)
against ds4moe_route on the same inputs, two calls in a row each.

The file name sorts last so the test also runs after every other GPU test; it builds its
own handles and inputs and passes alone as well.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

CASES = [
    # (workload, T): a decode batch, a ragged T over several 64-token blocks, the limit
    ("decode_t16_h4096_e256_k8", 16),
    ("prefill_t2048_h4096_e256_k8_bias", 200),
    ("prefill_t2048_h4096_e256_k8_bias", 256),
]


def _outputs(torch, T, k, E):
    dev = "cuda"
    return (torch.full((T, k), -1, dtype=torch.int32, device=dev), torch.full((T, k), -1.0, device=dev),
            torch.full((E + 1,), -1, dtype=torch.int32, device=dev),
            torch.full((T * k,), -1, dtype=torch.int32, device=dev),
            torch.full((T * k,), -1, dtype=torch.int32, device=dev),
            torch.full((T * k,), -1, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("name,T", CASES)
def test_route_static_matches_route(name, T):
    import torch
    import bit_quantized_routed_sqrt_b200 as ds4
    w = synth.workload(name)
    lw = synth.make_layer(w)
    layer = ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=T)
    layer.load(lw)
    for call in range(2):
        # each call routes other tokens, so a word of the shared scratch left over from the
        # first call cannot stand in for one the second call must write
        x = synth.make_tokens(w, tokens=T, stream=call)
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        ref = _outputs(torch, T, w.top_k, w.n_experts)
        layer.ds4moe_route(xd, T, *ref)
        torch.cuda.synchronize()
        layer.ds4moe_sync_status()
        ref = [t.cpu().numpy() for t in ref]
        out = _outputs(torch, T, w.top_k, w.n_experts)
        layer.ds4moe_route_static(xd, T, *out)
        torch.cuda.synchronize()
        layer.ds4moe_sync_status()
        got = [t.cpu().numpy() for t in out]
        tag = "%s T=%d call %d" % (name, T, call)
        # indices and the permutation are bit-exact; the weights agree to fp32 rounding
        assert np.array_equal(got[0], ref[0]), tag
        np.testing.assert_allclose(got[1], ref[1], rtol=1e-6, atol=0, err_msg=tag)
        for g, r, what in zip(got[2:], ref[2:], ("offsets", "sorted_token", "sorted_slot", "inv_pos")):
            assert np.array_equal(g, r), (tag, what)
    layer.close()


def test_route_static_rejects_more_tokens_than_its_scratch():
    import torch
    import bit_quantized_routed_sqrt_b200 as ds4
    w = synth.workload("tiny_t4_h256_e8_k2")
    lw = synth.make_layer(w)
    T = ds4.ROUTE_STATIC_MAX_TOKENS + 1
    layer = ds4.Ds4Moe(w.hidden, w.n_experts, w.top_k, w.inter, w.shared_inter, max_tokens=T)
    layer.load(lw)
    x = synth.make_tokens(w, tokens=T)
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    out = _outputs(torch, T, w.top_k, w.n_experts)
    with pytest.raises(ds4.Ds4MoeError, match="static routing scratch"):
        layer.ds4moe_route_static(xd, T, *out)
    with pytest.raises(ds4.Ds4MoeError, match="required"):
        layer.ds4moe_route_static(xd, 4, out[0], out[1], None, out[3], out[4], out[5])
    layer.close()
