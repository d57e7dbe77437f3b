"""The allocation-free routing entry point, against the layer's own routing
and against the oracle.

moe_route_topk_noalloc serves callers that may not allocate device memory (a
plugin whose host framework owns all device memory, or a serving loop that
must not hit the device-wide synchronisation of cudaMalloc/cudaFree). Its
scratch is a fixed array inside the library. Through the C ABI, two calls in
a row must give the routing of moe_layer_forward + moe_layer_get_routing, and
the oracle's top-k selection, weights, counts and offsets (indices, counts and
offsets bit-exact, weights within 1e-6); requests beyond the array's capacity
are refused before any launch, and the exact capacity is accepted. The file
is named to run last so that a stop-at-first-failure run has already run every
other test.
"""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle as orc
from moe_testlib import make_blocks, make_layer

pytestmark = pytest.mark.gpu

MOE_ERR_TOO_LARGE = 9
FLAG_NO_TOPK_RENORM = 1


def _logits(T, E, key):
    # seeded N(0,1) logits with a Zipf skew, drawn on the host
    L = ms.gaussian((T, E), 1.0, [90, T, E, key], "cpu", torch.float32)
    L = L + torch.from_numpy(ms.zipf_bias(E, 1.1, [90, E])).float()[None, :]
    return L.contiguous()


def _noalloc(bq, logits_d, k, flags=0):
    T, E = logits_d.shape
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    bq.moe_route_topk_noalloc(logits_d, k, idx, w, counts, offsets, flags=flags)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy()


def _check_against_oracle(got, logits, k, renorm):
    idx, w, counts, offsets = got
    ridx, rw = orc.route(logits.numpy(), k, renorm=renorm)
    rcounts, roffsets, _, _ = orc.bucket(ridx, logits.shape[1])
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(w - rw)) <= 1e-6
    assert np.array_equal(counts, rcounts)
    assert np.array_equal(offsets, roffsets)


@pytest.mark.parametrize("name,T", [("mixtral_decode", 64), ("dsv2lite_decode", 256)])
def test_noalloc_routing_matches_layer_and_oracle(name, T):
    import bit_quantized_moe_top_b200 as bq
    cfg = ms.scaled_config(ms.make_config(name), K=256, N=256)
    cfg.experts = [ms.ExpertSpec(ms.FMT_INT_ASYM, (4, 4), 64, 0) for _ in range(cfg.E)]
    blocks = make_blocks(cfg, "cuda")
    L = make_layer(cfg, blocks, max_tokens=T)
    k = cfg.top_k
    for call in range(2):
        X, logits = ms.make_inputs(cfg, T, "cuda", key_extra=call)
        L.forward(X, logits, k)
        assert L.sync_status() == 0
        ref = L.routing(T, k)
        got = _noalloc(bq, logits, k)
        idx, w, counts, offsets = got
        assert np.array_equal(idx, ref["idx"].cpu().numpy()), call
        assert np.max(np.abs(w - ref["w"].cpu().numpy())) <= 1e-6, call
        assert np.array_equal(counts, ref["counts"].cpu().numpy()), call
        assert np.array_equal(offsets, ref["offsets"].cpu().numpy()), call
        _check_against_oracle(got, logits.cpu(), k, renorm=True)
    L.close()


@pytest.mark.parametrize("T,E,k,flags", [
    (64, 8, 2, FLAG_NO_TOPK_RENORM),   # full-softmax probabilities of the selected experts
    (33, 8, 2, 0),                     # a partial last block of 16 tokens
    (1024, 256, 8, 0),                 # all eight logit registers per lane in use; 64 x 256 = capacity
    (4096, 64, 6, 0),                  # exactly the capacity: 256 token blocks x 64 experts
])
def test_noalloc_against_oracle(T, E, k, flags):
    import bit_quantized_moe_top_b200 as bq
    for call in range(2):
        logits = _logits(T, E, call)
        got = _noalloc(bq, logits.cuda(), k, flags)
        _check_against_oracle(got, logits, k, renorm=not (flags & FLAG_NO_TOPK_RENORM))


def test_noalloc_rejects_oversized_request():
    import bit_quantized_moe_top_b200 as bq
    logits = torch.zeros(4097, 64, device="cuda")
    out = torch.empty(4097 * 2, dtype=torch.int32, device="cuda")
    wout = torch.empty(4097 * 2, dtype=torch.float32, device="cuda")
    c = torch.empty(64, dtype=torch.int32, device="cuda")
    o = torch.empty(65, dtype=torch.int32, device="cuda")
    with pytest.raises(bq.MoEError) as ei:
        bq.moe_route_topk_noalloc(logits, 2, out, wout, c, o)
    assert ei.value.status == MOE_ERR_TOO_LARGE
    # a token count near the int range is refused too, before any launch
    lib = bq._lib()
    st = lib.moe_route_topk_noalloc(logits.data_ptr(), 2**31 - 1, 64, 2, 0, out.data_ptr(), wout.data_ptr(),
                                    c.data_ptr(), o.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == MOE_ERR_TOO_LARGE
