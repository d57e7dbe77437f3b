"""The allocation-free routing entry point against the layer's own routing.

moe_route_topk_noalloc serves callers that may not allocate device memory (a
plugin whose host framework owns all device memory, or a serving loop that
must not hit the device-wide synchronisation of cudaMalloc/cudaFree). Its
scratch is a fixed array inside the library; this test checks, through the C
ABI, that two calls in a row give the same routing as moe_layer_forward +
moe_layer_get_routing, and that oversized requests are refused. The file is
named to run last so that a stop-at-first-failure run has already run every
other test.
"""
import numpy as np
import pytest
import torch

import moe_synth as ms
from moe_testlib import make_blocks, make_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("mixtral_decode", 64), ("dsv2lite_decode", 256)])
def test_noalloc_routing_matches_layer(name, T):
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
        idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
        counts = torch.full((cfg.E,), -1, dtype=torch.int32, device="cuda")
        offsets = torch.full((cfg.E + 1,), -1, dtype=torch.int32, device="cuda")
        bq.moe_route_topk_noalloc(logits, k, idx, w, counts, offsets)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref["idx"]), call
        assert np.max(np.abs(w.cpu().numpy() - ref["w"].cpu().numpy())) <= 1e-6, call
        assert torch.equal(counts, ref["counts"]), call
        assert torch.equal(offsets, ref["offsets"]), call
    L.close()


def test_noalloc_rejects_oversized_request():
    import bit_quantized_moe_top_b200 as bq
    logits = torch.zeros(4097, 64, device="cuda")
    out = torch.empty(4097 * 2, dtype=torch.int32, device="cuda")
    wout = torch.empty(4097 * 2, dtype=torch.float32, device="cuda")
    c = torch.empty(64, dtype=torch.int32, device="cuda")
    o = torch.empty(65, dtype=torch.int32, device="cuda")
    with pytest.raises(bq.MoEError) as ei:
        bq.moe_route_topk_noalloc(logits, 2, out, wout, c, o)
    assert ei.value.status == 9  # MOE_ERR_TOO_LARGE
