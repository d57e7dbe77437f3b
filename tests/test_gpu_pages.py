"""Weight-page movement of bit-plane blocks through the C ABI (PagedWeight:
Efficient MoE LLM Serving with Dynamic Quality-Aware Weight Quantization,
Figure 4: planes are released from GPU memory after the committed bitwidth is
lowered, and restored before a higher bitwidth is committed)."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle as orc
from moe_testlib import assert_parity, make_blocks, make_layer, oracle_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg():
    base = ms.make_config("mixtral_decode")
    cfg = ms.scaled_config(base, E=4, K=512, N=256, top_k=2)
    cfg.experts = [ms.ExpertSpec(ms.FMT_BITPLANE_LUT, (4, 4), 0, 16) for _ in range(4)]
    return cfg


@pytest.mark.parametrize("path", [1, 2])
def test_release_and_reload_planes(path):
    import bit_quantized_moe_top_b200 as bq
    cfg = _cfg()
    blocks = make_blocks(cfg, DEV)
    T = 40 if path == 1 else 300
    L = make_layer(cfg, blocks, max_tokens=T)
    L.set_path(path)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y4 = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    assert L.page_state(1, 0) == (4, 4, 0)
    side = torch.cuda.Stream()
    # lower the committed bits, then release planes 2..3 of every W1 block on a side stream
    for e in range(cfg.E):
        L.set_bits(e, 0, 2)
        L.release_planes(e, 0, 2, stream=side.cuda_stream)
    Y2 = L.forward(X, logits, cfg.top_k)
    side.synchronize()
    assert L.sync_status() == 0
    assert L.page_state(1, 0) == (2, 2, 2)
    ref2 = oracle_forward(cfg, blocks, X, logits, cfg.top_k, bits_override={(e, 0): 2 for e in range(cfg.E)})
    assert_parity(Y2, ref2["Y"], "after release")
    # planes that are not resident cannot be committed
    with pytest.raises(bq.MoEError) as ei:
        L.set_bits(0, 0, 3)
    assert ei.value.status == 5
    with pytest.raises(bq.MoEError) as ei:
        L.release_planes(0, 0, 1)
    assert ei.value.status == 1
    # restore from the host copies on the side stream; set_bits waits for them
    for e in range(cfg.E):
        L.reload_planes(e, 0, 4, stream=side.cuda_stream)
        L.set_bits(e, 0, 4)
    assert L.page_state(2, 0) == (4, 4, 2)
    Y4b = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    assert torch.equal(Y4, Y4b)
    got = L.debug_unpack(3, 0).cpu().numpy()
    assert np.array_equal(got, orc.bitplane_codes(blocks[(3, 0)].codes.cpu().numpy(), 4))
    # a second release reuses the cached host copies (no copy, only the free)
    L.set_bits(2, 0, 3)
    L.release_planes(2, 0, 3, stream=side.cuda_stream)
    side.synchronize()
    assert L.page_state(2, 0) == (3, 3, 2)
    L.close()


def test_page_calls_reject_other_formats():
    import bit_quantized_moe_top_b200 as bq
    base = ms.make_config("mixtral_decode")
    cfg = ms.scaled_config(base, E=2, K=256, N=256, top_k=1)
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=8)
    with pytest.raises(bq.MoEError) as ei:
        L.release_planes(0, 0, 3)
    assert ei.value.status == 4
    with pytest.raises(bq.MoEError) as ei:
        L.reload_planes(0, 0, 4)
    assert ei.value.status == 4
    assert L.page_state(0, 0)[:2] == (3, 3)
    L.close()
