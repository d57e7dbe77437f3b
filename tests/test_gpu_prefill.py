"""GPU parity of the prefill path (tcgen05 grouped GEMMs) and of the bit-plane
format (both paths, with set_bits), through the C ABI, against the oracle."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle as orc
from moe_testlib import (assert_parity, make_blocks, make_layer, oracle_forward, oracle_forward_pool,
                         prefill_sample_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(E=8, K=512, N=384, fmt=ms.FMT_INT_ASYM, bits=(3, 3), group=128, rank=32, top_k=2, zipf=0.0, mult=1.0):
    base = ms.make_config("mixtral_decode", comp_std_mult=mult)
    cfg = ms.scaled_config(base, E=E, K=K, N=N, top_k=top_k)
    cfg.experts = [ms.ExpertSpec(fmt, bits, group, rank) for _ in range(E)]
    cfg.zipf_s = zipf
    return cfg


def _run(cfg, T, path, max_tokens=None, flags=0):
    import bit_quantized_moe_top_b200 as bq
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=max_tokens or T, flags=flags)
    L.set_path(path)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y = L.forward(X, logits, cfg.top_k)
    st = L.sync_status()
    assert st == 0, bq.moe_status_string(st)
    return L, blocks, X, logits, Y


@pytest.mark.parametrize("T", [40, 300, 520])
@pytest.mark.parametrize("bits,group", [(3, 128), (4, 64), (2, 64)])
def test_prefill_int_parity(T, bits, group):
    import bit_quantized_moe_top_b200 as bq
    cfg = _cfg(bits=(bits, bits), group=group)
    L, blocks, X, logits, Y = _run(cfg, T, bq.PATH_PREFILL)
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Y, ref["Y"], f"prefill T={T} b={bits}")
    L.close()


def test_prefill_matches_decode_path():
    import bit_quantized_moe_top_b200 as bq
    cfg = _cfg()
    L, blocks, X, logits, Yp = _run(cfg, 200, bq.PATH_PREFILL)
    L.set_path(bq.PATH_DECODE)
    Yd = L.forward(X, logits, cfg.top_k)
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Yp, ref["Y"], "prefill")
    assert_parity(Yd, ref["Y"], "decode")
    L.close()


def test_prefill_tiny_config():
    import bit_quantized_moe_top_b200 as bq
    cfg = ms.make_config("tiny")
    L, blocks, X, logits, Y = _run(cfg, 16, bq.PATH_PREFILL)
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Y, ref["Y"], "tiny prefill")
    L.close()


def test_prefill_compensator_amplified():
    import bit_quantized_moe_top_b200 as bq
    cfg = _cfg(mult=10.0, rank=64)
    L, blocks, X, logits, Y = _run(cfg, 260, bq.PATH_PREFILL)
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Y, ref["Y"], "prefill x10")
    L.close()


@pytest.mark.parametrize("path", [1, 2])
def test_bitplane_mixed_bits_and_set_bits(path):
    """Bit-plane + LUT experts with per-block bits drawn from {2,3,4}, then a
    set_bits re-draw (only descriptors change) checked against the oracle at
    the new bits."""
    E = 16
    cfg = _cfg(E=E, K=512, N=256, fmt=ms.FMT_BITPLANE_LUT, group=0, rank=32, top_k=4, zipf=1.2)
    rng = np.random.default_rng(5)
    cfg.experts = [ms.ExpertSpec(ms.FMT_BITPLANE_LUT, tuple(int(b) for b in rng.choice([2, 3, 4], 2)), 0, 32)
                   for _ in range(E)]
    T = 48 if path == 1 else 300
    L, blocks, X, logits, Y = _run(cfg, T, path)
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Y, ref["Y"], "bit-plane")
    newbits = {}
    for e in range(E):
        for b in (0, 1):
            nb = int(rng.choice([2, 3, 4]))
            L.set_bits(e, b, nb)
            newbits[(e, b)] = nb
    Y2 = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    ref2 = oracle_forward(cfg, blocks, X, logits, cfg.top_k, bits_override=newbits)
    assert_parity(Y2, ref2["Y"], "bit-plane after set_bits")
    for (e, b), nb in list(newbits.items())[:4]:
        got = L.debug_unpack(e, b).cpu().numpy()
        assert np.array_equal(got, orc.bitplane_codes(blocks[(e, b)].codes.cpu().numpy(), nb))
    L.close()


def test_set_bits_errors():
    import bit_quantized_moe_top_b200 as bq
    cfg = _cfg(E=2, K=256, N=256, fmt=ms.FMT_BITPLANE_LUT, group=0, rank=0)
    cfg.experts = [ms.ExpertSpec(ms.FMT_BITPLANE_LUT, (3, 3), 0, 0) for _ in range(2)]
    L, blocks, X, logits, Y = _run(cfg, 8, 1)
    with pytest.raises(bq.MoEError) as ei:
        L.set_bits(0, 0, 5)
    assert ei.value.status == 5  # MOE_ERR_BITS_UNAVAILABLE
    with pytest.raises(bq.MoEError) as ei:
        L.set_bits(0, 0, 1)
    assert ei.value.status == 1
    L.close()
    # INT codes cannot be truncated: set_bits invalidates the block until reloaded
    cfg = _cfg(E=2, K=256, N=256, rank=0)
    L, blocks, X, logits, Y = _run(cfg, 8, 1)
    L.set_bits(1, 0, 2)
    with pytest.raises(bq.MoEError) as ei:
        L.forward(X, logits, cfg.top_k)
    assert ei.value.status == 3  # MOE_ERR_NOT_LOADED
    L.close()


# ---------------------------------------------------------------------------- full-size configurations

def test_dsv2lite_decode_full_size_all_rows():
    """64 experts, top-6, 2048 x 1408, per-expert bits {2,3,4} g64, ranks
    {0,16,32,64}, Zipf(1.1)-skewed routing, T = 256; every row."""
    cfg = ms.make_config("dsv2lite_decode")
    L, blocks, X, logits, Y = _run(cfg, 256, 0)
    ref = oracle_forward_pool(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Y, ref["Y"], "dsv2lite")
    L.close()


def test_mixtral_prefill_full_size_sampled_rows():
    """Mixtral-8x7B prefill layer: INT4 g128, rank 16, T = 8192 (tcgen05
    path). Rows: the first and last of every expert bucket, both sides of the
    128-token tile boundaries, the last partial pair of tiles, random rows."""
    cfg = ms.make_config("mixtral_prefill")
    L, blocks, X, logits, Y = _run(cfg, 8192, 0)
    rows = prefill_sample_rows(logits, cfg.top_k)
    assert len(rows) >= 32
    ref = oracle_forward_pool(cfg, blocks, X, logits, cfg.top_k, rows=rows)
    assert_parity(Y[rows], ref["Y"], "mixtral prefill")
    L.close()


def _redraw_bits(L, cfg, seed=11):
    rng = np.random.default_rng(seed)
    newbits = {}
    for e in range(cfg.E):
        for b in (0, 1):
            nb = int(rng.choice([2, 3, 4]))
            L.set_bits(e, b, nb)
            newbits[(e, b)] = nb
    return newbits


def test_dsv3_bitplane_decode_full_size_all_rows():
    """256 bit-plane experts, top-8, 7168 x 2048, bits {2,3,4} per block,
    rank 32, Zipf(1.2) routing, T = 128, every row; then one set_bits
    re-draw of every block."""
    cfg = ms.make_config("dsv3_bitplane")
    T = 128
    L, blocks, X, logits, Y = _run(cfg, T, 0)
    ref = oracle_forward_pool(cfg, blocks, X, logits, cfg.top_k)
    assert_parity(Y, ref["Y"], "dsv3 decode")
    newbits = _redraw_bits(L, cfg)
    Y2 = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    ref2 = oracle_forward_pool(cfg, blocks, X, logits, cfg.top_k, bits_override=newbits)
    assert_parity(Y2, ref2["Y"], "dsv3 decode after set_bits")
    L.close()


def test_dsv3_bitplane_prefill_full_size_sampled_rows():
    """The DeepSeek-V3-shaped bit-plane layer at T = 4096 on the prefill path,
    rows by the prefill sampling rule, before and after one set_bits re-draw
    of every block."""
    cfg = ms.make_config("dsv3_bitplane")
    T = 4096
    L, blocks, X, logits, Y = _run(cfg, T, 0)
    rows = prefill_sample_rows(logits, cfg.top_k, extra=16)
    assert len(rows) >= 32
    ref = oracle_forward_pool(cfg, blocks, X, logits, cfg.top_k, rows=rows)
    assert_parity(Y[rows], ref["Y"], "dsv3 prefill")
    newbits = _redraw_bits(L, cfg)
    Y2 = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    ref2 = oracle_forward_pool(cfg, blocks, X, logits, cfg.top_k, rows=rows, bits_override=newbits)
    assert_parity(Y2[rows], ref2["Y"], "dsv3 prefill after set_bits")
    L.close()


@pytest.mark.parametrize("path,T", [(1, 48), (2, 300)])
def test_top_n_compensation(path, T):
    """BEAM-style compensation of only the first n routing slots, both paths."""
    cfg = _cfg(mult=10.0, top_k=3)
    L, blocks, X, logits, Y = _run(cfg, T, path)
    L.set_comp_top_n(1)
    Y1 = L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    ref1 = oracle_forward(cfg, blocks, X, logits, cfg.top_k, comp_top_n=1)
    assert_parity(Y1, ref1["Y"], "top-n 1")
    ref = oracle_forward(cfg, blocks, X, logits, cfg.top_k)
    assert np.max(np.abs(ref1["Y"] - ref["Y"])) > 0.05 * np.max(np.abs(ref["Y"]))
    L.set_comp_top_n(0)
    Y0 = L.forward(X, logits, cfg.top_k)
    assert torch.equal(Y0, Y)
    L.close()
