"""GPU parity of the decode path (tcgen05 grouped GEMMs with the unpacked
weights in tensor memory) against the oracle, through the C ABI: routing
bit-exact, unpacked codes bit-exact, layer outputs within the row tolerance."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle as orc
from moe_testlib import (assert_parity, make_blocks, make_layer, oracle_forward, oracle_forward_pool, row_errors)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import bit_quantized_moe_top_b200 as bq  # noqa: F401
    assert torch.cuda.is_available()


def _small_mixtral(E=8, K=512, N=384, bits=3, group=128, rank=32, mult=1.0):
    base = ms.make_config("mixtral_decode", comp_std_mult=mult)
    cfg = ms.scaled_config(base, E=E, K=K, N=N)
    cfg.experts = [ms.ExpertSpec(ms.FMT_INT_ASYM, (bits, bits), group, rank) for _ in range(E)]
    return cfg


# ---------------------------------------------------------------------------- routing

@pytest.mark.parametrize("name,T", [("tiny", 16), ("dsv2lite_decode", 256), ("mixtral_decode", 1),
                                    ("mixtral_decode", 200)])
def test_routing_bitexact(name, T):
    cfg = ms.make_config(name)
    cfg = ms.scaled_config(cfg, K=256, N=256)
    cfg.experts = [ms.ExpertSpec(ms.FMT_INT_ASYM, (4, 4), 64, 0) for _ in range(cfg.E)]
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=T)
    X, logits = ms.make_inputs(cfg, T, DEV)
    L.forward(X, logits, cfg.top_k)
    assert L.sync_status() == 0
    r = L.routing(T, cfg.top_k)
    idx, w = orc.route(logits.cpu().numpy(), cfg.top_k)
    counts, offsets, perm, inv = orc.bucket(idx, cfg.E)
    assert np.array_equal(r["idx"].cpu().numpy(), idx)
    assert np.max(np.abs(r["w"].cpu().numpy() - w)) <= 1e-6
    assert np.array_equal(r["counts"].cpu().numpy(), counts)
    assert np.array_equal(r["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(r["perm_token"].cpu().numpy(), perm)
    assert np.array_equal(r["inv_pos"].cpu().numpy(), inv)
    L.close()


def test_routing_ties_and_full_softmax():
    import bit_quantized_moe_top_b200 as bq
    cfg = _small_mixtral(E=8, K=256, N=256, rank=0)
    blocks = make_blocks(cfg, DEV)
    T = 40
    L = make_layer(cfg, blocks, max_tokens=T, max_top_k=3, flags=bq.FLAG_NO_TOPK_RENORM)
    X, _ = ms.make_inputs(cfg, T, DEV)
    # heavy ties: logits on a coarse grid
    g = torch.Generator(device="cpu").manual_seed(3)
    logits = torch.randint(0, 3, (T, cfg.E), generator=g).float().to(DEV)
    L.forward(X, logits, 3)
    r = L.routing(T, 3)
    idx, w = orc.route(logits.cpu().numpy(), 3, renorm=False)
    assert np.array_equal(r["idx"].cpu().numpy(), idx)
    assert np.max(np.abs(r["w"].cpu().numpy() - w)) <= 1e-6
    L.close()


# ---------------------------------------------------------------------------- unpack

@pytest.mark.parametrize("fmt,bits,group", [(ms.FMT_INT_ASYM, 2, 64), (ms.FMT_INT_ASYM, 3, 128),
                                            (ms.FMT_INT_ASYM, 4, 64), (ms.FMT_INT_ASYM, 3, 64),
                                            (ms.FMT_BITPLANE_LUT, 2, 0), (ms.FMT_BITPLANE_LUT, 3, 0),
                                            (ms.FMT_BITPLANE_LUT, 4, 0)])
def test_debug_unpack_bitexact(fmt, bits, group):
    cfg = _small_mixtral(E=2, K=384, N=256, bits=bits, group=group or 128, rank=0)
    cfg.experts = [ms.ExpertSpec(fmt, (bits, bits), group, 0) for _ in range(2)]
    blocks = {}
    for e in range(2):
        for b in (0, 1):
            blocks[(e, b)] = ms.make_block(cfg, e, b, device=DEV, keep_raw=True)
    L = make_layer(cfg, blocks, max_tokens=4)
    for (e, b), blk in blocks.items():
        got = L.debug_unpack(e, b).cpu().numpy()
        if fmt == ms.FMT_INT_ASYM:
            ref = orc.unpack_int_rows(blk.codes.cpu().numpy(), bits, blk.K_in)
        else:
            ref = orc.bitplane_codes(blk.codes.cpu().numpy(), bits)
        assert np.array_equal(got, ref), (e, b)
    L.close()


# ---------------------------------------------------------------------------- layer parity

def test_tiny_config_parity():
    """E=4, top-2, T=16, K=256, N=512, INT4 g64, rank-8 truncated-SVD compensators."""
    cfg = ms.make_config("tiny")
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=16)
    X, logits = ms.make_inputs(cfg, 16, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = oracle_forward(cfg, blocks, X, logits, 2)
    assert_parity(Y, ref["Y"], "tiny")
    L.close()


@pytest.mark.parametrize("T", [1, 3, 8, 33, 64])
@pytest.mark.parametrize("bits,group", [(3, 128), (2, 64), (4, 64)])
def test_small_mixtral_parity(T, bits, group):
    cfg = _small_mixtral(bits=bits, group=group)
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=64)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = oracle_forward(cfg, blocks, X, logits, 2)
    assert_parity(Y, ref["Y"], f"T={T} b={bits}")
    L.close()


def test_compensator_amplified_and_delta():
    """Compensators x10 (about a third of the output) and the delta
    Y(r) - Y(r=0) against the oracle's delta."""
    cfg = _small_mixtral(mult=10.0)
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=32)
    X, logits = ms.make_inputs(cfg, 32, DEV)
    Y = L.forward(X, logits, 2)
    ref = oracle_forward(cfg, blocks, X, logits, 2)
    assert_parity(Y, ref["Y"], "x10")
    cfg0 = _small_mixtral(rank=0)
    blocks0 = {k: ms.BlockWeights(**{**v.__dict__, "rank": 0, "A": None, "B": None}) for k, v in blocks.items()}
    L0 = make_layer(cfg0, blocks0, max_tokens=32)
    Y0 = L0.forward(X, logits, 2)
    ref0 = oracle_forward(cfg0, blocks0, X, logits, 2)
    dg = (Y.float() - Y0.float()).cpu().numpy()
    dr = ref["Y"] - ref0["Y"]
    rel = np.linalg.norm(dg - dr) / np.linalg.norm(dr)
    assert rel <= 2e-2, rel
    L.close()
    L0.close()


def test_top1_and_rank0_and_idle_experts():
    cfg = _small_mixtral(E=16, rank=0)
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=8, max_top_k=2)
    X, logits = ms.make_inputs(cfg, 5, DEV)
    Y = L.forward(X, logits, 1)
    ref = oracle_forward(cfg, blocks, X, logits, 1)
    assert_parity(Y, ref["Y"], "top1")
    L.close()


def test_dense16_rank0_matches_dense_matmul():
    cfg = _small_mixtral(E=4, K=256, N=256, rank=0)
    cfg.experts = [ms.ExpertSpec(ms.FMT_DENSE16, (16, 16), 0, 0) for _ in range(4)]
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=16)
    X, logits = ms.make_inputs(cfg, 16, DEV)
    Y = L.forward(X, logits, 2)
    ref = oracle_forward(cfg, blocks, X, logits, 2)
    assert_parity(Y, ref["Y"], "dense16")
    L.close()


def test_repeat_is_bitwise_deterministic():
    cfg = _small_mixtral()
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=64)
    X, logits = ms.make_inputs(cfg, 48, DEV)
    Y1 = L.forward(X, logits, 2).clone()
    for _ in range(3):
        Y2 = L.forward(X, logits, 2)
        assert torch.equal(Y1, Y2)
    L.close()


def test_forward_host_matches_device():
    cfg = _small_mixtral()
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=64)
    X, logits = ms.make_inputs(cfg, 17, DEV)
    Yd = L.forward(X, logits, 2)
    Yh = L.forward_host(X.cpu().pin_memory(), logits.cpu().pin_memory(), 2)
    assert torch.equal(Yd.cpu(), Yh)
    L.close()


# ---------------------------------------------------------------------------- full size

@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_mixtral_decode_full_size_all_rows(T):
    """Mixtral-8x7B decode layer (E=8, top-2, 4096 x 14336, INT3 g128, rank 32)
    at each token count of the workload, on the benchmark's launch
    configuration (a layer sized for T tokens); every output row checked
    against the oracle."""
    cfg = ms.make_config("mixtral_decode")
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=T)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = oracle_forward_pool(cfg, blocks, X, logits, 2)
    assert_parity(Y, ref["Y"], "mixtral full")
    L.close()


@pytest.mark.parametrize("KN", [(128, 128), (384, 128), (128, 384)])
def test_128_wide_dimensions(KN):
    """d_model or d_ff of 128 (one 128-row block, fewer columns than one
    256-wide K slice or split), and 384 (not a multiple of 256), both paths."""
    K, N = KN
    cfg = _small_mixtral(E=4, K=K, N=N, bits=3, group=64, rank=16)
    blocks = make_blocks(cfg, DEV)
    for path, T in ((1, 8), (2, 200)):
        L = make_layer(cfg, blocks, max_tokens=T)
        L.set_path(path)
        X, logits = ms.make_inputs(cfg, T, DEV)
        Y = L.forward(X, logits, 2)
        assert L.sync_status() == 0
        ref = oracle_forward(cfg, blocks, X, logits, 2)
        assert_parity(Y, ref["Y"], f"K={K} N={N} path={path}")
        L.close()
