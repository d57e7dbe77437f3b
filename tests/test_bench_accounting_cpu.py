"""The algorithmic work that bench.py divides by (roofline `achieved`), against
closed forms worked out by hand for the workload shapes: bytes of one expert's
weights per format, flops of the layer, and the tiled shared compensator's
factor bytes. CPU only; no GPU and no library call."""
import importlib.util
import os
import sys

import pytest

import moe_synth as ms

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def _expert_bytes(bench, cfg, e):
    tot = 0
    for b in (0, 1):
        wb, bb, ab = bench.block_bytes(cfg, cfg.experts[e], b)
        tot += wb + bb + ab
    return tot


def test_mixtral_expert_bytes(bench):
    # INT3 g128, rank 32, W1 [28672, 4096], W2 [4096, 14336]:
    # codes 3 * (28672*4096 + 4096*14336) / 8 = 66 060 288
    # scales + zeros 4 * (28672*4096 + 4096*14336) / 128 = 5 505 024
    # factors 2 * 32 * ((28672 + 4096) + (4096 + 14336)) = 3 276 800
    cfg = ms.make_config("mixtral_decode")
    assert _expert_bytes(bench, cfg, 0) == 66060288 + 5505024 + 3276800


def test_mixtral_layer_bytes_all_experts(bench):
    cfg = ms.make_config("mixtral_decode")
    T = 64
    counts = [16] * 8
    # eight experts + X (bf16) + logits (fp32) + Y (bf16)
    assert bench.layer_bytes(cfg, counts, T) == 8 * 74842112 + 2 * T * 4096 + 4 * T * 8 + 2 * T * 4096


def test_dsv2_expert_bytes_at_three_bits(bench):
    # K = 2048, N = 1408, g64, b = 3, r = 32: codes 3 * 3 * 1408 * 2048 / 8,
    # scales 4 * 3 * 1408 * 2048 / 64, factors 2 * 32 * (2816 + 2048 + 2048 + 1408)
    cfg = ms.make_config("dsv2lite_decode")
    cfg.experts = [ms.ExpertSpec(ms.FMT_INT_ASYM, (3, 3), 64, 32)] * cfg.E
    assert _expert_bytes(bench, cfg, 0) == 3244032 + 540672 + 532480


def test_bitplane_expert_bytes(bench):
    # K = 7168, N = 2048, b = (2, 4): planes b * M * K / 8, LUT 2 * 2^b, factors 2 r (M + K)
    cfg = ms.make_config("dsv3_bitplane")
    cfg.experts = [ms.ExpertSpec(ms.FMT_BITPLANE_LUT, (2, 4), 0, 32)] * cfg.E
    w1 = 2 * 4096 * 7168 // 8 + 2 * 4 + 2 * 32 * (4096 + 7168)
    w2 = 4 * 7168 * 2048 // 8 + 2 * 16 + 2 * 32 * (7168 + 2048)
    assert _expert_bytes(bench, cfg, 0) == w1 + w2


def test_prefill_flops(bench):
    # 2 * rows * 3NK + 2 * rows * r * (2K + 3N), rows = T k = 16384
    cfg = ms.make_config("mixtral_prefill")
    counts = [2048] * 8
    main = 2 * 16384 * 3 * 14336 * 4096
    comp = 2 * 16384 * 16 * (2 * 4096 + 3 * 14336)
    assert bench.layer_flops(cfg, counts) == pytest.approx(main + comp, rel=0, abs=0.5)
    assert abs((main + comp) / 1e12 - 5.80) < 0.01
    # the gate/up launch alone: 2 * rows * 2N * (K + r)
    assert bench.gemm1_flops(cfg, counts) == pytest.approx(2 * 16384 * 2 * 14336 * (4096 + 16), abs=0.5)


def test_decode_gemm1_bytes(bench):
    # codes + scales + B1 of the touched experts, routed rows in (K + r) and out (N), fp16
    cfg = ms.make_config("mixtral_decode")
    counts = [16, 0, 16, 0, 0, 0, 0, 0]
    per = 3 * 28672 * 4096 // 8 + 4 * 28672 * 4096 // 128 + 2 * 32 * 28672
    rows = 2 * 16 * (4096 + 32) + 2 * 16 * 14336
    assert bench.gemm1_bytes(cfg, counts) == 2 * per + 2 * rows


def test_tileq_factor_bytes(bench):
    # both blocks, r = 32, 1024 x 1024 tiles, every expert touched:
    # W1: U 28672 x 32, V 32 x 4096, cores 8 * 28 * 4 * 32 * 32; W2: U 4096 x 32,
    # V 32 x 14336, cores 8 * 4 * 14 * 32 * 32; all bf16
    cfg = ms.make_config("mixtral_decode")
    b, _ = bench.tileq_bytes_flops(cfg, [16] * 8, 64, (32, 1024, 1024))
    w1 = 2 * (28672 * 32 + 32 * 4096) + 8 * 2 * 28 * 4 * 32 * 32
    w2 = 2 * (4096 * 32 + 32 * 14336) + 8 * 2 * 4 * 14 * 32 * 32
    assert b == w1 + w2
    assert abs(b / 1e6 - 6.03) < 0.01
