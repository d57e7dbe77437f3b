"""GPU parity of the 2D-tiled shared low-rank compensators (TileQ: Efficient
Low-Rank Quantization of Mixture-of-Experts with 2D Tiling, abstract: factors
shared across the experts' input and output dimensions, the experts' low-rank
terms evaluated in one pass) through the C ABI, on both kernel paths, against
the oracle's dense per-expert tiles U_p C[e,p,q] V_q."""
import numpy as np
import pytest
import torch

import moe_synth as ms
from oracle import tileq as otq
from moe_testlib import OracleExperts, assert_parity, make_blocks, make_layer, oracle_forward

pytestmark = pytest.mark.gpu

DEV = "cuda"
PATHS = {"decode": 1, "prefill": 2}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import bit_quantized_moe_top_b200 as bq  # noqa: F401
    assert torch.cuda.is_available()


def _cfg(E=8, K=512, N=768, bits=3, group=128, rank=0, top_k=2):
    base = ms.make_config("mixtral_decode")
    cfg = ms.scaled_config(base, E=E, K=K, N=N, top_k=top_k)
    cfg.experts = [ms.ExpertSpec(ms.FMT_INT_ASYM, (bits, bits), group, rank) for _ in range(E)]
    return cfg


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


class TileqExperts(OracleExperts):
    """Oracle experts whose blocks listed in ``tq`` carry the dense tiled
    compensator D1 / D2 in place of their own factors. With ``fold`` the
    compensator is added to the dequantised weights instead (x W^T + x dW^T
    = x (W + dW)^T: one fp64 matrix per block instead of two, for the
    full-size case; it then applies to every routing slot)."""

    def __init__(self, blocks, tq, fold=False):
        super().__init__(blocks)
        self.tq = tq  # block -> (U, V, C, tile_m, tile_k) as torch tensors
        self.fold = fold

    def __call__(self, e):
        if e not in self.cache:
            d = dict(super().__call__(e))
            for b, nm in ((0, "1"), (1, "2")):
                if b in self.tq:
                    U, V, C, tm, tk = self.tq[b]
                    D = otq.tileq_delta(_np(U), _np(V), _np(C[e]), tm, tk)
                    if self.fold:
                        d["W" + nm] = d["W" + nm] + D
                    else:
                        d["D" + nm] = D
                    d.pop("A" + nm, None)
                    d.pop("B" + nm, None)
            self.cache[e] = d
        return self.cache[e]


def _oracle(cfg, blocks, tq, X, logits, top_k, rows=None, comp_top_n=0, fold=False):
    from oracle import moe_oracle as mo
    return mo.moe_forward(_np(X), logits.cpu().numpy(), top_k, TileqExperts(blocks, tq, fold), cfg.N, rows=rows,
                          comp_top_n=comp_top_n)


def _tileq(cfg, L, blocks_tq, rank, tiles):
    """Sets the tiled compensators of the listed block types; returns the
    factors for the oracle."""
    tq = {}
    for b in blocks_tq:
        tm, tk = tiles[b]
        U, V, C = ms.make_tileq(cfg, b, rank, tm, tk, DEV)
        L.set_tileq(b, rank, tm, tk, U, V, C)
        tq[b] = (U, V, C, tm, tk)
    return tq


# W1 [2N, K] = [1536, 512]: 6 row tiles (3 gate, 3 up) x 2 column tiles;
# W2 [K, N] = [512, 768]: 2 row tiles x 3 column tiles
TILES = {0: (256, 256), 1: (256, 256)}


@pytest.mark.parametrize("path", ["decode", "prefill"])
@pytest.mark.parametrize("T,rank", [(1, 32), (8, 16), (33, 32), (64, 32), (300, 16)])
def test_tileq_parity(path, T, rank):
    cfg = _cfg()
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=max(T, 64))
    L.set_path(PATHS[path])
    tq = _tileq(cfg, L, (0, 1), rank, TILES)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = _oracle(cfg, blocks, tq, X, logits, 2)
    assert_parity(Y, ref["Y"], f"{path} T={T} r={rank}")
    L.close()


@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_tileq_delta_and_clear(path):
    """The compensator's own contribution Y(tiled) - Y(none) against the
    oracle's, and clear_tileq restoring the uncompensated output bit for bit."""
    cfg = _cfg()
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=64)
    L.set_path(PATHS[path])
    X, logits = ms.make_inputs(cfg, 40, DEV)
    Y0 = L.forward(X, logits, 2)
    tq = _tileq(cfg, L, (0, 1), 32, TILES)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = _oracle(cfg, blocks, tq, X, logits, 2)
    ref0 = oracle_forward(cfg, blocks, X, logits, 2)
    dr = ref["Y"] - ref0["Y"]
    dg = (Y.float() - Y0.float()).cpu().numpy()
    assert np.linalg.norm(dr) > 0.1 * np.linalg.norm(ref0["Y"])  # the term is a visible part of the output
    rel = np.linalg.norm(dg - dr) / np.linalg.norm(dr)
    assert rel <= 2e-2, rel
    L.clear_tileq(0)
    L.clear_tileq(1)
    Yc = L.forward(X, logits, 2)
    assert torch.equal(Yc, Y0)
    L.close()


def test_tileq_on_one_block_with_expert_factors_on_the_other():
    """Tiled compensator on W1 only; W2 keeps each expert's own rank-32 pair."""
    cfg = _cfg(rank=32)
    cfg.comp_std_mult = 10.0
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=64)
    tq = _tileq(cfg, L, (0,), 16, TILES)
    X, logits = ms.make_inputs(cfg, 24, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = _oracle(cfg, blocks, tq, X, logits, 2)
    assert_parity(Y, ref["Y"], "W1 tiled, W2 per expert")
    L.close()


@pytest.mark.parametrize("path,T", [("decode", 48), ("prefill", 300)])
def test_tileq_top_n(path, T):
    cfg = _cfg(top_k=3)
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=T)
    L.set_path(PATHS[path])
    tq = _tileq(cfg, L, (0, 1), 32, TILES)
    L.set_comp_top_n(1)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y = L.forward(X, logits, 3)
    assert L.sync_status() == 0
    ref = _oracle(cfg, blocks, tq, X, logits, 3, comp_top_n=1)
    assert_parity(Y, ref["Y"], f"{path} top-n 1")
    L.close()


def test_tileq_rejects_bad_shapes():
    import bit_quantized_moe_top_b200 as bq
    cfg = _cfg()
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=8)
    U, V, C = ms.make_tileq(cfg, 0, 32, 256, 256, DEV)
    for args in [(0, 24, 256, 256), (0, 32, 128, 256), (0, 32, 256, 128), (0, 32, 512, 256), (2, 32, 256, 256),
                 (1, 32, 256, 512)]:
        with pytest.raises(bq.MoEError) as ei:
            L.set_tileq(*args, U, V, C)
        assert ei.value.status == 1  # MOE_ERR_INVALID_ARG
    L.clear_tileq(0)  # nothing set: no-op
    L.close()


def test_mixtral_tileq_full_size_sampled_rows():
    """Mixtral-8x7B-shaped decode layer (INT3 g128) with rank-32 tiled shared
    compensators on both blocks (1024 x 1024 tiles), T = 64, sampled rows."""
    cfg = ms.make_config("mixtral_decode")
    cfg.experts = [ms.ExpertSpec(ms.FMT_INT_ASYM, (3, 3), 128, 0) for _ in range(cfg.E)]
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=64)
    tq = _tileq(cfg, L, (0, 1), 32, {0: (1024, 1024), 1: (1024, 1024)})
    X, logits = ms.make_inputs(cfg, 64, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    rows = [0, 63]
    ref = _oracle(cfg, blocks, tq, X, logits, 2, rows=rows, fold=True)
    assert_parity(Y[rows], ref["Y"], "mixtral tiled full")
    L.close()


@pytest.mark.parametrize("path,T", [("decode", 24), ("prefill", 300)])
def test_tileq_on_bitplane_experts_and_set_bits(path, T):
    """Tiled shared compensators on bit-plane + LUT experts (PagedWeight format),
    then one set_bits on a block: the shared factors stay in force."""
    base = ms.make_config("dsv3_bitplane")
    cfg = ms.scaled_config(base, E=8, K=512, N=768, top_k=2)
    cfg.experts = [ms.ExpertSpec(ms.FMT_BITPLANE_LUT, (3, 4), 0, 0) for _ in range(cfg.E)]
    blocks = make_blocks(cfg, DEV)
    L = make_layer(cfg, blocks, max_tokens=T)
    L.set_path(PATHS[path])
    tq = _tileq(cfg, L, (0, 1), 32, TILES)
    X, logits = ms.make_inputs(cfg, T, DEV)
    Y = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    ref = _oracle(cfg, blocks, tq, X, logits, 2)
    assert_parity(Y, ref["Y"], f"{path} bit-plane tiled")
    L.set_bits(3, 0, 2)
    Y2 = L.forward(X, logits, 2)
    assert L.sync_status() == 0
    from oracle import moe_oracle as mo
    ex = TileqExperts(blocks, tq)
    ex.bits_override = {(3, 0): 2}
    ref2 = mo.moe_forward(_np(X), logits.cpu().numpy(), 2, ex, cfg.N)
    assert_parity(Y2, ref2["Y"], f"{path} bit-plane tiled after set_bits")
    L.close()
