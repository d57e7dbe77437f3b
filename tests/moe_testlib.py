"""Test helpers: build a GPU layer and the matching oracle experts from one set
of generated tensors, and compare outputs with the parity tolerance.

Tolerance (fp16 tensor-core operands, fp32 accumulation, bf16 output):
every output row has relative L2 error <= 4e-3 and max abs error
<= 1e-2 * max|Y_ref| against the fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import moe_synth as ms
import oracle as orc

ROW_REL_L2 = 4e-3
MAX_ABS_FRAC = 1e-2


def block_to_oracle(blk: ms.BlockWeights, bits=None) -> dict:
    """Dequantised fp64 weights of a generated block (oracle), plus factors."""
    d = {"fmt": blk.fmt, "bits": bits or blk.bits, "group": blk.group, "K_in": blk.K_in,
         "codes": blk.codes.cpu().numpy() if blk.fmt != ms.FMT_DENSE16 else blk.codes.float().cpu().numpy(),
         "scales": None if blk.scales is None else blk.scales.cpu().numpy(),
         "zeros_or_lut": None if blk.zeros_or_lut is None else blk.zeros_or_lut.cpu().numpy()}
    out = {"W": orc.dequant_block(d)}
    if blk.rank > 0:
        out["A"] = blk.A.float().cpu().numpy().astype(np.float64)
        out["B"] = blk.B.float().cpu().numpy().astype(np.float64)
    return out


def attach_svd(cfg: ms.LayerConfig, blk: ms.BlockWeights, rank: int):
    """Truncated-SVD compensator of the block's quantisation residual, built by
    the oracle (MiLo abstract: compensators of the quantisation loss)."""
    W = blk.dense.double().cpu().numpy()
    What = orc.dequant_block({"fmt": blk.fmt, "bits": blk.bits, "group": blk.group, "K_in": blk.K_in,
                              "codes": blk.codes.cpu().numpy(), "scales": blk.scales.cpu().numpy(),
                              "zeros_or_lut": blk.zeros_or_lut.cpu().numpy()})
    A, B = orc.svd_compensator(W - What, rank)
    dev = blk.codes.device
    blk.A = torch.from_numpy(A).to(torch.bfloat16).to(dev).contiguous()
    blk.B = torch.from_numpy(B).to(torch.bfloat16).to(dev).contiguous()
    blk.rank = rank


def make_blocks(cfg: ms.LayerConfig, device: str, experts=None):
    blocks = {}
    for e in (range(cfg.E) if experts is None else experts):
        for b in (0, 1):
            keep = cfg.comp == "svd"
            blk = ms.make_block(cfg, e, b, device=device, keep_dense=keep)
            if cfg.comp == "svd" and cfg.experts[e].rank > 0:
                attach_svd(cfg, blk, cfg.experts[e].rank)
            blocks[(e, b)] = blk
    return blocks


def descs_of(cfg: ms.LayerConfig):
    import ctypes
    import bit_quantized_moe_top_b200 as bq
    return [bq.ExpertDesc((ctypes.c_int * 2)(*sp.bits), sp.fmt, sp.group, sp.rank) for sp in cfg.experts[:cfg.E]]


def make_layer(cfg: ms.LayerConfig, blocks, max_tokens: int, max_top_k=None, flags=0):
    import bit_quantized_moe_top_b200 as bq
    L = bq.MoELayer(cfg.E, cfg.K, cfg.N, max_tokens, max_top_k or cfg.top_k, descs_of(cfg), flags)
    for (e, b), blk in blocks.items():
        L.set_expert_weights(e, b, blk.codes.contiguous(),
                             None if blk.scales is None else blk.scales.contiguous(),
                             None if blk.zeros_or_lut is None else blk.zeros_or_lut.contiguous(),
                             None if blk.rank == 0 else blk.A.contiguous(),
                             None if blk.rank == 0 else blk.B.contiguous())
    return L


class OracleExperts:
    """Lazily dequantised experts for ``oracle.moe_forward``."""

    def __init__(self, blocks, bits_override=None):
        self.blocks = blocks
        self.cache = {}
        self.bits_override = bits_override or {}

    def __call__(self, e):
        if e not in self.cache:
            d = {}
            for b, nm in ((0, "1"), (1, "2")):
                o = block_to_oracle(self.blocks[(e, b)], self.bits_override.get((e, b)))
                d["W" + nm] = o["W"]
                if "A" in o:
                    d["A" + nm] = o["A"]
                    d["B" + nm] = o["B"]
            self.cache[e] = d
        return self.cache[e]


def oracle_forward(cfg, blocks, X, logits, top_k, rows=None, renorm=True, bits_override=None, comp_top_n=0):
    Xn = X.float().cpu().numpy().astype(np.float64)
    Ln = logits.cpu().numpy()
    return orc.moe_forward(Xn, Ln, top_k, OracleExperts(blocks, bits_override), cfg.N, renorm=renorm, rows=rows,
                           comp_top_n=comp_top_n)


def _block_job_dict(blk: ms.BlockWeights, bits=None) -> dict:
    d = {"fmt": blk.fmt, "bits": bits or blk.bits, "group": blk.group, "K_in": blk.K_in,
         "codes": blk.codes.cpu().numpy() if blk.fmt != ms.FMT_DENSE16 else blk.codes.float().cpu().numpy(),
         "scales": None if blk.scales is None else blk.scales.cpu().numpy(),
         "zeros_or_lut": None if blk.zeros_or_lut is None else blk.zeros_or_lut.cpu().numpy()}
    out = {"blk": d, "A": None, "B": None}
    if blk.rank > 0:
        out["A"] = blk.A.float().cpu().numpy().astype(np.float64)
        out["B"] = blk.B.float().cpu().numpy().astype(np.float64)
    return out


def oracle_forward_pool(cfg, blocks, X, logits, top_k, rows=None, renorm=True, bits_override=None, comp_top_n=0):
    """``oracle_forward`` with the experts dequantised and run in a pool of
    spawned processes (for full-size layers)."""
    import oracle_pool
    bo = bits_override or {}

    def block_of(e):
        return {b: _block_job_dict(blocks[(e, b)], bo.get((e, b))) for b in (0, 1)}

    return oracle_pool.forward(X.float().cpu().numpy().astype(np.float64), logits.cpu().numpy(), top_k, block_of,
                               cfg.N, renorm=renorm, rows=rows, comp_top_n=comp_top_n)


def prefill_sample_rows(logits, top_k, tile=128, extra=8, seed=0):
    """Tokens whose outputs a full-size prefill test compares: for every
    expert bucket (the oracle's routing and bucketing), its first and last
    rows, the rows on both sides of each 128-row token-tile boundary within
    the first pair of tiles (positions 127, 128, 255, 256), and the first row
    of its last, partially filled pair of tiles; plus a few random tokens."""
    L = logits.cpu().numpy()
    idx, _ = orc.route(L, top_k)
    E = L.shape[1]
    counts, offsets, perm, _ = orc.bucket(idx, E)
    rows = set()
    for e in range(E):
        n, lo = int(counts[e]), int(offsets[e])
        if n == 0:
            continue
        for pos in (0, n - 1, tile - 1, tile, 2 * tile - 1, 2 * tile, (n - 1) // (2 * tile) * (2 * tile)):
            if 0 <= pos < n:
                rows.add(int(perm[lo + pos]))
    rng = np.random.default_rng(seed)
    rows.update(int(t) for t in rng.integers(0, L.shape[0], size=extra))
    return sorted(rows)


def row_errors(Y: torch.Tensor, Yref: np.ndarray):
    Yg = Y.float().cpu().numpy().astype(np.float64)
    num = np.linalg.norm(Yg - Yref, axis=1)
    den = np.linalg.norm(Yref, axis=1)
    rel = num / np.maximum(den, 1e-30)
    mabs = np.max(np.abs(Yg - Yref))
    return rel, mabs


def assert_parity(Y: torch.Tensor, Yref: np.ndarray, what=""):
    rel, mabs = row_errors(Y, Yref)
    lim = MAX_ABS_FRAC * np.max(np.abs(Yref))
    assert np.all(np.isfinite(rel)), what
    assert rel.max() <= ROW_REL_L2, f"{what}: worst row rel L2 {rel.max():.3e} (row {rel.argmax()})"
    assert mabs <= lim, f"{what}: max abs {mabs:.3e} > {lim:.3e}"
    return rel.max(), mabs
