"""Seeded synthetic inputs for the quantized MoE expert layer.

This module is shared by the tests, the benchmark and the CPU oracle's checks.
It only draws random tensors and writes them in the storage formats the layer
consumes; it holds none of the layer's forward arithmetic (no dequantisation,
routing, GEMM, SwiGLU or combine).

What it produces, per expert linear block (W1 = gate||up [2N, K], W2 = down
[K, N]):

* dense weights ~ N(0, 0.02) in fp32;
* for the integer format: asymmetric min-max round-to-nearest codes with one
  fp16 scale and one fp16 zero per group of ``g`` along K, packed as a
  little-endian bit-stream per row (code k occupies bits [b*k, b*k+b));
* for the bit-plane format: a 4-bit code from a uniform 16-level min-max grid
  over the whole block, stored as 4 bit-planes (plane 0 = most significant bit,
  bit i of 32-bit word w = element 32*w+i), plus one fp16 lookup table per
  bitwidth b in {2,3,4} holding the mean of the weights whose top-b code is c;
* low-rank factors A [r, K_in], B [M_out, r] (bf16, Gaussian);
* activations X bf16 N(0,1) and router logits fp32 N(0,1) (+ a Zipf bias).

The quantisers are input synthesis: the pages leave the offline quantiser
unspecified (MiLo abstract: "highly quantized MoEs"; PagedWeight Figure 3:
"bitwidth-specific centroid values"), and the oracle and the GPU library both
consume exactly the stored values written here.

Every tensor is drawn from a ``torch.Generator`` seeded from a tuple through
``numpy.random.SeedSequence``; the same tuple on the same device gives the same
bits. CPU and CUDA generators give different streams, so a test compares two
implementations on one set of tensors, never across devices.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

FMT_INT_ASYM = 0
FMT_BITPLANE_LUT = 1
FMT_DENSE16 = 2

# offsets of LUT_b inside the 28-entry per-block table (b = 2, 3, 4)
LUT_OFFSET = {2: 0, 3: 4, 4: 12}
LUT_ENTRIES = 28


def seed_of(*key: int) -> int:
    """64-bit seed from an integer tuple (SeedSequence hashing)."""
    st = np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key]).generate_state(2, dtype=np.uint32)
    return int(st[0]) | (int(st[1] & 0x7FFFFFFF) << 32)


def generator(key: Sequence[int], device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(*key))
    return g


def gaussian(shape, std: float, key: Sequence[int], device="cpu", dtype=torch.float32) -> torch.Tensor:
    g = generator(key, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


# ----------------------------------------------------------------------------
# integer format: asymmetric min-max RTN, group g along K
# ----------------------------------------------------------------------------

def rtn_int_asym(W: torch.Tensor, bits: int, group: int):
    """Quantise W [M, K] (fp32) -> q uint8 [M, K], s fp16 [M, K/g], z fp16 [M, K/g].

    Per group: lo/hi = min/max, s = fp16((hi-lo)/(2^b-1)), z = clamp(rne(-lo/s)),
    q = clamp(rne(w/s) + z). Quantising against the stored fp16 scale keeps the
    codes consistent with what is stored. Degenerate groups (hi == lo) use s = 1.
    """
    M, K = W.shape
    assert K % group == 0
    qmax = (1 << bits) - 1
    Wg = W.to(torch.float64).reshape(M, K // group, group)
    lo = Wg.amin(dim=2)
    hi = Wg.amax(dim=2)
    s = ((hi - lo) / qmax).to(torch.float16)
    s = torch.where(hi == lo, torch.ones_like(s), s)
    s64 = s.to(torch.float64)
    z = torch.clamp(torch.round(-lo / s64), 0, qmax)
    q = torch.clamp(torch.round(Wg / s64[:, :, None]) + z[:, :, None], 0, qmax)
    return q.reshape(M, K).to(torch.uint8), s, z.to(torch.float16)


def pack_int_rows(q: torch.Tensor, bits: int) -> torch.Tensor:
    """Pack codes [M, K] (values < 2^bits) into a little-endian bit-stream per row.

    Code k of a row occupies bits [bits*k, bits*k + bits) of the row's stream;
    bit j of the stream is bit (j % 8) of byte j // 8. Returns uint8 [M, K*bits/8].
    """
    M, K = q.shape
    assert (K * bits) % 8 == 0
    shifts = torch.arange(bits, device=q.device, dtype=torch.int32)
    bitsarr = ((q.to(torch.int32)[:, :, None] >> shifts) & 1).reshape(M, K * bits // 8, 8)
    weights = (1 << torch.arange(8, device=q.device, dtype=torch.int32))
    return (bitsarr * weights).sum(dim=2).to(torch.uint8)


# ----------------------------------------------------------------------------
# bit-plane + LUT format
# ----------------------------------------------------------------------------

def bitplane_quantize(W: torch.Tensor):
    """4-bit codes of W [M, K] on a uniform 16-level min-max grid over the block,
    and the per-bitwidth LUTs (fp16, 28 entries: LUT_2 | LUT_3 | LUT_4).

    LUT_b[c] = mean of the weights whose 4-bit code shifted right by (4-b)
    equals c; an empty bucket takes the centre of its interval.
    """
    W64 = W.to(torch.float64)
    lo = W64.min()
    hi = W64.max()
    step = (hi - lo) / 16.0 if hi > lo else torch.tensor(1.0, dtype=torch.float64, device=W.device)
    code4 = torch.clamp(torch.floor((W64 - lo) / step), 0, 15).to(torch.int64)
    lut = torch.zeros(LUT_ENTRIES, dtype=torch.float64, device=W.device)
    flat_w = W64.reshape(-1)
    for b in (2, 3, 4):
        cb = (code4 >> (4 - b)).reshape(-1)
        nb = 1 << b
        sums = torch.zeros(nb, dtype=torch.float64, device=W.device).index_add_(0, cb, flat_w)
        cnts = torch.zeros(nb, dtype=torch.float64, device=W.device).index_add_(0, cb, torch.ones_like(flat_w))
        width = (hi - lo) / nb if hi > lo else torch.tensor(1.0, dtype=torch.float64, device=W.device)
        centre = lo + (torch.arange(nb, dtype=torch.float64, device=W.device) + 0.5) * width
        vals = torch.where(cnts > 0, sums / torch.clamp(cnts, min=1), centre)
        lut[LUT_OFFSET[b]:LUT_OFFSET[b] + nb] = vals
    return code4.to(torch.uint8), lut.to(torch.float16)


def pack_bitplanes(code4: torch.Tensor) -> torch.Tensor:
    """4-bit codes [M, K] -> planes uint32-as-int32 [4, M, K/32]; plane 0 = MSB;
    bit i of word w of a row is element 32*w + i."""
    M, K = code4.shape
    assert K % 32 == 0
    c = code4.to(torch.int64)
    out = []
    weights = (torch.ones(32, dtype=torch.int64, device=code4.device) << torch.arange(32, device=code4.device))
    for p in range(4):
        bit = ((c >> (3 - p)) & 1).reshape(M, K // 32, 32)
        words = (bit * weights).sum(dim=2)  # < 2^32
        out.append(words)
    planes = torch.stack(out, 0)
    planes = torch.where(planes >= (1 << 31), planes - (1 << 32), planes).to(torch.int32)
    return planes


# ----------------------------------------------------------------------------
# configurations (shapes of the pages' workloads)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class ExpertSpec:
    fmt: int
    bits: Tuple[int, int]   # (W1, W2); 16 for dense
    group: int
    rank: int


@dataclasses.dataclass
class LayerConfig:
    cid: int
    name: str
    E: int
    top_k: int
    K: int              # d_model
    N: int              # d_ff
    tokens: Tuple[int, ...]
    experts: List[ExpertSpec]
    comp: str = "gauss"        # "gauss" | "svd" | "none"
    comp_std_mult: float = 1.0
    zipf_s: float = 0.0
    dense_std: float = 0.02


def _draw_choice(key, choices, n):
    g = np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))
    return [int(choices[i]) for i in g.integers(0, len(choices), size=n)]


def make_config(name: str, comp_std_mult: float = 1.0) -> LayerConfig:
    """The five workload shapes, by name."""
    if name == "tiny":
        E = 4
        ex = [ExpertSpec(FMT_INT_ASYM, (4, 4), 64, 8) for _ in range(E)]
        return LayerConfig(0, name, E, 2, 256, 512, (16,), ex, comp="svd", comp_std_mult=comp_std_mult)
    if name == "mixtral_decode":
        E = 8
        ex = [ExpertSpec(FMT_INT_ASYM, (3, 3), 128, 32) for _ in range(E)]
        return LayerConfig(1, name, E, 2, 4096, 14336, (1, 8, 32, 64), ex, comp_std_mult=comp_std_mult)
    if name == "dsv2lite_decode":
        E = 64
        bits = _draw_choice([2, 7, 1], (2, 3, 4), E)
        ranks = _draw_choice([2, 7, 2], (0, 16, 32, 64), E)
        ex = [ExpertSpec(FMT_INT_ASYM, (bits[e], bits[e]), 64, ranks[e]) for e in range(E)]
        return LayerConfig(2, name, E, 6, 2048, 1408, (256,), ex, zipf_s=1.1, comp_std_mult=comp_std_mult)
    if name == "mixtral_prefill":
        E = 8
        ex = [ExpertSpec(FMT_INT_ASYM, (4, 4), 128, 16) for _ in range(E)]
        return LayerConfig(3, name, E, 2, 4096, 14336, (8192,), ex, comp_std_mult=comp_std_mult)
    if name == "dsv3_bitplane":
        E = 256
        b1 = _draw_choice([4, 7, 1], (2, 3, 4), E)
        b2 = _draw_choice([4, 7, 2], (2, 3, 4), E)
        ex = [ExpertSpec(FMT_BITPLANE_LUT, (b1[e], b2[e]), 0, 32) for e in range(E)]
        return LayerConfig(4, name, E, 8, 7168, 2048, (128, 4096), ex, zipf_s=1.2, comp_std_mult=comp_std_mult)
    raise KeyError(name)


def scaled_config(base: LayerConfig, E=None, K=None, N=None, top_k=None, name=None) -> LayerConfig:
    """Same formats and seeds as ``base`` with smaller dimensions (parity cases)."""
    c = dataclasses.replace(base)
    c.E = E or base.E
    c.K = K or base.K
    c.N = N or base.N
    c.top_k = top_k or base.top_k
    c.experts = [base.experts[e % len(base.experts)] for e in range(c.E)]
    c.name = name or (base.name + "_scaled")
    return c


# ----------------------------------------------------------------------------
# per-block weights
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class BlockWeights:
    """One expert linear block in its stored form (tensors on one device)."""
    fmt: int
    bits: int
    group: int
    rank: int
    M: int
    K_in: int
    codes: torch.Tensor                   # INT: uint8 [M, K*b/8]; BITPLANE: int32 [4, M, K/32]; DENSE16: bf16 [M, K]
    scales: Optional[torch.Tensor]        # INT: fp16 [M, K/g]
    zeros_or_lut: Optional[torch.Tensor]  # INT: fp16 [M, K/g]; BITPLANE: fp16 [28]
    A: Optional[torch.Tensor]             # bf16 [r, K_in]
    B: Optional[torch.Tensor]             # bf16 [M, r]
    dense: Optional[torch.Tensor] = None  # fp32 [M, K] (kept only when asked)
    raw_codes: Optional[torch.Tensor] = None  # uint8 [M, K] unpacked codes (INT) or 4-bit codes (BITPLANE)


def block_shape(cfg: LayerConfig, block: int) -> Tuple[int, int]:
    return (2 * cfg.N, cfg.K) if block == 0 else (cfg.K, cfg.N)


def make_block(cfg: LayerConfig, expert: int, block: int, device="cpu", keep_dense=False,
               keep_raw=False, with_comp=True) -> BlockWeights:
    """Weights of (expert, block) for ``cfg``; seeds [cid, expert, block, tensor_id].

    Compensators of the "svd" kind are not made here (they need the residual of
    the dequantised weights); the caller attaches them.
    """
    spec = cfg.experts[expert]
    M, K_in = block_shape(cfg, block)
    W = gaussian((M, K_in), cfg.dense_std, [cfg.cid, expert, block, 0], device)
    bits = spec.bits[block]
    r = spec.rank if (with_comp and cfg.comp != "none") else 0
    A = B = None
    if r > 0 and cfg.comp == "gauss":
        std = 0.02 / math.sqrt(r) * cfg.comp_std_mult
        A = gaussian((r, K_in), std, [cfg.cid, expert, block, 1], device, torch.bfloat16)
        B = gaussian((M, r), std, [cfg.cid, expert, block, 2], device, torch.bfloat16)
    raw = None
    if spec.fmt == FMT_INT_ASYM:
        q, s, z = rtn_int_asym(W, bits, spec.group)
        codes = pack_int_rows(q, bits)
        scales, zl = s, z
        raw = q
    elif spec.fmt == FMT_BITPLANE_LUT:
        code4, lut = bitplane_quantize(W)
        codes = pack_bitplanes(code4)
        scales, zl = None, lut
        raw = code4
    elif spec.fmt == FMT_DENSE16:
        codes = W.to(torch.bfloat16)
        scales = zl = None
    else:
        raise ValueError(spec.fmt)
    return BlockWeights(spec.fmt, bits, spec.group, r, M, K_in, codes, scales, zl, A, B,
                        dense=W if keep_dense else None, raw_codes=raw if keep_raw else None)


def make_tileq(cfg: LayerConfig, block: int, rank: int, tile_m: int, tile_k: int, device="cpu",
               core_std: float = 0.005):
    """Seeded 2D-tiled shared compensator factors of one block type, bf16:
    U [M, r] and V [r, K_in] ~ N(0, 1/r), cores [E, P, Q, r, r] ~ N(0, core_std^2)
    (so that one tile of an expert's compensator has entries of about core_std).
    Seeds [cid, 2000 + block, tensor_id]."""
    M, K_in = block_shape(cfg, block)
    P, Q = M // tile_m, K_in // tile_k
    std = 1.0 / math.sqrt(rank)
    U = gaussian((M, rank), std, [cfg.cid, 2000 + block, 0], device, torch.bfloat16)
    V = gaussian((rank, K_in), std, [cfg.cid, 2000 + block, 1], device, torch.bfloat16)
    C = gaussian((cfg.E, P, Q, rank, rank), core_std, [cfg.cid, 2000 + block, 2], device, torch.bfloat16)
    return U, V, C


def zipf_bias(E: int, s: float, key: Sequence[int]) -> np.ndarray:
    """bias_e = -s * ln(pi(e) + 1) for a seeded permutation pi of 0..E-1 (the
    logarithm of a Zipf(s) pmf, up to a constant)."""
    g = np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))
    pi = g.permutation(E)
    return (-s * np.log(pi + 1.0)).astype(np.float32)


def make_inputs(cfg: LayerConfig, T: int, device="cpu", key_extra: int = 0):
    """X bf16 [T, K] ~ N(0,1); logits fp32 [T, E] ~ N(0,1) + Zipf bias."""
    X = gaussian((T, cfg.K), 1.0, [cfg.cid, 1000, T, key_extra], device, torch.bfloat16)
    L = gaussian((T, cfg.E), 1.0, [cfg.cid, 2000, T, key_extra], device, torch.float32)
    if cfg.zipf_s > 0:
        L = L + torch.from_numpy(zipf_bias(cfg.E, cfg.zipf_s, [cfg.cid, 3000])).to(device)[None, :]
    return X, L.contiguous()
