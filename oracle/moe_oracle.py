"""Plain fp64 CPU oracle of the quantized MoE expert layer forward pass.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module: only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
legs of ``bench.py`` may call it. It shares no code with the CUDA library.

The oracle writes out the plain definition of each step, in fp64, with numpy:

1. dequantise every expert linear block from its stored form
   (group-wise asymmetric integer codes, or bit-planes + lookup table);
2. route each token to its top-k experts with softmax weights;
3. bucket the routed (token, slot) pairs per expert;
4. per expert: h = W1^ x + B1 (A1 x); z = silu(h_gate) * h_up;
   o = W2^ z + B2 (A2 z);
5. combine y_t = sum_j w_tj * o_tj.

Sources (page titles and the passage each step follows):

* MiLo: Efficient Quantized MoE Inference with Mixture of Low-Rank
  Compensators, abstract: highly quantized experts plus low-rank compensators
  that recover the quantisation loss (step 4, the B(Ax) terms).
* PagedWeight: Efficient MoE LLM Serving with Dynamic Quality-Aware Weight
  Quantization, Figure 3 caption: bit-plane storage where subsets of planes
  give different effective bitwidths, each tensor with a LUT of
  bitwidth-specific centroids (step 1, bit-plane branch); "What carries the
  argument": a weight page is one expert linear block (the unit of bits).
* Bandwidth-Efficient Adaptive Mixture-of-Experts via Low-Rank Compensation,
  abstract: top-k routing per token with the compensators applied per routed
  expert (steps 2 and 4).
* MxMoE: Mixed-precision Quantization for MoE with Accuracy and Performance
  Co-Design, abstract: bitwidths that differ between linear blocks and experts
  (step 1 takes each block's own bits).
* TileQ: Efficient Low-Rank Quantization of Mixture-of-Experts with 2D Tiling,
  abstract: low-rank expert terms evaluated with the quantized GEMM (step 4);
  its shared 2D-tiled factors enter step 4 as dense compensators D1, D2
  (oracle/tileq.py).

Readings where the pages are silent:

* integer format: w^ = (q - z) * s with one fp16 scale s and one fp16 zero z
  per group of g consecutive elements along K; codes packed little-endian per
  row, code k at bits [b*k, b*k + b);
* bit-plane format: 4 planes, plane 0 = most significant bit; at bitwidth b
  the code is the top b planes, c = sum_{p<b} bit_p * 2^(b-1-p), and
  w^ = LUT_b[c]; the per-block table stores LUT_2 | LUT_3 | LUT_4 (28 fp16);
* routing: top-k by exact comparison of the fp32 logits, ties to the lower
  expert index, slots in descending order; weights are the softmax over the k
  selected logits (or, with ``renorm=False``, the full-softmax probabilities);
* bucketing: expert-major, token-ascending; inv_pos[t, j] is the row of
  (t, j) in that order;
* W1 = [gate; up] stacked along rows (gate = rows 0..N-1);
  silu(a) = a / (1 + exp(-a));
* each block (W1 and W2) has its own compensator pair with the expert's rank.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

LUT_OFFSET = {2: 0, 3: 4, 4: 12}


# ----------------------------------------------------------------------------
# 1. storage formats
# ----------------------------------------------------------------------------

def unpack_int_rows(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Codes [M, K] from the per-row little-endian bit-stream [M, K*bits/8].

    Code k starts at stream bit bits*k, i.e. bit (bits*k) % 8 of byte
    (bits*k) // 8, and may run into the next byte.
    """
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    M = packed.shape[0]
    padded = np.concatenate([packed, np.zeros((M, 1), np.uint8)], axis=1).astype(np.uint32)
    k = np.arange(K)
    start = bits * k
    byte = start // 8
    shift = (start % 8).astype(np.uint32)
    window = padded[:, byte] | (padded[:, byte + 1] << 8)
    return ((window >> shift) & ((1 << bits) - 1)).astype(np.uint8)


def pack_int_rows(q: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of ``unpack_int_rows`` (one Python integer per row)."""
    q = np.asarray(q)
    M, K = q.shape
    nbytes = K * bits // 8
    out = np.zeros((M, nbytes), np.uint8)
    for m in range(M):
        acc = 0
        for k in range(K):
            acc |= int(q[m, k]) << (bits * k)
        out[m] = np.frombuffer(acc.to_bytes(nbytes, "little"), np.uint8)
    return out


def dequant_int(q: np.ndarray, s: np.ndarray, z: np.ndarray, group: int) -> np.ndarray:
    """w^[m, k] = (q[m, k] - z[m, k // g]) * s[m, k // g], in fp64."""
    M, K = q.shape
    gi = np.arange(K) // group
    s64 = np.asarray(s, np.float64)[:, gi]
    z64 = np.asarray(z, np.float64)[:, gi]
    return (q.astype(np.float64) - z64) * s64


def bitplane_codes(planes: np.ndarray, bits: int) -> np.ndarray:
    """b-bit codes [M, K] from planes [4, M, K/32]: bit i of word w of a row is
    element 32*w + i; the code is the top ``bits`` planes, plane 0 the MSB."""
    P = np.asarray(planes).view(np.uint32)
    _, M, W = P.shape
    i = np.arange(32, dtype=np.uint32)
    code = np.zeros((M, W * 32), np.int64)
    for p in range(bits):
        bit = ((P[p][:, :, None] >> i) & 1).reshape(M, W * 32).astype(np.int64)
        code += bit << (bits - 1 - p)
    return code


def dequant_bitplane(planes: np.ndarray, lut: np.ndarray, bits: int) -> np.ndarray:
    """w^[m, k] = LUT_b[c_b[m, k]], in fp64."""
    c = bitplane_codes(planes, bits)
    table = np.asarray(lut, np.float64)[LUT_OFFSET[bits]:LUT_OFFSET[bits] + (1 << bits)]
    return table[c]


def dequant_block(blk: Dict) -> np.ndarray:
    """Dense fp64 weights of one block given as a dict of numpy arrays:
    fmt (0 int, 1 bit-plane, 2 dense), bits, group, K_in, codes, scales,
    zeros_or_lut."""
    fmt = blk["fmt"]
    if fmt == 0:
        q = unpack_int_rows(blk["codes"], blk["bits"], blk["K_in"])
        return dequant_int(q, blk["scales"], blk["zeros_or_lut"], blk["group"])
    if fmt == 1:
        return dequant_bitplane(blk["codes"], blk["zeros_or_lut"], blk["bits"])
    if fmt == 2:
        return np.asarray(blk["codes"], np.float64)
    raise ValueError(fmt)


# ----------------------------------------------------------------------------
# 2-3. routing and bucketing
# ----------------------------------------------------------------------------

def route(logits: np.ndarray, top_k: int, renorm: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """idx int64 [T, k] (descending logit, ties to the lower expert index) and
    weights fp64 [T, k]."""
    L = np.asarray(logits, np.float32)
    T, E = L.shape
    idx = np.zeros((T, top_k), np.int64)
    w = np.zeros((T, top_k), np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(L[t, e]), e))
        sel = order[:top_k]
        idx[t] = sel
        l64 = L[t].astype(np.float64)
        lmax = l64[sel[0]]
        num = np.exp(l64[sel] - lmax)
        den = num.sum() if renorm else np.exp(l64 - lmax).sum()
        w[t] = num / den
    return idx, w


def bucket(idx: np.ndarray, E: int):
    """counts [E], offsets [E+1], perm_token [T*k], inv_pos [T, k] for the
    expert-major, token-ascending order of the routed pairs."""
    T, k = idx.shape
    counts = np.zeros(E, np.int64)
    offsets = np.zeros(E + 1, np.int64)
    perm = np.zeros(T * k, np.int64)
    inv = np.full((T, k), -1, np.int64)
    p = 0
    for e in range(E):
        offsets[e] = p
        ts, js = np.nonzero(idx == e)      # row-major: tokens ascending
        n = len(ts)
        perm[p:p + n] = ts
        inv[ts, js] = np.arange(p, p + n)
        counts[e] = n
        p += n
    offsets[E] = p
    return counts, offsets, perm, inv


# ----------------------------------------------------------------------------
# 4-5. expert FFN and combine
# ----------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def expert_ffn(x: np.ndarray, W1: np.ndarray, W2: np.ndarray, N: int,
               A1=None, B1=None, A2=None, B2=None, D1=None, D2=None) -> np.ndarray:
    """Rows x [n, K] -> o [n, K] for one expert (all fp64). D1 / D2 are dense
    compensators (the 2D-tiled shared form, oracle/tileq.py) that take the
    place of B1 A1 / B2 A2."""
    h = x @ W1.T
    if D1 is not None:
        h = h + x @ D1.T
    elif A1 is not None and A1.shape[0] > 0:
        h = h + (x @ A1.T) @ B1.T
    z = silu(h[:, :N]) * h[:, N:]
    o = z @ W2.T
    if D2 is not None:
        o = o + z @ D2.T
    elif A2 is not None and A2.shape[0] > 0:
        o = o + (z @ A2.T) @ B2.T
    return o


def routed_jobs(X: np.ndarray, logits: np.ndarray, top_k: int, E: int, renorm: bool = True,
                rows: Optional[Sequence[int]] = None, comp_top_n: int = 0) -> Dict:
    """Steps 2-3 and the work list of step 4: routing, bucketing, and per
    expert the bucket rows p whose token is wanted, split into those that get
    the compensator and those that do not (``comp_top_n`` > 0 compensates only
    the first n routing slots of each token: Bandwidth-Efficient Adaptive
    Mixture-of-Experts via Low-Rank Compensation, abstract, Top-n (n < k)
    compensation)."""
    T = np.asarray(X).shape[0]
    idx, w = route(logits, top_k, renorm)
    counts, offsets, perm, inv = bucket(idx, E)
    want = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    wanted = set(int(t) for t in want)
    slot = {int(inv[t, j]): j for t in range(T) for j in range(top_k)}
    jobs = []
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        ps = [p for p in range(lo, hi) if int(perm[p]) in wanted]
        if not ps:
            continue
        comp = [p for p in ps if comp_top_n <= 0 or slot[p] < comp_top_n]
        plain = [p for p in ps if not (comp_top_n <= 0 or slot[p] < comp_top_n)]
        jobs.append((e, comp, plain))
    return {"idx": idx, "w": w, "counts": counts, "offsets": offsets, "perm_token": perm, "inv_pos": inv,
            "want": want, "jobs": jobs}


def expert_job(X: np.ndarray, perm: np.ndarray, ex: Dict, N: int, comp: Sequence[int],
               plain: Sequence[int]) -> Dict[int, np.ndarray]:
    """Step 4 for one expert: the outputs o of its bucket rows p (rows in
    ``comp`` with the compensators, rows in ``plain`` without)."""
    X64 = np.asarray(X, np.float64)
    O = {}
    if comp:
        o = expert_ffn(X64[perm[list(comp)]], ex["W1"], ex["W2"], N, ex.get("A1"), ex.get("B1"), ex.get("A2"),
                       ex.get("B2"), ex.get("D1"), ex.get("D2"))
        for i, p in enumerate(comp):
            O[p] = o[i]
    if plain:
        o = expert_ffn(X64[perm[list(plain)]], ex["W1"], ex["W2"], N)
        for i, p in enumerate(plain):
            O[p] = o[i]
    return O


def combine(want: Sequence[int], w: np.ndarray, inv: np.ndarray, O: Dict[int, np.ndarray], K: int) -> np.ndarray:
    """Step 5: y_t = sum_j w[t, j] * o_(t, j), slots in order."""
    Y = np.zeros((len(want), K), np.float64)
    for i, t in enumerate(want):
        for j in range(w.shape[1]):
            Y[i] += w[t, j] * O[int(inv[t, j])]
    return Y


def moe_forward(X: np.ndarray, logits: np.ndarray, top_k: int,
                expert: Callable[[int], Dict], N: int, renorm: bool = True,
                rows: Optional[Sequence[int]] = None, comp_top_n: int = 0) -> Dict:
    """The layer's forward pass: routed_jobs, then expert_job for every expert
    that holds a wanted row, then combine.

    ``expert(e)`` returns a dict with fp64 arrays W1 [2N, K], W2 [K, N] and
    optional A1, B1, A2, B2, or dense compensators D1 [2N, K], D2 [K, N] (it
    is called only for experts that receive wanted rows). ``rows`` restricts
    the output to those tokens (routing and bucketing are still computed for
    all tokens). Returns a dict with Y fp64 ([T, K] or [len(rows), K]) and the
    routing arrays.
    """
    X64 = np.asarray(X, np.float64)
    E = np.asarray(logits).shape[1]
    r = routed_jobs(X64, logits, top_k, E, renorm, rows, comp_top_n)
    O = {}
    for e, comp, plain in r["jobs"]:
        O.update(expert_job(X64, r["perm_token"], expert(e), N, comp, plain))
    Y = combine(r["want"], r["w"], r["inv_pos"], O, X64.shape[1])
    return {"Y": Y, "idx": r["idx"], "w": r["w"], "counts": r["counts"], "offsets": r["offsets"],
            "perm_token": r["perm_token"], "inv_pos": r["inv_pos"]}


# ----------------------------------------------------------------------------
# compensator construction (offline; MiLo abstract, low-rank compensation of
# the quantisation residual)
# ----------------------------------------------------------------------------

def svd_compensator(R: np.ndarray, rank: int) -> Tuple[np.ndarray, np.ndarray]:
    """Rank-r factors of the residual R = W - W^ [M, K]: R ~ B A with
    B = U_r S_r^(1/2) [M, r], A = S_r^(1/2) V_r^T [r, K] (balanced split)."""
    U, S, Vt = np.linalg.svd(np.asarray(R, np.float64), full_matrices=False)
    root = np.sqrt(S[:rank])
    return root[:, None] * Vt[:rank], U[:, :rank] * root[None, :]
