"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
examples (tests/golden/format_examples.json), an independent packer (the
input generator), closed forms (SVD / Eckart-Young), textbook constants, the
round-to-nearest error bound, invariants and brute force.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle as orc

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "format_examples.json")))


# --------------------------------------------------------------------------- O1

def test_int3_pack_hand_example():
    ex = GOLD["int3_pack"]
    codes = np.array([ex["codes"]], np.uint8)
    assert orc.unpack_int_rows(np.array([ex["bytes"]], np.uint8), 3, 8).tolist() == [ex["codes"]]
    assert orc.pack_int_rows(codes, 3).tolist() == [ex["bytes"]]


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("K", [32, 64, 96, 1408])
def test_pack_unpack_roundtrip(bits, K):
    g = np.random.default_rng([bits, K])
    q = g.integers(0, 1 << bits, size=(5, K)).astype(np.uint8)
    # the generator's packer (bit expansion) against the oracle's unpacker (byte windows)
    packed_gen = ms.pack_int_rows(torch.from_numpy(q), bits).numpy()
    assert np.array_equal(orc.unpack_int_rows(packed_gen, bits, K), q)
    # the oracle's own packer both ways
    packed = orc.pack_int_rows(q, bits)
    assert np.array_equal(packed, packed_gen)
    assert np.array_equal(orc.unpack_int_rows(packed, bits, K), q)
    raw = g.integers(0, 256, size=(3, K * bits // 8)).astype(np.uint8)
    assert np.array_equal(orc.pack_int_rows(orc.unpack_int_rows(raw, bits, K), bits), raw)


def test_bitplane_hand_example():
    ex = GOLD["bitplane"]
    planes = np.array(ex["planes_u32"], np.uint32).reshape(4, 1, 1)
    c4 = orc.bitplane_codes(planes, 4)[0]
    assert c4.tolist() == [i % 16 for i in range(32)]
    lut = np.array(ex["lut28"], np.float16)
    w2 = orc.dequant_bitplane(planes, lut, 2)[0]
    assert w2[:8].tolist() == ex["b2_values_elements_0_to_7"]
    assert orc.dequant_bitplane(planes, lut, 3)[0, 13] == ex["b3_value_element_13"]
    assert orc.dequant_bitplane(planes, lut, 4)[0, 29] == ex["b4_value_element_29"]
    # the generator writes the same planes for the same codes
    gen = ms.pack_bitplanes(torch.tensor([[i % 16 for i in range(32)]], dtype=torch.uint8)).numpy()
    assert np.array_equal(gen.view(np.uint32).reshape(4), np.array(ex["planes_u32"], np.uint32))


@pytest.mark.parametrize("K", [32, 96, 256])
def test_bitplane_roundtrip(K):
    g = np.random.default_rng(K)
    c4 = g.integers(0, 16, size=(6, K)).astype(np.uint8)
    planes = ms.pack_bitplanes(torch.from_numpy(c4)).numpy()
    assert np.array_equal(orc.bitplane_codes(planes, 4), c4)
    for b in (2, 3):
        assert np.array_equal(orc.bitplane_codes(planes, b), c4 >> (4 - b))


def test_int_dequant_hand_example():
    ex = GOLD["int_dequant"]
    w = orc.dequant_int(np.array(ex["q"], np.uint8), np.array(ex["s"], np.float16),
                        np.array(ex["z"], np.float16), ex["group"])
    assert w.tolist() == ex["w"]


# --------------------------------------------------------------------------- O8

@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (4, 64), (4, 32)])
def test_rtn_error_bound(bits, group):
    """Every element not clamped to the code range dequantises to within half a
    step (+ fp16 slack) of the original weight; a wrong group index, a swapped
    scale/zero or a sign error breaks this."""
    W = ms.gaussian((48, 512), 0.02, [9, bits, group])
    q, s, z = ms.rtn_int_asym(W, bits, group)
    packed = ms.pack_int_rows(q, bits).numpy()
    qo = orc.unpack_int_rows(packed, bits, 512)
    assert qo.max() <= (1 << bits) - 1
    what = orc.dequant_int(qo, s.numpy(), z.numpy(), group)
    gi = np.arange(512) // group
    s64 = s.numpy().astype(np.float64)[:, gi]
    z64 = z.numpy().astype(np.float64)[:, gi]
    W64 = W.numpy().astype(np.float64)
    interior = (np.round(W64 / s64) + z64 >= 0) & (np.round(W64 / s64) + z64 <= (1 << bits) - 1)
    err = np.abs(W64 - what)
    assert interior.mean() > 0.95
    assert np.all(err[interior] <= 0.5 * s64[interior] * (1 + 1e-9) + 1e-12)
    # clamped elements sit at most one step (+ the fp16 rounding of s) beyond
    assert np.all(err <= 1.6 * s64)


def test_bitplane_lut_error_bound():
    """LUT_4[c] is the mean of its bucket, so each weight lies within one
    bucket width of its dequantised value (fp16 slack)."""
    W = ms.gaussian((64, 256), 0.02, [10])
    code4, lut = ms.bitplane_quantize(W)
    planes = ms.pack_bitplanes(code4).numpy()
    W64 = W.numpy().astype(np.float64)
    step = (W64.max() - W64.min()) / 16
    for b in (2, 3, 4):
        what = orc.dequant_bitplane(planes, lut.numpy(), b)
        width = step * (1 << (4 - b))
        assert np.max(np.abs(W64 - what)) <= width * 1.001 + 1e-6
    # the error shrinks with more planes
    errs = [np.linalg.norm(W64 - orc.dequant_bitplane(planes, lut.numpy(), b)) for b in (2, 3, 4)]
    assert errs[0] > errs[1] > errs[2]


# --------------------------------------------------------------------------- routing

def test_routing_hand_example():
    ex = GOLD["routing"]
    L = np.array(ex["logits"], np.float32)
    idx, w = orc.route(L, 2)
    assert idx.tolist() == ex["idx"]
    assert np.allclose(w, ex["w"], rtol=0, atol=1e-15)
    idx3, w3 = orc.route(L, 3)
    assert idx3.tolist() == ex["top3_idx"]
    assert np.allclose(w3, ex["top3_w"], rtol=0, atol=1e-10)


def test_routing_full_softmax_flag():
    L = np.array([[0.0, 1.0, 2.0]], np.float32)
    idx, w = orc.route(L, 1, renorm=False)
    assert idx.tolist() == [[2]]
    # softmax([0,1,2])[2] = e^2 / (1 + e + e^2)
    assert abs(w[0, 0] - math.exp(2) / (1 + math.e + math.exp(2))) < 1e-15
    _, w1 = orc.route(L, 1, renorm=True)
    assert w1[0, 0] == 1.0


def test_bucket_against_sort():
    g = np.random.default_rng(3)
    T, E, k = 40, 7, 3
    idx = np.stack([g.permutation(E)[:k] for _ in range(T)])
    counts, offsets, perm, inv = orc.bucket(idx, E)
    assert np.array_equal(counts, np.bincount(idx.reshape(-1), minlength=E))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    tt, jj = np.meshgrid(np.arange(T), np.arange(k), indexing="ij")
    order = np.lexsort((tt.reshape(-1), idx.reshape(-1)))
    assert np.array_equal(perm, tt.reshape(-1)[order])
    for p, o in enumerate(order):
        assert inv[tt.reshape(-1)[o], jj.reshape(-1)[o]] == p


# --------------------------------------------------------------------------- FFN (O5)

def test_swiglu_ffn_hand_example():
    ex = GOLD["swiglu_ffn"]
    x = np.array([ex["x"]], np.float64)
    W1 = np.array(ex["W1_rows"], np.float64)
    W2 = np.array(ex["W2_rows"], np.float64)
    o = orc.expert_ffn(x, W1, W2, ex["N"])
    assert np.allclose(o[0], ex["o_no_comp"], rtol=0, atol=1e-15)
    o2 = orc.expert_ffn(x, W1, W2, ex["N"], np.array(ex["A1"], np.float64), np.array(ex["B1"], np.float64))
    assert np.allclose(o2[0], ex["o_with_comp"], rtol=0, atol=1e-15)
    o3 = orc.expert_ffn(x, W1, W2, ex["N"], None, None, np.array(ex["A2"], np.float64), np.array(ex["B2"], np.float64))
    assert np.allclose(o3[0], ex["o_with_comp2"], rtol=0, atol=1e-15)


def test_top1_equals_single_expert():
    """Top-1 routing with renormalised weight 1 gives one expert's FFN per token."""
    g = np.random.default_rng(5)
    T, E, K, N = 9, 3, 16, 8
    ex = {e: {"W1": g.normal(size=(2 * N, K)), "W2": g.normal(size=(K, N))} for e in range(E)}
    X = g.normal(size=(T, K))
    L = g.normal(size=(T, E)).astype(np.float32)
    out = orc.moe_forward(X, L, 1, lambda e: ex[e], N)
    assert np.all(out["w"] == 1.0)
    for t in range(T):
        e = int(np.argmax(L[t]))
        x = X[t]
        h = ex[e]["W1"] @ x
        z = h[:N] / (1 + np.exp(-h[:N])) * h[N:]
        assert np.allclose(out["Y"][t], ex[e]["W2"] @ z, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- O3 / O4 (SVD)

def _tiny_block(bits=4, group=64, M=64, K=128, seed=11):
    W = ms.gaussian((M, K), 0.02, [seed])
    q, s, z = ms.rtn_int_asym(W, bits, group)
    what = orc.dequant_int(q.numpy(), s.numpy(), z.numpy(), group)
    return W.numpy().astype(np.float64), what


def test_full_rank_svd_compensator_reconstructs():
    W, what = _tiny_block()
    R = W - what
    A, B = orc.svd_compensator(R, min(R.shape))
    rel = np.linalg.norm(W - (what + B @ A)) / np.linalg.norm(W)
    assert rel <= 1e-10


def test_truncated_svd_eckart_young():
    W, what = _tiny_block()
    R = W - what
    r = 8
    A, B = orc.svd_compensator(R, r)
    err = np.linalg.norm(R - B @ A)
    assert err < np.linalg.norm(R)
    # tail energy from the eigenvalues of R R^T (a different routine than the SVD)
    lam = np.sort(np.linalg.eigvalsh(R @ R.T))[::-1]
    tail = math.sqrt(max(lam[r:].sum(), 0.0))
    assert abs(err - tail) / tail < 1e-10
    # optimality against random rank-r factors
    g = np.random.default_rng(0)
    for _ in range(3):
        Br, Ar = g.normal(size=B.shape) * 0.01, g.normal(size=A.shape) * 0.01
        assert err <= np.linalg.norm(R - Br @ Ar)
    # balanced split: matching column / row norms
    assert np.allclose(np.linalg.norm(B, axis=0), np.linalg.norm(A, axis=1), rtol=1e-10)


# --------------------------------------------------------------------------- O2 / O6 / O7

def _brute_force(X, L, k, experts, N, renorm=True, comp_top_n=0):
    """Every expert on every token, combined with a 0/1 selection mask; the
    selection uses a stable argsort (no bucketing, no permutation). With
    comp_top_n > 0 only the experts ranked below n keep their compensators."""
    T = X.shape[0]
    E = L.shape[1]
    Y = np.zeros_like(X, dtype=np.float64)
    for t in range(T):
        order = np.argsort(-L[t].astype(np.float64), kind="stable")[:k]
        sel = np.zeros(E, bool)
        sel[order] = True
        rank = {int(e): j for j, e in enumerate(order)}
        p = np.exp(L[t].astype(np.float64) - L[t].astype(np.float64).max())
        wts = p * sel / ((p * sel).sum() if renorm else p.sum())
        for e in range(E):
            ex = experts[e]
            use = comp_top_n <= 0 or rank.get(e, k) < comp_top_n
            o = orc.expert_ffn(X[t:t + 1], ex["W1"], ex["W2"], N, ex.get("A1") if use else None,
                               ex.get("B1") if use else None, ex.get("A2") if use else None,
                               ex.get("B2") if use else None)[0]
            Y[t] += wts[e] * o
    return Y


def _quantized_experts(E, K, N, bits, group, rank, seed):
    cfg = ms.LayerConfig(99, "t", E, 2, K, N, (8,),
                         [ms.ExpertSpec(ms.FMT_INT_ASYM, (bits, bits), group, rank) for _ in range(E)])
    cfg.cid = seed
    experts = {}
    for e in range(E):
        d = {}
        for b, nm in ((0, "1"), (1, "2")):
            blk = ms.make_block(cfg, e, b)
            d["W" + nm] = orc.dequant_block({"fmt": 0, "bits": bits, "group": group, "K_in": blk.K_in,
                                             "codes": blk.codes.numpy(), "scales": blk.scales.numpy(),
                                             "zeros_or_lut": blk.zeros_or_lut.numpy()})
            if rank:
                d["A" + nm] = blk.A.float().numpy().astype(np.float64)
                d["B" + nm] = blk.B.float().numpy().astype(np.float64)
        experts[e] = d
    return experts


@pytest.mark.parametrize("k,renorm", [(1, True), (2, True), (3, False)])
def test_brute_force_agrees(k, renorm):
    E, K, N, T = 4, 64, 64, 8
    experts = _quantized_experts(E, K, N, 3, 32, 4, 21)
    g = np.random.default_rng(7)
    X = g.normal(size=(T, K))
    L = g.normal(size=(T, E)).astype(np.float32)
    out = orc.moe_forward(X, L, k, lambda e: experts[e], N, renorm=renorm)
    Yb = _brute_force(X, L, k, experts, N, renorm)
    assert np.max(np.abs(out["Y"] - Yb)) <= 1e-13 * max(1.0, np.max(np.abs(Yb)))


@pytest.mark.parametrize("n", [1, 2])
def test_top_n_compensation_brute_force(n):
    """Compensators only on the first n routing slots (BEAM abstract)."""
    E, K, N, T, k = 4, 64, 64, 7, 3
    experts = _quantized_experts(E, K, N, 3, 32, 8, 51)
    g = np.random.default_rng(12)
    X = g.normal(size=(T, K))
    L = g.normal(size=(T, E)).astype(np.float32)
    out = orc.moe_forward(X, L, k, lambda e: experts[e], N, comp_top_n=n)
    Yb = _brute_force(X, L, k, experts, N, comp_top_n=n)
    assert np.max(np.abs(out["Y"] - Yb)) <= 1e-13 * max(1.0, np.max(np.abs(Yb)))
    full = orc.moe_forward(X, L, k, lambda e: experts[e], N)["Y"]
    assert np.max(np.abs(out["Y"] - full)) > 1e-6  # the compensators do matter here
    same = orc.moe_forward(X, L, k, lambda e: experts[e], N, comp_top_n=k)["Y"]
    assert np.array_equal(same, full)


def test_dense16_rank0_is_dense_matmul():
    """bits = 16 (stored bf16 weights), rank 0: the bucketed layer equals the
    dense computation with the same weights, on every token."""
    E, K, N, T = 3, 32, 32, 6
    g = np.random.default_rng(8)
    experts = {}
    for e in range(E):
        W1 = torch.from_numpy(g.normal(scale=0.1, size=(2 * N, K))).to(torch.bfloat16)
        W2 = torch.from_numpy(g.normal(scale=0.1, size=(K, N))).to(torch.bfloat16)
        experts[e] = {"W1": orc.dequant_block({"fmt": 2, "codes": W1.float().numpy()}),
                      "W2": orc.dequant_block({"fmt": 2, "codes": W2.float().numpy()})}
    X = g.normal(size=(T, K))
    L = g.normal(size=(T, E)).astype(np.float32)
    out = orc.moe_forward(X, L, 2, lambda e: experts[e], N)
    Yb = _brute_force(X, L, 2, experts, N)
    assert np.max(np.abs(out["Y"] - Yb)) <= 1e-13 * max(1.0, np.max(np.abs(Yb)))


def test_token_permutation_invariance():
    E, K, N, T = 4, 64, 64, 10
    experts = _quantized_experts(E, K, N, 4, 64, 8, 31)
    g = np.random.default_rng(9)
    X = g.normal(size=(T, K))
    L = g.normal(size=(T, E)).astype(np.float32)
    Y = orc.moe_forward(X, L, 2, lambda e: experts[e], N)["Y"]
    pi = g.permutation(T)
    Yp = orc.moe_forward(X[pi], L[pi], 2, lambda e: experts[e], N)["Y"]
    assert np.max(np.abs(Yp - Y[pi])) <= 1e-13 * np.max(np.abs(Y))


def test_rows_subset_matches_full():
    E, K, N, T = 4, 64, 64, 10
    experts = _quantized_experts(E, K, N, 2, 64, 0, 41)
    g = np.random.default_rng(10)
    X = g.normal(size=(T, K))
    L = g.normal(size=(T, E)).astype(np.float32)
    full = orc.moe_forward(X, L, 2, lambda e: experts[e], N)["Y"]
    part = orc.moe_forward(X, L, 2, lambda e: experts[e], N, rows=[7, 2])["Y"]
    # BLAS may block a batch differently: equal up to fp64 rounding
    assert np.max(np.abs(part - full[[7, 2]])) <= 1e-13 * np.max(np.abs(full))
