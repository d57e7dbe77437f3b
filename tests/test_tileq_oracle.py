"""Pins of the 2D-tiled shared low-rank compensator oracle (TileQ: Efficient
Low-Rank Quantization of Mixture-of-Experts with 2D Tiling, abstract: factors
shared across the input and output dimensions of the experts by 2D tiling).

Each pin checks the oracle against something other than its own formula: the
plain rank-r product it must reduce to, the support a single core must have, a
Kronecker-product identity evaluated by ``np.kron``, brute force element by
element, and the layer forward through the factored (A, B) path."""
import numpy as np

from oracle import moe_oracle as mo
from oracle import tileq as tq


def _factors(rng, M, K, r, E, tile_m, tile_k):
    U = rng.standard_normal((M, r))
    V = rng.standard_normal((r, K))
    C = rng.standard_normal((E, M // tile_m, K // tile_k, r, r))
    return U, V, C


def test_identity_cores_reduce_to_plain_low_rank():
    rng = np.random.default_rng(1)
    M, K, r = 12, 10, 3
    U, V, _ = _factors(rng, M, K, r, 1, 4, 5)
    I = np.broadcast_to(np.eye(r), (3, 2, r, r))
    np.testing.assert_allclose(tq.tileq_delta(U, V, I, 4, 5), U @ V, rtol=0, atol=1e-12)


def test_single_core_changes_only_its_tile():
    rng = np.random.default_rng(2)
    M, K, r, tm, tk = 12, 8, 2, 4, 4  # P = 3 row tiles, Q = 2 column tiles (P != Q catches swapped indices)
    U, V, C = _factors(rng, M, K, r, 1, tm, tk)
    for p0, q0 in [(2, 0), (0, 1), (1, 1)]:
        Z = np.zeros_like(C[0])
        Z[p0, q0] = C[0, p0, q0]
        D = tq.tileq_delta(U, V, Z, tm, tk)
        mask = np.zeros((M, K), bool)
        mask[p0 * tm:(p0 + 1) * tm, q0 * tk:(q0 + 1) * tk] = True
        assert np.all(D[~mask] == 0.0)
        assert np.count_nonzero(D[mask]) == mask.sum()


def test_kronecker_identity_per_tile():
    # vec(U_p C V_q) = (V_q^T kron U_p) vec(C), vec stacking columns
    rng = np.random.default_rng(3)
    M, K, r, tm, tk = 9, 8, 3, 3, 4
    U, V, C = _factors(rng, M, K, r, 1, tm, tk)
    D = tq.tileq_delta(U, V, C[0], tm, tk)
    for p in range(M // tm):
        for q in range(K // tk):
            Up = U[p * tm:(p + 1) * tm]
            Vq = V[:, q * tk:(q + 1) * tk]
            want = np.kron(Vq.T, Up) @ C[0, p, q].reshape(-1, order="F")
            got = D[p * tm:(p + 1) * tm, q * tk:(q + 1) * tk].reshape(-1, order="F")
            np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_brute_force_elementwise():
    rng = np.random.default_rng(4)
    M, K, r, tm, tk = 6, 6, 2, 2, 3
    U, V, C = _factors(rng, M, K, r, 1, tm, tk)
    D = tq.tileq_delta(U, V, C[0], tm, tk)
    for m in range(M):
        for k in range(K):
            s = 0.0
            for i in range(r):
                for j in range(r):
                    s += U[m, i] * C[0, m // tm, k // tk, i, j] * V[j, k]
            assert abs(D[m, k] - s) < 1e-12


def test_experts_differ_only_through_their_cores():
    rng = np.random.default_rng(5)
    M, K, r, tm, tk = 8, 8, 2, 4, 4
    U, V, C = _factors(rng, M, K, r, 2, tm, tk)
    C[1] = C[0]
    C[1, 1, 0] += np.eye(r)
    D0 = tq.tileq_delta(U, V, C[0], tm, tk)
    D1 = tq.tileq_delta(U, V, C[1], tm, tk)
    diff = D1 - D0
    assert np.all(diff[:4] == 0.0) and np.all(diff[4:, 4:] == 0.0)
    np.testing.assert_allclose(diff[4:, :4], U[4:] @ V[:, :4], atol=1e-12)


def test_layer_forward_with_identity_cores_equals_factored_path():
    # a layer whose TileQ cores are identities must equal the same layer with
    # per-expert compensators B = U, A = V (the factored path of the oracle)
    rng = np.random.default_rng(6)
    E, K, N, T, k, r = 3, 8, 8, 5, 2, 2
    W1 = rng.standard_normal((E, 2 * N, K)) * 0.3
    W2 = rng.standard_normal((E, K, N)) * 0.3
    U1, V1 = rng.standard_normal((2 * N, r)) * 0.2, rng.standard_normal((r, K)) * 0.2
    U2, V2 = rng.standard_normal((K, r)) * 0.2, rng.standard_normal((r, N)) * 0.2
    I1 = np.broadcast_to(np.eye(r), (2 * N // 4, K // 4, r, r))
    I2 = np.broadcast_to(np.eye(r), (K // 4, N // 4, r, r))
    X = rng.standard_normal((T, K))
    logits = rng.standard_normal((T, E))

    def tiled(e):
        return {"W1": W1[e], "W2": W2[e], "D1": tq.tileq_delta(U1, V1, I1, 4, 4),
                "D2": tq.tileq_delta(U2, V2, I2, 4, 4)}

    def factored(e):
        return {"W1": W1[e], "W2": W2[e], "A1": V1, "B1": U1, "A2": V2, "B2": U2}

    a = mo.moe_forward(X, logits, k, tiled, N)["Y"]
    b = mo.moe_forward(X, logits, k, factored, N)["Y"]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_factor_count_closed_form():
    # Mixtral-shaped W1 (2*14336 x 4096), 8 experts, r = 32, 1024 x 1024 tiles
    n = tq.factor_elements(2 * 14336, 4096, 8, 32, 1024, 1024)
    assert n == 2 * 14336 * 32 + 32 * 4096 + 8 * 28 * 4 * 32 * 32
    per_expert = 8 * (2 * 14336 + 4096) * 32
    assert per_expert / n > 4.0


def test_top_n_with_tiled_compensators_matches_factored_path():
    # top-n compensation (only the first n routing slots compensated) must
    # treat the dense tiled form exactly as the factored (A, B) form
    rng = np.random.default_rng(7)
    E, K, N, T, k, r = 4, 8, 8, 6, 3, 2
    W1 = rng.standard_normal((E, 2 * N, K)) * 0.3
    W2 = rng.standard_normal((E, K, N)) * 0.3
    U1, V1 = rng.standard_normal((2 * N, r)), rng.standard_normal((r, K))
    U2, V2 = rng.standard_normal((K, r)), rng.standard_normal((r, N))
    I1 = np.broadcast_to(np.eye(r), (2 * N // 4, K // 4, r, r))
    I2 = np.broadcast_to(np.eye(r), (K // 4, N // 4, r, r))
    X = rng.standard_normal((T, K))
    logits = rng.standard_normal((T, E))

    def tiled(e):
        return {"W1": W1[e], "W2": W2[e], "D1": tq.tileq_delta(U1, V1, I1, 4, 4),
                "D2": tq.tileq_delta(U2, V2, I2, 4, 4)}

    def factored(e):
        return {"W1": W1[e], "W2": W2[e], "A1": V1, "B1": U1, "A2": V2, "B2": U2}

    for n in (1, 2):
        a = mo.moe_forward(X, logits, k, tiled, N, comp_top_n=n)["Y"]
        b = mo.moe_forward(X, logits, k, factored, N, comp_top_n=n)["Y"]
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    full = mo.moe_forward(X, logits, k, tiled, N)["Y"]
    assert np.max(np.abs(full - mo.moe_forward(X, logits, k, tiled, N, comp_top_n=1)["Y"])) > 1e-3
