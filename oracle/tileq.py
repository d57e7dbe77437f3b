"""Plain fp64 restatement of the 2D-tiled shared low-rank compensator.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` (and through them nothing
else); the CUDA library shares no code with it.

TileQ: Efficient Low-Rank Quantization of Mixture-of-Experts with 2D Tiling,
abstract: the experts' low-rank factors are shared across both the input and
the output dimension through a 2D tiling of the weight matrices, and the
experts' low-rank terms are evaluated together in one pass.

Reading where the page is silent (the page gives the abstract only): one
block type (W1 = [gate; up], or W2) of all E experts is cut
into P x Q tiles of tile_m rows x tile_k columns. The output-side factor U_p
[tile_m, r] of row tile p is shared by every column tile and every expert;
the input-side factor V_q [r, tile_k] of column tile q is shared by every row
tile and every expert; what belongs to one expert and one tile is an r x r
core C[e, p, q]. Expert e's compensator on tile (p, q) is U_p C[e, p, q] V_q,
so that W^_e + dW_e replaces W^_e + B_e A_e. U is stored as the stack of the
U_p [M, r] and V as the concatenation of the V_q [r, K_in].

Pins (tests/test_tileq_oracle.py): identity cores reduce it to the plain
rank-r product U V; a single nonzero core changes exactly its own tile; the
Kronecker identity vec(U_p C V_q) = (V_q^T kron U_p) vec(C); brute force element
by element on tiny shapes.
"""
from __future__ import annotations

import numpy as np


def tileq_delta(U: np.ndarray, V: np.ndarray, cores_e: np.ndarray, tile_m: int, tile_k: int) -> np.ndarray:
    """Dense compensator dW [M, K_in] of one expert: tile (p, q) = U_p C[p, q] V_q.

    U [M, r], V [r, K_in], cores_e [P, Q, r, r] (the expert's cores), fp64."""
    U = np.asarray(U, np.float64)
    V = np.asarray(V, np.float64)
    C = np.asarray(cores_e, np.float64)
    M, r = U.shape
    K = V.shape[1]
    P, Q = M // tile_m, K // tile_k
    assert P * tile_m == M and Q * tile_k == K and C.shape == (P, Q, r, r)
    D = np.zeros((M, K), np.float64)
    for p in range(P):
        rows = slice(p * tile_m, (p + 1) * tile_m)
        for q in range(Q):
            cols = slice(q * tile_k, (q + 1) * tile_k)
            D[rows, cols] = U[rows] @ C[p, q] @ V[:, cols]
    return D


def factor_elements(M: int, K: int, E: int, r: int, tile_m: int, tile_k: int) -> int:
    """Stored numbers of one block type: U, V and the cores of all experts."""
    return M * r + r * K + E * (M // tile_m) * (K // tile_k) * r * r
