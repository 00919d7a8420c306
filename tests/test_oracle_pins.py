"""Pins that tie the CPU oracle to what the pages and the mathematics fix.

Each pin is independent of the oracle's own formulas: worked examples and
counts the pages print (``tests/golden/``), algebraic invariants
(associativity, unit, composition), special cases that reduce to a library
routine (q = 1 is numpy's matmul), and brute force on tiny inputs.  The
mutation tests at the end plant plausible mistakes in the oracle, on the CPU,
and check that at least one pin catches each of them.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest

import oracle
from associative_algebra_block_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_blocks(name):
    out, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line[0].isalpha():
                cur = line
                out[cur] = []
            else:
                out[cur].append([float(v) for v in line.split()])
    return {k: np.array(v) for k, v in out.items()}


def _read_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# --------------------------------------------------------------------------
# Worked example and counts from the pages
# --------------------------------------------------------------------------

def test_q2_scalar_worked_example():
    g = _read_blocks("q2_scalar_example.txt")
    Z = oracle.square_product("Q", 2, g["X"], g["W"])
    assert np.array_equal(Z, g["Z"])
    # the dense product differs exactly by the two edge*edge terms
    assert np.array_equal(g["X"] @ g["W"], g["DENSE"])
    removed = g["DENSE"] - Z
    assert removed[0, 0] == g["X"][0, 1] * g["W"][1, 0]
    assert removed[1, 1] == g["X"][1, 0] * g["W"][0, 1]
    assert removed[0, 1] == 0 and removed[1, 0] == 0


def test_q2_removed_products_are_the_edge_cycle():
    # Of the 8 dense block products X_ia W_ak at q = 2, exactly the two
    # edge*edge ones (a != i and a != k) are missing.
    S = oracle.block_table("Q", 2)
    kept = {(i, a, k) for i in range(2) for k in range(2) for a in S[i][k]}
    dense = {(i, a, k) for i in range(2) for k in range(2) for a in range(2)}
    assert dense - kept == {(0, 1, 0), (1, 0, 1)}
    assert len(kept) == 6


@pytest.mark.parametrize("row", _read_rows("counts.txt"))
def test_block_product_counts(row):
    law, q, per_row, square = row[0], int(row[1]), int(row[2]), int(row[3])
    assert oracle.block_product_count(law, q, row_typed=True) == per_row
    assert oracle.block_product_count(law, q, row_typed=False) == square
    S = oracle.block_table(law, q)
    # every row type performs the same number of block products
    for i in range(q):
        assert sum(len(S[i][k]) for k in range(q)) == per_row
    assert math.isclose(oracle.mac_ratio(law, q), per_row / (q * q))


def test_alder_strassen_bound_is_met():
    for q, m, v, bound in (map(int, r) for r in _read_rows("alder_strassen.txt")):
        # m: slots of the algebra (basis elements that ever appear), v: vertices
        slots = {(i, k) for i in range(q) for k in range(q)
                 for a in range(q) if oracle.basis_product("Q", q, (i, a), (a, k))}
        verts = {(i, i) for i in range(q)
                 if oracle.basis_product("Q", q, (i, i), (i, i)) == (i, i)}
        assert len(slots) == m and len(verts) == v
        assert 2 * m - v == bound == oracle.block_product_count("Q", q, False)


def test_tensor_square_has_16_coordinates_and_is_not_q4():
    # 16 coordinates (basis slots) for Q2 (x) Q2
    slots = {(i, k) for i in range(4) for k in range(4)
             for a in range(4) if oracle.basis_product("Q2xQ2", 4, (i, a), (a, k))}
    assert len(slots) == 16
    # not isomorphic to Q4: different numbers of block products
    assert oracle.block_product_count("Q", 4, False) == 28
    assert oracle.block_product_count("Q2xQ2", 4, False) == 36
    assert oracle.mac_ratio("Q2xQ2", 4) == 9 / 16
    assert oracle.mac_ratio("Q", 4) == 7 / 16


def test_tensor_square_table_is_product_of_factor_tables():
    # Closed form of the tensor square: S((i1,i2),(k1,k2)) = S(i1,k1) x S(i2,k2)
    S2 = oracle.block_table("Q", 2)
    S4 = oracle.block_table("Q2xQ2", 4)
    for i in range(4):
        for k in range(4):
            expect = sorted(2 * a1 + a2 for a1 in S2[i // 2][k // 2] for a2 in S2[i % 2][k % 2])
            assert list(S4[i][k]) == expect


# --------------------------------------------------------------------------
# Algebraic invariants, bit-exact on small integers
# --------------------------------------------------------------------------

LAW_CASES = [("Q", 1), ("Q", 2), ("Q", 3), ("Q", 4), ("Q2xQ2", 4)]


def _int_mats(n, seed, count=3):
    return [m.f64 for m in inputs.integer_square_inputs(n, count=count, seed=seed)]


@pytest.mark.parametrize("law,q", LAW_CASES)
def test_associativity_exact(law, q):
    # config 1's check: 2x2-block matrices of 16x16 integer blocks in [-3, 3]
    # (and the same for the other laws, block size 16)
    X, W, Z = _int_mats(16 * q, seed=q)
    left = oracle.square_product(law, q, oracle.square_product(law, q, X, W), Z)
    right = oracle.square_product(law, q, X, oracle.square_product(law, q, W, Z))
    assert np.array_equal(left, right)


@pytest.mark.parametrize("law,q", LAW_CASES)
def test_basis_associativity_exhaustive(law, q):
    # (e_a e_b) e_c == e_a (e_b e_c) on every triple of basis slots
    slots = [(i, j) for i in range(q) for j in range(q)]

    def mul(x, y):
        if x is None or y is None:
            return None
        return oracle.basis_product(law, q, x, y)

    for x in slots:
        for y in slots:
            xy = mul(x, y)
            for z in slots:
                assert mul(xy, z) == mul(x, mul(y, z))


@pytest.mark.parametrize("law,q", LAW_CASES)
def test_unit_exact(law, q):
    X = _int_mats(8 * q, seed=10 + q, count=1)[0]
    one = oracle.unit(q, 8)
    assert np.array_equal(oracle.square_product(law, q, X, one), X)
    assert np.array_equal(oracle.square_product(law, q, one, X), X)


def test_products_keep_outer_indices():
    # every nonzero basis product e_ij e_lk lands on slot (i, k); the tile
    # oracle for large q relies on this
    for law, q in LAW_CASES:
        for i in range(q):
            for j in range(q):
                for l in range(q):
                    for k in range(q):
                        s = oracle.basis_product(law, q, (i, j), (l, k))
                        assert s is None or s == (i, k)


def test_q1_is_dense_gemm():
    s = inputs.Stream(3)
    X = s.normal(7, 12, 1.0, "f32").f64
    W = s.normal(12, 5, 1.0, "f32").f64
    assert np.array_equal(oracle.project("Q", 1, np.zeros(7, np.int64), X, W), X @ W)


# --------------------------------------------------------------------------
# Row-typed projection
# --------------------------------------------------------------------------

@pytest.mark.parametrize("law,q", LAW_CASES)
def test_projection_rows_equal_square_row_blocks(law, q):
    # a token of type i is a row of block-row i of the square product
    b = 4
    X, W = _int_mats(b * q, seed=20 + q, count=2)
    types = np.arange(b * q) // b
    assert np.array_equal(oracle.project(law, q, types, X, W), oracle.square_product(law, q, X, W))


@pytest.mark.parametrize("law,q", LAW_CASES)
def test_projection_composition_closure(law, q):
    # Phi_{W2}(Phi_{W1}(X)) == Phi_{W1 * W2}(X), exact on integers
    b = 3
    X = inputs.Stream(30 + q).integers(11, b * q, -3, 3, "f32").f64
    W1, W2 = _int_mats(b * q, seed=40 + q, count=2)
    types = np.arange(11) % q
    lhs = oracle.project(law, q, types, oracle.project(law, q, types, X, W1), W2)
    rhs = oracle.project(law, q, types, X, oracle.square_product(law, q, W1, W2))
    assert np.array_equal(lhs, rhs)


def _masked_dense(S, q, t, W):
    """W with block (a, k) zeroed unless a is in S(t, k)."""
    din, dout = W.shape
    bi, bo = din // q, dout // q
    Wm = np.zeros_like(W)
    for k in range(q):
        for a in S[t][k]:
            Wm[a * bi:(a + 1) * bi, k * bo:(k + 1) * bo] = W[a * bi:(a + 1) * bi, k * bo:(k + 1) * bo]
    return Wm


@pytest.mark.parametrize("law,q,din,dout", [("Q", 2, 6, 4), ("Q", 3, 6, 9), ("Q2xQ2", 4, 8, 12), ("Q", 5, 10, 5)])
def test_projection_brute_force_masked_dense(law, q, din, dout):
    s = inputs.Stream(50)
    M = 13
    X = s.normal(M, din, 1.0, "f32").f64
    W = s.normal(din, dout, 1.0, "f32").f64
    types = s.labels(M, q)
    S = oracle.block_table(law, q)
    Y = oracle.project(law, q, types, X, W)
    for r in range(M):
        ref = np.zeros(dout)
        Wm = _masked_dense(S, q, types[r], W)
        for c in range(dout):
            ref[c] = sum(X[r, j] * Wm[j, c] for j in range(din))
        assert np.allclose(Y[r], ref, rtol=1e-13, atol=1e-13)


def test_mac_counter_matches_closed_form():
    for law, q, M, din, dout in (("Q", 4, 40, 16, 8), ("Q2xQ2", 4, 24, 8, 16), ("Q", 32, 64, 64, 32)):
        c = oracle.MacCounter()
        types = np.arange(M) % q
        X = np.ones((M, din))
        W = np.ones((din, dout))
        oracle.project(law, q, types, X, W, counter=c)
        per_row = {"Q": 2 * q - 1, "Q2xQ2": 9}[law]
        assert c.macs == M * (din // q) * (dout // q) * per_row


def test_row_locality_and_decode():
    # decoding computes only the new position's row: it equals that row of
    # the full-sequence projection, whatever the other rows hold
    s = inputs.Stream(60)
    q, L = 4, 24
    X = s.normal(L, 8, 1.0, "f32").f64
    W = s.normal(8, 12, 1.0, "f32").f64
    pos = inputs.packed_positions(L, L)
    full = oracle.project("Q2xQ2", q, oracle.row_types("Q2xQ2", q, pos), X, W)
    for p in (0, 5, 17, 23):
        one = oracle.decode("Q2xQ2", q, np.array([p]), X[p:p + 1], W)
        assert np.array_equal(one[0], full[p])
        X2 = X.copy()
        X2[np.arange(L) != p] = 99.0
        again = oracle.project("Q2xQ2", q, oracle.row_types("Q2xQ2", q, pos), X2, W)
        assert np.array_equal(again[p], full[p])


def test_row_types_q2_first_types_use_first_block_row():
    # hotpaper.ai summary: with q = 2 the two row types take block rows
    # (A, U) and (V, D) of X = [[A, U], [V, D]].  With type = position mod 2,
    # position 0 is the first type, position 1 the second.
    assert list(oracle.row_types("Q", 2, [0, 1, 2, 3])) == [0, 1, 0, 1]
    X = np.array([[1.0, 2.0], [3.0, 4.0]])   # rows: (A, U) and (V, D) with b = 1
    W = np.array([[5.0, 6.0], [7.0, 8.0]])
    Y = oracle.decode("Q", 2, np.array([0, 1]), X, W)
    assert np.array_equal(Y, oracle.square_product("Q", 2, X, W))


# --------------------------------------------------------------------------
# Backward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("law,q", LAW_CASES)
def test_backward_adjoint_identities_exact(law, q):
    # the projection is bilinear: <dY, f(X, W)> = <dX, X> = <dW, W>, exact on
    # integer inputs
    s = inputs.Stream(70 + q)
    M, din, dout = 19, 3 * q, 2 * q
    X = s.integers(M, din, -3, 3, "f32").f64
    W = s.integers(din, dout, -3, 3, "f32").f64
    dY = s.integers(M, dout, -3, 3, "f32").f64
    types = s.labels(M, q)
    Y = oracle.project(law, q, types, X, W)
    dX, dW = oracle.project_bwd(law, q, types, X, W, dY)
    lhs = float(np.sum(dY * Y))
    assert lhs == float(np.sum(dX * X)) == float(np.sum(dW * W))


@pytest.mark.parametrize("law,q", [("Q", 2), ("Q", 3), ("Q2xQ2", 4)])
def test_backward_brute_force(law, q):
    # per row: dx = dy Wm_t^T and dW = sum_r x_r^T dy_r restricted to the mask
    s = inputs.Stream(80)
    M, din, dout = 9, 2 * q, 3 * q
    X = s.normal(M, din, 1.0, "f32").f64
    W = s.normal(din, dout, 1.0, "f32").f64
    dY = s.normal(M, dout, 1.0, "f32").f64
    types = s.labels(M, q)
    S = oracle.block_table(law, q)
    dX, dW = oracle.project_bwd(law, q, types, X, W, dY)
    refW = np.zeros_like(W)
    for r in range(M):
        Wm = _masked_dense(S, q, types[r], W)
        mask = _masked_dense(S, q, types[r], np.ones_like(W))
        assert np.allclose(dX[r], Wm @ dY[r], rtol=1e-13, atol=1e-13)
        refW += np.outer(X[r], dY[r]) * mask
    assert np.allclose(dW, refW, rtol=1e-13, atol=1e-13)


def test_backward_finite_difference():
    s = inputs.Stream(90)
    law, q, M, din, dout = "Q", 3, 5, 6, 6
    X = s.normal(M, din, 1.0, "f32").f64
    W = s.normal(din, dout, 1.0, "f32").f64
    dY = s.normal(M, dout, 1.0, "f32").f64
    types = s.labels(M, q)
    dX, dW = oracle.project_bwd(law, q, types, X, W, dY)
    h = 1e-6
    for (r, c) in ((0, 0), (2, 5), (4, 3)):
        Xp = X.copy(); Xp[r, c] += h
        Xm = X.copy(); Xm[r, c] -= h
        fd = (np.sum(dY * oracle.project(law, q, types, Xp, W)) - np.sum(dY * oracle.project(law, q, types, Xm, W))) / (2 * h)
        assert abs(fd - dX[r, c]) < 1e-6
    for (r, c) in ((0, 1), (3, 3), (5, 0)):
        Wp = W.copy(); Wp[r, c] += h
        Wm = W.copy(); Wm[r, c] -= h
        fd = (np.sum(dY * oracle.project(law, q, types, X, Wp)) - np.sum(dY * oracle.project(law, q, types, X, Wm))) / (2 * h)
        assert abs(fd - dW[r, c]) < 1e-6


# --------------------------------------------------------------------------
# SwiGLU and its parts
# --------------------------------------------------------------------------

def test_silu_definition_points():
    z = np.array([0.0, 1.0, -1.0, 40.0, -40.0])
    got = oracle.silu(z)
    ref = [0.0, 1.0 / (1.0 + math.exp(-1.0)), -1.0 / (1.0 + math.exp(1.0)), 40.0, -40.0 * math.exp(-40.0) / (1.0 + math.exp(-40.0))]
    assert np.allclose(got, ref, rtol=1e-15, atol=1e-300)


def test_swiglu_q1_is_dense_swiglu():
    s = inputs.Stream(95)
    X = s.normal(6, 8, 1.0, "f32").f64
    Wg = s.normal(8, 12, 0.3, "f32").f64
    Wu = s.normal(8, 12, 0.3, "f32").f64
    Wd = s.normal(12, 8, 0.3, "f32").f64
    H, Y = oracle.swiglu("Q", 1, np.zeros(6, np.int64), X, Wg, Wu, Wd)
    G = X @ Wg
    Hd = G / (1.0 + np.exp(-G)) * (X @ Wu)
    assert np.allclose(H, Hd, rtol=1e-14) and np.allclose(Y, Hd @ Wd, rtol=1e-13)


def test_swiglu_rows_match_full():
    s = inputs.Stream(96)
    X = s.normal(16, 8, 1.0, "f32").f64
    Wg, Wu = s.normal(8, 16, 0.3, "f32").f64, s.normal(8, 16, 0.3, "f32").f64
    Wd = s.normal(16, 8, 0.3, "f32").f64
    types = np.arange(16) % 4
    H, Y = oracle.swiglu("Q2xQ2", 4, types, X, Wg, Wu, Wd)
    h2, y2 = oracle.swiglu_rows("Q2xQ2", 4, types, X, Wg, Wu, Wd, [3, 9])
    assert np.array_equal(y2, Y[[3, 9]]) and np.array_equal(h2, H[[3, 9]])


def test_swiglu_bwd_q1_matches_torch_autograd():
    # at q = 1 the algebraic FFN is the dense one; torch's float64 autograd on
    # the CPU differentiates it independently of the oracle's chain rule
    import torch
    s = inputs.Stream(99)
    X = s.normal(5, 8, 1.0, "f32").f64
    Wg, Wu = s.normal(8, 12, 0.4, "f32").f64, s.normal(8, 12, 0.4, "f32").f64
    Wd = s.normal(12, 8, 0.4, "f32").f64
    dY = s.normal(5, 8, 1.0, "f32").f64
    got = oracle.swiglu_bwd("Q", 1, np.zeros(5, np.int64), X, Wg, Wu, Wd, dY)
    t = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (X, Wg, Wu, Wd)]
    Y = (torch.nn.functional.silu(t[0] @ t[1]) * (t[0] @ t[2])) @ t[3]
    (Y * torch.tensor(dY)).sum().backward()
    for g, ti in zip(got, t):
        assert np.allclose(g, ti.grad.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("law,q", [("Q2xQ2", 4), ("Q", 3)])
def test_swiglu_bwd_matches_autograd_of_masked_dense(law, q):
    # each row type's projection is a dense product with the weight blocks
    # outside its table row zeroed; torch's float64 autograd through those
    # masked dense products is an independent derivation of the gradients
    import torch
    s = inputs.Stream(120 + q)
    M, D, F = 3 * q, 2 * q, 4 * q
    X = s.normal(M, D, 1.0, "f32").f64
    Wg, Wu = s.normal(D, F, 0.5, "f32").f64, s.normal(D, F, 0.5, "f32").f64
    Wd = s.normal(F, D, 0.5, "f32").f64
    dY = s.normal(M, D, 1.0, "f32").f64
    types = np.arange(M) % q
    S = oracle.block_table_array(law, q)  # S[t, k, a]

    def mask(t, din, dout):
        bi, bo = din // q, dout // q
        m = np.zeros((din, dout))
        for k in range(q):
            for a in range(q):
                if S[t, k, a]:
                    m[a * bi:(a + 1) * bi, k * bo:(k + 1) * bo] = 1.0
        return torch.tensor(m)

    t = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (X, Wg, Wu, Wd)]
    rows = []
    for r in range(M):
        ty = int(types[r])
        x = t[0][r:r + 1]
        g = x @ (t[1] * mask(ty, D, F))
        u = x @ (t[2] * mask(ty, D, F))
        h = torch.nn.functional.silu(g) * u
        rows.append(h @ (t[3] * mask(ty, F, D)))
    Y = torch.cat(rows)
    (Y * torch.tensor(dY)).sum().backward()
    got = oracle.swiglu_bwd(law, q, types, X, Wg, Wu, Wd, dY)
    for g, ti in zip(got, t):
        assert np.allclose(g, ti.grad.numpy(), rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("law,q", [("Q2xQ2", 4), ("Q", 3)])
def test_swiglu_bwd_finite_differences(law, q):
    s = inputs.Stream(100 + q)
    M, D, F = 2 * q, 2 * q, 3 * q
    X = s.normal(M, D, 1.0, "f32").f64
    Wg, Wu = s.normal(D, F, 0.5, "f32").f64, s.normal(D, F, 0.5, "f32").f64
    Wd = s.normal(F, D, 0.5, "f32").f64
    dY = s.normal(M, D, 1.0, "f32").f64
    types = np.arange(M) % q
    grads = oracle.swiglu_bwd(law, q, types, X, Wg, Wu, Wd, dY)
    args = [X, Wg, Wu, Wd]

    def loss(a):
        return float(np.sum(dY * oracle.swiglu(law, q, types, *a)[1]))

    h = 1e-6
    for which in range(4):
        for (r, c) in ((0, 0), (1, 2), (M - 1 if which == 0 else 2, 1)):
            up = [a.copy() for a in args]
            dn = [a.copy() for a in args]
            up[which][r, c] += h
            dn[which][r, c] -= h
            fd = (loss(up) - loss(dn)) / (2 * h)
            assert abs(fd - grads[which][r, c]) < 1e-6 * max(1.0, abs(fd))


def test_swiglu_decode_is_the_prefill_row_at_that_position():
    # a decode step at position p equals row p of the prefill SwiGLU of a
    # sequence that contains it: the FFN is row-local and the row type comes
    # from the position alone
    s = inputs.Stream(97)
    L = 12
    X = s.normal(L, 8, 1.0, "f32").f64
    Wg, Wu = s.normal(8, 16, 0.3, "f32").f64, s.normal(8, 16, 0.3, "f32").f64
    Wd = s.normal(16, 8, 0.3, "f32").f64
    H, Y = oracle.swiglu("Q2xQ2", 4, oracle.row_types("Q2xQ2", 4, np.arange(L)), X, Wg, Wu, Wd)
    pos = np.array([7, 0, 11, 5, 5])
    h, y = oracle.swiglu_decode("Q2xQ2", 4, pos, X[pos], Wg, Wu, Wd)
    assert np.array_equal(h, H[pos]) and np.array_equal(y, Y[pos])


def test_swiglu_decode_q1_is_dense_swiglu_and_gate_up_not_symmetric():
    s = inputs.Stream(98)
    x = s.normal(3, 8, 1.0, "f32").f64
    Wg, Wu = s.normal(8, 12, 0.3, "f32").f64, s.normal(8, 12, 0.3, "f32").f64
    Wd = s.normal(12, 8, 0.3, "f32").f64
    h, y = oracle.swiglu_decode("Q", 1, np.array([4, 9, 2]), x, Wg, Wu, Wd)
    G, U = x @ Wg, x @ Wu
    hd = G / (1.0 + np.exp(-G)) * U
    assert np.allclose(h, hd, rtol=1e-14) and np.allclose(y, hd @ Wd, rtol=1e-13)
    # exchanging gate and up changes the result (silu is applied to the gate)
    h2, _ = oracle.swiglu_decode("Q", 1, np.array([4, 9, 2]), x, Wu, Wg, Wd)
    assert not np.allclose(h2, h)


# --------------------------------------------------------------------------
# The tile form of the square product (used for large q)
# --------------------------------------------------------------------------

def _assemble_from_tiles(tile_fn, law, q, X, W):
    """Z assembled tile by tile from ``tile_fn`` over every output block."""
    b = X.shape[0] // q
    Z = np.zeros_like(X)

    def xb(r, c):
        return X[r * b:(r + 1) * b, c * b:(c + 1) * b]

    def wb(r, c):
        return W[r * b:(r + 1) * b, c * b:(c + 1) * b]

    for i in range(q):
        for k in range(q):
            Z[i * b:(i + 1) * b, k * b:(k + 1) * b] = tile_fn(law, q, i, k, xb, wb)
    return Z


SQUARE_TILE_CASES = [("Q", 2), ("Q", 3), ("Q", 4), ("Q", 5), ("Q2xQ2", 4)]


def _square_tile_pin(tile_fn):
    """The tile form equals the full definition (all q^4 block pairs) exactly
    on small-integer matrices, and a tile at q = 2 matches the hand-worked
    entry: Z_01 = X_00 W_01 + X_01 W_11 (source vertex times edge plus edge
    times target vertex)."""
    try:
        for law, q in SQUARE_TILE_CASES:
            X, W = _int_mats(3 * q, seed=80 + q, count=2)
            if not np.array_equal(_assemble_from_tiles(tile_fn, law, q, X, W),
                                  oracle.square_product(law, q, X, W)):
                return False
        X, W = _int_mats(6, seed=90, count=2)
        xb = lambda r, c: X[3 * r:3 * r + 3, 3 * c:3 * c + 3]  # noqa: E731
        wb = lambda r, c: W[3 * r:3 * r + 3, 3 * c:3 * c + 3]  # noqa: E731
        by_hand = xb(0, 0) @ wb(0, 1) + xb(0, 1) @ wb(1, 1)
        if not np.array_equal(tile_fn("Q", 2, 0, 1, xb, wb), by_hand):
            return False
        if not np.array_equal(tile_fn("Q", 2, 1, 1, xb, wb), xb(1, 1) @ wb(1, 1)):
            return False
    except (ValueError, IndexError, TypeError):
        return False
    return True


def test_square_tile_equals_square_product_exact():
    assert _square_tile_pin(oracle.square_tile)


def _tile_swapped_x(law, q, i, k, x_block, w_block):
    return sum(x_block(a, i) @ w_block(a, k) for a in oracle.table_entry(law, q, i, k))


def _tile_swapped_w(law, q, i, k, x_block, w_block):
    return sum(x_block(i, a) @ w_block(k, a) for a in oracle.table_entry(law, q, i, k))


def _tile_wrong_chain(law, q, i, k, x_block, w_block):
    return sum(x_block(i, a) @ w_block(i, k) for a in oracle.table_entry(law, q, i, k))


def _tile_first_member_only(law, q, i, k, x_block, w_block):
    a = oracle.table_entry(law, q, i, k)[0]
    return x_block(i, a) @ w_block(a, k)


@pytest.mark.parametrize("bad", [_tile_swapped_x, _tile_swapped_w, _tile_wrong_chain,
                                 _tile_first_member_only])
def test_planted_square_tile_mistakes_are_caught(bad):
    assert not _square_tile_pin(bad)


# --------------------------------------------------------------------------
# Mutations planted in the oracle: each must trip at least one pin
# --------------------------------------------------------------------------

def _pins_pass():
    """Run a compact set of the pins above; False as soon as one fails."""
    try:
        test_q2_scalar_worked_example()
        test_q2_removed_products_are_the_edge_cycle()
        for row in _read_rows("counts.txt"):
            test_block_product_counts(row)
        for law, q in LAW_CASES:
            test_associativity_exact(law, q)
            test_unit_exact(law, q)
            test_projection_rows_equal_square_row_blocks(law, q)
        test_tensor_square_table_is_product_of_factor_tables()
        test_row_types_q2_first_types_use_first_block_row()
    except (AssertionError, ValueError, IndexError):
        return False
    return True


def test_unmutated_oracle_passes_compact_pins():
    assert _pins_pass()


MUTATIONS = {
    # edge * edge kept: the dense block algebra
    "dense": lambda i, j, l, k: (i, k) if j == l else None,
    # edge * target-vertex dropped
    "no_edge_vertex": lambda i, j, l, k: (i, k) if j == l and i == j else None,
    # source-vertex * edge dropped
    "no_vertex_edge": lambda i, j, l, k: (i, k) if j == l and (l == k) else None,
    # wrong chaining index: pairs blocks on the outer indices
    "wrong_chain": lambda i, j, l, k: (j, l) if i == k and (i == j or l == k) else None,
    # transposed result slot
    "transposed_slot": lambda i, j, l, k: ((k, i) if j == l and (i == j or l == k) else None),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_structure_constant_mistakes_are_caught(monkeypatch, name):
    monkeypatch.setattr(oracle, "_complete_graph_product", MUTATIONS[name])
    assert not _pins_pass()


def test_planted_row_type_offset_is_caught(monkeypatch):
    real = oracle.row_types
    monkeypatch.setattr(oracle, "row_types", lambda law, q, p: real(law, q, np.asarray(p) + 1))
    assert not _pins_pass()


def test_planted_transposed_weight_block_is_caught(monkeypatch):
    real = oracle.project

    def bad(law, q, types, X, W, counter=None):
        W = np.asarray(W, dtype=np.float64)
        din, dout = W.shape
        if din == dout and din % q == 0 and q > 1:
            b = din // q
            W = W.copy()
            for a in range(q):
                for k in range(a + 1, q):
                    blk = W[a * b:(a + 1) * b, k * b:(k + 1) * b].copy()
                    W[a * b:(a + 1) * b, k * b:(k + 1) * b] = W[k * b:(k + 1) * b, a * b:(a + 1) * b]
                    W[k * b:(k + 1) * b, a * b:(a + 1) * b] = blk
        return real(law, q, types, X, W, counter)

    monkeypatch.setattr(oracle, "project", bad)
    assert not _pins_pass()
