"""CPU oracle for the associative-algebra block product, in float64 (numpy).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never calls it and shares no code with it.

What it computes, and where the pages define it (all from "Change the
Product, Keep the Parameters: Associative Algebra Layers for Transformers",
Koziev & Oseledets, arXiv:2609.32814; the pages cited are the agihunt.info
digest, the hotpaper.ai summary and the author's post on feed.hirify.me):

* The multiplication table comes from a directed graph: the diagonal slots
  of a q x q block matrix are its vertices, the kept off-diagonal slots its
  edges, and an edge times an edge is zero.  The complete graph on q feature
  groups gives the law Q_q: a diagonal block multiplies only its own group,
  and an off-diagonal output block is the source group's diagonal block times
  the edge block plus the edge block times the target group's diagonal block
  (agihunt.info digest, paragraph on the multiplication table).  This module
  encodes exactly that rule as structure constants on basis elements e_ij
  (``basis_product``) and derives everything else from them.
* The pilot law is the tensor square Q2 (x) Q2: 16 coordinates, 36 block
  products on the square, 9/16 of the dense MACs per projection row
  (agihunt.info digest, paragraph on the tensor-square pilot).
* Row typing: each token takes a row type from its absolute position and
  evaluates only that row of the table (agihunt.info digest, paragraph on
  mapping to the Transformer; hotpaper.ai summary, "row-typed rectangular
  projections").  The position -> type map is position mod (number of
  groups), the plainest reading of "absolute position".
* Projections are Y = X W with X [tokens, din], W [din, dout] (agihunt.info
  digest, opening paragraph); din and dout are each cut into q equal groups.

Every function here is a plain loop over the table with a float64 matmul as
its only library step.  Pins that tie these functions to the pages (and not
to themselves) live in ``tests/test_oracle_pins.py``.  The SwiGLU order
(silu(G) * U then the down projection) is a reading of the pages' "FFN
projections" and is pinned only through its parts (SiLU at fixed points,
the projections, and the q = 1 case against a dense SwiGLU).
"""
from __future__ import annotations

import math

import numpy as np

LAWS = ("Q", "Q2xQ2")


# ---------------------------------------------------------------------------
# Structure constants
# ---------------------------------------------------------------------------

def _complete_graph_product(i: int, j: int, l: int, k: int):
    """Basis product e_ij * e_lk in the complete-graph law Q_q.

    Slot (g, g) is the vertex of group g; slot (g, h), g != h, is the edge
    g -> h.  Returns the slot of the product (coefficient 1) or None (zero).
    """
    if j != l:               # blocks that do not chain multiply to zero
        return None
    left_vertex = i == j
    right_vertex = l == k
    if left_vertex or right_vertex:
        # vertex*vertex -> vertex; vertex*edge and edge*vertex -> the edge
        return (i, k)
    return None              # edge * edge = 0


def _pair(g: int):
    """Group g of the tensor square <-> pair (g1, g2) with g = 2*g1 + g2."""
    return g // 2, g % 2


def _tensor_square_product(i: int, j: int, l: int, k: int):
    """Basis product in Q2 (x) Q2: (e (x) f)(e' (x) f') = (e e') (x) (f f')."""
    i1, i2 = _pair(i)
    j1, j2 = _pair(j)
    l1, l2 = _pair(l)
    k1, k2 = _pair(k)
    first = _complete_graph_product(i1, j1, l1, k1)
    second = _complete_graph_product(i2, j2, l2, k2)
    if first is None or second is None:
        return None
    return (2 * first[0] + second[0], 2 * first[1] + second[1])


def basis_product(law: str, q: int, left, right):
    """Slot of e_left * e_right under ``law`` with q groups, or None."""
    i, j = left
    l, k = right
    for g in (i, j, l, k):
        if not 0 <= g < q:
            raise ValueError("group index out of range")
    if law == "Q":
        return _complete_graph_product(i, j, l, k)
    if law == "Q2xQ2":
        if q != 4:
            raise ValueError("Q2xQ2 has exactly 4 groups")
        return _tensor_square_product(i, j, l, k)
    raise ValueError(f"unknown law {law!r}")


def check_law(law: str, q: int):
    if law not in LAWS:
        raise ValueError(f"unknown law {law!r}")
    if q < 1:
        raise ValueError("q must be >= 1")
    if law == "Q2xQ2" and q != 4:
        raise ValueError("Q2xQ2 has exactly 4 groups")


def table_entry(law: str, q: int, i: int, k: int):
    """S(i, k): the inner groups a whose product e_ia * e_ak lands on slot
    (i, k).  Output block (i, k) of X * W is the sum over a in S(i, k) of
    X_ia W_ak."""
    return tuple(a for a in range(q) if basis_product(law, q, (i, a), (a, k)) == (i, k))


def block_table(law: str, q: int):
    """S as a nested list: S[i][k] = table_entry(law, q, i, k)."""
    check_law(law, q)
    return [[table_entry(law, q, i, k) for k in range(q)] for i in range(q)]


def block_table_array(law: str, q: int) -> np.ndarray:
    """S as a uint8 array [q, q, q] with S[i, k, a] = 1 iff a in S(i, k)."""
    S = np.zeros((q, q, q), dtype=np.uint8)
    for i, row in enumerate(block_table(law, q)):
        for k, members in enumerate(row):
            for a in members:
                S[i, k, a] = 1
    return S


def block_product_count(law: str, q: int, row_typed: bool) -> int:
    """Block products one row of the table needs (row_typed, summed over the
    row's output groups and taken for row type 0), or the whole square
    product needs."""
    S = block_table(law, q)
    if row_typed:
        return sum(len(S[0][k]) for k in range(q))
    return sum(len(S[i][k]) for i in range(q) for k in range(q))


# ---------------------------------------------------------------------------
# Square product X * W on q x q block matrices
# ---------------------------------------------------------------------------

def _block(A: np.ndarray, r: int, c: int, br: int, bc: int) -> np.ndarray:
    return A[r * br:(r + 1) * br, c * bc:(c + 1) * bc]


def square_product(law: str, q: int, X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """X * W from the definition: X = sum e_ij (x) X_ij, W = sum e_lk (x) W_lk
    and X * W = sum over all block pairs of (e_ij e_lk) (x) X_ij W_lk.
    Visits all q^4 block pairs; meant for small q."""
    check_law(law, q)
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    n_r, n_i = X.shape
    n_i2, n_c = W.shape
    if n_i != n_i2 or n_r % q or n_i % q or n_c % q:
        raise ValueError("shapes must agree and be divisible by q")
    br, bi, bc = n_r // q, n_i // q, n_c // q
    Z = np.zeros((n_r, n_c))
    for i in range(q):
        for j in range(q):
            for l in range(q):
                for k in range(q):
                    slot = basis_product(law, q, (i, j), (l, k))
                    if slot is None:
                        continue
                    r, c = slot
                    Z[r * br:(r + 1) * br, c * bc:(c + 1) * bc] += (
                        _block(X, i, j, br, bi) @ _block(W, l, k, bi, bc))
    return Z


def square_tile(law: str, q: int, i: int, k: int, x_block, w_block) -> np.ndarray:
    """Output block (i, k) of X * W for large q.

    ``x_block(i, a)`` and ``w_block(a, k)`` return float64 blocks.  Only
    pairs e_ij * e_lk whose product lands on (i, k) contribute; for the laws
    here a product keeps the outer indices, so those are the pairs
    (i, a) * (a, k) with a in S(i, k)."""
    acc = None
    for a in table_entry(law, q, i, k):
        term = np.asarray(x_block(i, a), dtype=np.float64) @ np.asarray(w_block(a, k), dtype=np.float64)
        acc = term if acc is None else acc + term
    return acc


def unit(q: int, b: int) -> np.ndarray:
    """The unit of the algebra on q x q blocks of size b: sum_i e_ii (x) I_b."""
    return np.eye(q * b)


# ---------------------------------------------------------------------------
# Row-typed projection
# ---------------------------------------------------------------------------

def row_types(law: str, q: int, positions) -> np.ndarray:
    """Row type of a token at absolute position p: p mod q (for Q2xQ2 the
    type t = p mod 4 is group (t // 2, t % 2) of the pair index)."""
    check_law(law, q)
    return (np.asarray(positions, dtype=np.int64) % q).astype(np.int64)


class MacCounter:
    """Counts the scalar multiply-adds the oracle performs."""

    def __init__(self):
        self.macs = 0


def project(law: str, q: int, types, X, W, counter: MacCounter | None = None) -> np.ndarray:
    """Row-typed projection Y = X * W: row r of type t plays the role of a
    row of block-row t, so for each output group k,
    y_k = sum over a in S(t, k) of x_a W_ak."""
    check_law(law, q)
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    types = np.asarray(types, dtype=np.int64)
    M, din = X.shape
    din2, dout = W.shape
    if din != din2 or din % q or dout % q or types.shape != (M,):
        raise ValueError("bad shapes")
    if M and (types.min() < 0 or types.max() >= q):
        raise ValueError("row type out of range")
    bi, bo = din // q, dout // q
    S = block_table(law, q)
    Y = np.zeros((M, dout))
    for t in range(q):
        rows = np.nonzero(types == t)[0]
        if rows.size == 0:
            continue
        Xt = X[rows]
        for k in range(q):
            acc = np.zeros((rows.size, bo))
            for a in S[t][k]:
                acc += Xt[:, a * bi:(a + 1) * bi] @ W[a * bi:(a + 1) * bi, k * bo:(k + 1) * bo]
                if counter is not None:
                    counter.macs += rows.size * bi * bo
            Y[rows, k * bo:(k + 1) * bo] = acc
    return Y


def project_rows(law: str, q: int, types, X, W, rows) -> np.ndarray:
    """The projection of a subset of rows only (rows are independent)."""
    rows = np.asarray(rows, dtype=np.int64)
    return project(law, q, np.asarray(types)[rows], np.asarray(X)[rows], W)


def project_bwd(law: str, q: int, types, X, W, dY):
    """Gradients of L = <dY, project(X, W)>: each term x_a W_ak of output
    group k sends dy_k W_ak^T to dx_a and x_a^T dy_k to dW_ak."""
    check_law(law, q)
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    types = np.asarray(types, dtype=np.int64)
    M, din = X.shape
    dout = W.shape[1]
    bi, bo = din // q, dout // q
    S = block_table(law, q)
    dX = np.zeros_like(X)
    dW = np.zeros_like(W)
    for t in range(q):
        rows = np.nonzero(types == t)[0]
        if rows.size == 0:
            continue
        Xt = X[rows]
        dYt = dY[rows]
        dXt = np.zeros((rows.size, din))
        for k in range(q):
            dyk = dYt[:, k * bo:(k + 1) * bo]
            for a in S[t][k]:
                Wak = W[a * bi:(a + 1) * bi, k * bo:(k + 1) * bo]
                dXt[:, a * bi:(a + 1) * bi] += dyk @ Wak.T
                dW[a * bi:(a + 1) * bi, k * bo:(k + 1) * bo] += Xt[:, a * bi:(a + 1) * bi].T @ dyk
        dX[rows] = dXt
    return dX, dW


def silu(z):
    """SiLU from its definition z * sigmoid(z) = z / (1 + exp(-z))."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def swiglu(law: str, q: int, types, X, Wg, Wu, Wd):
    """SwiGLU FFN with every projection algebraic and the same row types:
    H = silu(X * Wg) . (X * Wu), Y = H * Wd.  Returns (H, Y) in float64."""
    G = project(law, q, types, X, Wg)
    U = project(law, q, types, X, Wu)
    H = silu(G) * U
    return H, project(law, q, types, H, Wd)


def swiglu_bwd(law: str, q: int, types, X, Wg, Wu, Wd, dY):
    """Gradients of L = <dY, Y> for the algebraic SwiGLU FFN (Y from
    ``swiglu``): chain rule through the down projection, the product
    silu(G) . U (silu'(g) = s (1 + g (1 - s)), s the logistic function) and
    the two input projections, each through ``project_bwd``.
    Returns (dX, dWg, dWu, dWd) in float64."""
    X = np.asarray(X, dtype=np.float64)
    G = project(law, q, types, X, Wg)
    U = project(law, q, types, X, Wu)
    H = silu(G) * U
    dH, dWd = project_bwd(law, q, types, H, Wd, dY)
    sg = 1.0 / (1.0 + np.exp(-G))
    dG = dH * U * sg * (1.0 + G * (1.0 - sg))
    dU = dH * silu(G)
    dXg, dWg = project_bwd(law, q, types, X, Wg, dG)
    dXu, dWu = project_bwd(law, q, types, X, Wu, dU)
    return dXg + dXu, dWg, dWu, dWd


def swiglu_rows(law: str, q: int, types, X, Wg, Wu, Wd, rows):
    """SwiGLU on a subset of rows (the FFN is row-local)."""
    rows = np.asarray(rows, dtype=np.int64)
    return swiglu(law, q, np.asarray(types)[rows], np.asarray(X)[rows], Wg, Wu, Wd)


def decode(law: str, q: int, positions, x, W) -> np.ndarray:
    """One new token per batch entry at absolute position positions[b]: only
    that position's table row is evaluated."""
    return project(law, q, row_types(law, q, positions), x, W)


def swiglu_decode(law: str, q: int, positions, x, Wg, Wu, Wd):
    """Decode step of the algebraic SwiGLU FFN: for each new token at absolute
    position positions[b], its row of each projection with the activation in
    between (agihunt.info digest: decoding evaluates the new position's row;
    the FFN projections share the row types).  Returns (H, Y) in float64."""
    G = decode(law, q, positions, x, Wg)
    U = decode(law, q, positions, x, Wu)
    H = silu(G) * U
    return H, decode(law, q, positions, H, Wd)


def mac_ratio(law: str, q: int) -> float:
    """Fraction of a dense projection's MACs that one row type performs."""
    return block_product_count(law, q, True) / float(q * q)


def rel_err(got, ref) -> float:
    """max|got - ref| / max|ref| (0 when both are empty or ref is zero and
    got matches)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return num / den
