"""GPU parity: every libaal call against the CPU oracle on the same seeded
inputs.  bf16: max|err|/max|ref| <= 5e-3; fp32: <= 1e-5.  Integer work
(associativity and unit on small-integer matrices) is compared bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import associative_algebra_block_b200 as aal
from associative_algebra_block_b200 import inputs

from gpu_cases import (TOL, dev, host64, run_bwd, run_decode, run_project, run_square, run_swiglu,
                       run_swiglu_bwd, run_swiglu_decode)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    aal.load()


GENERAL = aal.AAL_PATH_GENERAL

# ----------------------------------------------------------------- Q_2 fp32
def test_c1_q2_fp32_projection():
    err, _ = run_project("Q", 2, 64, 64, 64, "f32", seq_len=64)
    assert err <= TOL["f32"], err


@pytest.mark.parametrize("law,q,n", [("Q", 2, 32), ("Q", 3, 48), ("Q2xQ2", 4, 64)])
def test_c1_integer_associativity_and_unit_exact(law, q, n):
    mats = inputs.integer_square_inputs(n, count=3, seed=q)
    X, W, Z = (m.t.cuda() for m in mats)

    def sq(A, B):
        out = torch.empty_like(A)
        aal.aal_square_product(law, q, A, B, out)
        return out

    left = sq(sq(X, W), Z)
    right = sq(X, sq(W, Z))
    torch.cuda.synchronize()
    assert torch.equal(left, right)
    ref = oracle.square_product(law, q, oracle.square_product(law, q, mats[0].f64, mats[1].f64), mats[2].f64)
    assert np.array_equal(host64(left), ref)
    one = torch.eye(n, device="cuda")
    assert torch.equal(sq(X, one), X) and torch.equal(sq(one, X), X)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_c1_all_calls_small(dtype):
    tol = TOL[dtype]
    e, _ = run_square("Q", 2, 64, dtype)
    assert e <= tol
    eh, ey, _ = run_swiglu("Q", 2, 64, 64, 128, dtype, seq_len=64)
    assert eh <= tol and ey <= tol
    edx, edw, _ = run_bwd("Q", 2, 64, 64, 64, dtype)
    assert edx <= tol and edw <= tol
    ed, _ = run_decode("Q", 2, 5, 64, 64, dtype)
    assert ed <= tol


# ------------------------------------------------- Q2 x Q2 SwiGLU (110M FFN)
TENSOR = aal.AAL_PATH_TENSOR


def test_c2_swiglu_full_size():
    # the launch configuration bench.py times (tensor-core path)
    eh, ey, path = run_swiglu("Q2xQ2", 4, 12288, 768, 1536, "bf16", seq_len=1536)
    assert eh <= TOL["bf16"] and ey <= TOL["bf16"], (eh, ey)
    assert path == TENSOR


@pytest.mark.parametrize("B", [1, 8, 64])
def test_c2_decode(B):
    err, path = run_decode("Q2xQ2", 4, B, 768, 1536, "bf16", seed=B)
    assert err <= TOL["bf16"], err
    assert path == aal.AAL_PATH_DECODE
    err, _ = run_decode("Q2xQ2", 4, B, 1536, 768, "bf16", seed=B + 1)
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("t", [0, 1, 2, 3])
def test_c2_decode_single_type(t):
    err, _ = run_decode("Q2xQ2", 4, 1, 768, 1536, "bf16", seed=40 + t, same_type=t)
    assert err <= TOL["bf16"], err


# Decode shapes around the tensor-core decode kernel's limits: ragged batches,
# the largest batch it takes (256) and the first it leaves to the SIMT
# kernels (257; 1100 reaches the cluster kernel), K slices of 16 rows, groups
# of 16 rows, q up to 32.
@pytest.mark.parametrize("law,q,B,din,dout", [
    ("Q2xQ2", 4, 100, 768, 1536),
    ("Q2xQ2", 4, 256, 1536, 768),
    ("Q2xQ2", 4, 257, 768, 1536),
    ("Q2xQ2", 4, 1100, 768, 1536),
    ("Q", 16, 33, 2048, 1024),
    ("Q", 32, 17, 4096, 2048),
    ("Q", 2, 7, 64, 128),
    ("Q", 8, 1, 128, 512),
    ("Q", 4, 64, 4096, 256),
])
def test_decode_shapes(law, q, B, din, dout):
    err, path = run_decode(law, q, B, din, dout, "bf16", seed=B + din)
    assert err <= TOL["bf16"], err
    assert path == aal.AAL_PATH_DECODE


def test_decode_negative_position_tensor_core_kernel():
    # 64-column output groups: the tensor-core decode kernel takes this call
    s = inputs.Stream(5)
    x = s.normal(3, 64, 1.0, "bf16")
    W = s.normal(64, 128, 0.125, "bf16")
    pos = np.array([3, -1, 6], dtype=np.int64)
    y = torch.full((3, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    aal.aal_decode_matvec("Q", 2, torch.from_numpy(pos).cuda(), x.t.cuda(), W.t.cuda(), y)
    assert aal.aal_get_device_status() == aal.AAL_ERR_DEVICE_BOUNDS
    got = host64(y)
    assert np.all(np.isnan(got[1]))  # the invalid entry is skipped
    keep = np.array([0, 2])
    ref = oracle.decode("Q", 2, pos[keep], x.f64[keep], W.f64)
    assert oracle.rel_err(got[keep], ref) <= TOL["bf16"]


# Whole-FFN decode step (fused gate/up/SiLU, then the down decode): the c2
# batches, a batch split into 128-entry launches, single row types, and the
# general path (fp32; 32-column groups).
@pytest.mark.parametrize("B", [1, 8, 64, 128, 200])
def test_swiglu_decode_c2(B):
    eh, ey, path = run_swiglu_decode("Q2xQ2", 4, B, 768, 1536, "bf16", seed=300 + B)
    assert eh <= TOL["bf16"] and ey <= TOL["bf16"], (eh, ey)
    assert path == aal.AAL_PATH_DECODE


@pytest.mark.parametrize("t", [0, 3])
def test_swiglu_decode_single_type(t):
    eh, ey, _ = run_swiglu_decode("Q2xQ2", 4, 1, 768, 1536, "bf16", seed=310 + t, same_type=t)
    assert eh <= TOL["bf16"] and ey <= TOL["bf16"], (eh, ey)


@pytest.mark.parametrize("law,q,B,D,F,dtype,path", [
    ("Q", 2, 5, 64, 128, "f32", aal.AAL_PATH_GENERAL),
    ("Q", 4, 9, 128, 128, "bf16", aal.AAL_PATH_GENERAL),
    ("Q", 16, 33, 2048, 1024, "bf16", aal.AAL_PATH_DECODE),
])
def test_swiglu_decode_other_shapes(law, q, B, D, F, dtype, path):
    eh, ey, got = run_swiglu_decode(law, q, B, D, F, dtype, seed=320 + B)
    assert eh <= TOL[dtype] and ey <= TOL[dtype], (eh, ey)
    assert got == path


@pytest.mark.parametrize("B,launches", [(1, 2), (64, 2), (128, 2), (200, 3)])
def test_swiglu_decode_launches(B, launches):
    # gate/up/SiLU decode (one launch per 128 entries), then the down decode
    # chained to it by a programmatic dependent launch
    s = inputs.Stream(330 + B)
    D, F = 768, 1536
    x = s.normal(B, D, 1.0, "bf16", want_f64=False).t.cuda()
    Wg, Wu = (s.normal(D, F, D ** -0.5, "bf16", want_f64=False).t.cuda() for _ in range(2))
    Wd = s.normal(F, D, F ** -0.5, "bf16", want_f64=False).t.cuda()
    pos = torch.from_numpy(s.positions(B, 1536)).cuda()
    h = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")
    aal.aal_launch_count(reset=True)
    aal.aal_swiglu_decode("Q2xQ2", 4, pos, x, Wg, Wu, Wd, h, y)
    assert aal.aal_launch_count(reset=True) == launches
    assert aal.aal_get_device_status() == aal.AAL_OK


_ONE_LAUNCH_CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + '/tests')
from gpu_cases import TOL, run_swiglu_decode
import associative_algebra_block_b200 as aal
for B, launches in ((1, 1), (8, 1), (64, 1), (128, 1), (200, 2)):
    aal.aal_launch_count(reset=True)
    eh, ey, path = run_swiglu_decode('Q2xQ2', 4, B, 768, 1536, 'bf16', seed=340 + B)
    assert path == aal.AAL_PATH_DECODE and eh <= TOL['bf16'] and ey <= TOL['bf16'], (B, eh, ey, path)
    assert aal.aal_launch_count(reset=True) == launches, B
for t in (0, 3):
    eh, ey, _ = run_swiglu_decode('Q2xQ2', 4, 1, 768, 1536, 'bf16', seed=360 + t, same_type=t)
    assert eh <= TOL['bf16'] and ey <= TOL['bf16'], (t, eh, ey)
eh, ey, _ = run_swiglu_decode('Q', 16, 33, 2048, 1024, 'bf16', seed=370)
assert eh <= TOL['bf16'] and ey <= TOL['bf16'], (eh, ey)
print('ok')
"""


def test_one_launch_ffn_decode_parity():
    # the opt-in one-launch FFN decode (gate/up CTAs and down CTAs in one
    # grid, meeting in a bounded grid barrier)
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _ONE_LAUNCH_CHILD, root], capture_output=True, text=True,
                       timeout=600, env=dict(os.environ, AAL_FFN_DECODE_FUSED="1"))
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_swiglu_decode_negative_position():
    s = inputs.Stream(7)
    x = s.normal(3, 128, 1.0, "bf16")
    Wg, Wu = s.normal(128, 256, 0.1, "bf16"), s.normal(128, 256, 0.1, "bf16")
    Wd = s.normal(256, 128, 0.06, "bf16")
    pos = np.array([5, -2, 8], dtype=np.int64)
    h = torch.full((3, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((3, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    aal.aal_swiglu_decode("Q", 2, torch.from_numpy(pos).cuda(), x.t.cuda(), Wg.t.cuda(), Wu.t.cuda(),
                          Wd.t.cuda(), h, y)
    assert aal.aal_get_device_status() == aal.AAL_ERR_DEVICE_BOUNDS
    gh, gy = host64(h), host64(y)
    assert np.all(np.isnan(gh[1])) and np.all(np.isnan(gy[1]))
    keep = np.array([0, 2])
    H, Y = oracle.swiglu_decode("Q", 2, pos[keep], x.f64[keep], Wg.f64, Wu.f64, Wd.f64)
    assert oracle.rel_err(gh[keep], H) <= TOL["bf16"] and oracle.rel_err(gy[keep], Y) <= TOL["bf16"]


# SwiGLU backward (dX, dWg, dWu, dWd): the expert-shaped FFN on the
# tensor-core path with the SiLU' chain in the dH epilogue, the pilot law,
# and the general path (fp32; explicit row types).
@pytest.mark.parametrize("law,q,M,D,F,dtype,explicit,path", [
    ("Q", 16, 2048, 2048, 768, "bf16", False, aal.AAL_PATH_TENSOR),
    ("Q2xQ2", 4, 1024, 768, 1536, "bf16", False, aal.AAL_PATH_TENSOR),
    ("Q", 2, 64, 64, 128, "f32", False, aal.AAL_PATH_GENERAL),
    ("Q", 4, 96, 128, 256, "bf16", True, aal.AAL_PATH_GENERAL),
])
def test_swiglu_bwd(law, q, M, D, F, dtype, explicit, path):
    errs, got = run_swiglu_bwd(law, q, M, D, F, dtype, seed=M + q, explicit=explicit)
    assert max(errs) <= TOL[dtype], errs
    assert got == path


def test_swiglu_autograd_wrapper():
    from associative_algebra_block_b200.autograd import swiglu
    ins = inputs.swiglu_inputs(256, 512, 512, seed=3, dtype="bf16")
    t = [dev(ins[k]).requires_grad_(True) for k in ("X", "Wg", "Wu", "Wd")]
    dYd = inputs.Stream(9).normal(512, 256, 1.0, "bf16")
    Y = swiglu("Q2xQ2", 4, aal.row_rule(seq_len=512), *t)
    Y.backward(dev(dYd))
    types = oracle.row_types("Q2xQ2", 4, np.arange(512))
    _, Yref = oracle.swiglu("Q2xQ2", 4, types, *(ins[k].f64 for k in ("X", "Wg", "Wu", "Wd")))
    assert oracle.rel_err(host64(Y.detach()), Yref) <= TOL["bf16"]
    ref = oracle.swiglu_bwd("Q2xQ2", 4, types, *(ins[k].f64 for k in ("X", "Wg", "Wu", "Wd")), dYd.f64)
    for ti, r in zip(t, ref):
        assert oracle.rel_err(host64(ti.grad), r) <= TOL["bf16"]


# -------------------------------------------------- Qwen3-8B-shaped Q_32
def test_c3_swiglu_full_size():
    eh, ey, path = run_swiglu("Q", 32, 2048, 4096, 12288, "bf16", seq_len=2048, w_sigma_rule="D")
    assert eh <= TOL["bf16"] and ey <= TOL["bf16"], (eh, ey)
    assert path == TENSOR


def test_c3_projection_full_size():
    err, path = run_project("Q", 32, 2048, 4096, 12288, "bf16", seq_len=2048)
    assert err <= TOL["bf16"] and path == TENSOR, err


# ------------------------------------------ Qwen3-30B-A3B-expert-shaped Q_16
@pytest.mark.parametrize("din,dout", [(2048, 768), (768, 2048)])
@pytest.mark.parametrize("ws", [False, True])
def test_c4_projection_fwd_bwd(din, dout, ws):
    # ws: with a workspace the heavy dX / dW tiles run as split K pieces
    err, path = run_project("Q", 16, 2048, din, dout, "bf16", seq_len=2048)
    assert err <= TOL["bf16"] and path == TENSOR, err
    edx, edw, path = run_bwd("Q", 16, 2048, din, dout, "bf16", seq_len=2048, ws=ws)
    assert edx <= TOL["bf16"] and edw <= TOL["bf16"], (edx, edw)
    assert path == TENSOR


def test_c4_swiglu():
    eh, ey, _ = run_swiglu("Q", 16, 2048, 2048, 768, "bf16", seq_len=2048)
    assert eh <= TOL["bf16"] and ey <= TOL["bf16"], (eh, ey)


# ------------------------------------------------- square product Q_256
def test_c5_square_full_size_sampled_tiles():
    # Z starts as NaN: a tile the kernel never writes stays non-finite.
    # Every tile is checked for that on the GPU; against the oracle: all of
    # tile-row 17, all of tile-column 200, the four corners and 26 random tiles.
    n, q = 32768, 256
    b = n // q
    ins = inputs.square_inputs(n, seed=0, dtype="bf16", want_f64=False)
    X, W = ins["X"].t.cuda(), ins["W"].t.cuda()
    Z = torch.full_like(X, float("nan"))
    aal.aal_square_product("Q", q, X, W, Z)
    torch.cuda.synchronize()
    assert aal.aal_last_path() == TENSOR
    assert aal.aal_get_device_status() == aal.AAL_OK
    finite = torch.isfinite(Z.view(q, b, q, b)).all(dim=3).all(dim=1)  # [q, q] per tile
    assert bool(finite.all()), int((~finite).sum())
    Xh, Wh = ins["X"].t, ins["W"].t
    rng = np.random.default_rng(123)
    row_i, col_k = 17, 200
    tiles = [(row_i, k) for k in range(q)] + [(i, col_k) for i in range(q) if i != row_i]
    tiles += [(0, 0), (0, q - 1), (q - 1, 0), (q - 1, q - 1)]
    tiles += [tuple(int(v) for v in rng.integers(0, q, 2)) for _ in range(26)]
    Zrow = Z[row_i * b:(row_i + 1) * b].to("cpu", torch.float64).numpy()
    Zcol = Z[:, col_k * b:(col_k + 1) * b].to("cpu", torch.float64).numpy()

    def blk(A, r, c):
        return A[r * b:(r + 1) * b, c * b:(c + 1) * b].to(torch.float64).numpy()

    worst = 0.0
    for i, k in tiles:
        ref = oracle.square_tile("Q", q, i, k, lambda r, c: blk(Xh, r, c), lambda r, c: blk(Wh, r, c))
        if i == row_i:
            got = Zrow[:, k * b:(k + 1) * b]
        elif k == col_k:
            got = Zcol[i * b:(i + 1) * b]
        else:
            got = Z[i * b:(i + 1) * b, k * b:(k + 1) * b].to("cpu", torch.float64).numpy()
        worst = max(worst, oracle.rel_err(got, ref))
    assert worst <= TOL["bf16"], worst


# Q_q with 128-wide blocks and even q runs column-block pairs; odd q one block a tile
@pytest.mark.parametrize("law,q,n", [("Q", 4, 512), ("Q", 16, 2048), ("Q2xQ2", 4, 256), ("Q", 3, 384)])
def test_square_medium(law, q, n):
    err, path = run_square(law, q, n, "bf16")
    assert err <= TOL["bf16"], err
    assert path == (TENSOR if (n // q) % 128 == 0 else aal.AAL_PATH_GENERAL)


@pytest.mark.parametrize("case", ["fwd_swap", "fwd_q2xq2", "swiglu_swap", "bwd_q4", "square_b256",
                                  "fwd_offset", "fwd_ragged_tokens", "fwd_swap_groups_offset",
                                  "swiglu_swap_48_rows", "fwd_swap_q2xq2", "fwd_group_pairs_q2",
                                  "fwd_group_pairs_48", "fwd_class_pairs_48_rows",
                                  "fwd_class_pairs_q4", "swiglu_group_pairs"])
def test_tensor_path_small_cases(case):
    T = TENSOR
    if case == "fwd_swap":
        r = run_project("Q", 8, 512, 1024, 1024, "bf16", seq_len=512, policy=T)
    elif case == "fwd_q2xq2":
        r = run_project("Q2xQ2", 4, 1024, 768, 1536, "bf16", seq_len=1024, policy=T)
    elif case == "swiglu_swap":
        eh, ey, p = run_swiglu("Q", 8, 512, 1024, 1024, "bf16", seq_len=512, policy=T)
        r = (max(eh, ey), p)
    elif case == "bwd_q4":
        edx, edw, p = run_bwd("Q", 4, 512, 512, 512, "bf16", seq_len=512, policy=T)
        r = (max(edx, edw), p)
    elif case == "square_b256":
        r = run_square("Q", 2, 512, "bf16", policy=T)
    elif case == "fwd_offset":
        r = run_project("Q", 8, 1024, 512, 1024, "bf16", seq_len=256, offset=5, policy=T)
    elif case == "fwd_swap_groups_offset":  # 32 rows a class: groups of 4 classes, offset 5
        r = run_project("Q", 16, 512, 1024, 2048, "bf16", seq_len=512, offset=5, policy=T)
    elif case == "swiglu_swap_48_rows":  # 48 rows a class: gate/up in pairs of classes, down in fours
        eh, ey, p = run_swiglu("Q", 8, 384, 1024, 2048, "bf16", seq_len=384, policy=T)
        r = (max(eh, ey), p)
    elif case == "fwd_swap_q2xq2":  # swapped layout without class groups (not Q_q)
        r = run_project("Q2xQ2", 4, 256, 512, 512, "bf16", seq_len=256, policy=T)
    elif case == "fwd_group_pairs_q2":  # one pair of output groups, 200 rows a class
        r = run_project("Q", 2, 400, 256, 128, "bf16", seq_len=400, policy=T)
    elif case == "fwd_group_pairs_48":  # 48-column groups in pairs, offset 3, a partial row block
        r = run_project("Q", 16, 16 * 160, 2048, 768, "bf16", seq_len=16 * 160, offset=3, policy=T)
    elif case == "fwd_class_pairs_48_rows":  # 48 rows a type: two types share a tile, offset 3
        r = run_project("Q", 16, 16 * 48, 512, 16 * 80, "bf16", seq_len=16 * 48, offset=3, policy=T)
    elif case == "fwd_class_pairs_q4":  # 64 rows a type, 96-column groups
        r = run_project("Q", 4, 256, 256, 384, "bf16", seq_len=256, policy=T)
    elif case == "swiglu_group_pairs":  # gate/up in output-group pairs, 160 rows a type (a partial block)
        eh, ey, p = run_swiglu("Q", 8, 8 * 160, 512, 8 * 48, "bf16", seq_len=8 * 160, policy=T)
        r = (max(eh, ey), p)
    else:  # tokens per class not a multiple of the 128-row tile
        r = run_project("Q", 4, 4 * 200, 256, 512, "bf16", seq_len=800, policy=T)
    assert r[0] <= TOL["bf16"] and r[1] == T, r


_ONE_CLASS_CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + '/tests')
from gpu_cases import TOL, run_project, run_swiglu
import associative_algebra_block_b200 as aal
T = aal.AAL_PATH_TENSOR
err, p = run_project("Q", 16, 512, 1024, 2048, "bf16", seq_len=512, offset=5, policy=T)
assert err <= TOL["bf16"] and p == T, (err, p)
eh, ey, p = run_swiglu("Q", 8, 384, 1024, 2048, "bf16", seq_len=384, policy=T)
assert max(eh, ey) <= TOL["bf16"] and p == T, (eh, ey, p)
print("ok")
"""


_ONE_GROUP_CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + '/tests')
from gpu_cases import TOL, run_project, run_square, run_swiglu
import associative_algebra_block_b200 as aal
T = aal.AAL_PATH_TENSOR
for q, M, din, dout, seq, off in ((16, 2048, 2048, 768, 2048, 0), (8, 1024, 512, 1024, 256, 5),
                                   (16, 768, 512, 1280, 768, 3)):
    err, p = run_project("Q", q, M, din, dout, "bf16", seq_len=seq, offset=off, policy=T)
    assert err <= TOL["bf16"] and p == T, (q, err, p)
err, p = run_square("Q", 4, 512, "bf16", policy=T)
assert err <= TOL["bf16"] and p == T, (err, p)
eh, ey, p = run_swiglu("Q", 16, 2048, 2048, 768, "bf16", seq_len=2048, policy=T)
assert max(eh, ey) <= TOL["bf16"] and p == T, (eh, ey, p)
# segment mode (explicit types through the workspace)
err, p = run_project("Q", 16, 2048, 2048, 768, "bf16", explicit=True, seed=5, ws=True, policy=T)
assert err <= TOL["bf16"] and p == T, (err, p)
eh, ey, p = run_swiglu("Q", 16, 2048, 2048, 768, "bf16", seq_len=2047, seed=6, ws=True, policy=T)
assert max(eh, ey) <= TOL["bf16"] and p == T, (eh, ey, p)
print("ok")
"""


def test_unswapped_projection_one_output_group_per_tile():
    # AAL_TC_GROUP_PAIRS=0 and AAL_TC_CLASS_PAIRS=0 (read once per process) keep one
    # output group and one row type per tile
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _ONE_GROUP_CHILD, root], capture_output=True, text=True,
                       timeout=600, env=dict(os.environ, AAL_TC_GROUP_PAIRS="0", AAL_TC_CLASS_PAIRS="0"))
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_swapped_forward_one_class_per_tile():
    # AAL_TC_CLASS_GROUPS=0 (read once per process) keeps one class per tile
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _ONE_CLASS_CHILD, root], capture_output=True, text=True,
                       timeout=600, env=dict(os.environ, AAL_TC_CLASS_GROUPS="0"))
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("M", [0, 1, 7, 130, 1000])
def test_ragged_and_empty_rows(M):
    for law, q, din, dout in (("Q", 4, 256, 512), ("Q2xQ2", 4, 256, 128)):
        if M == 0:
            X = torch.empty(0, din, dtype=torch.bfloat16, device="cuda")
            W = torch.randn(din, dout, device="cuda").to(torch.bfloat16)
            Y = torch.empty(0, dout, dtype=torch.bfloat16, device="cuda")
            aal.aal_project_fwd(law, q, aal.row_rule(seq_len=16), X, W, Y)
            continue
        err, _ = run_project(law, q, M, din, dout, "bf16", seq_len=M)
        assert err <= TOL["bf16"], (law, M, err)


@pytest.mark.parametrize("seq_len,offset", [(100, 0), (64, 3), (1536, 0), (37, 11)])
def test_sequence_packing_and_offset(seq_len, offset):
    err, _ = run_project("Q", 8, 600, 256, 256, "bf16", seq_len=seq_len, offset=offset)
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_explicit_types(dtype):
    err, _ = run_project("Q", 8, 333, 128, 256, dtype, explicit=True)
    assert err <= TOL[dtype], err
    edx, edw, _ = run_bwd("Q", 8, 333, 128, 256, dtype, explicit=True)
    assert edx <= TOL[dtype] and edw <= TOL[dtype]


def test_q1_is_dense():
    err, _ = run_project("Q", 1, 256, 128, 192, "bf16", seq_len=256)
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("q,M,din,dout,ws", [(4, 512, 256, 256, False), (8, 1600, 3072, 256, True)])
def test_bwd_accumulate(q, M, din, dout, ws):
    # dW += X^T dY; with ws the diagonal blocks are split and their reduction adds to dW
    edx, edw, _ = run_bwd("Q", q, M, din, dout, "bf16", seq_len=M, accumulate=True, ws=ws)
    assert edx <= TOL["bf16"] and edw <= TOL["bf16"], (edx, edw)


def test_bwd_split_heavy_tiles_ragged_rows():
    # Q_8 with 200 rows per class (a partial 128-row block) and two column
    # blocks per input group: the heavy dX tiles (a == t, K over every output
    # group) and dW tiles (diagonal blocks, K over every token) run as K pieces
    # whose fp32 partials a reduction kernel adds
    edx, edw, path = run_bwd("Q", 8, 1600, 3072, 256, "bf16", seq_len=1600, ws=True)
    assert edx <= TOL["bf16"] and edw <= TOL["bf16"], (edx, edw)
    assert path == TENSOR


def test_swiglu_bwd_split_heavy_tiles():
    # expert shape with a workspace: dX (both products in one accumulator),
    # dWg, dWu and dWd split their heavy tiles; dH keeps them whole
    errs, got = run_swiglu_bwd("Q", 16, 2048, 2048, 768, "bf16", seed=5, ws=True)
    assert max(errs) <= TOL["bf16"], errs
    assert got == TENSOR


# The general path's dW runs on tiles inside one block (a, k): groups that are
# not multiples of the 64-wide tile, steps of 32 rows with a short last one,
# both laws, accumulation, q = 1.
@pytest.mark.parametrize("law,q,M,din,dout,explicit,accumulate", [
    ("Q", 3, 301, 300, 210, True, False),      # 100 x 70 blocks: partial tiles
    ("Q", 8, 1000, 512, 64, False, True),      # 64 x 8 blocks, dW accumulated
    ("Q2xQ2", 4, 77, 320, 80, True, False),    # 80 x 20 blocks
    ("Q", 1, 45, 96, 48, False, False),        # one group: dense
])
def test_general_path_backward_tiles(law, q, M, din, dout, explicit, accumulate):
    edx, edw, path = run_bwd(law, q, M, din, dout, "f32", explicit=explicit, accumulate=accumulate,
                             seed=M, policy=GENERAL)
    assert edx <= TOL["f32"] and edw <= TOL["f32"] and path == GENERAL, (edx, edw, path)


# The general path's projection and dX run on 64-row tiles that keep, for each
# group of the contraction, only the rows the table applies it to: a partial
# last row tile, groups narrower or wider than a tile, both laws.
@pytest.mark.parametrize("law,q,M,din,dout,explicit,seq_len", [
    ("Q", 3, 301, 300, 210, True, None),
    ("Q2xQ2", 4, 77, 320, 80, True, None),
    ("Q", 8, 1000, 512, 64, False, 37),
    ("Q", 5, 130, 80, 650, False, 130),
])
def test_general_path_projection_tiles(law, q, M, din, dout, explicit, seq_len):
    err, path = run_project(law, q, M, din, dout, "f32", seq_len=seq_len, explicit=explicit, seed=M,
                            policy=GENERAL)
    assert err <= TOL["f32"] and path == GENERAL, (err, path)


def test_general_path_matches_oracle():
    err, path = run_project("Q", 16, 2048, 2048, 768, "bf16", seq_len=2048, policy=GENERAL)
    assert err <= TOL["bf16"] and path == aal.AAL_PATH_GENERAL


def test_out_of_range_explicit_type_sets_device_status():
    q, M, din, dout = 4, 64, 64, 64
    X = torch.randn(M, din, device="cuda").to(torch.bfloat16)
    W = torch.randn(din, dout, device="cuda").to(torch.bfloat16)
    Y = torch.zeros(M, dout, dtype=torch.bfloat16, device="cuda")
    types = torch.zeros(M, dtype=torch.int32, device="cuda")
    types[5] = 9
    aal.aal_project_fwd("Q", q, aal.row_rule(types=types), X, W, Y)
    assert aal.aal_get_device_status() == aal.AAL_ERR_DEVICE_BOUNDS
    assert aal.aal_get_device_status() == aal.AAL_OK  # cleared by the read
    assert torch.all(Y[5] == 0)


def test_negative_decode_position_sets_device_status():
    x = torch.randn(2, 64, device="cuda").to(torch.bfloat16)
    W = torch.randn(64, 64, device="cuda").to(torch.bfloat16)
    y = torch.zeros(2, 64, dtype=torch.bfloat16, device="cuda")
    aal.aal_decode_matvec("Q", 2, torch.tensor([3, -1], device="cuda"), x, W, y)
    assert aal.aal_get_device_status() == aal.AAL_ERR_DEVICE_BOUNDS


# ------------------------------------------------------ CTA-pair tcgen05 mode
_PAIR_CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + '/tests')
from gpu_cases import TOL, run_swiglu, run_project
import associative_algebra_block_b200 as aal
eh, ey, path = run_swiglu('Q2xQ2', 4, 3072, 768, 1536, 'bf16', seq_len=1536)
assert path == aal.AAL_PATH_TENSOR, path
assert eh <= TOL['bf16'] and ey <= TOL['bf16'], (eh, ey)
e, path = run_project('Q', 4, 2048, 512, 1024, 'bf16', seq_len=1024)
assert e <= TOL['bf16'], e
print('ok')
"""


@pytest.mark.gpu
def test_cta_pair_mode_parity():
    # the pair mode is chosen once per process from the environment
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _PAIR_CHILD, root], capture_output=True, text=True,
                       timeout=600, env=dict(os.environ, AAL_TC_PAIR="1"))
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


# ------------------------------------------------- bounded waits run out
_STALL_CHILD = r"""
import os, sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + '/tests')
import torch
from gpu_cases import TOL, run_project
import associative_algebra_block_b200 as aal
from associative_algebra_block_b200 import inputs
X = inputs.projection_inputs(512, 512, 512, seed=3)["X"].t.cuda()
W = inputs.projection_inputs(512, 512, 512, seed=4)["W"].t.cuda()
Y = torch.zeros(512, 512, dtype=torch.bfloat16, device="cuda")
os.environ["AAL_TEST_STALL"] = "1"
aal.aal_set_path_policy(aal.AAL_PATH_TENSOR)
aal.aal_project_fwd("Q", 4, aal.row_rule(seq_len=512), X, W, Y)
st = aal.aal_get_device_status()
del os.environ["AAL_TEST_STALL"]
aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
assert st == aal.AAL_ERR_DEVICE_TIMEOUT, st
assert aal.aal_get_device_status() == aal.AAL_OK  # cleared by the read
# the context is still usable: the same kernel, unstalled, matches the oracle
err, path = run_project("Q", 4, 512, 512, 512, "bf16", seq_len=512, policy=aal.AAL_PATH_TENSOR)
assert path == aal.AAL_PATH_TENSOR and err <= TOL["bf16"], (err, path)
print("ok")
"""


def test_tcgen05_wait_that_runs_out_reports_timeout_and_returns():
    # The test hook makes the MMA thread wait on a barrier nothing arrives on,
    # bounded at 50 ms: the kernel records AAL_ERR_DEVICE_TIMEOUT, lets its
    # copies land, frees TMEM and returns; the next call works normally.
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k != "AAL_TEST_STALL"}
    r = subprocess.run([sys.executable, "-c", _STALL_CHILD, root], capture_output=True, text=True,
                       timeout=600, env=env)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


# ------------------------------------- explicit and ragged row types, tensor path
# With a workspace set, explicit types and sequences that are not whole
# multiples of q run on the tensor cores: rows sorted by type on the device,
# the tcgen05 kernel in segment mode, outputs written back to their rows.
@pytest.mark.parametrize("law,q,M,din,dout,seq_len,explicit", [
    ("Q", 16, 2048, 2048, 768, None, True),        # expert shape, explicit types
    ("Q", 16, 2048, 768, 2048, None, True),
    ("Q2xQ2", 4, 12288, 768, 1536, None, True),    # pilot shape, explicit types
    ("Q2xQ2", 4, 12288, 768, 1536, 1537, False),   # sequences of 1537 positions
    ("Q", 8, 1003, 256, 512, 37, False),           # ragged rows and sequences
    ("Q", 32, 333, 4096, 2048, None, True),        # few rows per type (partial tiles)
    ("Q", 4, 7, 128, 256, None, True),             # fewer rows than types
    ("Q", 5, 1500, 320, 640, None, True),          # odd q: one output group a tile
    ("Q", 4, 1000, 256, 1024, None, True),         # groups too wide to pair
])
def test_explicit_and_ragged_types_tensor_path(law, q, M, din, dout, seq_len, explicit):
    err, path = run_project(law, q, M, din, dout, "bf16", seq_len=seq_len, explicit=explicit,
                            seed=M + q, ws=True, policy=TENSOR)
    assert err <= TOL["bf16"] and path == TENSOR, (err, path)


@pytest.mark.parametrize("law,q,M,D,F,explicit,seq_len", [
    ("Q2xQ2", 4, 3000, 768, 1536, True, None),
    ("Q", 16, 2048, 2048, 768, False, 2047),
])
def test_explicit_and_ragged_types_swiglu_tensor_path(law, q, M, D, F, explicit, seq_len):
    eh, ey, path = run_swiglu(law, q, M, D, F, "bf16", seq_len=seq_len or M, seed=q + M, ws=True,
                              explicit=explicit, policy=TENSOR)
    assert eh <= TOL["bf16"] and ey <= TOL["bf16"] and path == TENSOR, (eh, ey, path)


def test_explicit_types_without_workspace_take_the_general_path():
    err, path = run_project("Q", 8, 333, 128, 256, "bf16", explicit=True)
    assert err <= TOL["bf16"] and path == aal.AAL_PATH_GENERAL
    with pytest.raises(aal.AalError):
        run_project("Q", 8, 333, 128, 256, "bf16", explicit=True, policy=TENSOR)


def test_segment_path_skips_rows_with_an_invalid_type():
    from gpu_cases import workspace
    q, M, din, dout = 4, 300, 128, 256
    X = torch.randn(M, din, device="cuda").to(torch.bfloat16)
    W = torch.randn(din, dout, device="cuda").to(torch.bfloat16)
    Y = torch.zeros(M, dout, dtype=torch.bfloat16, device="cuda")
    types = torch.randint(0, q, (M,), dtype=torch.int32, device="cuda")
    types[17] = -3
    rule = aal.row_rule(types=types)
    with workspace(aal.AAL_CALL_PROJECT_FWD, "Q", q, rule, M, din):
        aal.aal_project_fwd("Q", q, rule, X, W, Y)
        torch.cuda.synchronize()
    assert aal.aal_last_path() == TENSOR
    assert aal.aal_get_device_status() == aal.AAL_ERR_DEVICE_BOUNDS
    assert torch.all(Y[17] == 0)
    keep = torch.arange(M, device="cuda") != 17
    tv = types.cpu().numpy().astype(np.int64)
    ref = oracle.project("Q", q, tv[keep.cpu().numpy()], host64(X)[keep.cpu().numpy()], host64(W))
    assert oracle.rel_err(host64(Y[keep]), ref) <= TOL["bf16"]


# --------------------------------- ragged blocks (groups not multiples of 16)
# The tensor-core path's ragged mode: an input group of 20 features is read
# from the 16-byte aligned start below it with the weight rows outside the
# group read as zeros; output tiles span the 16-column aligned window around
# the group and only the group's columns are written.
@pytest.mark.parametrize("q,M,din,dout,seq_len", [
    (16, 2048, 320, 1600, 2048),    # 20 x 100 blocks, as in the Qwen3-32B shape
    (16, 3200, 320, 1600, 3200),    # 200 tokens per type: partial token tiles
    (8, 1024, 192, 320, 1024),      # 24 x 40 blocks
    (4, 512, 80, 208, 512),         # 20 x 52 blocks
])
def test_ragged_blocks_tensor_path(q, M, din, dout, seq_len):
    err, path = run_project("Q", q, M, din, dout, "bf16", seq_len=seq_len, seed=din + dout, policy=TENSOR)
    assert err <= TOL["bf16"] and path == TENSOR, (err, path)


def test_qwen3_32b_shaped_projection_sampled_rows():
    # M = 32768, D = 5120 -> F = 25600, q = 256 (20 x 100 blocks): NaN-prefilled
    # output; every row finite, and 64 rows (all of one token block, plus rows
    # of other types) against the oracle over all 25600 columns
    law, q, M, D, F = "Q", 256, 32768, 5120, 25600
    ins = inputs.projection_inputs(M, D, F, seed=32, dtype="bf16", want_f64=False)
    X, W = ins["X"].t.cuda(), ins["W"].t.cuda()
    Y = torch.full((M, F), float("nan"), dtype=torch.bfloat16, device="cuda")
    aal.aal_project_fwd(law, q, aal.row_rule(seq_len=M), X, W, Y)
    torch.cuda.synchronize()
    assert aal.aal_last_path() == TENSOR
    assert aal.aal_get_device_status() == aal.AAL_OK
    assert bool(torch.isfinite(Y).all())
    rows = np.concatenate([np.arange(0, 256, 8), np.array([257, 1000, 4095, 9999, 16384, 20000, 30001,
                                                           32767]), np.arange(32512, 32768, 11)])[:64]
    types = oracle.row_types(law, q, inputs.packed_positions(M, M))
    Wf = ins["W"].t.to(torch.float64).numpy()
    Xs = ins["X"].t[torch.as_tensor(rows)].to(torch.float64).numpy()
    ref = oracle.project(law, q, types[rows], Xs, Wf)
    got = host64(Y[torch.as_tensor(rows, device="cuda")])
    assert oracle.rel_err(got, ref) <= TOL["bf16"]


def test_qwen3_1_7b_shaped_projection_full():
    # M = 2048, D = 2048 -> F = 6144, q = 32 (64 x 192 blocks)
    err, path = run_project("Q", 32, 2048, 2048, 6144, "bf16", seq_len=2048, seed=17)
    assert err <= TOL["bf16"] and path == TENSOR, err
