"""Shared helpers for the GPU parity tests: run a libaal call on seeded inputs
and the oracle on the same values, and report max|err| / max|ref|.

Tolerances: bf16 inputs with fp32 accumulation and bf16 outputs: 5e-3;
fp32 throughout: 1e-5 (relative to the largest reference magnitude)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import associative_algebra_block_b200 as aal
from associative_algebra_block_b200 import inputs

TOL = {"bf16": 5e-3, "f32": 1e-5}


def dev(d: inputs.Drawn) -> torch.Tensor:
    return d.t.cuda()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def packed_types(law, q, M, seq_len, offset=0):
    return oracle.row_types(law, q, inputs.packed_positions(M, seq_len, offset))


class workspace:
    """Context manager: a device workspace of the size the call needs, set for
    this thread (aal_set_workspace) while the block runs."""

    def __init__(self, call, law, q, rule, rows, d_in, d_hidden=0, extra=0):
        self.n = aal.aal_workspace_size(call, law, q, rule, rows, d_in, d_hidden) + extra

    def __enter__(self):
        self.buf = torch.empty(max(self.n, 256), dtype=torch.uint8, device="cuda")
        aal.aal_set_workspace(self.buf)
        return self

    def __exit__(self, *a):
        aal.aal_set_workspace(None)


def run_project(law, q, M, din, dout, dtype, seq_len=None, offset=0, explicit=False, seed=0,
                policy=aal.AAL_PATH_AUTO, ws=False):
    ins = inputs.projection_inputs(M, din, dout, seed=seed, dtype=dtype)
    X, W = dev(ins["X"]), dev(ins["W"])
    Y = torch.full((M, dout), float("nan"), dtype=X.dtype, device="cuda")
    if explicit:
        tv = inputs.Stream(seed + 1).labels(M, q)
        types_t = torch.from_numpy(tv).cuda()
        rule = aal.row_rule(types=types_t)
        types = tv.astype(np.int64)
    else:
        seq_len = seq_len or max(M, 1)
        rule = aal.row_rule(seq_len=seq_len, pos_offset=offset)
        types = packed_types(law, q, M, seq_len, offset)
    aal.aal_set_path_policy(policy)
    try:
        if ws:
            with workspace(aal.AAL_CALL_PROJECT_FWD, law, q, rule, M, din):
                aal.aal_project_fwd(law, q, rule, X, W, Y)
                torch.cuda.synchronize()
        else:
            aal.aal_project_fwd(law, q, rule, X, W, Y)
            torch.cuda.synchronize()
        path = aal.aal_last_path()
    finally:
        aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
    assert aal.aal_get_device_status() == aal.AAL_OK
    ref = oracle.project(law, q, types, ins["X"].f64, ins["W"].f64)
    return oracle.rel_err(host64(Y), ref), path


def run_square(law, q, n, dtype, seed=0, policy=aal.AAL_PATH_AUTO):
    ins = inputs.square_inputs(n, seed=seed, dtype=dtype)
    X, W = dev(ins["X"]), dev(ins["W"])
    Z = torch.full((n, n), float("nan"), dtype=X.dtype, device="cuda")
    aal.aal_set_path_policy(policy)
    try:
        aal.aal_square_product(law, q, X, W, Z)
        torch.cuda.synchronize()
        path = aal.aal_last_path()
    finally:
        aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
    ref = oracle.square_product(law, q, ins["X"].f64, ins["W"].f64) if q <= 8 else None
    if ref is None:
        b = n // q
        ref = np.zeros((n, n))
        Xf, Wf = ins["X"].f64, ins["W"].f64
        for i in range(q):
            for k in range(q):
                ref[i * b:(i + 1) * b, k * b:(k + 1) * b] = oracle.square_tile(
                    law, q, i, k, lambda r, c: Xf[r * b:(r + 1) * b, c * b:(c + 1) * b],
                    lambda r, c: Wf[r * b:(r + 1) * b, c * b:(c + 1) * b])
    return oracle.rel_err(host64(Z), ref), path


def run_swiglu(law, q, M, D, F, dtype, seq_len, w_sigma_rule="din", seed=0,
               policy=aal.AAL_PATH_AUTO, rows=None, ws=False, explicit=False):
    ins = inputs.swiglu_inputs(D, F, M, seed=seed, dtype=dtype, w_sigma_rule=w_sigma_rule)
    X, Wg, Wu, Wd = (dev(ins[k]) for k in ("X", "Wg", "Wu", "Wd"))
    H = torch.full((M, F), float("nan"), dtype=X.dtype, device="cuda")
    Y = torch.full((M, D), float("nan"), dtype=X.dtype, device="cuda")
    if explicit:
        tv = inputs.Stream(seed + 1).labels(M, q)
        rule = aal.row_rule(types=torch.from_numpy(tv).cuda())
        types = tv.astype(np.int64)
    else:
        rule = aal.row_rule(seq_len=seq_len)
        types = packed_types(law, q, M, seq_len)
    aal.aal_set_path_policy(policy)
    try:
        if ws:
            with workspace(aal.AAL_CALL_SWIGLU_FWD, law, q, rule, M, D, F):
                aal.aal_swiglu_fwd(law, q, rule, X, Wg, Wu, Wd, H, Y)
                torch.cuda.synchronize()
        else:
            aal.aal_swiglu_fwd(law, q, rule, X, Wg, Wu, Wd, H, Y)
            torch.cuda.synchronize()
        path = aal.aal_last_path()
    finally:
        aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
    if rows is None:
        Href, Yref = oracle.swiglu(law, q, types, ins["X"].f64, ins["Wg"].f64, ins["Wu"].f64, ins["Wd"].f64)
        Hg, Yg = host64(H), host64(Y)
    else:
        Href, Yref = oracle.swiglu_rows(law, q, types, ins["X"].f64, ins["Wg"].f64, ins["Wu"].f64,
                                        ins["Wd"].f64, rows)
        Hg, Yg = host64(H[torch.as_tensor(rows, device="cuda")]), host64(Y[torch.as_tensor(rows, device="cuda")])
    return oracle.rel_err(Hg, Href), oracle.rel_err(Yg, Yref), path


def run_bwd(law, q, M, din, dout, dtype, seq_len=None, explicit=False, seed=0, accumulate=False,
            policy=aal.AAL_PATH_AUTO, ws=False):
    ins = inputs.projection_inputs(M, din, dout, seed=seed, dtype=dtype, with_dy=True)
    X, W, dY = dev(ins["X"]), dev(ins["W"]), dev(ins["dY"])
    dX = torch.full((M, din), float("nan"), dtype=X.dtype, device="cuda")
    if accumulate:
        base = inputs.Stream(seed + 7).normal(din, dout, 1.0, dtype)
        dW = base.t.cuda()
    else:
        base = None
        dW = torch.full((din, dout), float("nan"), dtype=X.dtype, device="cuda")
    if explicit:
        tv = inputs.Stream(seed + 1).labels(M, q)
        rule = aal.row_rule(types=torch.from_numpy(tv).cuda())
        types = tv.astype(np.int64)
    else:
        seq_len = seq_len or max(M, 1)
        rule = aal.row_rule(seq_len=seq_len)
        types = packed_types(law, q, M, seq_len)
    aal.aal_set_path_policy(policy)
    try:
        if ws:
            with workspace(aal.AAL_CALL_PROJECT_BWD, law, q, rule, M, din, dout) as w:
                assert w.n > 0
                aal.aal_project_bwd(law, q, rule, X, W, dY, dX, dW, accumulate_dW=accumulate)
                torch.cuda.synchronize()
        else:
            aal.aal_project_bwd(law, q, rule, X, W, dY, dX, dW, accumulate_dW=accumulate)
            torch.cuda.synchronize()
        path = aal.aal_last_path()
    finally:
        aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
    assert aal.aal_get_device_status() == aal.AAL_OK
    rdX, rdW = oracle.project_bwd(law, q, types, ins["X"].f64, ins["W"].f64, ins["dY"].f64)
    if base is not None:
        rdW = rdW + base.f64
    return oracle.rel_err(host64(dX), rdX), oracle.rel_err(host64(dW), rdW), path


def run_decode(law, q, B, din, dout, dtype, seq_len=1536, seed=0, same_type=None):
    s = inputs.Stream(seed)
    x = s.normal(B, din, 1.0, dtype)
    W = s.normal(din, dout, din ** -0.5, dtype)
    pos = s.positions(B, seq_len)
    if same_type is not None:
        pos = (pos - pos % q + same_type).astype(np.int64)
    y = torch.full((B, dout), float("nan"), dtype=x.t.dtype, device="cuda")
    aal.aal_decode_matvec(law, q, torch.from_numpy(pos).cuda(), x.t.cuda(), W.t.cuda(), y)
    torch.cuda.synchronize()
    path = aal.aal_last_path()
    ref = oracle.decode(law, q, pos, x.f64, W.f64)
    return oracle.rel_err(host64(y), ref), path


def run_swiglu_decode(law, q, B, D, F, dtype, seq_len=1536, seed=0, same_type=None,
                      policy=aal.AAL_PATH_AUTO):
    s = inputs.Stream(seed)
    x = s.normal(B, D, 1.0, dtype)
    Wg = s.normal(D, F, D ** -0.5, dtype)
    Wu = s.normal(D, F, D ** -0.5, dtype)
    Wd = s.normal(F, D, F ** -0.5, dtype)
    pos = s.positions(B, seq_len)
    if same_type is not None:
        pos = (pos - pos % q + same_type).astype(np.int64)
    h = torch.full((B, F), float("nan"), dtype=x.t.dtype, device="cuda")
    y = torch.full((B, D), float("nan"), dtype=x.t.dtype, device="cuda")
    aal.aal_set_path_policy(policy)
    try:
        aal.aal_swiglu_decode(law, q, torch.from_numpy(pos).cuda(), x.t.cuda(), Wg.t.cuda(),
                              Wu.t.cuda(), Wd.t.cuda(), h, y)
        torch.cuda.synchronize()
        path = aal.aal_last_path()
    finally:
        aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
    assert aal.aal_get_device_status() == aal.AAL_OK
    H, Y = oracle.swiglu_decode(law, q, pos, x.f64, Wg.f64, Wu.f64, Wd.f64)
    return oracle.rel_err(host64(h), H), oracle.rel_err(host64(y), Y), path


def run_swiglu_bwd(law, q, M, D, F, dtype, seq_len=None, seed=0, explicit=False,
                   policy=aal.AAL_PATH_AUTO, ws=False):
    ins = inputs.swiglu_inputs(D, F, M, seed=seed, dtype=dtype)
    X, Wg, Wu, Wd = (dev(ins[k]) for k in ("X", "Wg", "Wu", "Wd"))
    dYd = inputs.Stream(seed + 7).normal(M, D, 1.0, dtype)
    dY = dev(dYd)
    if explicit:
        tv = inputs.Stream(seed + 1).labels(M, q)
        types_t = torch.from_numpy(tv).cuda()  # the rule holds only its pointer
        rule = aal.row_rule(types=types_t)
        types = tv.astype(np.int64)
    else:
        seq_len = seq_len or M
        rule = aal.row_rule(seq_len=seq_len)
        types = packed_types(law, q, M, seq_len)
    H = torch.empty(M, F, dtype=X.dtype, device="cuda")
    Y = torch.empty(M, D, dtype=X.dtype, device="cuda")
    aal.aal_set_path_policy(policy)
    try:
        aal.aal_swiglu_fwd(law, q, rule, X, Wg, Wu, Wd, H, Y)
        hs = [torch.full((M, F), float("nan"), dtype=X.dtype, device="cuda") for _ in range(4)]
        outs = [torch.full(t.shape, float("nan"), dtype=X.dtype, device="cuda") for t in (X, Wg, Wu, Wd)]
        if ws:
            with workspace(aal.AAL_CALL_SWIGLU_BWD, law, q, rule, M, D, F) as w:
                assert w.n > 0
                aal.aal_swiglu_bwd(law, q, rule, X, Wg, Wu, Wd, H, dY, *hs, *outs)
                torch.cuda.synchronize()
        else:
            aal.aal_swiglu_bwd(law, q, rule, X, Wg, Wu, Wd, H, dY, *hs, *outs)
            torch.cuda.synchronize()
        path = aal.aal_last_path()
    finally:
        aal.aal_set_path_policy(aal.AAL_PATH_AUTO)
    assert aal.aal_get_device_status() == aal.AAL_OK
    ref = oracle.swiglu_bwd(law, q, types, ins["X"].f64, ins["Wg"].f64, ins["Wu"].f64, ins["Wd"].f64,
                            dYd.f64)
    return [oracle.rel_err(host64(o), r) for o, r in zip(outs, ref)], path
