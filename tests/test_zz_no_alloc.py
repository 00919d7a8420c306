"""The FFN decode entry point that allocates nothing (aal_swiglu_decode_noalloc).

Callers that cannot allocate device memory (a plug-in whose host application
owns every device allocation, a real-time loop that may not take cudaMalloc's
device-wide synchronisation) use this variant: the activation h lives in the
library's fixed device array instead of a caller buffer.  Its results must
equal those of aal_swiglu_decode, which takes h from the caller, on the same
inputs; two calls in a row check that the shared array's leftover contents
from the first call do not leak into the second.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import associative_algebra_block_b200 as aal
from associative_algebra_block_b200 import inputs

TOL_BF16 = 5e-3  # max|err| / max|ref|, the bf16 tolerance of every parity test


def _ffn_weights(D, F, seed):
    s = inputs.Stream(seed)
    return [s.normal(D, F, D ** -0.5, "bf16", want_f64=False).t.cuda(),
            s.normal(D, F, D ** -0.5, "bf16", want_f64=False).t.cuda(),
            s.normal(F, D, F ** -0.5, "bf16", want_f64=False).t.cuda()]


def _decode_batch(B, D, seed):
    s = inputs.Stream(seed)
    x = s.normal(B, D, 1.0, "bf16", want_f64=False).t.cuda()
    pos = torch.from_numpy(s.positions(B, 1536)).cuda()
    return x, pos


def _rel(a, b):
    return oracle.rel_err(a.to("cpu", torch.float64).numpy(), b.to("cpu", torch.float64).numpy())


@pytest.mark.gpu
def test_noalloc_ffn_decode_equals_swiglu_decode_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    aal.load()
    law, q, D, F = "Q2xQ2", 4, 768, 1536
    Wg, Wu, Wd = _ffn_weights(D, F, seed=500)
    # two calls in a row with different inputs and batch sizes; the second
    # writes fewer rows of the shared array than the first left behind
    for call, B in enumerate((64, 8)):
        x, pos = _decode_batch(B, D, seed=510 + call)
        h_ref = torch.full((B, F), float("nan"), dtype=torch.bfloat16, device="cuda")
        y_ref = torch.full((B, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        aal.aal_swiglu_decode(law, q, pos, x, Wg, Wu, Wd, h_ref, y_ref)
        y = torch.full((B, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        aal.aal_swiglu_decode_noalloc(law, q, pos, x, Wg, Wu, Wd, y)
        torch.cuda.synchronize()
        assert aal.aal_get_device_status() == aal.AAL_OK
        assert bool(torch.isfinite(y).all()), f"call {call}: rows left unwritten"
        err = _rel(y, y_ref)
        assert err <= TOL_BF16, (call, err)


@pytest.mark.gpu
def test_noalloc_ffn_decode_rejects_a_batch_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    aal.load()
    D, F = 768, 1536
    B = 1366  # 1366 * 1536 bf16 values are more than the 4 MiB array holds
    Wg, Wu, Wd = _ffn_weights(D, F, seed=520)
    x, pos = _decode_batch(B, D, seed=521)
    y = torch.zeros(B, D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(aal.AalError) as e:
        aal.aal_swiglu_decode_noalloc("Q2xQ2", 4, pos, x, Wg, Wu, Wd, y)
    assert e.value.status == aal.AAL_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((y == 0).all())  # nothing was launched
    # the largest batch that fits still runs and matches aal_swiglu_decode
    B = 1365
    x, pos = _decode_batch(B, D, seed=522)
    h_ref = torch.empty(B, F, dtype=torch.bfloat16, device="cuda")
    y_ref = torch.empty(B, D, dtype=torch.bfloat16, device="cuda")
    aal.aal_swiglu_decode("Q2xQ2", 4, pos, x, Wg, Wu, Wd, h_ref, y_ref)
    y = torch.full((B, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    aal.aal_swiglu_decode_noalloc("Q2xQ2", 4, pos, x, Wg, Wu, Wd, y)
    torch.cuda.synchronize()
    assert aal.aal_get_device_status() == aal.AAL_OK
    assert _rel(y, y_ref) <= TOL_BF16
