"""torch.autograd wrapper of the algebraic SwiGLU FFN (libaal calls only).

``swiglu(law, q, rule, X, Wg, Wu, Wd)`` returns Y = (silu(X*Wg) . (X*Wu)) * Wd
with every product row-typed, and differentiates through ``aal_swiglu_bwd``.
The forward keeps its activation H for the backward; the backward allocates
the pre-activation and gradient workspaces it passes to the library.  All
arithmetic runs in the CUDA library.
"""
from __future__ import annotations

import torch

from . import aal_swiglu_bwd, aal_swiglu_fwd


class _SwiGLU(torch.autograd.Function):
    @staticmethod
    def forward(ctx, law, q, rule, X, Wg, Wu, Wd):
        M, D, F = X.shape[0], X.shape[1], Wg.shape[1]
        H = torch.empty(M, F, dtype=X.dtype, device=X.device)
        Y = torch.empty(M, D, dtype=X.dtype, device=X.device)
        aal_swiglu_fwd(law, q, rule, X, Wg, Wu, Wd, H, Y)
        ctx.law, ctx.q, ctx.rule = law, q, rule
        ctx.save_for_backward(X, Wg, Wu, Wd, H)
        return Y

    @staticmethod
    def backward(ctx, dY):
        X, Wg, Wu, Wd, H = ctx.saved_tensors
        dY = dY.contiguous()
        ws = [torch.empty_like(H) for _ in range(4)]  # G, U, dG, dU
        dX, dWg, dWu, dWd = (torch.empty_like(t) for t in (X, Wg, Wu, Wd))
        aal_swiglu_bwd(ctx.law, ctx.q, ctx.rule, X, Wg, Wu, Wd, H, dY, *ws, dX, dWg, dWu, dWd)
        return None, None, None, dX, dWg, dWu, dWd


def swiglu(law, q, rule, X, Wg, Wu, Wd):
    """Differentiable algebraic SwiGLU FFN on row-major CUDA tensors."""
    return _SwiGLU.apply(law, q, rule, X, Wg, Wu, Wd)
