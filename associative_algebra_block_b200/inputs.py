"""Seeded synthetic inputs for the row-typed block projection.

This module draws random numbers and nothing else: it holds none of the
algebra's arithmetic (no block table, no row-type rule, no products).  Both
the CUDA path (through the tests and the benchmark) and the CPU oracle take
their inputs from here, so the two sides see bit-identical operands.

Recipe (one numpy PCG64 stream per call, ``numpy.random.default_rng(seed)``):

* matrices are drawn in the order the caller asks for them, each as float32
  ``standard_normal`` times ``sigma`` (row chunks of the same stream for large
  matrices), then rounded to bfloat16 with round-to-nearest-even when the
  dtype is bf16;
* integer matrices are uniform in ``[lo, hi]``;
* decode positions are uniform in ``[0, seq_len)``.

Every tensor is returned twice: as a CPU ``torch`` tensor in the compute
dtype (what gets copied to the GPU) and as its exact float64 widening (what
the oracle reads).  Widening bf16 or fp32 to fp64 is exact.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

_CHUNK_ELEMS = 1 << 26  # row-chunked drawing for very large matrices


def _torch_dtype(dtype: str) -> torch.dtype:
    if dtype == "bf16":
        return torch.bfloat16
    if dtype == "f32":
        return torch.float32
    raise ValueError(f"unknown dtype {dtype!r}")


@dataclasses.dataclass
class Drawn:
    """One synthetic tensor: ``t`` in the compute dtype (CPU), ``f64`` exact."""

    t: torch.Tensor
    f64: np.ndarray


class Stream:
    """A seeded generator; successive draws continue the same stream."""

    def __init__(self, seed: int = 0):
        self.rng = np.random.default_rng(seed)

    def normal(self, rows: int, cols: int, sigma: float, dtype: str,
               want_f64: bool = True) -> Drawn:
        tdt = _torch_dtype(dtype)
        out = torch.empty((rows, cols), dtype=tdt)
        step = max(1, _CHUNK_ELEMS // max(cols, 1))
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            chunk = self.rng.standard_normal((r1 - r0, cols), dtype=np.float32)
            chunk *= np.float32(sigma)
            # torch's float32 -> bfloat16 conversion rounds to nearest even
            out[r0:r1] = torch.from_numpy(chunk).to(tdt)
        f64 = out.to(torch.float64).numpy() if want_f64 else None
        return Drawn(out, f64)

    def integers(self, rows: int, cols: int, lo: int, hi: int, dtype: str) -> Drawn:
        vals = self.rng.integers(lo, hi + 1, size=(rows, cols)).astype(np.float32)
        t = torch.from_numpy(vals).to(_torch_dtype(dtype))
        return Drawn(t, t.to(torch.float64).numpy())

    def positions(self, count: int, seq_len: int) -> np.ndarray:
        return self.rng.integers(0, seq_len, size=count).astype(np.int64)

    def labels(self, count: int, num: int) -> np.ndarray:
        """Uniform integers in [0, num): used for explicit per-row type arrays."""
        return self.rng.integers(0, num, size=count).astype(np.int32)


def packed_positions(rows: int, seq_len: int, offset: int = 0) -> np.ndarray:
    """Absolute position of each row when ``rows`` tokens are packed as
    back-to-back sequences of ``seq_len`` tokens (the last one may be short),
    each starting at ``offset``."""
    return (np.arange(rows, dtype=np.int64) % seq_len) + offset


# --------------------------------------------------------------------------
# The five workloads.  Each returns a dict of Drawn tensors plus the shape
# parameters; sizes follow the shapes of the pages' workloads.
# --------------------------------------------------------------------------

CONFIGS = {
    # Q_2, fp32, 64 tokens, 64 -> 64
    "c1": dict(law="Q", q=2, M=64, din=64, dout=64, seq_len=64, dtype="f32"),
    # Q2 (x) Q2 SwiGLU FFN of the 110M pilot: 8 sequences of 1536 tokens
    "c2": dict(law="Q2xQ2", q=4, M=12288, D=768, F=1536, seq_len=1536, dtype="bf16"),
    # Qwen3-8B-shaped SwiGLU under Q_32
    "c3": dict(law="Q", q=32, M=2048, D=4096, F=12288, seq_len=2048, dtype="bf16"),
    # Qwen3-30B-A3B-expert-shaped narrow FFN under Q_16
    "c4": dict(law="Q", q=16, M=2048, D=2048, F=768, seq_len=2048, dtype="bf16"),
    # fixed-block square product under Q_256
    "c5": dict(law="Q", q=256, n=32768, b=128, dtype="bf16"),
}


def swiglu_inputs(D: int, F: int, M: int, seed: int = 0, dtype: str = "bf16",
                  w_sigma_rule: str = "din", want_f64: bool = True):
    """X [M, D] ~ N(0,1); Wg, Wu [D, F] and Wd [F, D] ~ N(0, 1/fan), where
    fan is the projection's input width (``"din"``) or D for all three
    (``"D"``).  Draw order: X, Wg, Wu, Wd."""
    s = Stream(seed)
    X = s.normal(M, D, 1.0, dtype, want_f64)
    fan_d = D
    fan_f = D if w_sigma_rule == "D" else F
    Wg = s.normal(D, F, fan_d ** -0.5, dtype, want_f64)
    Wu = s.normal(D, F, fan_d ** -0.5, dtype, want_f64)
    Wd = s.normal(F, D, fan_f ** -0.5, dtype, want_f64)
    return dict(X=X, Wg=Wg, Wu=Wu, Wd=Wd)


def projection_inputs(M: int, din: int, dout: int, seed: int = 0,
                      dtype: str = "bf16", with_dy: bool = False,
                      want_f64: bool = True):
    """X [M, din] ~ N(0,1), W [din, dout] ~ N(0, 1/din), optionally
    dY [M, dout] ~ N(0,1).  Draw order: X, W, dY."""
    s = Stream(seed)
    out = dict(X=s.normal(M, din, 1.0, dtype, want_f64),
               W=s.normal(din, dout, din ** -0.5, dtype, want_f64))
    if with_dy:
        out["dY"] = s.normal(M, dout, 1.0, dtype, want_f64)
    return out


def square_inputs(n: int, seed: int = 0, dtype: str = "bf16", sigma: float | None = None,
                  want_f64: bool = True):
    """X, W [n, n] ~ N(0, sigma^2) with sigma = 1/sqrt(n) by default."""
    s = Stream(seed)
    sg = n ** -0.5 if sigma is None else sigma
    return dict(X=s.normal(n, n, sg, dtype, want_f64), W=s.normal(n, n, sg, dtype, want_f64))


def integer_square_inputs(n: int, count: int = 3, lo: int = -3, hi: int = 3,
                          seed: int = 0, dtype: str = "f32"):
    """``count`` n x n matrices of integers in [lo, hi] (exact in any dtype)."""
    s = Stream(seed)
    return [s.integers(n, n, lo, hi, dtype) for _ in range(count)]
