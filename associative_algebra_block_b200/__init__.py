"""Python binding of libaal (argument marshalling only).

Every function below has the name of the C entry point it calls and forwards
torch tensors as ``aal_mat`` descriptors (device pointer, dtype, rows, cols,
leading dimension).  All arithmetic happens in the CUDA library; this module
only checks that tensors are 2-D, row-major and on the GPU, and raises
``AalError`` for a non-OK status.  The library is loaded on first use and a
missing ``libaal.so`` is an error (build it with ``__graft_entry__.build()``
or ``python -m associative_algebra_block_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libaal.so")

# status codes (include/aal.h)
AAL_OK = 0
AAL_ERR_INVALID_ARG = 1
AAL_ERR_UNSUPPORTED = 2
AAL_ERR_ALIGNMENT = 3
AAL_ERR_CUDA = 4
AAL_ERR_DEVICE_TIMEOUT = 5
AAL_ERR_DEVICE_BOUNDS = 6
AAL_ERR_SCRATCH_LIMIT = 7

LAW = {"Q": 0, "Q2xQ2": 1}
AAL_BF16, AAL_F32 = 0, 1
AAL_TYPES_POSITION, AAL_TYPES_EXPLICIT = 0, 1
AAL_PATH_AUTO, AAL_PATH_TENSOR, AAL_PATH_GENERAL, AAL_PATH_DECODE = 0, 1, 2, 3
AAL_CALL_PROJECT_FWD, AAL_CALL_SWIGLU_FWD, AAL_CALL_PROJECT_BWD, AAL_CALL_SWIGLU_BWD = 1, 2, 3, 4

EXPORTS = ("aal_project_fwd", "aal_swiglu_fwd", "aal_project_bwd", "aal_decode_matvec",
           "aal_swiglu_decode", "aal_swiglu_bwd", "aal_square_product", "aal_block_table", "aal_block_product_count",
           "aal_get_device_status", "aal_status_string", "aal_set_path_policy",
           "aal_last_path", "aal_launch_count", "aal_version", "aal_set_timing_events",
           "aal_swiglu_decode_noalloc", "aal_workspace_size", "aal_set_workspace")
AAL_KERNEL_PROJECT, AAL_KERNEL_GATE_UP, AAL_KERNEL_BWD_DX = 1, 2, 3
AAL_KERNEL_BWD_DW, AAL_KERNEL_SQUARE, AAL_KERNEL_DECODE = 4, 5, 6
AAL_KERNEL_DECODE_GATE_UP, AAL_KERNEL_SWIGLU_BWD, AAL_KERNEL_FFN_DECODE = 7, 8, 9


class AalError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class AalMat(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("ld", ctypes.c_int64)]


class AalRowTypeRule(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("seq_len", ctypes.c_int64),
                ("pos_offset", ctypes.c_int64), ("types", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libaal.so (once) and declare the C signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libaal.so is not built ({p}); run __graft_entry__.build()")
        lib = ctypes.CDLL(p)
        i32, i64, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
        sig = {
            "aal_project_fwd": ([i32, i32, AalRowTypeRule, AalMat, AalMat, AalMat, vp], i32),
            "aal_swiglu_fwd": ([i32, i32, AalRowTypeRule, AalMat, AalMat, AalMat, AalMat, AalMat,
                                AalMat, vp], i32),
            "aal_swiglu_decode": ([i32, i32, vp, AalMat, AalMat, AalMat, AalMat, AalMat, AalMat, vp],
                                  i32),
            "aal_swiglu_bwd": ([i32, i32, AalRowTypeRule] + [AalMat] * 14 + [vp], i32),
            "aal_swiglu_decode_noalloc": ([i32, i32, vp, AalMat, AalMat, AalMat, AalMat, AalMat, vp],
                                          i32),
            "aal_project_bwd": ([i32, i32, AalRowTypeRule, AalMat, AalMat, AalMat, AalMat, AalMat,
                                 i32, vp], i32),
            "aal_decode_matvec": ([i32, i32, vp, AalMat, AalMat, AalMat, vp], i32),
            "aal_square_product": ([i32, i32, AalMat, AalMat, AalMat, vp], i32),
            "aal_block_table": ([i32, i32, vp], i32),
            "aal_block_product_count": ([i32, i32, i32], i64),
            "aal_get_device_status": ([vp], i32),
            "aal_status_string": ([i32], ctypes.c_char_p),
            "aal_set_path_policy": ([i32], i32),
            "aal_last_path": ([], i32),
            "aal_launch_count": ([i32], i64),
            "aal_version": ([], i32),
            "aal_set_timing_events": ([i32, vp, vp], i32),
            "aal_workspace_size": ([i32, i32, i32, AalRowTypeRule, i64, i64, i64], i64),
            "aal_set_workspace": ([vp, ctypes.c_uint64], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().aal_status_string(int(status)).decode()


def _law(law) -> int:
    if isinstance(law, str):
        return LAW[law]
    return int(law)


def _check(status: int, where: str):
    if status != AAL_OK:
        raise AalError(status, where)


def mat(t: torch.Tensor | None) -> AalMat:
    """aal_mat view of a 2-D row-major tensor (None -> a NULL descriptor)."""
    if t is None:
        return AalMat(None, AAL_BF16, 0, 0, 0)
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor")
    if t.dtype == torch.bfloat16:
        dt = AAL_BF16
    elif t.dtype == torch.float32:
        dt = AAL_F32
    else:
        raise ValueError(f"unsupported dtype {t.dtype}")
    rows, cols = t.shape
    if rows > 0 and cols > 1 and t.stride(1) != 1:
        raise ValueError("tensor must be row-major (unit column stride)")
    ld = t.stride(0) if rows > 1 else max(cols, 1)
    if t.numel() > 0 and not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    return AalMat(t.data_ptr() if t.numel() > 0 else None, dt, rows, cols, max(ld, cols))


def _index_vector(t: torch.Tensor, dtype: torch.dtype, n: int, what: str, like: torch.Tensor | None):
    """Checks an index tensor the kernels read directly: ``dtype``, 1-D,
    contiguous, exactly ``n`` entries, and (when it has entries) on the CUDA
    device of ``like``.  A host or short tensor would make a kernel read the
    wrong memory, so it is refused here."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{what} must be a torch tensor")
    if t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}")
    if t.dim() != 1:
        raise ValueError(f"{what} must be 1-D")
    if t.numel() != n:
        raise ValueError(f"{what} must have {n} entries (has {t.numel()})")
    if n == 0:
        return
    if not t.is_cuda:
        raise ValueError(f"{what} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if like is not None and like.numel() > 0 and like.device != t.device:
        raise ValueError(f"{what} is on {t.device}, the matrices on {like.device}")


def _checked_rule(rule, rows: int, like: torch.Tensor | None):
    """An explicit-type rule's tensor must hold one int32 type per row."""
    if rule.kind == AAL_TYPES_EXPLICIT:
        types = getattr(rule, "_types", None)
        if types is None:
            if rows > 0:
                raise ValueError("explicit row types: build the rule with row_rule(types=...)")
        else:
            _index_vector(types, torch.int32, rows, "types", like)
    return rule


def row_rule(seq_len: int | None = None, pos_offset: int = 0,
             types: torch.Tensor | None = None) -> AalRowTypeRule:
    """Row-type rule: position-derived (packed sequences of ``seq_len``) or
    an explicit int32 device tensor of types."""
    if types is not None:
        if types.dtype != torch.int32:
            raise ValueError("types must be int32")
        rule = AalRowTypeRule(AAL_TYPES_EXPLICIT, 0, 0, types.data_ptr() if types.numel() else None)
        rule._types = types  # the C struct holds only the pointer: keep the tensor alive with it
        return rule
    if seq_len is None:
        raise ValueError("give seq_len or types")
    return AalRowTypeRule(AAL_TYPES_POSITION, int(seq_len), int(pos_offset), None)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int | None:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def aal_project_fwd(law, q, rule, X, W, Y, stream=None):
    rule = _checked_rule(rule, X.shape[0], X)
    _check(load().aal_project_fwd(_law(law), q, rule, mat(X), mat(W), mat(Y), _stream(stream)),
           "aal_project_fwd")


def aal_swiglu_fwd(law, q, rule, X, Wg, Wu, Wd, H, Y, stream=None):
    rule = _checked_rule(rule, X.shape[0], X)
    _check(load().aal_swiglu_fwd(_law(law), q, rule, mat(X), mat(Wg), mat(Wu), mat(Wd), mat(H),
                                 mat(Y), _stream(stream)), "aal_swiglu_fwd")


def aal_project_bwd(law, q, rule, X, W, dY, dX=None, dW=None, accumulate_dW=False, stream=None):
    rule = _checked_rule(rule, X.shape[0], X)
    _check(load().aal_project_bwd(_law(law), q, rule, mat(X), mat(W), mat(dY), mat(dX), mat(dW),
                                  int(bool(accumulate_dW)), _stream(stream)), "aal_project_bwd")


def aal_decode_matvec(law, q, positions, x, W, y, stream=None):
    _index_vector(positions, torch.int64, x.shape[0], "positions", x)
    _check(load().aal_decode_matvec(_law(law), q, positions.data_ptr() if positions.numel() else None,
                                    mat(x), mat(W), mat(y), _stream(stream)), "aal_decode_matvec")


def aal_swiglu_bwd(law, q, rule, X, Wg, Wu, Wd, H, dY, G, U, dG, dU, dX, dWg, dWu, dWd, stream=None):
    rule = _checked_rule(rule, X.shape[0], X)
    _check(load().aal_swiglu_bwd(_law(law), q, rule, *(mat(t) for t in (X, Wg, Wu, Wd, H, dY, G, U, dG,
                                                                         dU, dX, dWg, dWu, dWd)),
                                 _stream(stream)), "aal_swiglu_bwd")


def aal_swiglu_decode(law, q, positions, x, Wg, Wu, Wd, h, y, stream=None):
    _index_vector(positions, torch.int64, x.shape[0], "positions", x)
    _check(load().aal_swiglu_decode(_law(law), q, positions.data_ptr() if positions.numel() else None,
                                    mat(x), mat(Wg), mat(Wu), mat(Wd), mat(h), mat(y), _stream(stream)),
           "aal_swiglu_decode")


def aal_swiglu_decode_noalloc(law, q, positions, x, Wg, Wu, Wd, y, stream=None):
    """aal_swiglu_decode with the activation kept in the library's fixed
    device array (for callers that cannot allocate device memory)."""
    _index_vector(positions, torch.int64, x.shape[0], "positions", x)
    _check(load().aal_swiglu_decode_noalloc(_law(law), q,
                                            positions.data_ptr() if positions.numel() else None,
                                            mat(x), mat(Wg), mat(Wu), mat(Wd), mat(y), _stream(stream)),
           "aal_swiglu_decode_noalloc")


def aal_square_product(law, q, X, W, Z, stream=None):
    _check(load().aal_square_product(_law(law), q, mat(X), mat(W), mat(Z), _stream(stream)),
           "aal_square_product")


def aal_block_table(law, q) -> np.ndarray:
    S = np.zeros(q * q * q, dtype=np.uint8)
    _check(load().aal_block_table(_law(law), q, S.ctypes.data), "aal_block_table")
    return S.reshape(q, q, q)


def aal_block_product_count(law, q, row_typed) -> int:
    return int(load().aal_block_product_count(_law(law), q, int(bool(row_typed))))


def aal_get_device_status(stream=None) -> int:
    return int(load().aal_get_device_status(_stream(stream)))


def aal_status_string(status) -> str:
    return status_string(status)


def aal_set_path_policy(policy: int):
    _check(load().aal_set_path_policy(int(policy)), "aal_set_path_policy")


def aal_last_path() -> int:
    return int(load().aal_last_path())


def aal_launch_count(reset: bool = False) -> int:
    return int(load().aal_launch_count(int(bool(reset))))


def aal_set_timing_events(kernel: int, before=None, after=None):
    """Record torch.cuda.Event ``before``/``after`` around the next launch of
    ``kernel`` (an AAL_KERNEL_* kind) on this thread."""
    b = before.cuda_event if before is not None else None
    a = after.cuda_event if after is not None else None
    _check(load().aal_set_timing_events(int(kernel), b, a), "aal_set_timing_events")


def aal_workspace_size(call, law, q, rule, rows, d_in, d_hidden=0) -> int:
    """Bytes of device workspace the call uses: the forward calls for explicit
    or ragged row types, the backward calls to split their heavy Q_q tiles
    (0: none used)."""
    n = int(load().aal_workspace_size(int(call), _law(law), q, rule, int(rows), int(d_in), int(d_hidden)))
    if n < 0:
        raise ValueError("aal_workspace_size: invalid arguments")
    return n


_workspace_keep = threading.local()


def aal_set_workspace(buf: torch.Tensor | None):
    """Device workspace (a CUDA tensor, kept alive by the binding until the
    next call here on this thread) for the following calls of this thread;
    None removes it."""
    if buf is None:
        _check(load().aal_set_workspace(None, 0), "aal_set_workspace")
        _workspace_keep.t = None
        return
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check(load().aal_set_workspace(buf.data_ptr(), buf.numel() * buf.element_size()), "aal_set_workspace")
    _workspace_keep.t = buf


def aal_version() -> int:
    return int(load().aal_version())
