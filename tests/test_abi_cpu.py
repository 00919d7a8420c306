"""CPU-side checks of the C-ABI library: it loads without a GPU, exports every
symbol include/aal.h declares, its integer table matches the oracle bit for
bit, and argument errors come back as status codes before any launch."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import associative_algebra_block_b200 as aal

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(aal.LIB_PATH):
        from associative_algebra_block_b200 import build
        build.build()
    return aal.load()


def _declared_symbols():
    names = set()
    with open(os.path.join(ROOT, "include", "aal.h")) as f:
        text = f.read()
    for m in re.finditer(r"^AAL_API\s+[\w\s\*]+?\b(aal_\w+)\s*\(", text, flags=re.M):
        names.add(m.group(1))
    return names


def test_header_declares_the_boundary_calls():
    names = _declared_symbols()
    for required in ("aal_project_fwd", "aal_swiglu_fwd", "aal_project_bwd",
                     "aal_decode_matvec", "aal_square_product", "aal_block_table",
                     "aal_block_product_count", "aal_get_device_status", "aal_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(aal.EXPORTS) <= _declared_symbols()


@pytest.mark.parametrize("law,q", [("Q", 1), ("Q", 2), ("Q", 3), ("Q", 7), ("Q", 16), ("Q", 32),
                                   ("Q2xQ2", 4)])
def test_block_table_matches_oracle_bit_exact(lib, law, q):
    got = aal.aal_block_table(law, q)
    ref = oracle.block_table_array(law, q)
    assert got.dtype == ref.dtype and np.array_equal(got, ref)


@pytest.mark.parametrize("law,q", [("Q", 1), ("Q", 2), ("Q", 5), ("Q", 16), ("Q", 32), ("Q", 256),
                                   ("Q2xQ2", 4)])
def test_block_product_counts_match_oracle(lib, law, q):
    for row_typed in (True, False):
        assert aal.aal_block_product_count(law, q, row_typed) == oracle.block_product_count(law, q, row_typed)


def test_invalid_law_and_q(lib):
    assert aal.aal_block_product_count("Q2xQ2", 3, True) == -1
    assert aal.aal_block_product_count(7, 2, True) == -1
    assert aal.aal_block_product_count("Q", 0, True) == -1
    S = np.zeros(27, np.uint8)
    assert lib.aal_block_table(1, 3, S.ctypes.data) == aal.AAL_ERR_INVALID_ARG
    assert lib.aal_block_table(0, 3, None) == aal.AAL_ERR_INVALID_ARG


def _m(ptr, rows, cols, ld=None, dtype=aal.AAL_BF16):
    return aal.AalMat(ptr, dtype, rows, cols, cols if ld is None else ld)


FAKE = 0x10000  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("case", ["shape", "q_divides", "null", "ld", "rule", "law", "dtype"])
def test_project_fwd_argument_errors(lib, case):
    rule = aal.AalRowTypeRule(0, 64, 0, None)
    X, W, Y = _m(FAKE, 64, 64), _m(FAKE, 64, 32), _m(FAKE, 64, 32)
    law, q = 0, 2
    expect = aal.AAL_ERR_INVALID_ARG
    if case == "shape":
        W = _m(FAKE, 32, 32)
    elif case == "q_divides":
        q = 3
    elif case == "null":
        X = _m(None, 64, 64)
    elif case == "ld":
        Y = _m(FAKE, 64, 32, ld=16)
    elif case == "rule":
        rule = aal.AalRowTypeRule(0, 0, 0, None)
    elif case == "law":
        law = 1
    elif case == "dtype":
        Y = _m(FAKE, 64, 32, dtype=aal.AAL_F32)
        expect = aal.AAL_ERR_UNSUPPORTED
    assert lib.aal_project_fwd(law, q, rule, X, W, Y, None) == expect


def test_other_calls_argument_errors(lib):
    rule = aal.AalRowTypeRule(0, 16, 0, None)
    bad_rule = aal.AalRowTypeRule(1, 0, 0, None)
    X, W = _m(FAKE, 16, 8), _m(FAKE, 8, 8)
    assert lib.aal_project_fwd(0, 2, bad_rule, X, W, _m(FAKE, 16, 8), None) == aal.AAL_ERR_INVALID_ARG
    # swiglu: H of the wrong width
    assert lib.aal_swiglu_fwd(0, 2, rule, X, _m(FAKE, 8, 12), _m(FAKE, 8, 12), _m(FAKE, 12, 8),
                              _m(FAKE, 16, 8), _m(FAKE, 16, 8), None) == aal.AAL_ERR_INVALID_ARG
    # bwd: dY of the wrong shape
    assert lib.aal_project_bwd(0, 2, rule, X, W, _m(FAKE, 16, 4), _m(None, 0, 0), _m(None, 0, 0),
                               0, None) == aal.AAL_ERR_INVALID_ARG
    # decode: null positions with rows
    assert lib.aal_decode_matvec(0, 2, None, _m(FAKE, 4, 8), W, _m(FAKE, 4, 8), None) == aal.AAL_ERR_INVALID_ARG
    # swiglu decode: Wd of the wrong shape, null positions, mixed dtypes
    Wg = _m(FAKE, 8, 12)
    assert lib.aal_swiglu_decode(0, 2, FAKE, _m(FAKE, 4, 8), Wg, Wg, _m(FAKE, 8, 12), _m(FAKE, 4, 12),
                                 _m(FAKE, 4, 8), None) == aal.AAL_ERR_INVALID_ARG
    assert lib.aal_swiglu_decode(0, 2, None, _m(FAKE, 4, 8), Wg, Wg, _m(FAKE, 12, 8), _m(FAKE, 4, 12),
                                 _m(FAKE, 4, 8), None) == aal.AAL_ERR_INVALID_ARG
    assert lib.aal_swiglu_decode(0, 2, FAKE, _m(FAKE, 4, 8), Wg, Wg, _m(FAKE, 12, 8), _m(FAKE, 4, 12),
                                 _m(FAKE, 4, 8, dtype=aal.AAL_F32), None) == aal.AAL_ERR_UNSUPPORTED
    # swiglu bwd: dWd of the wrong shape, mixed dtypes
    m_mf, m_md = _m(FAKE, 16, 12), _m(FAKE, 16, 8)
    good = [X, Wg, Wg, _m(FAKE, 12, 8), m_mf, m_md, m_mf, m_mf, m_mf, m_mf, m_md, Wg, Wg]
    assert lib.aal_swiglu_bwd(0, 2, rule, *good, _m(FAKE, 8, 12), None) == aal.AAL_ERR_INVALID_ARG
    assert lib.aal_swiglu_bwd(0, 2, rule, *good, _m(FAKE, 12, 8, dtype=aal.AAL_F32), None) == aal.AAL_ERR_UNSUPPORTED
    # square: not square / aliasing output
    assert lib.aal_square_product(0, 2, _m(FAKE, 8, 4), W, _m(FAKE + 4096, 8, 8), None) == aal.AAL_ERR_INVALID_ARG
    assert lib.aal_square_product(0, 2, X := _m(FAKE, 8, 8), W, _m(FAKE, 8, 8), None) == aal.AAL_ERR_INVALID_ARG
    # misaligned bf16 pointer
    assert lib.aal_square_product(0, 2, _m(FAKE + 1, 8, 8), W, _m(FAKE + 4096, 8, 8), None) == aal.AAL_ERR_INVALID_ARG


def test_empty_inputs_launch_nothing(lib):
    rule = aal.AalRowTypeRule(0, 16, 0, None)
    aal.aal_launch_count(reset=True)
    assert lib.aal_project_fwd(0, 2, rule, _m(None, 0, 8), _m(FAKE, 8, 8), _m(None, 0, 8), None) == aal.AAL_OK
    assert lib.aal_square_product(0, 2, _m(None, 0, 0), _m(None, 0, 0), _m(None, 0, 0), None) == aal.AAL_OK
    assert lib.aal_decode_matvec(0, 2, None, _m(None, 0, 8), _m(FAKE, 8, 8), _m(None, 0, 8), None) == aal.AAL_OK
    assert lib.aal_swiglu_decode(0, 2, None, _m(None, 0, 8), _m(FAKE, 8, 12), _m(FAKE, 8, 12),
                                 _m(FAKE, 12, 8), _m(None, 0, 12), _m(None, 0, 8), None) == aal.AAL_OK
    assert aal.aal_launch_count() == 0


def test_status_strings(lib):
    seen = set()
    for code in range(8):
        s = aal.aal_status_string(code)
        assert s and s not in seen
        seen.add(s)
    assert aal.aal_status_string(99) == "unknown status"


def test_path_policy_round_trip(lib):
    for p in (aal.AAL_PATH_TENSOR, aal.AAL_PATH_GENERAL, aal.AAL_PATH_AUTO):
        aal.aal_set_path_policy(p)
    with pytest.raises(aal.AalError):
        aal.aal_set_path_policy(7)
    assert aal.aal_version() >= 100


def test_plain_c_program_uses_the_boundary(lib, tmp_path):
    # the header and library work from C with no Python or torch in between
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    exe = tmp_path / "abi_host"
    pkg = os.path.dirname(aal.LIB_PATH)
    r = subprocess.run([gcc, "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_host.c"), "-o", str(exe),
                        "-L", pkg, "-l:libaal.so", "-Wl,-rpath," + pkg],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "table ok" in r.stdout and "counts ok" in r.stdout and "argument check ok" in r.stdout


def _declared_arity():
    """Parameter count of every AAL_API function in include/aal.h."""
    with open(os.path.join(ROOT, "include", "aal.h")) as f:
        text = f.read()
    out = {}
    for m in re.finditer(r"^AAL_API\s+[\w\s\*]+?\b(aal_\w+)\s*\(([^)]*)\)", text, flags=re.M | re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(lib):
    # the ctypes declarations of the binding have the header's arity
    arity = _declared_arity()
    assert arity, "no declarations parsed"
    for name, n in arity.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_new_entry_points_reject_bad_law_and_q(lib):
    rule = aal.AalRowTypeRule(0, 16, 0, None)
    x, Wg, Wd = _m(FAKE, 4, 8), _m(FAKE, 8, 12), _m(FAKE, 12, 8)
    h, y = _m(FAKE, 4, 12), _m(FAKE, 4, 8)
    for law, q in ((0, 0), (1, 3), (7, 2)):
        assert lib.aal_swiglu_decode(law, q, FAKE, x, Wg, Wg, Wd, h, y, None) == aal.AAL_ERR_INVALID_ARG
        mf, md = _m(FAKE, 16, 12), _m(FAKE, 16, 8)
        args = [md, Wg, Wg, Wd, mf, md, mf, mf, mf, mf, md, Wg, Wg, Wd]
        assert lib.aal_swiglu_bwd(law, q, rule, *args, None) == aal.AAL_ERR_INVALID_ARG


def test_binding_refuses_host_short_or_strided_index_tensors():
    # the kernels read positions / explicit types through raw pointers: the
    # binding refuses anything but a 1-D contiguous device tensor of the
    # right length and dtype before any call reaches the library
    import torch
    x = torch.empty(4, 8, dtype=torch.bfloat16)
    W = torch.empty(8, 8, dtype=torch.bfloat16)
    y = torch.empty(4, 8, dtype=torch.bfloat16)
    cases = [
        (torch.arange(4), "CUDA device"),              # a host tensor
        (torch.arange(3), "4 entries"),                # too short
        (torch.arange(4, dtype=torch.int32), "int64"), # wrong dtype
        (torch.arange(8).view(2, 4), "1-D"),           # not a vector
    ]
    for pos, msg in cases:
        for call in (lambda p: aal.aal_decode_matvec("Q", 2, p, x, W, y),
                     lambda p: aal.aal_swiglu_decode("Q", 2, p, x, W, W, W, y, y),
                     lambda p: aal.aal_swiglu_decode_noalloc("Q", 2, p, x, W, W, W, y)):
            with pytest.raises(ValueError, match=msg):
                call(pos)
    X = torch.empty(6, 8, dtype=torch.bfloat16)
    Y = torch.empty(6, 8, dtype=torch.bfloat16)
    for types, msg in ((torch.zeros(6, dtype=torch.int32), "CUDA device"),
                       (torch.zeros(5, dtype=torch.int32), "6 entries")):
        rule = aal.row_rule(types=types)
        with pytest.raises(ValueError, match=msg):
            aal.aal_project_fwd("Q", 2, rule, X, W, Y)
        with pytest.raises(ValueError, match=msg):
            aal.aal_project_bwd("Q", 2, rule, X, W, Y, X, W)


def test_every_compute_binding_runs_an_empty_call(lib):
    # all-empty tensors reach the library without a GPU (nothing is
    # launched), so each Python wrapper's argument marshalling and status
    # check run end to end here
    import torch
    z = torch.empty(0, 0, dtype=torch.bfloat16)
    pos = torch.empty(0, dtype=torch.int64)
    rule = aal.row_rule(seq_len=16)
    aal.aal_project_fwd("Q", 2, rule, z, z, z)
    aal.aal_swiglu_fwd("Q", 2, rule, z, z, z, z, z, z)
    aal.aal_project_bwd("Q", 2, rule, z, z, z, z, None)
    aal.aal_swiglu_bwd("Q", 2, rule, *([z] * 14))
    aal.aal_decode_matvec("Q", 2, pos, z, z, z)
    aal.aal_swiglu_decode("Q", 2, pos, z, z, z, z, z, z)
    aal.aal_swiglu_decode_noalloc("Q", 2, pos, z, z, z, z, z)
    aal.aal_square_product("Q", 2, z, z, z)
    assert aal.aal_workspace_size(aal.AAL_CALL_PROJECT_FWD, "Q", 2, rule, 0, 8) == 0
    assert aal.aal_workspace_size(aal.AAL_CALL_PROJECT_FWD, "Q", 2, aal.row_rule(seq_len=7), 10, 64) > 10 * 64 * 2
    aal.aal_set_workspace(None)


def test_backward_workspace_sizes():
    # the backward calls use a workspace for the split of their heavy Q_q tiles
    rule = aal.row_rule(seq_len=2048)
    n = aal.aal_workspace_size(aal.AAL_CALL_PROJECT_BWD, "Q", 16, rule, 2048, 2048, 768)
    assert n > 0 and n % (128 * 4) == 0
    assert aal.aal_workspace_size(aal.AAL_CALL_SWIGLU_BWD, "Q", 16, rule, 2048, 2048, 768) >= n
    # no heavy tiles to split: the Q2xQ2 law, q = 1
    assert aal.aal_workspace_size(aal.AAL_CALL_PROJECT_BWD, "Q2xQ2", 4, rule, 2048, 768, 1536) == 0
    assert aal.aal_workspace_size(aal.AAL_CALL_PROJECT_BWD, "Q", 1, rule, 2048, 2048, 768) == 0
    # rules that take the general path use none
    assert aal.aal_workspace_size(aal.AAL_CALL_PROJECT_BWD, "Q", 16, aal.row_rule(seq_len=7), 2048,
                                  2048, 768) == 0
    with pytest.raises(ValueError):
        aal.aal_workspace_size(5, "Q", 16, rule, 2048, 2048, 768)


def test_every_environment_switch_is_documented():
    # each AAL_* variable the library reads appears in the header's list of switches
    import glob
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    read = set()
    for f in glob.glob(os.path.join(root, "associative_algebra_block_b200", "csrc", "*.cu")):
        read |= set(re.findall(r'getenv\("(AAL_[A-Z0-9_]+)"\)', open(f).read()))
    header = open(os.path.join(root, "include", "aal.h")).read()
    documented = set(re.findall(r"(AAL_[A-Z0-9_]+)=", header))
    assert read, "no switches found"
    assert read <= documented, sorted(read - documented)
