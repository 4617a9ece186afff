"""The C ABI without a GPU: the library loads, exports every function that
include/moe_rt.h declares, and its host-only entry points (sizes, status text,
argument validation) behave as documented. No call here reaches the device."""

import ctypes
import subprocess

import pytest

import combine_moe_route_tokens_b200 as moe
from combine_moe_route_tokens_b200 import _native
from combine_moe_route_tokens_b200.build import LIB_PATH, build


@pytest.fixture(scope="module")
def lib():
    build()
    return _native.lib()


def test_exports_every_declared_symbol(lib):
    declared = _native.declared_functions()
    assert "moe_dispatch_layout" in declared and "moe_combine" in declared
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [name for name in declared if name not in exported]
    assert not missing, missing
    for name in declared:
        assert hasattr(lib, name)
    # nothing but the C ABI leaks out of the library
    assert {n for n in exported if n.startswith("moe_")} == set(declared)


def test_abi_version_and_status_strings(lib):
    assert lib.moe_abi_version() == _native.ABI_VERSION
    for code in (0, -1, -2, -3, 1, 2, 4, 12345):
        assert isinstance(_native.status_string(code), str) and _native.status_string(code)
    assert "invalid" in _native.status_string(-1)


@pytest.mark.parametrize(
    "kw,rows",
    [
        (dict(N=4096, H=7168, k=8, E_log=256, R=4), 32768),
        (dict(N=16384, H=2048, k=2, E_log=64, R=2, capacity=640), 40960),
        (dict(N=8192, H=7168, k=8, E_log=256, R=8, num_replicas=8), 65536),
        (dict(N=0, H=8, k=1, E_log=1, R=1), 0),
        (dict(N=0, H=8, k=2, E_log=4, R=2, capacity=3), 12),
        (dict(N=4096, H=7168, k=8, E_log=256, R=4, row_align=16), 32768 + 256 * 15),
        (dict(N=10, H=8, k=2, E_log=4, R=2, capacity=32, row_align=16), 128),
        (dict(N=100, H=8, k=3, E_log=8, R=2, tp_size=3, tp_rank=1), (300 + 8 * 2) // 3),
        (dict(N=100, H=8, k=3, E_log=8, R=2, capacity=10, tp_size=3), 8 * 4),
    ],
)
def test_rows_max(lib, kw, rows):
    assert moe.Problem(**kw).rows_max == rows


@pytest.mark.parametrize(
    "kw",
    [
        dict(N=-1, H=8, k=1, E_log=4, R=1),
        dict(N=4, H=12, k=1, E_log=4, R=1),  # H not a multiple of 8
        dict(N=4, H=0, k=1, E_log=4, R=1),
        dict(N=4, H=8, k=0, E_log=4, R=1),
        dict(N=4, H=8, k=1, E_log=6, R=4),  # E_log % R
        dict(N=4, H=8, k=1, E_log=8, R=4, num_replicas=2),  # replicas % R
        dict(N=4, H=8, k=1, E_log=4, R=2, num_replicas=6),  # more replicas than experts
        dict(N=4, H=8, k=1, E_log=4, R=1, capacity=-1),
        dict(N=2**31, H=8, k=2, E_log=4, R=1),  # N*k overflows int32
        dict(N=4, H=8, k=1, E_log=4, R=1, flags=0x2),  # unknown flag
        dict(N=4, H=8, k=1, E_log=4, R=1, row_align=-2),
        dict(N=4, H=8, k=1, E_log=4, R=1, capacity=10, row_align=4),  # capacity not a multiple of the alignment
        dict(N=4, H=8, k=1, E_log=4, R=1, tp_size=2, tp_rank=2),  # rank outside the peers
        dict(N=4, H=8, k=1, E_log=4, R=1, tp_size=9),  # more peers than MOE_MAX_TP
        dict(N=4, H=8, k=1, E_log=4, R=1, capacity=10, row_align=8, tp_size=3),  # ceil(10/3) % 8 != 0
    ],
)
def test_invalid_problems_rejected(lib, kw):
    p = moe.Problem(**kw).c_struct()
    assert lib.moe_rows_max(ctypes.byref(p)) == _native.MOE_ERR_INVALID
    n = ctypes.c_size_t(0)
    assert lib.moe_layout_workspace_bytes(ctypes.byref(p), ctypes.byref(n)) == _native.MOE_ERR_INVALID
    L = _native.MoeLayout()
    assert lib.moe_dispatch_layout(ctypes.byref(p), None, None, ctypes.byref(L), None, 0, None) == \
        _native.MOE_ERR_INVALID
    assert lib.moe_permute(ctypes.byref(p), ctypes.byref(L), None, None, None) == _native.MOE_ERR_INVALID
    assert lib.moe_combine(ctypes.byref(p), ctypes.byref(L), None, None, None, None) == _native.MOE_ERR_INVALID


@pytest.mark.parametrize(
    "kw",
    [
        dict(N=4, H=8, k=33, E_log=64, R=1),  # k above the kernels' 32
        dict(N=4, H=8, k=2, E_log=4096, R=1),  # E_log above 2048
        dict(N=4, H=8, k=2, E_log=256, R=128, num_replicas=128),  # placement over 64 ranks
    ],
)
def test_unsupported_problems(lib, kw):
    p = moe.Problem(**kw).c_struct()
    L = _native.MoeLayout()
    assert lib.moe_dispatch_layout(ctypes.byref(p), None, None, ctypes.byref(L), None, 0, None) == \
        _native.MOE_ERR_UNSUPPORTED


def test_workspace_size(lib):
    p = moe.Problem(N=4096, H=7168, k=8, E_log=256, R=4)
    assert p.workspace_bytes == 256 + 128 * 256 * 8  # ticket word, then 64-bit look-back words per block and expert


def test_layout_requires_outputs_and_workspace(lib):
    p = moe.Problem(N=4, H=8, k=2, E_log=4, R=2).c_struct()
    L = _native.MoeLayout()
    # every required output NULL -> invalid before any device work
    assert lib.moe_dispatch_layout(ctypes.byref(p), ctypes.c_void_p(16), None, ctypes.byref(L),
                                   ctypes.c_void_p(256), 1 << 20, None) == _native.MOE_ERR_INVALID


def test_layout_rejects_undersized_or_misaligned_workspace(lib):
    # every output pointer set (fake addresses: the checks run on the host, before any
    # device work), so only the workspace decides
    p = moe.Problem(N=4, H=8, k=2, E_log=4, R=2)
    L = _native.MoeLayout(**{name: 4096 * (i + 1) for i, name in enumerate(_native.LAYOUT_FIELDS)})
    need = p.workspace_bytes
    f = lib.moe_dispatch_layout
    args = (ctypes.byref(p.c_struct()), ctypes.c_void_p(1 << 20), None, ctypes.byref(L))
    assert f(*args, ctypes.c_void_p(1 << 24), need - 1, None) == _native.MOE_ERR_INVALID  # one byte short
    assert f(*args, ctypes.c_void_p((1 << 24) + 128), need, None) == _native.MOE_ERR_INVALID  # not 256-byte aligned
    assert f(*args, None, need, None) == _native.MOE_ERR_INVALID


def test_route_argument_checks(lib):
    f = lib.moe_route_topk
    assert f(None, None, 4, 8, 0, None, None, None) == _native.MOE_ERR_INVALID  # k = 0
    assert f(None, None, 4, 8, 9, None, None, None) == _native.MOE_ERR_INVALID  # k > E
    assert f(None, None, -1, 8, 2, None, None, None) == _native.MOE_ERR_INVALID
    assert f(None, None, 4, 2048, 8, None, None, None) == _native.MOE_ERR_UNSUPPORTED
    assert f(None, None, 4, 64, 40, None, None, None) == _native.MOE_ERR_UNSUPPORTED
    assert f(None, None, 4, 64, 8, None, None, None) == _native.MOE_ERR_INVALID  # NULL buffers
    assert f(None, None, 0, 64, 8, None, None, None) == _native.MOE_OK  # nothing to do


def test_misaligned_buffers_rejected(lib):
    p = moe.Problem(N=4, H=8, k=2, E_log=4, R=2).c_struct()
    L = _native.MoeLayout(dest_row=64, pad_mask=128, status=192)
    assert lib.moe_permute(ctypes.byref(p), ctypes.byref(L), ctypes.c_void_p(4096 + 8), ctypes.c_void_p(8192),
                           None) == _native.MOE_ERR_INVALID
    assert lib.moe_combine(ctypes.byref(p), ctypes.byref(L), ctypes.c_void_p(4096), None,
                           ctypes.c_void_p(8192 + 4), None) == _native.MOE_ERR_INVALID


def test_product_package_does_not_import_oracle():
    import sys

    before = set(sys.modules)
    import importlib

    importlib.reload(moe)
    src = open(moe.__file__).read() + open(_native.__file__).read()
    assert "oracle" not in src
    assert not any(m == "oracle" or m.startswith("oracle.") for m in set(sys.modules) - before)
