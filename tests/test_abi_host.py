"""CPU-only checks of the C ABI: the library loads without a GPU, exports
every function include/gift.h declares, and rejects bad arguments on the
host before any CUDA call (the status codes gift.h documents).

Only argument combinations that fail host validation are passed here; the
fake addresses below are never dereferenced because validation returns
first.
"""
import ctypes
import os
import re

import pytest

from geometry_aware_fp8_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, SHAPE, ALIGN, WORKSPACE = 0, 1, 2, 3, 4
A16 = 0x10000          # aligned fake address (never dereferenced)
A_ODD = 0x10004        # 4-byte but not 16-byte aligned


def declared_functions():
    src = open(os.path.join(ROOT, "include", "gift.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gift_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    try:
        return ops.lib()
    except RuntimeError as e:
        pytest.fail(str(e))


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ops.EXPORTED)


def test_version_and_status_strings(L):
    # the library reports the version of the header it was built from
    m = re.search(r"#define GIFT_VERSION (\d+)", open(os.path.join(ROOT, "include", "gift.h")).read())
    assert m and L.gift_version() == int(m.group(1))
    for s in range(7):
        assert L.gift_status_string(s).startswith(b"GIFT_")


def test_encode_rejects_bad_arguments(L):
    s = None
    # null pointers (an empty gradient, d_out == 0, may pass nulls)
    assert L.gift_encode(None, 1, 4, 128, None, None, None, 0, A16, A16, None, s) == INVALID
    assert L.gift_encode(None, 1, 0, 128, None, None, None, 0, None, None, None, s) == OK
    # bad dtype
    assert L.gift_encode(A16, 7, 4, 128, None, None, None, 0, A16, A16, None, s) == INVALID
    # d_in not a multiple of 128
    assert L.gift_encode(A16, 1, 4, 100, None, None, None, 0, A16, A16, None, s) == SHAPE
    # rank above 32
    assert L.gift_encode(A16, 1, 4, 128, A16, A16, A16, 33, A16, A16, None, s) == SHAPE
    # whitened without factors
    assert L.gift_encode(A16, 1, 4, 128, None, None, None, 32, A16, A16, None, s) == INVALID
    # misaligned gradient / codes
    assert L.gift_encode(A_ODD, 1, 4, 128, None, None, None, 0, A16, A16, None, s) == ALIGN
    assert L.gift_encode(A16, 1, 4, 128, None, None, None, 0, A_ODD, A16, None, s) == ALIGN
    # negative sizes
    assert L.gift_encode(A16, 1, -1, 128, None, None, None, 0, A16, A16, None, s) == INVALID


def test_codec_status_word_alignment_and_stall_hook_arguments(L):
    s = None
    assert L.gift_encode(A16, 1, 4, 128, None, None, None, 0, A16, A16, A16 + 2, s) == ALIGN
    assert L.gift_decode(A16, A16, 4, 128, None, None, None, 0, A16, 1, A16 + 1, s) == ALIGN
    import torch
    arr = ops.make_layers([ops.LayerArgs(d_out=256, d_in=256, rank=32, dtype=torch.bfloat16)])
    assert L.gift_encode_many(arr, 1, A16 + 2, None) == ALIGN
    assert L.gift_codec_stall_test(None, 1, 100, A16, s) == INVALID
    assert L.gift_codec_stall_test(arr, 1, 0, A16, s) == INVALID      # stall_polls must be positive
    assert L.gift_codec_stall_test(arr, 1, 100, None, s) == INVALID   # the status word is required
    assert L.gift_codec_stall_test(arr, 1, 100, A16, s) == INVALID    # layer without tensors


def test_decode_rejects_bad_arguments(L):
    s = None
    assert L.gift_decode(None, A16, 4, 128, None, None, None, 0, A16, 1, None, s) == INVALID
    assert L.gift_decode(A16, A16, 4, 256 + 64, None, None, None, 0, A16, 1, None, s) == SHAPE
    assert L.gift_decode(A16, A16, 4, 128, None, None, None, 0, A16, 3, None, s) == INVALID
    assert L.gift_decode(A16, A16, 4, 128, None, None, None, 0, A_ODD, 1, None, s) == ALIGN


def test_nvfp4_rejects_bad_arguments(L):
    s = None
    UNSUPPORTED = 6
    enc, dec = L.gift_encode_nvfp4, L.gift_decode_nvfp4
    # empty gradient: nothing is touched
    assert enc(None, 1, 0, 128, None, None, None, 0, None, None, None, None, s) == OK
    # null outputs
    assert enc(A16, 1, 4, 128, None, None, None, 0, A16, A16, None, None, s) == INVALID
    # Euclidean blocks of 16: d_in % 16; whitened: d_in % 128
    assert enc(A16, 1, 4, 24, None, None, None, 0, A16, A16, A16, None, s) == SHAPE
    assert enc(A16, 1, 4, 144, A16, A16, A16, 32, A16, A16, A16, None, s) == SHAPE
    # whitened NVFP4 runs on the tensor cores only: rank 32, bf16
    assert enc(A16, 1, 4, 128, A16, A16, A16, 7, A16, A16, A16, None, s) == UNSUPPORTED
    assert enc(A16, 0, 4, 128, A16, A16, A16, 32, A16, A16, A16, None, s) == UNSUPPORTED
    assert enc(A16, 1, 4, 128, A16, A16, A16, 33, A16, A16, A16, None, s) == SHAPE
    # alignment: codes 16 B, block scales 8 B, tensor scale 4 B
    assert enc(A16, 1, 4, 128, None, None, None, 0, A_ODD, A16, A16, None, s) == ALIGN
    assert enc(A16, 1, 4, 128, None, None, None, 0, A16, A16 + 4, A16, None, s) == ALIGN
    assert enc(A16, 1, 4, 128, None, None, None, 0, A16, A16, A16 + 2, None, s) == ALIGN
    assert dec(A16, A16, A16, 4, 128, None, None, None, 0, None, 1, None, s) == INVALID
    assert dec(A16, A16, A16, 4, 128, None, None, None, 0, A16, 5, None, s) == INVALID
    assert dec(A16, A16, A16, 4, 128, A16, A16, A16, 32, A16, 0, None, s) == UNSUPPORTED


def test_refresh_rejects_bad_arguments(L):
    s = None
    n = ctypes.c_size_t(0)
    assert L.gift_refresh_workspace_size(1024, 512, 32, 16, 0, ctypes.byref(n)) == OK
    need = n.value
    assert need >= 512 * 512 * 4  # A lives in the workspace when A_out is not given
    assert L.gift_refresh_workspace_size(1024, 512, 32, 16, 1, ctypes.byref(n)) == OK
    assert n.value < need
    assert L.gift_refresh_workspace_size(1024, 500, 32, 16, 0, ctypes.byref(n)) == SHAPE
    assert L.gift_refresh_workspace_size(1024, 512, 48, 17, 0, ctypes.byref(n)) == SHAPE
    assert L.gift_refresh_workspace_size(0, 512, 32, 16, 0, ctypes.byref(n)) == INVALID
    args = dict(X=A16, xdt=1, N=1024, d=512, r=32, p=16, it=4, seed=0, U=A16, lam=A16, rho=A16, A=None)

    def call(ws, ws_bytes, **kw):
        a = dict(args, **kw)
        return L.gift_factor_refresh(a["X"], a["xdt"], a["N"], a["d"], a["r"], a["p"], a["it"], a["seed"], a["U"],
                                     a["lam"], a["rho"], a["A"], ws, ws_bytes, None, s)

    assert call(None, 0) == WORKSPACE
    assert call(A16, need - 1) == WORKSPACE
    assert call(A16, need, X=None) == INVALID
    assert call(A16, need, xdt=5) == INVALID
    assert call(A16, need, X=A_ODD) == ALIGN
    assert call(A16, need, it=-1) == INVALID
    assert call(A16, need, r=0) == INVALID


def test_error_rejects_bad_arguments(L):
    n = ctypes.c_size_t(0)
    assert L.gift_error_workspace_size(16, 256, ctypes.byref(n)) == OK and n.value >= 16
    assert L.gift_roundtrip_error(A16, A16, 1, 16, 256, A16, None, 0, None) == WORKSPACE
    assert L.gift_roundtrip_error(A16, None, 1, 16, 256, A16, A16, n.value, None) == INVALID
    assert L.gift_roundtrip_error(A16, A_ODD, 1, 16, 256, A16, A16, n.value, None) == ALIGN


def test_many_rejects_a_bad_layer_before_launching(L):
    good = ops.Layer(A16, A16, A16, A16, None, None, None, 8, 256, 0, 1)
    bad = ops.Layer(A16, A16, A16, A16, None, None, None, 8, 200, 0, 1)
    arr = (ops.Layer * 2)(good, bad)
    assert L.gift_encode_many(arr, 2, None, None) == SHAPE
    assert L.gift_encode_many(None, 3, None, None) == INVALID
    assert L.gift_encode_many(arr, 0, None, None) == OK


def test_product_path_has_no_oracle_import():
    pkg = os.path.join(ROOT, "geometry_aware_fp8_b200")
    pat = re.compile(r"^\s*(from|import)\s+oracle\b|gift_oracle|#include\s+\"[^\"]*oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not pat.search(txt), f


def test_codec_split_rejects_bad_arguments(L):
    import torch
    out = ctypes.c_int(-1)
    eu = ops.make_layers([ops.LayerArgs(d_out=256, d_in=256, rank=0, dtype=torch.bfloat16)])
    assert L.gift_codec_split(eu, 1, 1, None) == INVALID
    assert L.gift_codec_split(None, 1, 1, ctypes.byref(out)) == INVALID
    assert L.gift_codec_split(eu, -1, 1, ctypes.byref(out)) == INVALID
    bad = ops.make_layers([ops.LayerArgs(d_out=256, d_in=200, rank=32, dtype=torch.bfloat16)])
    assert L.gift_codec_split(bad, 1, 1, ctypes.byref(out)) == SHAPE
    # no layer on the tensor-core path (Euclidean): nothing to plan, no device needed
    assert L.gift_codec_split(eu, 1, 0, ctypes.byref(out)) == OK and out.value == 0
    assert L.gift_codec_split(eu, 0, 1, ctypes.byref(out)) == OK and out.value == 0


def test_split_u_and_layer_split_arguments(L):
    s = None
    assert L.gift_split_u(None, 128, 32, A16, s) == INVALID
    assert L.gift_split_u(A16, 128, 32, None, s) == INVALID
    assert L.gift_split_u(A16, 128, 16, A16, s) == INVALID    # the split serves the rank-32 codec only
    assert L.gift_split_u(A16, 0, 32, A16, s) == INVALID
    assert L.gift_split_u(A_ODD, 128, 32, A16, s) == ALIGN
    assert L.gift_split_u(A16, 128, 32, A_ODD, s) == ALIGN
    # a grouped layer whose U split is misaligned is rejected before any launch
    arr = (ops.Layer * 1)()
    arr[0] = ops.Layer(A16, A16, A16, A16, A16, A16, A16, 256, 256, 32, 1, A_ODD)
    assert L.gift_encode_many(arr, 1, None, None) == ALIGN
    assert L.gift_decode_many(arr, 1, None, None) == ALIGN
