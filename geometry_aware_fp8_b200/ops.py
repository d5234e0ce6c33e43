"""ctypes binding of libgift (include/gift.h): argument marshalling only.

Every function here checks tensor placement/dtype, allocates missing outputs
with torch (device memory is torch's job), passes raw pointers and the
current CUDA stream to the C ABI, and raises GiftError on a non-OK status.
No step of the codec is computed here; if libgift.so is missing every call
raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgift.so")

GIFT_F32, GIFT_BF16 = 0, 1
E4M3_BLOCK = 128
DEV_RHO_FLOORED, DEV_RANK_DEFICIENT, DEV_NONFINITE, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8
STATUS = {0: "GIFT_OK", 1: "GIFT_ERR_INVALID_ARG", 2: "GIFT_ERR_SHAPE", 3: "GIFT_ERR_ALIGN",
          4: "GIFT_ERR_WORKSPACE", 5: "GIFT_ERR_CUDA", 6: "GIFT_ERR_UNSUPPORTED"}

EXPORTED = ("gift_status_string", "gift_version", "gift_refresh_workspace_size", "gift_factor_refresh",
            "gift_factor_refresh_noalloc", "gift_factor_refresh_many", "gift_encode", "gift_decode", "gift_encode_many", "gift_decode_many",
            "gift_error_workspace_size", "gift_roundtrip_error", "gift_encode_nvfp4", "gift_decode_nvfp4",
            "gift_codec_split", "gift_whitened_error_workspace_size", "gift_whitened_error",
            "gift_codec_stall_test", "gift_dense_factor_workspace_size", "gift_dense_factor", "gift_dense_split",
            "gift_dense_encode", "gift_dense_decode", "gift_decode_sum", "gift_split_u",
            "gift_split_u_many")
DENSE_CHOLESKY, DENSE_INVSQRT = 1, 2


class GiftError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class RefreshJob(ctypes.Structure):
    """Mirror of gift_refresh_job."""
    _fields_ = [("X", ctypes.c_void_p), ("xdt", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("N", ctypes.c_int64), ("d_in", ctypes.c_int64), ("seed", ctypes.c_uint64),
                ("U", ctypes.c_void_p), ("lambda_", ctypes.c_void_p), ("rho", ctypes.c_void_p),
                ("A_out", ctypes.c_void_p), ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t),
                ("dev_status", ctypes.c_void_p)]


class Layer(ctypes.Structure):
    """Mirror of gift_layer."""
    _fields_ = [("G", ctypes.c_void_p), ("G_hat", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("U", ctypes.c_void_p), ("lambda_", ctypes.c_void_p),
                ("rho", ctypes.c_void_p), ("d_out", ctypes.c_int64), ("d_in", ctypes.c_int64),
                ("rank", ctypes.c_int32), ("dtype", ctypes.c_int32), ("U_split", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Open libgift.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m geometry_aware_fp8_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.gift_status_string.restype = ctypes.c_char_p
        L.gift_status_string.argtypes = [i32]
        L.gift_version.restype = i32
        L.gift_refresh_workspace_size.argtypes = [i64, i64, i32, i32, i32, ctypes.POINTER(sz)]
        L.gift_factor_refresh.argtypes = [vp, i32, i64, i64, i32, i32, i32, ctypes.c_uint64, vp, vp, vp, vp,
                                          vp, sz, vp, vp]
        L.gift_factor_refresh_noalloc.argtypes = [vp, i32, i64, i64, i32, i32, i32, ctypes.c_uint64, vp, vp, vp,
                                                  vp, vp, vp]
        L.gift_factor_refresh_many.argtypes = [ctypes.POINTER(RefreshJob), i32, i32, i32, i32, vp]
        L.gift_encode.argtypes = [vp, i32, i64, i64, vp, vp, vp, i32, vp, vp, vp, vp]
        L.gift_decode.argtypes = [vp, vp, i64, i64, vp, vp, vp, i32, vp, i32, vp, vp]
        L.gift_encode_many.argtypes = [ctypes.POINTER(Layer), i32, vp, vp]
        L.gift_split_u.argtypes = [vp, i64, i32, vp, vp]
        L.gift_split_u_many.argtypes = [ctypes.POINTER(Layer), i32, vp]
        L.gift_decode_many.argtypes = [ctypes.POINTER(Layer), i32, vp, vp]
        L.gift_codec_stall_test.argtypes = [ctypes.POINTER(Layer), i32, ctypes.c_uint32, vp, vp]
        L.gift_codec_split.argtypes = [ctypes.POINTER(Layer), i32, i32, ctypes.POINTER(i32)]
        L.gift_error_workspace_size.argtypes = [i64, i64, ctypes.POINTER(sz)]
        L.gift_roundtrip_error.argtypes = [vp, vp, i32, i64, i64, vp, vp, sz, vp]
        L.gift_whitened_error_workspace_size.argtypes = [i64, i64, ctypes.POINTER(sz)]
        L.gift_whitened_error.argtypes = [vp, vp, i32, i64, i64, vp, vp, vp, i32, vp, vp, sz, vp]
        L.gift_encode_nvfp4.argtypes = [vp, i32, i64, i64, vp, vp, vp, i32, vp, vp, vp, vp, vp]
        L.gift_decode_nvfp4.argtypes = [vp, vp, vp, i64, i64, vp, vp, vp, i32, vp, i32, vp, vp]
        L.gift_decode_sum.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i64, i64, vp, vp, vp, i32,
                                      ctypes.c_float, vp, i32, vp, vp]
        L.gift_dense_factor_workspace_size.argtypes = [i64, i32, ctypes.POINTER(sz)]
        L.gift_dense_factor.argtypes = [vp, i64, i32, vp, vp, vp, vp, vp, sz, vp, vp]
        L.gift_dense_split.argtypes = [vp, i64, i32, vp, vp]
        L.gift_dense_encode.argtypes = [vp, i64, i64, vp, i32, vp, vp, vp, vp]
        L.gift_dense_decode.argtypes = [vp, vp, i64, i64, vp, i32, vp, i32, vp, vp]
        for name in EXPORTED:
            if name not in ("gift_status_string", "gift_version"):
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def _check(st: int, where: str):
    if st != 0:
        raise GiftError(st, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GIFT_BF16
    if t.dtype == torch.float32:
        return GIFT_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensor must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensor must be contiguous")


# ---------------------------------------------------------------------------
def refresh_workspace_size(N: int, d_in: int, rank: int = 32, oversample: int = 16,
                           a_out_given: bool = False) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().gift_refresh_workspace_size(N, d_in, rank, oversample, int(a_out_given), ctypes.byref(n)),
           "gift_refresh_workspace_size")
    return n.value


def factor_refresh(X: torch.Tensor, rank: int = 32, oversample: int = 16, iters: int = 4, seed: int = 0,
                   A_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   dev_status: Optional[torch.Tensor] = None, stream=None, out=None):
    """(U, lambda, rho, dev_status) of the input factor A = X^T X / N (see gift_factor_refresh)."""
    _cuda(X, A_out, ws, dev_status)
    N, d = X.shape
    dev = X.device
    if out is None:
        U = torch.empty((d, rank), device=dev, dtype=torch.float32)
        lam = torch.empty((rank,), device=dev, dtype=torch.float32)
        rho = torch.empty((1,), device=dev, dtype=torch.float32)
    else:
        U, lam, rho = out
    need = refresh_workspace_size(N, d, rank, oversample, A_out is not None)
    if ws is None:
        ws = torch.empty((max(need, 16),), device=dev, dtype=torch.uint8)
    if dev_status is None:
        dev_status = torch.zeros((1,), device=dev, dtype=torch.int32)
    _check(lib().gift_factor_refresh(_ptr(X), _dt(X), N, d, rank, oversample, iters, seed & (2**64 - 1),
                                     _ptr(U), _ptr(lam), _ptr(rho), _ptr(A_out), _ptr(ws), ws.numel(),
                                     _ptr(dev_status), _stream(stream)), "gift_factor_refresh")
    return U, lam, rho, dev_status


def factor_refresh_noalloc(X: torch.Tensor, A_out: torch.Tensor, rank: int = 32, oversample: int = 16,
                           iters: int = 4, seed: int = 0, dev_status: Optional[torch.Tensor] = None,
                           stream=None, out=None):
    """Same result as factor_refresh, for callers that cannot supply a workspace.

    The library keeps the scratch in a fixed array on each GPU, so this call
    allocates nothing on the device besides the outputs created here when
    `out` / `dev_status` are not passed.  A_out (d_in x d_in fp32) is
    required; d_in <= 4096 and rank + oversample <= 64.  Calls must not
    overlap on the GPU.
    """
    _cuda(X, A_out, dev_status)
    N, d = X.shape
    dev = X.device
    if out is None:
        U = torch.empty((d, rank), device=dev, dtype=torch.float32)
        lam = torch.empty((rank,), device=dev, dtype=torch.float32)
        rho = torch.empty((1,), device=dev, dtype=torch.float32)
    else:
        U, lam, rho = out
    if dev_status is None:
        dev_status = torch.zeros((1,), device=dev, dtype=torch.int32)
    _check(lib().gift_factor_refresh_noalloc(_ptr(X), _dt(X), N, d, rank, oversample, iters, seed & (2**64 - 1),
                                             _ptr(U), _ptr(lam), _ptr(rho), _ptr(A_out), _ptr(dev_status),
                                             _stream(stream)), "gift_factor_refresh_noalloc")
    return U, lam, rho, dev_status


def make_refresh_jobs(items):
    """Pack [(X, U, lam, rho, ws, dev_status, seed, A_out or None), ...] into a gift_refresh_job array."""
    arr = (RefreshJob * max(len(items), 1))()
    for i, (X, U, lam, rho, ws, st, seed, A_out) in enumerate(items):
        _cuda(X, U, lam, rho, ws, st, A_out)
        arr[i] = RefreshJob(_ptr(X), _dt(X), 0, X.shape[0], X.shape[1], seed & (2**64 - 1), _ptr(U), _ptr(lam),
                            _ptr(rho), _ptr(A_out), _ptr(ws), 0 if ws is None else ws.numel(), _ptr(st))
    return arr


def factor_refresh_many(jobs, n: int, rank: int = 32, oversample: int = 16, iters: int = 4, stream=None):
    """Refresh n layers' factors in one batched sequence (see gift_factor_refresh_many)."""
    _check(lib().gift_factor_refresh_many(jobs, n, rank, oversample, iters, _stream(stream)),
           "gift_factor_refresh_many")


def encode(G: torch.Tensor, U=None, lam=None, rho=None, rank: Optional[int] = None,
           codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, stream=None,
           dev_status: Optional[torch.Tensor] = None):
    """(codes uint8 [d_out, d_in], scales fp32 [d_out, d_in/128]); rank 0 / U None = Euclidean.
    dev_status: optional int32 device word the call ORs GIFT_DEV_* bits into."""
    _cuda(G, U, lam, rho, codes, scales, dev_status)
    d_out, d_in = G.shape
    if rank is None:
        rank = 0 if U is None else U.shape[1]
    if codes is None:
        codes = torch.empty((d_out, d_in), device=G.device, dtype=torch.uint8)
    if scales is None:
        scales = torch.empty((d_out, max(d_in // E4M3_BLOCK, 1)), device=G.device, dtype=torch.float32)
    _check(lib().gift_encode(_ptr(G), _dt(G), d_out, d_in, _ptr(U), _ptr(lam), _ptr(rho), rank,
                             _ptr(codes), _ptr(scales), _ptr(dev_status), _stream(stream)), "gift_encode")
    return codes, scales


def decode(codes: torch.Tensor, scales: torch.Tensor, U=None, lam=None, rho=None, rank: Optional[int] = None,
           out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None, stream=None,
           dev_status: Optional[torch.Tensor] = None):
    """G_hat [d_out, d_in] in out_dtype (bf16 or fp32)."""
    _cuda(codes, scales, U, lam, rho, out, dev_status)
    d_out, d_in = codes.shape
    if rank is None:
        rank = 0 if U is None else U.shape[1]
    if out is None:
        out = torch.empty((d_out, d_in), device=codes.device, dtype=out_dtype)
    _check(lib().gift_decode(_ptr(codes), _ptr(scales), d_out, d_in, _ptr(U), _ptr(lam), _ptr(rho), rank,
                             _ptr(out), _dt(out), _ptr(dev_status), _stream(stream)), "gift_decode")
    return out


NVFP4_BLOCK = 16


def encode_nvfp4(G: torch.Tensor, U=None, lam=None, rho=None, rank: Optional[int] = None,
                 codes: Optional[torch.Tensor] = None, block_scales: Optional[torch.Tensor] = None,
                 tensor_scale: Optional[torch.Tensor] = None, stream=None,
                 dev_status: Optional[torch.Tensor] = None):
    """(codes uint8 [d_out, d_in/2], block scales uint8 [d_out, d_in/16], tensor scale fp32 [1])."""
    _cuda(G, U, lam, rho, codes, block_scales, tensor_scale, dev_status)
    d_out, d_in = G.shape
    if rank is None:
        rank = 0 if U is None else U.shape[1]
    if codes is None:
        codes = torch.empty((d_out, d_in // 2), device=G.device, dtype=torch.uint8)
    if block_scales is None:
        block_scales = torch.empty((d_out, max(d_in // NVFP4_BLOCK, 1)), device=G.device, dtype=torch.uint8)
    if tensor_scale is None:
        tensor_scale = torch.empty((1,), device=G.device, dtype=torch.float32)
    _check(lib().gift_encode_nvfp4(_ptr(G), _dt(G), d_out, d_in, _ptr(U), _ptr(lam), _ptr(rho), rank,
                                   _ptr(codes), _ptr(block_scales), _ptr(tensor_scale), _ptr(dev_status),
                                   _stream(stream)),
           "gift_encode_nvfp4")
    return codes, block_scales, tensor_scale


def decode_nvfp4(codes: torch.Tensor, block_scales: torch.Tensor, tensor_scale: torch.Tensor, U=None, lam=None,
                 rho=None, rank: Optional[int] = None, out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
                 stream=None, dev_status: Optional[torch.Tensor] = None):
    """G_hat [d_out, d_in] in out_dtype from NVFP4 codes."""
    _cuda(codes, block_scales, tensor_scale, U, lam, rho, out, dev_status)
    d_out, d_in = codes.shape[0], codes.shape[1] * 2
    if rank is None:
        rank = 0 if U is None else U.shape[1]
    if out is None:
        out = torch.empty((d_out, d_in), device=codes.device, dtype=out_dtype)
    _check(lib().gift_decode_nvfp4(_ptr(codes), _ptr(block_scales), _ptr(tensor_scale), d_out, d_in, _ptr(U),
                                   _ptr(lam), _ptr(rho), rank, _ptr(out), _dt(out), _ptr(dev_status),
                                   _stream(stream)),
           "gift_decode_nvfp4")
    return out


@dataclass
class LayerArgs:
    d_out: int
    d_in: int
    rank: int
    dtype: torch.dtype
    G: Optional[torch.Tensor] = None
    G_hat: Optional[torch.Tensor] = None
    codes: Optional[torch.Tensor] = None
    scales: Optional[torch.Tensor] = None
    U: Optional[torch.Tensor] = None
    lam: Optional[torch.Tensor] = None
    rho: Optional[torch.Tensor] = None
    U_split: Optional[torch.Tensor] = None  # split_u(U), or None: the kernels split U themselves


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return GIFT_BF16
    if dt == torch.float32:
        return GIFT_F32
    raise TypeError(f"unsupported gradient dtype {dt} (bf16 or fp32)")


def make_layers(layers: Sequence[LayerArgs]):
    """Pack a list of LayerArgs into a ctypes gift_layer array (kept alive by the caller)."""
    arr = (Layer * max(len(layers), 1))()
    for i, L in enumerate(layers):
        for t in (L.G, L.G_hat):
            if t is not None and t.dtype != L.dtype:
                raise TypeError(f"layer {i}: tensor dtype {t.dtype} differs from the layer's {L.dtype}")
        arr[i] = Layer(_ptr(L.G), _ptr(L.G_hat), _ptr(L.codes), _ptr(L.scales), _ptr(L.U), _ptr(L.lam),
                       _ptr(L.rho), L.d_out, L.d_in, L.rank, _dtype_code(L.dtype), _ptr(L.U_split))
    return arr


def split_u(U: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The (2, d_in, 64) int16 U split that LayerArgs.U_split takes (gift_split_u)."""
    _cuda(U, out)
    d_in, rank = U.shape
    if out is None:
        out = torch.empty((2, d_in, 64), device=U.device, dtype=torch.int16)
    _check(lib().gift_split_u(_ptr(U), d_in, rank, _ptr(out), _stream(stream)), "gift_split_u")
    return out


def split_u_many(packed, n: int, stream=None):
    """gift_split_u_many over a make_layers() array: every layer with a U_split
    and rank 32 gets the split of its current U, in one launch."""
    _check(lib().gift_split_u_many(packed, n, _stream(stream)), "gift_split_u_many")


def encode_many(packed, n: int, stream=None, dev_status: Optional[torch.Tensor] = None):
    _cuda(dev_status)
    _check(lib().gift_encode_many(packed, n, _ptr(dev_status), _stream(stream)), "gift_encode_many")


def decode_many(packed, n: int, stream=None, dev_status: Optional[torch.Tensor] = None):
    _cuda(dev_status)
    _check(lib().gift_decode_many(packed, n, _ptr(dev_status), _stream(stream)), "gift_decode_many")


def decode_sum(codes: Sequence[torch.Tensor], scales: Sequence[torch.Tensor], U=None, lam=None, rho=None,
               rank: Optional[int] = None, alpha: float = 1.0, out_dtype=torch.float32,
               out: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None, stream=None):
    """alpha * sum_r decode(codes[r], scales[r]) through one inverse transform (gift_decode_sum)."""
    n = len(codes)
    if n != len(scales) or n < 1:
        raise ValueError("codes and scales must be equally long, non-empty lists")
    _cuda(*codes, *scales, U, lam, rho, out, dev_status)
    d_out, d_in = codes[0].shape
    if rank is None:
        rank = 0 if U is None else U.shape[1]
    if out is None:
        out = torch.empty((d_out, d_in), device=codes[0].device, dtype=out_dtype)
    cp = (ctypes.c_void_p * n)(*[c.data_ptr() for c in codes])
    sp = (ctypes.c_void_p * n)(*[x.data_ptr() for x in scales])
    _check(lib().gift_decode_sum(cp, sp, n, d_out, d_in, _ptr(U), _ptr(lam), _ptr(rho), rank, float(alpha), _ptr(out),
                                 _dt(out), _ptr(dev_status), _stream(stream)), "gift_decode_sum")
    return out


def codec_stall_test(layer: LayerArgs, encode: bool, stall_polls: int, dev_status: torch.Tensor, stream=None):
    """Test hook (gift_codec_stall_test): the tensor-core codec kernel on this
    layer gives up a bounded wait on a barrier nothing arrives at before any
    work, skips the layer and ORs GIFT_DEV_TIMEOUT into dev_status."""
    _cuda(dev_status)
    arr = make_layers([layer])
    _check(lib().gift_codec_stall_test(arr, 1 if encode else 0, stall_polls, _ptr(dev_status), _stream(stream)),
           "gift_codec_stall_test")


def codec_split(packed, n: int, encode: bool = True) -> int:
    """CTAs per 128-row panel (1, 2 or 4; 0 if no layer takes the tensor-core
    path) that the whitened codec plans for its first launch over these layers."""
    out = ctypes.c_int32(-1)
    _check(lib().gift_codec_split(packed, n, 1 if encode else 0, ctypes.byref(out)), "gift_codec_split")
    return out.value


def error_workspace_size(d_out: int, d_in: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().gift_error_workspace_size(d_out, d_in, ctypes.byref(n)), "gift_error_workspace_size")
    return n.value


def roundtrip_error(G: torch.Tensor, G_hat: torch.Tensor, out: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Device tensor [rel_err, ||G_hat-G||^2, ||G||^2] (fp64)."""
    _cuda(G, G_hat, out, ws)
    if G.dtype != G_hat.dtype or G.shape != G_hat.shape:
        raise ValueError("G and G_hat must match in shape and dtype")
    d_out, d_in = G.shape
    if out is None:
        out = torch.empty((3,), device=G.device, dtype=torch.float64)
    if ws is None:
        ws = torch.empty((error_workspace_size(d_out, d_in),), device=G.device, dtype=torch.uint8)
    _check(lib().gift_roundtrip_error(_ptr(G), _ptr(G_hat), _dt(G), d_out, d_in, _ptr(out), _ptr(ws),
                                      ws.numel(), _stream(stream)), "gift_roundtrip_error")
    return out


def whitened_error_workspace_size(d_out: int, d_in: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().gift_whitened_error_workspace_size(d_out, d_in, ctypes.byref(n)),
           "gift_whitened_error_workspace_size")
    return n.value


def whitened_error(G: torch.Tensor, G_hat: torch.Tensor, U=None, lam=None, rho=None,
                   out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Device tensor [||(G_hat-G) M|| / ||G M||, ||(G_hat-G) M||^2, ||G M||^2] (fp64), M from (U, lam, rho)."""
    _cuda(G, G_hat, U, lam, rho, out, ws)
    if G.dtype != G_hat.dtype or G.shape != G_hat.shape:
        raise ValueError("G and G_hat must match in shape and dtype")
    d_out, d_in = G.shape
    rank = 0 if U is None else U.shape[1]
    if out is None:
        out = torch.empty((3,), device=G.device, dtype=torch.float64)
    if ws is None:
        ws = torch.empty((whitened_error_workspace_size(d_out, d_in),), device=G.device, dtype=torch.uint8)
    _check(lib().gift_whitened_error(_ptr(G), _ptr(G_hat), _dt(G), d_out, d_in, _ptr(U), _ptr(lam), _ptr(rho), rank,
                                     _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "gift_whitened_error")
    return out


# ---------------------------------------------------------------------------
# Dense input-side transforms (full-rank A^{-1/2} and Cholesky L^{-T} variants)
# ---------------------------------------------------------------------------
def dense_factor_workspace_size(d: int, kind: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().gift_dense_factor_workspace_size(d, kind, ctypes.byref(n)), "gift_dense_factor_workspace_size")
    return n.value


def dense_factor(A: torch.Tensor, kind: int, ws: Optional[torch.Tensor] = None,
                 dev_status: Optional[torch.Tensor] = None, stream=None):
    """(M, M_inv, M_split (3 bf16 parts), M_inv_split (2 parts), dev_status) of
    gift_dense_factor for A (d x d fp32); the parts are stored as int16."""
    _cuda(A, ws, dev_status)
    d = A.shape[0]
    dev = A.device
    M = torch.empty((d, d), device=dev, dtype=torch.float32)
    Mi = torch.empty_like(M)
    Ms = torch.empty((3, d, d), device=dev, dtype=torch.int16)
    Mis = torch.empty((2, d, d), device=dev, dtype=torch.int16)
    if ws is None:
        ws = torch.empty((dense_factor_workspace_size(d, kind),), device=dev, dtype=torch.uint8)
    if dev_status is None:
        dev_status = torch.zeros((1,), device=dev, dtype=torch.int32)
    _check(lib().gift_dense_factor(_ptr(A), d, kind, _ptr(M), _ptr(Mi), _ptr(Ms), _ptr(Mis), _ptr(ws), ws.numel(),
                                   _ptr(dev_status), _stream(stream)), "gift_dense_factor")
    return M, Mi, Ms, Mis, dev_status


def dense_split(M: torch.Tensor, parts: int = 3, stream=None) -> torch.Tensor:
    """bf16 parts (parts x d x d, stored as int16) of an fp32 d x d transform:
    3 for the encoder's M, 2 for the decoder's M^{-1}."""
    _cuda(M)
    d = M.shape[0]
    out = torch.empty((parts, d, d), device=M.device, dtype=torch.int16)
    _check(lib().gift_dense_split(_ptr(M), d, parts, _ptr(out), _stream(stream)), "gift_dense_split")
    return out


def dense_encode(G: torch.Tensor, M_split: torch.Tensor, upper: bool = False, codes=None, scales=None,
                 dev_status: Optional[torch.Tensor] = None, stream=None):
    """(codes, scales) of W = G M (G bf16, M given as its three bf16 parts)."""
    _cuda(G, M_split, codes, scales, dev_status)
    if G.dtype != torch.bfloat16:
        raise TypeError("gift_dense_encode takes bf16 gradients")
    d_out, d_in = G.shape
    if codes is None:
        codes = torch.empty((d_out, d_in), device=G.device, dtype=torch.uint8)
    if scales is None:
        scales = torch.empty((d_out, max(d_in // E4M3_BLOCK, 1)), device=G.device, dtype=torch.float32)
    _check(lib().gift_dense_encode(_ptr(G), d_out, d_in, _ptr(M_split), int(upper), _ptr(codes), _ptr(scales),
                                   _ptr(dev_status), _stream(stream)), "gift_dense_encode")
    return codes, scales


def dense_decode(codes: torch.Tensor, scales: torch.Tensor, M_inv_split: torch.Tensor, upper: bool = False,
                 out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
                 dev_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """G_hat = W_hat M_inv (M_inv given as its bf16 pair)."""
    _cuda(codes, scales, M_inv_split, out, dev_status)
    d_out, d_in = codes.shape
    if out is None:
        out = torch.empty((d_out, d_in), device=codes.device, dtype=out_dtype)
    _check(lib().gift_dense_decode(_ptr(codes), _ptr(scales), d_out, d_in, _ptr(M_inv_split), int(upper), _ptr(out),
                                   _dt(out), _ptr(dev_status), _stream(stream)), "gift_dense_decode")
    return out
