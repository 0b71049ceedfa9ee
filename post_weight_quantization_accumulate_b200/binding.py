"""ctypes binding of libgptq.so: argument marshalling only.

Every function here has the name of the C entry point it calls and takes
torch tensors (device memory unless stated) instead of raw pointers; the
current torch stream of the tensors' device is passed as the CUDA stream.
Nothing is computed in Python: there is no CPU fallback, and loading fails
loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgptq.so")

GPTQ_OK = 0
STATUS_NAMES = {0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID_ARG", 2: "GPTQ_ERR_NOT_PD",
                3: "GPTQ_ERR_NONFINITE", 4: "GPTQ_ERR_CUDA", 5: "GPTQ_ERR_TIMEOUT",
                6: "GPTQ_ERR_WORKSPACE", 7: "GPTQ_ERR_UNSUPPORTED", 8: "GPTQ_ERR_NO_MEMORY"}

# (name, restype, argtypes) of every exported symbol, in header order
_P, _I64, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = [
    ("gptq_status_string", ctypes.c_char_p, [_I]),
    ("gptq_last_cuda_error", ctypes.c_char_p, []),
    ("gptq_version", _I, []),
    ("gptq_launch_count", ctypes.c_uint64, []),
    ("gptq_device_status", _I, []),
    ("gptq_workspace_bytes", _SZ, [_I64, _I64, _I]),
    ("gptq_workspace_min_bytes", _SZ, [_I64, _I64, _I]),
    ("gptq_hessian_accumulate", _I, [_P, _P, _I64, _I64, _P]),
    ("gptq_hessian_accumulate_host", _I, [_P, _P, _I64, _I64, _P, _I64, _P]),
    ("gptq_hessian_f32_workspace_bytes", _SZ, [_I64, _I64]),
    ("gptq_hessian_accumulate_f32", _I, [_P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    ("gptq_prepare", _I, [_P, _I64, _F, _I, _P, _P, _P, _SZ, _P]),
    ("gptq_prepare_async", _I, [_P, _I64, _F, _I, _P, _P, _P, _SZ, _P, _P]),
    ("gptq_quantize", _I, [_P, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    ("gptq_quantize_q4k", _I, [_P, _P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                               _SZ, _P]),
    ("gptq_quantize_static_scratch", _I, [_P, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    ("gptq_quantize_timed", _I, [_P, _P, _P, _I64, _I64, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                 _P, _P, _P, _P]),
    ("gptq_selftest_bounded_wait", _I, [_I64]),
    ("gptq_selftest_quotient", _I, [_I64, ctypes.c_uint64, _P]),
    ("gptq_w4a16_gemm", _I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _P]),
    ("gptq_bf16_to_f32", _I, [_P, _P, _I64, _P]),
]

W4A16_AUTO, W4A16_TENSOR_CORE, W4A16_GENERAL, W4A16_DECODE = 0, 1, 2, 3

_lib = None
_lock = threading.Lock()


class GptqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} -> {STATUS_NAMES.get(status, status)}"
        if status == 4:
            msg += f" ({lib().gptq_last_cuda_error().decode()})"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "python -m post_weight_quantization_accumulate_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            for name, res, args in SIGNATURES:
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return ctypes.c_void_p(t.data_ptr())
    return ctypes.c_void_p(int(t))


def _stream(t: torch.Tensor | None, stream=None):
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    dev = t.device if t is not None and t.is_cuda else torch.device("cuda", torch.cuda.current_device())
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(fn: str, st: int):
    if st != GPTQ_OK:
        raise GptqError(fn, st)


def _need(t: torch.Tensor, dtype, name):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError(f"{name} must be a {dtype} tensor")


def gptq_status_string(status: int) -> str:
    return lib().gptq_status_string(status).decode()


def gptq_version() -> int:
    return lib().gptq_version()


def gptq_launch_count() -> int:
    return int(lib().gptq_launch_count())


def gptq_device_status() -> int:
    return lib().gptq_device_status()


def gptq_workspace_bytes(d_out: int, d_in: int, block_size: int = 128) -> int:
    return int(lib().gptq_workspace_bytes(d_out, d_in, block_size))


def gptq_workspace_min_bytes(d_out: int, d_in: int, block_size: int = 128) -> int:
    return int(lib().gptq_workspace_min_bytes(d_out, d_in, block_size))


def workspace(d_out: int, d_in: int, block_size: int = 128, device=None) -> torch.Tensor:
    """A uint8 device buffer large enough for gptq_prepare and gptq_quantize
    (torch's allocator returns 256-byte-aligned blocks)."""
    n = gptq_workspace_bytes(d_out, d_in, block_size)
    if n == 0:
        raise ValueError("invalid sizes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def gptq_hessian_accumulate(H: torch.Tensor, X: torch.Tensor, stream=None):
    """H (+)= 2 X^T X.  H float32 [d, d] on the device; X bf16 [n, d]."""
    _need(H, torch.float32, "H")
    _need(X, torch.bfloat16, "X")
    n, d = X.shape
    _check("gptq_hessian_accumulate",
           lib().gptq_hessian_accumulate(_ptr(H), _ptr(X), n, d, _stream(H, stream)))
    return H


def gptq_hessian_accumulate_host(H: torch.Tensor, X_host: torch.Tensor, staging: torch.Tensor,
                                 chunk_tokens: int, stream=None):
    """H (+)= 2 X^T X with X bf16 [n, d] in (pinned) host memory, streamed
    through `staging` (device bf16, >= 2 * chunk_tokens * d elements)."""
    _need(H, torch.float32, "H")
    _need(X_host, torch.bfloat16, "X_host")
    _need(staging, torch.bfloat16, "staging")
    n, d = X_host.shape
    if X_host.is_cuda or staging.numel() < 2 * chunk_tokens * d:
        raise ValueError("X_host must be host memory; staging too small")
    _check("gptq_hessian_accumulate_host",
           lib().gptq_hessian_accumulate_host(_ptr(H), _ptr(X_host), n, d, _ptr(staging),
                                              chunk_tokens, _stream(H, stream)))
    return H


def gptq_hessian_f32_workspace_bytes(d_in: int, chunk_tokens: int) -> int:
    return int(lib().gptq_hessian_f32_workspace_bytes(d_in, chunk_tokens))


def gptq_hessian_accumulate_f32(H: torch.Tensor, X: torch.Tensor, ws: torch.Tensor,
                                chunk_tokens: int = 8192, stream=None):
    """H float32 [d, d] += 2 X^T X for float32 X [n, d] on the device."""
    _need(H, torch.float32, "H")
    _need(X, torch.float32, "X")
    n, d = X.shape
    _check("gptq_hessian_accumulate_f32",
           lib().gptq_hessian_accumulate_f32(_ptr(H), _ptr(X), n, d, chunk_tokens, _ptr(ws),
                                             ws.numel() * ws.element_size(), _stream(H, stream)))


def gptq_prepare(H: torch.Tensor, damp: float, act_order: bool, perm: torch.Tensor,
                 Hinv_chol: torch.Tensor, ws: torch.Tensor, stream=None):
    """perm (int32 [d]) and Hinv_chol (float32 [d, d], upper) are outputs."""
    _need(H, torch.float32, "H")
    _need(perm, torch.int32, "perm")
    _need(Hinv_chol, torch.float32, "Hinv_chol")
    d = H.shape[0]
    _check("gptq_prepare",
           lib().gptq_prepare(_ptr(H), d, float(damp), int(bool(act_order)), _ptr(perm),
                              _ptr(Hinv_chol), _ptr(ws), ws.numel(), _stream(H, stream)))


def gptq_prepare_async(H: torch.Tensor, damp: float, act_order: bool, perm: torch.Tensor,
                       Hinv_chol: torch.Tensor, ws: torch.Tensor, status: torch.Tensor, stream=None):
    """gptq_prepare without waiting: the factorisation status lands in
    status (int32, one element, on the device or in pinned host memory) when
    the stream reaches it; read it after synchronising."""
    _need(H, torch.float32, "H")
    _need(perm, torch.int32, "perm")
    _need(Hinv_chol, torch.float32, "Hinv_chol")
    _need(status, torch.int32, "status")
    if status.numel() < 1 or not (status.is_cuda or status.is_pinned()):
        raise ValueError("status must be an int32 device tensor or pinned host tensor")
    d = H.shape[0]
    _check("gptq_prepare_async",
           lib().gptq_prepare_async(_ptr(H), d, float(damp), int(bool(act_order)), _ptr(perm),
                                    _ptr(Hinv_chol), _ptr(ws), ws.numel(), _ptr(status),
                                    _stream(H, stream)))


def gptq_quantize(W: torch.Tensor, Hinv_chol: torch.Tensor, perm: torch.Tensor | None, bits: int,
                  group_size: int, block_size: int, scales: torch.Tensor, zeros: torch.Tensor,
                  ws: torch.Tensor, codes: torch.Tensor | None = None,
                  packed_int4: torch.Tensor | None = None, g_idx: torch.Tensor | None = None,
                  err_sq: torch.Tensor | None = None, stream=None):
    """W float32 [d_out, d_in] is overwritten with the dequantized weights."""
    _need(W, torch.float32, "W")
    d_out, d_in = W.shape
    _check("gptq_quantize",
           lib().gptq_quantize(_ptr(W), _ptr(Hinv_chol), _ptr(perm), d_out, d_in, bits,
                               group_size, block_size, _ptr(codes), _ptr(scales), _ptr(zeros),
                               _ptr(packed_int4), _ptr(g_idx), _ptr(err_sq), _ptr(ws),
                               ws.numel(), _stream(W, stream)))


def gptq_quantize_timed(W: torch.Tensor, Hinv_chol: torch.Tensor, perm: torch.Tensor | None, bits: int,
                        group_size: int, block_size: int, scales: torch.Tensor, zeros: torch.Tensor,
                        ws: torch.Tensor, codes: torch.Tensor | None = None,
                        packed_int4: torch.Tensor | None = None, g_idx: torch.Tensor | None = None,
                        err_sq: torch.Tensor | None = None, stream=None):
    """gptq_quantize with per-class device times: returns (column-loop ms,
    lazy-batch product ms, other ms) of this call (synchronises the stream).
    The first two are the kernels' own spans in the production launch
    sequence; other is the rest of the call's device time."""
    _need(W, torch.float32, "W")
    d_out, d_in = W.shape
    out = [ctypes.c_float(0.0) for _ in range(3)]
    _check("gptq_quantize_timed",
           lib().gptq_quantize_timed(_ptr(W), _ptr(Hinv_chol), _ptr(perm), d_out, d_in, bits,
                                     group_size, block_size, _ptr(codes), _ptr(scales), _ptr(zeros),
                                     _ptr(packed_int4), _ptr(g_idx), _ptr(err_sq), _ptr(ws),
                                     ws.numel(), _stream(W, stream), *(ctypes.byref(o) for o in out)))
    return tuple(o.value for o in out)


def gptq_quantize_q4k(W: torch.Tensor, Hinv_chol: torch.Tensor, perm: torch.Tensor | None,
                      out: dict, ws: torch.Tensor, codes: torch.Tensor | None = None,
                      packed_int4: torch.Tensor | None = None, g_idx: torch.Tensor | None = None,
                      err_sq: torch.Tensor | None = None, stream=None):
    """GPTQ onto the Q4_K grid; `out` holds the device tensors sc6, m6
    (uint8 [d_out, d_in/32]), dsup, dmin (float32 [d_out, d_in/256]) and
    scales, offsets (float32 [d_out, d_in/32])."""
    _need(W, torch.float32, "W")
    for k in ("sc6", "m6"):
        _need(out.get(k), torch.uint8, k)
    for k in ("dsup", "dmin", "scales", "offsets"):
        _need(out.get(k), torch.float32, k)
    d_out, d_in = W.shape
    _check("gptq_quantize_q4k",
           lib().gptq_quantize_q4k(_ptr(W), _ptr(Hinv_chol), _ptr(perm), d_out, d_in, _ptr(codes),
                                   _ptr(out["sc6"]), _ptr(out["m6"]), _ptr(out["dsup"]),
                                   _ptr(out["dmin"]), _ptr(out["scales"]), _ptr(out["offsets"]),
                                   _ptr(packed_int4), _ptr(g_idx), _ptr(err_sq), _ptr(ws),
                                   ws.numel(), _stream(W, stream)))


def gptq_quantize_static_scratch(W: torch.Tensor, Hinv_chol: torch.Tensor, perm: torch.Tensor | None,
                                 bits: int, group_size: int, block_size: int, scales: torch.Tensor,
                                 zeros: torch.Tensor, codes: torch.Tensor | None = None,
                                 packed_int4: torch.Tensor | None = None,
                                 g_idx: torch.Tensor | None = None,
                                 err_sq: torch.Tensor | None = None, stream=None):
    """gptq_quantize using the library's fixed scratch array (no workspace)."""
    _need(W, torch.float32, "W")
    d_out, d_in = W.shape
    _check("gptq_quantize_static_scratch",
           lib().gptq_quantize_static_scratch(_ptr(W), _ptr(Hinv_chol), _ptr(perm), d_out, d_in,
                                              bits, group_size, block_size, _ptr(codes),
                                              _ptr(scales), _ptr(zeros), _ptr(packed_int4),
                                              _ptr(g_idx), _ptr(err_sq), _stream(W, stream)))


def gptq_selftest_bounded_wait(limit_cycles: int) -> int:
    """Status of a deliberately unsatisfied, bounded device wait (expect 5)."""
    return lib().gptq_selftest_bounded_wait(int(limit_cycles))


def gptq_selftest_quotient(n_pairs: int, seed: int = 0) -> int:
    """Mismatches of the column loop's division-free quotient against IEEE
    division over n_pairs device-generated operand pairs (expect 0)."""
    out = ctypes.c_int64(-1)
    _check("gptq_selftest_quotient",
           lib().gptq_selftest_quotient(int(n_pairs), ctypes.c_uint64(seed), ctypes.byref(out)))
    return out.value


def gptq_w4a16_gemm(Y: torch.Tensor, X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                    zeros: torch.Tensor, g_idx: torch.Tensor | None, group_size: int,
                    path: int = W4A16_AUTO, stream=None):
    """Y float32 [M, N] = X (bf16 [M, K]) times the dequantized packed 4-bit
    weights (uint8 [N, K/2]) transposed."""
    _need(Y, torch.float32, "Y")
    _need(X, torch.bfloat16, "X")
    _need(packed, torch.uint8, "packed")
    M, K = X.shape
    N = packed.shape[0]
    if Y.shape != (M, N) or packed.shape[1] * 2 != K:
        raise ValueError("shape mismatch")
    _check("gptq_w4a16_gemm",
           lib().gptq_w4a16_gemm(_ptr(Y), _ptr(X), _ptr(packed), _ptr(scales), _ptr(zeros),
                                 _ptr(g_idx), M, N, K, group_size, path, _stream(Y, stream)))


def gptq_bf16_to_f32(dst: torch.Tensor, src: torch.Tensor, stream=None):
    _need(dst, torch.float32, "dst")
    _need(src, torch.bfloat16, "src")
    if dst.numel() != src.numel():
        raise ValueError("size mismatch")
    _check("gptq_bf16_to_f32",
           lib().gptq_bf16_to_f32(_ptr(dst), _ptr(src), src.numel(), _stream(dst, stream)))
