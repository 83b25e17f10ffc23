"""ctypes binding of libgptq_b200.so: argument marshalling only.

Every function here passes raw device pointers, sizes and the current CUDA stream to the C ABI
declared in include/gptq.h; all arithmetic runs in the library's CUDA kernels. Loading fails
loudly when the shared library has not been built -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgptq_b200.so")

GPTQ_OK, GPTQ_EINVAL, GPTQ_ENOTPD, GPTQ_ECUDA, GPTQ_EUNSUPPORTED, GPTQ_ETIMEOUT, \
    GPTQ_EWORKSPACE = range(7)
GPTQ_BF16, GPTQ_FP32 = 0, 1
GPTQ_INFO_TIMEOUT = -1
GPTQ_INFO_BAD_HESSIAN = -2
GPTQ_INFO_BAD_CODE = -3
GPTQ_WS_PREPARE, GPTQ_WS_QUANTIZE = 1, 2
GPTQ_ROUTE_DEFAULT, GPTQ_ROUTE_THREE_STEP, GPTQ_ROUTE_REVERSED = 0, 1, 2
GPTQ_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
GPTQ_OBQ_NATURAL, GPTQ_OBQ_GREEDY = 0, 1

# name -> (restype, argtypes)
_P, _I64, _I32, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "gptq_hessian_accumulate": (_I32, [_P, _I64, _P, _I32, _I64, _I64, _P, _P]),
    "gptq_prepare_hinv": (_I32, [_P, _P, _I64, _I64, _F, _P, _SZ, _P, _P]),
    "gptq_prepare_hinv_route": (_I32, [_P, _P, _I64, _I64, _F, _I32, _P, _SZ, _P, _P]),
    "gptq_quantize_layer": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I32, _I32, _I32, _P, _P, _P,
                                   _P, _P, _P, _SZ, _P, _P]),
    "gptq_workspace_size": (_SZ, [_I32, _I64, _I64, _I32]),
    "gptq_info_status": (_I32, [ctypes.c_int32]),
    "gptq_status_string": (ctypes.c_char_p, [_I32]),
    "gptq_version": (ctypes.c_char_p, []),
    "gptq_quantize_layer_noalloc": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I32, _I32, _I32, _P,
                                           _P, _P, _P, _P, _P, _P]),
    "gptq_kernel_launches": (ctypes.c_uint64, []),
    "gptq_pack_codes_4bit": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "gptq_pack_codes_3bit": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "gptq_hadamard_block": (_I32, [_I64]),
    "gptq_obq_quantize": (_I32, [_P, _I64, _I64, _I64, _P, _I32, _I32, _P, _P, _P, _P, _P, _P,
                                 _P]),
    "gptq_hadamard_rotate": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _I32, _I64, _P]),
    "gptq_w4a16_matmul": (_I32, [_P, _P, _P, _I64, _I64, _I32, _P, _I32, _I64, _I64, _P, _I64, _P,
                                 _P]),
    "gptq_selftest_gemm": (_I32, [_P, _I64, _I32, _P, _I64, _I32, _P, _I64, _I32, _I32, _I32,
                                  _F, _F, _I32, _I32, _I32, _P, _P, _P, _SZ, _P, _P]),
    "gptq_selftest_wait_timeout": (_I32, [_P, _I32, _P]),
    "gptq_selftest_flag_timeout": (_I32, [_P, _P, _I32, _P]),
}

_lib = None


class GPTQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load():
    """Load libgptq_b200.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m post_weight_quantization_12_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().gptq_status_string(int(status)).decode()


def info_status(info: int) -> int:
    return int(load().gptq_info_status(int(info)))


def workspace_size(which: int, rows: int, cols: int, block: int) -> int:
    return int(load().gptq_workspace_size(which, rows, cols, block))


def kernel_launches() -> int:
    """Kernels the library has enqueued since it was loaded (diagnostic counter)."""
    return int(load().gptq_kernel_launches())


def selftest_wait_timeout(info, limit_ms: int, stream=None):
    """Enqueue a bounded wait that nothing will satisfy; it must end with GPTQ_INFO_TIMEOUT."""
    _check(load().gptq_selftest_wait_timeout(_ptr(info), int(limit_ms), _stream(stream)),
           "gptq_selftest_wait_timeout")


def selftest_flag_timeout(flag, info, limit_ms: int, stream=None):
    """One device thread waits (bounded) for the int32 flag to reach 1 (gptq_selftest_flag_timeout)."""
    _check(load().gptq_selftest_flag_timeout(_ptr(flag), _ptr(info), int(limit_ms), _stream(stream)),
           "gptq_selftest_flag_timeout")


def _check(st: int, where: str):
    if st != GPTQ_OK:
        raise GPTQError(st, where)


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return GPTQ_BF16
    if t.dtype == torch.float32:
        return GPTQ_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _row_major_ld(t, name):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    return t.stride(0)


def hessian_accumulate(S, X, info, stream=None):
    """S[cols, cols] (fp32) += X^T X for token-major X[n_tokens, >= cols] (bf16 or fp32)."""
    ldx = _row_major_ld(X, "X")
    st = load().gptq_hessian_accumulate(_ptr(S), S.shape[0], _ptr(X), _dtype_code(X), X.shape[0],
                                        ldx, _ptr(info), _stream(stream))
    _check(st, "gptq_hessian_accumulate")


def prepare_hinv(S_H, R, n_total, damp_rel, ws, info, stream=None, route=None):
    """S_H: S in, H = 2S/N out (both triangles); R: upper factor of (H + lambda I)^-1.

    route: None for gptq_prepare_hinv (the library's default route), else a GPTQ_ROUTE_* value
    passed to gptq_prepare_hinv_route."""
    args = (_ptr(S_H), _ptr(R), S_H.shape[0], int(n_total), float(damp_rel))
    tail = (_ptr(ws), ws.numel() * ws.element_size(), _ptr(info), _stream(stream))
    if route is None:
        st = load().gptq_prepare_hinv(*args, *tail)
    else:
        st = load().gptq_prepare_hinv_route(*args, int(route), *tail)
    _check(st, "gptq_prepare_hinv")


def quantize_layer(W, R, bits, group, block, W_hat, codes, scales, zeros, err_sq, ws, info,
                   stream=None):
    """GPTQ column loop over W[rows, cols] with the factor R; outputs are caller tensors."""
    ldw = _row_major_ld(W, "W")
    st = load().gptq_quantize_layer(
        _ptr(W), _dtype_code(W), W.shape[0], W.shape[1], ldw, _ptr(R), int(bits), int(group),
        int(block), _ptr(W_hat), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(err_sq), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(info), _stream(stream))
    _check(st, "gptq_quantize_layer")


def quantize_layer_noalloc(W, R, bits, group, block, W_hat, codes, scales, zeros, err_sq, info,
                           stream=None):
    """As quantize_layer, but with the library's built-in scratch instead of a workspace (for
    callers that cannot allocate device memory; limited to layers whose quantize workspace fits
    in GPTQ_NOALLOC_SCRATCH_BYTES; concurrent calls race on the shared scratch)."""
    ldw = _row_major_ld(W, "W")
    st = load().gptq_quantize_layer_noalloc(
        _ptr(W), _dtype_code(W), W.shape[0], W.shape[1], ldw, _ptr(R), int(bits), int(group),
        int(block), _ptr(W_hat), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(err_sq), _ptr(info),
        _stream(stream))
    _check(st, "gptq_quantize_layer_noalloc")


def pack_codes_4bit(codes, packed, info=None, stream=None):
    """uint8 codes[rows, >= cols] -> packed[rows, cols // 8] (int32 or uint32 tensor, the 32-bit
    words of the layout in include/gptq.h); cols = 8 * packed.shape[1]."""
    ldc = _row_major_ld(codes, "codes")
    if packed.dim() != 2 or not packed.is_contiguous() or packed.element_size() != 4:
        raise ValueError("packed must be a contiguous 2-D tensor of 32-bit words")
    st = load().gptq_pack_codes_4bit(_ptr(codes), codes.shape[0], 8 * packed.shape[1], ldc,
                                     _ptr(packed), _ptr(info), _stream(stream))
    _check(st, "gptq_pack_codes_4bit")


def pack_codes_3bit(codes, packed, info=None, stream=None):
    """uint8 codes[rows, >= cols] (values < 8) -> packed[rows, 3 cols // 32] (int32 or uint32
    tensor, the 32-bit words of the 3-bit layout in include/gptq.h); cols = 32 * packed.shape[1]
    // 3."""
    ldc = _row_major_ld(codes, "codes")
    if packed.dim() != 2 or not packed.is_contiguous() or packed.element_size() != 4 or \
            packed.shape[1] % 3:
        raise ValueError("packed must be a contiguous 2-D tensor of 32-bit words, 3 per 32 codes")
    st = load().gptq_pack_codes_3bit(_ptr(codes), codes.shape[0], 32 * (packed.shape[1] // 3),
                                     ldc, _ptr(packed), _ptr(info), _stream(stream))
    _check(st, "gptq_pack_codes_3bit")


def w4a16_matmul(packed, scales, zeros, group, X, Y, info=None, stream=None):
    """Y[n, rows] (fp32) = X[n, cols] (bf16) @ W_hat^T with W_hat dequantized from the packed
    4-bit codes[rows, cols // 8] and the scales / zeros [rows, G]."""
    if packed.dim() != 2 or not packed.is_contiguous() or packed.element_size() != 4:
        raise ValueError("packed must be a contiguous 2-D tensor of 32-bit words")
    ldx = _row_major_ld(X, "X")
    ldy = _row_major_ld(Y, "Y")
    st = load().gptq_w4a16_matmul(_ptr(packed), _ptr(scales), _ptr(zeros), packed.shape[0],
                                  8 * packed.shape[1], int(group), _ptr(X), _dtype_code(X),
                                  X.shape[0], ldx, _ptr(Y), ldy, _ptr(info), _stream(stream))
    _check(st, "gptq_w4a16_matmul")


def hadamard_block(n: int) -> int:
    """Order b of the Hadamard blocks the rotation uses for width n (0 for n <= 0)."""
    return int(load().gptq_hadamard_block(int(n)))


def hadamard_rotate(X, Y, sign_bits=None, stream=None):
    """Y[rows, n] = X[rows, n] Q (bf16 or fp32 each; Y may be X). sign_bits: int32/uint32 tensor
    of n // 32 words (bit j % 32 of word j // 32 set: column j negated) or None."""
    ldx, ldy = _row_major_ld(X, "X"), _row_major_ld(Y, "Y")
    if X.shape != Y.shape:
        raise ValueError("X and Y must have the same shape")
    st = load().gptq_hadamard_rotate(_ptr(X), _dtype_code(X), X.shape[0], X.shape[1], ldx,
                                     _ptr(sign_bits), _ptr(Y), _dtype_code(Y), ldy,
                                     _stream(stream))
    _check(st, "gptq_hadamard_rotate")


def obq_quantize(W, Hinv, bits, codes, W_hat, order=None, loss=None, scales=None, zeros=None,
                 greedy=True, stream=None):
    """OBQ on W[rows, cols <= 128] (fp32) with the shared fp64 inverse Hessian Hinv[cols, cols];
    outputs are caller tensors (codes uint8 / W_hat fp32 [rows, cols], order int32 [rows, cols],
    loss fp64 [rows], scales fp32 / zeros uint8 [rows]; the last four optional)."""
    ldw = _row_major_ld(W, "W")
    st = load().gptq_obq_quantize(
        _ptr(W), W.shape[0], W.shape[1], ldw, _ptr(Hinv), int(bits),
        GPTQ_OBQ_GREEDY if greedy else GPTQ_OBQ_NATURAL, _ptr(codes), _ptr(W_hat), _ptr(order),
        _ptr(loss), _ptr(scales), _ptr(zeros), _stream(stream))
    _check(st, "gptq_obq_quantize")


def selftest_gemm(A, a_mn, B, b_mn, C, M, N, K, alpha=1.0, beta=0.0, lower=False,
                  klo_from_m=False, klo_from_n=False, C_big=None, C_small=None, info=None,
                  stream=None):
    """The library's tensor-core (3xTF32) matrix product on fp32 device tensors (self-test)."""
    import torch
    lda, ldb = _row_major_ld(A, "A"), _row_major_ld(B, "B")
    ldc = _row_major_ld(C, "C") if C is not None else (C_big.stride(0) if C_big is not None else 4)
    ws = torch.empty(2 * (A.shape[0] * lda + B.shape[0] * ldb) * 4 + 2048, dtype=torch.uint8,
                     device=A.device)
    st = load().gptq_selftest_gemm(_ptr(A), lda, int(a_mn), _ptr(B), ldb, int(b_mn), _ptr(C), ldc,
                                   int(M), int(N), int(K), float(alpha), float(beta), int(lower),
                                   int(klo_from_m), int(klo_from_n), _ptr(C_big), _ptr(C_small),
                                   _ptr(ws), ws.numel(), _ptr(info), _stream(stream))
    _check(st, "gptq_selftest_gemm")
