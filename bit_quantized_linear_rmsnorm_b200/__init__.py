"""Python binding of libbq.so, the sm_100a quantized linear layer.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind ``include/bq.h``.  PyTorch supplies device memory and the
current stream.  The functions carry the C names; each takes torch tensors,
allocates outputs (and workspaces) with torch when they are not given, and
raises ``BQError`` on a status other than BQ_OK.  There is no fallback: if
the library is missing or the device is not sm_100, calls fail loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbq.so")

# enums of bq.h
BQ_OK, BQ_ERR_INVALID_ARG, BQ_ERR_UNSUPPORTED, BQ_ERR_MISALIGNED, BQ_ERR_WORKSPACE, BQ_ERR_CUDA, BQ_ERR_TIMEOUT = range(7)
BQ_F32, BQ_BF16, BQ_F16 = 0, 1, 2
BQ_W_NK, BQ_W_KN = 0, 1
(BQ_OP_ACT_QUANT_INT8, BQ_OP_WEIGHT_QUANT_TERNARY_PACK, BQ_OP_WEIGHT_PACK_INT4_GROUPED,
 BQ_OP_GEMM_I8_PERTOKEN, BQ_OP_BITLINEAR_W2A8, BQ_OP_LINEAR_W4_GROUPED, BQ_OP_LINEAR_W4A4,
 BQ_OP_BITLINEAR_W2A8_BACKWARD, BQ_OP_LINEAR_W4A4_BACKWARD) = range(9)

EXPORTED = [
    "bq_act_quant_int8", "bq_weight_quant_ternary_pack", "bq_weight_pack_int4_grouped",
    "bq_gemm_i8_pertoken", "bq_gemm_i8_pertoken_batched", "bq_bitlinear_w2a8", "bq_act_quant_int8_layernorm",
    "bq_bitlinear_w2a8_layernorm", "bq_weight_quant_int4_pack", "bq_act_quant_int4", "bq_linear_w4a4",
    "bq_bitconv1d_weight_pack_workspace_bytes", "bq_bitconv1d_weight_pack", "bq_bitconv1d_workspace_bytes",
    "bq_bitconv1d", "bq_bitlinear_w2a8_backward", "bq_linear_w4a4_backward", "bq_linear_w4_grouped",
    "bq_workspace_bytes",
    "bq_bitlinear_workspace_layout", "bq_status_string", "bq_device_status", "bq_version",
    "bq_bitlinear_w2a8_noalloc", "bq_bitlinear_w2a8_path", "bq_diag_gemm_withheld_arrival",
]
(BQ_PATH_DECODE_STREAM, BQ_PATH_DECODE_MMA, BQ_PATH_DECODE_SMEM, BQ_PATH_ACT_QUANT_GEMV, BQ_PATH_TC_SINGLE,
 BQ_PATH_TC_PAIR) = range(1, 7)
BQ_NOALLOC_SCRATCH_BYTES = 2 * 1024 * 1024

_DTYPE = {torch.float32: BQ_F32, torch.bfloat16: BQ_BF16, torch.float16: BQ_F16}

P = ctypes.c_void_p
I64 = ctypes.c_int64
I32 = ctypes.c_int
SZ = ctypes.c_size_t
F32 = ctypes.c_float

_SIGS = {
    "bq_act_quant_int8": (I32, [P, I32, I64, I64, I64, F32, P, I64, P, P, P]),
    "bq_weight_quant_ternary_pack": (I32, [P, I32, I64, I64, P, P, P, SZ, P]),
    "bq_weight_pack_int4_grouped": (I32, [P, P, I64, I64, I64, P, P, P]),
    "bq_gemm_i8_pertoken": (I32, [P, I64, P, I32, I64, P, P, P, I64, I64, I64, I32, P, I64, P]),
    "bq_gemm_i8_pertoken_batched": (I32, [P, I64, I64, I32, P, I32, I64, I64, P, I64, P, I64, P, I64, I64, I64, I64,
                                          I32, P, I64, I64, P]),
    "bq_bitlinear_w2a8": (I32, [P, I32, I64, I64, P, P, I64, P, F32, I32, P, P, SZ, P]),
    "bq_act_quant_int8_layernorm": (I32, [P, I32, I64, I64, I64, P, P, F32, P, I64, P, P, P]),
    "bq_bitlinear_w2a8_layernorm": (I32, [P, I32, I64, I64, P, P, P, P, I64, P, F32, I32, P, P, SZ, P]),
    "bq_linear_w4_grouped": (I32, [P, I64, I64, P, P, P, P, I64, I64, P, P, SZ, P]),
    "bq_bitlinear_w2a8_noalloc": (I32, [P, I32, I64, I64, P, P, I64, P, F32, I32, P, P]),
    "bq_bitlinear_w2a8_path": (I32, [P, I32, I64, I64, I64, ctypes.POINTER(I32)]),
    "bq_diag_gemm_withheld_arrival": (I32, [P, P, P, P, P, ctypes.c_uint64, P]),
    "bq_weight_quant_int4_pack": (I32, [P, I32, I64, I64, P, I32, F32, P, P]),
    "bq_act_quant_int4": (I32, [P, I32, I64, I64, I64, P, F32, P, I64, P]),
    "bq_linear_w4a4": (I32, [P, I32, I64, I64, P, P, P, I32, I64, P, F32, I32, P, P, SZ, P]),
    "bq_bitconv1d_weight_pack_workspace_bytes": (SZ, [I64, I64, I64]),
    "bq_bitconv1d_weight_pack": (I32, [P, I32, I64, I64, I64, P, P, P, SZ, P]),
    "bq_bitconv1d_workspace_bytes": (SZ, [I64, I64, I64, I64, I64, I64, I64, I64]),
    "bq_bitconv1d": (I32, [P, I32, I64, I64, I64, P, P, P, P, I64, I64, I64, I64, I64, P, F32, I32, P, P, SZ, P]),
    "bq_bitlinear_w2a8_backward": (I32, [P, I32, P, I64, I64, P, P, I64, F32, P, P, P, SZ, P]),
    "bq_linear_w4a4_backward": (I32, [P, I32, P, P, I64, I64, I64, P, P, I32, F32, P, P, P, P, SZ, P]),
    "bq_workspace_bytes": (SZ, [I32, I64, I64, I64, I64]),
    "bq_bitlinear_workspace_layout": (None, [I64, I64, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
    "bq_status_string": (ctypes.c_char_p, [I32]),
    "bq_device_status": (I32, [P, ctypes.POINTER(ctypes.c_uint32)]),
    "bq_version": (I32, []),
}

_lib = None


class BQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {bq_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded libbq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                               "(nvcc, sm_100a); there is no fallback implementation")
        _lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != BQ_OK:
        raise BQError(status, where)


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a row-major 2-D tensor with unit inner stride")
    return t.stride(0)


def bq_status_string(status: int) -> str:
    return lib().bq_status_string(int(status)).decode()


def bq_version() -> int:
    return lib().bq_version()


def bq_workspace_bytes(op: int, M: int, N: int, K: int, group_size: int = 0) -> int:
    return int(lib().bq_workspace_bytes(op, M, N, K, group_size))


def bq_bitlinear_workspace_layout(M: int, K: int):
    a, b, c = SZ(), SZ(), SZ()
    lib().bq_bitlinear_workspace_layout(M, K, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return a.value, b.value, c.value


def bq_device_status(stream=None):
    detail = ctypes.c_uint32(0)
    st = lib().bq_device_status(_stream(stream), ctypes.byref(detail))
    return st, detail.value


def _workspace(nbytes: int, device, workspace=None):
    if workspace is not None:
        return workspace
    # 256-byte aligned (the caching allocator returns >= 512-byte aligned blocks)
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def bq_act_quant_int8(x: torch.Tensor, eps: float = 1e-5, xq=None, act_scale=None, rowsum=None,
                      want_rowsum: bool = True, stream=None):
    """(xq int8 [M,K], act_scale fp32 [M], rowsum int32 [M] or None)."""
    M, K = x.shape
    if xq is None:
        ldq = (K + 15) // 16 * 16
        xq = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
    if act_scale is None:
        act_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    if rowsum is None and want_rowsum:
        rowsum = torch.empty(M, dtype=torch.int32, device=x.device)
    st = lib().bq_act_quant_int8(_ptr(x), _DTYPE[x.dtype], M, K, _ld(x), float(eps), _ptr(xq), _ld(xq),
                                 _ptr(act_scale), _ptr(rowsum), _stream(stream))
    _check(st, "bq_act_quant_int8")
    return xq, act_scale, rowsum


def bq_act_quant_int8_layernorm(x: torch.Tensor, eps: float = 1e-5, ln_weight=None, ln_bias=None, xq=None,
                                act_scale=None, rowsum=None, want_rowsum: bool = True, stream=None):
    """LayerNorm (optional affine) + per-token int8 quantization:
    (xq int8 [M,K], act_scale fp32 [M], rowsum int32 [M] or None)."""
    M, K = x.shape
    if xq is None:
        ldq = (K + 15) // 16 * 16
        xq = torch.empty((M, ldq), dtype=torch.int8, device=x.device)[:, :K]
    if act_scale is None:
        act_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    if rowsum is None and want_rowsum:
        rowsum = torch.empty(M, dtype=torch.int32, device=x.device)
    st = lib().bq_act_quant_int8_layernorm(_ptr(x), _DTYPE[x.dtype], M, K, _ld(x), _ptr(ln_weight), _ptr(ln_bias),
                                           float(eps), _ptr(xq), _ld(xq), _ptr(act_scale), _ptr(rowsum),
                                           _stream(stream))
    _check(st, "bq_act_quant_int8_layernorm")
    return xq, act_scale, rowsum


def bq_bitlinear_w2a8_layernorm(x: torch.Tensor, wpacked: torch.Tensor, w_scale: torch.Tensor, N: int,
                                ln_weight=None, ln_bias=None, bias=None, eps: float = 1e-5, out_dtype=torch.bfloat16,
                                out=None, workspace=None, stream=None):
    """BitLinear forward with the LayerNorm normaliser."""
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    nbytes = bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8, M, N, K)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_bitlinear_w2a8_layernorm(_ptr(x), _DTYPE[x.dtype], M, K, _ptr(ln_weight), _ptr(ln_bias),
                                           _ptr(wpacked), _ptr(w_scale), N, _ptr(bias), float(eps), _DTYPE[out.dtype],
                                           _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_bitlinear_w2a8_layernorm")
    return out


def bq_weight_quant_ternary_pack(w: torch.Tensor, wpacked=None, w_scale=None, workspace=None, stream=None):
    """(wpacked uint32-as-int32 [N,K/16], w_scale fp32 [1])."""
    N, K = w.shape
    if wpacked is None:
        wpacked = torch.empty((N, K // 16), dtype=torch.int32, device=w.device)
    if w_scale is None:
        w_scale = torch.empty(1, dtype=torch.float32, device=w.device)
    nbytes = bq_workspace_bytes(BQ_OP_WEIGHT_QUANT_TERNARY_PACK, 0, N, K)
    ws = _workspace(nbytes, w.device, workspace)
    st = lib().bq_weight_quant_ternary_pack(_ptr(w), _DTYPE[w.dtype], N, K, _ptr(wpacked), _ptr(w_scale),
                                            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_weight_quant_ternary_pack")
    return wpacked, w_scale


def bq_weight_pack_int4_grouped(q: torch.Tensor, zeros: torch.Tensor, group_size: int, qweight=None, qzeros=None,
                                stream=None):
    """(qweight int32 [N,K/8], qzeros int32 [N,ceil(G/8)]) from uint8 codes."""
    N, K = q.shape
    G = K // group_size
    if qweight is None:
        qweight = torch.empty((N, K // 8), dtype=torch.int32, device=q.device)
    if qzeros is None:
        qzeros = torch.empty((N, (G + 7) // 8), dtype=torch.int32, device=q.device)
    st = lib().bq_weight_pack_int4_grouped(_ptr(q), _ptr(zeros), N, K, group_size, _ptr(qweight), _ptr(qzeros),
                                           _stream(stream))
    _check(st, "bq_weight_pack_int4_grouped")
    return qweight, qzeros


def bq_gemm_i8_pertoken(x: torch.Tensor, w: torch.Tensor, deq_scale: torch.Tensor, per_token_scale: torch.Tensor,
                        bias=None, w_layout: int = BQ_W_NK, out_dtype=torch.bfloat16, out=None, stream=None):
    """out[m,n] = (acc * deq_scale[n]) * per_token_scale[m] (+ bias[n])."""
    M, K = x.shape
    N = w.shape[0] if w_layout == BQ_W_NK else w.shape[1]
    if out is None:
        esz = torch.tensor([], dtype=out_dtype).element_size()
        pad = 16 // esz
        ldo = (N + pad - 1) // pad * pad
        out = torch.empty((M, ldo), dtype=out_dtype, device=x.device)[:, :N]
    st = lib().bq_gemm_i8_pertoken(_ptr(x), _ld(x), _ptr(w), w_layout, _ld(w), _ptr(deq_scale),
                                   _ptr(per_token_scale), _ptr(bias), M, N, K, _DTYPE[out.dtype], _ptr(out), _ld(out),
                                   _stream(stream))
    _check(st, "bq_gemm_i8_pertoken")
    return out


def _ld3(t: torch.Tensor):
    """(leading dimension, batch stride) of a [B, rows, cols] tensor with unit inner stride."""
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("expected a 3-D tensor with unit inner stride")
    return t.stride(1), t.stride(0)


def bq_gemm_i8_pertoken_batched(x: torch.Tensor, w: torch.Tensor, deq_scale: torch.Tensor,
                                per_token_scale: torch.Tensor, bias=None, w_layout: int = BQ_W_NK,
                                trans_a: bool = False, out_dtype=torch.bfloat16, out=None, stream=None):
    """Batched per-token W8A8 matmul.  x int8 [B,M,K] ([B,K,M] with trans_a);
    w int8 [B,N,K] (BQ_W_NK) or [B,K,N] (BQ_W_KN); deq_scale [N] / [B,N] and
    per_token_scale [M] / [B,M] (1-D: shared by every batch)."""
    B = x.shape[0]
    M, K = (x.shape[2], x.shape[1]) if trans_a else (x.shape[1], x.shape[2])
    N = w.shape[1] if w_layout == BQ_W_NK else w.shape[2]
    if out is None:
        esz = torch.tensor([], dtype=out_dtype).element_size()
        pad = 16 // esz
        ldo = (N + pad - 1) // pad * pad
        out = torch.empty((B, M, ldo), dtype=out_dtype, device=x.device)[:, :, :N]
    ldx, sx = _ld3(x)
    ldw, sw = _ld3(w)
    ldo_, so = _ld3(out)
    sd = deq_scale.stride(0) if deq_scale.dim() == 2 else 0
    sp = per_token_scale.stride(0) if per_token_scale.dim() == 2 else 0
    st = lib().bq_gemm_i8_pertoken_batched(_ptr(x), ldx, sx, int(bool(trans_a)), _ptr(w), w_layout, ldw, sw,
                                           _ptr(deq_scale), sd, _ptr(per_token_scale), sp, _ptr(bias), B, M, N, K,
                                           _DTYPE[out.dtype], _ptr(out), ldo_, so, _stream(stream))
    _check(st, "bq_gemm_i8_pertoken_batched")
    return out


def bq_bitlinear_w2a8(x: torch.Tensor, wpacked: torch.Tensor, w_scale: torch.Tensor, N: int, bias=None,
                      eps: float = 1e-5, out_dtype=torch.bfloat16, out=None, workspace=None, stream=None):
    """BitLinear forward: act quant into the workspace, ternary integer linear, rescale."""
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    nbytes = bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8, M, N, K)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_bitlinear_w2a8(_ptr(x), _DTYPE[x.dtype], M, K, _ptr(wpacked), _ptr(w_scale), N, _ptr(bias),
                                 float(eps), _DTYPE[out.dtype], _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream))
    _check(st, "bq_bitlinear_w2a8")
    return out


def bq_linear_w4_grouped(x: torch.Tensor, qweight: torch.Tensor, scales_f16: torch.Tensor, qzeros: torch.Tensor,
                         group_size: int, bias=None, out=None, workspace=None, stream=None):
    """out[m,n] = bias[n] + sum_k x[m,k] * s[n,g] * (q[n,k] - z[n,g])."""
    M, K = x.shape
    N = qweight.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    nbytes = bq_workspace_bytes(BQ_OP_LINEAR_W4_GROUPED, M, N, K, group_size)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_linear_w4_grouped(_ptr(x), M, K, _ptr(qweight), _ptr(scales_f16), _ptr(qzeros), _ptr(bias), N,
                                    group_size, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_linear_w4_grouped")
    return out


def bq_bitlinear_w2a8_noalloc(x: torch.Tensor, wpacked: torch.Tensor, w_scale: torch.Tensor, N: int, bias=None,
                              eps: float = 1e-5, out_dtype=torch.bfloat16, out=None, stream=None):
    """BitLinear forward that allocates nothing on the device beyond the output
    given (or allocated here by torch when `out` is None): the library keeps
    its scratch in a fixed static device array (see include/bq.h)."""
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    st = lib().bq_bitlinear_w2a8_noalloc(_ptr(x), _DTYPE[x.dtype], M, K, _ptr(wpacked), _ptr(w_scale), N, _ptr(bias),
                                         float(eps), _DTYPE[out.dtype], _ptr(out), _stream(stream))
    _check(st, "bq_bitlinear_w2a8_noalloc")
    return out


def bq_bitlinear_w2a8_path(x: torch.Tensor, N: int) -> int:
    """Which kernels bq_bitlinear_w2a8 runs for x [M,K] and N outputs (a BQ_PATH_* value)."""
    M, K = x.shape
    path = I32(0)
    st = lib().bq_bitlinear_w2a8_path(_ptr(x), _DTYPE[x.dtype], M, N, K, ctypes.byref(path))
    _check(st, "bq_bitlinear_w2a8_path")
    return path.value


def bq_weight_quant_int4_pack(w: torch.Tensor, scale_w: torch.Tensor, eps: float, wpacked=None, stream=None):
    """Signed 4-bit codes of w [N,K] with step max(scale_w, eps) (scale_w one
    value or [N]), packed eight per word: int32 [N, K/8]."""
    N, K = w.shape
    if wpacked is None:
        wpacked = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    per_channel = 1 if scale_w.numel() == N and N > 1 else 0
    st = lib().bq_weight_quant_int4_pack(_ptr(w), _DTYPE[w.dtype], N, K, _ptr(scale_w), per_channel, float(eps),
                                         _ptr(wpacked), _stream(stream))
    _check(st, "bq_weight_quant_int4_pack")
    return wpacked


def bq_act_quant_int4(x: torch.Tensor, scale_a: torch.Tensor, eps: float, xq=None, stream=None):
    """Signed 4-bit codes of x [M,K] (as int8) with step max(scale_a, eps)."""
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    st = lib().bq_act_quant_int4(_ptr(x), _DTYPE[x.dtype], M, K, _ld(x), _ptr(scale_a), float(eps), _ptr(xq), _ld(xq),
                                 _stream(stream))
    _check(st, "bq_act_quant_int4")
    return xq


def bq_linear_w4a4(x: torch.Tensor, scale_a: torch.Tensor, wpacked: torch.Tensor, scale_w: torch.Tensor, N: int,
                   eps: float, bias=None, out_dtype=torch.bfloat16, out=None, workspace=None, stream=None):
    """Forward of the 4-bit activation / 4-bit weight linear with given steps."""
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    per_channel = 1 if scale_w.numel() == N and N > 1 else 0
    nbytes = bq_workspace_bytes(BQ_OP_LINEAR_W4A4, M, N, K)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_linear_w4a4(_ptr(x), _DTYPE[x.dtype], M, K, _ptr(scale_a), _ptr(wpacked), _ptr(scale_w),
                              per_channel, N, _ptr(bias), float(eps), _DTYPE[out.dtype], _ptr(out), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_linear_w4a4")
    return out


def bq_bitconv1d_weight_pack(w: torch.Tensor, wpacked=None, w_scale=None, workspace=None, stream=None):
    """Ternary codes of a Conv1d weight [C_out, Cg, KS] packed per tap:
    (wpacked int32 [KS, C_out, Cgp/16], w_scale fp32 [1])."""
    C_out, Cg, KS = w.shape
    Cgp = (Cg + 63) // 64 * 64
    if wpacked is None:
        wpacked = torch.empty((KS, C_out, Cgp // 16), dtype=torch.int32, device=w.device)
    if w_scale is None:
        w_scale = torch.empty(1, dtype=torch.float32, device=w.device)
    ws = _workspace(int(lib().bq_bitconv1d_weight_pack_workspace_bytes(C_out, Cg, KS)), w.device, workspace)
    st = lib().bq_bitconv1d_weight_pack(_ptr(w.contiguous()), _DTYPE[w.dtype], C_out, Cg, KS, _ptr(wpacked),
                                        _ptr(w_scale), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_bitconv1d_weight_pack")
    return wpacked, w_scale


def bq_bitconv1d(x: torch.Tensor, wpacked: torch.Tensor, w_scale: torch.Tensor, C_out: int, kernel_size: int,
                 stride: int = 1, padding: int = 0, groups: int = 1, ln_weight=None, ln_bias=None, bias=None,
                 eps: float = 1e-5, out_dtype=torch.bfloat16, out=None, workspace=None, stream=None):
    """Ternary Conv1d forward: x (B, C_in, L) -> (B, C_out, L_out)."""
    B, C_in, L = x.shape
    L_out = (L + 2 * padding - kernel_size) // stride + 1
    if out is None:
        out = torch.empty((B, C_out, L_out), dtype=out_dtype, device=x.device)
    nbytes = int(lib().bq_bitconv1d_workspace_bytes(B, C_in, L, C_out, kernel_size, stride, padding, groups))
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_bitconv1d(_ptr(x), _DTYPE[x.dtype], B, C_in, L, _ptr(ln_weight), _ptr(ln_bias), _ptr(wpacked),
                            _ptr(w_scale), C_out, kernel_size, stride, padding, groups, _ptr(bias), float(eps),
                            _DTYPE[out.dtype], _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_bitconv1d")
    return out


def bq_bitlinear_w2a8_backward(x: torch.Tensor, dout: torch.Tensor, wpacked: torch.Tensor, w_scale: torch.Tensor,
                               eps: float = 1e-5, dx=None, dw=None, workspace=None, stream=None):
    """Straight-through backward of the BitLinear forward: (dx fp32 [M,K], dw fp32 [N,K])."""
    M, K = x.shape
    N = dout.shape[1]
    if dx is None:
        dx = torch.empty((M, K), dtype=torch.float32, device=x.device)
    if dw is None:
        dw = torch.empty((N, K), dtype=torch.float32, device=x.device)
    nbytes = bq_workspace_bytes(BQ_OP_BITLINEAR_W2A8_BACKWARD, M, N, K)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_bitlinear_w2a8_backward(_ptr(x), _DTYPE[x.dtype], _ptr(dout), M, K, _ptr(wpacked), _ptr(w_scale), N,
                                          float(eps), _ptr(dx), _ptr(dw), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream(stream))
    _check(st, "bq_bitlinear_w2a8_backward")
    return dx, dw


def bq_linear_w4a4_backward(x: torch.Tensor, w: torch.Tensor, dout: torch.Tensor, scale_a: torch.Tensor,
                            scale_w: torch.Tensor, eps: float, dx=None, dw=None, dscale_a=None, workspace=None,
                            stream=None):
    """Straight-through backward of the 4-bit activation / 4-bit weight linear:
    (dx fp32 [M,K], dw fp32 [N,K], dscale_a fp32 [1])."""
    M, K = x.shape
    N = w.shape[0]
    per_channel = 1 if scale_w.numel() == N and N > 1 else 0
    if dx is None:
        dx = torch.empty((M, K), dtype=torch.float32, device=x.device)
    if dw is None:
        dw = torch.empty((N, K), dtype=torch.float32, device=x.device)
    if dscale_a is None:
        dscale_a = torch.empty(1, dtype=torch.float32, device=x.device)
    nbytes = bq_workspace_bytes(BQ_OP_LINEAR_W4A4_BACKWARD, M, N, K)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().bq_linear_w4a4_backward(_ptr(x), _DTYPE[x.dtype], _ptr(w), _ptr(dout), M, K, N, _ptr(scale_a),
                                       _ptr(scale_w), per_channel, float(eps), _ptr(dx), _ptr(dw), _ptr(dscale_a),
                                       _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "bq_linear_w4a4_backward")
    return dx, dw, dscale_a
