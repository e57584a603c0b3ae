"""Oracle for the quantized linear layer (test infrastructure only).

Plain double-precision host C in ``bq_oracle.c``, wrapped here with ctypes
and numpy for argument marshalling.  Only the tests, ``__graft_entry__.smoke``
and the benchmark's CPU-baseline leg may import this package; the product
path (``bit_quantized_linear_rmsnorm_b200``) never does, and the two share no
code.  See ``bq_oracle.c`` for the page citations and the readings taken where
the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# No fast-math and no contraction into fused multiply-add: every operation in
# the oracle is one correctly rounded binary64 operation.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc if it is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None

P = ctypes.c_void_p
I64 = ctypes.c_int64
F64 = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        sig = {
            "bq_oracle_round_half_even": (F64, [F64]),
            "bq_oracle_act_quant": (None, [P, I64, I64, F64, P, P, P, P, P]),
            "bq_oracle_act_quant_layernorm": (None, [P, I64, I64, F64, P, P, P, P, P, P, P]),
            "bq_oracle_ternary_quant": (ctypes.c_int, [P, I64, I64, P, P, P]),
            "bq_oracle_ternary_bake": (None, [P, F64, I64, P]),
            "bq_oracle_ternary_pack": (None, [P, I64, I64, P]),
            "bq_oracle_ternary_unpack": (I64, [P, I64, I64, P]),
            "bq_oracle_int4_pack": (None, [P, I64, I64, P]),
            "bq_oracle_int4_unpack": (None, [P, I64, I64, P]),
            "bq_oracle_half_to_double": (F64, [ctypes.c_uint16]),
            "bq_oracle_gemm_i8_pertoken": (I64, [P, I64, P, ctypes.c_int, I64, P, P, P, I64, I64, I64, P]),
            "bq_oracle_gemm_i8_pertoken_batched": (I64, [P, I64, I64, ctypes.c_int, P, ctypes.c_int, I64, I64, P, I64,
                                                          P, I64, P, I64, I64, I64, I64, P]),
            "bq_oracle_bitlinear_from_codes": (None, [P, P, P, F64, P, I64, I64, I64, P, P]),
            "bq_oracle_linear_w4_grouped": (None, [P, I64, I64, P, P, P, P, I64, I64, P]),
            "bq_oracle_q4_quant": (None, [P, I64, I64, P, I64, F64, P, P]),
            "bq_oracle_bitlinear_backward": (None, [P, P, P, I64, I64, I64, F64, P, P]),
            "bq_oracle_bitconv1d_from_codes": (None, [P, P, P, F64, P, I64, I64, I64, I64, I64, I64, I64, I64, P]),
            "bq_oracle_linear_w4a4_from_codes": (None, [P, P, P, P, I64, F64, P, I64, I64, I64, P]),
            "bq_oracle_s4_pack": (None, [P, I64, I64, P]),
            "bq_oracle_linear_w4a4_backward": (None, [P, P, P, P, P, I64, F64, I64, I64, I64, P, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _c(a, dtype):
    """Contiguous array of the given dtype (a copy only when needed)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def round_half_even(v: float) -> float:
    return lib().bq_oracle_round_half_even(float(v))


def act_quant(x, eps: float = 1e-5, want_pre: bool = False, want_y: bool = False):
    """RMSNorm + per-token absmax int8 quantization of x [M,K] (float32 values).

    Returns dict with xq int8 [M,K], act_scale f64 [M], rowsum int64 [M] and,
    when asked, the pre-rounding values ``pre`` and the normalised ``y``.
    """
    x = _c(x, np.float32)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sc = np.empty(M, np.float64)
    rs = np.empty(M, np.int64)
    pre = np.empty((M, K), np.float64) if want_pre else None
    y = np.empty((M, K), np.float64) if want_y else None
    lib().bq_oracle_act_quant(_p(x), M, K, float(eps), _p(xq), _p(sc), _p(rs), _p(pre), _p(y))
    out = {"xq": xq, "act_scale": sc, "rowsum": rs}
    if want_pre:
        out["pre"] = pre
    if want_y:
        out["y"] = y
    return out


def act_quant_layernorm(x, eps: float = 1e-5, ln_weight=None, ln_bias=None, want_pre: bool = False,
                        want_y: bool = False):
    """LayerNorm (optional affine ln_weight / ln_bias [K]) + per-token absmax
    int8 quantization of x [M,K]; returns the same dict as act_quant."""
    x = _c(x, np.float32)
    M, K = x.shape
    gw = None if ln_weight is None else _c(ln_weight, np.float32)
    gb = None if ln_bias is None else _c(ln_bias, np.float32)
    xq = np.empty((M, K), np.int8)
    sc = np.empty(M, np.float64)
    rs = np.empty(M, np.int64)
    pre = np.empty((M, K), np.float64) if want_pre else None
    y = np.empty((M, K), np.float64) if want_y else None
    lib().bq_oracle_act_quant_layernorm(_p(x), M, K, float(eps), _p(gw), _p(gb), _p(xq), _p(sc), _p(rs), _p(pre),
                                        _p(y))
    out = {"xq": xq, "act_scale": sc, "rowsum": rs}
    if want_pre:
        out["pre"] = pre
    if want_y:
        out["y"] = y
    return out


def bitlinear_layernorm(x, w, eps: float = 1e-5, ln_weight=None, ln_bias=None, bias=None):
    """BitLinear forward with the LayerNorm normaliser."""
    a = act_quant_layernorm(x, eps, ln_weight, ln_bias)
    t = ternary_quant(w)
    out = bitlinear_from_codes(a["xq"], a["act_scale"], t["wq"], t["gamma"], bias)
    return out, a, t


def ternary_quant(w, want_pre: bool = False):
    """Absmean ternary quantization with the bake rule; w float32 [N,K]."""
    w = _c(w, np.float32)
    N, K = w.shape
    g = np.zeros(1, np.float64)
    wq = np.empty((N, K), np.int8)
    pre = np.empty((N, K), np.float64) if want_pre else None
    baked = lib().bq_oracle_ternary_quant(_p(w), N, K, _p(g), _p(wq), _p(pre))
    out = {"wq": wq, "gamma": float(g[0]), "already_ternary": bool(baked)}
    if want_pre:
        out["pre"] = pre
    return out


def ternary_bake(wq, gamma: float):
    wq = _c(wq, np.int8)
    out = np.empty(wq.shape, np.float32)
    lib().bq_oracle_ternary_bake(_p(wq), float(gamma), wq.size, _p(out))
    return out


def ternary_pack(wq):
    wq = _c(wq, np.int8)
    N, K = wq.shape
    assert K % 16 == 0
    out = np.empty((N, K // 16), np.uint32)
    lib().bq_oracle_ternary_pack(_p(wq), N, K, _p(out))
    return out


def ternary_unpack(packed, K: int):
    packed = _c(packed, np.uint32)
    N = packed.shape[0]
    wq = np.empty((N, K), np.int8)
    bad = lib().bq_oracle_ternary_unpack(_p(packed), N, K, _p(wq))
    return wq, int(bad)


def int4_pack(q):
    q = _c(q, np.uint8)
    rows, cols = q.shape
    out = np.empty((rows, (cols + 7) // 8), np.uint32)
    lib().bq_oracle_int4_pack(_p(q), rows, cols, _p(out))
    return out


def int4_unpack(packed, cols: int):
    packed = _c(packed, np.uint32)
    rows = packed.shape[0]
    q = np.empty((rows, cols), np.uint8)
    lib().bq_oracle_int4_unpack(_p(packed), rows, cols, _p(q))
    return q


def half_to_double(bits: int) -> float:
    return lib().bq_oracle_half_to_double(int(bits) & 0xFFFF)


def gemm_i8_pertoken(x, w, deq_scale, per_token_scale, bias=None, layout: int = 0):
    """acc = x @ weight, out = acc * deqScale[n] * perTokenScale[m] (+ bias[n]).

    x int8 [M,K]; w int8 [N,K] (layout 0) or [K,N] (layout 1).  Returns
    (out f64 [M,N], number of accumulators outside int32).
    """
    x = _c(x, np.int8)
    w = _c(w, np.int8)
    M, K = x.shape
    N = w.shape[0] if layout == 0 else w.shape[1]
    deq = _c(deq_scale, np.float32)
    pts = _c(per_token_scale, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((M, N), np.float64)
    ovf = lib().bq_oracle_gemm_i8_pertoken(_p(x), K, _p(w), int(layout), w.shape[1], _p(deq), _p(pts),
                                           _p(b), M, N, K, _p(out))
    return out, int(ovf)


def gemm_i8_pertoken_batched(x, w, deq_scale, per_token_scale, bias=None, layout: int = 0, trans_a: bool = False,
                             shared_scales: bool = True):
    """Batched per-token W8A8 matmul.  x int8 [B,M,K] ([B,K,M] with trans_a);
    w int8 [B,N,K] (layout 0) or [B,K,N] (layout 1); deq_scale [N] and
    per_token_scale [M] shared by every batch (shared_scales) or [B,N] and
    [B,M].  Returns (out f64 [B,M,N], number of accumulators outside int32)."""
    x = _c(x, np.int8)
    w = _c(w, np.int8)
    B = x.shape[0]
    M, K = (x.shape[2], x.shape[1]) if trans_a else (x.shape[1], x.shape[2])
    N = w.shape[1] if layout == 0 else w.shape[2]
    deq = _c(deq_scale, np.float32)
    pts = _c(per_token_scale, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((B, M, N), np.float64)
    ovf = lib().bq_oracle_gemm_i8_pertoken_batched(
        _p(x), x.shape[2], x.shape[1] * x.shape[2], int(bool(trans_a)), _p(w), int(layout), w.shape[2],
        w.shape[1] * w.shape[2], _p(deq), 0 if shared_scales else N, _p(pts), 0 if shared_scales else M, _p(b),
        B, M, N, K, _p(out))
    return out, int(ovf)


def bitlinear_from_codes(xq, act_scale, wq, gamma: float, bias=None, want_acc: bool = False):
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    sc = _c(act_scale, np.float64)
    M, K = xq.shape
    N = wq.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((M, N), np.float64)
    acc = np.empty((M, N), np.int64) if want_acc else None
    lib().bq_oracle_bitlinear_from_codes(_p(xq), _p(sc), _p(wq), float(gamma), _p(b), M, N, K, _p(out), _p(acc))
    return (out, acc) if want_acc else out


def bitlinear(x, w, eps: float = 1e-5, bias=None):
    """Whole BitLinear forward: act quant, ternary quant, integer linear, rescale."""
    a = act_quant(x, eps)
    t = ternary_quant(w)
    out = bitlinear_from_codes(a["xq"], a["act_scale"], t["wq"], t["gamma"], bias)
    return out, a, t


def linear_w4_grouped(x, qweight, scales_f16_bits, qzeros, bias, group_size: int):
    x = _c(x, np.float32)
    M, K = x.shape
    qw = _c(qweight, np.uint32)
    N = qw.shape[0]
    sc = _c(scales_f16_bits, np.uint16)
    qz = _c(qzeros, np.uint32)
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((M, N), np.float64)
    lib().bq_oracle_linear_w4_grouped(_p(x), M, K, _p(qw), _p(sc), _p(qz), _p(b), N, int(group_size), _p(out))
    return out


def q4_quant(v, scale, eps: float, per_row: bool = False, want_pre: bool = False):
    """Signed 4-bit codes of v [rows, cols] with step max(scale, eps): one
    step (scale of one element) or one per row (scale [rows])."""
    v = _c(v, np.float32)
    rows, cols = v.shape
    sc = _c(np.atleast_1d(scale), np.float32)
    q = np.empty((rows, cols), np.int8)
    pre = np.empty((rows, cols), np.float64) if want_pre else None
    lib().bq_oracle_q4_quant(_p(v), rows, cols, _p(sc), 1 if per_row else 0, float(eps), _p(q), _p(pre))
    return (q, pre) if want_pre else q


def linear_w4a4_from_codes(xq, wq, scale_a, scale_w, eps: float, bias=None, per_channel: bool = False):
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    sa = _c(np.atleast_1d(scale_a), np.float32)
    sw = _c(np.atleast_1d(scale_w), np.float32)
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((M, N), np.float64)
    lib().bq_oracle_linear_w4a4_from_codes(_p(xq), _p(wq), _p(sa), _p(sw), 1 if per_channel else 0, float(eps),
                                           _p(b), M, N, K, _p(out))
    return out


def linear_w4a4(x, w, scale_a, scale_w, eps: float, bias=None, per_channel: bool = False):
    """The whole W4A4 forward: 4-bit codes of x and w, integer linear, rescale."""
    xq = q4_quant(x, scale_a, eps)
    wq = q4_quant(w, scale_w, eps, per_row=per_channel)
    return linear_w4a4_from_codes(xq, wq, scale_a, scale_w, eps, bias, per_channel), xq, wq


def linear_w4a4_backward(x, w, dout, scale_a, scale_w, eps: float, per_channel: bool = False):
    """Straight-through backward of the W4A4 forward: dict of dx f64 [M,K],
    dw f64 [N,K], dscale_a (float) and g f64 [M,K] (the gradient reaching the
    dequantized activations, before the range mask)."""
    x = _c(x, np.float32)
    w = _c(w, np.float32)
    dout = _c(dout, np.float32)
    M, K = x.shape
    N = w.shape[0]
    sa = _c(np.atleast_1d(scale_a), np.float32)
    sw = _c(np.atleast_1d(scale_w), np.float32)
    dx = np.empty((M, K), np.float64)
    dw = np.empty((N, K), np.float64)
    ds = np.zeros(1, np.float64)
    g = np.empty((M, K), np.float64)
    lib().bq_oracle_linear_w4a4_backward(_p(x), _p(w), _p(dout), _p(sa), _p(sw), 1 if per_channel else 0,
                                         float(eps), M, N, K, _p(dx), _p(dw), _p(ds), _p(g))
    return {"dx": dx, "dw": dw, "dscale_a": float(ds[0]), "g": g}


def s4_pack(q):
    q = _c(q, np.int8)
    rows, cols = q.shape
    assert cols % 8 == 0
    out = np.empty((rows, cols // 8), np.uint32)
    lib().bq_oracle_s4_pack(_p(q), rows, cols, _p(out))
    return out


def bitconv1d_act_quant(x, eps: float = 1e-5, ln_weight=None, ln_bias=None, want_pre: bool = False):
    """Per-position LayerNorm over the channels + int8 quantization of x (B, C, L):
    the act quant of the rows of x transposed to (B, L, C).  Returns the
    act_quant_layernorm dict with xq [B*L, C] and act_scale [B*L]."""
    x = _c(x, np.float32)
    B, C, L = x.shape
    rows = np.ascontiguousarray(x.transpose(0, 2, 1).reshape(B * L, C))
    return act_quant_layernorm(rows, eps, ln_weight, ln_bias, want_pre=want_pre)


def bitconv1d_from_codes(xq, act_scale, wq, gamma: float, B: int, L: int, stride: int = 1, pad: int = 0,
                         groups: int = 1, bias=None):
    """Ternary Conv1d from position-major codes xq [B*L, C_in], act_scale [B*L]
    and weight codes wq [C_out, C_in/groups, KS]; returns out f64 (B, C_out, L_out)."""
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    sc = _c(act_scale, np.float64)
    C_in = xq.shape[1]
    C_out, _, KS = wq.shape
    L_out = (L + 2 * pad - KS) // stride + 1
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((B, C_out, L_out), np.float64)
    lib().bq_oracle_bitconv1d_from_codes(_p(xq), _p(sc), _p(wq), float(gamma), _p(b), B, C_in, L, C_out, KS, stride,
                                         pad, groups, _p(out))
    return out


def bitconv1d(x, w, eps: float = 1e-5, stride: int = 1, pad: int = 0, groups: int = 1, ln_weight=None, ln_bias=None,
              bias=None):
    """Whole BitConv1d forward: per-position LayerNorm + int8 quant, ternary
    weight quant, convolution of the dequantized values."""
    x = _c(x, np.float32)
    B, C, L = x.shape
    a = bitconv1d_act_quant(x, eps, ln_weight, ln_bias)
    t = ternary_quant(np.ascontiguousarray(w, np.float32).reshape(w.shape[0], -1))
    wq = t["wq"].reshape(w.shape)
    out = bitconv1d_from_codes(a["xq"], a["act_scale"], wq, t["gamma"], B, L, stride, pad, groups, bias)
    return out, a, t


def bitlinear_backward(x, w, dout, eps: float = 1e-5):
    """STE backward of the BitLinear forward: (dx f64 [M,K], dw f64 [N,K])."""
    x = _c(x, np.float32)
    w = _c(w, np.float32)
    dout = _c(dout, np.float32)
    M, K = x.shape
    N = w.shape[0]
    dx = np.empty((M, K), np.float64)
    dw = np.empty((N, K), np.float64)
    lib().bq_oracle_bitlinear_backward(_p(x), _p(w), _p(dout), M, N, K, float(eps), _p(dx), _p(dw))
    return dx, dw
