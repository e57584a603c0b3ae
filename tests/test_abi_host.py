"""C-ABI checks that need no GPU: the library loads, exports every call the
header declares, and rejects invalid arguments before launching anything."""
import ctypes
import os
import re

import pytest

import bit_quantized_linear_rmsnorm_b200 as bq
from bit_quantized_linear_rmsnorm_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return bq.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "bq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_six_calls():
    names = _declared()
    for n in ["bq_act_quant_int8", "bq_weight_quant_ternary_pack", "bq_weight_pack_int4_grouped",
              "bq_gemm_i8_pertoken", "bq_bitlinear_w2a8", "bq_linear_w4_grouped"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in _declared():
        assert hasattr(L, n), n
    assert set(_declared()) <= set(bq.EXPORTED)


def test_version_and_strings(L):
    assert bq.bq_version() >= 100
    assert bq.bq_status_string(bq.BQ_OK) == "ok"
    assert "workspace" in bq.bq_status_string(bq.BQ_ERR_WORKSPACE)
    assert bq.bq_status_string(99) == "unknown status"


def test_workspace_sizes(L):
    assert bq.bq_workspace_bytes(bq.BQ_OP_GEMM_I8_PERTOKEN, 4096, 4096, 4096) == 0
    n = bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 16, 11008, 4096)
    xo, so, ro = bq.bq_bitlinear_workspace_layout(16, 4096)
    assert xo == 0 and so >= 16 * 4096 and ro >= so + 16 * 4 and n >= ro + 16 * 4
    assert so % 256 == 0 and ro % 256 == 0
    assert bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4_GROUPED, 32, 14336, 4096, 128) >= 3 * 32 * 4096
    assert bq.bq_workspace_bytes(bq.BQ_OP_WEIGHT_QUANT_TERNARY_PACK, 0, 4096, 4096) > 0
    assert bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4_GROUPED, 1, 1, 128, 0) == 0


FAKE = ctypes.c_void_p(0x10000)      # 64 KiB-aligned, never dereferenced
ODD = ctypes.c_void_p(0x10001)


def test_act_quant_rejects(L):
    f = L.bq_act_quant_int8
    assert f(None, bq.BQ_F32, 4, 64, 64, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, 7, 4, 64, 64, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F16, 4, 64, 64, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F32, 4, 0, 64, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F32, 4, 64, 32, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F32, 4, 64, 64, float("nan"), FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F32, 4, 64, 64, -1.0, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F32, 4, 64, 64, 1e-5, ODD, 64, FAKE, None, None) == bq.BQ_ERR_MISALIGNED
    assert f(FAKE, bq.BQ_F32, 4, 64, 64, 1e-5, FAKE, 72, FAKE, None, None) == bq.BQ_ERR_MISALIGNED
    # empty batch is a valid no-op
    assert f(None, bq.BQ_F32, 0, 64, 64, 1e-5, None, 64, None, None, None) == bq.BQ_OK


def test_ternary_pack_rejects(L):
    f = L.bq_weight_quant_ternary_pack
    assert f(FAKE, bq.BQ_F32, 8, 24, FAKE, FAKE, FAKE, 1 << 20, None) == bq.BQ_ERR_INVALID_ARG  # K % 16
    assert f(FAKE, bq.BQ_F32, 8, 32, FAKE, FAKE, None, 0, None) == bq.BQ_ERR_WORKSPACE
    assert f(FAKE, bq.BQ_F32, 8, 32, FAKE, FAKE, FAKE, 1, None) == bq.BQ_ERR_WORKSPACE
    assert f(ODD, bq.BQ_F32, 8, 32, FAKE, FAKE, FAKE, 1 << 20, None) == bq.BQ_ERR_MISALIGNED
    assert f(None, bq.BQ_F32, 0, 32, None, None, None, 0, None) == bq.BQ_OK


def test_int4_pack_rejects(L):
    f = L.bq_weight_pack_int4_grouped
    assert f(FAKE, FAKE, 4, 12, 4, FAKE, FAKE, None) == bq.BQ_ERR_INVALID_ARG   # K % 8
    assert f(FAKE, FAKE, 4, 64, 48, FAKE, FAKE, None) == bq.BQ_ERR_INVALID_ARG  # gs does not divide K
    assert f(FAKE, FAKE, 4, 64, 0, FAKE, FAKE, None) == bq.BQ_ERR_INVALID_ARG
    assert f(ODD, FAKE, 4, 64, 16, FAKE, FAKE, None) == bq.BQ_ERR_MISALIGNED


def _gemm(L, x=FAKE, ldx=64, w=FAKE, wl=0, ldw=64, deq=FAKE, pts=FAKE, bias=None, M=4, N=64, K=64, od=bq.BQ_BF16,
          out=FAKE, ldo=64):
    return L.bq_gemm_i8_pertoken(x, ldx, w, wl, ldw, deq, pts, bias, M, N, K, od, out, ldo, None)


def test_gemm_rejects(L):
    assert _gemm(L, K=0) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, K=131072, ldx=131072, ldw=131072) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, wl=5) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, od=9) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, ldx=32) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, ldo=32) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, x=None) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, deq=None) == bq.BQ_ERR_INVALID_ARG
    assert _gemm(L, x=ODD) == bq.BQ_ERR_MISALIGNED
    assert _gemm(L, ldx=72) == bq.BQ_ERR_MISALIGNED
    assert _gemm(L, ldo=68) == bq.BQ_ERR_MISALIGNED          # 68 * 2 bytes is not a multiple of 16
    assert _gemm(L, deq=ctypes.c_void_p(0x10010)) == bq.BQ_ERR_MISALIGNED  # deqScale 32-byte rule
    assert _gemm(L, M=0) == bq.BQ_OK
    assert _gemm(L, N=0, ldo=64) == bq.BQ_OK


def test_bitlinear_rejects(L):
    f = L.bq_bitlinear_w2a8
    ok = dict(x=FAKE, xt=bq.BQ_BF16, M=32, K=128, wp=FAKE, ws_=FAKE, N=64, bias=None, eps=1e-5, od=bq.BQ_BF16,
              out=FAKE, work=FAKE, nbytes=1 << 24)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["x"], a["xt"], a["M"], a["K"], a["wp"], a["ws_"], a["N"], a["bias"], a["eps"], a["od"], a["out"],
                 a["work"], a["nbytes"], None)
    assert call(K=40) == bq.BQ_ERR_INVALID_ARG
    assert call(xt=bq.BQ_F16) == bq.BQ_ERR_INVALID_ARG
    assert call(work=None) == bq.BQ_ERR_WORKSPACE
    assert call(nbytes=16) == bq.BQ_ERR_WORKSPACE
    assert call(work=ctypes.c_void_p(0x10040)) == bq.BQ_ERR_MISALIGNED
    assert call(x=ODD) == bq.BQ_ERR_MISALIGNED
    assert call(out=ctypes.c_void_p(0x10008)) == bq.BQ_ERR_MISALIGNED
    assert call(M=0) == bq.BQ_OK
    assert call(N=0, wp=None) == bq.BQ_OK
    # ragged N and K % 64 != 0 are valid at any M (the tensor-core path stages
    # them through the workspace), so validation lets them through
    for kw in (dict(N=61), dict(K=144), dict(N=61, K=144, od=bq.BQ_F16)):
        assert call(**kw) not in (bq.BQ_ERR_INVALID_ARG, bq.BQ_ERR_MISALIGNED, bq.BQ_ERR_WORKSPACE), kw


def test_bitlinear_workspace_grows_for_tensor_core_tails(L):
    base = bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 300, 64, 128)
    assert bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 300, 61, 128) >= base + 300 * 64 * 4
    assert bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 300, 64, 144) >= base + 64 * 192 // 4
    # up to 16 tokens (decode kernels) nothing is staged
    xo, so, ro = bq.bq_bitlinear_workspace_layout(16, 144)
    assert bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 16, 61, 144) == ro + 256


def test_noalloc_checks_arguments_like_the_workspace_entry_point(L):
    """bq_bitlinear_w2a8_noalloc answers every invalid call exactly as
    bq_bitlinear_w2a8 does (minus the workspace, which it does not take),
    before it looks at its scratch limit or at the device."""
    ok = dict(x=FAKE, xt=bq.BQ_BF16, M=32, K=128, wp=FAKE, ws_=FAKE, N=64, bias=None, eps=1e-5, od=bq.BQ_BF16,
              out=FAKE)

    def both(**kw):
        a = dict(ok, **kw)
        na = L.bq_bitlinear_w2a8_noalloc(a["x"], a["xt"], a["M"], a["K"], a["wp"], a["ws_"], a["N"], a["bias"],
                                         a["eps"], a["od"], a["out"], None)
        wa = L.bq_bitlinear_w2a8(a["x"], a["xt"], a["M"], a["K"], a["wp"], a["ws_"], a["N"], a["bias"], a["eps"],
                                 a["od"], a["out"], FAKE, 1 << 40, None)
        return na, wa
    # invalid arguments, even where the scratch would also be too small
    for kw in (dict(K=40), dict(K=131072 + 16, M=4096), dict(K=131088), dict(xt=bq.BQ_F16), dict(od=7),
               dict(eps=float("nan")), dict(eps=-1.0), dict(M=-1), dict(x=None), dict(out=None), dict(ws_=None),
               dict(M=4096, K=4096, x=None)):
        na, wa = both(**kw)
        assert na == wa == bq.BQ_ERR_INVALID_ARG, (kw, na, wa)
    for kw in (dict(x=ODD), dict(out=ctypes.c_void_p(0x10008)), dict(bias=ODD), dict(M=4096, K=4096, x=ODD)):
        na, wa = both(**kw)
        assert na == wa == bq.BQ_ERR_MISALIGNED, (kw, na, wa)
    # valid empty calls: nothing to do
    for kw in (dict(M=0), dict(N=0), dict(M=0, x=None, out=None)):
        na, wa = both(**kw)
        assert na == wa == bq.BQ_OK, (kw, na, wa)
    # only a valid call too large for the static scratch gets BQ_ERR_WORKSPACE
    na, _ = both(M=1024, K=4096)
    assert na == bq.BQ_ERR_WORKSPACE


def test_linear_w4_rejects(L):
    f = L.bq_linear_w4_grouped

    def call(M=1, K=256, gs=128, N=8, work=FAKE, nbytes=1 << 24, x=FAKE):
        return f(x, M, K, FAKE, FAKE, FAKE, None, N, gs, FAKE, work, nbytes, None)
    assert call(K=100) == bq.BQ_ERR_INVALID_ARG
    assert call(gs=12) == bq.BQ_ERR_INVALID_ARG
    assert call(gs=96) == bq.BQ_ERR_INVALID_ARG
    assert call(K=65544, gs=8) == bq.BQ_ERR_INVALID_ARG
    assert call(work=None) == bq.BQ_ERR_WORKSPACE
    assert call(x=ODD) == bq.BQ_ERR_MISALIGNED
    assert call(M=0) == bq.BQ_OK


def test_gemm_batched_rejects(L):
    f = L.bq_gemm_i8_pertoken_batched

    def call(x=FAKE, ldx=64, sx=64 * 64, ta=0, w=FAKE, wl=0, ldw=64, sw=64 * 64, deq=FAKE, sd=0, pts=FAKE, sp=0,
             bias=None, B=2, M=64, N=64, K=64, od=bq.BQ_BF16, out=FAKE, ldo=64, so=64 * 64):
        return f(x, ldx, sx, ta, w, wl, ldw, sw, deq, sd, pts, sp, bias, B, M, N, K, od, out, ldo, so, None)
    assert call(B=-1) == bq.BQ_ERR_INVALID_ARG
    assert call(ta=2) == bq.BQ_ERR_INVALID_ARG
    assert call(sx=64 * 63) == bq.BQ_ERR_INVALID_ARG          # batches would overlap
    assert call(sw=16) == bq.BQ_ERR_INVALID_ARG
    assert call(so=64) == bq.BQ_ERR_INVALID_ARG
    assert call(sd=32) == bq.BQ_ERR_INVALID_ARG               # a per-batch deqScale needs N entries
    assert call(sp=-64) == bq.BQ_ERR_INVALID_ARG
    assert call(ta=1, ldx=32) == bq.BQ_ERR_INVALID_ARG        # transposed x is [K][ldx >= M]
    assert call(sx=64 * 64 + 8) == bq.BQ_ERR_MISALIGNED
    assert call(sd=66) == bq.BQ_ERR_MISALIGNED                # each batch's deqScale 32-byte aligned
    assert call(B=0) == bq.BQ_OK
    assert call(B=1, sx=0, sw=0, so=0, x=ODD) == bq.BQ_ERR_MISALIGNED
    # batch 1 ignores the strides
    assert call(B=1, sx=0, sw=0, so=0, sd=0) not in (bq.BQ_ERR_INVALID_ARG, bq.BQ_ERR_MISALIGNED)


def test_layernorm_calls_reject(L):
    f = L.bq_act_quant_int8_layernorm
    assert f(FAKE, bq.BQ_F32, 4, 64, 64, None, None, 1e-5, FAKE, 64, FAKE, None, None) not in (
        bq.BQ_ERR_INVALID_ARG, bq.BQ_ERR_MISALIGNED)
    assert f(FAKE, bq.BQ_F16, 4, 64, 64, None, None, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_INVALID_ARG
    assert f(FAKE, bq.BQ_F32, 4, 64, 64, ODD, None, 1e-5, FAKE, 64, FAKE, None, None) == bq.BQ_ERR_MISALIGNED
    assert f(None, bq.BQ_F32, 0, 64, 64, None, None, 1e-5, None, 64, None, None, None) == bq.BQ_OK
    g = L.bq_bitlinear_w2a8_layernorm
    assert g(FAKE, bq.BQ_BF16, 32, 40, None, None, FAKE, FAKE, 64, None, 1e-5, bq.BQ_BF16, FAKE, FAKE, 1 << 24,
             None) == bq.BQ_ERR_INVALID_ARG
    assert g(FAKE, bq.BQ_BF16, 32, 128, None, ODD, FAKE, FAKE, 64, None, 1e-5, bq.BQ_BF16, FAKE, FAKE, 1 << 24,
             None) == bq.BQ_ERR_MISALIGNED
    assert g(FAKE, bq.BQ_BF16, 32, 128, None, None, FAKE, FAKE, 64, None, 1e-5, bq.BQ_BF16, FAKE, None, 0,
             None) == bq.BQ_ERR_WORKSPACE


def test_w4a4_calls_reject(L):
    f = L.bq_linear_w4a4

    def call(x=FAKE, xt=bq.BQ_BF16, M=32, K=128, sa=FAKE, wp=FAKE, sw=FAKE, pc=1, N=64, bias=None, eps=1e-6,
             od=bq.BQ_BF16, out=FAKE, work=FAKE, nbytes=1 << 24):
        return f(x, xt, M, K, sa, wp, sw, pc, N, bias, eps, od, out, work, nbytes, None)
    assert call(K=48) == bq.BQ_ERR_INVALID_ARG          # K % 32
    assert call(eps=0.0) == bq.BQ_ERR_INVALID_ARG
    assert call(pc=2) == bq.BQ_ERR_INVALID_ARG
    assert call(sa=None) == bq.BQ_ERR_INVALID_ARG
    assert call(wp=ctypes.c_void_p(0x10008)) == bq.BQ_ERR_MISALIGNED
    assert call(work=None) == bq.BQ_ERR_WORKSPACE
    assert call(nbytes=64) == bq.BQ_ERR_WORKSPACE
    assert call(M=0) == bq.BQ_OK
    g = L.bq_weight_quant_int4_pack
    assert g(FAKE, bq.BQ_F32, 8, 12, FAKE, 0, 1e-6, FAKE, None) == bq.BQ_ERR_INVALID_ARG   # K % 8
    assert g(FAKE, bq.BQ_F32, 8, 16, None, 0, 1e-6, FAKE, None) == bq.BQ_ERR_INVALID_ARG
    assert g(None, bq.BQ_F32, 0, 16, None, 0, 1e-6, None, None) == bq.BQ_OK
    a = L.bq_act_quant_int4
    assert a(FAKE, bq.BQ_F16, 4, 16, 16, FAKE, 1e-6, FAKE, 16, None) == bq.BQ_ERR_INVALID_ARG
    assert a(FAKE, bq.BQ_F32, 4, 16, 8, FAKE, 1e-6, FAKE, 16, None) == bq.BQ_ERR_INVALID_ARG
    ws = bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4A4, 300, 61, 256)
    assert ws >= 300 * 256 + 300 * 4 + 61 * 4 + 300 * 64 * 4


def test_bitconv1d_calls_reject(L):
    f = L.bq_bitconv1d

    def call(x=FAKE, xt=bq.BQ_BF16, B=2, C_in=64, Lx=32, lw=None, lb=None, wp=FAKE, ws_=FAKE, C_out=32, KS=3,
             stride=1, pad=1, groups=1, bias=None, eps=1e-5, od=bq.BQ_BF16, out=FAKE, work=FAKE, nbytes=1 << 26):
        return f(x, xt, B, C_in, Lx, lw, lb, wp, ws_, C_out, KS, stride, pad, groups, bias, eps, od, out, work, nbytes,
                 None)
    assert call(C_in=40) == bq.BQ_ERR_INVALID_ARG           # C_in % 16
    assert call(groups=3) == bq.BQ_ERR_INVALID_ARG          # groups divides C_in and C_out
    assert call(groups=2, C_out=36) == bq.BQ_ERR_INVALID_ARG  # (C_out / groups) % 4
    assert call(KS=40, pad=0) == bq.BQ_ERR_INVALID_ARG      # no output position
    assert call(stride=0) == bq.BQ_ERR_INVALID_ARG
    assert call(work=None) == bq.BQ_ERR_WORKSPACE
    assert call(x=ODD) == bq.BQ_ERR_MISALIGNED
    assert call(B=0) == bq.BQ_OK
    assert bq.lib().bq_bitconv1d_workspace_bytes(2, 64, 32, 32, 3, 1, 1, 1) > 3 * 2 * 32 * 32 * 4
    g = L.bq_bitconv1d_weight_pack
    assert g(FAKE, bq.BQ_F32, 32, 24, 3, FAKE, FAKE, FAKE, 1 << 24, None) == bq.BQ_ERR_INVALID_ARG  # Cg % 16
    assert g(FAKE, bq.BQ_F32, 32, 32, 3, FAKE, FAKE, None, 0, None) == bq.BQ_ERR_WORKSPACE


def test_backward_rejects(L):
    f = L.bq_bitlinear_w2a8_backward

    def call(x=FAKE, xt=bq.BQ_BF16, d=FAKE, M=32, K=128, wp=FAKE, ws_=FAKE, N=64, eps=1e-5, dx=FAKE, dw=FAKE,
             work=FAKE, nbytes=1 << 26):
        return f(x, xt, d, M, K, wp, ws_, N, eps, dx, dw, work, nbytes, None)
    assert call(K=40) == bq.BQ_ERR_INVALID_ARG
    assert call(N=60) == bq.BQ_ERR_INVALID_ARG     # N % 8 (bf16 rows of dout, 16-byte pitch)
    assert call(d=None) == bq.BQ_ERR_INVALID_ARG
    assert call(d=ODD) == bq.BQ_ERR_MISALIGNED
    assert call(work=None) == bq.BQ_ERR_WORKSPACE
    assert call(M=0, dw=None) == bq.BQ_ERR_INVALID_ARG  # M == 0 writes dw as zeros: it must exist
    assert call(M=0, N=0) == bq.BQ_OK                    # no gradient to write
    assert bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8_BACKWARD, 32, 64, 128) >= 32 * 128 * 5 + 64 * 128 * 2


def test_w4a4_backward_rejects(L):
    f = L.bq_linear_w4a4_backward

    def call(x=FAKE, xt=bq.BQ_BF16, w=FAKE, d=FAKE, M=32, K=128, N=64, sa=FAKE, sw=FAKE, pc=0, eps=1e-6, dx=FAKE,
             dw=FAKE, ds=FAKE, work=FAKE, nbytes=1 << 26):
        return f(x, xt, w, d, M, K, N, sa, sw, pc, eps, dx, dw, ds, work, nbytes, None)
    assert call(K=40) == bq.BQ_ERR_INVALID_ARG     # K % 16
    assert call(N=60) == bq.BQ_ERR_INVALID_ARG     # N % 8
    assert call(eps=0.0) == bq.BQ_ERR_INVALID_ARG  # the steps need eps > 0
    assert call(pc=2) == bq.BQ_ERR_INVALID_ARG
    assert call(xt=bq.BQ_F16) == bq.BQ_ERR_INVALID_ARG
    assert call(ds=None) == bq.BQ_ERR_INVALID_ARG
    assert call(w=ODD) == bq.BQ_ERR_MISALIGNED
    assert call(dx=ODD) == bq.BQ_ERR_MISALIGNED
    assert call(work=None) == bq.BQ_ERR_WORKSPACE
    assert call(nbytes=16) == bq.BQ_ERR_WORKSPACE
    assert call(M=0, dw=None) == bq.BQ_ERR_INVALID_ARG
    need = bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4A4_BACKWARD, 32, 64, 128)
    assert need >= 32 * 128 * (2 + 4) + 2 * 64 * 128 * 2 + 32 * 2 * 64 * 2
