"""The allocation-free BitLinear entry point, bq_bitlinear_w2a8_noalloc.

It exists for callers that may not allocate device memory (a plugin whose
host framework owns every allocation, a decode loop where cudaMalloc would
synchronize the device): the scratch lives in a fixed static device array of
the library.  Every call reuses that array, so each case runs two calls in a
row on different shapes; each call's output must be bit-identical to the
workspace entry point's (bq_bitlinear_w2a8, same kernels, same inputs) and
within the parity tolerance of the oracle.  The sequences cover every way the
scratch is used: written by the fused decode kernels only, written by the
activation-quantization kernel and read by the GEMV kernel, and read by the
tensor-core GEMM together with its re-pitched weights and staged outputs.
This file runs last (test_zz_*), alone or after the other GPU tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_linear_rmsnorm_b200 as bq
import synth
from gpu_helpers import assert_out, bf16_dev, bitlinear_expected, bitlinear_rel32, dev, host

pytestmark = pytest.mark.gpu

_OUT = {torch.bfloat16: bq.BQ_BF16, torch.float16: bq.BQ_F16, torch.float32: bq.BQ_F32}
_IN = {torch.bfloat16: bq.BQ_BF16, torch.float32: bq.BQ_F32}


@pytest.fixture(scope="module", autouse=True)
def _ready():
    from bit_quantized_linear_rmsnorm_b200 import _build
    _build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    torch.cuda.init()
    yield
    st, detail = bq.bq_device_status()
    assert st == bq.BQ_OK, f"device status word {detail:#x}"


def _noalloc(x, wp, ws, N, bias, out):
    """Calls the C entry point directly through ctypes."""
    M, K = x.shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return bq.lib().bq_bitlinear_w2a8_noalloc(p(x), _IN[x.dtype], M, K, p(wp), p(ws), N, p(bias), 1e-5,
                                              _OUT[out.dtype], p(out),
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(M, N, K, xdtype, bias, seed):
    g = synth.rng((120, seed))
    w = synth.normal_f32(g, (N, K), 0.02)
    wp, ws = bq.bq_weight_quant_ternary_pack(dev(w))
    if xdtype == torch.bfloat16:
        bits, xf = synth.bf16_activations(M, K, (120, seed, 1), outlier_frac=0.01)
        x = bf16_dev(bits)
    else:
        xf = synth.normal_f32(g, (M, K))
        x = dev(xf)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    return x, xf, w, wp, ws, b


def _dev_or_none(a):
    return None if a is None else dev(a)


_SEQUENCES = [
    # tensor-core GEMM (scratch: codes, scales, row sums), then the activation-
    # quantization kernel writing the scratch and the GEMV kernel reading it
    [(300, 512, 1024, torch.bfloat16, torch.bfloat16, True, bq.BQ_PATH_TC_SINGLE),
     (4, 1000, 1040, torch.bfloat16, torch.float32, False, bq.BQ_PATH_ACT_QUANT_GEMV)],
    # fused decode (writes the scratch only), then the GEMM on fp32 inputs
    [(16, 11008, 4096, torch.bfloat16, torch.bfloat16, False, bq.BQ_PATH_DECODE_MMA),
     (64, 256, 2048, torch.float32, torch.float32, True, bq.BQ_PATH_TC_SINGLE)],
    # GEMM with re-pitched weights and staged output rows, then one-token decode
    [(300, 61, 144, torch.bfloat16, torch.float16, True, bq.BQ_PATH_TC_SINGLE),
     (1, 300, 1024, torch.bfloat16, torch.bfloat16, False, bq.BQ_PATH_DECODE_SMEM)],
]


@pytest.mark.parametrize("seq", _SEQUENCES, ids=["gemm-then-gemv", "decode-then-gemm", "tails-then-decode"])
def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row(seq):
    for i, (M, N, K, xd, od, bias, path) in enumerate(seq):
        x, xf, w, wp, ws, b = _case(M, N, K, xd, bias, seed=(M, N, K, i))
        bd = _dev_or_none(b)
        assert bq.bq_bitlinear_w2a8_path(x, N) == path
        out = torch.full((M, N), float("nan"), dtype=od, device="cuda")
        assert _noalloc(x, wp, ws, N, bd, out) == bq.BQ_OK
        work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K), dtype=torch.uint8,
                           device="cuda")
        ref_out = bq.bq_bitlinear_w2a8(x, wp, ws, N, bd, 1e-5, od, workspace=work)
        torch.cuda.synchronize()
        what = f"noalloc call {i + 1} {M}x{N}x{K}"
        # same kernels on the same inputs: the same bits
        bits = torch.int32 if od == torch.float32 else torch.int16
        assert torch.equal(out.view(bits), ref_out.view(bits)), what + ": not bit-identical"
        # and the oracle, on the same seeded inputs
        _, so, _ = bq.bq_bitlinear_workspace_layout(M, K)
        g_sc = host(work[so:so + 4 * M].view(torch.float32))
        ref, extra, scale, a, t = bitlinear_expected(xf, w, b, 1e-5)
        rel32 = bitlinear_rel32(g_sc, a["act_scale"], host(ws)[0], t["gamma"])
        assert_out(host(out), ref, od, what, extra=extra, scale=scale, rel32=rel32)


def test_noalloc_rejects_scratch_beyond_the_limit():
    M, N, K = 1024, 64, 4096  # 4 MB of int8 activations > the 2 MB scratch
    assert bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K) > bq.BQ_NOALLOC_SCRATCH_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    wp = torch.zeros((N, K // 16), dtype=torch.int32, device="cuda")
    ws = torch.ones(1, dtype=torch.float32, device="cuda")
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(x, wp, ws, N, None, out) == bq.BQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
