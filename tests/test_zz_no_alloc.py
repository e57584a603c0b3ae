"""The allocation-free BitLinear entry point, bq_bitlinear_w2a8_noalloc.

It exists for callers that may not allocate device memory (a plugin whose
host framework owns every allocation, a decode loop where cudaMalloc would
synchronize the device): the scratch lives in a fixed static device array of
the library.  Its output must match the workspace entry point's
(bq_bitlinear_w2a8) within the parity tolerance, call after call, although
every call reuses the same scratch.  This file runs last (test_zz_*), alone
or after the other GPU tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_linear_rmsnorm_b200 as bq
import synth
from gpu_helpers import assert_out, bf16_dev, dev, host

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


def _case(M, N, K, xdtype, odtype, bias, seed):
    g = synth.rng((120, seed))
    w = synth.normal_f32(g, (N, K), 0.02)
    wp, ws = bq.bq_weight_quant_ternary_pack(dev(w))
    if xdtype == torch.bfloat16:
        bits, _ = synth.bf16_activations(M, K, (120, seed, 1), outlier_frac=0.01)
        x = bf16_dev(bits)
    else:
        x = dev(synth.normal_f32(g, (M, K)))
    b = dev(synth.normal_f32(g, (N,), 0.1)) if bias else None
    return x, wp, ws, b


@pytest.mark.parametrize("first,second", [
    ((300, 512, 1024, torch.bfloat16, torch.bfloat16, True), (5, 2048, 4096, torch.bfloat16, torch.bfloat16, False)),
    ((16, 11008, 4096, torch.bfloat16, torch.bfloat16, False), (64, 256, 2048, torch.float32, torch.float32, True)),
])
def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row(first, second):
    for i, (M, N, K, xd, od, bias) in enumerate((first, second)):
        x, wp, ws, b = _case(M, N, K, xd, od, bias, seed=(M, N, K, i))
        out = torch.full((M, N), float("nan"), dtype=od, device="cuda")
        assert _noalloc(x, wp, ws, N, b, out) == bq.BQ_OK
        ref = bq.bq_bitlinear_w2a8(x, wp, ws, N, b, 1e-5, od)
        torch.cuda.synchronize()
        r = host(ref).astype(np.float64)
        scale = None
        if b is not None:
            bb = host(b).astype(np.float64)
            scale = np.abs(r - bb) + np.abs(bb)
        assert_out(host(out), r, od, f"noalloc call {i + 1} {M}x{N}x{K}", scale=scale)


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
