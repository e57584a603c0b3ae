"""Failure detection on the GPU without a fault.

Every wait of the tensor-core GEMM is bounded.  The diagnostic entry point
bq_diag_gemm_withheld_arrival runs the single-CTA kernel on one tile with a
short limit while its producer withholds the copies of one K block, so a
wait runs out: the kernel must record BQ_ERR_TIMEOUT with the site of the
wait, drain its own asynchronous work, free its tensor memory and return, the
host must read that status, and the next ordinary call must run correctly.
Nothing here traps, faults or waits without a limit.
"""
import time

import numpy as np
import pytest
import torch

import bit_quantized_linear_rmsnorm_b200 as bq
import oracle
import synth
from gpu_helpers import assert_out, dev, host

pytestmark = pytest.mark.gpu

SITE_GEMM_MMA, SITE_GEMM_EPILOGUE = 2, 3


@pytest.fixture(scope="module", autouse=True)
def _ready():
    from bit_quantized_linear_rmsnorm_b200 import _build
    _build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    torch.cuda.init()
    assert bq.bq_device_status()[0] == bq.BQ_OK
    yield


def _inputs():
    d = synth.gemm_w8a8(128, 256, 256, seed=21)
    return d, dev(d["x"]), dev(d["w"]), dev(d["deq_scale"]), dev(d["per_token_scale"])


@pytest.mark.parametrize("limit_ns", [1_000_000, 200_000])
def test_withheld_arrival_times_out_and_the_next_call_runs(limit_ns):
    d, x, w, deq, pts = _inputs()
    out = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    ptr = lambda t: t.data_ptr()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st = bq.lib().bq_diag_gemm_withheld_arrival(ptr(x), ptr(w), ptr(deq), ptr(pts), ptr(out), limit_ns,
                                                torch.cuda.current_stream().cuda_stream)
    assert st == bq.BQ_OK
    status, detail = bq.bq_device_status()  # synchronizes the stream
    elapsed = time.perf_counter() - t0
    assert status == bq.BQ_ERR_TIMEOUT, f"status word {detail:#x}"
    assert (detail >> 8) in (SITE_GEMM_MMA, SITE_GEMM_EPILOGUE), f"site {detail >> 8}"
    assert elapsed < 1.0, f"the kernel took {elapsed:.3f} s to give up"
    assert bq.bq_device_status()[0] == bq.BQ_OK  # read and cleared
    # the context is intact: an ordinary call on the same inputs is correct
    o = bq.bq_gemm_i8_pertoken(x, w, deq, pts)
    torch.cuda.synchronize()
    ref, _ = oracle.gemm_i8_pertoken(d["x"], d["w"], d["deq_scale"], d["per_token_scale"])
    assert_out(host(o), ref, torch.bfloat16, "GEMM after a timeout")
    assert bq.bq_device_status()[0] == bq.BQ_OK


def test_withheld_arrival_rejects_bad_limits():
    _, x, w, deq, pts = _inputs()
    out = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    f = bq.lib().bq_diag_gemm_withheld_arrival
    s = torch.cuda.current_stream().cuda_stream
    assert f(x.data_ptr(), w.data_ptr(), deq.data_ptr(), pts.data_ptr(), out.data_ptr(), 10, s) == \
        bq.BQ_ERR_INVALID_ARG
    assert f(x.data_ptr(), w.data_ptr(), deq.data_ptr(), pts.data_ptr(), out.data_ptr(), 3_000_000_000, s) == \
        bq.BQ_ERR_INVALID_ARG
    assert f(None, w.data_ptr(), deq.data_ptr(), pts.data_ptr(), out.data_ptr(), 1_000_000, s) == \
        bq.BQ_ERR_INVALID_ARG
    assert bq.bq_device_status()[0] == bq.BQ_OK
