"""Parity of every C-ABI call with the oracle, on identical seeded inputs.

Sizes span several tiles with ragged tails; the benchmark workloads run at
full size (outputs compared on whole rows sampled by the oracle).  Integer
results are bit-exact except codes whose exact pre-rounding value lies within
1e-6 (relative) of a .5 boundary; dequantized outputs are within 1 bf16/fp16
ulp or 1e-5 relative (fp32); grouped INT4 outputs within 1e-4*sqrt(K/128)
absolute.
"""
import math

import numpy as np
import pytest
import torch

import bit_quantized_linear_rmsnorm_b200 as bq
import oracle
import synth
from gpu_helpers import (assert_codes, assert_out, bf16_dev, bitlinear_expected, bitlinear_rel32, dev, host,
                         padded, tie_band)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _ready():
    from bit_quantized_linear_rmsnorm_b200 import _build
    _build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    torch.cuda.init()
    yield
    st, detail = bq.bq_device_status()
    assert st == bq.BQ_OK, f"device status word {detail:#x}"


# ----------------------------------------------------------------- act quant

def _check_act(x_f32, x_dev, eps, what):
    xq, sc, rs = bq.bq_act_quant_int8(x_dev, eps)
    torch.cuda.synchronize()
    ref = oracle.act_quant(x_f32, eps, want_pre=True)
    g_xq = host(xq)
    assert_codes(g_xq, ref["xq"], ref["pre"], what)
    np.testing.assert_allclose(host(sc), ref["act_scale"], rtol=1e-5, err_msg=what)
    np.testing.assert_array_equal(host(rs), g_xq.astype(np.int64).sum(axis=1))
    return g_xq


@pytest.mark.parametrize("M,K,dtype", [(8, 256, "f32"), (37, 1000, "bf16"), (5, 4096, "bf16"),
                                       (300, 4096, "bf16"), (3, 6000, "f32"), (64, 8200, "bf16"),
                                       (1, 7, "f32"), (17, 33, "bf16"),
                                       # many rows: one CTA per row at a time (chunk counts 1..8 per thread)
                                       (1300, 4096, "bf16"), (700, 4096, "f32"), (2000, 512, "bf16"),
                                       (650, 1000, "f32"), (900, 8192, "bf16")])
def test_act_quant(M, K, dtype):
    g = synth.rng((101, M, K))
    x = synth.normal_f32(g, (M, K))
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(x)
        x = synth.bf16_bits_to_f32(bits)
        xd = bf16_dev(bits)
    else:
        xd = dev(x)
    _check_act(x, xd, 1e-5, f"act_quant {M}x{K} {dtype}")


def test_act_quant_special_rows():
    K = 512
    x = synth.normal_f32(synth.rng(102), (6, K))
    x[0] = 0.0                 # zero row
    x[1] = 0.75                # constant row
    x[2] = 0.0
    x[2, 100] = -3.0           # one-hot row
    x[3] *= 1e-6               # tiny row: eps dominates the RMS
    x[4, :] = np.float32(2.0 ** -20)
    _check_act(x, dev(x), 1e-5, "special rows")
    xq, sc, _ = bq.bq_act_quant_int8(dev(x), 1e-5)
    assert np.all(host(xq)[0] == 0) and host(sc)[0] == pytest.approx(1e-5 / 127, rel=1e-6)
    assert np.all(host(xq)[1] == 127)


def test_act_quant_unaligned_rows_scalar_path():
    M, K = 9, 300
    x = synth.normal_f32(synth.rng(103), (M, K + 1))
    xd = dev(x)[:, 1:]  # base 4 bytes off 16, stride 301 floats
    _check_act(np.ascontiguousarray(x[:, 1:]), xd, 1e-5, "unaligned")


def test_act_quant_outlier_channels_prefill_rows():
    bits, xf = synth.bf16_activations(256, 4096, (5, 1), outlier_frac=0.01)
    _check_act(xf, bf16_dev(bits), 1e-5, "outliers")


# ------------------------------------------------------------ ternary pack

def _check_ternary(w_f32, w_dev, what):
    wp, ws = bq.bq_weight_quant_ternary_pack(w_dev)
    torch.cuda.synchronize()
    ref = oracle.ternary_quant(w_f32, want_pre=True)
    gamma = float(host(ws)[0])
    assert gamma == pytest.approx(ref["gamma"], rel=1e-6), what
    K = w_f32.shape[1]
    codes, bad = oracle.ternary_unpack(host(wp).view(np.uint32), K)
    assert bad == 0, f"{what}: invalid 2-bit code"
    assert_codes(codes, ref["wq"], ref["pre"] + 0.0, what)
    if not tie_band(ref["pre"]).any():
        np.testing.assert_array_equal(host(wp).view(np.uint32), oracle.ternary_pack(ref["wq"]))
    return wp, ws, ref


@pytest.mark.parametrize("N,K,dtype", [(128, 256, "f32"), (300, 512, "f32"), (64, 4096, "bf16"), (5, 16, "f32")])
def test_ternary_pack(N, K, dtype):
    w = synth.normal_f32(synth.rng((104, N, K)), (N, K), 0.02)
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(w)
        _check_ternary(synth.bf16_bits_to_f32(bits), bf16_dev(bits), f"ternary {N}x{K} bf16")
    else:
        _check_ternary(w, dev(w), f"ternary {N}x{K}")


def test_ternary_pack_full_decode_weight():
    w = synth.bitlinear_weight(11008, 4096, 3)
    _check_ternary(w, dev(w), "ternary 11008x4096")


def test_ternary_pack_bake_rule_and_edges():
    w = np.zeros((16, 64), np.float32)
    _, ws, ref = _check_ternary(w, dev(w), "all zero")
    assert float(host(ws)[0]) == pytest.approx(1e-5, rel=1e-6)
    g = synth.rng(105)
    w = (g.integers(-1, 2, (32, 64)) * 0.37).astype(np.float32)
    _, ws, ref = _check_ternary(w, dev(w), "already ternary")
    assert ref["already_ternary"] and float(host(ws)[0]) == np.float32(0.37)
    # bake(W) packs to the same words and scale as W itself
    w = synth.normal_f32(g, (48, 128), 0.02)
    wp1, ws1, r1 = _check_ternary(w, dev(w), "master")
    baked = oracle.ternary_bake(r1["wq"], r1["gamma"])
    wp2, ws2, _ = _check_ternary(baked, dev(baked), "baked")
    np.testing.assert_array_equal(host(wp1), host(wp2))
    assert float(host(ws2)[0]) == pytest.approx(float(host(ws1)[0]), rel=1e-6)


# --------------------------------------------------------------- INT4 pack

@pytest.mark.parametrize("N,K,gs", [(14336, 4096, 128), (7, 192, 8), (3, 40, 8), (5, 64, 64)])
def test_int4_pack(N, K, gs):
    g = synth.rng((106, N, K))
    q = synth.nibbles(g, (N, K))
    z = synth.nibbles(g, (N, K // gs))
    qw, qz = bq.bq_weight_pack_int4_grouped(dev(q), dev(z), gs)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(qw).view(np.uint32), oracle.int4_pack(q))
    np.testing.assert_array_equal(host(qz).view(np.uint32), oracle.int4_pack(z))


def test_int4_pack_flags_codes_above_15():
    q = np.full((2, 16), 3, np.uint8)
    q[1, 5] = 0x13
    z = np.zeros((2, 2), np.uint8)
    qw, _ = bq.bq_weight_pack_int4_grouped(dev(q), dev(z), 8)
    st, detail = bq.bq_device_status()
    assert st == bq.BQ_ERR_INVALID_ARG
    assert (detail >> 8) == 16
    assert bq.bq_device_status()[0] == bq.BQ_OK  # read-and-clear
    q[1, 5] = 3
    np.testing.assert_array_equal(host(qw).view(np.uint32), oracle.int4_pack(q))


# ------------------------------------------------------------- W8A8 GEMM

_TORCH_OUT = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


def _gemm_case(M, N, K, layout, out, bias, seed):
    d = synth.gemm_w8a8(M, N, K, seed)
    w = d["w"] if layout == bq.BQ_W_NK else np.ascontiguousarray(d["w"].T)
    b = synth.normal_f32(synth.rng((seed, 7)), (N,), 0.5) if bias else None
    xd = padded(d["x"], 16)
    wd = padded(w, 16)
    deq = dev(d["deq_scale"])
    pts = dev(d["per_token_scale"])
    o = bq.bq_gemm_i8_pertoken(xd, wd, deq, pts, None if b is None else dev(b), w_layout=layout,
                               out_dtype=_TORCH_OUT[out])
    torch.cuda.synchronize()
    ref, ovf = oracle.gemm_i8_pertoken(d["x"], w, d["deq_scale"], d["per_token_scale"], b, layout=layout)
    assert ovf == 0
    scale = None
    if b is not None:
        scale = np.abs(ref - b.astype(np.float64)) + np.abs(b.astype(np.float64))
    assert_out(host(o), ref, _TORCH_OUT[out], f"gemm {M}x{N}x{K} layout {layout} {out}", scale=scale)


def test_gemm_atb_worked_example(golden_dir):
    import json
    import os
    with open(os.path.join(golden_dir, "atb_per_token_example.json")) as f:
        ex = json.load(f)
    x = np.array(ex["x"], np.int8)
    w = np.array(ex["weight"], np.int8)  # [k, n]
    for out in ("bf16", "f16", "f32"):
        o = bq.bq_gemm_i8_pertoken(padded(x, 16), padded(w, 16), dev(np.array(ex["deqScale"], np.float32)),
                                   dev(np.array(ex["perTokenScale"], np.float32)), w_layout=bq.BQ_W_KN,
                                   out_dtype=_TORCH_OUT[out])
        np.testing.assert_array_equal(host(o), np.array(ex["output"], np.float64))
        o = bq.bq_gemm_i8_pertoken(padded(x, 16), padded(np.ascontiguousarray(w.T), 16),
                                   dev(np.array(ex["deqScale"], np.float32)),
                                   dev(np.array(ex["perTokenScale"], np.float32)), w_layout=bq.BQ_W_NK,
                                   out_dtype=_TORCH_OUT[out])
        np.testing.assert_array_equal(host(o), np.array(ex["output"], np.float64))


@pytest.mark.parametrize("M,N,K,layout,out,bias", [
    (300, 520, 400, bq.BQ_W_NK, "bf16", False),
    (129, 257, 128, bq.BQ_W_NK, "f32", True),
    (200, 384, 264, bq.BQ_W_KN, "f16", False),
    (77, 200, 1000, bq.BQ_W_KN, "bf16", True),
    (1, 8, 16, bq.BQ_W_NK, "bf16", False),
    (513, 1030, 2048, bq.BQ_W_NK, "bf16", True),
    (260, 2100, 96, bq.BQ_W_NK, "f32", False),
    # more tiles than SMs with a short last wave: its tiles run as 128 x 128 halves
    (1024, 5000, 64, bq.BQ_W_NK, "bf16", True),
    (1100, 4400, 96, bq.BQ_W_KN, "f32", False),
    (2000, 2560, 48, bq.BQ_W_NK, "f16", False),
    # enough 256 x 256 tiles for a wave of CTA pairs (tcgen05 cta_group::2), with and without half tiles
    (2500, 4600, 64, bq.BQ_W_NK, "bf16", True),
    (1536, 4864, 48, bq.BQ_W_NK, "f32", False),
    (2048, 2560, 80, bq.BQ_W_NK, "f16", True),
])
def test_gemm_ragged(M, N, K, layout, out, bias):
    _gemm_case(M, N, K, layout, out, bias, seed=M + N + K)


def test_gemm_full_size_sampled_rows():
    d = synth.gemm_w8a8()
    o = bq.bq_gemm_i8_pertoken(dev(d["x"]), dev(d["w"]), dev(d["deq_scale"]), dev(d["per_token_scale"]))
    torch.cuda.synchronize()
    rows = np.sort(synth.rng(107).choice(4096, 48, replace=False))
    rows = np.concatenate([[0, 127, 128, 4095], rows])
    ref, _ = oracle.gemm_i8_pertoken(d["x"][rows], d["w"], d["deq_scale"], d["per_token_scale"][rows])
    assert_out(host(o)[rows], ref, torch.bfloat16, "gemm 4096^3 sampled rows")


def test_gemm_closed_form_all_ones():
    M, N, K = 200, 300, 1000
    x = np.ones((M, K), np.int8)
    w = np.ones((N, K), np.int8)
    o = bq.bq_gemm_i8_pertoken(padded(x, 16), padded(w, 16), dev(np.ones(N, np.float32)),
                               dev(np.ones(M, np.float32)), out_dtype=torch.float32)
    np.testing.assert_array_equal(host(o), np.full((M, N), float(K)))


# ------------------------------------------------------------- BitLinear

def _bitlinear_check(x_f32, x_dev, w_f32, N, out, bias, what, rows=None, path=None):
    """Runs the GPU pack + BitLinear, then checks the workspace codes and the
    output against the oracle computed from the same inputs (and, when given,
    which kernels the call ran)."""
    eps = 1e-5
    M, K = x_f32.shape
    wp, ws_ = bq.bq_weight_quant_ternary_pack(dev(w_f32))
    if path is not None:
        assert bq.bq_bitlinear_w2a8_path(x_dev, N) == path, what
    nbytes = bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K)
    work = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    b = None if bias is None else dev(bias)
    o = bq.bq_bitlinear_w2a8(x_dev, wp, ws_, N, b, eps, _TORCH_OUT[out], workspace=work)
    torch.cuda.synchronize()
    xo, so, _ = bq.bq_bitlinear_workspace_layout(M, K)
    g_xq = host(work[xo:xo + M * K].view(torch.int8).view(M, K))
    g_sc = host(work[so:so + 4 * M].view(torch.float32))
    sel = np.arange(M) if rows is None else rows
    ref, extra, scale, a, t = bitlinear_expected(x_f32, w_f32, bias, eps, rows=sel)
    assert_codes(g_xq[sel], a["xq"], a["pre"], what + " xq")
    np.testing.assert_allclose(g_sc[sel], a["act_scale"], rtol=1e-5)
    rel32 = bitlinear_rel32(g_sc[sel], a["act_scale"], host(ws_)[0], t["gamma"])
    assert_out(host(o)[sel], ref, _TORCH_OUT[out], what, extra=extra, scale=scale, rel32=rel32)


def test_bitlinear_tiny_config():
    d = synth.bitlinear_tiny(0)
    _bitlinear_check(d["x"], dev(d["x"]), d["w"], 128, "f32", None, "bitlinear tiny")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_bitlinear_decode_full_size(M):
    d = synth.bitlinear_decode(M)
    path = bq.BQ_PATH_DECODE_STREAM if M == 1 else bq.BQ_PATH_DECODE_MMA
    _bitlinear_check(d["x"], bf16_dev(d["x_bf16"]), d["w"], 11008, "bf16", None, f"decode M={M}", path=path)


# shapes the register-streaming kernels leave to the shared-memory decode
# kernel: one token with K < 2048 or more rows per CTA than the stream kernel
# keeps in flight, and 2..16 tokens with K % 512 == 0 but K not 2048 / 4096
@pytest.mark.parametrize("M,N,K,out,bias,xin", [(1, 300, 1024, "bf16", False, "bf16"),
                                                (1, 12800, 4096, "f32", True, "bf16"),
                                                (4, 1000, 8192, "bf16", True, "f32"),
                                                (2, 700, 1536, "f16", False, "bf16"),
                                                (16, 400, 8192, "bf16", False, "bf16"),
                                                (7, 900, 512, "f32", True, "f32")])
def test_bitlinear_decode_shared_memory_kernel(M, N, K, out, bias, xin):
    g = synth.rng((116, M, N, K))
    if xin == "bf16":
        bits, x = synth.bf16_activations(M, K, (116, M, K))
        x_dev = bf16_dev(bits)
    else:
        x = synth.normal_f32(g, (M, K))
        x_dev = dev(x)
    w = synth.normal_f32(g, (N, K), 0.02)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    _bitlinear_check(x, x_dev, w, N, out, b, f"decode smem {M}x{N}x{K} {xin}", path=bq.BQ_PATH_DECODE_SMEM)


@pytest.mark.parametrize("M,N,K,out,bias", [(3, 100, 48, "f16", True), (7, 64, 4096, "f32", False),
                                            (16, 72, 192, "bf16", True)])
def test_bitlinear_decode_ragged(M, N, K, out, bias):
    g = synth.rng((108, M, N, K))
    x = synth.normal_f32(g, (M, K))
    w = synth.normal_f32(g, (N, K), 0.02)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    path = bq.BQ_PATH_ACT_QUANT_GEMV if K % 512 else None
    _bitlinear_check(x, dev(x), w, N, out, b, f"decode ragged {M}x{N}x{K}", path=path)


# one token: dp4a register-streaming kernel (fp32 and bf16 inputs, K = 2048 / 8192,
# fewer rows than SMs); 2..4 tokens: the one-launch mma.sync kernel; 5..16
# tokens: the two-launch mma.sync kernel (K = 2048 / 4096, one or two token
# groups, up to 80 rows per CTA, fewer rows than SMs) and, past its row limit,
# the shared-memory kernel
@pytest.mark.parametrize("M,N,K,out,bias,xin", [(1, 300, 2048, "f32", True, "f32"), (1, 100, 4096, "f16", True, "bf16"),
                                                (1, 5000, 8192, "bf16", False, "bf16"),
                                                (2, 1000, 4096, "bf16", True, "bf16"),
                                                (1, 11008, 4096, "f32", False, "f32"),
                                                (5, 3000, 2048, "f16", True, "f32"), (12, 777, 4096, "f32", True, "bf16"),
                                                (9, 150, 2048, "bf16", False, "bf16"), (16, 11900, 4096, "bf16", True, "f32"),
                                                (16, 11008, 4096, "bf16", True, "f32"), (8, 4096, 4096, "f16", False, "f32"),
                                                (3, 40, 4096, "bf16", True, "bf16"), (16, 11840, 4096, "f32", False, "bf16"),
                                                (7, 8000, 2048, "bf16", True, "bf16"), (4, 3000, 2048, "f16", True, "f32"),
                                                (2, 11840, 4096, "bf16", False, "f32")])
def test_bitlinear_decode_stream_shapes(M, N, K, out, bias, xin):
    g = synth.rng((110, M, N, K))
    if xin == "bf16":
        bits, x = synth.bf16_activations(M, K, (110, M, K))
        x_dev = bf16_dev(bits)
    else:
        x = synth.normal_f32(g, (M, K))
        x_dev = dev(x)
    w = synth.normal_f32(g, (N, K), 0.02)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    _bitlinear_check(x, x_dev, w, N, out, b, f"decode stream {M}x{N}x{K} {xin}")


@pytest.mark.parametrize("M,N,K,out,bias", [(17, 256, 128, "bf16", False), (300, 520, 512, "bf16", True),
                                            (129, 264, 640, "f32", False), (200, 1000, 1024, "f16", True),
                                            # CTA-pair path, with and without half tiles in the last wave
                                            (2500, 4600, 128, "bf16", True), (1536, 4864, 256, "f32", False)])
def test_bitlinear_prefill_ragged(M, N, K, out, bias):
    g = synth.rng((109, M, N, K))
    bits, xf = synth.bf16_activations(M, K, (109, M), outlier_frac=0.01)
    w = synth.normal_f32(g, (N, K), 0.02)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    _bitlinear_check(xf, bf16_dev(bits), w, N, out, b, f"prefill ragged {M}x{N}x{K}")


# more than 16 tokens with K % 64 != 0 (packed rows re-pitched in the
# workspace) and / or N * size % 16 != 0 (output rows staged in the workspace)
@pytest.mark.parametrize("M,N,K,out,bias", [(300, 61, 144, "f16", False), (257, 1001, 528, "bf16", True),
                                            (17, 9, 16, "bf16", False), (40, 77, 80, "f32", True),
                                            (130, 300, 1040, "bf16", False), (2500, 4601, 144, "f16", True)])
def test_bitlinear_prefill_unaligned_tails(M, N, K, out, bias):
    g = synth.rng((117, M, N, K))
    bits, xf = synth.bf16_activations(M, K, (117, M), outlier_frac=0.01)
    w = synth.normal_f32(g, (N, K), 0.02)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    x_dev = bf16_dev(bits)
    path = bq.BQ_PATH_TC_PAIR if (M >= 2048 and N >= 4096) else bq.BQ_PATH_TC_SINGLE
    _bitlinear_check(xf, x_dev, w, N, out, b, f"prefill tails {M}x{N}x{K}", path=path)


def test_bitlinear_prefill_full_size_sampled_rows():
    d = synth.bitlinear_prefill()
    rows = np.sort(np.concatenate([[0, 1, 127, 128, 8191], synth.rng(110).choice(8192, 27, replace=False)]))
    rows = np.unique(rows)
    _bitlinear_check(d["x"], bf16_dev(d["x_bf16"]), d["w"], 4096, "bf16", None, "prefill 8192x4096x4096",
                     rows=rows)


# ------------------------------------------------------------- INT4 linear

def _w4_check(M, N, K, gs, seed, rows=None, full=None):
    if full is None:
        g = synth.rng(seed)
        q = synth.nibbles(g, (N, K))
        z = synth.nibbles(g, (N, K // gs))
        s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
        b = synth.normal_f32(g, (N,), 0.01)
        x = synth.normal_f32(g, (M, K))
    else:
        q, z, s, b, x = full
    qw, qz = bq.bq_weight_pack_int4_grouped(dev(q), dev(z), gs)
    o = bq.bq_linear_w4_grouped(dev(x), qw, dev(s.view(np.int16)), qz, gs, None if b is None else dev(b))
    torch.cuda.synchronize()
    sel = np.arange(M) if rows is None else rows
    ref = oracle.linear_w4_grouped(x[sel], oracle.int4_pack(q), s.view(np.uint16), oracle.int4_pack(z), b, gs)
    tol = 1e-4 * math.sqrt(K / 128)
    err = np.abs(host(o)[sel] - ref)
    assert err.max() <= tol, f"INT4 {M}x{N}x{K} g{gs}: max |err| {err.max():.3e} > {tol:.3e}"
    return err.max()


@pytest.mark.parametrize("M,N,K,gs", [(3, 100, 384, 64), (5, 33, 200, 8), (2, 7, 96, 96), (6, 300, 1024, 128),
                                      (1, 64, 64, 32), (9, 129, 512, 256)])
def test_linear_w4_ragged(M, N, K, gs):
    _w4_check(M, N, K, gs, seed=(111, M, N, K))


# one token: the single-launch TMA-fed mma.sync kernel (K = 2048 .. 8192,
# groups of 128 / 256, more 8-row boxes than SMs and fewer, row counts that
# end inside a box, with and without bias), and shapes it leaves to the
# general path (groups of 32 / 64, K = 1024)
@pytest.mark.parametrize("N,K,gs,bias", [(300, 2048, 64, True), (5000, 8192, 256, True), (100, 1024, 32, False),
                                         (900, 2048, 128, True), (3000, 8192, 128, False),
                                         (16000, 4096, 128, True), (7, 4096, 128, False),
                                         (14336, 4096, 128, True), (1001, 4096, 256, False),
                                         (2301, 2048, 128, False)])
def test_linear_w4_one_token(N, K, gs, bias):
    g = synth.rng((113, N, K, gs))
    q = synth.nibbles(g, (N, K))
    z = synth.nibbles(g, (N, K // gs))
    s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
    b = synth.normal_f32(g, (N,), 0.01) if bias else None
    x = synth.normal_f32(g, (1, K))
    _w4_check(1, N, K, gs, None, full=(q, z, s, b, x))


# 2..32 tokens: the tensor-core path (planes prologue, tcgen05 kind::i8 with
# the codes minus the zero-point expanded in shared memory, K-slice reduction)
@pytest.mark.parametrize("M,N,K,gs,bias", [(2, 1000, 2048, 128, True), (32, 3000, 4096, 256, True),
                                           (31, 640, 8192, 128, False), (4, 130, 1024, 128, True)])
def test_linear_w4_tensor_core(M, N, K, gs, bias):
    g = synth.rng((114, M, N, K, gs))
    q = synth.nibbles(g, (N, K))
    z = synth.nibbles(g, (N, K // gs))
    s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
    b = synth.normal_f32(g, (N,), 0.01) if bias else None
    x = synth.normal_f32(g, (M, K))
    _w4_check(M, N, K, gs, None, full=(q, z, s, b, x))


def test_linear_w4_tensor_core_zero_point_equals_code_gives_bias():
    g = synth.rng(115)
    N, K, gs = 200, 1024, 128
    z = synth.nibbles(g, (N, K // gs))
    q = np.repeat(z, gs, axis=1)
    s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
    b = synth.normal_f32(g, (N,), 0.01)
    x = synth.normal_f32(g, (8, K))
    _w4_check(8, N, K, gs, None, full=(q, z, s, b, x))


@pytest.mark.parametrize("M", [1, 32])
def test_linear_w4_full_size(M):
    w = synth.linear_w4_weights()
    x = synth.linear_w4_activations(M)
    rows = None if M == 1 else np.array([0, 5, 17, 31])
    _w4_check(M, 14336, 4096, 128, None, rows=rows,
              full=(w["q"], w["zeros"], w["scales_f16"], w["bias"], x))


def test_linear_w4_zero_point_equals_code_gives_bias():
    g = synth.rng(112)
    N, K, gs = 40, 256, 64
    z = synth.nibbles(g, (N, K // gs))
    q = np.repeat(z, gs, axis=1)
    s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
    b = synth.normal_f32(g, (N,), 0.01)
    x = synth.normal_f32(g, (3, K))
    _w4_check(3, N, K, gs, None, full=(q, z, s, b, x))


# ------------------------------------------------- batched / transposed W8A8

def _dev3(a: np.ndarray, align_elems: int = 16):
    """Device copy of a [B, R, C] array with rows padded to align_elems (the
    batch stride is R * padded row), sliced back to [B, R, C]."""
    B, R, C = a.shape
    ld = (C + align_elems - 1) // align_elems * align_elems
    buf = np.zeros((B, R, ld), a.dtype)
    buf[:, :, :C] = a
    return dev(buf)[:, :, :C]


def test_gemm_batched_atb_example(golden_dir):
    import json
    import os
    with open(os.path.join(golden_dir, "atb_per_token_example.json")) as f:
        ex = json.load(f)
    x = np.array(ex["x"], np.int8)
    w = np.array(ex["weight"], np.int8)  # [k, n]
    want = np.stack([np.array(ex["output"], np.float64)] * 3)
    deq = dev(np.array(ex["deqScale"], np.float32))
    pts = dev(np.array(ex["perTokenScale"], np.float32))
    for trans in (False, True):
        xs = np.stack([x.T if trans else x] * 3)
        for layout, ws in ((bq.BQ_W_KN, np.stack([w] * 3)), (bq.BQ_W_NK, np.stack([w.T] * 3))):
            for out in ("bf16", "f16", "f32"):
                o = bq.bq_gemm_i8_pertoken_batched(_dev3(np.ascontiguousarray(xs)), _dev3(np.ascontiguousarray(ws)),
                                                   deq, pts, w_layout=layout, trans_a=trans,
                                                   out_dtype=_TORCH_OUT[out])
                np.testing.assert_array_equal(host(o), want, err_msg=f"trans {trans} layout {layout} {out}")


@pytest.mark.parametrize("B,M,N,K,layout,trans,out,bias,shared", [
    (3, 200, 300, 160, bq.BQ_W_NK, False, "bf16", False, True),
    (2, 129, 257, 96, bq.BQ_W_KN, False, "f32", True, False),
    (1, 300, 520, 400, bq.BQ_W_NK, True, "bf16", True, True),
    (4, 130, 200, 64, bq.BQ_W_KN, True, "f16", False, False),
    (2, 257, 384, 1000, bq.BQ_W_NK, True, "f32", False, True),
    # enough 256 x 256 tiles over the batches for CTA pairs
    (4, 1024, 2048, 128, bq.BQ_W_NK, False, "bf16", True, False),
    (6, 700, 1300, 48, bq.BQ_W_NK, False, "f16", False, True),
])
def test_gemm_batched_ragged(B, M, N, K, layout, trans, out, bias, shared):
    g = synth.rng((118, B, M, N, K))
    x = synth.int8_uniform(g, (B, M, K))
    w = synth.int8_uniform(g, (B, N, K))
    deq = synth.uniform_f32(g, (N,) if shared else (B, N), 0.001, 0.01)
    pts = synth.uniform_f32(g, (M,) if shared else (B, M), 0.001, 0.01)
    b = synth.normal_f32(g, (N,), 0.5) if bias else None
    xs = np.ascontiguousarray(x.transpose(0, 2, 1)) if trans else x
    ws = w if layout == bq.BQ_W_NK else np.ascontiguousarray(w.transpose(0, 2, 1))
    deq_d = dev(deq) if shared else _dev3(deq[:, None, :], 8)[:, 0, :]
    o = bq.bq_gemm_i8_pertoken_batched(_dev3(xs), _dev3(ws), deq_d, dev(pts), None if b is None else dev(b),
                                       w_layout=layout, trans_a=trans, out_dtype=_TORCH_OUT[out])
    torch.cuda.synchronize()
    ref, ovf = oracle.gemm_i8_pertoken_batched(xs, ws, deq, pts, b, layout=layout, trans_a=trans,
                                               shared_scales=shared)
    assert ovf == 0
    scale = None
    if b is not None:
        scale = np.abs(ref - b.astype(np.float64)) + np.abs(b.astype(np.float64))
    assert_out(host(o), ref, _TORCH_OUT[out], f"batched {B}x{M}x{N}x{K} layout {layout} trans {trans} {out}",
               scale=scale)


def test_gemm_transposed_a_full_size_sampled_rows():
    # the 4096^3 workload with x stored [K, M] (transposeA)
    d = synth.gemm_w8a8()
    xt = np.ascontiguousarray(d["x"].T)
    o = bq.bq_gemm_i8_pertoken_batched(dev(xt)[None], dev(d["w"])[None], dev(d["deq_scale"]),
                                       dev(d["per_token_scale"]), trans_a=True)
    torch.cuda.synchronize()
    rows = np.sort(np.concatenate([[0, 127, 128, 4095], synth.rng(119).choice(4096, 28, replace=False)]))
    ref, _ = oracle.gemm_i8_pertoken(d["x"][rows], d["w"], d["deq_scale"], d["per_token_scale"][rows])
    assert_out(host(o)[0][rows], ref, torch.bfloat16, "gemm 4096^3 transposeA sampled rows")


# ---------------------------------------------------- LayerNorm normaliser

def _ln_params(g, K, affine):
    if not affine:
        return None, None
    return (1.0 + 0.2 * g.standard_normal(K)).astype(np.float32), (0.1 * g.standard_normal(K)).astype(np.float32)


@pytest.mark.parametrize("M,K,dtype,affine", [(8, 256, "f32", False), (37, 1000, "bf16", True),
                                              (300, 4096, "bf16", True), (5, 4096, "f32", False),
                                              (1, 7, "f32", True), (2000, 512, "bf16", False)])
def test_act_quant_layernorm(M, K, dtype, affine):
    g = synth.rng((121, M, K))
    x = synth.normal_f32(g, (M, K)) + np.float32(0.75)  # a nonzero mean for the LayerNorm to remove
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(x)
        x = synth.bf16_bits_to_f32(bits)
        xd = bf16_dev(bits)
    else:
        xd = dev(x)
    lw, lb = _ln_params(g, K, affine)
    xq, sc, rs = bq.bq_act_quant_int8_layernorm(xd, 1e-5, None if lw is None else dev(lw),
                                                None if lb is None else dev(lb))
    torch.cuda.synchronize()
    ref = oracle.act_quant_layernorm(x, 1e-5, lw, lb, want_pre=True)
    g_xq = host(xq)
    assert_codes(g_xq, ref["xq"], ref["pre"], f"layernorm quant {M}x{K} {dtype}")
    np.testing.assert_allclose(host(sc), ref["act_scale"], rtol=1e-5)
    np.testing.assert_array_equal(host(rs), g_xq.astype(np.int64).sum(axis=1))


@pytest.mark.parametrize("affine", [False, True])
def test_act_quant_layernorm_degenerate_rows_many(affine):
    # sixteen rows (the warp-per-row kernel): rows whose mean is far from zero relative to their
    # spread take its binary64 passes, ordinary rows its fp32 passes; all are compared alike
    M, K = 16, 512
    g = synth.rng((123, affine))
    x = synth.normal_f32(g, (M, K))
    x[0] = 1e5                                                       # constant, large
    x[1] = 3.0                                                       # constant, small
    x[2] = np.float32(1e4) + np.float32(1e-3) * synth.normal_f32(g, (K,))  # tiny spread, large offset
    x[3] = np.float32(-250.0) + synth.normal_f32(g, (K,))            # offset 250 sigma
    x[4] = 0.0
    x[4, 9] = -7.0                                                   # one-hot
    x[5, ::7] = np.float32(1e-40)                                    # subnormal and zero elements
    x[5, 3::11] = 0.0
    lw, lb = _ln_params(g, K, affine)
    xq, sc, rs = bq.bq_act_quant_int8_layernorm(dev(x), 1e-5, None if lw is None else dev(lw),
                                                None if lb is None else dev(lb))
    torch.cuda.synchronize()
    ref = oracle.act_quant_layernorm(x, 1e-5, lw, lb, want_pre=True)
    assert_codes(host(xq), ref["xq"], ref["pre"], f"layernorm degenerate rows affine={affine}")
    np.testing.assert_allclose(host(sc), ref["act_scale"], rtol=1e-5)
    np.testing.assert_array_equal(host(rs), host(xq).astype(np.int64).sum(axis=1))
    if not affine:
        assert np.all(host(xq)[0] == 0) and np.all(host(xq)[1] == 0)


def test_act_quant_layernorm_special_rows():
    K = 512
    x = synth.normal_f32(synth.rng(122), (4, K))
    x[0] = 3.0                   # constant row: zero after the mean is removed
    x[1] = 0.0
    x[1, 7] = 5.0                # one-hot row
    x[2] += np.float32(1000.0)   # large common offset
    xq, sc, _ = bq.bq_act_quant_int8_layernorm(dev(x), 1e-5)
    torch.cuda.synchronize()
    ref = oracle.act_quant_layernorm(x, 1e-5, want_pre=True)
    assert_codes(host(xq), ref["xq"], ref["pre"], "layernorm special rows")
    np.testing.assert_allclose(host(sc), ref["act_scale"], rtol=1e-5)
    assert np.all(host(xq)[0] == 0)


@pytest.mark.parametrize("M,N,K,out,bias,affine", [(4, 11008, 4096, "bf16", False, False),
                                                   (16, 300, 2048, "f32", True, True),
                                                   (300, 520, 512, "bf16", True, True),
                                                   (300, 61, 144, "f16", False, True),
                                                   (2048, 4096, 256, "bf16", False, False),
                                                   (1, 11008, 4096, "bf16", True, True),     # one token: fused
                                                   (1, 300, 2048, "f32", False, False),
                                                   (1, 5000, 8192, "bf16", False, True)])
def test_bitlinear_layernorm(M, N, K, out, bias, affine):
    g = synth.rng((123, M, N, K))
    bits, xf = synth.bf16_activations(M, K, (123, M, K), outlier_frac=0.01)
    w = synth.normal_f32(g, (N, K), 0.02)
    b = synth.normal_f32(g, (N,), 0.1) if bias else None
    lw, lb = _ln_params(g, K, affine)
    wp, ws_ = bq.bq_weight_quant_ternary_pack(dev(w))
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, M, N, K), dtype=torch.uint8, device="cuda")
    o = bq.bq_bitlinear_w2a8_layernorm(bf16_dev(bits), wp, ws_, N, None if lw is None else dev(lw),
                                       None if lb is None else dev(lb), None if b is None else dev(b), 1e-5,
                                       _TORCH_OUT[out], workspace=work)
    torch.cuda.synchronize()
    xo, so, _ = bq.bq_bitlinear_workspace_layout(M, K)
    g_xq = host(work[xo:xo + M * K].view(torch.int8).view(M, K))
    g_sc = host(work[so:so + 4 * M].view(torch.float32))
    what = f"bitlinear layernorm {M}x{N}x{K}"
    ref, extra, scale, a, t = bitlinear_expected(xf, w, b, 1e-5, ln=(lw, lb))
    assert_codes(g_xq, a["xq"], a["pre"], what + " xq")
    rel32 = bitlinear_rel32(g_sc, a["act_scale"], host(ws_)[0], t["gamma"])
    assert_out(host(o), ref, _TORCH_OUT[out], what, extra=extra, scale=scale, rel32=rel32)


@pytest.mark.parametrize("row,affine", [("constant", False), ("constant", True), ("offset", True), ("tiny", False)])
def test_bitlinear_layernorm_one_token_degenerate(row, affine):
    # one token through the fused kernel: a constant row far from zero and a tiny spread on a large
    # offset take its binary64 passes, a 250-sigma offset its fp32 ones
    N, K = 2000, 4096
    g = synth.rng((125, ["constant", "offset", "tiny"].index(row), int(affine)))
    xf = synth.normal_f32(g, (1, K))
    if row == "constant":
        xf[:] = 1e5
    elif row == "offset":
        xf += np.float32(250.0)
    else:
        xf = np.float32(1e4) + np.float32(1e-2) * xf
    bits = synth.f32_to_bf16_bits(xf)
    xf = synth.bf16_bits_to_f32(bits)
    w = synth.normal_f32(g, (N, K), 0.02)
    lw, lb = _ln_params(g, K, affine)
    wp, ws_ = bq.bq_weight_quant_ternary_pack(dev(w))
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_BITLINEAR_W2A8, 1, N, K), dtype=torch.uint8, device="cuda")
    o = bq.bq_bitlinear_w2a8_layernorm(bf16_dev(bits), wp, ws_, N, None if lw is None else dev(lw),
                                       None if lb is None else dev(lb), None, 1e-5, torch.float32, workspace=work)
    torch.cuda.synchronize()
    xo, so, _ = bq.bq_bitlinear_workspace_layout(1, K)
    g_xq = host(work[xo:xo + K].view(torch.int8).view(1, K))
    g_sc = host(work[so:so + 4].view(torch.float32))
    what = f"bitlinear layernorm one token {row} affine={affine}"
    ref, extra, scale, a, t = bitlinear_expected(xf, w, None, 1e-5, ln=(lw, lb))
    assert_codes(g_xq, a["xq"], a["pre"], what + " xq")
    np.testing.assert_allclose(g_sc, a["act_scale"], rtol=1e-5)
    rel32 = bitlinear_rel32(g_sc, a["act_scale"], host(ws_)[0], t["gamma"])
    assert_out(host(o), ref, torch.float32, what, extra=extra, scale=scale, rel32=rel32)


# ------------------------------------------------------- W4A4 (Q4Linear)

def _q4_inputs(M, N, K, seed, per_channel, xin):
    g = synth.rng((124, seed))
    x = synth.normal_f32(g, (M, K))
    if xin == "bf16":
        bits = synth.f32_to_bf16_bits(x)
        x = synth.bf16_bits_to_f32(bits)
        xd = bf16_dev(bits)
    else:
        xd = dev(x)
    w = synth.normal_f32(g, (N, K), 0.02)
    # steps: about a quarter of a standard deviation for x, max|w_n| / 7.5 per weight row
    sa = np.array([0.27], np.float32)
    sw = (np.abs(w).max(axis=1) / 7.5).astype(np.float32) if per_channel else np.array([0.006], np.float32)
    return x, xd, w, sa, sw


def _q4_band_extra(xq, x_pre, wq, w_pre, sa, sw_n, eps):
    xband = tie_band(x_pre).astype(np.float64)
    wband = tie_band(w_pre).astype(np.float64)
    s_a = max(float(sa[0]), eps)
    s_w = np.maximum(sw_n.astype(np.float64), eps)
    return (xband @ np.abs(wq).T.astype(np.float64) + np.abs(xq).astype(np.float64) @ wband.T) * s_a * s_w[None, :]


@pytest.mark.parametrize("N,K,per_channel,win", [(300, 256, True, "f32"), (64, 4096, False, "bf16"), (7, 8, True, "f32")])
def test_q4_weight_pack(N, K, per_channel, win):
    _, _, w, _, sw = _q4_inputs(1, N, K, (N, K), per_channel, "f32")
    eps = 1e-6
    if win == "bf16":
        bits = synth.f32_to_bf16_bits(w)
        w = synth.bf16_bits_to_f32(bits)
        wd = bf16_dev(bits)
    else:
        wd = dev(w)
    wp = bq.bq_weight_quant_int4_pack(wd, dev(sw), eps)
    torch.cuda.synchronize()
    wq, pre = oracle.q4_quant(w, sw, eps, per_row=per_channel, want_pre=True)
    u = oracle.int4_unpack(host(wp).view(np.uint32), K).astype(np.int16)
    codes = np.where(u >= 8, u - 16, u)
    assert_codes(codes, wq, pre, f"q4 pack {N}x{K}")
    if not tie_band(pre).any():
        np.testing.assert_array_equal(host(wp).view(np.uint32), oracle.s4_pack(wq))


@pytest.mark.parametrize("M,N,K,per_channel,bias,out,xin", [
    (1, 11008, 4096, True, False, "bf16", "bf16"),
    (5, 300, 1024, False, True, "f32", "f32"),
    (16, 1000, 2048, True, True, "f16", "bf16"),
    (17, 257, 256, True, False, "bf16", "f32"),
    (300, 61, 512, False, True, "f16", "bf16"),
    (300, 520, 1024, True, True, "bf16", "bf16"),
    (2500, 4608, 256, True, False, "bf16", "bf16"),  # CTA pairs
])
def test_linear_w4a4(M, N, K, per_channel, bias, out, xin):
    eps = 1e-6
    x, xd, w, sa, sw = _q4_inputs(M, N, K, (M, N, K), per_channel, xin)
    b = synth.normal_f32(synth.rng((125, N)), (N,), 0.1) if bias else None
    wp = bq.bq_weight_quant_int4_pack(dev(w), dev(sw), eps)
    work = torch.empty(bq.bq_workspace_bytes(bq.BQ_OP_LINEAR_W4A4, M, N, K), dtype=torch.uint8, device="cuda")
    o = bq.bq_linear_w4a4(xd, dev(sa), wp, dev(sw), N, eps, None if b is None else dev(b), _TORCH_OUT[out],
                          workspace=work)
    torch.cuda.synchronize()
    xq, x_pre = oracle.q4_quant(x, sa, eps, want_pre=True)
    wq, w_pre = oracle.q4_quant(w, sw, eps, per_row=per_channel, want_pre=True)
    assert_codes(host(work[:M * K].view(torch.int8).view(M, K)), xq, x_pre, f"w4a4 act codes {M}x{K}")
    ref = oracle.linear_w4a4_from_codes(xq, wq, sa, sw, eps, b, per_channel=per_channel)
    sw_n = sw if per_channel else np.full(N, sw[0], np.float32)
    extra = _q4_band_extra(xq, x_pre, wq, w_pre, sa, sw_n, eps)
    scale = None
    if b is not None:
        scale = np.abs(ref - b.astype(np.float64)) + np.abs(b.astype(np.float64))
    assert_out(host(o), ref, _TORCH_OUT[out], f"w4a4 {M}x{N}x{K}", extra=extra, scale=scale)


# -------------------------------------------------------------- BitConv1d

@pytest.mark.parametrize("B,C_in,L,C_out,KS,stride,pad,groups,xin,out,bias,affine", [
    (2, 64, 37, 48, 3, 1, 1, 1, "bf16", "bf16", True, True),
    (1, 128, 100, 96, 4, 2, 0, 2, "f32", "f32", False, False),
    (3, 32, 9, 8, 5, 1, 2, 1, "f32", "f16", True, False),
    (2, 80, 20, 40, 3, 1, 1, 1, "bf16", "bf16", False, True),       # channels re-pitched to 128
    (4, 512, 256, 512, 3, 1, 1, 1, "bf16", "bf16", True, False),     # several GEMM tiles per tap
    (2, 256, 64, 64, 1, 1, 0, 4, "bf16", "f32", False, True),
    (2, 128, 50, 64, 3, 1, 1, 2, "bf16", "bf16", True, True),       # groups with padding at stride 1
    (1, 64, 5, 32, 7, 1, 3, 1, "f32", "f32", False, False),          # padding wide against L
    (2, 32, 4, 16, 6, 1, 1, 1, "f32", "bf16", False, False),         # one output position
])
def test_bitconv1d(B, C_in, L, C_out, KS, stride, pad, groups, xin, out, bias, affine):
    g = synth.rng((126, B, C_in, L, C_out, KS))
    x = synth.normal_f32(g, (B, C_in, L)) + np.float32(0.3)
    if xin == "bf16":
        bits = synth.f32_to_bf16_bits(x)
        x = synth.bf16_bits_to_f32(bits)
        xd = bf16_dev(bits)
    else:
        xd = dev(x)
    w = synth.normal_f32(g, (C_out, C_in // groups, KS), 0.02)
    b = synth.normal_f32(g, (C_out,), 0.1) if bias else None
    lw, lb = _ln_params(g, C_in, affine)
    wp, ws_ = bq.bq_bitconv1d_weight_pack(dev(w))
    o = bq.bq_bitconv1d(xd, wp, ws_, C_out, KS, stride, pad, groups, None if lw is None else dev(lw),
                        None if lb is None else dev(lb), None if b is None else dev(b), 1e-5, _TORCH_OUT[out])
    torch.cuda.synchronize()
    a = oracle.bitconv1d_act_quant(x, 1e-5, lw, lb, want_pre=True)
    t = oracle.ternary_quant(w.reshape(C_out, -1), want_pre=True)
    assert float(host(ws_)[0]) == pytest.approx(t["gamma"], rel=1e-6)
    wq = t["wq"].reshape(w.shape)
    conv = lambda xc, wc, bb=None: oracle.bitconv1d_from_codes(xc, a["act_scale"], wc, t["gamma"], B, L, stride, pad,
                                                               groups, bb)
    ref = conv(a["xq"], wq, b)
    # term magnitude and tie-band widening, from the oracle's conv of absolute codes / band indicators
    absx, absw = np.abs(a["xq"].astype(np.int16)).astype(np.int8), np.abs(wq)
    mag = conv(absx, absw)
    extra = conv(tie_band(a["pre"]).astype(np.int8), absw) + \
        conv(absx, tie_band(t["pre"]).reshape(w.shape).astype(np.int8))
    if b is not None:
        mag = mag + np.abs(b.astype(np.float64))[None, :, None]
    rel32 = (KS + 7) * 2.0 ** -24  # fp32 tap products and tap sum (scales are binary64 rounded once)
    assert_out(host(o), ref, _TORCH_OUT[out], f"bitconv1d {B}x{C_in}x{L} -> {C_out} k{KS} s{stride} p{pad} g{groups}",
               extra=extra, scale=mag, rel32=rel32)


# ------------------------------------------------- BitLinear STE backward

@pytest.mark.parametrize("M,N,K,xin", [(8, 128, 256, "f32"), (300, 520, 1024, "bf16"), (129, 264, 640, "f32"),
                                       (1024, 2048, 512, "bf16"), (2, 64, 64, "bf16")])
def test_bitlinear_backward(M, N, K, xin):
    u = 2.0 ** -24
    g = synth.rng((127, M, N, K))
    if xin == "bf16":
        bits, x = synth.bf16_activations(M, K, (127, M, K), outlier_frac=0.01)
        xd = bf16_dev(bits)
    else:
        x = synth.normal_f32(g, (M, K))
        xd = dev(x)
    w = synth.normal_f32(g, (N, K), 0.02)
    dbits = synth.f32_to_bf16_bits(synth.normal_f32(g, (M, N)))
    dout = synth.bf16_bits_to_f32(dbits)
    wp, ws_ = bq.bq_weight_quant_ternary_pack(dev(w))
    dx, dw = bq.bq_bitlinear_w2a8_backward(xd, bf16_dev(dbits), wp, ws_, 1e-5)
    torch.cuda.synchronize()
    rdx, rdw = oracle.bitlinear_backward(x, w, dout, 1e-5)
    a = oracle.act_quant(x, 1e-5, want_pre=True, want_y=True)
    t = oracle.ternary_quant(w, want_pre=True)
    s, gam = a["act_scale"], t["gamma"]
    ad = np.abs(dout.astype(np.float64))
    # dw: hi + lo split of dout * s (2^-16 relative), fp32 accumulation over 2M terms
    mag_dw = ad.T @ (np.abs(a["xq"]).astype(np.float64) * s[:, None])
    ex_dw = ad.T @ (tie_band(a["pre"]).astype(np.float64) * s[:, None])
    tol_dw = (2.0 ** -16 + (2 * M + 2) * u) * (mag_dw + ex_dw) + ex_dw + 1e-30
    err = np.abs(host(dw).astype(np.float64) - rdw)
    assert (err <= tol_dw).all(), f"dw {M}x{N}x{K}: worst {float((err - tol_dw).max()):.3e} over"
    # dx: dy exact products, fp32 accumulation over N terms and the gamma scale,
    # then the RMSNorm backward (binary64 reductions, one fp32 rounding)
    mag_dy = gam * (ad @ np.abs(t["wq"]).astype(np.float64))
    ex_dy = gam * (ad @ tie_band(t["pre"]).astype(np.float64))
    tol_dy = (N + 2) * u * (mag_dy + ex_dy) + ex_dy
    y = a["y"]
    r = np.sqrt((x.astype(np.float64) ** 2).mean(axis=1) + 1e-5)[:, None]
    tol_dx = (tol_dy + np.abs(y) * (tol_dy * np.abs(y)).mean(axis=1, keepdims=True)) / r + 2 * u * np.abs(rdx) + 1e-30
    err = np.abs(host(dx).astype(np.float64) - rdx)
    assert (err <= tol_dx).all(), f"dx {M}x{N}x{K}: worst {float((err - tol_dx).max()):.3e} over"


# ------------------------------------------------- W4A4 straight-through backward

def _range_band(pre):
    """Quotients within TIE_REL (relative) of the clamp-range ends -8 and 7."""
    return (np.abs(pre + 8.0) <= 8e-6) | (np.abs(pre - 7.0) <= 7e-6)


@pytest.mark.parametrize("M,N,K,xin,per_channel", [(8, 64, 128, "f32", False), (300, 520, 1024, "bf16", True),
                                                   (129, 264, 640, "f32", True), (1024, 2048, 512, "bf16", False),
                                                   (2, 8, 64, "bf16", True)])
def test_w4a4_backward(M, N, K, xin, per_channel):
    u = 2.0 ** -24
    eps = 1e-6
    g = synth.rng((131, M, N, K))
    x = synth.normal_f32(g, (M, K))
    if xin == "bf16":
        bits = synth.f32_to_bf16_bits(x)
        x = synth.bf16_bits_to_f32(bits)
        xd = bf16_dev(bits)
    else:
        xd = dev(x)
    w = synth.normal_f32(g, (N, K), 0.02)
    # steps that leave some quotients outside [-8, 7] on both operands
    sa = np.array([0.15], np.float32)
    sw = (np.abs(w).max(axis=1) / 9.0).astype(np.float32) if per_channel else np.array([0.003], np.float32)
    dbits = synth.f32_to_bf16_bits(synth.normal_f32(g, (M, N)))
    dout = synth.bf16_bits_to_f32(dbits)
    dx, dw, ds = bq.bq_linear_w4a4_backward(xd, dev(w), bf16_dev(dbits), dev(sa), dev(sw), eps)
    torch.cuda.synchronize()
    r = oracle.linear_w4a4_backward(x, w, dout, sa, sw, eps, per_channel=per_channel)
    xq, xpre = oracle.q4_quant(x, sa, eps, want_pre=True)
    wq, wpre = oracle.q4_quant(w, sw, eps, per_row=per_channel, want_pre=True)
    s_a = float(sa[0])
    s_w = sw.astype(np.float64) if per_channel else np.full(N, float(sw[0]))
    ad = np.abs(dout.astype(np.float64))
    # g: exact products accumulated in fp32 over N terms (per-channel steps: hi + lo parts, 2^-16)
    mag_g = ad @ (np.abs(wq).astype(np.float64) * s_w[:, None])
    ex_g = ad @ (tie_band(wpre).astype(np.float64) * s_w[:, None])
    rel_g = (2.0 ** -16 + (2 * N + 2) * u) if per_channel else (N + 2) * u
    tol_g = rel_g * (mag_g + ex_g) + ex_g
    xin_band = _range_band(xpre)
    tol_dx = tol_g + np.where(xin_band, np.abs(r["g"]) + tol_g, 0.0) + 1e-30
    err = np.abs(host(dx).astype(np.float64) - r["dx"])
    assert (err <= tol_dx).all(), f"dx {M}x{N}x{K}: worst {float((err - tol_dx).max()):.3e} over"
    # dw: exact products accumulated in fp32 over M terms, then the step
    mag_dw = s_a * (ad.T @ np.abs(xq).astype(np.float64))
    ex_dw = s_a * (ad.T @ tie_band(xpre).astype(np.float64))
    tol_dw = (M + 2) * u * (mag_dw + ex_dw) + ex_dw
    tol_dw = tol_dw + np.where(_range_band(wpre), np.abs(r["dw"]) + tol_dw, 0.0) + 1e-30
    err = np.abs(host(dw).astype(np.float64) - r["dw"])
    assert (err <= tol_dw).all(), f"dw {M}x{N}x{K}: worst {float((err - tol_dw).max()):.3e} over"
    # dscale_a: g's error times |term|, the fp32 quotient (2^-24 |u|) and code or mask flips times |g|
    inside = (xpre >= -8) & (xpre <= 7)
    term = np.where(inside, xq - xpre, xq.astype(np.float64))
    ag = np.abs(r["g"])
    tol_ds = float((tol_g * np.abs(term)).sum() + (ag * (u * np.abs(xpre) + tie_band(xpre) + 8.0 * xin_band)).sum()
                   + u * abs(r["dscale_a"]) + 1e-30)
    got = float(host(ds)[0])
    assert abs(got - r["dscale_a"]) <= tol_ds + 2 * u * abs(r["dscale_a"]), (got, r["dscale_a"], tol_ds)
    assert (~inside).any() and inside.any()  # both sides of the range were exercised


def test_w4a4_backward_scale_below_eps_and_empty():
    g = synth.rng(133)
    M, N, K = 16, 32, 64
    x = synth.normal_f32(g, (M, K))
    w = synth.normal_f32(g, (N, K), 0.02)
    dbits = synth.f32_to_bf16_bits(synth.normal_f32(g, (M, N)))
    sa, sw = np.array([1e-9], np.float32), np.array([0.003], np.float32)
    dx, dw, ds = bq.bq_linear_w4a4_backward(dev(x), dev(w), bf16_dev(dbits), dev(sa), dev(sw), 1e-6)
    torch.cuda.synchronize()
    r = oracle.linear_w4a4_backward(x, w, synth.bf16_bits_to_f32(dbits), sa, sw, 1e-6)
    assert float(host(ds)[0]) == 0.0 and r["dscale_a"] == 0.0
    np.testing.assert_array_equal(host(dx), r["dx"].astype(np.float32))  # every quotient is outside: all zero
    # empty shapes write zero gradients
    dx0 = torch.full((M, K), 7.0, device="cuda")
    ds0 = torch.full((1,), 7.0, device="cuda")
    bq.bq_linear_w4a4_backward(dev(x), dev(w[:0]), torch.empty((M, 0), dtype=torch.bfloat16, device="cuda"),
                               dev(sa), dev(np.array([0.003], np.float32)), 1e-6, dx=dx0,
                               dw=torch.empty((0, K), device="cuda"), dscale_a=ds0)
    torch.cuda.synchronize()
    assert float(dx0.abs().max()) == 0.0 and float(ds0[0]) == 0.0
