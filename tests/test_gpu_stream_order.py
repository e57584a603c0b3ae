"""Stream order of the weight-streaming decode kernels.

The one-launch decode kernels (RMSNorm at one to sixteen tokens, LayerNorm at
one token) read nothing before their dependency wait but prefetch their
weights into L2 there; the LayerNorm decode at 2..16 tokens issues its weight
loads before its wait, which is correct only because the LayerNorm quantizer
launched ahead of it in the same call waits for everything earlier in the
stream before it releases it.  Here the packed weights are rewritten in place by the packing
kernel on the same stream directly before each call, with a different weight
matrix each time and no host synchronisation in between; every output must be
bit-identical to the same call made after a full synchronisation (the same
kernels, so the same bits).  A kernel that read its weights too early would
see the previous matrix.
"""
import numpy as np
import pytest
import torch

import bit_quantized_linear_rmsnorm_b200 as bq
import synth

pytestmark = pytest.mark.gpu

N, K = 11008, 4096  # a large matrix, so that packing runs for tens of microseconds


@pytest.fixture(scope="module", autouse=True)
def _ready():
    from bit_quantized_linear_rmsnorm_b200 import _build
    _build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    torch.cuda.init()
    yield
    st, detail = bq.bq_device_status()
    assert st == bq.BQ_OK, f"device status word {detail:#x}"


def _call(ln, x, wp, ws, lw, lb, out):
    if ln:
        return bq.bq_bitlinear_w2a8_layernorm(x, wp, ws, N, lw, lb, None, 1e-5, torch.bfloat16, out=out)
    return bq.bq_bitlinear_w2a8(x, wp, ws, N, None, 1e-5, torch.bfloat16, out=out)


@pytest.mark.parametrize("M,ln", [(1, False), (4, False), (16, False), (1, True), (4, True), (16, True)])
def test_weights_packed_just_before_the_call(M, ln):
    dev = "cuda"
    # three different weight matrices, each scaled differently so that a stale read changes every output
    ws_f32 = [torch.from_numpy(synth.bitlinear_weight(N, K, 40 + i, std=0.02 * (i + 1))).to(dev) for i in range(3)]
    x = torch.from_numpy(synth.bitlinear_decode(M)["x_bf16"].view(np.int16)).to(dev).view(torch.bfloat16)
    g = synth.rng((77, M))
    lw = torch.from_numpy((1.0 + 0.2 * g.standard_normal(K)).astype(np.float32)).to(dev) if ln else None
    lb = torch.from_numpy((0.1 * g.standard_normal(K)).astype(np.float32)).to(dev) if ln else None
    wp = torch.empty((N, K // 16), dtype=torch.int32, device=dev)
    wsc = torch.empty(1, dtype=torch.float32, device=dev)

    # reference: pack, synchronise, call, synchronise
    refs = []
    for w in ws_f32:
        bq.bq_weight_quant_ternary_pack(w, wpacked=wp, w_scale=wsc)
        torch.cuda.synchronize()
        refs.append(_call(ln, x, wp, wsc, lw, lb, torch.empty((M, N), dtype=torch.bfloat16, device=dev)))
        torch.cuda.synchronize()

    # the same sequence twice over without any synchronisation
    outs = []
    for _ in range(2):
        for w in ws_f32:
            bq.bq_weight_quant_ternary_pack(w, wpacked=wp, w_scale=wsc)
            outs.append(_call(ln, x, wp, wsc, lw, lb, torch.empty((M, N), dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        r = refs[i % 3]
        assert torch.equal(o.view(torch.int16), r.view(torch.int16)), f"call {i}: output differs from the synchronised call"
    # and consecutive references really differ, so a stale read could not pass
    assert not torch.equal(refs[0], refs[1]) and not torch.equal(refs[1], refs[2])


@pytest.mark.parametrize("M", [1, 4])
def test_w4a4_weights_packed_just_before_the_call(M):
    # the 4-bit path: act-quant kernel, then the GEMV launched as its programmatic dependent
    dev = "cuda"
    K4, N4 = 4096, 11008
    g = synth.rng((78, M))
    ws_f32 = [torch.from_numpy(synth.normal_f32(g, (N4, K4), 0.02 * (i + 1))).to(dev) for i in range(3)]
    x = torch.from_numpy(synth.normal_f32(g, (M, K4))).to(dev)
    sa = torch.tensor([0.27], dtype=torch.float32, device=dev)
    sw = torch.tensor([0.006], dtype=torch.float32, device=dev)
    wp = torch.empty((N4, K4 // 8), dtype=torch.int32, device=dev)
    refs = []
    for w in ws_f32:
        bq.bq_weight_quant_int4_pack(w, sw, 1e-6, wpacked=wp)
        torch.cuda.synchronize()
        refs.append(bq.bq_linear_w4a4(x, sa, wp, sw, N4, 1e-6, out_dtype=torch.float32))
        torch.cuda.synchronize()
    outs = []
    for _ in range(2):
        for w in ws_f32:
            bq.bq_weight_quant_int4_pack(w, sw, 1e-6, wpacked=wp)
            outs.append(bq.bq_linear_w4a4(x, sa, wp, sw, N4, 1e-6, out_dtype=torch.float32))
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o, refs[i % 3]), f"call {i}: output differs from the synchronised call"
    assert not torch.equal(refs[0], refs[1])
