"""Pins of the oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself:
values the pages print (the ATB worked example), closed forms, invariants the
pages state, special cases that reduce to a library routine (numpy/torch in
float64), and hand-worked golden words.  A plausible mistake in the oracle (a
dropped eps, a wrong scale constant, a transposed operand, a wrong bit
position, round-half-up instead of half-to-even) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- rounding

def test_round_half_even_ties():
    cases = {0.5: 0.0, 1.5: 2.0, 2.5: 2.0, -0.5: 0.0, -1.5: -2.0, -2.5: -2.0,
             126.5: 126.0, 127.5: 128.0, 0.49999999: 0.0, 0.50000001: 1.0, -3.7: -4.0}
    for v, want in cases.items():
        assert oracle.round_half_even(v) == want, v


def test_round_half_even_matches_numpy_rint():
    g = synth.rng(11)
    v = np.concatenate([g.uniform(-300, 300, 2000), np.arange(-260, 260) + 0.5])
    got = np.array([oracle.round_half_even(t) for t in v])
    np.testing.assert_array_equal(got, np.rint(v))


# ---------------------------------------------------------- activation quant

def test_rmsnorm_matches_torch_rms_norm():
    x = synth.normal_f32(synth.rng(1), (16, 300))
    x[3] *= 1e-4  # a row where eps matters
    eps = 1e-5
    y = oracle.act_quant(x, eps, want_y=True)["y"]
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (300,), eps=eps).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=0)


def test_act_quant_invariants_random():
    x = synth.normal_f32(synth.rng(2), (64, 512))
    r = oracle.act_quant(x, 1e-5, want_pre=True)
    xq, pre = r["xq"].astype(np.int64), r["pre"]
    assert xq.min() >= -127 and xq.max() <= 127  # [-128,127] range; 127/absmax never reaches -128
    am = np.argmax(np.abs(x), axis=1)
    rows = np.arange(64)
    np.testing.assert_array_equal(xq[rows, am], np.sign(x[rows, am]).astype(np.int64) * 127)
    assert np.all(np.abs(xq - pre) <= 0.5 + 1e-12)  # rounding moves by at most half a step
    np.testing.assert_array_equal(r["rowsum"], xq.sum(axis=1))
    # dequantized value x_q * act_scale approximates the normalised y within half a step
    y = oracle.act_quant(x, 1e-5, want_y=True)["y"]
    assert np.all(np.abs(xq * r["act_scale"][:, None] - y) <= 0.5 * r["act_scale"][:, None] * (1 + 1e-12))


def test_act_quant_codes_scale_invariant():
    x = synth.normal_f32(synth.rng(3), (32, 256))
    a = oracle.act_quant(x)["xq"]
    b = oracle.act_quant(x * np.float32(8.0))["xq"]
    c = oracle.act_quant(x * np.float32(0.25))["xq"]
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a, c)


@pytest.mark.parametrize("c", [1.0, -0.75, 3.0e-3, 250.0])
def test_act_quant_constant_row_closed_form(c):
    K, eps = 96, 1e-5
    x = np.full((1, K), c, np.float32)
    r = oracle.act_quant(x, eps)
    cf = float(np.float32(c))
    assert np.all(r["xq"] == (127 if c > 0 else -127))
    want = 1.0 / (127.0 * math.sqrt(1.0 + eps / (cf * cf)))
    assert r["act_scale"][0] == pytest.approx(want, rel=1e-14)


def test_act_quant_one_hot_closed_form():
    K, eps, j, c = 200, 1e-5, 37, -2.5
    x = np.zeros((1, K), np.float32)
    x[0, j] = c
    r = oracle.act_quant(x, eps)
    want_q = np.zeros(K, np.int8)
    want_q[j] = -127
    np.testing.assert_array_equal(r["xq"][0], want_q)
    assert r["act_scale"][0] == pytest.approx(abs(c) / (127.0 * math.sqrt(c * c / K + eps)), rel=1e-14)
    assert r["rowsum"][0] == -127


def test_act_quant_zero_row():
    r = oracle.act_quant(np.zeros((2, 64), np.float32))
    assert np.all(r["xq"] == 0)
    np.testing.assert_array_equal(r["act_scale"], np.full(2, 1e-5 / 127.0))


# ------------------------------------------------------------ ternary quant

def test_ternary_hand_cases(golden_dir):
    d = _load(golden_dir, "ternary_hand_cases.json")
    for case in d["cases"]:
        w = np.array(case["w"], np.float32)
        t = oracle.ternary_quant(w)
        np.testing.assert_array_equal(t["wq"], np.array(case["wq"], np.int8), err_msg=case["name"])
        assert t["already_ternary"] == case["already_ternary"], case["name"]
        tol = case["gamma_rel_tol"]
        assert abs(t["gamma"] - case["gamma"]) <= tol * case["gamma"], case["name"]


def test_ternary_invariants_and_statistics():
    sigma = 0.02
    w = synth.normal_f32(synth.rng(4), (1024, 1024), sigma)
    t = oracle.ternary_quant(w, want_pre=True)
    assert set(np.unique(t["wq"]).tolist()) <= {-1, 0, 1}
    # gamma -> sigma * sqrt(2/pi) for a normal weight; zero fraction -> erf(0.5/sqrt(pi))
    assert t["gamma"] == pytest.approx(sigma * math.sqrt(2 / math.pi), rel=5e-3)
    zero_frac = float(np.mean(t["wq"] == 0))
    assert zero_frac == pytest.approx(math.erf(0.5 / math.sqrt(math.pi)), abs=3e-3)
    # codes agree with sign and the 0.5 threshold of the pre-rounding value
    pre = t["pre"]
    want = np.where(pre > 0.5, 1, np.where(pre < -0.5, -1, 0))
    np.testing.assert_array_equal(t["wq"], want)


def test_ternary_bake_idempotent():
    w = synth.normal_f32(synth.rng(5), (64, 128), 0.02)
    t1 = oracle.ternary_quant(w)
    baked = oracle.ternary_bake(t1["wq"], t1["gamma"])
    t2 = oracle.ternary_quant(baked)
    assert t2["already_ternary"]
    np.testing.assert_array_equal(t2["wq"], t1["wq"])
    assert t2["gamma"] == float(np.float32(t1["gamma"]))
    np.testing.assert_array_equal(oracle.ternary_bake(t2["wq"], t2["gamma"]), baked)
    # without the bake rule the scale would drift to gamma * (fraction nonzero)
    nz = float(np.mean(t1["wq"] != 0))
    assert abs(t2["gamma"] - t1["gamma"] * nz) > 0.1 * t1["gamma"]


# ------------------------------------------------------------------ packing

def test_ternary_pack_golden_words(golden_dir):
    d = _load(golden_dir, "pack_words.json")
    for case in d["ternary"]:
        wq = np.array([case["wq"]], np.int8)
        assert int(oracle.ternary_pack(wq)[0, 0]) == int(case["word"], 16)


def test_ternary_pack_roundtrip():
    g = synth.rng(6)
    wq = g.integers(-1, 2, (37, 160)).astype(np.int8)
    packed = oracle.ternary_pack(wq)
    back, bad = oracle.ternary_unpack(packed, 160)
    assert bad == 0
    np.testing.assert_array_equal(back, wq)


def test_int4_pack_golden_words(golden_dir):
    d = _load(golden_dir, "pack_words.json")
    for case in d["int4"]:
        q = np.array([case["q"]], np.uint8)
        assert int(oracle.int4_pack(q)[0, 0]) == int(case["word"], 16)


def test_int4_pack_roundtrip():
    q = synth.nibbles(synth.rng(7), (19, 77))
    np.testing.assert_array_equal(oracle.int4_unpack(oracle.int4_pack(q), 77), q)


def test_half_decode_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(got[finite], ref[finite])
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.all(got[np.isinf(ref)] == ref[np.isinf(ref)])


# ------------------------------------------------------------------- W8A8

def test_gemm_atb_worked_example(golden_dir):
    d = _load(golden_dir, "atb_per_token_example.json")
    x = np.array(d["x"], np.int8)
    w = np.array(d["weight"], np.int8)  # [k, n]
    out, ovf = oracle.gemm_i8_pertoken(x, w, np.array(d["deqScale"], np.float32),
                                       np.array(d["perTokenScale"], np.float32), layout=1)
    assert ovf == 0
    np.testing.assert_array_equal(out, np.array(d["output"], np.float64))
    # the same numbers with the weight in the nn.Linear [n, k] layout
    out_nk, _ = oracle.gemm_i8_pertoken(x, w.T.copy(), np.array(d["deqScale"], np.float32),
                                        np.array(d["perTokenScale"], np.float32), layout=0)
    np.testing.assert_array_equal(out_nk, out)


def test_gemm_unit_scales_is_integer_matmul():
    g = synth.rng(8)
    x, w = synth.int8_uniform(g, (23, 70)), synth.int8_uniform(g, (31, 70))
    out, _ = oracle.gemm_i8_pertoken(x, w, np.ones(31, np.float32), np.ones(23, np.float32))
    np.testing.assert_array_equal(out, (x.astype(np.int64) @ w.astype(np.int64).T).astype(np.float64))


def test_gemm_scales_and_bias_match_numpy():
    g = synth.rng(9)
    x, w = synth.int8_uniform(g, (17, 45)), synth.int8_uniform(g, (29, 45))
    deq, pts = synth.uniform_f32(g, (29,), 0.001, 0.01), synth.uniform_f32(g, (17,), 0.001, 0.01)
    bias = synth.normal_f32(g, (29,), 0.1)
    out, _ = oracle.gemm_i8_pertoken(x, w, deq, pts, bias)
    acc = (x.astype(np.int64) @ w.astype(np.int64).T).astype(np.float64)
    ref = pts.astype(np.float64)[:, None] * acc * deq.astype(np.float64)[None, :] + bias.astype(np.float64)
    np.testing.assert_allclose(out, ref, rtol=1e-15, atol=1e-15)
    # layout [K,N] with the transposed weight gives identical results
    out_kn, _ = oracle.gemm_i8_pertoken(x, w.T.copy(), deq, pts, bias, layout=1)
    np.testing.assert_array_equal(out_kn, out)


def test_gemm_reports_int32_overflow():
    # (-128)*(-128) = 2^14 per term: K = 2^17 terms reach 2^31, one past INT32_MAX
    K = 131072
    x = np.full((1, K), -128, np.int8)
    w = np.full((1, K), -128, np.int8)
    _, ovf = oracle.gemm_i8_pertoken(x, w, np.ones(1, np.float32), np.ones(1, np.float32))
    assert ovf == 1
    _, ovf = oracle.gemm_i8_pertoken(x[:, :K - 1], w[:, :K - 1], np.ones(1, np.float32), np.ones(1, np.float32))
    assert ovf == 0


# -------------------------------------------------------------- BitLinear

def test_bitlinear_constant_weight_closed_form():
    # every weight equal to c is already ternary: gamma = c, codes all +1, so
    # out[m,n] = c * act_scale[m] * rowsum(x_q)[m]
    x = synth.normal_f32(synth.rng(10), (5, 64))
    w = np.full((7, 64), 0.03, np.float32)
    out, a, t = oracle.bitlinear(x, w)
    assert t["already_ternary"] and t["gamma"] == float(np.float32(0.03))
    want = t["gamma"] * a["act_scale"] * a["rowsum"].astype(np.float64)
    np.testing.assert_allclose(out, np.repeat(want[:, None], 7, axis=1), rtol=1e-15)


def test_bitlinear_matches_integer_matmul_of_codes():
    d = synth.bitlinear_tiny(0)
    out, a, t = oracle.bitlinear(d["x"], d["w"], d["eps"])
    acc = a["xq"].astype(np.int64) @ t["wq"].astype(np.int64).T
    ref = acc.astype(np.float64) * a["act_scale"][:, None] * t["gamma"]
    np.testing.assert_allclose(out, ref, rtol=1e-15)
    # dequantized result approximates the float linear of the normalised input
    y = oracle.act_quant(d["x"], d["eps"], want_y=True)["y"]
    dense = y @ (t["wq"].astype(np.float64) * t["gamma"]).T
    assert np.max(np.abs(out - dense)) < 0.05 * np.max(np.abs(dense))


# ----------------------------------------------------------------- INT4

def _w4_case(g, M, N, K, gs):
    q = synth.nibbles(g, (N, K))
    z = synth.nibbles(g, (N, K // gs))
    s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
    b = synth.normal_f32(g, (N,), 0.01)
    x = synth.normal_f32(g, (M, K))
    return x, q, z, s, b


def test_w4_matches_dequantized_matmul():
    g = synth.rng(12)
    for (M, N, K, gs) in [(3, 20, 256, 128), (2, 9, 192, 64), (1, 5, 64, 64), (4, 11, 96, 8)]:
        x, q, z, s, b = _w4_case(g, M, N, K, gs)
        out = oracle.linear_w4_grouped(x, oracle.int4_pack(q), s.view(np.uint16), oracle.int4_pack(z), b, gs)
        deq = np.repeat(s.astype(np.float64), gs, axis=1) * (q.astype(np.float64) - np.repeat(z, gs, axis=1))
        ref = x.astype(np.float64) @ deq.T + b.astype(np.float64)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_w4_zero_point_equal_code_gives_bias():
    g = synth.rng(13)
    N, K, gs = 6, 128, 32
    z = synth.nibbles(g, (N, K // gs))
    q = np.repeat(z, gs, axis=1)
    s = g.uniform(0.005, 0.02, (N, K // gs)).astype(np.float16)
    b = synth.normal_f32(g, (N,), 0.01)
    out = oracle.linear_w4_grouped(synth.normal_f32(g, (3, K)), oracle.int4_pack(q), s.view(np.uint16),
                                   oracle.int4_pack(z), b, gs)
    np.testing.assert_array_equal(out, np.repeat(b.astype(np.float64)[None, :], 3, axis=0))


def test_w4_one_hot_gathers_x():
    g = synth.rng(14)
    N, K, gs = 8, 64, 16
    cols = g.integers(0, K, N)
    q = np.zeros((N, K), np.uint8)
    q[np.arange(N), cols] = 1
    z = np.zeros((N, K // gs), np.uint8)
    s = np.ones((N, K // gs), np.float16)
    x = synth.normal_f32(g, (2, K))
    out = oracle.linear_w4_grouped(x, oracle.int4_pack(q), s.view(np.uint16), oracle.int4_pack(z), None, gs)
    np.testing.assert_array_equal(out, x[:, cols].astype(np.float64))


def test_w4_one_hot_with_per_group_scale_picks_its_group():
    # one nonzero code per weight row, at a column k_n in a known group, with a
    # scale that differs per group and per row and no zero-point:
    # out[m,n] = s[n, k_n // gs] * x[m, k_n]  (every value exact in binary64)
    g = synth.rng(16)
    N, K, gs = 12, 256, 32
    G = K // gs
    cols = g.integers(0, K, N)
    cols[:G] = np.arange(G) * gs + 5  # every group is hit at least once
    q = np.zeros((N, K), np.uint8)
    q[np.arange(N), cols] = 1
    z = np.zeros((N, G), np.uint8)
    s = (0.5 * (np.arange(G)[None, :] + 1) + 0.125 * (np.arange(N)[:, None] % 4)).astype(np.float16)
    x = synth.normal_f32(g, (3, K))
    out = oracle.linear_w4_grouped(x, oracle.int4_pack(q), s.view(np.uint16), oracle.int4_pack(z), None, gs)
    want = np.empty((3, N))
    for n in range(N):
        want[:, n] = float(s[n, cols[n] // gs]) * x[:, cols[n]].astype(np.float64)
    np.testing.assert_array_equal(out, want)
    # zero-point 3 in that group only: its 31 zero codes weigh -3 and the one
    # code weighs 1 - 3, so out = s * (x[k_n] - 3 * sum of x over the group)
    z2 = z.copy()
    z2[np.arange(N), cols // gs] = 3
    out2 = oracle.linear_w4_grouped(x, oracle.int4_pack(q), s.view(np.uint16), oracle.int4_pack(z2), None, gs)
    want2 = np.empty((3, N))
    for n in range(N):
        g0 = (cols[n] // gs) * gs
        xg = x[:, g0:g0 + gs].astype(np.float64)
        want2[:, n] = float(s[n, cols[n] // gs]) * (x[:, cols[n]].astype(np.float64) - 3.0 * xg.sum(axis=1))
    np.testing.assert_allclose(out2, want2, rtol=1e-13, atol=1e-14)


def test_w4_single_group_is_plain_int4_linear():
    # group_size = K leaves one scale and zero-point per row: the grouped
    # affine form reduces to s_n * (x . q_n - z_n * sum(x)), i.e. the plain
    # unpack-on-demand INT4 dot product of the linear_4bit module, scaled and
    # shifted; with s = 1, z = 0 it is the integer-code matmul itself
    g = synth.rng(17)
    M, N, K = 4, 9, 128
    q = synth.nibbles(g, (N, K))
    x = synth.normal_f32(g, (M, K))
    one = np.ones((N, 1), np.float16)
    zero = np.zeros((N, 1), np.uint8)
    plain = oracle.linear_w4_grouped(x, oracle.int4_pack(q), one.view(np.uint16), oracle.int4_pack(zero), None, K)
    np.testing.assert_allclose(plain, x.astype(np.float64) @ q.astype(np.float64).T, rtol=1e-13, atol=1e-12)
    s = g.uniform(0.005, 0.02, (N, 1)).astype(np.float16)
    z = synth.nibbles(g, (N, 1))
    out = oracle.linear_w4_grouped(x, oracle.int4_pack(q), s.view(np.uint16), oracle.int4_pack(z), None, K)
    xs = x.astype(np.float64).sum(axis=1, keepdims=True)
    want = (plain - xs * z.astype(np.float64).T) * s.astype(np.float64).T
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


def test_bitlinear_one_code_per_row_pins_weight_indexing():
    # W has one nonzero per output row, +-c at column k_n: it is already
    # ternary, so gamma = c and out[m,n] = +-xq[m,k_n] * act_scale[m] * c.
    # M, N and K all differ, so a transposed operand or a swapped index fails.
    g = synth.rng(18)
    M, N, K = 5, 11, 48
    c = np.float32(0.0625)
    cols = g.permutation(K)[:N]
    sign = np.where(g.integers(0, 2, N) == 1, 1.0, -1.0).astype(np.float32)
    w = np.zeros((N, K), np.float32)
    w[np.arange(N), cols] = sign * c
    x = synth.normal_f32(g, (M, K))
    out, a, t = oracle.bitlinear(x, w)
    assert t["already_ternary"] and t["gamma"] == float(c)
    want = a["xq"][:, cols].astype(np.float64) * sign[None, :] * a["act_scale"][:, None] * float(c)
    np.testing.assert_array_equal(out, want)
    # the same through the codes entry point with a bias
    b = synth.normal_f32(g, (N,), 0.1)
    out_b = oracle.bitlinear_from_codes(a["xq"], a["act_scale"], t["wq"], t["gamma"], b)
    np.testing.assert_array_equal(out_b, want + b.astype(np.float64)[None, :])


# --------------------------------------------------------- batched W8A8

def test_gemm_batched_atb_example_stacked(golden_dir):
    # the worked example twice as a batch of 2 ([batch,m,k] x [batch,k,n]),
    # and with x stored transposed ([batch,k,m], transposeA): the printed
    # output for every batch
    d = _load(golden_dir, "atb_per_token_example.json")
    x = np.array(d["x"], np.int8)
    w = np.array(d["weight"], np.int8)  # [k, n]
    want = np.array(d["output"], np.float64)
    deq, pts = np.array(d["deqScale"], np.float32), np.array(d["perTokenScale"], np.float32)
    xb, wb = np.stack([x, x]), np.stack([w, w])
    out, ovf = oracle.gemm_i8_pertoken_batched(xb, wb, deq, pts, layout=1)
    assert ovf == 0
    np.testing.assert_array_equal(out, np.stack([want, want]))
    out_t, _ = oracle.gemm_i8_pertoken_batched(np.ascontiguousarray(xb.transpose(0, 2, 1)), wb, deq, pts,
                                                layout=1, trans_a=True)
    np.testing.assert_array_equal(out_t, np.stack([want, want]))
    out_nk, _ = oracle.gemm_i8_pertoken_batched(xb, np.ascontiguousarray(wb.transpose(0, 2, 1)), deq, pts,
                                                 layout=0)
    np.testing.assert_array_equal(out_nk, np.stack([want, want]))


def test_gemm_batched_is_per_batch_matmul_with_its_scales():
    # different data per batch: each batch equals the integer matmul of its
    # own operands (numpy int64), scaled by the shared or per-batch vectors
    g = synth.rng(19)
    B, M, N, K = 3, 5, 7, 40
    x, w = synth.int8_uniform(g, (B, M, K)), synth.int8_uniform(g, (B, N, K))
    deq_b, pts_b = synth.uniform_f32(g, (B, N), 0.001, 0.01), synth.uniform_f32(g, (B, M), 0.001, 0.01)
    out, _ = oracle.gemm_i8_pertoken_batched(x, w, deq_b, pts_b, shared_scales=False)
    for b in range(B):
        acc = (x[b].astype(np.int64) @ w[b].astype(np.int64).T).astype(np.float64)
        ref = pts_b[b].astype(np.float64)[:, None] * acc * deq_b[b].astype(np.float64)[None, :]
        np.testing.assert_allclose(out[b], ref, rtol=1e-15, atol=0)
    # shared scales: batch b uses deq[n] and pts[m] of the one vector each
    out_s, _ = oracle.gemm_i8_pertoken_batched(x, w, deq_b[1], pts_b[2])
    for b in range(B):
        acc = (x[b].astype(np.int64) @ w[b].astype(np.int64).T).astype(np.float64)
        ref = pts_b[2].astype(np.float64)[:, None] * acc * deq_b[1].astype(np.float64)[None, :]
        np.testing.assert_allclose(out_s[b], ref, rtol=1e-15, atol=0)


# ------------------------------------------------ LayerNorm normaliser

def test_layernorm_matches_torch_layer_norm():
    g = synth.rng(20)
    x = synth.normal_f32(g, (12, 300)) + np.float32(3.0)
    x[4] *= 1e-4  # eps matters
    w = (1.0 + 0.1 * g.standard_normal(300)).astype(np.float32)
    b = (0.05 * g.standard_normal(300)).astype(np.float32)
    for gw, gb in ((None, None), (w, b)):
        y = oracle.act_quant_layernorm(x, 1e-5, gw, gb, want_y=True)["y"]
        ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (300,),
                                             None if gw is None else torch.from_numpy(gw).double(),
                                             None if gb is None else torch.from_numpy(gb).double(),
                                             eps=1e-5).numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_layernorm_quant_shift_invariant_and_centred():
    # without the affine part the codes ignore a constant shift of the row
    # (RMSNorm's codes would not) and are those of x - mean(x)
    x = synth.normal_f32(synth.rng(21), (16, 256))
    a = oracle.act_quant_layernorm(x)
    b = oracle.act_quant_layernorm(x + np.float32(0.5))
    c = oracle.act_quant(x - x.astype(np.float64).mean(axis=1, keepdims=True).astype(np.float32))
    agree = (a["xq"] == b["xq"]).mean()
    assert agree > 0.999  # the shift is exact in fp32 only up to rounding of x + 0.5
    assert (a["xq"] == c["xq"]).mean() > 0.999
    r = oracle.act_quant(x + np.float32(0.5))
    assert (r["xq"] != a["xq"]).mean() > 0.1


def test_layernorm_quant_constant_row_and_affine_closed_forms():
    K = 64
    x = np.full((1, K), 2.5, np.float32)
    r = oracle.act_quant_layernorm(x)
    assert np.all(r["xq"] == 0) and r["act_scale"][0] == 1e-5 / 127.0
    # constant row with an affine bias: y = b exactly, so the codes quantize b
    b = np.linspace(-1.0, 1.0, K).astype(np.float32)
    r = oracle.act_quant_layernorm(x, ln_bias=b, want_pre=True)
    np.testing.assert_allclose(r["pre"][0], b.astype(np.float64) * 127.0 / np.abs(b).max(), rtol=1e-15)
    assert r["act_scale"][0] == pytest.approx(1.0 / 127.0, rel=1e-15)


# ------------------------------------------------------- W4A4 (Q4Linear)

def test_q4_quant_hand_cases():
    # step 0.5: values on the grid, half-step ties to even, clamping at -8 / 7
    v = np.array([[0.0, 0.5, -0.5, 0.25, 0.75, -0.25, -0.75, 1.25, 3.5, 3.75, 4.0, -4.0, -4.25, 100.0, -100.0,
                   0.2499]], np.float32)
    want = [0, 1, -1, 0, 2, 0, -2, 2, 7, 7, 7, -8, -8, 7, -8, 0]
    np.testing.assert_array_equal(oracle.q4_quant(v, np.float32(0.5), 1e-8)[0], want)
    # a step below eps is replaced by eps (no division by zero)
    np.testing.assert_array_equal(oracle.q4_quant(np.array([[0.0, 1e-6, -3e-6]], np.float32), np.float32(0.0), 1e-6)[0],
                                  [0, 1, -3])
    # per-row steps
    q = oracle.q4_quant(np.array([[1.0, 2.0], [1.0, 2.0]], np.float32), np.array([1.0, 0.5], np.float32), 1e-8,
                        per_row=True)
    np.testing.assert_array_equal(q, [[1, 2], [2, 4]])


def test_w4a4_unit_steps_is_integer_matmul():
    # integer inputs inside [-8, 7] with unit steps are their own codes, so
    # the forward is the integer matmul (numpy int64), plus the bias
    g = synth.rng(22)
    x = g.integers(-8, 8, (6, 48)).astype(np.float32)
    w = g.integers(-8, 8, (9, 48)).astype(np.float32)
    b = synth.normal_f32(g, (9,), 0.1)
    out, xq, wq = oracle.linear_w4a4(x, w, np.float32(1.0), np.float32(1.0), 1e-6, b)
    np.testing.assert_array_equal(xq, x.astype(np.int8))
    ref = x.astype(np.int64) @ w.astype(np.int64).T
    np.testing.assert_array_equal(out, ref.astype(np.float64) + b.astype(np.float64))


def test_w4a4_scales_pin_order_and_channel():
    # per-channel weight steps: out[m,n] = acc * s_w[n] * s_a exactly (powers of two)
    g = synth.rng(23)
    xq = g.integers(-8, 8, (4, 32)).astype(np.int8)
    wq = g.integers(-8, 8, (5, 32)).astype(np.int8)
    sw = np.array([0.5, 0.25, 2.0, 1.0, 0.125], np.float32)
    out = oracle.linear_w4a4_from_codes(xq, wq, np.float32(0.0625), sw, 1e-9, per_channel=True)
    acc = xq.astype(np.int64) @ wq.astype(np.int64).T
    np.testing.assert_array_equal(out, acc * sw.astype(np.float64)[None, :] * 0.0625)


def test_s4_pack_golden_and_roundtrip():
    q = np.array([[0, 1, -1, 7, -8, 2, -3, 5]], np.int8)
    # nibbles low first: 0x0, 0x1, 0xF, 0x7, 0x8, 0x2, 0xD, 0x5
    assert int(oracle.s4_pack(q)[0, 0]) == 0x5D287F10
    g = synth.rng(24)
    q = g.integers(-8, 8, (7, 64)).astype(np.int8)
    u = oracle.int4_unpack(oracle.s4_pack(q), 64).astype(np.int16)
    np.testing.assert_array_equal(np.where(u >= 8, u - 16, u), q)


# ------------------------------------------------------------- BitConv1d

def test_bitconv1d_matches_torch_conv1d_of_dequantized_values():
    # the convolution of the dequantized operands (xq * act_scale, wq * gamma)
    # by torch's conv1d in float64, for strides, padding and groups
    g = synth.rng(25)
    for (B, C_in, L, C_out, KS, stride, pad, groups) in [(2, 16, 11, 8, 3, 1, 1, 1), (1, 12, 9, 6, 2, 2, 0, 3),
                                                          (3, 8, 5, 4, 5, 1, 2, 2)]:
        x = synth.normal_f32(g, (B, C_in, L))
        w = synth.normal_f32(g, (C_out, C_in // groups, KS), 0.02)
        bias = synth.normal_f32(g, (C_out,), 0.1)
        out, a, t = oracle.bitconv1d(x, w, stride=stride, pad=pad, groups=groups, bias=bias)
        xd = (a["xq"].astype(np.float64) * a["act_scale"][:, None]).reshape(B, L, C_in).transpose(0, 2, 1)
        wd = t["wq"].reshape(w.shape).astype(np.float64) * t["gamma"]
        ref = torch.nn.functional.conv1d(torch.from_numpy(np.ascontiguousarray(xd)), torch.from_numpy(wd),
                                         torch.from_numpy(bias.astype(np.float64)), stride=stride, padding=pad,
                                         groups=groups).numpy()
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)


def test_bitconv1d_kernel_one_is_bitlinear_per_position():
    # kernel size 1, stride 1, no padding: each position is a BitLinear of
    # its LayerNorm-normalised channel vector
    g = synth.rng(26)
    B, C_in, L, C_out = 2, 32, 7, 5
    x = synth.normal_f32(g, (B, C_in, L))
    w = synth.normal_f32(g, (C_out, C_in, 1), 0.02)
    out, _, _ = oracle.bitconv1d(x, w)
    rows = np.ascontiguousarray(x.transpose(0, 2, 1).reshape(B * L, C_in))
    ref, _, _ = oracle.bitlinear_layernorm(rows, w[:, :, 0])
    np.testing.assert_allclose(out, ref.reshape(B, L, C_out).transpose(0, 2, 1), rtol=1e-14, atol=0)


# ------------------------------------------------- BitLinear STE backward

def test_bitlinear_backward_matches_autograd_of_the_ste_surrogate():
    # torch autograd (fp64) of the straight-through forward written with
    # detach: y + (xt - y).detach() and w + (wt - w).detach(), where xt and wt
    # are the oracle's dequantized operands, through torch's own RMSNorm
    g = synth.rng(27)
    M, N, K = 6, 10, 48
    x = synth.normal_f32(g, (M, K))
    w = synth.normal_f32(g, (N, K), 0.02)
    dout = synth.normal_f32(g, (M, N))
    eps = 1e-5
    dx, dw = oracle.bitlinear_backward(x, w, dout, eps)
    a = oracle.act_quant(x, eps)
    t = oracle.ternary_quant(w)
    xt = torch.from_numpy(a["xq"].astype(np.float64) * a["act_scale"][:, None])
    wt = torch.from_numpy(t["wq"].astype(np.float64) * t["gamma"])
    xx = torch.from_numpy(x.astype(np.float64)).requires_grad_()
    ww = torch.from_numpy(w.astype(np.float64)).requires_grad_()
    y = torch.nn.functional.rms_norm(xx, (K,), eps=eps)
    out = (y + (xt - y).detach()) @ (ww + (wt - ww).detach()).T
    out.backward(torch.from_numpy(dout.astype(np.float64)))
    np.testing.assert_allclose(dx, xx.grad.numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(dw, ww.grad.numpy(), rtol=1e-10, atol=1e-13)


# ------------------------------------------------- Q4Linear straight-through backward

def test_w4a4_backward_hand_worked():
    # x = (1.375, 5), s_a = 0.5: u = (2.75, 10), codes (3, 7 clamped); w = (0.625, -0.25), s_w = 0.25:
    # v = (2.5, -1), codes (2, -1) (2.5 ties to even), wh = (0.5, -0.25); dout = 2:
    # g = (1, -0.5); dx = (1, 0) (the second quotient is outside [-8, 7]);
    # dw = 2 * xh = 2 * (1.5, 3.5) = (3, 7); dscale_a = 1 * (3 - 2.75) + (-0.5) * 7 = -3.25
    r = oracle.linear_w4a4_backward(np.array([[1.375, 5.0]], np.float32), np.array([[0.625, -0.25]], np.float32),
                                    np.array([[2.0]], np.float32), 0.5, 0.25, 1e-6)
    np.testing.assert_array_equal(r["g"], [[1.0, -0.5]])
    np.testing.assert_array_equal(r["dx"], [[1.0, 0.0]])
    np.testing.assert_array_equal(r["dw"], [[3.0, 7.0]])
    assert r["dscale_a"] == -3.25
    # a weight quotient outside the range masks its weight gradient: w = 2.5 at s_w = 0.25 gives v = 10
    r = oracle.linear_w4a4_backward(np.array([[1.375]], np.float32), np.array([[2.5]], np.float32),
                                    np.array([[2.0]], np.float32), 0.5, 0.25, 1e-6)
    np.testing.assert_array_equal(r["dw"], [[0.0]])
    np.testing.assert_array_equal(r["g"], [[2.0 * 0.25 * 7]])


def _ste_dequant(v, s):
    # s * clamp(rne(v / s), -8, 7) in value; rounding passed straight through, the clamp's
    # gradient taken on the unrounded quotient
    u = v / s
    cu = torch.clamp(u, -8.0, 7.0)
    q = torch.clamp(torch.round(u), -8.0, 7.0)
    return s * (cu + (q - cu).detach())


@pytest.mark.parametrize("per_channel,scale_a", [(False, 0.15), (True, 0.15), (False, 1e-9)])
def test_w4a4_backward_matches_autograd_of_the_ste_surrogate(per_channel, scale_a):
    g = synth.rng((29, per_channel))
    M, N, K = 5, 9, 40
    eps = 1e-6
    x = synth.normal_f32(g, (M, K))
    w = synth.normal_f32(g, (N, K), 0.02)
    dout = synth.normal_f32(g, (M, N))
    sw = (np.float32(0.003) * (1 + g.random(N))).astype(np.float32) if per_channel else np.float32(0.003)
    r = oracle.linear_w4a4_backward(x, w, dout, scale_a, sw, eps, per_channel=per_channel)
    xx = torch.from_numpy(x.astype(np.float64)).requires_grad_()
    ww = torch.from_numpy(w.astype(np.float64)).requires_grad_()
    sa = torch.tensor(float(np.float32(scale_a)), dtype=torch.float64, requires_grad=True)
    swt = torch.from_numpy(np.atleast_1d(sw).astype(np.float64))
    s_a = torch.clamp(sa, min=eps)
    s_w = torch.clamp(swt, min=eps)[:, None] if per_channel else torch.clamp(swt, min=eps)
    out = _ste_dequant(xx, s_a) @ _ste_dequant(ww, s_w).T
    out.backward(torch.from_numpy(dout.astype(np.float64)))
    # the case must exercise both sides of the range
    u = x.astype(np.float64) / max(float(np.float32(scale_a)), eps)
    if scale_a > eps:
        assert ((u < -8) | (u > 7)).any() and ((u >= -8) & (u <= 7)).any()
    np.testing.assert_allclose(r["dx"], xx.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["dw"], ww.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert abs(r["dscale_a"] - float(sa.grad)) <= 1e-10 * (1 + abs(float(sa.grad)))
    if scale_a < eps:
        assert r["dscale_a"] == 0.0
