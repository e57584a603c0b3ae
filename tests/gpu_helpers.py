"""Shared helpers of the GPU parity tests: tensor transfer, tolerances and the
rounding-tie exemption.  Expected values always come from ``oracle`` run on
the same seeded inputs as the CUDA path; nothing computed on the GPU is fed
back into the oracle."""
import numpy as np
import torch

TIE_REL = 1e-6  # a code whose exact pre-rounding value lies this close to a .5 boundary may round either way


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits):
    return dev(bits.view(np.int16), torch.bfloat16)


def padded(a: np.ndarray, align_elems: int):
    """Device copy of a 2-D array whose row stride is rounded up to align_elems."""
    M, K = a.shape
    ld = (K + align_elems - 1) // align_elems * align_elems
    buf = np.zeros((M, ld), a.dtype)
    buf[:, :K] = a
    return dev(buf)[:, :K]


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.cpu().numpy()


def tie_band(pre: np.ndarray) -> np.ndarray:
    """Elements whose pre-rounding value lies within TIE_REL (relative) of a .5 boundary."""
    frac = pre - np.floor(pre)
    return np.abs(frac - 0.5) <= TIE_REL * np.maximum(np.abs(pre), 1e-30)


def assert_codes(gpu: np.ndarray, ref: np.ndarray, pre: np.ndarray, what: str):
    """Bit-exact integer codes, except that tie-band elements may differ by one."""
    gpu = gpu.astype(np.int64)
    ref = ref.astype(np.int64)
    diff = gpu != ref
    band = tie_band(pre)
    bad = diff & ~band
    assert not bad.any(), f"{what}: {int(bad.sum())} codes differ outside the tie band, first at {np.argwhere(bad)[:5]}"
    assert np.all(np.abs(gpu - ref)[diff] == 1), f"{what}: a tie-band code moved by more than one"
    return int(diff.sum())


def ulp(v: np.ndarray, dtype) -> np.ndarray:
    a = np.abs(v)
    if dtype == torch.bfloat16:
        return 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -126))) - 7)
    if dtype == torch.float16:
        return 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -14))) - 10)
    raise ValueError(dtype)


U32 = 2.0 ** -24  # unit roundoff of fp32

# The GPU epilogue computes out = ((float(acc) * s1) * s2) + bias in fp32 and
# rounds once to the output type.  Three roundings on the product p (the int
# to float conversion and two multiplies) and one on the sum bound its fp32
# error by 4u(|p| + |bias|), u = 2^-24 (first order).
EPILOGUE_REL = 4 * U32


def assert_out(gpu: np.ndarray, ref: np.ndarray, dtype, what: str, extra=None, scale=None, rel32=EPILOGUE_REL):
    """Dequantized outputs against the oracle's binary64 value `ref`.

    bf16/fp16: |gpu - ref| <= 1 ulp(|ref| + ex) + rel32 * (mag + ex) + ex, i.e.
    one unit in the last place of the output type plus the fp32 epilogue's own
    error bound, which only matters where a bias cancels the product.
    fp32: |gpu - ref| <= 1e-5 * (mag + ex) + ex.
    `mag` is the magnitude of the terms, |product| + |bias| (`scale`; defaults
    to |ref|); `ex` (`extra`) is what tie-band codes can move the value by;
    `rel32` may be an array broadcast against `ref` (per-row scale errors)."""
    err = np.abs(gpu.astype(np.float64) - ref)
    ex = 0.0 if extra is None else extra
    mag = np.abs(ref) if scale is None else scale
    if dtype == torch.float32:
        tol = 1e-5 * (mag + ex) + 1e-30
    else:
        # tie-band codes may move the value by up to `ex` and across a binade,
        # so the rounding step is the one at |ref| + ex
        tol = ulp(np.abs(ref) + ex, dtype) + rel32 * (mag + ex)
    tol = tol + ex
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst "
                           f"{float(np.max(err - tol)):.3e} over at {np.unravel_index(np.argmax(err - tol), err.shape)}")


def bitlinear_expected(x_f32, w_f32, bias, eps=1e-5, rows=None, ln=None):
    """Oracle BitLinear output for rows `rows` of x (all when None) with what
    the tolerance needs: the tie-band widening `extra`, the term magnitude
    `scale` (None without bias) and the oracle's steps `a` (act quant) and `t`
    (ternary quant).  `ln` = (ln_weight, ln_bias) selects the LayerNorm
    normaliser.  Everything here comes from the oracle alone."""
    import oracle
    M = x_f32.shape[0]
    sel = np.arange(M) if rows is None else rows
    if ln is None:
        a = oracle.act_quant(x_f32[sel], eps, want_pre=True)
    else:
        a = oracle.act_quant_layernorm(x_f32[sel], eps, ln[0], ln[1], want_pre=True)
    t = oracle.ternary_quant(w_f32, want_pre=True)
    ref = oracle.bitlinear_from_codes(a["xq"], a["act_scale"], t["wq"], t["gamma"], bias)
    # codes in the tie band may round either way: widen by what they can move
    xband = tie_band(a["pre"]).astype(np.float64)
    wband = tie_band(t["pre"]).astype(np.float64)
    extra = (xband @ np.abs(t["wq"]).T.astype(np.float64) + np.abs(a["xq"]).astype(np.float64) @ wband.T) \
        * a["act_scale"][:, None] * t["gamma"]
    scale = None
    if bias is not None:
        b = bias.astype(np.float64)
        scale = np.abs(ref - b) + np.abs(b)
    return ref, extra, scale, a, t


def bitlinear_rel32(gpu_act_scale, ref_act_scale, gpu_gamma, ref_gamma):
    """fp32 error bound of the BitLinear epilogue per row: the epilogue's own
    4u plus the relative deviation of the GPU's act_scale (row) and gamma from
    the oracle's, which the tests bound separately (1e-5 relative)."""
    da = np.abs(np.asarray(gpu_act_scale, np.float64) - ref_act_scale) / ref_act_scale
    dg = abs(float(gpu_gamma) - ref_gamma) / ref_gamma
    assert da.max() <= 1e-5 and dg <= 1e-5, f"scales off: act_scale {da.max():.2e}, gamma {dg:.2e}"
    return EPILOGUE_REL + da[:, None] + dg
