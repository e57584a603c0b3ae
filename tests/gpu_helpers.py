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


def assert_out(gpu: np.ndarray, ref: np.ndarray, dtype, what: str, extra=None, scale=None):
    """Dequantized outputs: within 1 ulp of the oracle value (bf16/fp16) or 1e-5
    relative to the magnitude of the terms (fp32).  `extra` widens the bound
    elementwise by what tie-band codes can move; `scale` is the term magnitude
    used for fp32 (defaults to |ref|)."""
    err = np.abs(gpu.astype(np.float64) - ref)
    ex = 0.0 if extra is None else extra
    mag = np.abs(ref) if scale is None else scale
    if dtype == torch.float32:
        tol = 1e-5 * (mag + ex) + 1e-30
    else:
        # tie-band codes may move the value by up to `ex` and across a binade,
        # so the rounding step is the one at |ref| + ex; where a bias cancels
        # the product, the fp32 terms' 1e-5 relative bound is the wider one
        tol = np.maximum(ulp(np.abs(ref) + ex, dtype), 1e-5 * (mag + ex))
    tol = tol + ex
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst "
                           f"{float(np.max(err - tol)):.3e} over at {np.unravel_index(np.argmax(err - tol), err.shape)}")
