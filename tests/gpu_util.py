"""Shared helpers for the GPU parity tests."""

import numpy as np
import pytest
import torch

# Tolerances: fp16/bf16 inputs with fp32 accumulation, output requested in
# fp32 -> max abs error 2e-3; fp32 inputs -> 1e-5.
# With the output in the input's 16-bit dtype the kernel returns RNE(y) for
# its fp32 result y.  If |y - x| <= EPS16 for the float64 oracle x, then
# |RNE(y) - RNE(x)| <= 1 ulp + EPS16, which is what is checked (a bare "1 ulp"
# cannot hold near zero, where an ulp is far below any fp32 error bound).
TOL = {torch.float16: 2e-3, torch.bfloat16: 2e-3, torch.float32: 1e-5}
EPS16 = 1e-5
# Precision regression bound on the fp32 output of the 16-bit kernels.  The
# dominant rounding is the two-term split of each softmax weight p into 16-bit
# parts for the tensor-core p.V product: relative error <= 2^-16 (bf16) or
# 2^-22 (fp16) per weight, so |error| <= 2^-16 * max|v| (+ fp32 rounding).
# For N(0, 1) values (|v| < 6) that is below 1e-4 (bf16) / 1e-5 (fp16); a
# dropped or mis-paired term exceeds it by an order of magnitude.
PRECISION = {torch.bfloat16: 1e-4, torch.float16: 1e-5, torch.float32: 1e-5}
MANTISSA_BITS = {torch.float16: 10, torch.bfloat16: 7}

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a tensor (for bitwise comparisons)."""
    view = {2: torch.int16, 4: torch.int32, 8: torch.int64}[t.element_size()]
    return t.detach().contiguous().view(view).cpu().numpy()


def ulp_of(x: np.ndarray, dtype) -> np.ndarray:
    """Spacing of the 16-bit format at each value's magnitude (normal range)."""
    mant = MANTISSA_BITS[dtype]
    ax = np.abs(x).astype(np.float64)
    tiny = {torch.float16: 2.0 ** -24, torch.bfloat16: 2.0 ** -133}[dtype]
    e = np.floor(np.log2(np.maximum(ax, 1e-300)))
    return np.maximum(2.0 ** (e - mant), tiny)


def assert_close_to_oracle(out: torch.Tensor, ref: np.ndarray, in_dtype, what=""):
    """fp32 output: max abs error within TOL; 16-bit output: within 1 ulp + EPS16 of RNE(ref)."""
    got = out.detach().float().cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    if out.dtype == torch.float32:
        err = np.abs(got - ref).max() if got.size else 0.0
        assert err <= TOL[in_dtype], f"{what}: max abs error {err:.3e} > {TOL[in_dtype]:.0e}"
        return err
    err = np.abs(got - ref).max() if got.size else 0.0
    rne = torch.from_numpy(ref).to(out.dtype).double().numpy()
    diff = np.abs(got - rne)
    lim = ulp_of(rne, out.dtype) * 1.0000001 + EPS16
    bad = diff > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements further than 1 ulp + {EPS16:.0e} "
                           f"from the rounded oracle (worst {diff[bad].max():.3e})")
    return float(err)


def assert_precise(out: torch.Tensor, ref: np.ndarray, in_dtype, what=""):
    """fp32 output within the precision regression bound of the 16-bit kernels."""
    assert out.dtype == torch.float32
    err = float(np.abs(out.detach().cpu().numpy().astype(np.float64) - ref).max())
    assert err <= PRECISION[in_dtype], f"{what}: max abs error {err:.3e} > {PRECISION[in_dtype]:.0e}"
    return err
