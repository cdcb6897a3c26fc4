"""Helpers of the GPU parity tests: device transfers and the comparison metrics.

Tolerances (derived in the design notes):
  * fp32 paths: max|got - ref| <= 1e-5 * max|ref| (normwise relative);
  * bf16 inputs, fp32 outputs: max|got - ref| <= 1e-2 * RMS(ref) (outputs rescaled
    to unit RMS), LSE within 1e-3 absolute;
  * bf16 outputs additionally allow the output rounding itself, 2^-8 |ref|;
  * G, C: relative Frobenius error <= 1e-3; dW: <= 1e-2;
  * epsilon: |got - ref| <= tol * r2 (the scale of the terms that cancel).
"""
import numpy as np
import torch

DEV = "cuda"


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV).to(dtype).contiguous()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def nan_like(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device=DEV)


def max_over_rms(got, ref):
    return float(np.abs(got - ref).max() / np.sqrt(np.mean(ref ** 2)))


def rel_fro(got, ref):
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def normwise(got, ref):
    return float(np.abs(got - ref).max() / np.abs(ref).max())


def assert_bf16_out(got, ref, tol=1e-2):
    rms = np.sqrt(np.mean(ref ** 2))
    bound = tol * rms + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"max excess {float((err - bound).max())}, rms {rms}"


def assert_lse(got, ref, tol):
    both_inf = np.isneginf(got) & np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    # mask before subtracting: -inf - (-inf) is NaN
    d = np.abs(np.where(both_inf, 0.0, got) - np.where(both_inf, 0.0, ref))
    assert float(d.max()) <= tol, float(d.max())
