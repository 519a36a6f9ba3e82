"""Helpers for the GPU parity tests (test-only)."""
import os

import numpy as np

from tests import npref

# Output tolerance of the layer (bf16 outputs against the oracle's fp64 values):
# max |err| <= 2e-2 * max |ref| and sum |err| / sum |ref| <= 5e-3.
MAX_TOL = 2e-2
MEAN_TOL = 5e-3
# Routing weights: the GPU computes w_j = expf(l_j - m) / sum in fp32 from the
# same fp32 logits; the subtraction, expf (<= 2 ulp), the sum of <= 32 terms and
# the division stay well inside 64 ulp of fp32 (2^-24 * 64 = 3.8e-6 relative).
W_RTOL = 4e-6

THREADS = max(1, min(32, os.cpu_count() or 1))


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(
        torch.bfloat16).cuda()


def from_dev_bf16(t):
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_output(y_bits, ref_f64, label=""):
    y = npref.bf16_bits_to_f64(y_bits)
    err = np.abs(y - ref_f64)
    mx = float(err.max() / np.abs(ref_f64).max())
    mean = float(err.sum() / np.abs(ref_f64).sum())
    assert np.all(np.isfinite(y)), label
    assert mx <= MAX_TOL, f"{label}: max err {mx:.3e} > {MAX_TOL}"
    assert mean <= MEAN_TOL, f"{label}: mean rel err {mean:.3e} > {MEAN_TOL}"
    return mx, mean
