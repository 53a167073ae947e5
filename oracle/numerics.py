"""Rounding helpers of the oracle (float64 throughout, rounded only at the
precision contract points: bf16 for activations that feed a bf16 matrix
product, fp32 for the residual stream and accumulator outputs).

Pinned by: tests that compare bf16_round with the IEEE definition on
hand-made halfway cases and with torch's CPU bfloat16 conversion of float32
inputs (a library routine)."""

import numpy as np


def bf16_round(x):
    """Round float64 values straight to the nearest bfloat16 (ties to even);
    returns float64 values that are exactly representable in bf16."""
    x = np.asarray(x, dtype=np.float64)
    b = x.view(np.uint64).copy()
    sign = b & np.uint64(0x8000000000000000)
    mag = b & np.uint64(0x7FFFFFFFFFFFFFFF)
    # keep 7 explicit mantissa bits: drop the low 45 bits of the double mantissa
    low = mag & np.uint64((1 << 45) - 1)
    keep = mag >> np.uint64(45)
    half = np.uint64(1 << 44)
    up = (low > half) | ((low == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    out = (keep << np.uint64(45)) | sign
    r = out.view(np.float64)
    # values that underflow below the float normal range flush to zero, as in
    # the bf16 storage format used here (never reached by the workloads)
    return np.where(np.abs(x) < 2.0 ** -126, 0.0 * x, r)


def f32_round(x):
    """Round float64 values to float32 (nearest even), returned as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_bits_to_f64(bits):
    """Decode stored bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x):
    """Encode bf16-representable float64 values as uint16 bit patterns."""
    f = bf16_round(x).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
