"""CPU oracle: the MXFP4 weight format, in numpy (an independent restatement
of the C++ oracle's MXFP4 pack and decode, written apart from it).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module.

The pages list MXFP4 beside NVFP4 as an expert format ("FlashML-org /
FreeToken" about page, quantization formats; model guide, CPU executor
formats) without defining it; the reading is the OCP Microscaling Formats
(MX) v1.0 specification:

* elements are E2M1 codes (the same 4-bit format as NVFP4's);
* every 32 consecutive elements along K of one row share one E8M0 scale
  byte s: 2^(s - 127), 255 = NaN, no sign and no zero;
* value = e2m1(code) * 2^(s - 127); there is no per-tensor scale;
* conversion from fp32: the shared exponent is floor(log2 max|w|) minus the
  largest exponent of E2M1 (2, as 6 = 1.5 * 2^2), clamped to [-127, 127]
  (-127 for an all-zero block); each element is w / 2^x rounded to the
  nearest E2M1 value, ties to the even code, saturating at 6, sign kept.
"""
from __future__ import annotations

import math

import numpy as np

from .nvfp4 import e2m1_value

# E2M1 magnitudes, ascending, indexed by the 3 low code bits
_MAG = np.array([e2m1_value(c) for c in range(8)], dtype=np.float64)


def e8m0_value(byte: int) -> float:
    return float("nan") if byte == 255 else math.ldexp(1.0, byte - 127)


def _nearest_code(a: float) -> int:
    """Index of the E2M1 magnitude nearest to a >= 0 (ties to the even index,
    saturating above 6), by comparing against every magnitude."""
    if a >= _MAG[-1]:
        return 7
    d = np.abs(_MAG - a)
    best = np.flatnonzero(d == d.min())
    return int(best[0]) if len(best) == 1 or best[0] % 2 == 0 else int(best[1])


def pack(w: np.ndarray):
    """fp32 [N, K] (K % 32 == 0) -> (codes uint8 [N, K/2], scales uint8 [N, K/32])."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    if not np.isfinite(w).all():
        raise ValueError("non-finite input")
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // 32), np.uint8)
    for n in range(N):
        for b in range(K // 32):
            blk = w[n, 32 * b:32 * b + 32].astype(np.float64)
            amax = float(np.max(np.abs(blk)))
            # floor(log2 amax) is the frexp exponent minus 1 (amax = f * 2^e, f in [0.5, 1))
            x = -127 if amax == 0.0 else max(-127, min(127, math.frexp(amax)[1] - 1 - 2))
            scales[n, b] = x + 127
            for i in range(32):
                v = math.ldexp(float(blk[i]), -x)
                c = _nearest_code(abs(v)) | (8 if math.copysign(1.0, v) < 0 else 0)
                k = 32 * b + i
                if k % 2 == 0:
                    codes[n, k // 2] |= c
                else:
                    codes[n, k // 2] |= c << 4
    return codes, scales


def decode(codes: np.ndarray, scales: np.ndarray, K: int) -> np.ndarray:
    """MXFP4 [N, K] -> fp64 values."""
    N = codes.shape[0]
    out = np.zeros((N, K), np.float64)
    for n in range(N):
        for k in range(K):
            byte = int(codes[n, k // 2])
            c = (byte >> 4) if k % 2 else (byte & 15)
            out[n, k] = e2m1_value(c) * e8m0_value(int(scales[n, k // 32]))
    return out
