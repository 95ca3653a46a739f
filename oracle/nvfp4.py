"""CPU oracle, part 1: the NVFP4 weight format (decode from bits, and pack).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module;
only the tests, the package's smoke check and the bench's CPU-baseline leg do.

The pages name the format but do not spell it out: experts are served as
"NVFP4" (FreeToken model guide, "--quant-backend moe.nvfp4" in the MoE
scheduling section; sm89-moe-offload fork README, "Production configuration"
and "Key customizations", wide-load NVFP4 prefill MoE kernel).  The plainest
reading, used here, is the standard NVFP4 layout:

* each weight is a 4-bit E2M1 code: bit 3 sign, bits 2..1 exponent (bias 1),
  bit 0 mantissa; exponent 0 is subnormal (0 or 0.5);
* every 16 consecutive weights along K of one output row share one E4M3 (FN
  variant: bias 7, subnormals, no infinities, S.1111.111 = NaN, max 448)
  scale byte;
* each weight tensor has one fp32 global scale;
* dequantised weight = e2m1(code) * e4m3(scale) * global.

Byte layout (a reading; the pages are silent): codes are packed two per byte,
row-major [N, K/2], element k in the low nibble when k is even; scales are
row-major [N, ld_scale] bytes with ld_scale >= K/16 (padding bytes are zero).

All arithmetic is fp64 unless a step is stated to be fp32.  Parity pins: see
tests/test_oracle_nvfp4.py (hand-worked tables, closed forms, exhaustive
bf16-exactness, round-trip and error bounds).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


# ---------------------------------------------------------------- decode ---

def e2m1_value(code: int) -> float:
    """Value of one E2M1 code, from its bit fields."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        mag = 0.5 * m                       # subnormal: m * 2^(1-bias) * 1/2
    else:
        mag = (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return -mag if s else mag


def e4m3_value(byte: int) -> float:
    """Value of one E4M3 (FN) byte, from its bit fields.  NaN for S.1111.111."""
    s = (byte >> 7) & 1
    e = (byte >> 3) & 15
    m = byte & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** -6
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)


def unpack_codes(codes: np.ndarray, N: int, K: int) -> np.ndarray:
    """uint8 [N, K/2] -> uint8 [N, K] of 4-bit codes (even k = low nibble)."""
    c = np.asarray(codes, dtype=np.uint8).reshape(N, K // 2)
    out = np.empty((N, K), dtype=np.uint8)
    out[:, 0::2] = c & 0x0F
    out[:, 1::2] = c >> 4
    return out


def decode(codes: np.ndarray, scales: np.ndarray, global_scale: float,
           N: int, K: int, ld_scale: int) -> np.ndarray:
    """NVFP4 tensor -> fp64 [N, K] (exact: every product fits in fp64)."""
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    q = E2M1_TABLE[unpack_codes(codes, N, K)]
    sb = np.asarray(scales, dtype=np.uint8).reshape(N, ld_scale)[:, : K // 16]
    s = E4M3_TABLE[sb]
    if np.isnan(s).any():
        raise ValueError("NaN E4M3 scale byte")
    return q * np.repeat(s, 16, axis=1) * float(np.float32(global_scale))


# ------------------------------------------------------------------ pack ---

# Non-negative finite E4M3 values, indexed by code 0..126 (ascending).
_E4M3_POS = E4M3_TABLE[:127].copy()
# Non-negative E2M1 magnitudes, indexed by code 0..7 (ascending).
_E2M1_POS = E2M1_TABLE[:8].copy()


def _round_to_grid(v: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the nearest grid value to each v >= 0; ties go to the even
    index (the code whose mantissa LSB is 0); values above the top saturate."""
    v = np.asarray(v, dtype=np.float64)
    hi = np.searchsorted(grid, v, side="left")           # grid[hi-1] < v <= grid[hi]
    hi = np.clip(hi, 1, len(grid) - 1)
    lo = hi - 1
    dlo = v - grid[lo]
    dhi = grid[hi] - v
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(v >= grid[-1], len(grid) - 1, idx)
    idx = np.where(v <= grid[0], 0, idx)
    return idx.astype(np.uint8)


def e4m3_rne_sat(v: np.ndarray) -> np.ndarray:
    """Non-negative value -> E4M3 byte (nearest, ties to even, saturating)."""
    return _round_to_grid(v, _E4M3_POS)


def e2m1_rne_sat(v: np.ndarray) -> np.ndarray:
    """Signed value -> E2M1 code (nearest, ties to even, saturating at 6).
    The sign bit follows the sign bit of the input (so -0.1 -> -0)."""
    v = np.asarray(v, dtype=np.float32)
    mag = _round_to_grid(np.abs(v).astype(np.float64), _E2M1_POS)
    return (mag | (np.signbit(v).astype(np.uint8) << 3)).astype(np.uint8)


def global_scale_of(w: np.ndarray) -> np.float32:
    """fp32 global scale: amax / (6 * 448), or 1 for an all-zero tensor."""
    amax = np.float32(np.max(np.abs(np.asarray(w, dtype=np.float32)))) if w.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX))


def pack(w: np.ndarray, ld_scale: int | None = None):
    """fp32 [N, K] -> (codes uint8 [N, K/2], scales uint8 [N, ld_scale], global fp32).

    Steps, each an IEEE fp32 operation rounded to nearest:
      g       = amax / 2688                      (amax over the whole tensor)
      r_b     = amax_b / (6 * g)                 (amax_b over one 16-block)
      s_b     = E4M3(r_b)                        (nearest, ties to even, saturate)
      q       = E2M1(w / (dec(s_b) * g))         (nearest, ties to even, saturate)
    A block whose scale decodes to 0 stores code 0 everywhere.
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    ld = K // 16 if ld_scale is None else ld_scale
    g = global_scale_of(w)
    blocks = np.abs(w).reshape(N, K // 16, 16)
    amax_b = blocks.max(axis=2).astype(np.float32)
    denom = np.float32(np.float32(6.0) * g)
    r = (amax_b / denom).astype(np.float32)
    s_code = e4m3_rne_sat(r.astype(np.float64))
    s_val = E4M3_TABLE[s_code].astype(np.float32)
    qden = (s_val * g).astype(np.float32)                      # [N, K/16]
    qden_full = np.repeat(qden, 16, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (w / qden_full).astype(np.float32)
    code = e2m1_rne_sat(v)
    code[np.repeat(s_val == 0, 16, axis=1)] = 0
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    scales = np.zeros((N, ld), dtype=np.uint8)
    scales[:, : K // 16] = s_code
    return packed, scales, np.float32(g)
