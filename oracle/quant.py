"""Quantiser emulation for the low-precision read copy -- TEST INFRASTRUCTURE.

The ReplaySSM reports keep a high-precision checkpoint for the recurrent update
and a low-precision copy that only outputs are read from ("Deux precisions pour
le prix d'une", irisproject.cloud; item 5 of "Co sie zmienilo?",
ainews.tenesys.com).  They do not fix the formats; the readings used here:

* bf16: round-to-nearest-even from the fp32 value (IEEE binary32 -> bfloat16).
* fp8 e4m3 ("fn" variant: bias 7, no infinities, max finite 448, subnormal step
  2^-9), round-to-nearest-even, saturating to +-448, with one fp32 scale per row
  (a row = the N contiguous elements of one state row): scale = amax/448
  (scale = 1 when the row is all zeros), code = e4m3(value / scale) with the
  division done in fp32, dequantised value = float(code) * scale in fp32.

Everything is written from the formats' definitions with integer/bit
arithmetic on numpy arrays; tests pin it against torch's CPU casts.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def bf16_rne(x) -> np.ndarray:
    """fp32 -> bf16 (round to nearest, ties to even), returned as float32 values."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(f)
    out[nan] = np.nan
    return out


def _round_half_even(v: np.ndarray) -> np.ndarray:
    return np.round(v)  # numpy rounds halves to even


def e4m3_rne(x) -> np.ndarray:
    """fp32 values -> nearest e4m3fn value (ties to even, saturate at +-448), as float64.

    Representable magnitudes: 0, k * 2^-9 for k = 1..7 (subnormal), and
    (1 + m/8) * 2^e for e = -6..8, m = 0..7, except (1 + 7/8) * 2^8 (= 480, the NaN code).
    """
    v = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.sign(v)
    a = np.abs(v)
    out = np.empty_like(a)
    sub = a < 2.0 ** -6
    out[sub] = _round_half_even(a[sub] / 2.0 ** -9) * 2.0 ** -9
    nrm = ~sub
    if np.any(nrm):
        _, e2 = np.frexp(a[nrm])  # a = m * 2^e2 with m in [0.5, 1)
        e = e2.astype(np.int64) - 1  # a in [2^e, 2^(e+1))
        ulp = np.ldexp(1.0, e - 3)
        out[nrm] = _round_half_even(a[nrm] / ulp) * ulp
    out = np.minimum(out, E4M3_MAX)
    out = sign * out
    out[np.isnan(v)] = np.nan
    return out


def e4m3_rows(S_f32: np.ndarray):
    """Per-row scaled e4m3 copy of S[..., N] (fp32 values).

    Returns (codes as float64 values in [-448, 448], scale[...] as fp32 values).
    """
    S = np.asarray(S_f32, dtype=np.float32)
    amax = np.max(np.abs(S), axis=-1)
    scale = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32), np.float32(1.0))
    scale = scale.astype(np.float32)
    ratio = (S / scale[..., None]).astype(np.float32)
    return e4m3_rne(ratio), scale


def dequant_e4m3_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """float(code) * scale in fp32, returned as float64."""
    return (codes.astype(np.float32) * np.asarray(scale, np.float32)[..., None]).astype(
        np.float32).astype(np.float64)


def read_copy(S: np.ndarray, dtype: str) -> np.ndarray:
    """The dequantised read copy the outputs see, from state values S (float64).

    "f64": S itself (the exact algebra, no storage rounding).  Otherwise the
    checkpoint is held in fp32, so S is first rounded to fp32; then "f32": as is;
    "bf16": RNE to bf16; "fp8": per-row scaled e4m3.
    """
    if dtype == "f64":
        return np.array(S, dtype=np.float64, copy=True)
    s32 = np.asarray(S, dtype=np.float32)
    if dtype == "f32":
        return s32.astype(np.float64)
    if dtype == "bf16":
        return bf16_rne(s32).astype(np.float64)
    if dtype == "fp8":
        codes, scale = e4m3_rows(s32)
        return dequant_e4m3_rows(codes, scale)
    raise ValueError(dtype)
