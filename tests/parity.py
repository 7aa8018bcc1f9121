"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the published acceptance bar for this path, with the readings
recorded in the design notes):
* INT4 codes are bit-exact, except where the oracle's pre-round value lies
  within 1e-3 of a code step from a .5 rounding boundary; there the two sides
  may differ by one code.
* fp32 scales within 1e-5 relative. fp16 scales and zero points are equal,
  except where the oracle's unrounded scale sits within 1e-4 relative of an
  fp16 rounding boundary (the GPU rounds its fp32 value, the oracle its fp64
  value); such groups are counted and their codes are not compared.
* bf16 outputs: |gpu - oracle| <= max(2e-2, 0.5 ulp_bf16(oracle) * (1 + 1e-3)).
  fp32 outputs: |gpu - oracle| <= 1e-5 * ||oracle row||_2.
"""
from __future__ import annotations

import numpy as np

TIE_BAND = 1e-3


def unpack_signed(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1, n // 2)
    c = np.empty((p.shape[0], n), dtype=np.int32)
    c[:, 0::2] = p & 0xF
    c[:, 1::2] = p >> 4
    return np.where(c >= 8, c - 16, c)


def unpack_unsigned(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1, n // 2)
    c = np.empty((p.shape[0], n), dtype=np.int32)
    c[:, 0::2] = p & 0xF
    c[:, 1::2] = p >> 4
    return c


def near_half(pre: np.ndarray, band: float = TIE_BAND) -> np.ndarray:
    """True where pre lies within `band` of a k + 1/2 rounding boundary."""
    f = np.abs(pre - np.floor(pre) - 0.5)
    return f <= band


def check_codes(gpu: np.ndarray, orc: np.ndarray, pre: np.ndarray, what: str = "codes") -> int:
    """Assert code parity with the tie exemption; return the number of exempt mismatches."""
    gpu = np.asarray(gpu).ravel()
    orc = np.asarray(orc).ravel()
    pre = np.asarray(pre).ravel()
    bad = gpu != orc
    if not bad.any():
        return 0
    idx = np.nonzero(bad)[0]
    ok = near_half(pre[idx]) & (np.abs(gpu[idx] - orc[idx]) == 1)
    if not ok.all():
        j = idx[~ok][:8]
        raise AssertionError(f"{what}: {int((~ok).sum())} mismatches outside the tie band, e.g. at {j.tolist()}: "
                             f"gpu {gpu[j].tolist()} oracle {orc[j].tolist()} pre {pre[j].tolist()}")
    return int(bad.sum())


def check_rel(gpu, orc, rtol: float, what: str) -> None:
    gpu = np.asarray(gpu, dtype=np.float64).ravel()
    orc = np.asarray(orc, dtype=np.float64).ravel()
    err = np.abs(gpu - orc)
    lim = rtol * np.abs(orc)
    if not (err <= lim).all():
        j = np.nonzero(err > lim)[0][:8]
        raise AssertionError(f"{what}: rel error above {rtol} at {j.tolist()}: gpu {gpu[j].tolist()} "
                             f"oracle {orc[j].tolist()}")


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_bf16(gpu_f: np.ndarray, orc: np.ndarray, what: str) -> None:
    gpu_f = np.asarray(gpu_f, dtype=np.float64)
    orc = np.asarray(orc, dtype=np.float64)
    lim = np.maximum(2e-2, 0.5 * bf16_ulp(orc) * (1 + 1e-3))
    err = np.abs(gpu_f - orc)
    if not (err <= lim).all():
        j = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: bf16 error {err[j]} above {lim[j]} at {j} (gpu {gpu_f[j]}, oracle {orc[j]})")


def check_f32_rows(gpu: np.ndarray, orc: np.ndarray, what: str, rtol: float = 1e-5) -> None:
    gpu = np.asarray(gpu, dtype=np.float64)
    orc = np.asarray(orc, dtype=np.float64)
    norms = np.linalg.norm(orc, axis=-1, keepdims=True)
    err = np.abs(gpu - orc)
    if not (err <= rtol * np.maximum(norms, 1e-30)).all():
        r = np.unravel_index(np.argmax(err / np.maximum(norms, 1e-30)), err.shape)
        raise AssertionError(f"{what}: error {err[r]} above {rtol} x row norm {norms[r[:-1]]} at {r}")


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
