"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the published acceptance bar for this path, with the readings
recorded in the design notes):
* INT4 codes are bit-exact, except where the oracle's pre-round value lies
  within 1e-3 of a code step from a .5 rounding boundary; there the two sides
  may differ by one code.
* fp32 scales within 1e-5 relative. fp16 scales and zero points are equal,
  except where the oracle's unrounded scale sits within 1e-6 relative of an
  fp16 rounding boundary (the GPU rounds its fp32 value, the oracle its fp64
  value; an fp32 evaluation of that step is within 3.3e-7 relative of the fp64
  one on the R3 workload). Such a group must carry the other fp16 neighbour,
  and its zero point and codes are compared with the oracle's for that step.
  The zero point is an INT4 code (-lo/s rounded): like a code, it may differ
  by one where the oracle's unrounded value lies within 1e-3 of a .5 boundary,
  and the group's codes are then compared with the oracle's for that zero point.
* bf16 outputs: |gpu - oracle| <= max(2e-2, 0.5 ulp_bf16(oracle) * (1 + 1e-3)).
  fp32 outputs: |gpu - oracle| <= 1e-5 * ||oracle row||_2.
"""
from __future__ import annotations

import numpy as np
import torch

TIE_BAND = 1e-3
F16_BOUNDARY_BAND = 1e-6


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


def bf16_bits_of(orc_f64: np.ndarray) -> np.ndarray:
    """bf16 bit patterns nearest (through fp32) to fp64 values: a fast prefilter
    for check_bf16_bits (an element equal to it is within the bf16 tolerance)."""
    f = torch.from_numpy(np.ascontiguousarray(orc_f64, dtype=np.float64).astype(np.float32))
    return f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def check_bf16_bits(gpu_bits: np.ndarray, orc: np.ndarray, what: str) -> int:
    """bf16 tolerance on every element; elements whose bits equal the nearest
    bf16 of the oracle value pass at once, the rest go through check_bf16.
    Returns the number of elements that differ from the nearest bf16."""
    gpu_bits = np.asarray(gpu_bits).view(np.uint16)
    diff = gpu_bits != bf16_bits_of(orc)
    if diff.any():
        check_bf16(bf16_bits_to_f64(gpu_bits[diff]), np.asarray(orc)[diff], what)
    return int(diff.sum())


def check_r4_bulk(orc, bits, clip, signs, q_gpu, s_gpu, no_rotate=False, what="r4", threads=None) -> int:
    """Every row of an R4 INT4 batch against the oracle: the oracle's threaded batch
    path gives packed codes and fp32 steps for all rows; steps within 1e-5; rows
    whose packed codes differ are re-run one by one for the rounding-tie exemption.
    Returns (rows with an exempt code difference, the oracle's packed codes, steps)."""
    threads = threads or orc.max_threads()
    n = bits.shape[1]
    packed, scales = orc.r4_rows(bits, clip, signs, no_rotate=no_rotate, threads=threads)
    check_rel(s_gpu, scales, 1e-5, f"{what} steps")
    rows = np.nonzero((np.asarray(q_gpu) != packed).any(axis=1))[0]
    for t in rows:
        r = orc.r4_row(bits[t], clip, signs=signs, no_rotate=no_rotate)
        check_codes(unpack_signed(q_gpu[t], n)[0], r["codes"], r["pre"], f"{what} codes row {t}")
    return len(rows), packed, scales


def check_kron_bulk(orc, bits, m, clip, signs, q_gpu, s_gpu, what="kron", threads=None) -> int:
    """Every row of an INT4 batch of n = m b against the oracle's threaded Kronecker
    batch path, as check_r4_bulk does for powers of two. Returns the rows re-run."""
    threads = threads or orc.max_threads()
    n = bits.shape[1]
    packed, scales = orc.r4_rows_kron(bits, m, clip, signs, threads=threads)
    check_rel(s_gpu, scales, 1e-5, f"{what} steps")
    rows = np.nonzero((np.asarray(q_gpu) != packed).any(axis=1))[0]
    for t in rows:
        r = orc.r4_row_kron(bits[t], m, clip, signs=signs)
        check_codes(unpack_signed(q_gpu[t], n)[0], r["codes"], r["pre"], f"{what} codes row {t}")
    return len(rows)


def other_f16_neighbour(orc, ref_s16: int, unrounded: float) -> int:
    """The fp16 pattern on the other side of `unrounded` from the oracle's
    rounded step (positive fp16 patterns are ordered like their values)."""
    return ref_s16 + 1 if unrounded > orc.f16_to_f64([ref_s16])[0] else ref_s16 - 1


def check_asym_group(orc, clip, gpu_packed, gpu_s, gpu_z, ref_packed, ref_s, ref_z, pre, values, what) -> int:
    """One asymmetric INT4 group. A different fp16 step is accepted only when the
    oracle's unrounded step lies within F16_BOUNDARY_BAND (relative) of the fp16
    midpoint between its rounding and the GPU's; a different zero point (an INT4
    code, -lo/s rounded) only when the oracle's unrounded zero point lies within the
    code tie band of a .5 boundary and the GPU's is its other rounding. The codes are
    then compared with the oracle's for the step and zero point the GPU used, both
    taken from the oracle's candidates. Returns 1 for a group on such a boundary."""
    excused = 0
    s16 = ref_s
    if gpu_s != ref_s:
        u = orc.asym_unrounded_scale(values, clip)
        other = other_f16_neighbour(orc, ref_s, u)
        mid = (orc.f16_to_f64([ref_s])[0] + orc.f16_to_f64([other])[0]) / 2
        assert gpu_s == other and abs(u - mid) <= F16_BOUNDARY_BAND * u, (
            f"{what}: step {gpu_s:#06x} vs oracle {ref_s:#06x} (unrounded {u!r}, fp16 midpoint {mid!r})")
        codes, _, z16, pre = orc.quant_asym_int4_at(values, clip, other)
        ref_packed, ref_z, s16 = orc.pack_nibbles(codes), z16, other
        excused = 1
    if gpu_z != ref_z:
        zr = orc.f16_to_f64([ref_z])[0]
        _, zpre, _ = orc.asym_codes_at(values, clip, s16, zr)
        alt = zr + (1.0 if zpre > zr else -1.0)
        assert near_half(np.array([zpre]))[0] and 0.0 <= alt <= 15.0 and gpu_z == orc.f64_to_f16([alt])[0], (
            f"{what}: zero {gpu_z:#06x} vs {ref_z:#06x} (unrounded {zpre!r})")
        codes, _, pre = orc.asym_codes_at(values, clip, s16, alt)
        ref_packed = orc.pack_nibbles(codes)
        excused = 1
    n = 2 * np.asarray(gpu_packed).size
    check_codes(unpack_unsigned(gpu_packed, n)[0], unpack_unsigned(ref_packed, n)[0], pre, what)
    return excused
