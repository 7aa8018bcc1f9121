"""ctypes wrapper around the fp64 CPU oracle (oracle/spin_oracle.c).

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  Nothing in the CUDA
library imports this package, and this package imports nothing from it.

The arithmetic lives in the C file; this module only moves numpy arrays in
and out of it.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

NO_ROTATE = 1
METHOD_FWHT = 0
METHOD_EXPLICIT = 1

_lib = None

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_i8p = np.ctypeslib.ndpointer(dtype=np.int8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    L = C.CDLL(path)
    vp = C.c_void_p
    L.orc_rounding_is_nearest.restype = C.c_int
    L.orc_rne.argtypes = [C.c_double]
    L.orc_rne.restype = C.c_double
    L.orc_bf16_to_f64.argtypes = [C.c_uint16]
    L.orc_bf16_to_f64.restype = C.c_double
    L.orc_f64_to_bf16.argtypes = [C.c_double]
    L.orc_f64_to_bf16.restype = C.c_uint16
    L.orc_f16_to_f64.argtypes = [C.c_uint16]
    L.orc_f16_to_f64.restype = C.c_double
    L.orc_f64_to_f16.argtypes = [C.c_double]
    L.orc_f64_to_f16.restype = C.c_uint16
    L.orc_sylvester_matrix.argtypes = [C.c_int, _i8p]
    L.orc_hadamard_entry.argtypes = [C.c_uint64, C.c_uint64]
    L.orc_hadamard_entry.restype = C.c_int
    L.orc_wht_explicit.argtypes = [_dp, C.c_int, _dp]
    L.orc_fwht.argtypes = [_dp, C.c_int]
    L.orc_rotate.argtypes = [_dp, C.c_int, vp, C.c_int, _dp]
    L.orc_rotate.restype = C.c_int
    L.orc_quant_sym_int4.argtypes = [_dp, C.c_int, C.c_double, vp, _i8p]
    L.orc_quant_sym_int4.restype = C.c_double
    L.orc_legendre.argtypes = [C.c_int64, C.c_int64]
    L.orc_legendre.restype = C.c_int
    L.orc_paley_type.argtypes = [C.c_int]
    L.orc_paley_type.restype = C.c_int
    L.orc_paley_hadamard.argtypes = [C.c_int, _i8p]
    L.orc_paley_hadamard.restype = C.c_int
    L.orc_rotate_kron.argtypes = [_dp, C.c_int, C.c_int, vp, _dp]
    L.orc_rotate_kron.restype = C.c_int
    L.orc_r4_row_kron.argtypes = [_u16p, C.c_int, C.c_int, C.c_double, vp, vp, vp, _i8p, vp, vp]
    L.orc_r4_row_kron.restype = C.c_int
    L.orc_r4_rows_kron.argtypes = [_u16p, C.c_int64, C.c_int, C.c_int, C.c_double, vp, _u8p,
                                   np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS"), C.c_int]
    L.orc_r4_rows_kron.restype = C.c_int
    L.orc_quant_sym_int8.argtypes = [_dp, C.c_int, C.c_double, vp, _i8p]
    L.orc_quant_sym_int8.restype = C.c_double
    L.orc_r4_row_int8.argtypes = [_u16p, C.c_int, C.c_double, vp, C.c_uint32, C.c_int, vp, vp, _i8p,
                                  vp, vp]
    L.orc_r4_row_int8.restype = C.c_int
    L.orc_quant_asym_int4.argtypes = [_dp, C.c_int, C.c_double, vp, _u8p,
                                      C.POINTER(C.c_uint16), C.POINTER(C.c_uint16)]
    L.orc_quant_asym_int4_at.argtypes = [_dp, C.c_int, C.c_double, C.c_uint16, vp, _u8p,
                                         C.POINTER(C.c_uint16)]
    L.orc_quant_asym_int4_at.restype = C.c_uint16
    L.orc_asym_codes_at.argtypes = [_dp, C.c_int, C.c_double, C.c_uint16, C.c_double, vp, _u8p]
    L.orc_asym_codes_at.restype = C.c_double
    L.orc_asym_unrounded_scale.argtypes = [_dp, C.c_int, C.c_double]
    L.orc_asym_unrounded_scale.restype = C.c_double
    L.orc_pack_nibbles.argtypes = [_i32p, C.c_int, _u8p]
    L.orc_unpack_nibbles.argtypes = [_u8p, C.c_int, C.c_int, _i32p]
    L.orc_r4_row.argtypes = [_u16p, C.c_int, C.c_double, vp, C.c_uint32, C.c_int,
                             vp, vp, vp, _u8p, C.POINTER(C.c_double), C.POINTER(C.c_float)]
    L.orc_r4_row.restype = C.c_int
    L.orc_r4_rows.argtypes = [_u16p, C.c_int64, C.c_int, C.c_double, vp, C.c_uint32, _u8p,
                              np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS"), C.c_int]
    L.orc_r4_rows.restype = C.c_int
    L.orc_w4a4_gemm.argtypes = [_u8p, _f32p, C.c_int64, _u8p, _f32p, C.c_int, C.c_int, _dp, C.c_int]
    L.orc_w4a4_gemm.restype = C.c_int
    L.orc_max_threads.restype = C.c_int
    L.orc_rope_half.argtypes = [_dp, C.c_int, C.c_double, C.c_double]
    L.orc_r3_token.argtypes = [_u16p, _u16p, _u16p, C.c_double, C.c_double, C.c_int, C.c_int,
                               C.c_int, C.c_double, vp, _u16p, vp, vp, vp, _u8p, _u8p,
                               _u16p, _u16p, _u16p, _u16p]
    L.orc_r3_token.restype = C.c_int
    L.orc_r3_batch.argtypes = [_u16p, _u16p, _u16p, _i32p, C.c_double, C.c_int, C.c_int, C.c_int,
                               C.c_int, C.c_int, C.c_double, _u16p, _u8p, _u8p, _u16p, _u16p,
                               _u16p, _u16p, C.c_int, C.c_int, C.c_int]
    L.orc_r3_batch.restype = C.c_int
    L.orc_dequant_inverse_row.argtypes = [_u8p, C.c_int, C.c_int, C.c_double, C.c_double, vp,
                                          C.c_uint32, C.c_int, _dp]
    L.orc_dequant_inverse_row.restype = C.c_int
    L.orc_dequant_inverse_rows.argtypes = [_u8p, C.c_int64, C.c_int, C.c_int, _dp, vp, vp, C.c_uint32, _dp,
                                           C.c_int]
    L.orc_dequant_inverse_rows.restype = C.c_int
    L.orc_decode_attention_batch.argtypes = [_u16p, _u8p, _u8p, _u16p, _u16p, _u16p, _u16p, _i32p, C.c_int,
                                             C.c_int, C.c_int, C.c_int, C.c_int, C.c_double, _dp, C.c_int]
    L.orc_decode_attention_batch.restype = C.c_int
    L.orc_rmsnorm.argtypes = [_dp, C.c_int, C.c_double, _dp]
    L.orc_mse.argtypes = [_dp, _dp, C.c_int64]
    L.orc_mse.restype = C.c_double
    if not L.orc_rounding_is_nearest():
        raise RuntimeError("oracle requires round-to-nearest floating-point mode")
    _lib = L
    return L


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _signs(signs):
    if signs is None:
        return None
    s = np.ascontiguousarray(signs, dtype=np.uint32)
    return s


# ---------------------------------------------------------------- converters
def bf16_to_f64(bits) -> np.ndarray:
    L = lib()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([L.orc_bf16_to_f64(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def f64_to_bf16(x) -> np.ndarray:
    L = lib()
    a = np.asarray(x, dtype=np.float64)
    return np.array([L.orc_f64_to_bf16(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


def f16_to_f64(bits) -> np.ndarray:
    L = lib()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([L.orc_f16_to_f64(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def f64_to_f16(x) -> np.ndarray:
    L = lib()
    a = np.asarray(x, dtype=np.float64)
    return np.array([L.orc_f64_to_f16(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


def rne(v: float) -> float:
    return lib().orc_rne(float(v))


# ---------------------------------------------------------------- Hadamard
def sylvester_matrix(n: int) -> np.ndarray:
    H = np.zeros((n, n), dtype=np.int8)
    lib().orc_sylvester_matrix(n, H)
    return H


def hadamard_entry(i: int, j: int) -> int:
    return lib().orc_hadamard_entry(i, j)


def wht_explicit(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib().orc_wht_explicit(x, x.size, y)
    return y


def fwht(x) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    lib().orc_fwht(y, y.size)
    return y


def rotate(x, signs=None, method=METHOD_FWHT) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    s = _signs(signs)
    y = np.empty_like(x)
    rc = lib().orc_rotate(x, x.size, _ptr(s), method, y)
    if rc:
        raise ValueError(f"orc_rotate failed ({rc})")
    return y


# ---------------------------------------------------------------- quantisers
def quant_sym_int4(y, clip):
    y = np.ascontiguousarray(y, dtype=np.float64)
    pre = np.empty_like(y)
    codes = np.empty(y.size, dtype=np.int8)
    s = lib().orc_quant_sym_int4(y, y.size, float(clip), _ptr(pre), codes)
    return s, pre, codes


def quant_sym_int8(y, clip):
    y = np.ascontiguousarray(y, dtype=np.float64)
    pre = np.empty_like(y)
    codes = np.empty(y.size, dtype=np.int8)
    s = lib().orc_quant_sym_int8(y, y.size, float(clip), _ptr(pre), codes)
    return s, pre, codes


def quant_asym_int4(x, clip):
    x = np.ascontiguousarray(x, dtype=np.float64)
    pre = np.empty_like(x)
    codes = np.empty(x.size, dtype=np.uint8)
    s16 = C.c_uint16()
    z16 = C.c_uint16()
    lib().orc_quant_asym_int4(x, x.size, float(clip), _ptr(pre), codes, C.byref(s16), C.byref(z16))
    return codes, int(s16.value), int(z16.value), pre


def quant_asym_int4_at(x, clip, s16):
    """Codes and zero point of an asymmetric group for the given fp16 step pattern.
    Returns (codes, s16 used, z16, pre)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    pre = np.empty_like(x)
    codes = np.empty(x.size, dtype=np.uint8)
    z16 = C.c_uint16()
    used = lib().orc_quant_asym_int4_at(x, x.size, float(clip), int(s16), _ptr(pre), codes, C.byref(z16))
    return codes, int(used), int(z16.value), pre


def asym_codes_at(x, clip, s16, z):
    """Codes for the given fp16 step pattern and integer zero point; also the zero
    point before rounding (-lo/s). Returns (codes, zero_pre, pre)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    pre = np.empty_like(x)
    codes = np.empty(x.size, dtype=np.uint8)
    zpre = lib().orc_asym_codes_at(x, x.size, float(clip), int(s16), float(z), _ptr(pre), codes)
    return codes, float(zpre), pre


def asym_unrounded_scale(x, clip) -> float:
    x = np.ascontiguousarray(x, dtype=np.float64)
    return lib().orc_asym_unrounded_scale(x, x.size, float(clip))


def pack_nibbles(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.int32)
    out = np.empty(c.size // 2, dtype=np.uint8)
    lib().orc_pack_nibbles(c, c.size, out)
    return out


def unpack_nibbles(packed, n, signed) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.empty(n, dtype=np.int32)
    lib().orc_unpack_nibbles(p, n, 1 if signed else 0, out)
    return out


# ---------------------------------------------------------------- R4
def r4_row(x_bits, clip, signs=None, no_rotate=False, method=METHOD_FWHT):
    """One token through the R4 path; returns a dict of every intermediate."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n = x.size
    y = np.empty(n, dtype=np.float64)
    pre = np.empty(n, dtype=np.float64)
    codes = np.empty(n, dtype=np.int8)
    packed = np.empty(n // 2, dtype=np.uint8)
    s64 = C.c_double()
    s32 = C.c_float()
    s = _signs(signs)
    rc = lib().orc_r4_row(x, n, float(clip), _ptr(s), NO_ROTATE if no_rotate else 0, method,
                          _ptr(y), _ptr(pre), _ptr(codes), packed, C.byref(s64), C.byref(s32))
    if rc:
        raise ValueError(f"orc_r4_row failed ({rc})")
    return dict(y=y, pre=pre, codes=codes, packed=packed, scale64=s64.value,
                scale32=np.float32(s32.value))


def r4_row_int8(x_bits, clip, signs=None, no_rotate=False, method=METHOD_FWHT):
    """One token through the R4 path with per-token INT8 codes."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n = x.size
    y = np.empty(n, dtype=np.float64)
    pre = np.empty(n, dtype=np.float64)
    codes = np.empty(n, dtype=np.int8)
    s64 = C.c_double()
    s32 = C.c_float()
    s = _signs(signs)
    rc = lib().orc_r4_row_int8(x, n, float(clip), _ptr(s), NO_ROTATE if no_rotate else 0, method,
                               _ptr(y), _ptr(pre), codes, C.byref(s64), C.byref(s32))
    if rc:
        raise ValueError(f"orc_r4_row_int8 failed ({rc})")
    return dict(y=y, pre=pre, codes=codes, scale64=s64.value, scale32=np.float32(s32.value))


def max_threads() -> int:
    """Threads the oracle's batch loop uses by default (the host's cores)."""
    return int(lib().orc_max_threads())


# ---------------------------------------------------------------- n = m * 2^k
def legendre(a, q) -> int:
    return int(lib().orc_legendre(int(a), int(q)))


def paley_type(m) -> int:
    """1 or 2 when Paley's construction gives a Hadamard matrix of order m, else 0."""
    return int(lib().orc_paley_type(int(m)))


def paley_hadamard(m) -> np.ndarray:
    H = np.empty((m, m), dtype=np.int8)
    rc = lib().orc_paley_hadamard(int(m), H)
    if rc:
        raise ValueError(f"no Paley Hadamard matrix of order {m}")
    return H


def rotate_kron(x, m, signs=None) -> np.ndarray:
    """(H_m (x) H_b) D x / sqrt(n) for a row of n = m b values (b a power of two)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    s = _signs(signs)
    rc = lib().orc_rotate_kron(x, int(m), x.size // int(m), _ptr(s), y)
    if rc:
        raise ValueError(f"orc_rotate_kron failed ({rc})")
    return y


def r4_row_kron(x_bits, m, clip, signs=None):
    """One token of n = m b values through the Kronecker rotation and INT4 quantiser."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n = x.size
    y = np.empty(n, dtype=np.float64)
    pre = np.empty(n, dtype=np.float64)
    codes = np.empty(n, dtype=np.int8)
    s64 = C.c_double()
    s32 = C.c_float()
    s = _signs(signs)
    rc = lib().orc_r4_row_kron(x, int(m), n // int(m), float(clip), _ptr(s), _ptr(y), _ptr(pre), codes,
                               C.byref(s64), C.byref(s32))
    if rc:
        raise ValueError(f"orc_r4_row_kron failed ({rc})")
    return dict(y=y, pre=pre, codes=codes, scale64=s64.value, scale32=np.float32(s32.value))


def r4_rows_kron(x_bits, m, clip, signs=None, threads=1):
    """Rows [T, n = m b] through the Kronecker rotation and INT4 quantiser over
    `threads` OpenMP threads: (packed codes [T, n/2], fp32 steps [T])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    T, n = x.shape
    packed = np.empty((T, n // 2), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float32)
    rc = lib().orc_r4_rows_kron(x, T, int(m), n // int(m), float(clip), _ptr(_signs(signs)), packed, scales,
                                int(threads))
    if rc:
        raise ValueError(f"orc_r4_rows_kron failed ({rc})")
    return packed, scales


def r4_rows(x_bits, clip, signs=None, no_rotate=False, threads=1):
    """Rows [T, n] through the R4 path with the fast transform, over `threads`
    OpenMP threads (rows are independent; the results do not depend on it)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    T, n = x.shape
    packed = np.empty((T, n // 2), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float32)
    s = _signs(signs)
    rc = lib().orc_r4_rows(x, T, n, float(clip), _ptr(s), NO_ROTATE if no_rotate else 0,
                           packed, scales, int(threads))
    if rc:
        raise ValueError(f"orc_r4_rows failed ({rc})")
    return packed, scales


# ---------------------------------------------------------------- W4A4 GEMM
def bake_weights(w_bits, signs=None, clip=1.0, threads=1):
    """Offline weight baking: each output row w_o of W [n_out, k] (bf16 bits) becomes a
    row of W R^T = (R w_o)^T with R = H D / sqrt(k), the rotation the activations get
    online, quantised per output channel by the same symmetric INT4 rule ("SpinQuant
    Guide", "Production Engineering and Cluster Deployment Best Practices": compute
    W R^T offline, quantise it and pack INT4 nibbles). Returns (codes [n_out, k/2],
    scales [n_out])."""
    return r4_rows(w_bits, clip, signs=signs, threads=threads)


def w4a4_gemm(xq, xs, wq, ws, threads=1) -> np.ndarray:
    """y [tokens, n_out] = (s_x q_x)(s_w q_w)^T from packed INT4 codes ("SpinQuant Guide",
    "End-to-End Implementation": the quantised output is the product of the dequantised
    activations and weights), exact integer sums scaled once in fp64."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    xs = np.ascontiguousarray(xs, dtype=np.float32)
    ws = np.ascontiguousarray(ws, dtype=np.float32)
    T, kh = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != kh or xs.shape != (T,) or ws.shape != (N,):
        raise ValueError("w4a4_gemm: shapes do not match")
    y = np.empty((T, N), dtype=np.float64)
    if lib().orc_w4a4_gemm(xq, xs, T, wq, ws, N, 2 * kh, y, int(threads)):
        raise ValueError("orc_w4a4_gemm failed")
    return y


# ---------------------------------------------------------------- R3
def rope_half(x, pos, theta) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    lib().orc_rope_half(y, y.size, float(pos), float(theta))
    return y


def r3_token(q_bits, k_bits, v_bits, pos, theta, clip):
    """One token: q [hq, d], k/v [hkv, d] bf16 bit patterns."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    hq, d = q.shape
    hkv = k.shape[0]
    out = dict(
        q_f64=np.empty((hq, d)), q_bf16=np.empty((hq, d), dtype=np.uint16),
        k_f64=np.empty((hkv, d)), k_pre=np.empty((hkv, d)), v_pre=np.empty((hkv, d)),
        k_packed=np.empty((hkv, d // 2), dtype=np.uint8), v_packed=np.empty((hkv, d // 2), dtype=np.uint8),
        k_s=np.empty(hkv, dtype=np.uint16), k_z=np.empty(hkv, dtype=np.uint16),
        v_s=np.empty(hkv, dtype=np.uint16), v_z=np.empty(hkv, dtype=np.uint16))
    rc = lib().orc_r3_token(q, k, v, float(pos), float(theta), d, hq, hkv, float(clip),
                            _ptr(out["q_f64"]), out["q_bf16"], _ptr(out["k_f64"]),
                            _ptr(out["k_pre"]), _ptr(out["v_pre"]), out["k_packed"],
                            out["v_packed"], out["k_s"], out["k_z"], out["v_s"], out["v_z"])
    if rc:
        raise ValueError(f"orc_r3_token failed ({rc})")
    return out


def r3_batch(q_bits, k_bits, v_bits, pos, theta, clip, cache_len=None, cache_offset=0, threads=1):
    """The whole R3 batch into a cache of cache_len slots (token (b, s) at slot
    cache_offset + s; other slots stay zero); tokens spread over `threads`."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    p = np.ascontiguousarray(pos, dtype=np.int32)
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    L = cache_len if cache_len is not None else S + cache_offset
    out = dict(
        q_out=np.empty_like(q),
        k_cache=np.zeros((B, hkv, L, d // 2), dtype=np.uint8),
        v_cache=np.zeros((B, hkv, L, d // 2), dtype=np.uint8),
        k_scale=np.zeros((B, hkv, L), dtype=np.uint16), k_zero=np.zeros((B, hkv, L), dtype=np.uint16),
        v_scale=np.zeros((B, hkv, L), dtype=np.uint16), v_zero=np.zeros((B, hkv, L), dtype=np.uint16))
    rc = lib().orc_r3_batch(q, k, v, p, float(theta), d, B, S, hq, hkv, float(clip), out["q_out"],
                            out["k_cache"], out["v_cache"], out["k_scale"], out["k_zero"],
                            out["v_scale"], out["v_zero"], L, cache_offset, int(threads))
    if rc:
        raise ValueError(f"orc_r3_batch failed ({rc})")
    return out


# ---------------------------------------------------------------- inverse
def dequant_inverse_row(packed, n, mode, scale, zero=0.0, signs=None, no_rotate=False,
                        method=METHOD_FWHT) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.empty(n, dtype=np.float64)
    s = _signs(signs)
    rc = lib().orc_dequant_inverse_row(p, n, int(mode), float(scale), float(zero), _ptr(s),
                                       NO_ROTATE if no_rotate else 0, method, out)
    if rc:
        raise ValueError(f"orc_dequant_inverse_row failed ({rc})")
    return out


def dequant_inverse_rows(packed, n, mode, scale, zero=None, signs=None, no_rotate=False, threads=1):
    """Rows [rows, n/2] of codes -> [rows, n] fp64 (fast transform), rows over `threads`."""
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1, n // 2)
    rows = p.shape[0]
    sc = np.ascontiguousarray(scale, dtype=np.float64).ravel()
    z = None if zero is None else np.ascontiguousarray(zero, dtype=np.float64).ravel()
    if sc.size != rows or (z is not None and z.size != rows):
        raise ValueError("one scale (and zero) per row")
    out = np.empty((rows, n), dtype=np.float64)
    s = _signs(signs)
    rc = lib().orc_dequant_inverse_rows(p, rows, n, int(mode), sc, _ptr(z), _ptr(s),
                                        NO_ROTATE if no_rotate else 0, out, int(threads))
    if rc:
        raise ValueError(f"orc_dequant_inverse_rows failed ({rc})")
    return out


# ---------------------------------------------------------------- decode attention
def decode_attention(q_bits, cache, lens, softmax_scale=None, threads=1):
    """One decode step per batch row over the INT4 KV cache: q [B, hq, d] bf16
    patterns; cache dict of numpy arrays (k_cache, v_cache [B, hkv, L, d/2] uint8;
    k_scale, k_zero, v_scale, v_zero [B, hkv, L] fp16 patterns); lens [B] slots
    attended. Returns out [B, hq, d] fp64."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    B, hq, d = q.shape
    kc = np.ascontiguousarray(cache["k_cache"], dtype=np.uint8)
    hkv, L = kc.shape[1], kc.shape[2]
    arr = {k: np.ascontiguousarray(cache[k]).view(np.uint16) for k in ("k_scale", "k_zero", "v_scale", "v_zero")}
    ln = np.ascontiguousarray(np.broadcast_to(np.asarray(lens, dtype=np.int32), (B,)))
    out = np.empty((B, hq, d), dtype=np.float64)
    sc = 1.0 / np.sqrt(d) if softmax_scale is None else float(softmax_scale)
    rc = lib().orc_decode_attention_batch(q, kc, np.ascontiguousarray(cache["v_cache"], dtype=np.uint8),
                                          arr["k_scale"], arr["k_zero"], arr["v_scale"], arr["v_zero"], ln, B, hq,
                                          hkv, d, L, sc, out, int(threads))
    if rc:
        raise ValueError(f"orc_decode_attention_batch failed ({rc})")
    return out


# ---------------------------------------------------------------- self-test helpers
def rmsnorm(h, eps=0.0) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.float64)
    out = np.empty_like(h)
    lib().orc_rmsnorm(h, h.size, float(eps), out)
    return out


def mse(a, b) -> float:
    a = np.ascontiguousarray(a, dtype=np.float64).ravel()
    b = np.ascontiguousarray(b, dtype=np.float64).ravel()
    return lib().orc_mse(a, b, a.size)


LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspin_oracle.so")
