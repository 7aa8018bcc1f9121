"""Dequantise + inverse rotation (spin_dequant_hadamard_inverse) vs the fp64
oracle. Both sides receive the same codes and scales, produced by the oracle
(symmetric rows from the oracle's R4; asymmetric rows are random codes with
random fp16 scales and integer zero points)."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_signs

pytestmark = pytest.mark.gpu


def gpu_inverse(spin, packed, n, scale, zero, mode, signs, direct, out_dtype):
    codes = torch.from_numpy(np.ascontiguousarray(packed)).cuda()
    sc = torch.from_numpy(np.ascontiguousarray(scale)).cuda()
    zr = torch.from_numpy(np.ascontiguousarray(zero)).cuda() if zero is not None else None
    out = spin.dequant_hadamard_inverse(codes, n, sc, zr, mode=mode, signs=to_dev_signs(signs), no_rotate=direct,
                                        out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("k", [7, 8, 9, 11, 12, 14, 15])
@pytest.mark.parametrize("with_signs", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_sym_inverse(spin_gpu, orc, k, with_signs, out_dtype):
    n = 1 << k
    tokens = 37 if k <= 12 else 5
    bits = synthetic.sweep(k, tokens=tokens, seed=2000 + k)
    signs = synthetic.sign_bits(n, 7 + k) if with_signs else None
    packed = np.empty((tokens, n // 2), np.uint8)
    scales = np.empty(tokens, np.float32)
    for t in range(tokens):
        r = orc.r4_row(bits[t], 0.9, signs=signs)
        packed[t], scales[t] = r["packed"], r["scale32"]
    for direct in (False, True):
        got = gpu_inverse(spin_gpu, packed, n, scales, None, 0, signs, direct, out_dtype)
        ref = np.stack([orc.dequant_inverse_row(packed[t], n, 0, float(scales[t]), signs=signs, no_rotate=direct)
                        for t in range(tokens)])
        if out_dtype == torch.float32:
            parity.check_f32_rows(got, ref, f"sym inverse n={n}")
        else:
            parity.check_bf16(got, ref, f"sym inverse bf16 n={n}")


@pytest.mark.parametrize("k", [7, 10, 13])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_asym_inverse(spin_gpu, orc, k, out_dtype):
    n = 1 << k
    rows = 41
    rng = np.random.default_rng(k)
    codes = rng.integers(0, 16, size=(rows, n))
    packed = np.stack([orc.pack_nibbles(c) for c in codes])
    scale16 = orc.f64_to_f16(rng.uniform(0.01, 3.0, rows))
    zero16 = orc.f64_to_f16(rng.integers(0, 16, rows).astype(np.float64))
    for direct in (False, True):
        got = gpu_inverse(spin_gpu, packed, n, scale16.view(np.float16), zero16.view(np.float16), 1, None, direct,
                          out_dtype)
        s = orc.f16_to_f64(scale16)
        z = orc.f16_to_f64(zero16)
        ref = np.stack([orc.dequant_inverse_row(packed[t], n, 1, s[t], z[t], no_rotate=direct) for t in range(rows)])
        if out_dtype == torch.float32:
            parity.check_f32_rows(got, ref, f"asym inverse n={n}")
        else:
            parity.check_bf16(got, ref, f"asym inverse bf16 n={n}")


def test_inverse_of_forward_round_trip(spin_gpu, orc):
    """GPU forward then GPU inverse equals the oracle's round trip (same codes)."""
    n = 4096
    bits = synthetic.sweep(12, tokens=16, seed=5)
    signs = synthetic.sign_bits(n, 5)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    q, s = spin_gpu.hadamard_quant_int4(x, 1.0, to_dev_signs(signs))
    xr = spin_gpu.dequant_hadamard_inverse(q, n, s, signs=to_dev_signs(signs), out_dtype=torch.float32)
    torch.cuda.synchronize()
    q, s, xr = q.cpu().numpy(), s.cpu().numpy(), xr.cpu().numpy()
    xf = synthetic.bf16_bits_to_f32(bits).astype(np.float64)
    for t in range(16):
        r = orc.r4_row(bits[t], 1.0, signs=signs)
        ref = orc.dequant_inverse_row(r["packed"], n, 0, r["scale64"], signs=signs)
        # both reconstructions sit within sqrt(n) * step / 2 of the input
        assert np.linalg.norm(xr[t] - xf[t]) <= np.sqrt(n) * s[t] / 2 * (1 + 1e-4)
        assert abs(orc.mse(xr[t], xf[t]) / orc.mse(ref, xf[t]) - 1) < 5e-3


def test_kv_cache_rows(spin_gpu, orc):
    """The inverse reads a [B, hkv, L, d/2] cache as B*hkv*L rows of d codes."""
    B, H, L, d = 2, 3, 5, 128
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 16, size=(B * H * L, d))
    packed = np.stack([orc.pack_nibbles(c) for c in codes]).reshape(B, H, L, d // 2)
    s16 = orc.f64_to_f16(rng.uniform(0.05, 1, B * H * L)).reshape(B, H, L)
    z16 = orc.f64_to_f16(rng.integers(0, 16, B * H * L).astype(float)).reshape(B, H, L)
    got = gpu_inverse(spin_gpu, packed, d, s16.view(np.float16), z16.view(np.float16), 1, None, False, torch.float32)
    assert got.shape == (B, H, L, d)
    ref = np.stack([orc.dequant_inverse_row(packed.reshape(-1, d // 2)[i], d, 1, orc.f16_to_f64(s16.ravel()[i:i + 1])[0],
                                            orc.f16_to_f64(z16.ravel()[i:i + 1])[0]) for i in range(B * H * L)])
    parity.check_f32_rows(got.reshape(-1, d), ref, "kv rows")
