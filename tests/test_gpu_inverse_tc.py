"""The tensor-core dequantise + inverse kernels vs the fp64 oracle, and vs the
all-CUDA-core kernel selected with SPIN_CUDA_CORES_ONLY. Codes are expanded to
exact fp16 integers; at n = 128 and 256 the rows are the MMA's M against a
constant H_128 (H_2 of n = 256 in the epilogue), at n = 512 .. 32768 the first
Kronecker factor (H_64 (+) H_64 at n = 512) runs on tcgen05 and the second in
registers, and rows of 64 bytes or more (bf16 from n = 4096, fp32 from 2048) leave
through TMA tensor stores from swizzled staging tiles. Both kernels transform
exact integers and scale once at the end, so their outputs must agree bit for
bit. Row counts leave partial MMA groups (128 rows per group at n = 128 and 256;
64 at n = 512, whose odd row counts split a two-row tile; 32, 16, 8, 4, 2 and 1 from
1024)."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_signs

pytestmark = pytest.mark.gpu

SIZES = [128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768]


def inverse(spin, packed, n, scale, zero, mode, signs, out_dtype, cores_only=False):
    codes = torch.from_numpy(np.ascontiguousarray(packed)).cuda()
    sc = torch.from_numpy(np.ascontiguousarray(scale)).cuda()
    zr = torch.from_numpy(np.ascontiguousarray(zero)).cuda() if zero is not None else None
    out = spin.dequant_hadamard_inverse(codes, n, sc, zr, mode=mode, signs=to_dev_signs(signs), out_dtype=out_dtype,
                                        cuda_cores_only=cores_only, tensor_cores=not cores_only)
    torch.cuda.synchronize()
    return out


def sym_rows(orc, n, rows, seed, signs):
    bits = synthetic.sweep(n.bit_length() - 1, tokens=rows, seed=seed)
    packed = np.empty((rows, n // 2), np.uint8)
    scales = np.empty(rows, np.float32)
    for t in range(rows):
        r = orc.r4_row(bits[t], 0.9, signs=signs)
        packed[t], scales[t] = r["packed"], r["scale32"]
    return packed, scales


@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("rows", [1, 3, 9, 37, 300])
@pytest.mark.parametrize("with_signs", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tc_sym_vs_oracle(spin_gpu, orc, n, rows, with_signs, out_dtype):
    signs = synthetic.sign_bits(n, 31 + rows) if with_signs else None
    packed, scales = sym_rows(orc, n, rows, 3000 + rows, signs)
    got = inverse(spin_gpu, packed, n, scales, None, 0, signs, out_dtype).float().cpu().numpy().astype(np.float64)
    ref = np.stack([orc.dequant_inverse_row(packed[t], n, 0, float(scales[t]), signs=signs) for t in range(rows)])
    if out_dtype == torch.float32:
        parity.check_f32_rows(got, ref, f"tc sym inverse n={n}")
    else:
        parity.check_bf16(got, ref, f"tc sym inverse bf16 n={n}")
    assert spin_gpu.device_status() == 0


@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tc_asym_vs_oracle(spin_gpu, orc, n, out_dtype):
    rows = 11
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 16, size=(rows, n))
    codes[0] = 15  # extreme rows: every code at the top, at the bottom
    codes[1] = 0
    packed = np.stack([orc.pack_nibbles(c) for c in codes])
    scale16 = orc.f64_to_f16(rng.uniform(0.01, 3.0, rows))
    zero16 = orc.f64_to_f16(rng.integers(0, 16, rows).astype(np.float64))
    zero16[0] = orc.f64_to_f16(np.array([0.0]))[0]
    zero16[1] = orc.f64_to_f16(np.array([15.0]))[0]
    got = inverse(spin_gpu, packed, n, scale16.view(np.float16), zero16.view(np.float16), 1, None, out_dtype)
    got = got.float().cpu().numpy().astype(np.float64)
    s, z = orc.f16_to_f64(scale16), orc.f16_to_f64(zero16)
    ref = np.stack([orc.dequant_inverse_row(packed[t], n, 1, s[t], z[t]) for t in range(rows)])
    if out_dtype == torch.float32:
        parity.check_f32_rows(got, ref, f"tc asym inverse n={n}")
    else:
        parity.check_bf16(got, ref, f"tc asym inverse bf16 n={n}")


@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("with_signs", [False, True])
def test_tc_matches_cuda_core_kernel(spin_gpu, orc, n, with_signs):
    rows = max(64, (1 << 21) // n) + 77
    rng = np.random.default_rng(n + 1)
    packed = rng.integers(0, 256, size=(rows, n // 2), dtype=np.uint8)
    scales = rng.uniform(0.001, 2.0, rows).astype(np.float32)
    signs = synthetic.sign_bits(n, 77) if with_signs else None
    for out_dtype in (torch.float32, torch.bfloat16):
        a = inverse(spin_gpu, packed, n, scales, None, 0, signs, out_dtype)
        b = inverse(spin_gpu, packed, n, scales, None, 0, signs, out_dtype, cores_only=True)
        assert torch.equal(a.view(torch.int16) if out_dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if out_dtype == torch.bfloat16 else b.view(torch.int32))


@pytest.mark.parametrize("n", SIZES)
def test_tc_leaves_tail_untouched(spin_gpu, orc, n):
    rows = 3
    packed, scales = sym_rows(orc, n, rows, 11, None)
    out = torch.full((rows + 2, n), -7.0, dtype=torch.float32, device="cuda")
    spin_gpu.dequant_hadamard_inverse(torch.from_numpy(packed).cuda(), n, torch.from_numpy(scales).cuda(),
                                      out=out[:rows], tensor_cores=True)
    torch.cuda.synchronize()
    assert torch.all(out[rows:] == -7.0)
    ref = np.stack([orc.dequant_inverse_row(packed[t], n, 0, float(scales[t])) for t in range(rows)])
    parity.check_f32_rows(out[:rows].cpu().numpy().astype(np.float64), ref, f"tc inverse n={n} into a slice")


@pytest.mark.parametrize("n", [128, 256, 512, 1024, 2048])
@pytest.mark.parametrize("mode", [0, 1])
def test_tc_small_n_many_groups(spin_gpu, orc, n, mode):
    """More 128-row groups than resident blocks (every block loops, every ring
    stage and both accumulators turn over), both code modes: bit-exact against
    the CUDA-core kernel, sampled rows against the oracle."""
    rows = 149 * 128 * 3 + 45
    rng = np.random.default_rng(n + mode)
    packed = rng.integers(0, 256, size=(rows, n // 2), dtype=np.uint8)
    if mode == 0:
        scales, zero = rng.uniform(0.001, 2.0, rows).astype(np.float32), None
    else:
        scales = orc.f64_to_f16(rng.uniform(0.01, 3.0, rows)).view(np.float16)
        zero = orc.f64_to_f16(rng.integers(0, 16, rows).astype(np.float64)).view(np.float16)
    signs = synthetic.sign_bits(n, 5)
    for out_dtype in (torch.float32, torch.bfloat16):
        a = inverse(spin_gpu, packed, n, scales, zero, mode, signs, out_dtype)
        b = inverse(spin_gpu, packed, n, scales, zero, mode, signs, out_dtype, cores_only=True)
        assert torch.equal(a.view(torch.int16) if out_dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if out_dtype == torch.bfloat16 else b.view(torch.int32))
    got = a.float().cpu().numpy().astype(np.float64)
    s = scales.astype(np.float64) if mode == 0 else orc.f16_to_f64(scales.view(np.uint16))
    z = None if mode == 0 else orc.f16_to_f64(zero.view(np.uint16))
    for t in list(rng.choice(rows, 24, replace=False)) + [0, rows - 1]:
        ref = orc.dequant_inverse_row(packed[t], n, mode, float(s[t]), 0.0 if z is None else float(z[t]),
                                      signs=signs)
        parity.check_bf16(got[t:t + 1], ref[None, :], f"tc inverse n={n} row {t}")
    assert spin_gpu.device_status() == 0
