"""The five workloads at full size, in the launch configuration the benchmark
times, checked against the oracle on sampled rows/tokens (every row where the
workload is small):

1. tiny: 64 x 256, channel 7 = 60, clip 1.0 -- full parity, MSE rotated vs direct.
2. R4 prefill: 8192 x 16384 SwiGLU-like, 0.1 % channels x100, +-1 diagonal, clip 0.9.
3. R3 + KV: batch 4 x seq 4096, 32/8 heads, d = 128, outlier dims x50, clip 0.95.
4. decode: 32 x {4096, 16384} Student-t(3), one channel x200 per row.
5. sweep: n = 2^7..2^15, 1 GiB of bf16 input each, forward and inverse.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16, to_dev_signs
from tests.test_gpu_r3 import compare_tokens, run_r3

pytestmark = pytest.mark.gpu


def r4_dev(spin, x_dev, clip, signs_dev, direct=False):
    q, s = spin.hadamard_quant_int4(x_dev, clip, signs_dev, no_rotate=direct)
    torch.cuda.synchronize()
    return q, s


def check_rows(orc, bits, clip, signs, q_np, s_np, rows, direct=False, method=0):
    n = bits.shape[1]
    for t in rows:
        r = orc.r4_row(bits[t], clip, signs=signs, no_rotate=direct, method=method)
        parity.check_rel([s_np[t]], [r["scale64"]], 1e-5, f"scale row {t}")
        parity.check_codes(parity.unpack_signed(q_np[t], n)[0], r["codes"], r["pre"], f"codes row {t}")


def test_config1_tiny(spin_gpu, orc):
    bits = synthetic.tiny()
    x = to_dev_bf16(bits)
    xf = synthetic.bf16_bits_to_f32(bits).astype(np.float64)
    mse = {}
    for direct in (False, True):
        q, s = r4_dev(spin_gpu, x, 1.0, None, direct)
        check_rows(orc, bits, 1.0, None, q.cpu().numpy(), s.cpu().numpy(), range(64), direct)
        xr = spin_gpu.dequant_hadamard_inverse(q, 256, s, no_rotate=direct, out_dtype=torch.float32)
        torch.cuda.synchronize()
        mse[direct] = orc.mse(xr.cpu().numpy(), xf)
    ref = {}
    for direct in (False, True):
        acc = []
        for t in range(64):
            r = orc.r4_row(bits[t], 1.0, no_rotate=direct)
            acc.append(orc.dequant_inverse_row(r["packed"], 256, 0, r["scale64"], no_rotate=direct))
        ref[direct] = orc.mse(np.stack(acc), xf)
    ratio_gpu, ratio_ref = mse[False] / mse[True], ref[False] / ref[True]
    assert abs(ratio_gpu / ratio_ref - 1) < 1e-3
    assert ratio_ref < 0.2  # rotation cuts the error several-fold on this workload


def test_config2_prefill(spin_gpu, orc):
    bits, signs, _ = synthetic.r4_prefill()
    x = to_dev_bf16(bits)
    q, s = r4_dev(spin_gpu, x, 0.9, to_dev_signs(signs))
    q_np, s_np = q.cpu().numpy(), s.cpu().numpy()
    assert np.all(np.isfinite(s_np)) and np.all(s_np > 0)
    rows = np.random.default_rng(0).choice(bits.shape[0], 32, replace=False).tolist() + [0, bits.shape[0] - 1]
    check_rows(orc, bits, 0.9, signs, q_np, s_np, rows)
    check_rows(orc, bits, 0.9, signs, q_np, s_np, rows[:1], method=1)  # explicit Sylvester sums


def test_config3_r3_kv(spin_gpu, orc):
    q, k, v, pos = synthetic.r3_kv()
    out = run_r3(spin_gpu, q, k, v, pos, 1e4, 0.95, 4096, 0)
    rng = np.random.default_rng(1)
    toks = [(int(b), int(s)) for b, s in zip(rng.integers(0, 4, 12), rng.integers(0, 4096, 12))]
    toks += [(0, 0), (3, 4095)]
    skipped = compare_tokens(orc, q, k, v, pos, 1e4, 0.95, out, 0, toks)
    assert skipped <= 2


@pytest.mark.parametrize("n", [4096, 16384])
def test_config4_decode(spin_gpu, orc, n):
    bits = synthetic.decode(32, n)
    q, s = r4_dev(spin_gpu, to_dev_bf16(bits), 1.0, None)
    check_rows(orc, bits, 1.0, None, q.cpu().numpy(), s.cpu().numpy(), range(32))


@pytest.mark.parametrize("k", list(range(7, 16)))
def test_config5_sweep(spin_gpu, orc, k):
    n = 1 << k
    bits = synthetic.sweep(k)
    T = bits.shape[0]
    x = to_dev_bf16(bits)
    rows = sorted(set(np.random.default_rng(k).choice(T, 12, replace=False).tolist() + [0, T - 1]))
    xf = synthetic.bf16_bits_to_f32(bits[rows]).astype(np.float64)
    mse_gpu, mse_ref = {}, {}
    for direct in (False, True):
        # forward at full size; sampled rows against the oracle
        q, s = r4_dev(spin_gpu, x, 1.0, None, direct)
        q_np, s_np = q[rows].cpu().numpy(), s[rows].cpu().numpy()
        check_rows(orc, bits[rows], 1.0, None, q_np, s_np, range(len(rows)), direct)
        if not direct:
            check_rows(orc, bits[rows], 1.0, None, q_np, s_np, [0], direct, method=1)
        # inverse at full size on the GPU's own codes: the reconstruction bound holds
        xr = spin_gpu.dequant_hadamard_inverse(q, n, s, no_rotate=direct, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        xr_rows = xr[rows].float().cpu().numpy().astype(np.float64)
        for i in range(len(rows)):
            bound = np.sqrt(n) * s_np[i] / 2 * (1 + 1e-3) + np.linalg.norm(xr_rows[i]) * 2.0 ** -8
            assert np.linalg.norm(xr_rows[i] - xf[i]) <= bound
        mse_gpu[direct] = np.mean((xr_rows - xf) ** 2)
        # inverse on the oracle's codes for the sampled rows: element parity
        ref_codes, ref_scales, ref_out = [], [], []
        for i, t in enumerate(rows):
            r = orc.r4_row(bits[t], 1.0, no_rotate=direct)
            ref_codes.append(r["packed"])
            ref_scales.append(r["scale32"])
            ref_out.append(orc.dequant_inverse_row(r["packed"], n, 0, float(r["scale32"]), no_rotate=direct))
        got = spin_gpu.dequant_hadamard_inverse(torch.from_numpy(np.stack(ref_codes)).cuda(), n,
                                                torch.from_numpy(np.array(ref_scales, np.float32)).cuda(),
                                                no_rotate=direct, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        ref_out = np.stack(ref_out)
        parity.check_bf16(got.float().cpu().numpy().astype(np.float64), ref_out, f"inverse n={n} direct={direct}")
        mse_ref[direct] = np.mean((ref_out - xf) ** 2)
        del q, s, xr
    assert mse_ref[False] < mse_ref[True]  # rotating first lowers the reconstruction error
    ratio_gpu, ratio_ref = mse_gpu[False] / mse_gpu[True], mse_ref[False] / mse_ref[True]
    assert abs(ratio_gpu / ratio_ref - 1) < 2e-2
