"""The five workloads at full size, in the launch configuration the benchmark
times, with every row (R4, inverse) and every token (R3 + KV) checked against
the oracle:

1. tiny: 64 x 256, channel 7 = 60, clip 1.0 -- parity, MSE rotated vs direct.
2. R4 prefill: 8192 x 16384 SwiGLU-like, 0.1 % channels x100, +-1 diagonal, clip 0.9.
3. R3 + KV: batch 4 x seq 4096, 32/8 heads, d = 128, outlier dims x50, clip 0.95.
4. decode: 32 x {4096, 16384} Student-t(3), one channel x200 per row.
5. sweep: n = 2^7..2^15, 1 GiB of bf16 input each, forward and inverse.

The oracle's threaded batch paths produce every row's expected result; rows
that differ in any byte are re-run through the single-row oracle, which
supplies the pre-round values the rounding-tie exemption needs.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import bf16_dev_to_bits, to_dev_bf16, to_dev_signs
from tests.test_gpu_r3 import compare_all_tokens, run_r3

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
    parity.check_r4_bulk(orc, bits, 0.9, signs, q_np, s_np, what="R4 prefill")  # all 8192 rows
    check_rows(orc, bits, 0.9, signs, q_np, s_np, [0, bits.shape[0] - 1], method=1)  # explicit Sylvester sums


def test_config3_r3_kv(spin_gpu, orc):
    q, k, v, pos = synthetic.r3_kv()
    out = run_r3(spin_gpu, q, k, v, pos, 1e4, 0.95, 4096, 0)
    compare_all_tokens(orc, q, k, v, pos, 1e4, 0.95, out, 0)  # all 16384 tokens, every head


@pytest.mark.parametrize("n", [4096, 16384])
def test_config4_decode(spin_gpu, orc, n):
    bits = synthetic.decode(32, n)
    q, s = r4_dev(spin_gpu, to_dev_bf16(bits), 1.0, None)
    check_rows(orc, bits, 1.0, None, q.cpu().numpy(), s.cpu().numpy(), range(32))


def _inverse_all_rows(spin, orc, n, packed, scales, direct, x_dev, chunk_elems=1 << 24):
    """The inverse kernel on the oracle's codes and steps for every row, compared
    element by element (bf16 bound) with the oracle's inverse; returns the oracle
    chain's reconstruction MSE over all rows."""
    T = packed.shape[0]
    got = spin.dequant_hadamard_inverse(torch.from_numpy(packed).cuda(), n, torch.from_numpy(scales).cuda(),
                                        no_rotate=direct, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = max(1, chunk_elems // n)
    sq = 0.0
    for t0 in range(0, T, rows):
        t1 = min(T, t0 + rows)
        ref = orc.dequant_inverse_rows(packed[t0:t1], n, 0, scales[t0:t1].astype(np.float64), no_rotate=direct,
                                       threads=orc.max_threads())
        parity.check_bf16_bits(bf16_dev_to_bits(got[t0:t1]), ref, f"inverse n={n} direct={direct} rows {t0}..")
        xf = x_dev[t0:t1].double().cpu().numpy()
        sq += float(((ref - xf) ** 2).sum())
    del got
    return sq / (T * n)


@pytest.mark.parametrize("k", list(range(7, 16)))
def test_config5_sweep(spin_gpu, orc, k):
    n = 1 << k
    bits = synthetic.sweep(k)
    T = bits.shape[0]
    x = to_dev_bf16(bits)
    mse_gpu, mse_ref = {}, {}
    for direct in (False, True):
        # forward at full size: every row against the oracle's batch path
        q, s = r4_dev(spin_gpu, x, 1.0, None, direct)
        q_np, s_np = q.cpu().numpy(), s.cpu().numpy()
        _, packed, scales = parity.check_r4_bulk(orc, bits, 1.0, None, q_np, s_np, no_rotate=direct,
                                                 what=f"sweep n={n} direct={direct}")
        if not direct:
            check_rows(orc, bits, 1.0, None, q_np, s_np, [0, T - 1], direct, method=1)
        # inverse at full size on the GPU's own codes: the reconstruction bound holds on every row
        xr = spin_gpu.dequant_hadamard_inverse(q, n, s, no_rotate=direct, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        err = (xr.double() - x.double()).norm(dim=1)
        bound = np.sqrt(n) * s.double() / 2 * (1 + 1e-3) + xr.double().norm(dim=1) * 2.0 ** -8
        assert bool((err <= bound).all()), f"reconstruction bound, n={n} direct={direct}"
        mse_gpu[direct] = float(((xr.double() - x.double()) ** 2).mean().item())
        del q, s, xr, err, bound
        # inverse on the oracle's codes for every row: element parity
        mse_ref[direct] = _inverse_all_rows(spin_gpu, orc, n, packed, scales, direct, x)
        del packed, scales
    assert mse_ref[False] < mse_ref[True]  # rotating first lowers the reconstruction error
    ratio_gpu, ratio_ref = mse_gpu[False] / mse_gpu[True], mse_ref[False] / mse_ref[True]
    assert abs(ratio_gpu / ratio_ref - 1) < 2e-2
