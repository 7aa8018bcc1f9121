"""W4A4 GEMM on packed INT4 codes (spin_w4a4_gemm) vs the fp64 oracle: random codes at
shapes with ragged token tiles, fp32 and bf16 outputs; the pipeline the GEMM serves (the
R4 kernel's codes against weight rows baked by the same kernel); and the bench's full
size (8192 tokens x 4096 outputs x k = 14336) on sampled rows. The integer sum is exact
on both sides, so fp32 outputs differ from the oracle only by the two fp32 roundings of
s_x s_w and of its product with the sum."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_signs

pytestmark = pytest.mark.gpu

F32_REL = 2.0 ** -22  # two fp32 roundings


def random_operands(T, N, K, seed):
    rng = np.random.default_rng(seed)
    xq = rng.integers(0, 256, (T, K // 2), dtype=np.uint8)
    wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    xs = (rng.random(T) * 0.05 + 1e-3).astype(np.float32)
    ws = (rng.random(N) * 0.05 + 1e-3).astype(np.float32)
    return xq, xs, wq, ws


def gpu_gemm(spin, xq, xs, wq, ws, out_dtype):
    dev = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (xq, xs, wq, ws)]
    out = spin.w4a4_gemm(*dev, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out


def check_f32(got, ref, what):
    err = np.abs(got - ref)
    bad = err > F32_REL * np.abs(ref)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err, 0)), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} outputs off, e.g. {i}: gpu {got[i]} oracle {ref[i]}")


@pytest.mark.parametrize("T,N,K", [(1, 256, 128), (37, 256, 384), (128, 512, 1024), (129, 768, 256),
                                   (300, 256, 2048)])
def test_w4a4_random_codes_vs_oracle(spin_gpu, orc, T, N, K):
    xq, xs, wq, ws = random_operands(T, N, K, T + N + K)
    ref = orc.w4a4_gemm(xq, xs, wq, ws, threads=orc.max_threads())
    got = gpu_gemm(spin_gpu, xq, xs, wq, ws, torch.float32).cpu().numpy().astype(np.float64)
    check_f32(got, ref, f"W4A4 fp32 T={T} N={N} K={K}")
    got16 = gpu_gemm(spin_gpu, xq, xs, wq, ws, torch.bfloat16).float().cpu().numpy().astype(np.float64)
    parity.check_bf16(got16, ref, f"W4A4 bf16 T={T} N={N} K={K}")
    assert spin_gpu.device_status() == 0


def test_w4a4_extreme_codes(spin_gpu, orc):
    """Every code -8 against every code -8 and 7 (the largest sums), and zero rows."""
    T, N, K = 130, 256, 4096
    xq = np.full((T, K // 2), 0x88, np.uint8)
    xq[5] = 0
    wq = np.where(np.arange(N)[:, None] % 2 == 0, 0x88, 0x77).astype(np.uint8).repeat(K // 2, axis=1)
    xs = np.full(T, 0.01, np.float32)
    ws = np.full(N, 0.02, np.float32)
    ref = orc.w4a4_gemm(xq, xs, wq, ws)
    got = gpu_gemm(spin_gpu, xq, xs, wq, ws, torch.float32).cpu().numpy().astype(np.float64)
    check_f32(got, ref, "extreme codes")
    assert np.all(got[5] == 0.0)


def test_w4a4_pipeline_on_r4_codes(spin_gpu, orc):
    """Activations through the R4 kernel and weight rows baked by the same kernel (same
    diagonal, clip 1.0): the GEMM on those GPU codes matches the oracle's GEMM on them, and
    the codes themselves are the oracle's R4 rows."""
    T, N, K = 300, 512, 2048
    x_bits = synthetic.sweep(11, tokens=T, seed=61)
    w = np.random.default_rng(62).standard_normal((N, K)) / np.sqrt(K)
    w_bits = orc.f64_to_bf16(w)
    sg = synthetic.sign_bits(K, 63)
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
    xq, xs = spin_gpu.hadamard_quant_int4(to_dev(x_bits), 1.0, to_dev_signs(sg))
    wq, ws = spin_gpu.hadamard_quant_int4(to_dev(w_bits), 1.0, to_dev_signs(sg))
    y = spin_gpu.w4a4_gemm(xq, xs, wq, ws, out_dtype=torch.float32)
    torch.cuda.synchronize()
    xq_h, xs_h, wq_h, ws_h = (a.cpu().numpy() for a in (xq, xs, wq, ws))
    ref = orc.w4a4_gemm(xq_h, xs_h, wq_h, ws_h, threads=orc.max_threads())
    check_f32(y.cpu().numpy().astype(np.float64), ref, "pipeline GEMM")
    oq, os_ = orc.bake_weights(w_bits, signs=sg, threads=orc.max_threads())
    assert np.max(np.abs(os_.astype(np.float64) / ws_h - 1.0)) < 1e-5  # the R4 steps' tolerance
    assert np.mean(oq != wq_h) < 1e-3  # codes agree up to the rounding-tie band


def test_w4a4_full_size_sampled_rows(spin_gpu, orc):
    """The bench's size, 8192 tokens x 4096 outputs x k = 14336 (every output tile, the
    full contraction), compared on sampled rows from several token tiles."""
    T, N, K = 8192, 4096, 14336
    xq, xs, wq, ws = random_operands(T, N, K, 99)
    got = gpu_gemm(spin_gpu, xq, xs, wq, ws, torch.float32)
    rows = np.array([0, 1, 127, 128, 4095, 6000, 8190, 8191])
    ref = orc.w4a4_gemm(xq[rows], xs[rows], wq, ws, threads=orc.max_threads())
    check_f32(got[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64), ref, "full size")
    assert spin_gpu.device_status() == 0


def test_w4a4_zero_tokens_and_errors(spin_gpu):
    xq = torch.zeros((0, 64), dtype=torch.uint8, device="cuda")
    xs = torch.zeros((0,), dtype=torch.float32, device="cuda")
    wq = torch.zeros((256, 64), dtype=torch.uint8, device="cuda")
    ws = torch.ones((256,), dtype=torch.float32, device="cuda")
    assert spin_gpu.w4a4_gemm(xq, xs, wq, ws).shape == (0, 256)
    with pytest.raises(spin_gpu.SpinError):
        spin_gpu.w4a4_gemm(torch.zeros((4, 64), dtype=torch.uint8, device="cuda"),
                           torch.ones((4,), dtype=torch.float32, device="cuda"), wq[:200].contiguous(), ws[:200])
