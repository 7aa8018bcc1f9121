"""The tensor-core R4 kernels vs the fp64 oracle, and vs the all-CUDA-core kernel
selected with SPIN_CUDA_CORES_ONLY:
  n = 128, 256: tokens as the MMA's M (128 tokens per MMA, the diagonal folded
    into the constant operand, H_2 of n = 256 in the epilogue);
  n = 1024 .. 16384: first H_128 Kronecker factor on tcgen05, second on CUDA
    cores; n = 512: two 64-row tokens per 128-row tile with H_64 (+) H_64 on
    tcgen05; n = 32768: H_2 and H_128 on tcgen05, without a sign diagonal.
Token counts leave partial MMA groups (256 / 128 / 64 tokens per group at n = 128 /
256 / 512; 32, 16, 8, 4 and 2 at n = 1024 .. 16384) and, at n = 512, odd tails that
split a two-token tile. At n = 32768 with sign_bits the CUDA-core kernel runs."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16, to_dev_signs

pytestmark = pytest.mark.gpu

SIZES = [128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768]


def run(spin, bits, clip, signs, cores_only=False):
    q, s = spin.hadamard_quant_int4(to_dev_bf16(bits), clip, to_dev_signs(signs), cuda_cores_only=cores_only,
                                    tensor_cores=not cores_only)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("N", SIZES)
@pytest.mark.parametrize("tokens", [1, 2, 3, 7, 9, 149, 300])
@pytest.mark.parametrize("clip,with_signs", [(1.0, False), (0.9, True)])
def test_tc_vs_oracle(spin_gpu, orc, N, tokens, clip, with_signs):
    bits = synthetic.r4_prefill(tokens=tokens, n=N, seed=50 + tokens)[0]
    signs = synthetic.sign_bits(N, 101) if with_signs else None
    q, s = run(spin_gpu, bits, clip, signs)
    codes = parity.unpack_signed(q, N)
    for t in range(tokens):
        r = orc.r4_row(bits[t], clip, signs=signs)
        parity.check_rel([s[t]], [r["scale64"]], 1e-5, f"scale row {t}")
        parity.check_codes(codes[t], r["codes"], r["pre"], f"codes row {t}")
    assert spin_gpu.device_status() == 0


@pytest.mark.parametrize("N", SIZES)
def test_tc_matches_cuda_core_kernel(spin_gpu, orc, N):
    bits, signs, _ = synthetic.r4_prefill(tokens=512, n=N, seed=9)
    if N == 32768:
        signs = None  # the tensor-core kernel takes no diagonal at this size
    q1, s1 = run(spin_gpu, bits, 0.9, signs)
    q2, s2 = run(spin_gpu, bits, 0.9, signs, cores_only=True)
    parity.check_rel(s1, s2, 1e-5, "tc vs cuda-core scales")
    c1, c2 = parity.unpack_signed(q1, N), parity.unpack_signed(q2, N)
    diff = np.nonzero((c1 != c2).any(axis=1))[0]
    for t in diff[:16]:  # any difference must be a rounding tie of the exact value
        r = orc.r4_row(bits[t], 0.9, signs=signs)
        parity.check_codes(c1[t], r["codes"], r["pre"], f"tc row {t}")
        parity.check_codes(c2[t], r["codes"], r["pre"], f"cuda-core row {t}")
    assert (c1 != c2).mean() < 1e-4


@pytest.mark.parametrize("N", SIZES)
def test_tc_special_rows(spin_gpu, orc, N):
    rows = [np.zeros(N, np.float32), np.full(N, 1.0, np.float32)]
    for j in sorted({0, 1, 127, 128 % N, N // 2 - 1, N - 1}):
        r = np.zeros(N, np.float32)
        r[j] = 60.0
        rows.append(r)
    rows.append(np.where(np.arange(N) % 3 == 0, 3.0e4, -2.0e4).astype(np.float32))
    bits = synthetic.to_bf16_bits(np.stack(rows))
    q, s = run(spin_gpu, bits, 1.0, None)
    codes = parity.unpack_signed(q, N)
    for t in range(len(rows)):
        r = orc.r4_row(bits[t], 1.0)
        parity.check_rel([s[t]], [r["scale64"]], 1e-5, f"scale row {t}")
        parity.check_codes(codes[t], r["codes"], r["pre"], f"codes row {t}")
    assert np.all(codes[0] == 0) and s[0] == np.float32(1e-8)
    for t in range(2, len(rows) - 1):
        assert np.all(np.abs(codes[t]) == 7)


@pytest.mark.parametrize("N", SIZES)
def test_tc_leaves_tail_untouched(spin_gpu, N):
    bits = synthetic.r4_prefill(tokens=5, n=N, seed=3)[0]
    out = torch.full((8, N // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((8,), -1.0, dtype=torch.float32, device="cuda")
    spin_gpu.hadamard_quant_int4(to_dev_bf16(bits), 1.0, out=out[:5], scales=sc[:5], tensor_cores=True)
    torch.cuda.synchronize()
    assert torch.all(out[5:] == 0xA5) and torch.all(sc[5:] == -1.0)
    assert torch.all(sc[:5] > 0)


@pytest.mark.parametrize("N,tokens", [(128, 149 * 256 + 77), (256, 149 * 128 + 77)])
@pytest.mark.parametrize("with_signs", [False, True])
def test_tc_small_n_many_groups(spin_gpu, orc, N, tokens, with_signs):
    """More MMA groups than resident blocks, so every block loops over several
    groups and both accumulators and every ring stage turn over."""
    bits, signs, _ = synthetic.r4_prefill(tokens=tokens, n=N, seed=17)
    if not with_signs:
        signs = None
    q1, s1 = run(spin_gpu, bits, 0.9, signs)
    q2, s2 = run(spin_gpu, bits, 0.9, signs, cores_only=True)
    parity.check_rel(s1, s2, 1e-5, "tc vs cuda-core scales")
    c1, c2 = parity.unpack_signed(q1, N), parity.unpack_signed(q2, N)
    rng = np.random.default_rng(N)
    sample = np.concatenate([rng.choice(tokens, 48, replace=False), [0, tokens - 1],
                             np.nonzero((c1 != c2).any(axis=1))[0][:16]])
    for t in sample:
        r = orc.r4_row(bits[t], 0.9, signs=signs)
        parity.check_rel([s1[t]], [r["scale64"]], 1e-5, f"scale row {t}")
        parity.check_codes(c1[t], r["codes"], r["pre"], f"tc row {t}")
    assert (c1 != c2).mean() < 1e-4
    assert spin_gpu.device_status() == 0
