"""R4 with per-token INT8 codes (spin_hadamard_quant_int8) vs the fp64 oracle:
every supported n, on the CUDA-core kernel and on the tensor-core kernels
(n = 128, 256 and 2048 .. 32768; n = 32768 without a diagonal), ragged token
counts, clip 1.0 / 0.9, with and without the +-1 diagonal, direct quantisation,
special rows, and more MMA groups than resident blocks."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16, to_dev_signs

pytestmark = pytest.mark.gpu

VARIANTS = {"plain": (1.0, False, False), "clip_signs": (0.9, True, False), "direct": (1.0, False, True)}
TC_SIZES = (128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768)


def run(spin, bits, clip, signs, direct=False, path="default"):
    q, s = spin.hadamard_quant_int8(to_dev_bf16(bits), clip, to_dev_signs(signs), no_rotate=direct,
                                    cuda_cores_only=path == "cuda_cores", tensor_cores=path == "tensor_cores")
    torch.cuda.synchronize()
    return q.cpu().numpy().astype(np.int32), s.cpu().numpy()


def compare(orc, bits, clip, signs, direct, q, s, rows, what):
    for t in rows:
        r = orc.r4_row_int8(bits[t], clip, signs=signs, no_rotate=direct)
        parity.check_rel([s[t]], [r["scale64"]], 1e-5, f"{what}: scale row {t}")
        parity.check_codes(q[t], r["codes"], r["pre"], f"{what}: codes row {t}")


@pytest.mark.parametrize("k", list(range(7, 16)))
@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("path", ["cuda_cores", "tensor_cores"])
def test_int8_all_sizes(spin_gpu, orc, k, variant, path):
    clip, with_signs, direct = VARIANTS[variant]
    n = 1 << k
    if path == "tensor_cores" and (n not in TC_SIZES or direct or (n == 32768 and with_signs)):
        pytest.skip("no tensor-core kernel for this case (the dispatch runs the CUDA-core one)")
    signs = synthetic.sign_bits(n, 300 + k) if with_signs else None
    for tokens in (1, 3, 149, 300):
        bits = synthetic.r4_prefill(tokens=tokens, n=n, seed=600 + k + tokens)[0]
        q, s = run(spin_gpu, bits, clip, signs, direct, path)
        compare(orc, bits, clip, signs, direct, q, s, range(tokens), f"n={n} {variant} {path} T={tokens}")
    assert spin_gpu.device_status() == 0


@pytest.mark.parametrize("n", TC_SIZES)
def test_int8_special_rows(spin_gpu, orc, n):
    rows = [np.zeros(n, np.float32), np.full(n, 1.0, np.float32)]
    for j in sorted({0, 1, 127, 128 % n, n // 2 - 1, n - 1}):
        r = np.zeros(n, np.float32)
        r[j] = 60.0
        rows.append(r)
    rows.append(np.where(np.arange(n) % 3 == 0, 3.0e4, -2.0e4).astype(np.float32))
    bits = synthetic.to_bf16_bits(np.stack(rows))
    for path in ("cuda_cores", "tensor_cores"):
        q, s = run(spin_gpu, bits, 1.0, None, path=path)
        compare(orc, bits, 1.0, None, False, q, s, range(len(rows)), f"n={n} special {path}")
        assert np.all(q[0] == 0) and s[0] == np.float32(1e-8)
        for t in range(2, len(rows) - 1):  # one-hot rows rotate to full scale
            assert np.all(np.abs(q[t]) == 127)


@pytest.mark.parametrize("n,tokens", [(128, 149 * 256 + 77), (256, 149 * 128 + 77), (16384, 149 * 2 * 3 + 1)])
def test_int8_many_groups(spin_gpu, orc, n, tokens):
    """More MMA groups than resident blocks; the default dispatch (tensor cores at
    this size) against the CUDA-core kernel, sampled rows against the oracle."""
    bits, signs, _ = synthetic.r4_prefill(tokens=tokens, n=n, seed=19)
    q1, s1 = run(spin_gpu, bits, 0.9, signs)
    q2, s2 = run(spin_gpu, bits, 0.9, signs, path="cuda_cores")
    parity.check_rel(s1, s2, 1e-5, "tc vs cuda-core scales")
    rng = np.random.default_rng(n)
    diff = np.nonzero((q1 != q2).any(axis=1))[0]
    sample = np.concatenate([rng.choice(tokens, 24, replace=False), [0, tokens - 1], diff[:16]])
    compare(orc, bits, 0.9, signs, False, q1, s1, sample, f"n={n} many groups")
    assert (q1 != q2).mean() < 1e-4
    assert spin_gpu.device_status() == 0


@pytest.mark.parametrize("n", [128, 512, 1024, 16384])
def test_int8_leaves_tail_untouched(spin_gpu, n):
    bits = synthetic.r4_prefill(tokens=5, n=n, seed=3)[0]
    out = torch.full((8, n), 0x5A, dtype=torch.int8, device="cuda")
    sc = torch.full((8,), -1.0, dtype=torch.float32, device="cuda")
    spin_gpu.hadamard_quant_int8(to_dev_bf16(bits), 1.0, out=out[:5], scales=sc[:5])
    torch.cuda.synchronize()
    assert torch.all(out[5:] == 0x5A) and torch.all(sc[5:] == -1.0)
    assert torch.all(sc[:5] > 0)
