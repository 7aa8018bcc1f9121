"""R4 kernel (spin_hadamard_quant_int4[_ex]) vs the fp64 oracle, element by
element: every supported n, ragged token counts, clip 1.0 / 0.9, with and
without the +-1 diagonal, direct quantisation, and special rows."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16, to_dev_signs

pytestmark = pytest.mark.gpu

VARIANTS = {"plain": (1.0, False, False), "clip_signs": (0.9, True, False), "direct": (1.0, False, True)}


def run(spin, bits, clip, signs, direct):
    q, s = spin.hadamard_quant_int4(to_dev_bf16(bits), clip, to_dev_signs(signs), no_rotate=direct)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def compare(orc, bits, clip, signs, direct, q, s, rows):
    n = bits.shape[1]
    codes = parity.unpack_signed(q, n)
    exempt = 0
    for t in rows:
        r = orc.r4_row(bits[t], clip, signs=signs, no_rotate=direct)
        parity.check_rel([s[t]], [r["scale64"]], 1e-5, f"scale row {t}")
        exempt += parity.check_codes(codes[t], r["codes"], r["pre"], f"codes row {t}")
    return exempt


@pytest.mark.parametrize("k", list(range(7, 16)))
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_r4_all_sizes(spin_gpu, orc, k, variant):
    clip, with_signs, direct = VARIANTS[variant]
    n = 1 << k
    signs = synthetic.sign_bits(n, 100 + k) if with_signs else None
    for tokens in (1, 3, 32, 257):
        bits = synthetic.sweep(k, tokens=tokens, seed=1000 + 7 * k + tokens)
        q, s = run(spin_gpu, bits, clip, signs, direct)
        compare(orc, bits, clip, signs, direct, q, s, range(tokens))


@pytest.mark.parametrize("k", [7, 10, 14, 15])
def test_r4_special_rows(spin_gpu, orc, k):
    n = 1 << k
    rows = [np.zeros(n, np.float32), np.full(n, 1.0, np.float32), np.full(n, -3.0, np.float32)]
    for j in (0, 5, n - 1):
        r = np.zeros(n, np.float32)
        r[j] = 60.0
        rows.append(r)
    alt = np.where(np.arange(n) % 2 == 0, 3.0e4, -3.0e4).astype(np.float32)
    rows.append(alt)
    tiny = np.full(n, 1e-30, np.float32)
    rows.append(tiny)
    bits = synthetic.to_bf16_bits(np.stack(rows))
    for clip, direct in ((1.0, False), (0.9, False), (1.0, True)):
        q, s = run(spin_gpu, bits, clip, None, direct)
        compare(orc, bits, clip, None, direct, q, s, range(len(rows)))
    q, s = run(spin_gpu, bits, 1.0, None, False)
    codes = parity.unpack_signed(q, n)
    assert np.all(codes[0] == 0) and s[0] == np.float32(1e-8)
    for i in (3, 4, 5):  # one-hot 60: every code is +-7
        assert np.all(np.abs(codes[i]) == 7)


def test_r4_rounding_ties_direct(spin_gpu, orc):
    """Direct quantisation of values sitting exactly on .5 boundaries: the two
    sides may only differ by one code, and only there."""
    n = 128
    base = np.array([7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, -3.5, 4.5, 5.5, 6.5, -6.5, -7.5], np.float32)
    row = np.zeros(n, np.float32)
    row[: base.size] = base
    bits = synthetic.to_bf16_bits(row[None, :])
    q, s = run(spin_gpu, bits, 1.0, None, True)
    compare(orc, bits, 1.0, None, True, q, s, [0])


def test_r4_empty_and_unaligned_tail(spin_gpu):
    """tokens = 0 is a no-op; outputs past the last row are never written."""
    n = 256
    x = torch.zeros((0, n), dtype=torch.bfloat16, device="cuda")
    q, s = spin_gpu.hadamard_quant_int4(x)
    assert q.shape == (0, n // 2)
    bits = synthetic.sweep(8, tokens=5, seed=3)
    out = torch.full((8, n // 2), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.full((8,), -1.0, dtype=torch.float32, device="cuda")
    spin_gpu.hadamard_quant_int4(to_dev_bf16(bits), 1.0, out=out[:5], scales=sc[:5])
    torch.cuda.synchronize()
    assert torch.all(out[5:] == 0xA5) and torch.all(sc[5:] == -1.0)


def test_r4_rejects_bad_arguments_on_gpu(spin_gpu):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(spin_gpu.SpinError):
        spin_gpu.hadamard_quant_int4(x, clip=1.5)
    with pytest.raises(spin_gpu.SpinError):
        spin_gpu.hadamard_quant_int4(torch.zeros((4, 96), dtype=torch.bfloat16, device="cuda"))
