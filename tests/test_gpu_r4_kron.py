"""R4 for row lengths that are not a power of two, n = m 2^k with Paley's H_m
(spin_hadamard_quant_kron) vs the fp64 oracle's Kronecker rotation: the LLaMA-3
8B down-projection width n = 14336 = 28 x 512 and the other supported sizes,
ragged token counts, with and without the diagonal, INT4 and INT8 codes, and the
output at a 16-byte offset."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16, to_dev_signs

pytestmark = pytest.mark.gpu

CASES = [(28, 14336), (12, 6144), (20, 10240), (12, 12288), (24, 6144), (48, 6144)]


def ref_rows(orc, bits, m, clip, signs, code_bits):
    out = []
    for t in range(bits.shape[0]):
        r = orc.r4_row_kron(bits[t], m, clip, signs=signs)
        if code_bits == 8:
            s, pre, codes = orc.quant_sym_int8(r["y"], clip)
            r = dict(y=r["y"], pre=pre, codes=codes, scale64=s)
        out.append(r)
    return out


def check(orc, bits, m, clip, signs, code_bits, q, s, what):
    n = bits.shape[1]
    for t, r in enumerate(ref_rows(orc, bits, m, clip, signs, code_bits)):
        parity.check_rel([s[t]], [r["scale64"]], 1e-5, f"{what}: step row {t}")
        got = parity.unpack_signed(q[t], n)[0] if code_bits == 4 else q[t].astype(np.int32)
        parity.check_codes(got, r["codes"], r["pre"], f"{what}: codes row {t}")


@pytest.mark.parametrize("m,n", sorted(set(CASES)))
@pytest.mark.parametrize("with_signs", [False, True])
@pytest.mark.parametrize("code_bits", [4, 8])
def test_kron_vs_oracle(spin_gpu, orc, m, n, with_signs, code_bits):
    signs = synthetic.sign_bits(n, 900 + m) if with_signs else None
    for tokens in (1, 3, 8, 301):
        bits = synthetic.r4_prefill(tokens=tokens, n=n, seed=950 + tokens + m)[0]
        q, s = spin_gpu.hadamard_quant_kron(to_dev_bf16(bits), m, 0.9, to_dev_signs(signs), bits=code_bits)
        torch.cuda.synchronize()
        check(orc, bits, m, 0.9, signs, code_bits, q.cpu().numpy(), s.cpu().numpy(),
              f"m={m} n={n} signs={with_signs} INT{code_bits} T={tokens}")
    assert spin_gpu.device_status() == 0


def test_kron_one_hot_rows_reach_full_scale(spin_gpu, orc):
    """A one-hot row rotates to +-1/sqrt(n) everywhere (H_m (x) H_b has +-1 entries),
    so every INT4 code is +-7 with the signs of the matrix column; checked at 14336."""
    m, n = 28, 14336
    rows = np.zeros((5, n), np.float32)
    for i, j in enumerate((0, 1, 511, 512, n - 1)):
        rows[i, j] = 3.0
    bits = synthetic.to_bf16_bits(rows)
    q, s = spin_gpu.hadamard_quant_kron(to_dev_bf16(bits), m, 1.0)
    torch.cuda.synchronize()
    codes = parity.unpack_signed(q.cpu().numpy(), n)
    assert np.all(np.abs(codes) == 7)
    check(orc, bits, m, 1.0, None, 4, q.cpu().numpy(), s.cpu().numpy(), "one-hot")


def test_kron_prefill_size_every_row(spin_gpu, orc):
    """8192 tokens x 14336 (the R4 prefill batch at the LLaMA-3 8B width), seeded
    diagonal, clip 0.9: every row against the oracle, plus canaries around a view of
    the codes at a 16-byte offset."""
    m, n, tokens = 28, 14336, 8192
    bits, signs, _ = synthetic.r4_prefill(tokens=tokens, n=n, seed=77)
    buf = torch.full((16 + tokens * n // 2 + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    q = buf[16:16 + tokens * n // 2].view(tokens, n // 2)
    q2, s = spin_gpu.hadamard_quant_kron(to_dev_bf16(bits), m, 0.9, to_dev_signs(signs), out=q)
    torch.cuda.synchronize()
    assert q2.data_ptr() == q.data_ptr() and spin_gpu.device_status() == 0
    b = buf.cpu().numpy()
    assert np.all(b[:16] == 0xA5) and np.all(b[16 + tokens * n // 2:] == 0xA5)
    qn, sn = q.cpu().numpy(), s.cpu().numpy()
    ref = np.array([orc.r4_row_kron(bits[t], m, 0.9, signs=signs)["scale64"] for t in range(0, tokens, 97)])
    parity.check_rel(sn[::97], ref, 1e-5, "kron prefill steps (every 97th row, fp64 single rows)")
    rows = parity.check_kron_bulk(orc, bits, m, 0.9, signs, qn, sn, "kron prefill")
    assert rows < tokens // 4
