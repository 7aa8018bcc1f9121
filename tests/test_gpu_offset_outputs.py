"""Outputs that start 16 bytes (not 32) past an aligned address: a caller's
view into a larger buffer. The tensor-core kernels store 32 bytes at a time
when the output pointer allows it and switch to 16-byte stores otherwise; these
tests run that second form of every tensor-core kernel (R4 INT4 and INT8 at
n = 128 .. 32768, with and without the diagonal, and both
tensor-core inverses, bf16 and fp32 out) against the oracle, with canary bytes
on both sides of the output."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16, to_dev_signs

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 64  # bytes of canary after the view
# tokens: several MMA groups plus a ragged tail (tokens per group: 256 at n = 128,
# 128 at n = 256, 64 at n = 512 (an odd tail splits a two-token box), 256 / (n / 128)
# from 1024, 1 at 32768)
TOKENS = {128: 3 * 256 + 77, 256: 3 * 128 + 37, 512: 3 * 64 + 33, 1024: 3 * 32 + 5, 2048: 5 * 16 + 7, 4096: 5 * 8 + 3, 8192: 9 * 4 + 1,
          16384: 11 * 2 + 1, 32768: 7}


def offset_view(nbytes: int, dtype: torch.dtype, shape, offset: int = 16):
    """A contiguous view of `shape` starting `offset` bytes into a canary-filled buffer."""
    buf = torch.full((offset + nbytes + PAD,), CANARY, dtype=torch.uint8, device="cuda")
    assert buf.data_ptr() % 256 == 0
    view = buf[offset:offset + nbytes].view(dtype).view(shape)
    assert view.data_ptr() % 32 == offset % 32
    return buf, view


def assert_canaries(buf, offset, nbytes, what):
    b = buf.cpu().numpy()
    assert np.all(b[:offset] == CANARY), f"{what}: bytes before the output changed"
    assert np.all(b[offset + nbytes:] == CANARY), f"{what}: bytes after the output changed"


@pytest.mark.parametrize("n", sorted(TOKENS))
@pytest.mark.parametrize("with_signs", [False, True])
@pytest.mark.parametrize("bits_", [4, 8])
def test_r4_tensor_core_output_at_16_byte_offset(spin_gpu, orc, n, with_signs, bits_):
    if n == 32768 and with_signs:
        pytest.skip("n = 32768 with a diagonal runs the CUDA-core kernel")
    tokens = TOKENS[n]
    assert spin_gpu.uses_tensor_cores(spin_gpu.OP_HADAMARD_QUANT, tokens, n, spin_gpu.TENSOR_CORES, with_signs)
    bits, signs, _ = synthetic.r4_prefill(tokens=tokens, n=n, seed=700 + n // 128 + bits_)
    if not with_signs:
        signs = None
    cols = n // 2 if bits_ == 4 else n
    dtype = torch.uint8 if bits_ == 4 else torch.int8
    qbuf, q = offset_view(tokens * cols, dtype, (tokens, cols))
    sbuf, s = offset_view(4 * tokens, torch.float32, (tokens,), offset=4)  # steps at a 4-byte offset
    quant = spin_gpu.hadamard_quant_int4 if bits_ == 4 else spin_gpu.hadamard_quant_int8
    quant(to_dev_bf16(bits), 0.9, to_dev_signs(signs), out=q, scales=s, tensor_cores=True)
    torch.cuda.synchronize()
    assert spin_gpu.device_status() == 0
    what = f"n={n} INT{bits_} signs={with_signs}"
    assert_canaries(qbuf, 16, tokens * cols, what + " codes")
    assert_canaries(sbuf, 4, 4 * tokens, what + " steps")
    q_np, s_np = q.cpu().numpy(), s.cpu().numpy()
    if bits_ == 4:
        parity.check_r4_bulk(orc, bits, 0.9, signs, q_np, s_np, what=what)
    else:
        for t in range(tokens):
            r = orc.r4_row_int8(bits[t], 0.9, signs=signs)
            parity.check_rel([s_np[t]], [r["scale64"]], 1e-5, f"{what}: step row {t}")
            parity.check_codes(q_np[t].astype(np.int32), r["codes"], r["pre"], f"{what}: codes row {t}")


@pytest.mark.parametrize("n,rows", [(128, 300), (256, 150), (512, 131), (1024, 67), (2048, 35), (4096, 19), (8192, 9),
                                    (16384, 5), (32768, 3)])
@pytest.mark.parametrize("with_signs", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_inverse_tensor_core_output_at_16_byte_offset(spin_gpu, orc, n, rows, with_signs, out_dtype):
    assert spin_gpu.uses_tensor_cores(spin_gpu.OP_DEQUANT_INVERSE, rows, n, spin_gpu.TENSOR_CORES)
    signs = synthetic.sign_bits(n, 40 + rows) if with_signs else None
    bits = synthetic.sweep(n.bit_length() - 1, tokens=rows, seed=800 + rows)
    packed, scales = orc.r4_rows(bits, 0.9, signs)
    esize = 4 if out_dtype == torch.float32 else 2
    obuf, out = offset_view(rows * n * esize, out_dtype, (rows, n))
    spin_gpu.dequant_hadamard_inverse(torch.from_numpy(packed).cuda(), n, torch.from_numpy(scales).cuda(),
                                      signs=to_dev_signs(signs), out=out, tensor_cores=True)
    torch.cuda.synchronize()
    assert spin_gpu.device_status() == 0
    what = f"inverse n={n} {out_dtype} signs={with_signs}"
    assert_canaries(obuf, 16, rows * n * esize, what)
    got = out.float().cpu().numpy().astype(np.float64)
    ref = orc.dequant_inverse_rows(packed, n, 0, scales.astype(np.float64), signs=signs)
    if out_dtype == torch.float32:
        parity.check_f32_rows(got, ref, what)
    else:
        parity.check_bf16(got, ref, what)
    # the 16-byte store form gives the same bits as the CUDA-core kernel
    ref_dev = spin_gpu.dequant_hadamard_inverse(torch.from_numpy(packed).cuda(), n, torch.from_numpy(scales).cuda(),
                                                signs=to_dev_signs(signs), out_dtype=out_dtype, cuda_cores_only=True)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16 if esize == 2 else torch.int32),
                       ref_dev.view(torch.int16 if esize == 2 else torch.int32)), what
