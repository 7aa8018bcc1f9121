"""Failure detection without a GPU fault: the tensor-core kernel's bounded waits
run out when one internal signal is withheld (test hook), the kernel returns
through its abort path, the device status word reports it, and the context
stays usable. Sizes cover both ways the epilogue leaves on an abort: one thread
deciding for its warpgroup (n = 4096) and every thread waiting itself, with the
warpgroup's reducing barrier making the decision uniform (n = 16384; n = 32768,
whose token spans both warpgroups)."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("k", [12, 14, 15])
def test_bounded_wait_expiry_sets_status_and_context_survives(spin_gpu, orc, k):
    n, tokens = 1 << k, 64
    bits = synthetic.sweep(k, tokens=tokens, seed=31)
    x = to_dev_bf16(bits)
    spin_gpu.device_status(reset=True)
    assert spin_gpu.device_status() == 0
    try:
        spin_gpu.test_stall_tensor_core_waits(True)
        spin_gpu.hadamard_quant_int4(x, 1.0, tensor_cores=True)
        torch.cuda.synchronize()  # returns: every wait is bounded
    finally:
        spin_gpu.test_stall_tensor_core_waits(False)
    assert spin_gpu.device_status(reset=True) != 0
    assert spin_gpu.device_status() == 0
    # the context is intact: the next launches are correct
    q, s = spin_gpu.hadamard_quant_int4(x, 1.0, tensor_cores=True)
    torch.cuda.synchronize()
    codes = parity.unpack_signed(q.cpu().numpy(), n)
    s = s.cpu().numpy()
    for t in range(0, tokens, 7):
        r = orc.r4_row(bits[t], 1.0)
        parity.check_rel([s[t]], [r["scale64"]], 1e-5, f"scale row {t}")
        parity.check_codes(codes[t], r["codes"], r["pre"], f"codes row {t}")
    assert spin_gpu.device_status() == 0
