"""spin_decode_attention_int4kv_noalloc, the decode-attention entry point for callers
that cannot allocate device memory (an engine plugin given no scratch, a serving loop
that must not call cudaMalloc): called through the C ABI with raw pointers and no
workspace, twice in a row, its output must match the workspace entry point's within
the fp32 output tolerance, and a call whose partials exceed the built-in scratch must
be refused. This file sorts last so that a run stopping at its first failure has
already run every other test; it also passes alone in a fresh process."""
import ctypes as C

import numpy as np
import pytest
import torch

import synthetic
from tests import parity

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 6  # SPIN_ERR_SCRATCH_LIMIT
SCRATCH_BYTES = 4 << 20  # SPIN_NOALLOC_SCRATCH_BYTES


def _entry(lib):
    f = lib.spin_decode_attention_int4kv_noalloc
    f.argtypes = [C.c_void_p] * 8 + [C.c_int32] * 5 + [C.c_float, C.c_void_p, C.c_int32, C.c_void_p]
    f.restype = C.c_int
    return f


def test_noalloc_matches_workspace_entry_point(spin_gpu, orc):
    B, S, hq, hkv, L = 3, 300, 32, 8, 320
    q, k, v, pos = synthetic.r3_kv(B, S, hq, hkv, 128, seed=123)
    ref = orc.r3_batch(q, k, v, pos, 1e4, 0.95, cache_len=L, threads=orc.max_threads())
    qd = torch.from_numpy(np.ascontiguousarray(ref["q_out"][:, S - 1]).view(np.int16)).view(torch.bfloat16).cuda()
    cache = {n: torch.from_numpy(np.ascontiguousarray(ref[n])).cuda() for n in ("k_cache", "v_cache")}
    for n in ("k_scale", "k_zero", "v_scale", "v_zero"):
        cache[n] = torch.from_numpy(np.ascontiguousarray(ref[n]).view(np.int16)).view(torch.float16).cuda()
    lens = torch.tensor([300, 1, 257], dtype=torch.int32, device="cuda")
    expected = spin_gpu.decode_attention_int4kv(qd, cache, lens)  # the workspace entry point
    torch.cuda.synchronize()
    exp_np = expected.cpu().numpy().astype(np.float64).reshape(B * hq, 128)

    f = _entry(spin_gpu.lib())
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):  # the second call reuses the scratch the first one left behind
        out = torch.full((B, hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        st = f(qd.data_ptr(), cache["k_cache"].data_ptr(), cache["v_cache"].data_ptr(), cache["k_scale"].data_ptr(),
               cache["k_zero"].data_ptr(), cache["v_scale"].data_ptr(), cache["v_zero"].data_ptr(), lens.data_ptr(),
               B, hq, hkv, 128, L, 1.0 / np.sqrt(128.0), out.data_ptr(), 1, stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64).reshape(B * hq, 128)
        parity.check_f32_rows(got, exp_np, f"no-alloc call {call} vs the workspace entry point")
    assert spin_gpu.device_status() == 0

    # partials beyond the built-in scratch are refused before anything is enqueued
    big_len = (SCRATCH_BYTES // (B * hq * 130 * 4) + 1) * 256
    assert spin_gpu.decode_attention_workspace_bytes(B, hq, big_len) > SCRATCH_BYTES
    st = f(qd.data_ptr(), cache["k_cache"].data_ptr(), cache["v_cache"].data_ptr(), cache["k_scale"].data_ptr(),
           cache["k_zero"].data_ptr(), cache["v_scale"].data_ptr(), cache["v_zero"].data_ptr(), lens.data_ptr(),
           B, hq, hkv, 128, big_len, 1.0 / np.sqrt(128.0), out.data_ptr(), 1, stream)
    assert st == SCRATCH_LIMIT
    assert spin_gpu.lib().spin_status_string(SCRATCH_LIMIT) == b"SPIN_ERR_SCRATCH_LIMIT"
