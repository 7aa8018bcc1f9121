"""R3 + INT4 KV cache kernel (spin_rope_hadamard_kvquant) vs the fp64 oracle:
rotated Q (bf16), K and V codes, fp16 scales and zero points, cache slot
placement, positions that differ from slots, ragged token groups, and cache
slots that must stay untouched. A group whose fp16 step differs from the
oracle's must sit on an fp16 rounding boundary and is then compared in full
with the oracle's result for the other step."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity
from tests.gpu_util import bf16_dev_to_bits, f16_dev_to_bits, to_dev_bf16

pytestmark = pytest.mark.gpu

CANARY_BYTE = 0xA5
CANARY_F16 = np.float16(-1234.0)


def run_r3(spin, q, k, v, pos, theta, clip, cache_len, cache_offset):
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    cache = spin.alloc_kv_cache(B, hkv, cache_len, d)
    for name in ("k_cache", "v_cache"):
        cache[name].fill_(CANARY_BYTE)
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        cache[name].fill_(float(CANARY_F16))
    qo = spin.rope_hadamard_kvquant(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v),
                                    torch.from_numpy(np.ascontiguousarray(pos)).cuda(), cache, theta=theta, clip=clip,
                                    cache_offset=cache_offset)
    torch.cuda.synchronize()
    out = {n: t.cpu().numpy() for n, t in cache.items()}
    for n in ("k_scale", "k_zero", "v_scale", "v_zero"):
        out[n] = f16_dev_to_bits(cache[n])
    out["q_out"] = bf16_dev_to_bits(qo)
    return out


def compare_tokens(orc, q, k, v, pos, theta, clip, out, cache_offset, tokens):
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    skipped = 0
    for (b, s) in tokens:
        r = orc.r3_token(q[b, s], k[b, s], v[b, s], pos[b, s], theta, clip)
        parity.check_bf16(parity.bf16_bits_to_f64(out["q_out"][b, s]), r["q_f64"], f"q_out ({b},{s})")
        slot = cache_offset + s
        for h in range(hkv):
            skipped += parity.check_asym_group(
                orc, clip, out["k_cache"][b, h, slot], int(out["k_scale"][b, h, slot]), int(out["k_zero"][b, h, slot]),
                r["k_packed"][h], int(r["k_s"][h]), int(r["k_z"][h]), r["k_pre"][h], r["k_f64"][h], f"K ({b},{s},{h})")
            vv = synthetic.bf16_bits_to_f32(v[b, s, h]).astype(np.float64)
            skipped += parity.check_asym_group(
                orc, clip, out["v_cache"][b, h, slot], int(out["v_scale"][b, h, slot]), int(out["v_zero"][b, h, slot]),
                r["v_packed"][h], int(r["v_s"][h]), int(r["v_z"][h]), r["v_pre"][h], vv, f"V ({b},{s},{h})")
    return skipped


def compare_all_tokens(orc, q, k, v, pos, theta, clip, out, cache_offset):
    """Every token of a batch: the oracle's threaded batch path gives rotated Q (as
    bf16), the caches, steps and zero points for all tokens; tokens where anything
    differs from it are re-checked one by one with the tolerances (bf16 bound for Q,
    rounding ties for codes, fp16 step boundary). Returns (tokens re-checked, groups
    on an fp16 step boundary)."""
    B, S = q.shape[:2]
    cache_len = out["k_cache"].shape[2]
    ref = orc.r3_batch(q, k, v, pos, theta, clip, cache_len=cache_len, cache_offset=cache_offset,
                       threads=orc.max_threads())
    sl = slice(cache_offset, cache_offset + S)
    differs = (out["q_out"] != ref["q_out"]).reshape(B, S, -1).any(axis=2)
    for name in ("k_cache", "v_cache"):
        differs |= (out[name][:, :, sl] != ref[name][:, :, sl]).any(axis=3).any(axis=1)
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        differs |= (out[name][:, :, sl] != ref[name][:, :, sl]).any(axis=1)
    toks = [(int(b), int(s)) for b, s in zip(*np.nonzero(differs))]
    return len(toks), compare_tokens(orc, q, k, v, pos, theta, clip, out, cache_offset, toks)


@pytest.mark.parametrize("shape", [(2, 37, 32, 8), (1, 5, 8, 8), (3, 2, 16, 2), (1, 1, 32, 8), (1, 9, 20, 10),
                                   (2, 3, 128, 32), (1, 3, 256, 64), (1, 7, 4, 1)])
def test_r3_small_shapes(spin_gpu, orc, shape):
    B, S, hq, hkv = shape
    q, k, v, _ = synthetic.r3_kv(B, S, hq, hkv, 128, seed=sum(shape))
    pos = (np.arange(S)[None, :] + 100 * np.arange(B)[:, None]).astype(np.int32)  # positions != slots
    cache_offset, cache_len = 3, S + 7
    out = run_r3(spin_gpu, q, k, v, pos, 1e4, 0.95, cache_len, cache_offset)
    compare_tokens(orc, q, k, v, pos, 1e4, 0.95, out, cache_offset, [(b, s) for b in range(B) for s in range(S)])
    # slots outside [offset, offset + S) are untouched
    for name in ("k_cache", "v_cache"):
        assert np.all(out[name][:, :, :cache_offset] == CANARY_BYTE)
        assert np.all(out[name][:, :, cache_offset + S:] == CANARY_BYTE)
    canary = np.array([CANARY_F16]).view(np.uint16)[0]
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        assert np.all(out[name][:, :, :cache_offset] == canary)
        assert np.all(out[name][:, :, cache_offset + S:] == canary)


def test_r3_in_place_q(spin_gpu, orc):
    B, S, hq, hkv = 1, 9, 32, 8
    q, k, v, pos = synthetic.r3_kv(B, S, hq, hkv, 128, seed=77)
    cache = spin_gpu.alloc_kv_cache(B, hkv, S)
    qd = to_dev_bf16(q)
    ret = spin_gpu.rope_hadamard_kvquant(qd, to_dev_bf16(k), to_dev_bf16(v), torch.from_numpy(pos).cuda(), cache,
                                         clip=0.95, q_out=qd)
    torch.cuda.synchronize()
    assert ret.data_ptr() == qd.data_ptr()
    got = parity.bf16_bits_to_f64(bf16_dev_to_bits(qd))
    for s in range(S):
        r = orc.r3_token(q[0, s], k[0, s], v[0, s], pos[0, s], 1e4, 0.95)
        parity.check_bf16(got[0, s], r["q_f64"], f"in-place q {s}")


def test_r3_large_positions(spin_gpu, orc):
    B, S, hq, hkv = 1, 4, 8, 8
    q, k, v, _ = synthetic.r3_kv(B, S, hq, hkv, 128, seed=5)
    pos = np.array([[0, 65535, 131071, 1000000]], dtype=np.int32)
    out = run_r3(spin_gpu, q, k, v, pos, 5e5, 1.0, S, 0)
    compare_tokens(orc, q, k, v, pos, 5e5, 1.0, out, 0, [(0, s) for s in range(S)])
