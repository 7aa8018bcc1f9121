"""Decode attention over the INT4 KV cache (spin_decode_attention_int4kv) vs the
fp64 oracle: caches and rotated queries come from the oracle's R3 batch on the
seeded attention-shaped workload; grouped query heads (1, 2, 4 and 8 per kv head),
ragged lengths, a cache longer than the attended slots, the R3 + KV workload's full
cache, fp32 and bf16 outputs, length clamping and argument errors."""
import numpy as np
import pytest
import torch

import synthetic
from tests import parity

pytestmark = pytest.mark.gpu


def oracle_cache(orc, B, S, hq, hkv, L, seed, threads=None):
    q, k, v, pos = synthetic.r3_kv(B, S, hq, hkv, 128, seed=seed)
    ref = orc.r3_batch(q, k, v, pos, 1e4, 0.95, cache_len=L, cache_offset=0,
                       threads=threads or orc.max_threads())
    return ref, ref["q_out"][:, S - 1]  # the last token's rotated query as this step's query


def to_dev(cache):
    out = {}
    for name in ("k_cache", "v_cache"):
        out[name] = torch.from_numpy(np.ascontiguousarray(cache[name])).cuda()
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        out[name] = torch.from_numpy(np.ascontiguousarray(cache[name]).view(np.int16)).view(torch.float16).cuda()
    return out


def run(spin, q_bits, cache_dev, lens, out_dtype=torch.float32):
    q = torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).view(torch.bfloat16).cuda()
    out = spin.decode_attention_int4kv(q, cache_dev, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                       out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out


def compare(got, ref, what):
    B, hq, d = ref.shape
    got = got.float().cpu().numpy().astype(np.float64)
    parity.check_f32_rows(got.reshape(B * hq, d), ref.reshape(B * hq, d), what)


@pytest.mark.parametrize("B,S,hq,hkv,L,lens", [(2, 37, 32, 8, 40, [37, 5]), (1, 300, 8, 8, 300, [300]),
                                               (2, 513, 16, 8, 600, [513, 257]), (1, 200, 64, 8, 256, [200]),
                                               (3, 260, 8, 4, 260, [1, 256, 260])])
def test_decode_attention_vs_oracle(spin_gpu, orc, B, S, hq, hkv, L, lens):
    cache, q = oracle_cache(orc, B, S, hq, hkv, L, seed=B + S + hq)
    ref = orc.decode_attention(q, cache, lens)
    dev = to_dev(cache)
    compare(run(spin_gpu, q, dev, lens), ref, f"fp32 out B={B} S={S} hq={hq} hkv={hkv}")
    got16 = run(spin_gpu, q, dev, lens, torch.bfloat16).float().cpu().numpy().astype(np.float64)
    parity.check_bf16(got16, ref, "bf16 out")


def test_decode_attention_r3_kv_workload_cache(spin_gpu, orc):
    """The R3 + KV workload's whole cache (batch 4 x 4096 slots, 32 / 8 heads)."""
    cache, q = oracle_cache(orc, 4, 4096, 32, 8, 4096, seed=2)
    lens = [4096, 4096, 4096, 4096]
    ref = orc.decode_attention(q, cache, lens, threads=orc.max_threads())
    got = run(spin_gpu, q, to_dev(cache), lens)
    compare(got, ref, "R3 + KV cache")
    again = run(spin_gpu, q, to_dev(cache), lens)
    assert torch.equal(got, again)  # no atomics: the same bits every call


def test_decode_attention_lengths_and_errors(spin_gpu, orc):
    cache, q = oracle_cache(orc, 2, 64, 8, 2, 64, seed=9)
    dev = to_dev(cache)
    # a length past the cache is clamped to it; a zero length gives zeros
    assert torch.equal(run(spin_gpu, q, dev, [64, 99]), run(spin_gpu, q, dev, [64, 64]))
    z = run(spin_gpu, q, dev, [0, 64])
    assert torch.all(z[0] == 0) and torch.all(torch.isfinite(z[1]))
    qd = torch.from_numpy(np.ascontiguousarray(q).view(np.int16)).view(torch.bfloat16).cuda()
    lens = torch.tensor([64, 64], dtype=torch.int32, device="cuda")
    small = torch.empty((16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(spin_gpu.SpinError) as e:
        spin_gpu.decode_attention_int4kv(qd, dev, lens, workspace=small)
    assert e.value.status == 1  # workspace too small
    one = {k: v[:, :1].contiguous() for k, v in dev.items()}  # one kv head for 8 query heads is fine ...
    assert spin_gpu.decode_attention_int4kv(qd, one, lens).shape == (2, 8, 128)
    q6 = torch.zeros((2, 6, 128), dtype=torch.bfloat16, device="cuda")  # ... 3 per kv head is not
    with pytest.raises(spin_gpu.SpinError) as e:
        spin_gpu.decode_attention_int4kv(q6, dev, lens)
    assert e.value.status == 2
