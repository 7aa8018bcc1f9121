"""C ABI checks that need no GPU: the library builds and loads, exports every
function include/spin.h declares, and rejects bad arguments on the host before
touching the device."""
import ctypes as C
import subprocess

import pytest

import online_hadamard_rotation_b200 as spin


@pytest.fixture(scope="module")
def L():
    from online_hadamard_rotation_b200 import build
    build.build()
    return spin.lib()


def test_header_declares_the_entry_points():
    names = spin.exported_symbols()
    for fn in ("spin_hadamard_quant_int4", "spin_hadamard_quant_int4_ex", "spin_hadamard_quant_int8",
               "spin_rope_hadamard_kvquant", "spin_dequant_hadamard_inverse", "spin_status_string",
               "spin_last_cuda_error", "spin_version"):
        assert fn in names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", spin.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    defined = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for fn in spin.exported_symbols():
        assert fn in defined, fn
        assert getattr(L, fn) is not None


def test_status_strings_and_version(L):
    assert L.spin_status_string(0) == b"SPIN_OK"
    assert L.spin_status_string(2) == b"SPIN_ERR_UNSUPPORTED_SIZE"
    assert L.spin_version() == 100
    assert L.spin_last_cuda_error() == 0


FAKE = 0x10000  # a 16-byte-aligned address that is never dereferenced by these calls


@pytest.mark.parametrize("n", [0, 64, 100, 129, 65536, -128])
def test_r4_rejects_sizes(L, n):
    assert L.spin_hadamard_quant_int4(FAKE, 4, n, 1.0, FAKE, FAKE, None) == 2


@pytest.mark.parametrize("clip", [0.0, -0.5, 1.5, float("nan")])
def test_r4_rejects_clip(L, clip):
    assert L.spin_hadamard_quant_int4(FAKE, 4, 256, clip, FAKE, FAKE, None) == 1


@pytest.mark.parametrize("n", [0, 64, 100, 65536])
def test_r4_int8_rejects_sizes_and_arguments(L, n):
    assert L.spin_hadamard_quant_int8(FAKE, 4, n, 1.0, None, 0, FAKE, FAKE, None) == 2
    assert L.spin_hadamard_quant_int8(FAKE, 4, 256, 1.5, None, 0, FAKE, FAKE, None) == 1
    assert L.spin_hadamard_quant_int8(FAKE, 4, 256, 1.0, None, 6, FAKE, FAKE, None) == 1  # both kernel bits
    assert L.spin_hadamard_quant_int8(FAKE, 4, 256, 1.0, None, 8, FAKE, FAKE, None) == 1  # unknown bit
    assert L.spin_hadamard_quant_int8(None, 0, 256, 1.0, None, 0, None, None, None) == 0  # empty: no-op
    assert L.spin_hadamard_quant_int8(FAKE, 4, 256, 1.0, None, 0, None, FAKE, None) == 1
    assert L.spin_hadamard_quant_int8(FAKE, 4, 256, 1.0, None, 0, FAKE + 4, FAKE, None) == 3


def test_r4_argument_checks(L):
    assert L.spin_hadamard_quant_int4(FAKE, -1, 256, 1.0, FAKE, FAKE, None) == 1
    assert L.spin_hadamard_quant_int4(None, 0, 256, 1.0, None, None, None) == 0  # empty: no-op
    assert L.spin_hadamard_quant_int4(None, 4, 256, 1.0, FAKE, FAKE, None) == 1
    assert L.spin_hadamard_quant_int4(FAKE + 2, 4, 256, 1.0, FAKE, FAKE, None) == 3
    assert L.spin_hadamard_quant_int4(FAKE, 4, 256, 1.0, FAKE + 8, FAKE, None) == 3
    assert L.spin_hadamard_quant_int4(FAKE, 4, 256, 1.0, FAKE, FAKE + 1, None) == 3
    assert L.spin_hadamard_quant_int4_ex(FAKE, 4, 256, 1.0, FAKE + 2, 0, FAKE, FAKE, None) == 3
    assert L.spin_hadamard_quant_int4_ex(FAKE, 4, 256, 1.0, None, 8, FAKE, FAKE, None) == 1
    assert L.spin_hadamard_quant_int4_ex(FAKE, 4, 256, 1.0, None, 6, FAKE, FAKE, None) == 1  # both kernel choices


def _r3(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, theta=1e4, head_dim=128, batch=2, seq=8, hq=32, hkv=8, clip=0.95,
             q_out=FAKE, kc=FAKE, vc=FAKE, ks=FAKE, kz=FAKE, vs=FAKE, vz=FAKE, cache_len=16, cache_offset=0)
    a.update(kw)
    return L.spin_rope_hadamard_kvquant(a["q"], a["k"], a["v"], a["pos"], a["theta"], a["head_dim"], a["batch"],
                                        a["seq"], a["hq"], a["hkv"], a["clip"], a["q_out"], a["kc"], a["vc"],
                                        a["ks"], a["kz"], a["vs"], a["vz"], a["cache_len"], a["cache_offset"],
                                        None)


def test_r3_argument_checks(L):
    assert _r3(L, head_dim=64) == 2
    assert _r3(L, head_dim=96) == 2
    assert _r3(L, hq=30) == 1  # not a multiple of hkv
    assert _r3(L, cache_len=7) == 1
    assert _r3(L, cache_offset=-1) == 1
    assert _r3(L, theta=0.0) == 1
    assert _r3(L, clip=0.0) == 1
    assert _r3(L, batch=0, q=None) == 0
    assert _r3(L, seq=0) == 0
    assert _r3(L, v=None) == 1
    assert _r3(L, q_out=FAKE + 4) == 3
    assert _r3(L, ks=FAKE + 1) == 3
    assert _r3(L, hq=400, hkv=40) == 2
    assert _r3(L, hq=264, hkv=8) == 2  # more than 256 query heads
    assert _r3(L, hq=256, hkv=128) == 2  # more than 384 head vectors per token
    assert _r3(L, batch=1 << 20, seq=1024, cache_len=1024) == 2  # batch * seq * hq >= 2^31


def test_dequant_argument_checks(L):
    f = L.spin_dequant_hadamard_inverse
    assert f(FAKE, 4, 200, 0, FAKE, None, None, 0, FAKE, 0, None) == 2
    assert f(FAKE, 4, 256, 2, FAKE, None, None, 0, FAKE, 0, None) == 1
    assert f(FAKE, 4, 256, 0, FAKE, None, None, 0, FAKE, 3, None) == 1
    assert f(FAKE, 4, 256, 1, FAKE, None, None, 0, FAKE, 0, None) == 1  # asym needs zero
    assert f(FAKE, -1, 256, 0, FAKE, None, None, 0, FAKE, 0, None) == 1
    assert f(None, 0, 256, 0, None, None, None, 0, None, 0, None) == 0
    assert f(FAKE + 8, 4, 256, 0, FAKE, None, None, 0, FAKE, 0, None) == 3
    assert f(FAKE, 4, 256, 0, FAKE + 2, None, None, 0, FAKE, 0, None) == 3
    assert f(FAKE, 4, 256, 1, FAKE + 2, FAKE + 1, None, 0, FAKE, 0, None) == 3
    assert f(FAKE, 4, 4096, 0, FAKE, None, None, 8, FAKE, 0, None) == 1  # unknown flag
    assert f(FAKE, 4, 4096, 0, FAKE, None, None, 6, FAKE, 0, None) == 1  # both kernel choices


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(spin, "_lib", None)
    monkeypatch.setattr(spin, "LIB_PATH", str(tmp_path / "libspin.so"))
    with pytest.raises(ImportError):
        spin.lib()


def test_binding_rejects_host_tensors():
    """A host pointer must never reach a kernel: the binding refuses tensors that are not
    on a CUDA device before it calls the library."""
    import torch
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    for fn in (spin.hadamard_quant_int4, spin.hadamard_quant_int8):
        with pytest.raises(ValueError, match="CUDA"):
            fn(x, 1.0)
    with pytest.raises(ValueError, match="CUDA"):
        spin.dequant_hadamard_inverse(torch.zeros((4, 128), dtype=torch.uint8), 256,
                                      torch.ones(4, dtype=torch.float32))
    q = torch.zeros((1, 2, 4, 128), dtype=torch.bfloat16)
    kv = torch.zeros((1, 2, 1, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        spin.rope_hadamard_kvquant(q, kv, kv, torch.zeros((1, 2), dtype=torch.int32), {}, clip=1.0)
    with pytest.raises(TypeError):
        spin.hadamard_quant_int4(torch.zeros((4, 256), dtype=torch.float32), 1.0)


def test_dispatch_query(L):
    """spin_uses_tensor_cores answers on the host with the entry points' own rules."""
    R4, INV = 0, 1
    q = L.spin_uses_tensor_cores
    q.argtypes = [C.c_int32, C.c_int64, C.c_int32, C.c_uint32, C.c_int32]
    q.restype = C.c_int
    assert q(R4, 8192, 16384, 0, 1) == 1              # R4 prefill: tensor cores
    assert q(R4, 32, 16384, 0, 0) == 0                # decode batch: CUDA cores
    assert q(R4, 1, 16384, 4, 0) == 1                 # SPIN_TENSOR_CORES at any batch
    assert q(R4, 8192, 16384, 2, 1) == 0              # SPIN_CUDA_CORES_ONLY
    assert q(R4, 8192, 16384, 1, 0) == 0              # SPIN_NO_ROTATE
    assert q(R4, 16384, 32768, 0, 1) == 0             # n = 32768 with a diagonal
    assert q(R4, 16384, 32768, 0, 0) == 1
    assert q(R4, 128 * 256, 128, 0, 0) == 1 and q(R4, 128 * 256 - 1, 128, 0, 0) == 0
    assert q(R4, 10 ** 6, 512, 0, 0) == 1 and q(R4, 10 ** 6, 1024, 4, 0) == 1   # tensor cores from n = 512
    assert q(R4, 128 * 64 - 1, 512, 0, 0) == 0 and q(R4, 128 * 32, 1024, 0, 0) == 1
    assert q(R4, 128 * 16, 2048, 0, 0) == 1
    assert q(INV, 128 * 128, 256, 0, 0) == 1 and q(INV, 128 * 128 - 1, 256, 0, 0) == 0
    assert q(INV, 10 ** 6, 2048, 0, 0) == 1 and q(INV, 128 * 8, 4096, 0, 0) == 1
    assert q(INV, 128 * 64, 512, 0, 0) == 1 and q(INV, 128 * 64 - 1, 512, 0, 0) == 0
    for bad in ((R4, 4, 100, 0, 0), (R4, -1, 256, 0, 0), (R4, 4, 256, 6, 0), (R4, 4, 256, 8, 0), (7, 4, 256, 0, 0),
                (7, 4, 256, 2, 0)):
        assert q(*bad) == -1
    # the entry points' row limits apply (no signed overflow in the size checks)
    assert q(R4, (1 << 47) - 1, 32768, 2, 0) == 0 and q(R4, 1 << 47, 32768, 0, 0) == -1
    assert q(R4, 1 << 56, 32768, 4, 0) == -1 and q(R4, 1 << 62, 128, 4, 0) == -1
    assert q(INV, (1 << 46) - 1, 32768, 2, 0) == 0 and q(INV, 1 << 46, 32768, 0, 0) == -1
    assert q(INV, 1 << 56, 32768, 4, 0) == -1


def test_bench_names_the_dispatched_kernel():
    import bench
    assert bench.r4_kernel_name(16384, 8192, True) == "k1_tc_rotate_quant"
    assert bench.r4_kernel_name(128, 1 << 22, False) == "k1_tcs_rotate_quant"
    assert bench.r4_kernel_name(1024, 1 << 19, False, 8) == "k1_tc_rotate_quant"
    assert bench.r4_kernel_name(1024, 32, False, 8) == "k1_rotate_quant_int8"  # a decode-size batch
    assert bench.k3_kernel_name(256, 1 << 21) == "k3_tcs_dequant_inverse"
    assert bench.k3_kernel_name(2048, 1 << 18) == "k3_tc_dequant_inverse"
    assert bench.k3_kernel_name(2048, 100) == "k3_dequant_inverse"


def test_kron_size_rules(L):
    """spin_hadamard_quant_kron accepts n = m 2^k with a Paley order m, 2^k >= 128 and
    n / 128 a multiple of 16 up to 128; with tokens = 0 the call returns before any
    device access, so the size rules are checked here without a GPU."""
    f = L.spin_hadamard_quant_kron
    f.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_int32, C.c_float, C.c_void_p, C.c_uint32, C.c_int32,
                  C.c_void_p, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    OK, BAD, SIZE = 0, 1, 2
    for m, n in ((28, 14336), (12, 6144), (12, 12288), (20, 10240), (24, 6144), (48, 6144), (4, 2048), (8, 4096)):
        assert f(None, 0, m, n, 1.0, None, 0, 4, None, None, None) == OK, (m, n)
    for m, n in ((16, 4096), (28, 7168), (36, 18432), (12, 3072), (20, 2560), (40, 10240), (28, 14336 * 2),
                 (28, 14000), (0, 2048), (-12, 6144), (12, 0)):
        assert f(None, 0, m, n, 1.0, None, 0, 4, None, None, None) == SIZE, (m, n)
    assert f(None, 0, 28, 14336, 1.0, None, 0, 5, None, None, None) == BAD      # bits
    assert f(None, 0, 28, 14336, 1.0, None, 1, 4, None, None, None) == BAD      # SPIN_NO_ROTATE is not a flag here
    assert f(None, 0, 28, 14336, 1.5, None, 0, 4, None, None, None) == BAD      # clip
    assert f(None, 4, 28, 14336, 1.0, None, 0, 4, None, None, None) == BAD      # null pointers


def test_w4a4_gemm_host_rules(L):
    """spin_w4a4_gemm takes n_out a multiple of 256 and k a multiple of 128 in
    [128, 65536]; tokens = 0 and every rejected argument return before any device
    access, so the rules are checked here without a GPU."""
    f = L.spin_w4a4_gemm
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p,
                  C.c_int32, C.c_void_p]
    f.restype = C.c_int
    OK, BAD, SIZE, MIS = 0, 1, 2, 3
    for n_out, k in ((256, 128), (4096, 14336), (14336, 4096), (11008, 4096), (256, 65536)):
        assert f(None, None, 0, None, None, n_out, k, None, 1, None) == OK, (n_out, k)
    for n_out, k in ((128, 4096), (4000, 4096), (4096, 64), (4096, 4000), (4096, 65536 + 128), (0, 128),
                     (256, 0), (-256, 128)):
        assert f(None, None, 0, None, None, n_out, k, None, 1, None) == SIZE, (n_out, k)
    assert f(None, None, -1, None, None, 256, 128, None, 1, None) == BAD      # tokens < 0
    assert f(None, None, 0, None, None, 256, 128, None, 2, None) == BAD       # out_dtype
    assert f(None, None, 4, None, None, 256, 128, None, 1, None) == BAD       # null pointers
    assert f(FAKE, FAKE + 4, 4, FAKE, FAKE + 4, 256, 128, FAKE, 1, None) == MIS   # w_scales not 16-byte aligned
    assert f(FAKE + 8, FAKE, 4, FAKE, FAKE, 256, 128, FAKE, 1, None) == MIS      # x_codes


def test_decode_attention_host_rules(L):
    """Workspace size and argument rules of the decode-attention entry point; batch = 0
    and every rejected argument return before any device access."""
    ws = L.spin_decode_attention_workspace_bytes
    ws.argtypes = [C.c_int32] * 3
    ws.restype = C.c_size_t
    assert ws(4, 32, 4096) == 4 * 32 * 16 * 130 * 4  # 16 chunks of 256 slots, 128 + 2 floats each
    assert ws(1, 8, 257) == 8 * 2 * 130 * 4 and ws(0, 8, 10) == 0 and ws(1, 8, 0) == 0
    f = L.spin_decode_attention_int4kv
    f.argtypes = [C.c_void_p] * 8 + [C.c_int32] * 5 + [C.c_float, C.c_void_p, C.c_int32, C.c_void_p, C.c_size_t,
                                                      C.c_void_p]
    f.restype = C.c_int
    z = [None] * 8
    assert f(*z, 0, 32, 8, 128, 4096, 0.088, None, 1, None, 0, None) == 0      # batch 0: no-op
    assert f(*z, 0, 32, 8, 64, 4096, 0.088, None, 1, None, 0, None) == 2       # head_dim
    assert f(*z, 0, 24, 8, 128, 4096, 0.088, None, 1, None, 0, None) == 2      # 3 query heads per kv head
    assert f(*z, 0, 30, 8, 128, 4096, 0.088, None, 1, None, 0, None) == 1      # not a multiple
    assert f(*z, 0, 32, 8, 128, 0, 0.088, None, 1, None, 0, None) == 1         # empty cache
    assert f(*z, 0, 32, 8, 128, 4096, -1.0, None, 1, None, 0, None) == 1       # softmax scale
    assert f(*z, 0, 32, 8, 128, 4096, 0.088, None, 7, None, 0, None) == 1      # out dtype
    assert f(*z, 2, 32, 8, 128, 4096, 0.088, None, 1, None, 0, None) == 1      # null pointers
