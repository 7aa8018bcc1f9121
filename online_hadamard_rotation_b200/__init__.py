"""Python binding for libspin.so: SpinQuant's online Hadamard rotations (R3,
R4) fused with INT4 quantisation, on NVIDIA B200.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/spin.h. PyTorch supplies device
memory and streams. The library must be built (``build.py``); importing this
package without it raises, and there is no CPU fallback.

The functions named ``spin_*`` take raw pointers exactly like the C ABI; the
other functions take torch tensors and return torch tensors.
"""
from __future__ import annotations

import ctypes as C
import os
import re

import torch

__all__ = [
    "lib", "SpinError", "hadamard_quant_int4", "hadamard_quant_int8", "hadamard_quant_int4_host",
    "hadamard_quant_host", "hadamard_quant_kron", "decode_attention_int4kv", "decode_attention_workspace_bytes",
    "rope_hadamard_kvquant",
    "dequant_hadamard_inverse", "alloc_kv_cache", "NO_ROTATE", "SYM_INT4_F32SCALE", "ASYM_INT4_F16SZ",
    "BF16", "F32", "HEADER", "LIB_PATH", "exported_symbols", "CUDA_CORES_ONLY", "TENSOR_CORES", "device_status",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libspin.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "spin.h")

NO_ROTATE = 1
CUDA_CORES_ONLY = 2
TENSOR_CORES = 4
SYM_INT4_F32SCALE = 0
ASYM_INT4_F16SZ = 1
BF16 = 0
F32 = 1

_STATUS = {0: "SPIN_OK", 1: "SPIN_ERR_INVALID_ARG", 2: "SPIN_ERR_UNSUPPORTED_SIZE",
           3: "SPIN_ERR_MISALIGNED", 4: "SPIN_ERR_CUDA", 5: "SPIN_ERR_DEVICE"}


class SpinError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{fn} returned {_STATUS.get(status, status)}"
        if status == 4:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


_lib = None


def lib() -> C.CDLL:
    """Load libspin.so from this package directory (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python online_hadamard_rotation_b200/build.py` (there is no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    vp, i64, i32, u32, f32 = C.c_void_p, C.c_int64, C.c_int32, C.c_uint32, C.c_float
    L.spin_hadamard_quant_int4.argtypes = [vp, i64, i32, f32, vp, vp, vp]
    L.spin_hadamard_quant_int4_ex.argtypes = [vp, i64, i32, f32, vp, u32, vp, vp, vp]
    L.spin_rope_hadamard_kvquant.argtypes = [vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, f32, vp, vp, vp,
                                             vp, vp, vp, vp, i32, i32, vp]
    L.spin_hadamard_quant_int8.argtypes = [vp, i64, i32, f32, vp, u32, vp, vp, vp]
    L.spin_dequant_hadamard_inverse.argtypes = [vp, i64, i32, i32, vp, vp, vp, u32, vp, i32, vp]
    L.spin_hadamard_quant_kron.argtypes = [vp, i64, i32, i32, f32, vp, u32, i32, vp, vp, vp]
    L.spin_decode_attention_int4kv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, i32,
                                               vp, C.c_size_t, vp]
    L.spin_w4a4_gemm.argtypes = [vp, vp, i64, vp, vp, i32, i32, vp, i32, vp]
    L.spin_decode_attention_workspace_bytes.argtypes = [i32, i32, i32]
    L.spin_decode_attention_workspace_bytes.restype = C.c_size_t
    for name in ("spin_hadamard_quant_int4", "spin_hadamard_quant_int4_ex", "spin_hadamard_quant_int8",
                 "spin_rope_hadamard_kvquant", "spin_dequant_hadamard_inverse", "spin_hadamard_quant_kron",
                 "spin_decode_attention_int4kv", "spin_w4a4_gemm"):
        getattr(L, name).restype = C.c_int
    L.spin_uses_tensor_cores.argtypes = [i32, i64, i32, u32, i32]
    L.spin_uses_tensor_cores.restype = C.c_int
    L.spin_test_stall_tensor_core_waits.argtypes = [C.c_int]
    L.spin_test_stall_tensor_core_waits.restype = None
    L.spin_device_status.argtypes = [C.POINTER(C.c_uint32), C.c_int]
    L.spin_device_status.restype = C.c_int
    L.spin_status_string.argtypes = [C.c_int]
    L.spin_status_string.restype = C.c_char_p
    L.spin_last_cuda_error.restype = C.c_int
    L.spin_version.restype = C.c_int
    _lib = L
    return L


def exported_symbols() -> list[str]:
    """Function names declared in include/spin.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(spin_\w+)\s*\(", text, flags=re.M)))


# ------------------------------------------------------------------ raw C ABI (pointers)
def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SpinError(fn, status, lib().spin_last_cuda_error())


def spin_hadamard_quant_int4(x_bf16, tokens, n, clip, q_packed_u8, scales_f32, stream) -> int:
    return lib().spin_hadamard_quant_int4(x_bf16, tokens, n, clip, q_packed_u8, scales_f32, stream)


def spin_hadamard_quant_int4_ex(x_bf16, tokens, n, clip, sign_bits, flags, q_packed_u8, scales_f32,
                                stream) -> int:
    return lib().spin_hadamard_quant_int4_ex(x_bf16, tokens, n, clip, sign_bits, flags, q_packed_u8,
                                             scales_f32, stream)


def spin_hadamard_quant_int8(x_bf16, tokens, n, clip, sign_bits, flags, q_i8, scales_f32, stream) -> int:
    return lib().spin_hadamard_quant_int8(x_bf16, tokens, n, clip, sign_bits, flags, q_i8, scales_f32, stream)


def spin_hadamard_quant_kron(x_bf16, tokens, m, n, clip, sign_bits, flags, bits, q, scales_f32, stream) -> int:
    return lib().spin_hadamard_quant_kron(x_bf16, tokens, m, n, clip, sign_bits, flags, bits, q, scales_f32, stream)


def spin_decode_attention_int4kv(*args) -> int:
    return lib().spin_decode_attention_int4kv(*args)


def spin_w4a4_gemm(*args) -> int:
    return lib().spin_w4a4_gemm(*args)


def spin_rope_hadamard_kvquant(*args) -> int:
    return lib().spin_rope_hadamard_kvquant(*args)


def spin_dequant_hadamard_inverse(*args) -> int:
    return lib().spin_dequant_hadamard_inverse(*args)


# ------------------------------------------------------------------ torch-level helpers
def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t: torch.Tensor, name: str, dtype, device=None, shape=None):
    """Argument checks before a pointer reaches the library: dtype, a contiguous CUDA
    tensor (a host pointer would reach a kernel), the expected device and shape."""
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _need_signs(signs, n: int, device) -> None:
    if signs is not None:
        _need(signs, "signs", torch.int32, device)
        if signs.numel() < max(1, n // 32):
            raise ValueError(f"signs: expected {max(1, n // 32)} words for n = {n}, got {signs.numel()}")


def _r4_args(x, out, scales, signs, code_dtype, code_cols):
    _need(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError(f"x: expected [tokens, n], got shape {tuple(x.shape)}")
    tokens, n = x.shape
    if out is None:
        out = torch.empty((tokens, code_cols(n)), dtype=code_dtype, device=x.device)
    _need(out, "out", code_dtype, x.device, (tokens, code_cols(n)))
    if scales is None:
        scales = torch.empty((tokens,), dtype=torch.float32, device=x.device)
    _need(scales, "scales", torch.float32, x.device, (tokens,))
    _need_signs(signs, n, x.device)
    return tokens, n, out, scales


def test_stall_tensor_core_waits(enable: bool) -> None:
    """Failure-detection test hook (see spin_test_stall_tensor_core_waits)."""
    lib().spin_test_stall_tensor_core_waits(1 if enable else 0)


OP_HADAMARD_QUANT = 0
OP_DEQUANT_INVERSE = 1


def uses_tensor_cores(op: int, rows: int, n: int, flags: int = 0, has_signs: bool = False) -> bool:
    """Whether a call would run a tensor-core kernel (host-only query of the library's
    dispatch; see spin_uses_tensor_cores)."""
    r = lib().spin_uses_tensor_cores(int(op), int(rows), int(n), int(flags), 1 if has_signs else 0)
    if r < 0:
        raise ValueError(f"invalid arguments for op {op}: rows={rows} n={n} flags={flags}")
    return bool(r)


def device_status(reset: bool = False) -> int:
    """Device status word (nonzero: a kernel gave up on an internal wait)."""
    v = C.c_uint32(0)
    _check("spin_device_status", lib().spin_device_status(C.byref(v), 1 if reset else 0))
    return int(v.value)


def hadamard_quant_int4(x: torch.Tensor, clip: float = 1.0, signs: torch.Tensor | None = None,
                        no_rotate: bool = False, out: torch.Tensor | None = None,
                        scales: torch.Tensor | None = None, stream=None, cuda_cores_only: bool = False,
                        tensor_cores: bool = False):
    """R4: x [tokens, n] bf16 (CUDA) -> (codes [tokens, n/2] uint8, scales [tokens] fp32)."""
    tokens, n, out, scales = _r4_args(x, out, scales, signs, torch.uint8, lambda n: n // 2)
    flags = ((NO_ROTATE if no_rotate else 0) | (CUDA_CORES_ONLY if cuda_cores_only else 0) |
             (TENSOR_CORES if tensor_cores else 0))
    st = spin_hadamard_quant_int4_ex(_ptr(x), tokens, n, float(clip), _ptr(signs), flags,
                                     _ptr(out), _ptr(scales), _stream(stream))
    _check("spin_hadamard_quant_int4_ex", st)
    return out, scales


def hadamard_quant_int8(x: torch.Tensor, clip: float = 1.0, signs: torch.Tensor | None = None,
                        no_rotate: bool = False, out: torch.Tensor | None = None,
                        scales: torch.Tensor | None = None, stream=None, cuda_cores_only: bool = False,
                        tensor_cores: bool = False):
    """R4 with INT8 codes: x [tokens, n] bf16 (CUDA) -> (codes [tokens, n] int8, scales [tokens] fp32)."""
    tokens, n, out, scales = _r4_args(x, out, scales, signs, torch.int8, lambda n: n)
    flags = ((NO_ROTATE if no_rotate else 0) | (CUDA_CORES_ONLY if cuda_cores_only else 0) |
             (TENSOR_CORES if tensor_cores else 0))
    st = spin_hadamard_quant_int8(_ptr(x), tokens, n, float(clip), _ptr(signs), flags, _ptr(out), _ptr(scales),
                                  _stream(stream))
    _check("spin_hadamard_quant_int8", st)
    return out, scales


_host_streams = {}


def _pipeline_streams(device):
    """Three streams per device (copy in, compute, copy out), created once."""
    key = torch.device(device).index
    if key not in _host_streams:
        _host_streams[key] = tuple(torch.cuda.Stream(device) for _ in range(3))
    return _host_streams[key]


def hadamard_quant_kron(x: torch.Tensor, m: int, clip: float = 1.0, signs: torch.Tensor | None = None,
                        bits: int = 4, out: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                        stream=None):
    """R4 for n = m 2^k (H_m of Paley (x) Sylvester H_{2^k}): x [tokens, n] bf16 (CUDA) ->
    (codes [tokens, n/2] uint8 for bits = 4, or [tokens, n] int8 for bits = 8; scales [tokens] fp32)."""
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    ctype, cols = (torch.uint8, lambda n: n // 2) if bits == 4 else (torch.int8, lambda n: n)
    tokens, n, out, scales = _r4_args(x, out, scales, signs, ctype, cols)
    st = spin_hadamard_quant_kron(_ptr(x), tokens, int(m), n, float(clip), _ptr(signs), 0, bits, _ptr(out),
                                  _ptr(scales), _stream(stream))
    _check("spin_hadamard_quant_kron", st)
    return out, scales


def w4a4_gemm(x_codes: torch.Tensor, x_scales: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor,
              out_dtype=torch.float32, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W4A4 GEMM on packed INT4 codes: x_codes [tokens, k/2] uint8 and x_scales [tokens]
    fp32 (as hadamard_quant_int4 / hadamard_quant_kron return them), w_codes [n_out, k/2]
    uint8 and w_scales [n_out] fp32 (weight rows packed the same way) -> out [tokens, n_out]
    = x_scales[t] w_scales[o] sum_k q_x q_w, fp32 or bf16."""
    _need(x_codes, "x_codes", torch.uint8)
    if x_codes.dim() != 2 or w_codes.dim() != 2:
        raise ValueError("x_codes and w_codes must be 2-D [rows, k/2]")
    tokens, kh = x_codes.shape
    n_out = w_codes.shape[0]
    _need(w_codes, "w_codes", torch.uint8, x_codes.device, (n_out, kh))
    _need(x_scales, "x_scales", torch.float32, x_codes.device, (tokens,))
    _need(w_scales, "w_scales", torch.float32, x_codes.device, (n_out,))
    if out is None:
        if out_dtype not in (torch.float32, torch.bfloat16):
            raise TypeError(f"out_dtype: expected torch.float32 or torch.bfloat16, got {out_dtype}")
        out = torch.empty((tokens, n_out), dtype=out_dtype, device=x_codes.device)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"out: expected torch.float32 or torch.bfloat16, got {out.dtype}")
    _need(out, "out", out.dtype, x_codes.device, (tokens, n_out))
    st = spin_w4a4_gemm(_ptr(x_codes), _ptr(x_scales), tokens, _ptr(w_codes), _ptr(w_scales), n_out, 2 * kh,
                        _ptr(out), F32 if out.dtype == torch.float32 else BF16, _stream(stream))
    _check("spin_w4a4_gemm", st)
    return out


def hadamard_quant_host(x_host: torch.Tensor, clip: float = 1.0, signs: torch.Tensor | None = None, bits: int = 4,
                        device=None, stream=None, buffers=None, chunks: int = 8, m: int | None = None):
    """End-to-end R4 from host memory: copy x (pinned, bf16 [tokens, n]) to the
    device, run the kernel, copy codes and steps back into pinned host tensors.
    The batch is cut into `chunks` slices of whole tokens that flow through three
    streams, so the copy in of one slice, the kernel of the previous one and the
    copy out of the one before overlap. Work is ordered after what is already
    enqueued on `stream` (default: the current stream), which is made to wait for
    all of it; the call synchronises `stream` before it returns (codes_host,
    steps_host). `buffers` (from a previous call's return of the same shape) may
    be passed to reuse the device and pinned buffers. With `m`, the row length is
    n = m 2^k and the kernel is hadamard_quant_kron's."""
    device = torch.device(device or "cuda")
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    if x_host.dim() != 2 or x_host.dtype != torch.bfloat16 or x_host.is_cuda:
        raise ValueError("x_host: expected a host [tokens, n] bfloat16 tensor")
    tokens, n = x_host.shape
    cols, ctype = (n // 2, torch.uint8) if bits == 4 else (n, torch.int8)
    if buffers is None:
        buffers = dict(
            x=torch.empty((tokens, n), dtype=torch.bfloat16, device=device),
            q=torch.empty((tokens, cols), dtype=ctype, device=device),
            s=torch.empty((tokens,), dtype=torch.float32, device=device),
            q_host=torch.empty((tokens, cols), dtype=ctype, pin_memory=True),
            s_host=torch.empty((tokens,), dtype=torch.float32, pin_memory=True))
    if m is not None:
        def quant(x, clip, signs, out, scales, stream):
            return hadamard_quant_kron(x, m, clip, signs, bits, out, scales, stream)
    else:
        quant = hadamard_quant_int4 if bits == 4 else hadamard_quant_int8
    s0 = stream or torch.cuda.current_stream(device)
    h2d, comp, d2h = _pipeline_streams(device)
    start = torch.cuda.Event()
    start.record(s0)
    for st in (h2d, comp, d2h):
        st.wait_event(start)
    step = max(1, -(-tokens // max(1, chunks)))
    for t0 in range(0, tokens, step):
        t1 = min(tokens, t0 + step)
        with torch.cuda.stream(h2d):
            buffers["x"][t0:t1].copy_(x_host[t0:t1], non_blocking=True)
        comp.wait_stream(h2d)
        quant(buffers["x"][t0:t1], clip, signs, out=buffers["q"][t0:t1], scales=buffers["s"][t0:t1], stream=comp)
        d2h.wait_stream(comp)
        with torch.cuda.stream(d2h):
            buffers["q_host"][t0:t1].copy_(buffers["q"][t0:t1], non_blocking=True)
            buffers["s_host"][t0:t1].copy_(buffers["s"][t0:t1], non_blocking=True)
    s0.wait_stream(d2h)
    s0.synchronize()
    return buffers["q_host"], buffers["s_host"], buffers


def hadamard_quant_int4_host(x_host: torch.Tensor, clip: float = 1.0, signs: torch.Tensor | None = None,
                             device=None, stream=None, buffers=None, chunks: int = 8):
    """hadamard_quant_host with INT4 codes; returns (codes_host, steps_host)."""
    q, s, _ = hadamard_quant_host(x_host, clip, signs, 4, device, stream, buffers, chunks)
    return q, s


def alloc_kv_cache(batch: int, n_kv_heads: int, cache_len: int, head_dim: int = 128, device="cuda"):
    """Caller-owned INT4 KV cache buffers in the layout the kernel writes."""
    return dict(
        k_cache=torch.zeros((batch, n_kv_heads, cache_len, head_dim // 2), dtype=torch.uint8, device=device),
        v_cache=torch.zeros((batch, n_kv_heads, cache_len, head_dim // 2), dtype=torch.uint8, device=device),
        k_scale=torch.zeros((batch, n_kv_heads, cache_len), dtype=torch.float16, device=device),
        k_zero=torch.zeros((batch, n_kv_heads, cache_len), dtype=torch.float16, device=device),
        v_scale=torch.zeros((batch, n_kv_heads, cache_len), dtype=torch.float16, device=device),
        v_zero=torch.zeros((batch, n_kv_heads, cache_len), dtype=torch.float16, device=device))


def rope_hadamard_kvquant(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
                          cache: dict, theta: float = 10000.0, clip: float = 1.0, cache_offset: int = 0,
                          q_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """R3 + INT4 KV: q [B,S,hq,d], k/v [B,S,hkv,d] bf16, pos [B,S] int32.
    Writes the cache dict (see alloc_kv_cache) and returns rotated Q (bf16)."""
    _need(q, "q", torch.bfloat16)
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k and v are [batch, seq, heads, head_dim]")
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    _need(k, "k", torch.bfloat16, q.device, (B, S, hkv, d))
    _need(v, "v", torch.bfloat16, q.device, (B, S, hkv, d))
    _need(pos, "pos", torch.int32, q.device, (B, S))
    if q_out is None:
        q_out = torch.empty_like(q)
    _need(q_out, "q_out", torch.bfloat16, q.device, (B, S, hq, d))
    cache_len = cache["k_cache"].shape[2]
    for name in ("k_cache", "v_cache"):
        _need(cache[name], name, torch.uint8, q.device, (B, hkv, cache_len, d // 2))
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        _need(cache[name], name, torch.float16, q.device, (B, hkv, cache_len))
    if cache_offset < 0 or cache_offset + S > cache_len:
        raise ValueError(f"cache slots {cache_offset} .. {cache_offset + S - 1} outside a cache of {cache_len}")
    st = spin_rope_hadamard_kvquant(
        _ptr(q), _ptr(k), _ptr(v), _ptr(pos), float(theta), d, B, S, hq, hkv, float(clip), _ptr(q_out),
        _ptr(cache["k_cache"]), _ptr(cache["v_cache"]), _ptr(cache["k_scale"]), _ptr(cache["k_zero"]),
        _ptr(cache["v_scale"]), _ptr(cache["v_zero"]), cache_len, cache_offset, _stream(stream))
    _check("spin_rope_hadamard_kvquant", st)
    return q_out


def decode_attention_workspace_bytes(batch: int, n_q_heads: int, cache_len: int) -> int:
    """Scratch bytes decode_attention_int4kv needs (see spin_decode_attention_workspace_bytes)."""
    return int(lib().spin_decode_attention_workspace_bytes(int(batch), int(n_q_heads), int(cache_len)))


def decode_attention_int4kv(q: torch.Tensor, cache: dict, lens: torch.Tensor, softmax_scale: float | None = None,
                            out_dtype=torch.float32, out: torch.Tensor | None = None,
                            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One decode step over the INT4 KV cache: q [B, hq, d] bf16 (rotated queries),
    cache as alloc_kv_cache returns it ([B, hkv, L, d/2] codes, [B, hkv, L] fp16 scale
    and zero), lens [B] int32 slots attended. Returns out [B, hq, d] (fp32 or bf16).
    `workspace` (uint8, at least decode_attention_workspace_bytes) is allocated
    through torch when not given."""
    _need(q, "q", torch.bfloat16)
    if q.dim() != 3:
        raise ValueError(f"q: expected [batch, n_q_heads, head_dim], got shape {tuple(q.shape)}")
    B, hq, d = q.shape
    hkv, L = cache["k_cache"].shape[1], cache["k_cache"].shape[2]
    for name in ("k_cache", "v_cache"):
        _need(cache[name], name, torch.uint8, q.device, (B, hkv, L, d // 2))
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        _need(cache[name], name, torch.float16, q.device, (B, hkv, L))
    _need(lens, "lens", torch.int32, q.device, (B,))
    if out is None:
        if out_dtype not in (torch.float32, torch.bfloat16):
            raise TypeError(f"out_dtype: expected torch.float32 or torch.bfloat16, got {out_dtype}")
        out = torch.empty((B, hq, d), dtype=out_dtype, device=q.device)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"out: expected torch.float32 or torch.bfloat16, got {out.dtype}")
    _need(out, "out", out.dtype, q.device, (B, hq, d))
    need = decode_attention_workspace_bytes(B, hq, L)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8, q.device)
    scale = float(softmax_scale) if softmax_scale is not None else 1.0 / float(d) ** 0.5
    st = spin_decode_attention_int4kv(
        _ptr(q), _ptr(cache["k_cache"]), _ptr(cache["v_cache"]), _ptr(cache["k_scale"]), _ptr(cache["k_zero"]),
        _ptr(cache["v_scale"]), _ptr(cache["v_zero"]), _ptr(lens), B, hq, hkv, d, L, scale, _ptr(out),
        F32 if out.dtype == torch.float32 else BF16, _ptr(workspace), workspace.numel(), _stream(stream))
    _check("spin_decode_attention_int4kv", st)
    return out


def dequant_hadamard_inverse(codes: torch.Tensor, n: int, scale: torch.Tensor, zero: torch.Tensor | None = None,
                             mode: int = SYM_INT4_F32SCALE, signs: torch.Tensor | None = None,
                             no_rotate: bool = False, out_dtype=torch.float32, out: torch.Tensor | None = None,
                             stream=None, cuda_cores_only: bool = False, tensor_cores: bool = False) -> torch.Tensor:
    """codes [..., n/2] uint8 -> out [..., n] (rows = codes.numel() / (n/2)).
    cuda_cores_only / tensor_cores select the kernel (SPIN_CUDA_CORES_ONLY /
    SPIN_TENSOR_CORES); by default the library picks."""
    _need(codes, "codes", torch.uint8)
    if n < 2 or codes.dim() < 1 or codes.shape[-1] != n // 2:
        raise ValueError(f"codes: expected [..., {n // 2}] for n = {n}, got shape {tuple(codes.shape)}")
    rows = codes.numel() // (n // 2)
    if mode not in (SYM_INT4_F32SCALE, ASYM_INT4_F16SZ):
        raise ValueError(f"mode {mode}: expected SYM_INT4_F32SCALE or ASYM_INT4_F16SZ")
    asym = mode == ASYM_INT4_F16SZ
    _need(scale, "scale", torch.float16 if asym else torch.float32, codes.device)
    if scale.numel() != rows:
        raise ValueError(f"scale: expected {rows} values, got {scale.numel()}")
    if asym:
        if zero is None:
            raise ValueError("zero is required for ASYM_INT4_F16SZ")
        _need(zero, "zero", torch.float16, codes.device)
        if zero.numel() != rows:
            raise ValueError(f"zero: expected {rows} values, got {zero.numel()}")
    _need_signs(signs, n, codes.device)
    if out is None:
        if out_dtype not in (torch.float32, torch.bfloat16):
            raise TypeError(f"out_dtype: expected torch.float32 or torch.bfloat16, got {out_dtype}")
        out = torch.empty(tuple(codes.shape[:-1]) + (n,), dtype=out_dtype, device=codes.device)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"out: expected torch.float32 or torch.bfloat16, got {out.dtype}")
    _need(out, "out", out.dtype, codes.device, tuple(codes.shape[:-1]) + (n,))
    dt = F32 if out.dtype == torch.float32 else BF16
    flags = (NO_ROTATE if no_rotate else 0) | (CUDA_CORES_ONLY if cuda_cores_only else 0) | \
        (TENSOR_CORES if tensor_cores else 0)
    st = spin_dequant_hadamard_inverse(_ptr(codes), rows, n, mode, _ptr(scale), _ptr(zero), _ptr(signs),
                                       flags, _ptr(out), dt, _stream(stream))
    _check("spin_dequant_hadamard_inverse", st)
    return out
