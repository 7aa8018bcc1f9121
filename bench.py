"""Benchmark of the fused online-Hadamard + INT4 path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl spin|reference] [--workload NAME]

A step is one pass of the R4 hot path (bf16 load, +-1 diagonal, Walsh-Hadamard
transform, per-token max, scale, round, clamp, nibble pack, store) over one
batch of the default workload: 8192 tokens x n = 16384, SwiGLU-like bf16
input with 0.1 % outlier channels, seeded +-1 diagonal, clip 0.9. Inputs are
synthetic and seeded (synthetic/), generated on the host and resident in HBM
before timing; the input (268 MB) is larger than L2 (126 MB) and two input and
output sets alternate between steps.

With N > 1 (torchrun, one process per GPU) every rank processes its own batch
(weak scaling, no data exchange: tokens are independent); the elapsed time is
the maximum over ranks and the value counts all ranks' tokens.

Printed as one JSON line on rank 0. `value` is the algorithmic HBM throughput
(bytes the method must move: bf16 in, packed codes and fp32 scales out) in
GB/s; tokens/s and the fraction of the measured HBM copy bandwidth are in the
same line. `--impl reference` times the fp64 CPU oracle on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused Hadamard+INT4-quant HBM GB/s (% of B200 peak) and tokens/s at n=16384"
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def metric_for(wl) -> str:
    """The headline metric, or its counterpart for the INT8, other-n, Kronecker-size,
    R3 + KV and decode-attention workloads."""
    if wl.get("kind") == "attn":
        return "decode attention over the INT4 KV cache: HBM GB/s (% of B200 peak) and us per step"
    if wl.get("kind") == "r3":
        return ("fused RoPE + Hadamard (R3) on Q/K + asymmetric INT4 KV-cache quant: HBM GB/s (% of B200 peak) "
                "and tokens/s at head_dim=128")
    if wl.get("kind") == "gemm":
        T, K = wl["bits"].shape
        return (f"W4A4 GEMM on the R4 kernel's INT4 codes (tcgen05 kind::i8): TOPS (% of int8 tensor peak) at "
                f"{T} x {wl['n_out']} x k={K}")
    m = METRIC.replace("INT4", "INT8") if wl.get("code_bits", 4) == 8 else METRIC
    n = int(wl["bits"].shape[1]) if "bits" in wl else 16384
    if wl.get("kron_m"):
        m = m.replace("at n=16384", f"at n={n} (H_{wl['kron_m']} Paley x Sylvester)")
    elif n != 16384:
        m = m.replace("at n=16384", f"at n={n}")
    return m


def algorithmic_bytes_r4(tokens: int, n: int, code_bits: int = 4) -> int:
    """bf16 in (2n) + codes out (n/2 packed INT4 or n INT8) + fp32 scale out (4), per token."""
    return tokens * (2 * n + n * code_bits // 8 + 4)


def oracle_r4_rows(oracle, bits, clip, signs, code_bits, threads=1, kron_m=None) -> int:
    """The oracle over rows: its C loop for INT4 (rows spread over `threads`; the
    Kronecker loop for n = m 2^k), one call per row for INT8 (one thread). Returns
    the threads used."""
    if kron_m:
        oracle.r4_rows_kron(bits, kron_m, clip, signs, threads=threads)
        return threads
    if code_bits == 4:
        oracle.r4_rows(bits, clip, signs, threads=threads)
        return threads
    for row in bits:
        oracle.r4_row_int8(row, clip, signs=signs)
    return 1


def r4_kernel_name(n: int, tokens: int, has_signs: bool, code_bits: int = 4) -> str:
    """The R4 kernel the library's dispatch picks by default, asked of the library
    itself (spin_uses_tensor_cores, a host-only query)."""
    import online_hadamard_rotation_b200 as spin
    if spin.uses_tensor_cores(spin.OP_HADAMARD_QUANT, tokens, n, 0, has_signs):
        return "k1_tcs_rotate_quant" if n <= 256 else "k1_tc_rotate_quant"
    return f"k1_rotate_quant_int{code_bits}"


def k3_kernel_name(n: int, rows: int) -> str:
    """The dequantise + inverse kernel the library's dispatch picks by default (asked
    of the library, as above)."""
    import online_hadamard_rotation_b200 as spin
    if spin.uses_tensor_cores(spin.OP_DEQUANT_INVERSE, rows, n):
        return "k3_tcs_dequant_inverse" if n <= 256 else "k3_tc_dequant_inverse"
    return "k3_dequant_inverse"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def int8_peak_tops():
    """Dense int8 tensor peak for a kernel timed inside a sustained loop: the measured
    sustained bf16 GEMM throughput times the nominal int8 : bf16 dense ratio (4.5 : 2.25
    PFLOP/s on B200)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return 2.0 * float(d["bf16_tflops_sustained"]), "2 x measured bf16_tflops_sustained (int8 : bf16 = 2)"
    return 2.0 * 1400.0, "2 x fallback sustained bf16 1.4 PFLOP/s (int8 : bf16 = 2)"


def kernel_source_digest(kernel: str) -> str:
    """Hash of the sources a kernel is built from: the .cu files of its family
    (k1_, k2_, k3_) and the shared device headers."""
    family = kernel.split("_")[0] + "_"
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "online_hadamard_rotation_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith(family) or name in ("spin_tile.cuh", "tc_ptx.cuh"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(key: str):
    """Per-launch DRAM bytes from the committed ncu summary (key "kernel:workload"),
    if it was taken on the current kernel source; None otherwise."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f).get(key)
    if not d or d.get("source_digest") != kernel_source_digest(key.split(":")[0]):
        return None
    return d.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    smax.append(float(p[2]))
                except ValueError:
                    continue
                for name, val in zip(names, p[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def max_over_ranks(value: float, device) -> float:
    """The largest value over all ranks (elapsed times are reported this way)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(world: int, unit_bytes: int, unit_count: int, steps: int, ms: float):
    """Whole-job GB/s and units/s: every rank processes `unit_count` units per
    step (weak scaling); `ms` is the maximum elapsed time over ranks."""
    sec = ms / 1e3
    return world * unit_bytes * steps / sec / 1e9, world * unit_count * steps / sec


def make_workload(name: str, rank: int, tokens: int | None = None):
    """The workload one rank processes; every rank draws its own shard (seed + rank)."""
    import synthetic
    if name in ("r4_prefill", "r4_prefill_int8"):
        bits, signs, _ = synthetic.r4_prefill(tokens=tokens or 8192, seed=1 + rank)
        code_bits = 8 if name.endswith("int8") else 4
        return dict(kind="r4", bits=bits, signs=signs, clip=0.9, code_bits=code_bits,
                    desc={"workload": "R4 prefill: 4x2048 tokens x n=16384 bf16, SwiGLU-like, 0.1% channels x100, "
                                      "seeded +-1 diagonal, H_16384 = H_128 (x) H_128, clip 0.9"
                                      + (", per-token INT8 codes" if code_bits == 8 else ""),
                          "tokens": int(bits.shape[0]), "n": int(bits.shape[1])})
    if name.startswith("decode_attn"):
        batch = int(name[len("decode_attn_b"):]) if name.startswith("decode_attn_b") else 4
        q, k, v, pos = synthetic.r3_kv(batch=batch, seed=2 + rank)
        return dict(kind="attn", q=q, k=k, v=v, pos=pos, clip=0.95,
                    desc={"workload": f"decode attention over the INT4 KV cache: batch {batch} x 4096 cached slots "
                                      "(the R3+KV workload's cache, written by the R3 kernel), 32 q / 8 kv heads, "
                                      "head_dim 128, one query token per row", "tokens": batch})
    if name == "w4a4_gemm":
        T = tokens or 8192
        bits, signs, _ = synthetic.r4_prefill(tokens=T, n=14336, seed=1 + rank)
        return dict(kind="gemm", bits=bits, w_bits=synthetic.weights(4096, 14336, seed=7 + rank), signs=signs,
                    kron_m=28, clip=0.9, n_out=4096,
                    desc={"workload": f"W4A4 GEMM at the LLaMA-3 8B down-projection shape: {T} tokens x k = 14336 "
                                      "(the R4 kernel's codes of the n = 14336 prefill: H_28 Paley (x) H_512, seeded "
                                      "+-1 diagonal, clip 0.9) against 4096 output channels (N(0, 1/k) bf16 weight "
                                      "rows baked by the same kernel, clip 1.0); bf16 output",
                          "tokens": T, "n_out": 4096, "k": 14336,
                          "l2": "operands (88 MB of codes) stay L2-resident across steps, as for any GEMM"})
    if name.startswith("kron"):
        n = int(name[len("kron"):] or 14336)
        m = {14336: 28, 6144: 12, 10240: 20, 12288: 12}[n]
        bits, signs, _ = synthetic.r4_prefill(tokens=tokens or 8192, n=n, seed=1 + rank)
        return dict(kind="r4", bits=bits, signs=signs, clip=0.9, code_bits=4, kron_m=m,
                    desc={"workload": f"R4 prefill at n={n} = {m} x {n // m} (H_{m} Paley (x) H_{n // m}): "
                                      f"{bits.shape[0]} tokens, SwiGLU-like bf16, 0.1% channels x100, seeded +-1 "
                                      "diagonal, clip 0.9", "tokens": int(bits.shape[0]), "n": n, "m": m})
    if name.startswith("decode"):
        n = int(name[len("decode"):] or 16384)
        bits = synthetic.decode(tokens or 32, n, seed=3 + rank)
        return dict(kind="r4", bits=bits, signs=None, clip=1.0, code_bits=4,
                    desc={"workload": f"decode: 32 tokens x n={n} Student-t(3), one channel x200 per row, clip 1.0",
                          "tokens": int(bits.shape[0]), "n": n})
    if name.startswith("sweep"):
        k = int(name[len("sweep"):])
        bits = synthetic.sweep(k, tokens=tokens, seed=4 + k + 100 * rank)
        return dict(kind="r4", bits=bits, signs=None, clip=1.0, code_bits=4,
                    desc={"workload": f"sweep: n=2^{k}, {'1 GiB' if tokens is None else f'{bits.nbytes >> 20} MiB'} "
                                      "bf16 input, N(0,1) with 0.1% channels x100, clip 1.0",
                          "tokens": int(bits.shape[0]), "n": 1 << k})
    if name == "r3_kv":
        q, k, v, pos = synthetic.r3_kv(seed=2 + rank)
        return dict(kind="r3", q=q, k=k, v=v, pos=pos, clip=0.95,
                    desc={"workload": "R3+KV: batch 4 x seq 4096, 32 q / 8 kv heads, head_dim 128, RoPE theta 1e4, "
                                      "asym INT4 KV cache, clip 0.95", "tokens": 4 * 4096})
    raise SystemExit(f"unknown workload {name}")


def config_for(wl, world: int, workload: str) -> dict:
    """The `config` object both arms print (same workload, same keys)."""
    l2 = ("inputs larger than L2 (268 MB bf16 input vs 126 MB L2); two buffer sets alternate"
          if workload.startswith("r4_prefill") else "two buffer sets alternate")
    return dict(wl["desc"], parallelism=f"dp{world}" if world > 1 else "single GPU", l2=wl["desc"].get("l2", l2))


def r3_bytes(tokens, hq=32, hkv=8, d=128):
    return tokens * (2 * hq * d * 2 + 2 * hkv * d * 2 + 2 * hkv * d // 2 + 4 * hkv * 2 + 4)


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle on the host cores
# ---------------------------------------------------------------------------
def attn_bytes(B, S, hq, hkv, d=128):
    """Bytes one decode-attention step must move: both caches' codes, fp16 scales and
    zeros, the bf16 queries and the fp32 output."""
    return B * hkv * S * (2 * d // 2 + 4 * 2) + B * hq * d * (2 + 4)


def run_reference_attn(args, wl):
    """The oracle's decode attention over the oracle's own cache of the workload, all
    batch rows spread over the host's cores."""
    import oracle
    oracle.lib()
    q, k, v, pos = wl["q"], wl["k"], wl["v"], wl["pos"]
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    threads = oracle.max_threads()
    ref = oracle.r3_batch(q, k, v, pos, 1e4, wl["clip"], cache_len=S, threads=threads)
    qs = ref["q_out"][:, S - 1]
    lens = [S] * B
    for _ in range(args.warmup):
        oracle.decode_attention(qs[:1], {n: a[:1] for n, a in ref.items() if n != "q_out"}, lens[:1])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.decode_attention(qs, ref, lens, threads=threads)
    dt = time.perf_counter() - t0
    gbs = attn_bytes(B, S, hq, hkv, d) * args.steps / dt / 1e9
    line = {"impl": "reference", "metric": metric_for(wl), "value": gbs, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_for(wl, args.gpus, args.workload),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"the whole batch ({B} rows x {S} slots) per step, fp64, rows over "
                                       f"{threads} host thread(s)"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_gemm(args, wl):
    """The oracle's pipeline on a bounded sample: the first 16 token rows through the R4
    rows and all weight rows baked once, then the GEMM of those rows against every output
    channel, all host cores; TOPS of the GEMM part."""
    import oracle
    oracle.lib()
    threads = oracle.max_threads()
    rows = 16
    xq, xs = oracle.r4_rows_kron(wl["bits"][:rows], wl["kron_m"], wl["clip"], wl["signs"], threads=threads)
    wq, ws = oracle.r4_rows_kron(wl["w_bits"], wl["kron_m"], 1.0, wl["signs"], threads=threads)
    for _ in range(args.warmup):
        oracle.w4a4_gemm(xq[:1], xs[:1], wq, ws, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.w4a4_gemm(xq, xs, wq, ws, threads=threads)
    dt = time.perf_counter() - t0
    tops = 2 * rows * wq.shape[0] * 2 * wq.shape[1] * args.steps / dt / 1e12
    line = {"impl": "reference", "metric": metric_for(wl), "value": tops, "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": config_for(wl, args.gpus, args.workload),
            "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": threads, "kind": "oracle",
                             "sample": f"{rows} of {wl['bits'].shape[0]} token rows per step against all "
                                       f"{wq.shape[0]} outputs, exact int64 sums, {threads} host thread(s)"},
            "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference(args, wl):
    import oracle
    oracle.lib()
    if wl["kind"] == "attn":
        return run_reference_attn(args, wl)
    if wl["kind"] == "gemm":
        return run_reference_gemm(args, wl)
    if wl["kind"] != "r4":
        raise SystemExit("the reference arm times the R4 and decode-attention workloads")
    bits, n = wl["bits"], wl["bits"].shape[1]
    sample = min(bits.shape[0], max(8, (1 << 22) // n))  # about 0.1-0.2 s of oracle work per step
    rows = bits[:sample]
    threads = oracle.max_threads()  # the host's cores
    for _ in range(args.warmup):
        oracle_r4_rows(oracle, rows[:1], wl["clip"], wl["signs"], wl["code_bits"], threads, wl.get("kron_m"))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cores = oracle_r4_rows(oracle, rows, wl["clip"], wl["signs"], wl["code_bits"], threads, wl.get("kron_m"))
    dt = time.perf_counter() - t0
    tok_s = args.steps * sample / dt
    gbs = algorithmic_bytes_r4(sample, n, wl["code_bits"]) * args.steps / dt / 1e9
    line = {"impl": "reference", "metric": metric_for(wl), "value": gbs, "unit": "GB/s", "tokens_per_s": tok_s,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_for(wl, args.gpus, args.workload),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"first {sample} of {bits.shape[0]} tokens per step, fp64 fast transform, "
                                       f"{cores} host thread(s), rows spread over threads"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline_leg(wl):
    """The fp64 oracle on this host over the workload's rows (all of them from
    n = 4096 up, else at most 65536): one pass on one thread, and one pass with the
    rows spread over the host's cores. Returns the baseline record and, for the
    spot check of the GPU's last timed step, (oracle module, packed codes, steps,
    rows) of the all-cores pass (INT4 workloads)."""
    import oracle
    oracle.lib()
    bits = wl["bits"]
    sample = bits.shape[0] if bits.shape[1] >= 4096 else min(bits.shape[0], 65536)
    cpu_bytes = algorithmic_bytes_r4(sample, bits.shape[1], wl["code_bits"])
    t0 = time.perf_counter()
    oracle_r4_rows(oracle, bits[:sample], wl["clip"], wl["signs"], wl["code_bits"], kron_m=wl.get("kron_m"))
    dt = time.perf_counter() - t0
    cpu = {"value": cpu_bytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle", "tokens_per_s": sample / dt,
           "sample": f"{sample} of {bits.shape[0]} tokens, one pass, fp64 fast transform, 1 thread"}
    ref = None
    t0 = time.perf_counter()
    if wl.get("kron_m"):
        used = oracle.max_threads()
        packed, scales = oracle.r4_rows_kron(bits[:sample], wl["kron_m"], wl["clip"], wl["signs"], threads=used)
        ref = (oracle, packed, scales.astype(np.float64), sample)
    elif wl["code_bits"] == 4:
        used = oracle.max_threads()
        packed, scales = oracle.r4_rows(bits[:sample], wl["clip"], wl["signs"], threads=used)
        ref = (oracle, packed, scales.astype(np.float64), sample)
    else:
        used = oracle_r4_rows(oracle, bits[:sample], wl["clip"], wl["signs"], wl["code_bits"], oracle.max_threads())
    dt = time.perf_counter() - t0
    cpu["all_cores"] = {"value": cpu_bytes / dt / 1e9, "unit": "GB/s", "cores": used, "tokens_per_s": sample / dt,
                        "sample": "the same rows, spread over the host's cores"}
    return cpu, ref


def cpu_baseline_gemm(xq, xs, wq, ws, out_dev, rows: int = 8):
    """The fp64 oracle GEMM on a bounded sample (the first `rows` token rows against every
    output channel), one thread and all host cores; the same rows of the GPU's last timed
    step must match it within the bf16 output tolerance."""
    import oracle
    oracle.lib()
    xq_h, xs_h = xq[:rows].cpu().numpy(), xs[:rows].cpu().numpy()
    wq_h, ws_h = wq.cpu().numpy(), ws.cpu().numpy()
    ops = 2 * rows * wq_h.shape[0] * 2 * wq_h.shape[1]
    t0 = time.perf_counter()
    oracle.w4a4_gemm(xq_h, xs_h, wq_h, ws_h, threads=1)
    dt1 = time.perf_counter() - t0
    used = oracle.max_threads()
    t0 = time.perf_counter()
    ref = oracle.w4a4_gemm(xq_h, xs_h, wq_h, ws_h, threads=used)
    dtn = time.perf_counter() - t0
    got = out_dev[:rows].float().cpu().numpy().astype(np.float64)
    lim = np.maximum(2e-2, np.abs(ref) * 2.0 ** -8)  # bf16 rounding of the output (round to nearest)
    bad = int(np.sum(np.abs(got - ref) > lim))
    return {"value": ops / dt1 / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
            "sample": f"{rows} token rows x {wq_h.shape[0]} outputs x k = {2 * wq_h.shape[1]}, exact int64 sums, "
                      "1 thread",
            "all_cores": {"value": ops / dtn / 1e12, "unit": "TOPS", "cores": used, "sample": "the same rows"},
            "spot_check": {"rows": rows, "outputs_off": bad, "ok": bad == 0}}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def timed_windows(step, steps, stream, dev, world, min_seconds, first=0):
    """Device time of windows of exactly `steps` calls of step(i), each window
    bracketed by a barrier (N > 1) and a device synchronisation, timed with CUDA
    events on `stream` and reduced to the maximum over ranks. Windows repeat until
    about `min_seconds` of device time is sampled (the count is fixed after the first
    window from its max-over-ranks time, so every rank runs the same number).
    Returns the list of window times in ms."""
    import torch
    import torch.distributed as dist
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    windows, target, i = [], None, first
    while target is None or len(windows) < target:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(steps):
            step(i)
            i += 1
        ev1.record(stream)
        ev1.synchronize()
        torch.cuda.synchronize()
        ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
        windows.append(ms)
        if target is None:
            target = windows_needed(ms, min_seconds)
    return windows


def windows_needed(first_ms: float, min_seconds: float) -> int:
    """Windows to time so that about `min_seconds` of device time is sampled,
    from the first window's (max-over-ranks) time; between 1 and 400."""
    return max(1, min(400, math.ceil(min_seconds * 1e3 / max(first_ms, 1e-3))))


def require_clean_status(spin, what):
    """The library's device status word must be zero after a timed loop: a kernel
    that gave up on a bounded wait stops early and would time as a faster run."""
    import torch
    torch.cuda.synchronize()
    st = spin.device_status(reset=True)
    if st:
        raise SystemExit(f"{what}: the device status word is {st:#x} (a kernel stopped early); no number reported")


def window_stats(windows, steps):
    med = statistics.median(windows)
    return med / steps, {"count": len(windows), "steps_each": steps, "ms_min": min(windows), "ms_median": med,
                         "ms_max": max(windows), "device_seconds": sum(windows) / 1e3}


def spot_check(oracle, wl, packed_ref, scales_ref, q_dev, s_dev, rows):
    """The GPU's codes and steps of `rows` (last timed step) against the oracle's
    batch output for the same rows: steps within 1e-5 relative; rows whose bytes
    differ are re-run through the single-row oracle, and every differing code must
    be one step away with the oracle's pre-round value within 1e-3 of a .5 tie."""
    q = q_dev[:rows].cpu().numpy()
    s = s_dev[:rows].cpu().numpy()
    rel = np.abs(s.astype(np.float64) - scales_ref) / np.abs(scales_ref)
    ok = bool(np.all(rel <= 1e-5))
    diff_rows = np.nonzero((q != packed_ref).any(axis=1))[0]
    bad_codes = 0
    n = wl["bits"].shape[1]
    for t in diff_rows[:4096]:
        if wl.get("kron_m"):
            r = oracle.r4_row_kron(wl["bits"][t], wl["kron_m"], wl["clip"], signs=wl["signs"])
        else:
            r = oracle.r4_row(wl["bits"][t], wl["clip"], signs=wl["signs"])
        g = q[t].astype(np.int32)
        c = np.empty(n, np.int32)
        c[0::2], c[1::2] = g & 0xF, g >> 4
        c = np.where(c >= 8, c - 16, c)
        d = c != r["codes"]
        pre = r["pre"][d]
        frac = np.abs(pre - np.floor(pre) - 0.5)
        bad_codes += int(np.sum(~((frac <= 1e-3) & (np.abs(c[d] - r["codes"][d]) == 1))))
    ok = ok and bad_codes == 0 and len(diff_rows) <= 4096
    return {"rows": int(rows), "rows_bit_identical": int(rows - len(diff_rows)),
            "rows_with_tie_band_codes": int(len(diff_rows)), "codes_outside_tie_band": bad_codes,
            "max_step_rel_err": float(rel.max()), "ok": ok}


def extra_workloads(spin, dev, world, rank, stream, args, peak):
    """Compact measurements of the other throughput workloads, carried in the
    default line: the 1 GiB sweeps at n = 4096 .. 32768 (the n >= 4096 target) and
    R3 + KV. Same timing method as the headline, about 0.25 s of device time each."""
    import torch
    out = {"sweep": [], "r3_kv": None}
    for k in (12, 13, 14, 15):
        wl = make_workload(f"sweep{k}", rank)
        n, tokens = 1 << k, wl["bits"].shape[0]
        x = torch.from_numpy(wl["bits"].view(np.int16)).view(torch.bfloat16).to(dev)
        del wl
        q = torch.empty((tokens, n // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((tokens,), dtype=torch.float32, device=dev)

        def step(i):
            spin.hadamard_quant_int4(x, 1.0, None, out=q, scales=s, stream=stream)

        for i in range(args.warmup):
            step(i)
        windows = timed_windows(step, args.steps, stream, dev, world, 0.25)
        require_clean_status(spin, f"sweep n={n}")
        ms, _ = window_stats(windows, args.steps)
        gbs = algorithmic_bytes_r4(tokens, n) / (ms / 1e3) / 1e9
        out["sweep"].append({"n": n, "tokens": tokens, "kernel": r4_kernel_name(n, tokens, False),
                             "ms_per_step": ms, "achieved_gbs": gbs * world, "frac": gbs / peak,
                             "windows": len(windows)})
        del x, q, s
    wl = make_workload("r3_kv", rank)
    qh, kh, vh, pos = wl["q"], wl["k"], wl["v"], wl["pos"]
    B, S, hq, d = qh.shape
    hkv = kh.shape[2]
    t = {name: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
         for name, a in (("q", qh), ("k", kh), ("v", vh))}
    pos_d = torch.from_numpy(pos).to(dev)
    qo = torch.empty((B, S, hq, d), dtype=torch.bfloat16, device=dev)
    cache = spin.alloc_kv_cache(B, hkv, S, d, device=dev)

    def r3_step(i):
        spin.rope_hadamard_kvquant(t["q"], t["k"], t["v"], pos_d, cache, clip=wl["clip"], q_out=qo, stream=stream)

    for i in range(args.warmup):
        r3_step(i)
    windows = timed_windows(r3_step, args.steps, stream, dev, world, 0.25)
    require_clean_status(spin, "R3 + KV")
    ms, _ = window_stats(windows, args.steps)
    gbs = r3_bytes(B * S, hq, hkv, d) / (ms / 1e3) / 1e9
    out["r3_kv"] = {"kernel": "k2_rope_hadamard_kvquant", "tokens": B * S, "ms_per_step": ms,
                    "achieved_gbs": gbs * world, "frac": gbs / peak, "tokens_per_s": world * B * S / (ms / 1e3),
                    "windows": len(windows)}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="spin", choices=["spin", "reference"])
    ap.add_argument("--workload", default="r4_prefill")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="leave out the sweep and R3 + KV sub-measurements of the default line")
    ap.add_argument("--min-seconds", type=float, default=0.5,
                    help="repeat the timed window of --steps steps until this much device time is sampled")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (R4 workloads; smaller cases for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        run_reference(args, make_workload(args.workload, 0, args.tokens))
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import online_hadamard_rotation_b200 as spin
    from online_hadamard_rotation_b200 import build
    build.build()
    spin.lib()
    spin.device_status(reset=True)

    wl = make_workload(args.workload, rank, args.tokens)
    stream = torch.cuda.Stream(dev)
    if wl["kind"] == "r4":
        bits, n = wl["bits"], wl["bits"].shape[1]
        tokens = bits.shape[0]
        host = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        code_bits = wl["code_bits"]
        qshape, qtype = ((tokens, n // 2), torch.uint8) if code_bits == 4 else ((tokens, n), torch.int8)
        quant = spin.hadamard_quant_int4 if code_bits == 4 else spin.hadamard_quant_int8
        if "kron_m" in wl:
            def quant(x, clip, signs, out, scales, stream, cuda_cores_only=False):  # noqa: F811
                return spin.hadamard_quant_kron(x, wl["kron_m"], clip, signs, out=out, scales=scales, stream=stream)
        sets = []
        for _ in range(2):
            sets.append(dict(x=host.to(dev), q=torch.empty(qshape, dtype=qtype, device=dev),
                             s=torch.empty((tokens,), dtype=torch.float32, device=dev)))
        signs = (torch.from_numpy(wl["signs"].view(np.int32)).to(dev) if wl["signs"] is not None else None)
        step_bytes = algorithmic_bytes_r4(tokens, n, code_bits)

        def step(i, cores_only=False):
            b = sets[i & 1]
            quant(b["x"], wl["clip"], signs, out=b["q"], scales=b["s"], stream=stream, cuda_cores_only=cores_only)
    elif wl["kind"] == "gemm":
        # activations through the R4 kernel, weight rows baked by the same kernel (same diagonal)
        T, K = wl["bits"].shape
        N = wl["n_out"]
        tokens = T
        signs = torch.from_numpy(wl["signs"].view(np.int32)).to(dev)
        to_dev = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        xq, xs = spin.hadamard_quant_kron(to_dev(wl["bits"]), wl["kron_m"], wl["clip"], signs)
        wq, ws = spin.hadamard_quant_kron(to_dev(wl["w_bits"]), wl["kron_m"], 1.0, signs)
        sets = [dict(out=torch.empty((T, N), dtype=torch.bfloat16, device=dev)) for _ in range(2)]
        torch.cuda.synchronize()
        step_ops = 2 * T * N * K
        step_bytes = T * (K // 2 + 4) + N * (K // 2 + 4) + 2 * T * N  # codes, steps, bf16 output

        def step(i, cores_only=False):
            spin.w4a4_gemm(xq, xs, wq, ws, out=sets[i & 1]["out"], stream=stream)
    elif wl["kind"] == "attn":
        # the cache as the R3 kernel writes it from the workload's Q, K, V; one query per row
        q, k, v, pos = wl["q"], wl["k"], wl["v"], wl["pos"]
        B, S, hq, d = q.shape
        hkv = k.shape[2]
        tokens = B
        sets = []
        for _ in range(2):
            cache = spin.alloc_kv_cache(B, hkv, S, d, device=dev)
            qo = spin.rope_hadamard_kvquant(*(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
                                              for a in (q, k, v)), torch.from_numpy(pos).to(dev), cache,
                                            clip=wl["clip"])
            sets.append(dict(q=qo[:, S - 1].contiguous(), cache=cache,
                             lens=torch.full((B,), S, dtype=torch.int32, device=dev),
                             out=torch.empty((B, hq, d), dtype=torch.float32, device=dev),
                             ws=torch.empty((spin.decode_attention_workspace_bytes(B, hq, S),), dtype=torch.uint8,
                                            device=dev)))
            del qo
        torch.cuda.synchronize()
        step_bytes = attn_bytes(B, S, hq, hkv, d)

        def step(i, cores_only=False):
            b = sets[i & 1]
            spin.decode_attention_int4kv(b["q"], b["cache"], b["lens"], out=b["out"], workspace=b["ws"],
                                         stream=stream)
    else:
        q, k, v, pos = wl["q"], wl["k"], wl["v"], wl["pos"]
        B, S, hq, d = q.shape
        hkv = k.shape[2]
        tokens = B * S
        sets = []
        for _ in range(2):
            sets.append(dict(q=torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(dev),
                             k=torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).to(dev),
                             v=torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev),
                             pos=torch.from_numpy(pos).to(dev), qo=torch.empty((B, S, hq, d), dtype=torch.bfloat16,
                                                                               device=dev),
                             cache=spin.alloc_kv_cache(B, hkv, S, d, device=dev)))
        step_bytes = r3_bytes(tokens, hq, hkv, d)

        def step(i, cores_only=False):
            b = sets[i & 1]
            spin.rope_hadamard_kvquant(b["q"], b["k"], b["v"], b["pos"], b["cache"], clip=wl["clip"], q_out=b["qo"],
                                       stream=stream)

    torch.cuda.synchronize()
    for i in range(args.warmup):
        step(i)
    stream.synchronize()
    require_clean_status(spin, "warm-up")

    # ---- device-timed region: inputs resident in HBM; windows of exactly --steps steps
    with ClockSampler(local_rank) as clocks:
        windows = timed_windows(step, args.steps, stream, dev, world, args.min_seconds)
    require_clean_status(spin, "timed region")
    ms_per_step, window_info = window_stats(windows, args.steps)
    last = sets[(args.steps * len(windows) - 1) & 1]  # buffers of the last timed step, kept for the spot check
    last = ({"q": last["q"].clone(), "s": last["s"].clone()} if wl["kind"] == "r4"
            else {"out": last["out"].clone()} if wl["kind"] == "gemm" else None)
    if wl["kind"] == "attn":  # per-call latency: the cache of the R3 + KV workload is L2-resident
        latency = {"us_per_call": ms_per_step * 1e3, "launches_per_call": 2}
    if world > 1:
        dist.barrier()
    gbs, tok_s = aggregate(world, step_bytes, tokens, args.steps, ms_per_step * args.steps)

    # ---- end to end through the public API from pinned host memory: the batch in
    # eight slices whose copy in, kernel and copy out overlap on three streams
    e2e = None
    if wl["kind"] == "r4":
        e2e_steps = max(3, args.steps // 5)
        bufs = None
        for _ in range(2):
            _, _, bufs = spin.hadamard_quant_host(host, wl["clip"], signs, code_bits, dev, stream, bufs,
                                                  m=wl.get("kron_m"))
        if world > 1:
            dist.barrier()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(e2e_steps):
            q_host, s_host, bufs = spin.hadamard_quant_host(host, wl["clip"], signs, code_bits, dev, stream, bufs,
                                                            m=wl.get("kron_m"))
        ev1.record(stream)
        ev1.synchronize()
        require_clean_status(spin, "end-to-end leg")
        ems = max_over_ranks(ev0.elapsed_time(ev1), dev)
        e_gbs, e_tok = aggregate(world, step_bytes, tokens, e2e_steps, ems)
        e2e = {"value": e_gbs, "unit": "GB/s", "tokens_per_s": e_tok,
               "h2d_bytes_per_step": int(host.numel() * 2), "d2h_bytes_per_step": int(q_host.numel() + 4 * tokens),
               "steps": e2e_steps, "pipeline": "8 token slices, copy in / kernel / copy out on three streams"}
        del bufs

    # ---- the same steps on the all-CUDA-core kernel, for comparison (not the headline)
    cores = None
    if wl["kind"] == "r4" and "kron_m" not in wl and \
            r4_kernel_name(n, tokens, wl["signs"] is not None) == "k1_tc_rotate_quant":
        for i in range(args.warmup):
            step(i, True)
        cwin = timed_windows(lambda i: step(i, True), args.steps, stream, dev, world, 0.1)
        require_clean_status(spin, "CUDA-core comparison leg")
        cms, _ = window_stats(cwin, args.steps)
        cores = {"kernel": f"k1_rotate_quant_int{code_bits} (all butterflies on CUDA cores)", "ms_per_step": cms,
                 "achieved_gbs": step_bytes / (cms / 1e3) / 1e9}

    # ---- bandwidth sweep: the dequantise -> inverse-rotate round trip on this step's
    # codes (its own kernel, timed alone), and the reconstruction error of the rotated
    # path against direct quantisation over the whole workload
    round_trip = None
    if args.workload.startswith("sweep"):
        b = sets[0]
        step(0)
        xr = torch.empty((tokens, n), dtype=torch.bfloat16, device=dev)

        def inverse(codes, scales, direct=False):
            spin.dequant_hadamard_inverse(codes, n, scales, no_rotate=direct, out_dtype=torch.bfloat16, out=xr,
                                          stream=stream)

        for _ in range(args.warmup):
            inverse(b["q"], b["s"])
        rwin = timed_windows(lambda i: inverse(b["q"], b["s"]), args.steps, stream, dev, world, 0.25)
        require_clean_status(spin, "round trip")
        rms, _ = window_stats(rwin, args.steps)
        rt_bytes = tokens * (n // 2 + 4 + 2 * n)
        x32 = b["x"].float()
        mse = {}
        for direct in (False, True):
            q_d = torch.empty_like(b["q"])
            s_d = torch.empty_like(b["s"])
            spin.hadamard_quant_int4(b["x"], wl["clip"], None, no_rotate=direct, out=q_d, scales=s_d, stream=stream)
            inverse(q_d, s_d, direct)
            stream.synchronize()
            mse[direct] = float(((xr.float() - x32) ** 2).mean().item())
            del q_d, s_d
        del x32, xr
        rt_gbs = rt_bytes / (rms / 1e3) / 1e9
        round_trip = {"kernel": k3_kernel_name(n, tokens), "ms_per_step": rms, "achieved_gbs": rt_gbs * world,
                      "frac": rt_gbs / measured_peaks()[0], "bytes_per_row": n // 2 + 4 + 2 * n,
                      "out_dtype": "bf16", "mse_rotated": mse[False], "mse_direct": mse[True],
                      "mse_ratio": mse[False] / mse[True] if mse[True] > 0 else None}

    # ---- decode: per-call latency, plain launches and CUDA-graph replay
    if wl["kind"] != "attn":
        latency = None
    if args.workload.startswith("decode") and wl["kind"] == "r4":
        calls = 1000
        b = sets[0]
        for _ in range(10):
            step(0)
        stream.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(calls):
            step(0)
        ev1.record(stream)
        ev1.synchronize()
        plain_us = ev0.elapsed_time(ev1) / calls * 1e3
        graph = torch.cuda.CUDAGraph()
        per_graph = 100
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(per_graph):
                spin.hadamard_quant_int4(b["x"], wl["clip"], signs, out=b["q"], scales=b["s"],
                                         stream=torch.cuda.current_stream())
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        ev0.record()
        for _ in range(calls // per_graph):
            graph.replay()
        ev1.record()
        ev1.synchronize()
        graph_us = ev0.elapsed_time(ev1) / calls * 1e3
        del graph
        require_clean_status(spin, "decode latency")
        latency = {"us_per_call_plain": plain_us, "us_per_call_graph": graph_us, "calls": calls,
                   "note": "inputs are L2-resident at this size (1.3 MB or less)"}

    peak, peak_kind = measured_peaks()
    if wl["kind"] == "attn":
        kname = "k4_attn_partial"
    elif wl["kind"] == "gemm":
        kname = "k5_w4a4_gemm"
    elif wl["kind"] == "r4" and "kron_m" in wl:
        kname = "k1_tc_rotate_quant"
    elif wl["kind"] == "r4":
        kname = r4_kernel_name(n, tokens, wl["signs"] is not None, wl["code_bits"])
    else:
        kname = "k2_rope_hadamard_kvquant"
    traffic = recorded_traffic(f"{kname}:{args.workload}")
    per_gpu_gbs = step_bytes / (ms_per_step / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": per_gpu_gbs, "peak": peak, "unit": "GB/s",
                "frac": per_gpu_gbs / peak, "traffic": traffic, "kernel": kname,
                "algorithmic_bytes_per_launch": step_bytes,
                "peak_source": f"{peak_kind} hbm_gbs (STREAM-style copy)"}
    value, unit = gbs, "GB/s"
    if wl["kind"] == "gemm":
        tops_peak, tops_src = int8_peak_tops()
        per_gpu_tops = step_ops / (ms_per_step / 1e3) / 1e12
        value, unit = per_gpu_tops * world, "TOPS"
        roofline = {"bound": "tensor", "achieved": per_gpu_tops, "peak": tops_peak, "unit": "TOPS",
                    "frac": per_gpu_tops / tops_peak, "traffic": traffic, "kernel": kname,
                    "algorithmic_ops_per_launch": step_ops, "peak_source": tops_src,
                    "operand_and_output_gbs": per_gpu_gbs}

    extras = None
    if args.workload == "r4_prefill" and not args.no_extras and args.tokens is None:
        extras = extra_workloads(spin, dev, world, rank, stream, args, peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and wl["kind"] == "gemm":
        cpu = cpu_baseline_gemm(xq, xs, wq, ws, last["out"])
        if not cpu["spot_check"]["ok"]:
            raise SystemExit(f"the last timed step disagrees with the oracle: {cpu['spot_check']}")
    if rank == 0 and world == 1 and not args.no_cpu_baseline and wl["kind"] == "r4":
        cpu, ref_out = cpu_baseline_leg(wl)
        cpu["spot_check"] = (spot_check(ref_out[0], wl, ref_out[1], ref_out[2], last["q"], last["s"], ref_out[3])
                             if ref_out is not None else None)
        if cpu["spot_check"] is not None and not cpu["spot_check"]["ok"]:
            raise SystemExit(f"the last timed step disagrees with the oracle: {cpu['spot_check']}")

    if rank == 0:
        line = {"metric": metric_for(wl), "value": value, "unit": unit, "tokens_per_s": tok_s,
                "pct_of_hbm_peak": 100.0 * per_gpu_gbs / peak, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "s8" if wl["kind"] == "gemm" else "f32", "data": "synthetic",
                "config": config_for(wl, world, args.workload),
                "gpu_launches": args.steps * (2 if wl["kind"] == "attn" else 1), "timed_windows": window_info, "e2e": e2e, "roofline": roofline,
                "cpu_baseline": cpu, "cuda_core_kernel": cores, "decode_latency": latency,
                "round_trip": round_trip, "other_workloads": extras, "clocks": clocks.summary()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
