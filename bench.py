"""Benchmark of the 64-layer decode weight stream on B200.

One step = one pass of the whole hot path over one decode token's weights:
the 257 group-quantised products of a dense 27B-shaped hybrid model (64 layers
of fused q|k|v, o, gate|up, down; the 16 attention layers' q|k|v|o and the
output head in q8 g32, everything else q4 g32), run as one stream-mode layer
stack: the activation preparation and one persistent kernel over all 257
products.  13.7 GB of packed weights are resident in HBM; x and y are small.

Metric: weight-stream GB/s (algorithmic weight bytes / device time per step)
at M = 1, with % of the measured HBM peak and the implied decode tok/s; the
same at M = 4 (one verification pass of 3 drafted tokens + 1) in "m4".  The
line also reports the ordered and graph stack modes, the end-to-end step
through the public API ("e2e"), the roofline of the dominant kernel, the CPU
oracle's rate ("cpu_baseline"), the SM clock under load, "chain" (the same
products as a dependent chain with the residual + RMSNorm and SwiGLU steps
between them, M = 1 and 4 as a CUDA graph, M = 1 also as one persistent
launch), "nvfp4" (the same stream with its 4-bit tensors
in NVFP4, the same bytes, M = 1 and 4), "widths" (the same with its 4-bit
tensors at 5 and 6 bits), "spec" (one MTP speculative step:
three mapped-vocabulary drafts, the M = 4 pass and the keep / reject step),
and "per_config":
microseconds per product of the single-tensor configurations (q4 4096 x 4096,
each projection of one layer at M = 1 and 4, the q8 vocabulary heads).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 it runs under torch.distributed (one process per GPU): every rank
streams its own replica of the weights (the single-token stream has no data
exchange to shard: replicas only), the device time is the max over ranks, and
the value is the bytes of all ranks over that time.  `--impl reference` times
the CPU oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "weight-stream GB/s & % of HBM peak (M=1,4); implied decode tok/s, 64 layers"
UNIT = "GB/s"
WORKLOAD = "64-layer decode weight stream + q8 output head (27B dense hybrid, 16 attn q8 / 48 DeltaNet q4, g32), M=1"


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for rel in ("bit_weight_gemv_q4_b200/csrc/q4gemv_kernels.cuh", "bit_weight_gemv_q4_b200/csrc/q4stack_kernel.cuh",
                "bit_weight_gemv_q4_b200/csrc/q4gemv.cu", "bit_weight_gemv_q4_b200/csrc/q4nvfp4_kernel.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "gemv_q4_traffic.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    per = re.search(r"dram_bytes_per_full_launch:\s*([0-9]+)", text)
    if not sha or not per or sha.group(1) != kernel_source_sha():
        return None
    return int(per.group(1))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples: list[int] = []
        self.reasons: set[str] = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # clocks are reported as unavailable
            self.nvml = None
            self.error = str(exc)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception as exc:
                self.error = str(exc)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "note": self.error or "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def nvml_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample of the workload
# ----------------------------------------------------------------------------
def _sample_inputs(tensors, rows_per_tensor, seed, M=1):
    """(tensor, q, s) of evenly strided whole rows of each tensor, and the
    activations per distinct K."""
    import numpy as np

    from bit_weight_gemv_q4_b200 import synth, workloads

    x = {K: synth.activations(seed, synth.act_stream(workloads.activation_stream_id(K)), M, K)
         for K in workloads.distinct_k(tensors)}
    inputs = []
    for t in tensors:
        n = min(rows_per_tensor, t.N)
        if n == t.N:
            q, s = synth.tensor(t.bits, seed, t.tensor_id, t.N, t.K)
        else:
            stride = t.N // n
            r0 = (seed * 7919) % stride
            qs = [synth.tensor(t.bits, seed, t.tensor_id, t.N, t.K, row0=r, nrows=1)
                  for r in range(r0, t.N, stride)[:n]]
            q, s = np.concatenate([a for a, _ in qs]), np.concatenate([b for _, b in qs])
        inputs.append((t, q, s))
    return inputs, x


def _oracle_pass(inputs, x):
    import oracle

    for t, q, s in inputs:
        oracle.gemv(t.bits, q, s, x[t.K])


def _sampled_rate(tensors, target_s, seed, M=1, max_rows=4096):
    """Grows whole-row samples of every tensor until one oracle pass takes
    about target_s (or the tensors are whole); returns (GB/s of weights,
    seconds, rows per tensor, sampled bytes)."""
    from bit_weight_gemv_q4_b200 import workloads

    rows = 2
    while True:
        inputs, x = _sample_inputs(tensors, rows, seed, M)
        nbytes = sum(workloads.weight_bytes(t.bits, q.shape[0], t.K) for t, q, _ in inputs)
        t0 = time.perf_counter()
        _oracle_pass(inputs, x)
        dt = time.perf_counter() - t0
        whole = all(q.shape[0] == t.N for t, q, _ in inputs)
        if dt >= 0.7 * target_s or whole or rows >= max_rows:
            return nbytes / dt / 1e9, dt, rows, nbytes
        rows = min(max_rows, max(2 * rows, int(rows * target_s / max(dt, 1e-3))))


def oracle_sample_rate(target_s: float = 12.0, seed: int = 0):
    """Times the CPU oracle on whole rows spread over every tensor of the decode
    stream; returns (GB/s of weights, threads, sample description, seconds)."""
    import oracle
    from bit_weight_gemv_q4_b200 import workloads

    tensors = workloads.decode_stream(fused=True)
    rate, dt, rows, nbytes = _sampled_rate(tensors, target_s, seed)
    desc = (f"{rows} whole rows (evenly strided) of each of the 257 tensors of the M=1 decode stream, "
            f"{nbytes / 1e6:.1f} MB of weights, fp64 oracle, {dt:.1f} s")
    return rate, oracle.threads(), desc, dt


def oracle_config_rates(budget_s: float, seed: int = 0):
    """The CPU oracle on each configuration (q4 4096 x 4096, one 27B-shaped q4
    layer at M = 1 and 4, the q8 heads of 65,536 and 248,320 rows, K = 5120,
    and the 257-product decode stream at M = 1), whole when that fits the
    budget per configuration, else on whole-row samples; GB/s of weights and
    the implied microseconds for the whole configuration, with the threads the
    oracle used."""
    import oracle
    from bit_weight_gemv_q4_b200 import workloads

    cases = [("q4_4096x4096_M1", [workloads.Tensor("w", 4, 4096, 4096, 3000)], 1),
             ("layer_q4_M1", workloads.layer_q4(), 1), ("layer_q4_M4", workloads.layer_q4(), 4)]
    cases += [(f"{h.name}_q8_{h.N}x{h.K}_M1", [h], 1) for h in workloads.draft_heads()]
    cases.append(("decode_stream_M1", workloads.decode_stream(fused=True), 1))
    out = {"threads": oracle.threads()}
    for name, tensors, M in cases:
        rate, dt, rows, nbytes = _sampled_rate(tensors, budget_s, seed, M, max_rows=1 << 20)
        total = workloads.total_bytes(tensors)
        out[name] = {"GBps": round(rate, 4), "us": round(total / (rate * 1e3), 1),
                     "sample": "whole" if nbytes == total else f"{nbytes / 1e6:.1f} of {total / 1e6:.1f} MB",
                     "seconds": round(dt, 2)}
    return out


def oracle_config_rates_in(threads: int, budget_s: float, seed: int = 0):
    """oracle_config_rates in a fresh process whose OpenMP runtime uses
    `threads` threads (the oracle as it stands; the thread count is the
    runtime's environment variable)."""
    import subprocess

    env = dict(os.environ, OMP_NUM_THREADS=str(threads))
    cmd = [sys.executable, os.path.abspath(__file__), "--oracle-configs", "--cpu-seconds", str(budget_s),
           "--seed", str(seed)]
    proc = subprocess.run(cmd, env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, timeout=900)
    if proc.returncode != 0:
        return {"error": proc.stderr.strip().splitlines()[-1:] or ["failed"]}
    return json.loads(proc.stdout.strip().splitlines()[-1])


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------
class Dist:
    """One process per GPU (torch.distributed.run sets RANK, LOCAL_RANK,
    WORLD_SIZE, MASTER_*).  The step has no data exchange (replicas): the
    process group only brackets the timed region with barriers and takes the
    max of the ranks' device times.  backend "gloo" (CPU tensors) serves the
    host-side tests."""

    def __init__(self, gpus: int, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        self.backend = backend
        if self.world != gpus:
            raise SystemExit(f"--gpus {gpus} needs torch.distributed.run with {gpus} processes "
                             f"(WORLD_SIZE is {self.world})")
        if self.world > 1:
            import torch
            import torch.distributed as dist

            timeout = datetime.timedelta(seconds=120)
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group(backend, timeout=timeout)
            self.pg = True

    @classmethod
    def single(cls):
        """Rank 0 of a multi-process launch doing host-only work: no process group."""
        d = cls.__new__(cls)
        d.world, d.rank, d.local, d.pg = 1, 0, int(os.environ.get("LOCAL_RANK", "0")), False
        return d

    def barrier(self):
        if self.pg:
            import torch.distributed as dist

            dist.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist

        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist

            dist.destroy_process_group()


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def time_region(torch, fn, steps, stream):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)  # ms


def per_config(args, d: Dist, torch, q4, workloads, peak):
    """Microseconds per product for the single-tensor configurations: a
    q4 4096 x 4096 product (M = 1), each projection of one 27B-shaped layer
    (M = 1 and M = 4) and the q8 vocabulary heads (M = 1).  Each shape is
    replicated until the copies exceed twice the L2, and the copies run in
    turn, so no launch finds its weights in L2.  `graph`: one q4_gemv /
    q8_gemv launch per product (captured as a graph with programmatic
    dependent launch, the single-call kernels back to back); `stream`: the
    same copies as one stream-mode stack.  Device time per product."""
    l2 = torch.cuda.get_device_properties(d.local).L2_cache_size
    stream = torch.cuda.current_stream()
    iters = max(3, min(20, args.steps // 10))

    def time_stack(stack):
        run = lambda: q4.layer_stack_run(stack)  # noqa: E731
        for _ in range(3):
            run()
        ms = d.max(time_region(torch, run, iters, stream) / iters)
        q4.layer_stack_check(stack)
        return ms

    def shape(name, bits, N, K, M, tid):
        one = workloads.weight_bytes(bits, N, K)
        copies = max(2, -(-2 * l2 // one))
        tensors = [workloads.Tensor(f"{name}.{i}", bits, N, K, tid + i) for i in range(copies)]
        out = {"N": N, "K": K, "bits": bits, "M": M, "bytes": one, "copies": copies}
        st = workloads.DeviceStream(tensors, M, seed=args.seed, flags=q4.Q4_STACK_GRAPH)
        for stack, key in ((st.stack, "graph"), (st.make_stack(q4.Q4_STACK_INDEPENDENT), "stream")):
            us = time_stack(stack) * 1e3 / copies
            out[key] = {"us": round(us, 2), "GBps": round(one / (us * 1e3), 1),
                        "pct_of_hbm_peak": round(100 * one / (us * 1e3) / peak, 1)}
            stack.close()
        st.close()
        del st
        torch.cuda.empty_cache()
        return out

    res = {"note": "device us per product, L2 defeated by rotating copies (> 2x L2)",
           "q4_4096x4096_M1": shape("w4096", 4, 4096, 4096, 1, 3000)}
    for M in (1, 4):
        layer = {}
        for t in workloads.layer_q4():
            layer[t.name] = shape(t.name, t.bits, t.N, t.K, M, 3100 + 100 * len(layer))
        layer["sum_us"] = {k: round(sum(v[k]["us"] for v in layer.values()), 2) for k in ("graph", "stream")}
        res[f"layer_q4_M{M}"] = layer
    for h in workloads.draft_heads():
        res[f"{h.name}_q8_{h.N}x{h.K}_M1"] = shape(h.name, h.bits, h.N, h.K, 1, 3900 + h.tensor_id)
    res["quantize"] = quantize_rates(args, d, torch, q4, peak)
    return res


def spec_step(args, d: Dist, torch, q4, workloads, stream, peak):
    """One MTP speculative step (3 drafts): each draft is the mapped draft
    head's product (65,536 x 5120 q8, M = 1) and a draw; then the decode
    stream at M = 4 and the keep / reject kernels.  Device time of the step
    and of its parts.  How many tokens a step yields depends on how often the
    drafts are kept, which needs trained weights; the step emits 1 to 4."""
    sp = workloads.DeviceSpec(seed=args.seed, temperature=1.0)
    n_it = max(3, args.steps // 4)

    def timed(fn, n):
        for _ in range(3):
            fn()
        return d.max(time_region(torch, fn, n, stream) / n)

    ms_step = timed(sp.run, n_it)
    ms_head = timed(lambda: q4.layer_stack_run(sp.draft_stacks[0]), 4 * n_it)
    ms_draft = timed(lambda: sp.draft(0), 4 * n_it)
    ms_pass = timed(sp.verify_stream.run, n_it)
    ms_verify = timed(sp.verify, 4 * n_it)
    sp.check()
    head_bytes = workloads.weight_bytes(8, sp.n_map, sp.K)
    step_bytes = sp.verify_stream.weight_bytes + sp.n * head_bytes
    # bytes the keep / reject kernels read: the target logits, the draft
    # logits and the inverse map (their floor; the kernels re-read from L2)
    verify_bytes = 4 * ((sp.n + 1) * sp.V + sp.n * sp.n_map + sp.V)
    out = {
        "drafts": sp.n, "vocab": sp.V, "mapped_vocab": sp.n_map, "temperature": sp.T,
        "step_ms": round(ms_step, 5),
        "step_weight_bytes": step_bytes,
        "step_GBps": round(step_bytes / (ms_step * 1e6), 1),
        "pct_of_hbm_peak": round(100 * step_bytes / (ms_step * 1e6) / peak, 2),
        "draft_head_us": round(ms_head * 1e3, 2),
        "draft_head_GBps": round(head_bytes / (ms_head * 1e6), 1),
        "draft_draw_us": round((ms_draft - ms_head) * 1e3, 2),
        "verify_pass_ms": round(ms_pass, 5),
        "verify_us": round(ms_verify * 1e3, 2),
        "verify_bytes": verify_bytes,
        "launches_per_step": sp.n * 3 + sp.verify_stream.stack.launches() + 2,
    }
    sp.close()
    del sp
    torch.cuda.empty_cache()
    return out


def quantize_rates(args, d: Dist, torch, q4, peak):
    """The offline quantiser on the device: bf16 weights of a gate|up-sized
    tensor (q4) and of the full vocabulary head (q8) to codes and scales; GB/s
    of bytes moved (2 B read per weight, codes and scales written)."""
    out = {}
    stream = torch.cuda.current_stream()
    for name, bits, mode, N, K in (("q4_signed_34816x5120", 4, q4.Q4_QUANT_SIGNED_MAX, 34816, 5120),
                                   ("q8_absmax_248320x5120", 8, q4.Q4_QUANT_ABSMAX, 248320, 5120)):
        g = torch.Generator(device="cuda")
        g.manual_seed(args.seed)
        w = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16).view(torch.int16)
        q = torch.empty(N * (K // 2 if bits == 4 else K), dtype=torch.uint8, device="cuda")
        s = torch.empty(N * (K // 32), dtype=torch.int16, device="cuda")
        run = lambda: q4.q4_quantize_device(bits, mode, w, N, K, q, s)  # noqa: E731
        for _ in range(3):
            run()
        n = 10
        ms = d.max(time_region(torch, run, n, stream) / n)
        moved = N * K * 2 + q.numel() + s.numel() * 2
        out[name] = {"us": round(ms * 1e3, 1), "GBps": round(moved / (ms * 1e6), 1),
                     "pct_of_hbm_peak": round(100 * moved / (ms * 1e6) / peak, 1), "bytes_moved": moved}
        del w, q, s
        torch.cuda.empty_cache()
    return out


def run_ours(args, d: Dist):
    import torch

    import bit_weight_gemv_q4_b200 as q4
    from bit_weight_gemv_q4_b200 import workloads

    torch.cuda.set_device(d.local)
    stream = torch.cuda.current_stream()
    tensors = workloads.decode_stream(fused=True)
    peak, peak_kind = measured_peaks()

    # the step: the 257 products of one decode token, independent (each reads
    # its own activation block), as one persistent stream-mode launch
    st = workloads.DeviceStream(tensors, 1, seed=args.seed, flags=q4.Q4_STACK_INDEPENDENT)
    n_launch = st.stack.launches()
    wbytes = st.weight_bytes

    for _ in range(args.warmup):
        st.run()
    torch.cuda.synchronize()
    st.check()

    sampler = ClockSampler(nvml_index(d.local))
    d.barrier()
    torch.cuda.synchronize()
    with sampler:
        ms = time_region(torch, st.run, args.steps, stream)
    d.barrier()
    st.check()
    ms_step = d.max(ms / args.steps)
    value = wbytes * d.world / (ms_step * 1e6)  # GB/s over all ranks
    # the step is one launch of stream_kernel, the dominant (only) kernel
    step_us = ms / args.steps * 1e3  # this rank's own step
    achieved = wbytes / (step_us * 1e-6) / 1e9

    # the same products with an ordering between consecutive products (each
    # product's outputs complete before the next reads its activations), as
    # one ordered persistent launch and as a graph of one launch per product
    other = {}
    for flags, name in ((q4.Q4_STACK_ORDERED, "ordered"), (q4.Q4_STACK_GRAPH, "graph")):
        alt = st.make_stack(flags)
        run_alt = lambda: q4.layer_stack_run(alt)  # noqa: E731
        for _ in range(max(3, args.warmup // 2)):
            run_alt()
        n_alt = max(3, args.steps // 4)
        ms_alt = d.max(time_region(torch, run_alt, n_alt, stream) / n_alt)
        q4.layer_stack_check(alt)
        other[name] = {"value": round(wbytes * d.world / (ms_alt * 1e6), 1), "ms_per_step": round(ms_alt, 5),
                       "pct_of_hbm_peak": round(100 * wbytes / (ms_alt * 1e6) / peak, 2),
                       "launches": alt.launches()}
        alt.close()

    # e2e through the public API: activations from pinned host memory in,
    # the stack, the logits (head output) back to pinned host memory
    x_host = {K: xb.cpu().pin_memory() for K, xb in st.x.items()}
    logits = st.y[-1]
    logits_host = torch.empty(logits.shape, dtype=logits.dtype, pin_memory=True)

    def e2e_step():
        for K, xb in st.x.items():
            xb.copy_(x_host[K], non_blocking=True)
        st.run()
        logits_host.copy_(logits, non_blocking=True)

    for _ in range(2):
        e2e_step()
    d.barrier()
    ms_e2e = d.max(time_region(torch, e2e_step, args.steps, stream) / args.steps)
    h2d = sum(v.numel() * v.element_size() for v in x_host.values())
    d2h = logits_host.numel() * logits_host.element_size()
    st.check()
    st.close()
    del st
    torch.cuda.empty_cache()

    # M = 4: one verification pass of three drafted tokens plus one
    st4 = workloads.DeviceStream(tensors, 4, seed=args.seed, flags=q4.Q4_STACK_INDEPENDENT)
    for _ in range(args.warmup):
        st4.run()
    d.barrier()
    ms4 = d.max(time_region(torch, st4.run, args.steps, stream) / args.steps)
    st4.check()
    st4.close()
    del st4
    torch.cuda.empty_cache()

    # the same stream with its 4-bit tensors in other formats: NVFP4 (E2M1
    # codes, E4M3 block scales of 16, fp32 tensor scale; the same bytes) and
    # q5 / q6 (more bytes per weight)
    def format_stream(fmt_tensors):
        fb = workloads.total_bytes(fmt_tensors)
        res = {"weight_bytes_per_step": fb}
        for M in (1, 4):
            sn = workloads.DeviceStream(fmt_tensors, M, seed=args.seed, flags=q4.Q4_STACK_INDEPENDENT)
            for _ in range(args.warmup):
                sn.run()
            d.barrier()
            n_f = max(3, args.steps // 2)
            ms_f = d.max(time_region(torch, sn.run, n_f, stream) / n_f)
            sn.check()
            res[f"M{M}"] = {"value": round(fb * d.world / (ms_f * 1e6), 1), "unit": UNIT,
                            "ms_per_step": round(ms_f, 5), "pct_of_hbm_peak": round(100 * fb / (ms_f * 1e6) / peak, 2),
                            "tok_per_s": round(1000.0 / ms_f, 1), "launches": sn.stack.launches()}
            sn.close()
            del sn
            torch.cuda.empty_cache()
        return res

    nv_tensors = workloads.as_nvfp4(tensors)
    assert workloads.total_bytes(nv_tensors) == wbytes
    # the secondary sections run at N = 1 only: with N > 1 the line reports the
    # headline step, M = 4, the other stack modes and e2e (replicas scale the same)
    secondary = d.world == 1 and not args.headline_only
    skipped = {"skipped": "measured at N = 1 only" if d.world > 1 else "--headline-only"}
    nvfp4 = format_stream(nv_tensors) if secondary else skipped
    widths = ({f"q{b}": format_stream(workloads.as_width(tensors, b)) for b in (5, 6)} if secondary else skipped)

    # the dependent chain: the same products with the steps between them
    # (residual + RMSNorm, SwiGLU), in the form layer_chain_create picks by
    # default (one CUDA graph with programmatic dependent launch) and as one
    # cooperative launch
    chain = {} if secondary else skipped
    for key, M, flags in ((("M1", 1, 0), ("M4", 4, 0), ("M1_persistent", 1, q4.Q4_CHAIN_PERSISTENT),
                           ("M4_persistent", 4, q4.Q4_CHAIN_PERSISTENT)) if secondary else ()):
        ch = workloads.DeviceChain(workloads.ChainShape(), M, seed=args.seed, flags=flags)
        try:
            for _ in range(3):
                ch.run()
            n_ch = max(3, args.steps // 4)
            ms_ch = d.max(time_region(torch, ch.run, n_ch, stream) / n_ch)
            ch.check()
        except q4.Q4Error as exc:
            # a bounded device wait gave up (the status word; the context stays
            # usable): report it in the line instead of losing the line
            chain[key] = {"error": str(exc)}
        else:
            chain[key] = {"value": round(wbytes * d.world / (ms_ch * 1e6), 1), "unit": UNIT,
                          "ms_per_step": round(ms_ch, 5),
                          "pct_of_hbm_peak": round(100 * wbytes / (ms_ch * 1e6) / peak, 2),
                          "tok_per_s": round(1000.0 / ms_ch, 1), "launches": ch.stack.launches()}
        ch.close()
        del ch
        torch.cuda.empty_cache()

    spec = spec_step(args, d, torch, q4, workloads, stream, peak) if secondary else skipped

    configs = None if args.no_configs or not secondary else per_config(args, d, torch, q4, workloads, peak)

    cpu = None
    if d.rank == 0 and d.world == 1 and not args.no_cpu_baseline:  # the oracle is timed at N = 1 only
        rate, threads, desc, _ = oracle_sample_rate(args.cpu_seconds, args.seed)
        cpu = {"value": round(rate, 4), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "per_config_all_cores": oracle_config_rates(args.cpu_seconds / 12, args.seed),
               "per_config_one_core": oracle_config_rates_in(1, args.cpu_seconds / 12, args.seed)}

    traffic = profiled_traffic()
    clocks = sampler.summary()
    gbs1 = wbytes / (ms_step * 1e6)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": d.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "q4/q8 g32 codes x fp16 (exact copy of the bf16 activations; bf16 when not exact), fp32 accumulate",
        "data": "synthetic (seeded generator: q uniform, fp16 scales |N(0,0.02)|, bf16 x N(0,1))",
        "config": {
            "workload": WORKLOAD,
            "tensors": len(tensors),
            "weight_bytes_per_step": wbytes,
            "M": 1,
            "mode": "stream (independent products, one persistent launch)",
            "parallelism": "replicas" if d.world > 1 else "single GPU",
            "l2": "inputs larger than L2 (13.7 GB of weights per step vs 126 MB L2); no flush",
        },
        "pct_of_hbm_peak": round(100 * gbs1 / peak, 2),
        "hbm_peak_gbs": peak,
        "hbm_peak_kind": peak_kind,
        "tok_per_s": round(1000.0 / ms_step, 1),
        "ordered": other["ordered"],
        "graph": other["graph"],
        "m4": {
            "value": round(wbytes * d.world / (ms4 * 1e6), 1),
            "unit": UNIT,
            "ms_per_step": round(ms4, 5),
            "pct_of_hbm_peak": round(100 * wbytes / (ms4 * 1e6) / peak, 2),
            "verify_passes_per_s": round(1000.0 / ms4, 1),
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "stream_kernel<M=1> (the whole decode stream in one launch; timed as the step, which also holds the activation preparation xprep_kernel, 0.4 % of its serialised time under ncu)",
            "achieved": round(achieved, 1),
            "peak": peak,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "bytes_per_launch": wbytes,
            "launch_us": round(step_us, 3),
            "launches_per_step": n_launch,
            "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy burst)" if peak_kind == "measured" else peak_kind,
        },
        "cpu_baseline": cpu,
        "e2e": {
            "value": round(wbytes * d.world / (ms_e2e * 1e6), 1),
            "unit": UNIT,
            "ms_per_step": round(ms_e2e, 5),
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
        },
        "chain": chain,
        "nvfp4": nvfp4,
        "widths": widths,
        "spec": spec,
        "per_config": configs,
        "gpu_launches": n_launch * args.steps,
        "clocks": clocks,
    }
    return line


def run_reference(args, d: Dist):
    """The CPU oracle on the host cores: each step is one pass of the oracle
    over the same bounded sample of the workload as cpu_baseline (whole rows
    of every tensor of the decode stream), sized so the whole --steps K
    --warmup W run takes about --reference-seconds; value = sampled weight
    bytes / time, same metric."""
    if d.rank != 0:
        return None
    import oracle
    from bit_weight_gemv_q4_b200 import workloads

    tensors = workloads.decode_stream(fused=True)
    per_step = max(0.05, args.reference_seconds / (args.steps + args.warmup))
    _, _, rows, nbytes = _sampled_rate(tensors, per_step, args.seed)
    inputs, x = _sample_inputs(tensors, rows, args.seed)
    for _ in range(args.warmup):
        _oracle_pass(inputs, x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_pass(inputs, x)
    dt = (time.perf_counter() - t0) / args.steps
    value = nbytes / dt / 1e9
    desc = (f"{rows} whole rows (evenly strided) of each of the 257 tensors of the M=1 decode stream per step, "
            f"{nbytes / 1e6:.1f} MB of weights, fp64 oracle")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": UNIT,
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp64 accumulate (oracle)",
        "data": "synthetic (seeded generator)",
        "config": {"workload": WORKLOAD, "tensors": len(tensors), "M": 1},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_profile_case(args):
    """Small cases for ncu.  Default: a q4 (or q8) 65536 x 5120 tensor (189 MB,
    larger than L2), `--profile-launches` launches at M = args.m.  With
    --profile-layers L: the first L layers of the decode stream (about 0.2 GB
    per layer) as one stream-mode stack launch; --profile-nvfp4 puts their
    4-bit tensors in NVFP4.  --profile-spec: the keep / reject kernels of a
    speculative step on seeded logits."""
    import torch

    import bit_weight_gemv_q4_b200 as q4
    from bit_weight_gemv_q4_b200 import workloads

    if args.profile_spec:
        # the keep / reject kernels alone on seeded logits (248,320 vocabulary,
        # 65,536 mapped, 3 drafts); drafts follow the target with noise
        import numpy as np

        rng = np.random.default_rng(args.seed)
        V, n = workloads.VOCAB, workloads.SPEC_DRAFTS
        vmap = workloads.vocab_map(args.seed, V)
        n_map = len(vmap)
        target = rng.normal(0, 3.0, (n + 1, V)).astype(np.float32)
        drafts = (target[:n][:, vmap] + rng.normal(0, 0.7, (n, n_map))).astype(np.float32)
        inv = np.full(V, -1, dtype=np.int32)
        inv[vmap] = np.arange(n_map, dtype=np.int32)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
        td, zd, md, invd = dev(target), dev(drafts), dev(vmap), dev(inv)
        rows = dev(rng.integers(0, n_map, n).astype(np.int32))
        u = dev(workloads.spec_uniforms(args.seed, 2 * n + 1))
        out = torch.zeros(3 * n + 3, dtype=torch.int32, device="cuda")
        for _ in range(args.profile_launches):
            q4.q4_spec_verify(td, V, zd, n_map, md, invd, rows, n, 1.0, u, out)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": "spec verify", "V": V, "n_map": n_map, "drafts": n,
                          "launches": args.profile_launches, "out": out.cpu().tolist()}))
        return
    if args.profile_chain_layers > 0:
        shape = workloads.ChainShape(layers=args.profile_chain_layers)
        ch = workloads.DeviceChain(shape, args.m, seed=args.seed, flags=q4.Q4_CHAIN_PERSISTENT)
        for _ in range(args.profile_launches):
            ch.run()
        torch.cuda.synchronize()
        ch.check()
        print(json.dumps({"profile_case": f"dependent chain of {args.profile_chain_layers} layers, one launch",
                          "M": args.m, "launches": args.profile_launches, "weight_bytes": ch.weight_bytes,
                          "kernel_source_sha": kernel_source_sha()}))
        ch.close()
        return
    if args.profile_shape:
        # single products (one gemv_kernel launch each) in copies rotated so
        # that no launch finds its weights in L2 (the per_config section's
        # "graph" figures)
        bits, N, K = (int(v) for v in args.profile_shape.split(","))
        one = workloads.weight_bytes(bits, N, K)
        l2 = torch.cuda.get_device_properties(0).L2_cache_size
        copies = max(2, -(-2 * l2 // one))
        tensors = [workloads.Tensor(f"shape.{i}", bits, N, K, 3000 + i) for i in range(copies)]
        st = workloads.DeviceStream(tensors, args.m, seed=args.seed, flags=q4.Q4_STACK_GRAPH)
        for _ in range(args.profile_launches):
            st.run()
        torch.cuda.synchronize()
        st.check()
        print(json.dumps({"profile_case": f"single products {bits},{N},{K} x {copies} copies, graph mode",
                          "M": args.m, "runs": args.profile_launches, "launches_per_run": copies,
                          "kernel_source_sha": kernel_source_sha()}))
        st.close()
        return
    if args.profile_layers > 0:
        tensors = workloads.decode_stream(fused=True)[: 4 * args.profile_layers]
        if args.profile_nvfp4:
            tensors = workloads.as_nvfp4(tensors)
        st = workloads.DeviceStream(tensors, args.m, seed=args.seed, flags=q4.Q4_STACK_INDEPENDENT)
        for _ in range(args.profile_launches):
            st.run()
        torch.cuda.synchronize()
        st.check()
        print(json.dumps({"profile_case": f"stream of {args.profile_layers} layers"
                          + (" (NVFP4)" if args.profile_nvfp4 else ""), "products": len(tensors),
                          "M": args.m, "launches": args.profile_launches, "weight_bytes": st.weight_bytes,
                          "kernel_source_sha": kernel_source_sha()}))
        st.close()
        return
    t = workloads.Tensor("profile.q4", 4 if args.profile_bits == 4 else 8, 65536, 5120, 900)
    st = workloads.DeviceStream([t], args.m, seed=args.seed)
    for _ in range(args.profile_launches):
        st.run()
    torch.cuda.synchronize()
    st.check()
    print(json.dumps({"profile_case": t.name, "bits": t.bits, "N": t.N, "K": t.K, "M": args.m,
                      "launches": args.profile_launches, "weight_bytes": t.bytes,
                      "kernel_source_sha": kernel_source_sha()}))
    st.close()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration product timings")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the format, width, chain and speculative sections (as every N > 1 run does)")
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="CPU time of the whole reference run (its per-step sample is sized from it)")
    ap.add_argument("--oracle-configs", action="store_true",
                    help="print the CPU oracle's per-configuration rates as one JSON line and exit")
    ap.add_argument("--profile-case", action="store_true", help="run the small ncu case and exit")
    ap.add_argument("--profile-bits", type=int, default=4)
    ap.add_argument("--profile-launches", type=int, default=3)
    ap.add_argument("--profile-layers", type=int, default=0)
    ap.add_argument("--profile-nvfp4", action="store_true")
    ap.add_argument("--profile-spec", action="store_true", help="profile case: the keep / reject kernels")
    ap.add_argument("--profile-chain-layers", type=int, default=0,
                    help="profile case: the dependent chain of this many layers as one launch (M = --m)")
    ap.add_argument("--profile-shape", default="",
                    help="profile case: bits,N,K of single products, in rotating copies (graph mode)")
    ap.add_argument("--m", type=int, default=1)
    args = ap.parse_args()
    if args.warmup < 3 and not args.profile_case:
        raise SystemExit("--warmup must be at least 3")

    if args.profile_case:
        run_profile_case(args)
        return
    if args.oracle_configs:  # host only: no CUDA
        print(json.dumps(oracle_config_rates(args.cpu_seconds, args.seed)), flush=True)
        return

    if args.impl == "reference" and int(os.environ.get("RANK", "0")) != 0:
        return  # the CPU oracle arm runs on rank 0 alone
    d = Dist(args.gpus) if args.impl == "ours" else Dist.single()
    try:
        line = run_reference(args, d) if args.impl == "reference" else run_ours(args, d)
        if d.rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        d.close()


if __name__ == "__main__":
    main()
