"""Benchmark of the paged-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-sweep]

One step = one pass of the hot path over its synthetic batches: the causal
GQA paged prefill (h16/kv1/d128/ps64, batch 8, lengths U[512, 4096]) and the
split-KV paged decode (b128/h32/kv8/d128/ps16, kv_len U[1024, 8192]), each
through pkv_run after an L2 flush, plus the absorbed-MLA prefill once its
kernel is built. `value` is the prefill's causal TFLOP/s (only visible
query/key pairs count); the decode's HBM GB/s (algorithmic bytes: K, V, Q, O,
LSE and page indices) rides along under "decode". Kernel times come from CUDA
events on the launching stream. `e2e` times the same prefill through the
public API from pinned host buffers: plan + upload, H2D of q / caches / page
table, run, D2H of O and LSE.

Beside the step (each timed alone between L2 flushes, not in its time): the
MLA decode, the FP8-KV decode, the paged KV append and, on one GPU, the
vector-sparse vs dense sweep of the pages' benchmark (`sparse_vs_dense`: page
size 1 with scattered slots against the contiguous layout of the same problem,
h32/kv8/d128 causal, every (B, L) of the sweep; `--no-sweep` skips it).

Multi-GPU (torchrun): requests are independent, so every rank runs its own
batch (weak scaling, no collective on the data path); the timed region is
bracketed by barriers and the max over ranks is reported.

--impl reference times the float64 CPU oracle (the only reference that exists
for this path) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import paged_kv_attention_38_b200 as pkv  # noqa: E402
from paged_kv_attention_38_b200 import workloads as W  # noqa: E402

METRIC = "causal paged-prefill TFLOP/s & % BF16 tensor peak; decode HBM GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------------- accounting

def causal_pairs(p: W.PagedProblem) -> int:
    """Visible (query, key) pairs: bottom-right causal, or all pairs."""
    total = 0
    for a, b in zip(p.qo_lens.tolist(), p.kv_lens.tolist()):
        if p.causal:
            d = b - a
            vis = np.clip(np.arange(a) + d + 1, 0, b)
            total += int(vis.sum())
        else:
            total += a * b
    return total


def attention_flops(p: W.PagedProblem) -> float:
    """2 FLOPs per multiply-add for Q.K^T (width head_dim [+ rope]) and P.V, per visible pair and head."""
    return 2.0 * (p.head_dim + p.head_dim_pe + p.head_dim_v) * p.num_qo_heads * causal_pairs(p)


def decode_bytes(p: W.PagedProblem) -> float:
    """Algorithmic HBM bytes of a decode pass: K and V rows of every request once,
    Q and O (bf16), LSE (fp32) and the page indices."""
    if p.is_mla:  # one latent row (ckv | kpe) per key serves as both K and V
        kv = 2 * (p.head_dim + p.head_dim_pe) * int(p.kv_lens.sum())
        q = 2 * p.total_q * p.num_qo_heads * (p.head_dim + p.head_dim_pe)
    else:  # K and V, 2 bytes per element (1 for an FP8 cache, plus its scales)
        el = 1 if p.is_fp8_kv else 2
        kv = 2 * el * p.num_kv_heads * p.head_dim * int(p.kv_lens.sum()) + (8 * p.num_kv_heads if el == 1 else 0)
        q = 2 * p.total_q * p.num_qo_heads * p.head_dim
    o = 2 * p.total_q * p.num_qo_heads * p.head_dim_v
    lse = 4 * p.total_q * p.num_qo_heads
    idx = 4 * len(p.kv_indices)
    return float(kv + q + o + lse + idx)


# ----------------------------------------------------------------- profile figures

PREFILL_SOURCES = ("prefill_sm100.cu", "sm100_ptx.cuh", "pkv_internal.h")
DECODE_SOURCES = ("decode_sm100.cu", "decode_core.cuh", "sm100_ptx.cuh", "pkv_internal.h")
DECODE_FP8_SOURCES = ("decode_fp8_sm100.cu", "sm100_ptx.cuh", "pkv_internal.h")
PREFILL_FP8_SOURCES = ("prefill_sm100.cu", "kv_fp8_expand.cu", "sm100_ptx.cuh", "pkv_internal.h")
MLA_SOURCES = ("mla_sm100.cu", "sm100_ptx.cuh", "pkv_internal.h")
MLA_DECODE_SOURCES = ("mla_decode_sm100.cu", "sm100_ptx.cuh", "pkv_internal.h")
APPEND_SOURCES = ("append.cu",)


def kernel_source_sha(files) -> str:
    """Short hash of the CUDA sources a kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_attention_38_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def profiled_traffic(summary: str, files, kv_tokens=None):
    """DRAM bytes per launch from a committed ncu summary under profiles/, or None
    when the summary is missing or was taken on other kernel sources. A summary
    taken on a smaller batch (it then records `kv_tokens`) is scaled to a launch
    with `kv_tokens` keys, for kernels whose traffic is proportional to them."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.split(":", 1)[0] in ("source_sha", "dram_bytes_per_launch", "kv_tokens"):
                k, v = line.split(":", 1)
                fields[k] = v.strip()
    if fields.get("source_sha") != kernel_source_sha(files) or "dram_bytes_per_launch" not in fields:
        return None
    traffic = float(fields["dram_bytes_per_launch"])
    if "kv_tokens" in fields and kv_tokens is not None:
        traffic *= kv_tokens / float(fields["kv_tokens"])
    return traffic


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle reasons sampled (NVML, every 2 ms) while the timed region runs.

    Falls back to `nvidia-smi -lms 100` if NVML is unavailable."""

    # NVML clocks-event-reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.index = index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None
        self._thread = None
        self._proc = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self._stop = threading.Event()

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                        bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        for b, n in self.REASONS.items():
                            if bits & b:
                                self.reasons.add(n)
                    except Exception:
                        pass
                    self._stop.wait(0.002)
            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception:
            q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap")
            try:
                self._proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                               "--format=csv,noheader,nounits", "-lms", "100"],
                                              stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self._proc = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=1)
        if self._proc is not None:
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
                out, _ = self._proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for l in out.splitlines():
                f = [x.strip() for x in l.split(",")]
                if len(f) < 6:
                    continue
                try:
                    self.samples.append(float(f[0]))
                    self.max_mhz = float(f[1])
                except ValueError:
                    continue
                for n, v in zip(names, f[2:6]):
                    if v.lower() == "active":
                        self.reasons.add(n)
        return False

    def summary(self):
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------- our arm

class Case:
    """A problem resident in HBM with its plan, ready to run."""

    def __init__(self, p: W.PagedProblem, device, **plan_kw):
        self.p = p
        self.idx = torch.from_numpy(p.kv_indices.astype(np.int32)).to(device)
        if p.is_mla:
            self.q_nope, self.q_pe = p.q_nope.to(device), p.q_pe.to(device)
            self.ckv, self.kpe = p.ckv_cache.to(device), p.kpe_cache.to(device)
            self.plan = pkv.plan_mla(p.qo_indptr, p.kv_indptr, self.idx, p.kv_last_page_len, p.num_qo_heads,
                                     p.head_dim, p.head_dim_pe, p.page_size, p.causal, p.sm_scale, **plan_kw)
            self.o = torch.empty(p.total_q, p.num_qo_heads, p.head_dim_v, dtype=torch.bfloat16, device=device)
        else:
            self.q, self.k, self.v = p.q.to(device), p.k_cache.to(device), p.v_cache.to(device)
            if p.is_fp8_kv:
                self.k_scale, self.v_scale = p.meta["k_scale"].to(device), p.meta["v_scale"].to(device)
                plan_kw.setdefault("kv_fp8", True)
            self.plan = pkv.plan(p.qo_indptr, p.kv_indptr, self.idx, p.kv_last_page_len, p.num_qo_heads,
                                 p.num_kv_heads, p.head_dim, p.page_size, p.causal, p.sm_scale, **plan_kw)
            self.o = torch.empty(p.total_q, p.num_qo_heads, p.head_dim_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(p.total_q, p.num_qo_heads, dtype=torch.float32, device=device)

    @property
    def launches(self) -> int:
        n = 1 + (1 if self.plan.num_merges > 0 else 0)  # the attention kernel and its split-KV merge
        if self.plan.kind == pkv.KIND_MLA:
            n += 1  # the latent rows packed before the MLA prefill kernel
        if self.p.is_fp8_kv and self.plan.kind == pkv.KIND_PREFILL:
            n += 1  # the FP8 pages expanded to bf16 before the prefill kernel
        return n

    def run(self):
        if self.p.is_mla:
            pkv.run_mla(self.plan, self.q_nope, self.q_pe, self.ckv, self.kpe, self.o, self.lse)
        elif self.p.is_fp8_kv:
            pkv.run_fp8_kv(self.plan, self.q, self.k, self.v, self.k_scale, self.v_scale, self.o, self.lse)
        else:
            pkv.run(self.plan, self.q, self.k, self.v, self.o, self.lse)


class AppendCase:
    """Paged KV append of a whole prefill batch: every request's rows written into
    its pages (the table after the append), K and V, resident in HBM."""

    def __init__(self, p: W.PagedProblem, device):
        self.p = p
        self.k, self.v = p.k_cache.to(device), p.v_cache.to(device)
        kv = p.kv_lens
        self.nnz = int(kv.sum())
        gen = torch.Generator().manual_seed(p.seed + 500)
        shape = (self.nnz, p.num_kv_heads, p.head_dim)
        self.k_new = torch.randn(shape, generator=gen).to(torch.bfloat16).to(device)
        self.v_new = torch.randn(shape, generator=gen).to(torch.bfloat16).to(device)
        dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)
        self.append_indptr = dev(np.concatenate([[0], np.cumsum(kv)]))
        self.kv_indptr, self.kv_indices, self.last = dev(p.kv_indptr), dev(p.kv_indices), dev(p.kv_last_page_len)
        self.launches = 1

    @property
    def bytes(self) -> float:
        """New K and V rows read once and written once, plus the index arrays."""
        rows = 2 * 2 * self.nnz * self.p.num_kv_heads * self.p.head_dim
        return float(2 * rows + 4 * (len(self.p.kv_indices) + 3 * (self.p.batch + 1)))

    def run(self):
        pkv.append_kv(self.k_new, self.v_new, self.append_indptr, self.kv_indptr, self.kv_indices, self.last,
                      self.k, self.v)


def time_case(case: Case, flush: torch.Tensor, steps: int, warmup: int):
    """Median and mean kernel time (ms) of `case.run`, L2 flushed before every launch."""
    for _ in range(warmup):
        flush.zero_()
        case.run()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        case.run()
        b.record()
        times.append((a, b))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in times]
    return float(np.median(ms)), float(np.mean(ms))


def e2e_prefill(p: W.PagedProblem, device, steps: int, warmup: int):
    """Prefill through the public API from pinned host buffers, copies inside the timed region."""
    hq = p.q.pin_memory()
    hk = p.k_cache.pin_memory()
    hv = p.v_cache.pin_memory()
    hidx = torch.from_numpy(p.kv_indices.astype(np.int32)).pin_memory()
    ho = torch.empty(p.total_q, p.num_qo_heads, p.head_dim_v, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(p.total_q, p.num_qo_heads, dtype=torch.float32).pin_memory()
    dq, dk, dv = torch.empty_like(hq, device=device), torch.empty_like(hk, device=device), torch.empty_like(hv, device=device)
    didx = torch.empty_like(hidx, device=device)
    do = torch.empty_like(ho, device=device)
    dl = torch.empty_like(hl, device=device)
    plans = []

    def step():
        didx.copy_(hidx, non_blocking=True)
        pl = pkv.plan(p.qo_indptr, p.kv_indptr, didx, p.kv_last_page_len, p.num_qo_heads, p.num_kv_heads,
                      p.head_dim, p.page_size, p.causal, p.sm_scale)
        plans.append(pl)  # keep the plan (and its pinned staging) alive until the stream drains
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        pkv.run(pl, dq, dk, dv, do, dl)
        ho.copy_(do, non_blocking=True)
        hl.copy_(dl, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    plans.clear()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + hidx.numel() * 4
    d2h = ho.numel() * 2 + hl.numel() * 4
    return ms, h2d, d2h


def _blas_threads() -> int:
    """Threads NumPy's BLAS runs with (the oracle's matmuls), else the CPU affinity."""
    try:
        import threadpoolctl
        n = [p["num_threads"] for p in threadpoolctl.threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except ImportError:
        pass
    return len(os.sched_getaffinity(0))


def _oracle_sample(p, order, seconds_target: float):
    """Whole requests of `p` in `order` through the oracle until the target time is spent."""
    import oracle
    t0 = time.perf_counter()
    flops, done = 0.0, []
    for b in order:
        oracle.paged_attention(p.q, p.k_cache, p.v_cache, p.qo_indptr, p.kv_indptr, p.kv_indices,
                               p.kv_last_page_len, p.page_size, True, p.sm_scale, requests=[b])
        L = int(p.qo_lens[b])
        flops += 2.0 * (2 * p.head_dim) * p.num_qo_heads * L * (L + 1) / 2
        done.append(L)
        if time.perf_counter() - t0 > seconds_target:
            break
    return flops, done, time.perf_counter() - t0


def cpu_baseline(seconds_target: float = 15.0):
    """The float64 oracle, as it stands, on a bounded sample of the prefill workload:
    whole requests of the h16/kv1/d128/ps64 batch, shortest first, until the target
    CPU time is spent, with every BLAS thread; then the shortest request again with
    BLAS limited to one thread. Returns TFLOP/s on the sample's causal FLOPs."""
    p = W.gqa_prefill()
    order = np.argsort(p.qo_lens).tolist()
    flops, done, dt = _oracle_sample(p, order, seconds_target)
    out = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{len(done)} of 8 requests of the h16/kv1/d128/ps64 prefill batch "
                     f"(qo_len {done}), float64 NumPy, {dt:.1f} s",
           "affinity": len(os.sched_getaffinity(0))}
    try:
        import threadpoolctl
        with threadpoolctl.threadpool_limits(1, user_api="blas"):
            f1, d1, t1 = _oracle_sample(p, order[:1], 0.0)
        out["value_1_thread"] = f1 / t1 / 1e12
        out["sample_1_thread"] = f"the shortest request (qo_len {d1[0]}) with one BLAS thread, {t1:.1f} s"
    except ImportError:
        pass
    return out


def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest of every rank's `x` (all ranks call it, in the same order)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device="cuda") -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def job_throughput(local_work: float, local_ms: float, world: int, device="cuda"):
    """Whole-job throughput of a weak-scaled run: the work every rank did, over
    the slowest rank's time. Returns (work per second, max ms)."""
    total = sum_over_ranks(local_work, world, device)
    ms = max_over_ranks(local_ms, world, device)
    return total / (ms * 1e-3), ms


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def run_ours(args):
    rank, world, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_kind = load_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    if args.only:
        return run_only(args, device, flush)
    # one independent batch per rank (weak scaling: no data-path collective)
    pre = Case(W.gqa_prefill(shard=rank), device)
    dec = Case(W.paged_decode(shard=rank), device)
    cases = [pre, dec]
    mla = None
    try:
        mla = Case(W.mla_prefill(shard=rank), device)
        mla.run()
        torch.cuda.synchronize()
        cases.append(mla)
    except pkv.PkvError:
        mla = None

    # warm-up steps
    for _ in range(args.warmup):
        for c in cases:
            flush.zero_()
            c.run()
    barrier(world)

    ev = {id(c): [] for c in cases}
    sampler = ClockSampler(local)
    with sampler:
        barrier(world)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record()
        for _ in range(args.steps):
            for c in cases:
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                c.run()
                b.record()
                ev[id(c)].append((a, b))
        t_end.record()
        barrier(world)
    clocks = sampler.summary()

    def mean_ms(c):
        return float(np.mean([a.elapsed_time(b) for a, b in ev[id(c)]]))

    pre_flops = attention_flops(pre.p)
    dec_bytes = decode_bytes(dec.p)
    job_flops_s, pre_ms = job_throughput(pre_flops, mean_ms(pre), world)
    job_bytes_s, dec_ms = job_throughput(dec_bytes, mean_ms(dec), world)
    mla_ms = max_over_ranks(mean_ms(mla), world) if mla else None
    step_ms = pre_ms + dec_ms + (mla_ms or 0.0)

    # Rows beyond the step (timed the same way, each alone between L2 flushes):
    # MLA decode, the FP8-KV decode and the paged KV append.
    extra_steps = max(3, min(args.steps, 20))
    mdec = Case(W.mla_decode(shard=rank), device)
    mdec_med, mdec_ms_local = time_case(mdec, flush, extra_steps, 3)
    mdec_ms = max_over_ranks(mdec_ms_local, world)
    fdec = Case(W.paged_decode_fp8(shard=rank), device)
    fdec_med, fdec_ms_local = time_case(fdec, flush, extra_steps, 3)
    fdec_ms = max_over_ranks(fdec_ms_local, world)
    pfp8 = Case(W.gqa_prefill_fp8(shard=rank), device)
    pfp8_med, pfp8_ms_local = time_case(pfp8, flush, extra_steps, 3)
    pfp8_ms = max_over_ranks(pfp8_ms_local, world)
    app = AppendCase(W.gqa_prefill(shard=rank), device)
    app_med, app_ms_local = time_case(app, flush, extra_steps, 3)
    app_ms = max_over_ranks(app_ms_local, world)
    tflops = job_flops_s / 1e12
    per_gpu_tflops = pre_flops / (pre_ms * 1e-3) / 1e12
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9

    # e2e through the public API with host buffers
    e2e_local_ms, h2d, d2h = e2e_prefill(pre.p, device, max(2, min(args.steps, 10)), 2)
    e2e_flops_s, e2e_ms = job_throughput(pre_flops, e2e_local_ms, world)

    peak_burst = float(peaks["bf16_tflops"])
    peak_sust = float(peaks.get("bf16_tflops_sustained", peak_burst))
    hbm = float(peaks["hbm_gbs"])
    roofs = {
        "prefill_kernel<128> (h16/kv1/d128/ps64)": {
            "bound": "tensor", "achieved": round(per_gpu_tflops, 2), "peak": peak_burst, "unit": "TFLOP/s",
            "frac": round(per_gpu_tflops / peak_burst, 4), "frac_of_sustained": round(per_gpu_tflops / peak_sust, 4),
            "traffic": profiled_traffic("prefill_gqa_h16_kv1_d128_ps64.md", PREFILL_SOURCES), "ms": round(pre_ms, 4)},
        "decode_kernel<128> (b128/h32/kv8/d128/ps16)": {
            "bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(dec_gbs / hbm, 4),
            "traffic": profiled_traffic("decode_b32_h32_kv8_d128_ps16.md", DECODE_SOURCES,
                                        kv_tokens=int(dec.p.kv_lens.sum())),
            "ms": round(dec_ms, 4)},
    }
    if mla:
        mla_tf = attention_flops(mla.p) / (mla_ms * 1e-3) / 1e12
        roofs["mla_kernel (h16/ckv512/kpe64/ps1)"] = {
            "bound": "tensor", "achieved": round(mla_tf, 2), "peak": peak_burst, "unit": "TFLOP/s",
            "frac": round(mla_tf / peak_burst, 4),
            "traffic": profiled_traffic("mla_h16_ckv512_kpe64_ps1.md", MLA_SOURCES), "ms": round(mla_ms, 4)}
    mdec_gbs = decode_bytes(mdec.p) / (mdec_ms * 1e-3) / 1e9
    roofs["mla_decode_kernel (b64/h16/ckv512/kpe64/ps1)"] = {
        "bound": "hbm", "achieved": round(mdec_gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(mdec_gbs / hbm, 4),
        "traffic": profiled_traffic("mla_decode_b64_h16_ckv512_kpe64_ps1.md", MLA_DECODE_SOURCES), "ms": round(mdec_ms, 4),
        "in_step": False}
    fdec_gbs = decode_bytes(fdec.p) / (fdec_ms * 1e-3) / 1e9
    roofs["decode_fp8_kernel<128> (b128/h32/kv8/d128/ps16, FP8 E4M3 KV)"] = {
        "bound": "hbm", "achieved": round(fdec_gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(fdec_gbs / hbm, 4),
        "traffic": profiled_traffic("decode_fp8_b32_h32_kv8_d128_ps16.md", DECODE_FP8_SOURCES,
                                    kv_tokens=int(fdec.p.kv_lens.sum())),
        "ms": round(fdec_ms, 4), "in_step": False}
    pfp8_tf = attention_flops(pfp8.p) / (pfp8_ms * 1e-3) / 1e12
    roofs["prefill_kernel<128> over an FP8 E4M3 KV cache (h16/kv1/d128/ps64; expand + prefill)"] = {
        "bound": "tensor", "achieved": round(pfp8_tf, 2), "peak": peak_burst, "unit": "TFLOP/s",
        "frac": round(pfp8_tf / peak_burst, 4),
        "traffic": profiled_traffic("prefill_fp8_h16_kv1_d128_ps64.md", PREFILL_FP8_SOURCES),
        "ms": round(pfp8_ms, 4), "in_step": False}
    app_gbs = app.bytes / (app_ms * 1e-3) / 1e9
    roofs["append_kernel (h16/kv1/d128/ps64 batch)"] = {
        "bound": "hbm", "achieved": round(app_gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(app_gbs / hbm, 4),
        "traffic": profiled_traffic("append_h16_kv1_d128_ps64.md", APPEND_SOURCES), "ms": round(app_ms, 4),
        "in_step": False}
    dominant = max((k for k in roofs if roofs[k].get("in_step", True)), key=lambda k: roofs[k]["ms"])
    roofline = dict(roofs[dominant], kernel=dominant,
                    peak_kind=f"{peak_kind} (burst bf16 for tensor-bound kernels timed alone between L2 flushes; "
                              "copy bandwidth for HBM-bound)")

    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded bf16 N(0,1), random page permutation)",
        "config": {
            "workload": "gqa_paged_prefill_causal_h16_kv1_d128_ps64: batch 8, qo_len=kv_len U[512,4096], "
                        "page_size 64, permuted pool",
            "lengths": pre.p.qo_lens.tolist(),
            "parallelism": f"dp{world} (independent batches per GPU)",
            "l2": "flushed (256 MiB write) before every timed launch",
            "step": "prefill h16/kv1/d128/ps64 + decode b128/h32/kv8/d128/ps16" + (" + MLA h16/ckv512/kpe64/ps1" if mla else ""),
        },
        "pct_bf16_peak": round(100 * per_gpu_tflops / peak_burst, 2),
        "prefill": {"ms": round(pre_ms, 4), "flops": pre_flops, "tflops_per_gpu": round(per_gpu_tflops, 2),
                    "units": pre.plan.num_units, "merges": pre.plan.num_merges},
        "decode": {"value": round(dec_gbs, 1), "job_value": round(job_bytes_s / 1e9, 1), "unit": "GB/s", "ms": round(dec_ms, 4), "bytes": dec_bytes,
                   "frac": round(dec_gbs / hbm, 4), "peak": hbm, "peak_kind": peak_kind,
                   "units": dec.plan.num_units, "merges": dec.plan.num_merges,
                   "workload": "paged_decode_b128_h32_kv8_d128_ps16, kv_len U[1024,8192]"},
        "roofline": roofline,
        "rooflines": roofs,
        "e2e": {"value": round(e2e_flops_s / 1e12, 2), "unit": "TFLOP/s",
                "ms": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "includes": "plan + upload + H2D(q, k, v, kv_indices) + run + D2H(o, lse)"},
        "gpu_launches": int(args.steps * sum(c.launches for c in cases)),
        "clocks": clocks,
    }
    if mla:
        mla_flops = attention_flops(mla.p)
        line["mla"] = {"value": round(mla_flops / (mla_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                       "ms": round(mla_ms, 4), "flops": mla_flops,
                       "workload": "mla_paged_prefill_causal_h16_ckv512_kpe64_ps1, batch 4, U[256,2048]"}
    line["mla_decode"] = {"value": round(mdec_gbs, 1), "unit": "GB/s", "ms": round(mdec_ms, 4),
                          "bytes": decode_bytes(mdec.p), "units": mdec.plan.num_units, "merges": mdec.plan.num_merges,
                          "workload": "mla_paged_decode_h16_ckv512_kpe64_ps1, batch 64, kv_len U[1024,8192]",
                          "timed": "alone, outside the step, L2 flushed before each launch"}
    line["decode_fp8"] = {"value": round(fdec_gbs, 1), "unit": "GB/s", "ms": round(fdec_ms, 4),
                          "bytes": decode_bytes(fdec.p), "units": fdec.plan.num_units,
                          "merges": fdec.plan.num_merges,
                          "workload": "paged_decode_b128_h32_kv8_d128_ps16 over an FP8 E4M3 KV cache with "
                                      "per-kv-head scales, kv_len U[1024,8192]",
                          "timed": "alone, outside the step, L2 flushed before each launch"}
    line["prefill_fp8"] = {"value": round(pfp8_tf, 2), "unit": "TFLOP/s", "ms": round(pfp8_ms, 4),
                           "flops": attention_flops(pfp8.p), "units": pfp8.plan.num_units,
                           "workload": "the config-2 prefill batch (h16/kv1/d128/ps64, causal, U[512,4096]) over "
                                       "an FP8 E4M3 KV cache with per-kv-head scales; the pages expanded to bf16, "
                                       "then the tensor-core prefill",
                           "timed": "alone, outside the step, L2 flushed before each launch pair"}
    line["append"] = {"value": round(app_gbs, 1), "unit": "GB/s", "ms": round(app_ms, 4), "bytes": app.bytes,
                      "rows": app.nnz, "workload": "append of the whole h16/kv1/d128/ps64 prefill batch (K and V)",
                      "timed": "alone, outside the step, L2 flushed before each launch"}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if world == 1 and not args.no_sweep:
        line["sparse_vs_dense"] = sparse_dense_sweep(device, flush, args)
    print(json.dumps(line), flush=True)


def run_only(args, device, flush):
    """One workload alone (for profiler captures): W warm-up and K timed launches."""
    makers = {"prefill": W.gqa_prefill, "decode": W.paged_decode, "mla": W.mla_prefill,
              "decode_small": lambda: W.paged_decode(batch=32),
              "sparse": lambda: W.sparse_vs_dense(16, 2048, False),
              "dense": lambda: W.sparse_vs_dense(16, 2048, True),
              "mla_decode": W.mla_decode, "decode_fp8": W.paged_decode_fp8,
              "decode_fp8_small": lambda: W.paged_decode_fp8(batch=32), "prefill_fp8": W.gqa_prefill_fp8}
    if args.only == "append":
        c = AppendCase(W.gqa_prefill(), device)
        sampler = ClockSampler(device.index or 0)
        with sampler:
            med, mean = time_case(c, flush, args.steps, args.warmup)
        print(json.dumps({"only": "append", "ms_median": med, "ms_mean": mean, "gbs": c.bytes / (med * 1e-3) / 1e9,
                          "rows": c.nnz, "clocks": sampler.summary()}), flush=True)
        return
    c = Case(makers[args.only](), device)
    sampler = ClockSampler(device.index or 0)
    with sampler:
        med, mean = time_case(c, flush, args.steps, args.warmup)
    f = attention_flops(c.p)
    print(json.dumps({"only": args.only, "ms_median": med, "ms_mean": mean,
                      "tflops": f / (med * 1e-3) / 1e12,
                      "gbs": decode_bytes(c.p) / (med * 1e-3) / 1e9 if "decode" in args.only else None,
                      "units": c.plan.num_units, "merges": c.plan.num_merges,
                      "clocks": sampler.summary()}), flush=True)


class DenseCase:
    """The dense (contiguous ragged) layout of a vector-sparse problem already in
    HBM: the same queries, and every request's K/V rows gathered on the device into
    order, described to the kernel as 64-slot pages with the identity page table
    (every length of the sweep is a multiple of 64)."""

    def __init__(self, sparse: Case):
        p = sparse.p
        hk, d = p.num_kv_heads, p.head_dim
        rows = sparse.idx.long()
        self.q = sparse.q
        self.k = sparse.k.view(-1, hk, d)[rows].view(-1, 64, hk, d)
        self.v = sparse.v.view(-1, hk, d)[rows].view(-1, 64, hk, d)
        kv_lens = p.kv_lens
        n_pages = kv_lens // 64
        kv_indptr = np.concatenate([[0], np.cumsum(n_pages)]).astype(np.int32)
        self.idx = torch.arange(int(kv_indptr[-1]), dtype=torch.int32, device=self.q.device)
        self.plan = pkv.plan(p.qo_indptr, kv_indptr, self.idx, np.full(p.batch, 64, np.int32), p.num_qo_heads, hk,
                             d, 64, True, p.sm_scale)
        self.o, self.lse = torch.empty_like(sparse.o), torch.empty_like(sparse.lse)
        self.launches = 1 + (1 if self.plan.num_merges > 0 else 0)

    def run(self):
        pkv.run(self.plan, self.q, self.k, self.v, self.o, self.lse)


def sparse_dense_sweep(device, flush, args):
    """Config 3 of the pages' benchmark: vector-sparse (page_size 1, token slots
    scattered over the pool) against the dense layout of the same problem, for
    every (B, L) of the sweep, each timed alone between L2 flushes (median of
    CUDA-event times). TFLOP/s count the causal FLOPs; ratio = dense time / sparse time."""
    out = []
    for B, L in W.SPARSE_DENSE_SWEEP:
        sp = W.sparse_vs_dense(B, L, contiguous=False)
        cs = Case(sp, device)
        cd = DenseCase(cs)
        ms_s, _ = time_case(cs, flush, max(10, args.steps), 3)
        ms_d, _ = time_case(cd, flush, max(10, args.steps), 3)
        f = attention_flops(sp)
        out.append({"B": B, "L": L, "sparse_tflops": round(f / ms_s / 1e9, 1),
                    "dense_tflops": round(f / ms_d / 1e9, 1), "ratio": round(ms_d / ms_s, 3),
                    "sparse_ms": round(ms_s, 4), "dense_ms": round(ms_d, 4)})
        del cs, cd
        torch.cuda.empty_cache()
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    import oracle
    p = W.gqa_prefill()
    b = int(np.argmin(p.qo_lens))
    L = int(p.qo_lens[b])
    flops = 2.0 * (2 * p.head_dim) * p.num_qo_heads * L * (L + 1) / 2
    for _ in range(args.warmup):
        pass  # the oracle has no state to warm; warm-up steps are not repeated on the CPU
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.paged_attention(p.q, p.k_cache, p.v_cache, p.qo_indptr, p.kv_indptr, p.kv_indices,
                               p.kv_last_page_len, p.page_size, True, p.sm_scale, requests=[b])
    dt = (time.perf_counter() - t0) / args.steps
    value = flops / dt / 1e12
    cores = _blas_threads()
    sample = (f"request {b} (qo_len = kv_len = {L}) of the h16/kv1/d128/ps64 prefill batch per step, "
              f"float64 NumPy oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "gqa_paged_prefill_causal_h16_kv1_d128_ps64 (one request per step)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sweep", action="store_true",
                    help="run the vector-sparse vs dense sweep (the default; kept as an alias)")
    ap.add_argument("--no-sweep", action="store_true", help="skip the vector-sparse vs dense sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["prefill", "decode", "decode_small", "mla", "mla_decode", "sparse", "dense", "append",
                                       "decode_fp8", "decode_fp8_small", "prefill_fp8"], default=None,
                    help="time one workload alone (profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
