"""Benchmark: exact split decode attention on B200.

One step = one decode step of the whole hot path (split-KV chunk statistics, their
log-depth merge and the final normalisation: one fused kernel launch) over the
long-context workload: batch 1, 32 query heads, 8 KV heads, head_dim 128, KV length
1,048,576, bf16 K/V ~ N(0,1) with 0.1% of keys scaled x4.  Inputs are synthetic and
seeded (4.3 GB of K/V, larger than the 126 MB L2, so no flush between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Prints one JSON line (rank 0).  Under torchrun with N > 1 every rank runs its own
replica of the workload (no data-path collective: the path does not shard), the
timed region is bracketed by a barrier and synchronisation, and the time is the max
over ranks.  `--impl reference` times the CPU oracle instead: every step is a full
step of the workload (all rows), threaded over (sequence, query head) rows.

Other workloads (--workload): the decode configurations, several query tokens per
sequence, paged caches, the shared-prefix (bifurcated) step and context encoding with
anchor blocks.  Each line's roofline is that of the step's main kernel, timed with CUDA
events that the library records around its launches (tree_attn_profile_events) in K steps
interleaved with the K timed steps, which carry no such events.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode-attn KV GB/s & % of B200 HBM peak at 1M ctx; µs/step, KV tokens/s"
UNIT = "GB/s"
ANCHOR_METRIC = "context-encoding attention TFLOP/s (anchor-block mask, exact); µs/step, tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# DRAM traffic per launch from committed ncu captures, per family of main kernel: the capture
# file and the sources it was taken from (a capture counts only while they are unchanged).
_CSRC = "exact_long_context_split_b200/csrc/"
TRAFFIC = {
    "split": ("split_kv_traffic.json", [_CSRC + "split_kv.cuh", _CSRC + "ptx.cuh"]),
    "tc_decode": ("bif_prefix_decode_traffic.json", [_CSRC + "bifurcated_tc.cuh", _CSRC + "ptx.cuh"]),
}


# ----------------------------------------------------------------------------------------------
# Host-side pieces shared by every rank (and covered by CPU tests)
# ----------------------------------------------------------------------------------------------


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(value: float, world: int) -> float:
    """The largest value over all ranks (every rank takes this collective step)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def kernel_hash(sources) -> str:
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    """(HBM GB/s, dense bf16 TF/s burst, kind): the measured copy and GEMM peaks of this
    pool's B200s, else the recorded fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def traffic_per_launch(spec, family) -> object:
    """DRAM bytes (read + write) of one launch of the family's main kernel from its committed ncu
    capture: the mean of the captured launches for the captured workload, reads scaled by K/V
    bytes for another one.  None without a capture, or when the kernel's sources changed since
    the counters were taken."""
    if family not in TRAFFIC:
        return None
    name, sources = TRAFFIC[family]
    try:
        with open(os.path.join(ROOT, "profiles", name)) as fh:
            d = json.load(fh)
    except Exception:
        return None
    if d.get("kernel_hash") != kernel_hash(sources):
        return None
    rd = statistics.mean(d["dram_bytes_read"])
    wr = statistics.mean(d["dram_bytes_write"])
    if spec.name != d["workload"]:
        rd *= spec.kv_bytes / d["kv_bytes"]
    return int(round(rd + wr))


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ClockSampler:
    """SM clock and clock-event (throttle) reasons read through NVML while the timed region
    runs: a host thread samples every 2 ms, and start() and stop() each take one sample
    themselves, so the window always holds its two edge samples even when it is shorter than
    the sampling period.  Only reads device state."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.idx = torch_device_index
        self.period = period_s
        self.samples = []
        self.window = [None, None]
        self.err = None
        self.max_mhz = None
        self._stop = False
        self._thread = None
        self._nv = None
        self._h = None

    def _handle(self, nv):
        import torch

        try:
            pr = torch.cuda.get_device_properties(self.idx)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.idx)

    def _sample(self):
        nv, h = self._nv, self._h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), int(get_reasons(h))))

    def _run(self):
        try:
            while not self._stop:
                self._sample()
                time.sleep(self.period)
        except Exception as e:  # never fail the bench on a sampling error
            self.err = f"nvml: {e}"

    def __enter__(self):
        import threading

        try:  # initialised here, before any timing, so the first sample cannot arrive late
            import pynvml as nv

            nv.nvmlInit()
            self._nv, self._h = nv, self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:
            self.err = f"nvml: {e}"
        return self

    def start(self):
        if self._nv is not None and self.err is None:
            self._sample()
        self.window[0] = time.perf_counter()

    def stop(self):
        self.window[1] = time.perf_counter()
        if self._nv is not None and self.err is None:
            self._sample()

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=5)
        if self._nv is not None:
            try:
                self._nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if self.err or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"], "samples": 0}
        t0, t1 = self.window
        # the edge samples taken by start() and stop() sit just outside [t0, t1]: widen by 1 ms
        inside = [s for s in self.samples if t0 is not None and t1 is not None and t0 - 1e-3 <= s[0] <= t1 + 1e-3]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples in the timed window"],
                    "samples": 0}
        reasons = sorted({name for _, _, r in inside for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside), "source": "nvml: 2 ms thread + start/stop edges"}


def workload_config(spec, n_gpus: int) -> dict:
    if isinstance(spec, synth.DecodeSpec):
        shape = {"batch": spec.batch, "seq_len": int(max(spec.seqlens)) if spec.seqlens else 0,
                 "query_tokens": spec.n_queries, **({"page_size": spec.page_size} if spec.page_size else {})}
    elif isinstance(spec, synth.BifurcatedSpec):
        shape = {"samples": spec.n_samples, "prefix_len": spec.prefix_len,
                 "suffix_len": int(max(spec.suffix_lens)) if spec.suffix_lens else 0}
    else:
        shape = {"seq_len": spec.seq_len, "block_size": spec.block_size}
    l2 = ("no flush: each step reads %.2f GB of K/V, more than the 126 MB L2" % (spec.kv_bytes / 1e9)
          if spec.kv_bytes > 2 * 126e6 else
          "L2 flushed before every step (a 512 MB write outside the timed span)")
    return {"workload": spec.name, **shape, "n_q_heads": spec.n_q_heads, "n_kv_heads": spec.n_kv_heads,
            "head_dim": spec.head_dim, "kv_bytes_per_step": spec.kv_bytes, "parallelism": f"replicas{n_gpus}",
            "l2": l2}


def make_record(*, metric, unit, value, n_gpus, steps, warmup, ms_per_step, spec, dtype, extra) -> dict:
    rec = {
        "metric": metric,
        "value": value,
        "unit": unit,
        "n_gpus": n_gpus,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic",
        "config": workload_config(spec, n_gpus),
    }
    rec.update(extra)
    return rec


# ----------------------------------------------------------------------------------------------
# The CPU oracle, threaded over (sequence, query head) rows
# ----------------------------------------------------------------------------------------------


def oracle_step_seconds(spec, inp, rows, threads: int) -> float:
    """Wall time of the CPU oracle computing the given (sequence, query head) rows of a decode
    workload, one row per task on `threads` threads (numpy releases the GIL in the oracle's array
    work; BLAS held to one thread per task).  The oracle is called as it stands; only its
    widening piece size, a memory setting, is lowered so that every thread's pieces fit."""
    import threadpoolctl

    import oracle
    from oracle import attention as oracle_attention

    def one(row):
        oracle.decode_attention(inp["q"], inp["k"], inp["v"], spec.seqlens, spec.n_q_heads, spec.n_kv_heads,
                                spec.head_dim, spec.scale, dtype=spec.dtype, pairs=[row])

    saved = oracle_attention.ROWS_PER_PIECE
    oracle_attention.ROWS_PER_PIECE = 1 << 18
    try:
        with threadpoolctl.threadpool_limits(1), cf.ThreadPoolExecutor(threads) as ex:
            t0 = time.perf_counter()
            list(ex.map(one, rows))
            return time.perf_counter() - t0
    finally:
        oracle_attention.ROWS_PER_PIECE = saved


def decode_rows(spec):
    return [(b, h) for b in range(spec.batch) for h in range(spec.n_q_heads)]


def cpu_baseline(spec, inp, budget_s: float = 30.0) -> dict:
    """The oracle on one full decode step (every row) when a probe says it fits in `budget_s`,
    else on a bounded sample of rows scaled to the step; threads = min(cores, rows)."""
    rows = decode_rows(spec)
    cores = host_cores()
    threads = max(1, min(cores, len(rows)))
    probe = oracle_step_seconds(spec, inp, rows[:threads], threads)  # one row per thread
    est = probe * len(rows) / threads
    if est <= budget_s:
        sec = oracle_step_seconds(spec, inp, rows, threads)
        sample = f"one full step: all {len(rows)} (sequence, query head) rows, {threads} threads"
    else:
        n = max(threads, int(len(rows) * budget_s / est) // threads * threads)
        stride = max(1, len(rows) // n)
        sub = rows[::stride][:n]
        sec = oracle_step_seconds(spec, inp, sub, threads) * len(rows) / len(sub)
        sample = (f"{len(sub)} of {len(rows)} (sequence, query head) rows (every {stride}th), {threads} threads; "
                  f"step time = sample time x {len(rows)}/{len(sub)}")
    return {"value": spec.kv_bytes / sec / 1e9, "unit": UNIT, "cores": threads, "host_cores": cores,
            "kind": "oracle", "sample": sample, "step_s": sec}


# ----------------------------------------------------------------------------------------------
# Reference arm: the CPU oracle
# ----------------------------------------------------------------------------------------------


def run_reference(args, spec) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    inp = synth.make_decode_inputs(spec)
    rows = decode_rows(spec)
    cores = host_cores()
    threads = max(1, min(cores, len(rows)))
    t_first = oracle_step_seconds(spec, inp, rows, threads)  # the first warm-up step, full
    budget = 180.0  # the whole run stays within a few minutes
    full = t_first * (args.warmup + args.steps) <= budget
    if full:
        sub = rows
        sample = f"each step: all {len(rows)} (sequence, query head) rows of the workload, {threads} threads"
    else:
        n = max(threads, int(len(rows) * budget / (t_first * (args.warmup + args.steps))) // threads * threads)
        stride = max(1, len(rows) // n)
        sub = rows[::stride][:n]
        sample = (f"each step: {len(sub)} of {len(rows)} rows (every {stride}th), {threads} threads; "
                  f"step time = sample time x {len(rows)}/{len(sub)}")
    for _ in range(max(0, args.warmup - 1)):
        oracle_step_seconds(spec, inp, sub, threads)
    times = [oracle_step_seconds(spec, inp, sub, threads) * len(rows) / len(sub) for _ in range(args.steps)]
    step_s = statistics.mean(times)
    value = spec.kv_bytes / step_s / 1e9
    rec = make_record(metric=METRIC, unit=UNIT, value=value, n_gpus=world, steps=args.steps, warmup=args.warmup,
                      ms_per_step=step_s * 1e3, spec=spec, dtype="f64", extra={
                          "impl": "reference",
                          "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "host_cores": cores,
                                           "kind": "oracle", "sample": sample},
                          "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                          "gpu_launches": 0,
                      })
    print(json.dumps(rec), flush=True)


# ----------------------------------------------------------------------------------------------
# The CUDA path
# ----------------------------------------------------------------------------------------------


def to_device_bf16(torch, arr):
    return torch.from_numpy(np.ascontiguousarray(arr).reshape(-1).view(np.int16)).view(torch.bfloat16).pin_memory()


class DecodeRun:
    """Device and pinned-host buffers of one decode workload and its step (one kernel launch)."""

    launches_per_step = 1
    metric, unit, bound = METRIC, UNIT, "hbm"

    def __init__(self, spec, torch, ta, keep_inputs=False, decode_path=0):
        self.spec, self.torch, self.ta = spec, torch, ta
        B, Hq, Hkv, D = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.seqlens = [int(s) for s in spec.seqlens]
        # ta_options.prefix_path for plain decode: 0 automatic, 1 tensor cores, 2 split kernel
        self.opts = ta.make_options(prefix_path=decode_path) if decode_path else None
        inp = synth.make_decode_inputs(spec)
        self.host = {n: to_device_bf16(torch, inp[n]) for n in ("q", "k", "v")}
        self.inputs = inp if keep_inputs else None
        del inp
        self.dev = {n: t.cuda() for n, t in self.host.items()}
        self.out = torch.empty(B, Hq, D, device="cuda")
        self.lse = torch.empty(B, Hq, device="cuda")
        self.ws = torch.empty(ta.tree_attn_workspace_size(self.seqlens, Hq, Hkv, D, "bf16", self.opts),
                              dtype=torch.uint8, device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        self.kv_bytes = spec.kv_bytes
        self.tokens = spec.tokens
        self.flops = 4 * D * Hq * sum(self.seqlens)
        self.kernel = f"split_kv_decode_kernel<bf16,{D},{Hq // Hkv},{'ShortTiles' if sum(self.seqlens) < 1024 * len(self.seqlens) else 'LongTiles'}>"
        self.family = "split"
        if D == 128 and ((Hq // Hkv == 8 and decode_path != 2) or decode_path == 1):  # tensor-core decode
            self.family = "tc_decode"
            self.launches_per_step = 2 * ((B + 127) // 128)
            self.kernel = f"bif_prefix_kernel (decode, {Hq // Hkv} rows per KV head)"

    def step(self, stream):
        sp = self.spec
        self.ta.tree_attn_decode_ex("bf16", self.dev["q"], self.dev["k"], self.dev["v"], self.seqlens, sp.n_q_heads,
                                    sp.n_kv_heads, sp.head_dim, sp.scale, self.out, self.lse, self.opts, self.ws,
                                    stream=stream)


def multi_visible_keys(seqlens, n):
    return sum(n * S - n * (n - 1) // 2 for S in seqlens)


class MultiRun(DecodeRun):
    """Several query tokens per sequence: one call = the tensor-core form (bf16, D = 128,
    8 <= G n <= 128) or ceil(n G / 8) split-KV passes."""

    def __init__(self, spec, torch, ta, keep_inputs=False):
        super().__init__(spec, torch, ta, keep_inputs)
        B, n, Hq, Hkv, D = spec.batch, spec.n_queries, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.out = torch.empty(B, n, Hq, D, device="cuda")
        self.lse = torch.empty(B, n, Hq, device="cuda")
        self.ws = torch.empty(ta.tree_attn_multi_workspace_size(self.seqlens, n, Hq, Hkv, D), dtype=torch.uint8,
                              device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        self.flops = 4 * D * Hq * multi_visible_keys(self.seqlens, n)
        G = Hq // Hkv
        if D == 128 and 8 <= G * n <= 128:
            # tensor-core form (the library's automatic choice for bf16): per group of up to 128
            # sequences one bif_prefix_kernel launch and one merge_chunks_kernel launch
            groups = (B + 127) // 128
            self.launches_per_step = 2 * groups
            self.kernel = f"bif_prefix_kernel (several query tokens, {G * n} rows per KV head)"
        else:
            passes, j = 0, 0
            while j < n:
                step = 1
                while 2 * step <= n - j and 2 * step * G <= 8:
                    step *= 2
                j += step
                passes += 1
            self.launches_per_step = passes
            self.kernel = f"split_kv_decode_kernel<bf16,{D},G*n'> x {passes} passes"

    def step(self, stream):
        sp = self.spec
        self.ta.tree_attn_decode_multi_ex("bf16", self.dev["q"], self.dev["k"], self.dev["v"], self.seqlens,
                                          sp.n_queries, sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.scale, self.out,
                                          self.lse, None, self.ws, stream=stream)


class PagedRun(DecodeRun):
    """A paged cache: the contiguous cache laid out in page_size-token blocks at seeded random
    places (built once on the device); each step reads it through the block table."""

    def __init__(self, spec, torch, ta, keep_inputs=False):
        super().__init__(spec, torch, ta, keep_inputs)
        Hkv, D, ps = spec.n_kv_heads, spec.head_dim, spec.page_size
        table, self.num_pages = synth.page_table(spec.seed, spec.seqlens, ps)
        self.table = torch.from_numpy(table).cuda()
        self.stride = table.shape[1]
        for name in ("k", "v"):
            pages = torch.zeros(self.num_pages, Hkv, ps, D, dtype=torch.bfloat16, device="cuda")
            off = 0
            for b, S in enumerate(self.seqlens):
                nb = -(-S // ps)
                blk = torch.zeros(Hkv, nb * ps, D, dtype=torch.bfloat16, device="cuda")
                blk[:, :S] = self.dev[name][off:off + Hkv * S * D].view(Hkv, S, D)
                off += Hkv * S * D
                pages[self.table[b, :nb].long()] = blk.view(Hkv, nb, ps, D).permute(1, 0, 2, 3)
            self.dev[name] = pages.view(-1)
            self.host[name] = pages.view(-1).cpu().pin_memory()  # the end-to-end leg uploads pages
        self.kernel += " (paged, %d-token blocks)" % ps

    def step(self, stream):
        sp = self.spec
        self.ta.tree_attn_decode_paged_ex("bf16", self.dev["q"], self.dev["k"], self.dev["v"], self.num_pages,
                                          sp.page_size, self.table, self.stride, self.seqlens, sp.n_q_heads,
                                          sp.n_kv_heads, sp.head_dim, sp.scale, self.out, self.lse, None, self.ws,
                                          stream=stream)


class PagedMultiRun(PagedRun):
    """Several query tokens per sequence over a paged cache (the tensor-core form when eligible)."""

    def __init__(self, spec, torch, ta, keep_inputs=False):
        super().__init__(spec, torch, ta, keep_inputs)
        B, n, Hq, Hkv, D = spec.batch, spec.n_queries, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.out = torch.empty(B, n, Hq, D, device="cuda")
        self.lse = torch.empty(B, n, Hq, device="cuda")
        self.ws = torch.empty(ta.tree_attn_multi_workspace_size(self.seqlens, n, Hq, Hkv, D), dtype=torch.uint8,
                              device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        self.flops = 4 * D * Hq * multi_visible_keys(self.seqlens, n)
        tc = D == 128 and 8 <= (Hq // Hkv) * n <= 128
        self.launches_per_step = 2 * ((B + 127) // 128) if tc else self.launches_per_step
        self.kernel = ("bif_prefix_kernel<paged>" if tc else self.kernel) + \
            " (%d query tokens, %d-token blocks)" % (n, spec.page_size)

    def step(self, stream):
        sp = self.spec
        self.ta.tree_attn_decode_multi_paged_ex("bf16", self.dev["q"], self.dev["k"], self.dev["v"], self.num_pages,
                                                sp.page_size, self.table, self.stride, self.seqlens, sp.n_queries,
                                                sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.scale, self.out,
                                                self.lse, None, self.ws, stream=stream)


class BifurcatedRun:
    """Shared-prefix workload: one call = the tensor-core prefix pass and the suffix pass, which
    folds the prefix chunks' statistics into each row as it writes it (two launches per group of
    128 samples).  The roofline is the prefix pass's dense contraction on the tensor cores."""

    launches_per_step = 2
    metric, unit, bound = METRIC, UNIT, "tensor"
    inputs = None

    def __init__(self, spec, torch, ta, keep_inputs=False):
        self.spec, self.torch, self.ta = spec, torch, ta
        N, Hq, Hkv, D = spec.n_samples, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.lens = [int(s) for s in spec.suffix_lens]
        inp = synth.make_bifurcated_inputs(spec)
        names = ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix")
        self.host = {n: to_device_bf16(torch, inp[n]) for n in names}
        del inp
        self.dev = {n: t.cuda() for n, t in self.host.items()}
        self.out = torch.empty(N, Hq, D, device="cuda")
        self.lse = torch.empty(N, Hq, device="cuda")
        nbytes = ta.tree_attn_bifurcated_workspace_size(spec.prefix_len, self.lens, Hq, Hkv, D)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        self.kv_bytes = spec.kv_bytes
        self.tokens = spec.prefix_len + sum(self.lens)
        self.launches_per_step = 2 * ((N + 127) // 128)
        self.flops = 4 * D * N * Hq * spec.prefix_len  # the prefix pass: S = Q K^T and O = P V
        self.kernel = "bif_prefix_kernel (shared-prefix pass; the step adds the suffix pass and the merge)"

    def step(self, stream):
        sp, d = self.spec, self.dev
        self.ta.tree_attn_decode_bifurcated_ex(d["q"], d["k_prefix"], d["v_prefix"], sp.prefix_len, d["k_suffix"],
                                               d["v_suffix"], self.lens, sp.n_q_heads, sp.n_kv_heads, sp.head_dim,
                                               sp.scale, self.out, self.lse, None, self.ws, stream=stream)


class AnchorRun:
    """Context encoding with anchor blocks: one tensor-core launch per step."""

    launches_per_step = 1
    metric, unit, bound = ANCHOR_METRIC, "TFLOP/s", "tensor"
    inputs = None

    def __init__(self, spec, torch, ta, keep_inputs=False):
        self.spec, self.torch, self.ta = spec, torch, ta
        S, Hq, Hkv, D = spec.seq_len, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        inp = synth.make_anchor_inputs(spec)
        self.host = {n: to_device_bf16(torch, inp[n]) for n in ("q", "k", "v")}
        del inp
        self.dev = {n: t.cuda() for n, t in self.host.items()}
        self.out = torch.empty(S, Hq, D, device="cuda")
        self.lse = torch.empty(S, Hq, device="cuda")
        self.ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        self.kv_bytes = spec.kv_bytes
        self.tokens = S
        self.flops = spec.flops
        self.kernel = f"bif_prefix_kernel (context encoding, {128 // (Hq // Hkv)} positions x {Hq // Hkv} heads per tile)"

    def step(self, stream):
        sp, d = self.spec, self.dev
        self.ta.tree_attn_anchor_prefill(d["q"], d["k"], d["v"], sp.seq_len, sp.block_size, sp.n_q_heads,
                                         sp.n_kv_heads, sp.head_dim, sp.scale, self.out, self.lse, None, self.ws,
                                         stream=stream)


def make_run(spec, torch, ta, keep_inputs=False, decode_path=0):
    if isinstance(spec, synth.BifurcatedSpec):
        return BifurcatedRun(spec, torch, ta)
    if isinstance(spec, synth.AnchorSpec):
        return AnchorRun(spec, torch, ta)
    if spec.n_queries > 1 and spec.page_size > 0:
        return PagedMultiRun(spec, torch, ta, keep_inputs)
    if spec.n_queries > 1:
        return MultiRun(spec, torch, ta, keep_inputs)
    if spec.page_size > 0:
        return PagedRun(spec, torch, ta, keep_inputs)
    return DecodeRun(spec, torch, ta, keep_inputs, decode_path)


def run_gpu(args, spec) -> None:
    import torch

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    import exact_long_context_split_b200 as ta

    want_cpu = world == 1 and not args.no_cpu_baseline and isinstance(spec, synth.DecodeSpec) and \
        spec.n_queries == 1 and spec.page_size == 0
    run = make_run(spec, torch, ta, keep_inputs=want_cpu, decode_path=DECODE_PATHS[args.decode_path])
    stream = torch.cuda.current_stream()
    small = spec.kv_bytes <= 2 * 126e6
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda") if small else None

    for _ in range(args.warmup):
        run.step(stream)
    torch.cuda.synchronize()
    assert ta.tree_attn_check(run.ws) == ta.TA_OK

    def events(n):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in ev:  # torch creates the CUDA event on its first record
            e.record(stream)
        return ev

    starts, ends = events(args.steps), events(args.steps)
    kstarts, kends = events(args.steps), events(args.steps)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        clocks.start()
        # The step time comes from steps with no library events inside them (an event between
        # two of the step's launches would serialise a launch meant to overlap its predecessor);
        # the main kernel's time from steps interleaved with them, with the library's events
        # around that kernel.
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)  # L2 flush outside the step's events
            starts[i].record(stream)
            run.step(stream)
            ends[i].record(stream)
            if flush is not None:
                flush.fill_((i + 128) & 0xFF)
            ta.tree_attn_profile_events(kstarts[i], kends[i])
            run.step(stream)
            ta.tree_attn_profile_events()
        torch.cuda.synchronize()
        clocks.stop()
        barrier(world)
    status = ta.tree_attn_check(run.ws)
    if status != ta.TA_OK:
        raise RuntimeError(ta.tree_attn_status_string(status))
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kernel_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(kstarts, kends))
    ms_per_step = max_over_ranks(statistics.mean(step_ms), world)
    elapsed_s = ms_per_step * 1e-3 * args.steps
    if run.unit == "TFLOP/s":
        value = world * run.flops / (ms_per_step * 1e-3) / 1e12
    else:
        value = world * run.kv_bytes / (ms_per_step * 1e-3) / 1e9

    # End to end through the public API: pinned host -> device copies of every input, the
    # call, and the device -> host read of out and lse, every step.
    e2e_steps = max(1, min(args.steps, 5))
    out_h = torch.empty(run.out.shape).pin_memory()
    lse_h = torch.empty(run.lse.shape).pin_memory()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for n in run.host:
            run.dev[n].copy_(run.host[n], non_blocking=True)
        run.step(stream)
        out_h.copy_(run.out, non_blocking=True)
        lse_h.copy_(run.lse, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for t in run.host.values())
    d2h = out_h.numel() * 4 + lse_h.numel() * 4
    e2e_value = world * (run.flops / 1e12 if run.unit == "TFLOP/s" else run.kv_bytes / 1e9) / (e2e_ms * 1e-3)

    hbm, bf16, peak_kind = measured_peaks()
    if run.bound == "tensor":
        achieved = run.flops / (kernel_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s", "frac": achieved / bf16,
                "peak_kind": peak_kind + " dense bf16 (burst)", "flops_per_launch": run.flops}
    else:
        achieved = run.kv_bytes / (kernel_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_kind": peak_kind + " copy bandwidth", "bytes_per_launch": run.kv_bytes}
    roof.update({"kernel": run.kernel, "kernel_us": kernel_ms * 1e3,
                 "traffic": traffic_per_launch(spec, run.family) if type(run) is DecodeRun else None})
    extra = {
        "us_per_step": ms_per_step * 1e3,
        "kv_tokens_per_s": world * run.tokens * args.steps / elapsed_s,
        "hbm_frac_of_" + peak_kind: world * run.kv_bytes / (ms_per_step * 1e-3) / 1e9 / world / hbm,
        "e2e": {"value": e2e_value, "unit": run.unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * run.launches_per_step,
        "roofline": roof,
        "clocks": clocks.summary(),
        "build_id": ta.tree_attn_build_id(),
    }
    if isinstance(run, (BifurcatedRun, AnchorRun)):
        extra["step_tflops"] = run.flops / (ms_per_step * 1e-3) / 1e12
    if isinstance(run, BifurcatedRun):
        extra["logical_kv_tokens_per_s"] = world * spec.n_samples * (spec.prefix_len + statistics.mean(run.lens)) * \
            args.steps / elapsed_s
    if want_cpu:
        extra["cpu_baseline"] = cpu_baseline(spec, run.inputs)
    rec = make_record(metric=run.metric, unit=run.unit, value=value, n_gpus=world, steps=args.steps,
                      warmup=args.warmup, ms_per_step=ms_per_step, spec=spec, dtype="bf16", extra=extra)
    if args.decode_path != "auto":
        rec["config"]["decode_path"] = args.decode_path
    if rank == 0:
        print(json.dumps(rec), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


DECODE_PATHS = {"auto": 0, "tensor": 1, "split": 2}


def all_workloads():
    return {**synth.decode_configs(), **synth.gqa8_configs(), **synth.capture_configs(),
            **synth.bifurcated_configs(), **synth.multi_query_configs(), **synth.paged_configs(),
            **synth.anchor_configs()}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    workloads = all_workloads()
    ap.add_argument("--workload", default="long_1m", choices=sorted(workloads))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-path", default="auto", choices=sorted(DECODE_PATHS),
                    help="plain decode workloads: the library's choice, or force the tensor-core or split kernel")
    args = ap.parse_args(argv)
    spec = workloads[args.workload]
    if args.impl == "reference":
        if not isinstance(spec, synth.DecodeSpec) or spec.n_queries != 1 or spec.page_size:
            raise SystemExit("the reference arm times the single-query decode workloads")
        run_reference(args, spec)
    else:
        run_gpu(args, spec)


if __name__ == "__main__":
    main()
