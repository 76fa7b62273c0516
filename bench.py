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
over ranks.  `--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
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
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["exact_long_context_split_b200/csrc/split_kv.cuh", "exact_long_context_split_b200/csrc/ptx.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "split_kv_traffic.json")


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


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_per_launch(spec) -> object:
    """DRAM bytes (read + write) of one launch from the committed ncu capture: the mean of the
    captured launches for the captured workload, reads scaled by K/V bytes for another one.
    None when the kernel sources changed since the counters were taken."""
    try:
        with open(TRAFFIC_FILE) as fh:
            d = json.load(fh)
    except Exception:
        return None
    if d.get("kernel_hash") != kernel_hash():
        return None
    rd = statistics.mean(d["dram_bytes_read"])
    wr = statistics.mean(d["dram_bytes_write"])
    if spec.name != d["workload"]:
        rd *= spec.kv_bytes / d["kv_bytes"]
    return int(round(rd + wr))


class ClockSampler:
    """SM clock and clock-event (throttle) reasons read through NVML every 2 ms by a host
    thread while the timed region runs (a step here lasts under a millisecond, far below
    nvidia-smi's 200 ms sampling).  Only reads device state."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.idx = torch_device_index
        self.period = period_s
        self.samples = []
        self.window = [None, None]
        self.err = None
        self._stop = False
        self._thread = None
        self._first = None  # set once the first sample (or an NVML error) exists

    def _handle(self, nv):
        import torch

        try:
            pr = torch.cuda.get_device_properties(self.idx)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.idx)

    def _run(self):
        import threading  # noqa: F401

        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            while not self._stop:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     int(get_reasons(h))))
                self._first.set()
                time.sleep(self.period)
            nv.nvmlShutdown()
        except Exception as e:  # NVML missing or refused: report it, never fail the bench
            self.err = f"nvml: {e}"
            self._first.set()

    def __enter__(self):
        import threading

        self._first = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        # NVML's first initialisation can take longer than a short timed region: start timing
        # only once the sampler is producing samples (bounded).
        self._first.wait(timeout=10.0)
        return self

    def start(self):
        self.window[0] = time.perf_counter()

    def stop(self):
        self.window[1] = time.perf_counter()

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if self.err or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"]}
        t0, t1 = self.window
        inside = [s for s in self.samples if t0 is not None and t1 is not None and t0 <= s[0] <= t1] or self.samples
        reasons = sorted({name for _, _, r in inside for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside), "source": "nvml, 2 ms"}


def make_record(*, value, n_gpus, steps, warmup, ms_per_step, spec, dtype, extra) -> dict:
    rec = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": n_gpus,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic",
        "config": {
            "workload": spec.name,
            **({"batch": spec.batch, "seq_len": int(max(spec.seqlens)) if spec.seqlens else 0,
                "query_tokens": spec.n_queries, **({"page_size": spec.page_size} if spec.page_size else {})}
               if isinstance(spec, synth.DecodeSpec) else
               {"samples": spec.n_samples, "prefix_len": spec.prefix_len,
                "suffix_len": int(max(spec.suffix_lens)) if spec.suffix_lens else 0}),
            "n_q_heads": spec.n_q_heads,
            "n_kv_heads": spec.n_kv_heads,
            "head_dim": spec.head_dim,
            "kv_bytes_per_step": spec.kv_bytes,
            "parallelism": f"replicas{n_gpus}",
            "l2": "no flush: each step reads %.2f GB of K/V, more than the 126 MB L2" % (spec.kv_bytes / 1e9),
        },
    }
    rec.update(extra)
    return rec


def oracle_sample_seconds(spec, h_kv: int, q_heads, n_tokens: int = 0) -> float:
    """Time the CPU oracle on the given query heads of KV head h_kv of sequence 0, over its first
    n_tokens tokens (0 = all).  Inputs are generated for that head only (the same bytes as the
    full workload's); only the oracle is timed."""
    import oracle

    S, D, Hq = spec.seqlens[0], spec.head_dim, spec.n_q_heads
    n = S * D
    k = synth.normal_bf16(spec.seed, synth.TID_K, n, start=h_kv * n)
    v = synth.normal_bf16(spec.seed, synth.TID_V, n, start=h_kv * n)
    if spec.spike_frac > 0:
        synth.spike_rows_bf16(k.reshape(S, D), spec.seed, h_kv, spec.n_spikes(S), spec.spike_factor)
    q = synth.normal_bf16(spec.seed, synth.TID_Q, Hq * D).reshape(Hq, D)
    T = n_tokens or S
    K, V = k.reshape(S, D)[:T], v.reshape(S, D)[:T]
    t0 = time.perf_counter()
    for h in q_heads:
        oracle.attention_one_bf16_cache(oracle.bf16_to_f64(q[h]), K, V, spec.scale)
    return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return 1


# ----------------------------------------------------------------------------------------------
# Reference arm: the CPU oracle
# ----------------------------------------------------------------------------------------------


REF_SLICE = 8  # the reference arm's per-step sample covers 1/REF_SLICE of the sequence


def run_reference(args, spec) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    G = spec.n_q_heads // spec.n_kv_heads
    rows = spec.batch * spec.n_q_heads
    T = spec.seqlens[0] // REF_SLICE
    for _ in range(args.warmup):
        oracle_sample_seconds(spec, 0, [0], T)
    times = [oracle_sample_seconds(spec, i % spec.n_kv_heads, [(i % spec.n_kv_heads) * G], T) for i in range(args.steps)]
    step_s = statistics.mean(times) * REF_SLICE * rows
    value = spec.kv_bytes / step_s / 1e9
    cores = blas_threads()
    sample = (f"each step: one (sequence, query head) row over the first {T} of {spec.seqlens[0]} tokens "
              f"(KV head cycling 0..{spec.n_kv_heads - 1}); step time = mean sample time x {REF_SLICE} x {rows} rows")
    rec = make_record(value=value, n_gpus=world, steps=args.steps, warmup=args.warmup, ms_per_step=step_s * 1e3,
                      spec=spec, dtype="f64", extra={
                          "impl": "reference",
                          "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                                           "sample": sample},
                          "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                          "gpu_launches": 0,
                      })
    print(json.dumps(rec), flush=True)


# ----------------------------------------------------------------------------------------------
# The CUDA path
# ----------------------------------------------------------------------------------------------


class DecodeRun:
    """Device and pinned-host buffers of one decode workload and its step (one kernel launch)."""

    launches_per_step = 1

    def __init__(self, spec, torch, ta):
        self.spec, self.torch, self.ta = spec, torch, ta
        B, Hq, Hkv, D = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.seqlens = [int(s) for s in spec.seqlens]
        inp = synth.make_decode_inputs(spec)
        self.host = {n: torch.from_numpy(inp[n].reshape(-1).view(np.int16)).view(torch.bfloat16).pin_memory()
                     for n in ("q", "k", "v")}
        del inp
        self.dev = {n: t.cuda() for n, t in self.host.items()}
        self.out = torch.empty(B, Hq, D, device="cuda")
        self.lse = torch.empty(B, Hq, device="cuda")
        self.ws = torch.empty(ta.tree_attn_workspace_size(self.seqlens, Hq, Hkv, D), dtype=torch.uint8, device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        self.kv_bytes = spec.kv_bytes
        self.tokens = spec.tokens
        self.kernel = f"split_kv_decode_kernel<bf16,{D},{Hq // Hkv},{'ShortTiles' if sum(self.seqlens) < 1024 * len(self.seqlens) else 'LongTiles'}>"

    def step(self, stream):
        sp = self.spec
        self.ta.tree_attn_decode_ex("bf16", self.dev["q"], self.dev["k"], self.dev["v"], self.seqlens, sp.n_q_heads,
                                    sp.n_kv_heads, sp.head_dim, sp.scale, self.out, self.lse, None, self.ws,
                                    stream=stream)


class MultiRun(DecodeRun):
    """Several query tokens per sequence: one call = the tensor-core form (bf16, D = 128,
    8 <= G n <= 128) or ceil(n G / 8) split-KV passes."""

    def __init__(self, spec, torch, ta):
        super().__init__(spec, torch, ta)
        B, n, Hq, Hkv, D = spec.batch, spec.n_queries, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.out = torch.empty(B, n, Hq, D, device="cuda")
        self.lse = torch.empty(B, n, Hq, device="cuda")
        self.ws = torch.empty(ta.tree_attn_multi_workspace_size(self.seqlens, n, Hq, Hkv, D), dtype=torch.uint8,
                              device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        G = Hq // Hkv
        if D == 128 and 8 <= G * n <= 128:
            # tensor-core form (the library's automatic choice for bf16): per group of up to 128
            # sequences one bif_prefix_kernel launch and one merge_chunks_kernel launch
            groups = (B + 127) // 128
            self.launches_per_step = 2 * groups
            self.kernel = f"bif_prefix_kernel (several query tokens, {G * n} rows per KV head) + merge_chunks_kernel"
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

    def __init__(self, spec, torch, ta):
        super().__init__(spec, torch, ta)
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

    def __init__(self, spec, torch, ta):
        super().__init__(spec, torch, ta)
        B, n, Hq, Hkv, D = spec.batch, spec.n_queries, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.out = torch.empty(B, n, Hq, D, device="cuda")
        self.lse = torch.empty(B, n, Hq, device="cuda")
        self.ws = torch.empty(ta.tree_attn_multi_workspace_size(self.seqlens, n, Hq, Hkv, D), dtype=torch.uint8,
                              device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        tc = D == 128 and 8 <= (Hq // Hkv) * n <= 128
        self.launches_per_step = 2 * ((B + 127) // 128) if tc else self.launches_per_step
        self.kernel = ("bif_prefix_kernel<paged> + merge_chunks_kernel" if tc else self.kernel) + \
            " (%d query tokens, %d-token blocks)" % (n, spec.page_size)

    def step(self, stream):
        sp = self.spec
        self.ta.tree_attn_decode_multi_paged_ex("bf16", self.dev["q"], self.dev["k"], self.dev["v"], self.num_pages,
                                                sp.page_size, self.table, self.stride, self.seqlens, sp.n_queries,
                                                sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.scale, self.out,
                                                self.lse, None, self.ws, stream=stream)


class BifurcatedRun:
    """Shared-prefix workload: one call = prefix pass, suffix pass and the exact merge."""

    launches_per_step = 3

    def __init__(self, spec, torch, ta):
        self.spec, self.torch, self.ta = spec, torch, ta
        N, Hq, Hkv, D = spec.n_samples, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
        self.lens = [int(s) for s in spec.suffix_lens]
        inp = synth.make_bifurcated_inputs(spec)
        names = ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix")
        self.host = {n: torch.from_numpy(inp[n].reshape(-1).view(np.int16)).view(torch.bfloat16).pin_memory()
                     for n in names}
        del inp
        self.dev = {n: t.cuda() for n, t in self.host.items()}
        self.out = torch.empty(N, Hq, D, device="cuda")
        self.lse = torch.empty(N, Hq, device="cuda")
        nbytes = ta.tree_attn_bifurcated_workspace_size(spec.prefix_len, self.lens, Hq, Hkv, D)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        ta.tree_attn_workspace_init(self.ws)
        self.kv_bytes = spec.kv_bytes
        self.tokens = spec.prefix_len + sum(self.lens)
        self.kernel = "bifurcated step (prefix pass + suffix pass + merge)"

    def step(self, stream):
        sp, d = self.spec, self.dev
        self.ta.tree_attn_decode_bifurcated_ex(d["q"], d["k_prefix"], d["v_prefix"], sp.prefix_len, d["k_suffix"],
                                               d["v_suffix"], self.lens, sp.n_q_heads, sp.n_kv_heads, sp.head_dim,
                                               sp.scale, self.out, self.lse, None, self.ws, stream=stream)


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

    if isinstance(spec, synth.BifurcatedSpec):
        run = BifurcatedRun(spec, torch, ta)
    elif spec.n_queries > 1 and spec.page_size > 0:
        run = PagedMultiRun(spec, torch, ta)
    elif spec.n_queries > 1:
        run = MultiRun(spec, torch, ta)
    elif spec.page_size > 0:
        run = PagedRun(spec, torch, ta)
    else:
        run = DecodeRun(spec, torch, ta)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        run.step(stream)
    torch.cuda.synchronize()
    assert ta.tree_attn_check(run.ws) == ta.TA_OK

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        clocks.start()
        t_begin.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            run.step(stream)
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        clocks.stop()
        barrier(world)
    status = ta.tree_attn_check(run.ws)
    if status != ta.TA_OK:
        raise RuntimeError(ta.tree_attn_status_string(status))
    elapsed_ms = max_over_ranks(t_begin.elapsed_time(t_end), world)
    kernel_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms_per_step = elapsed_ms / args.steps
    value = world * run.kv_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9

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

    peak, peak_kind = measured_peaks()
    achieved = run.kv_bytes / (kernel_ms * 1e-3) / 1e9
    extra = {
        "ms_per_step": ms_per_step,
        "us_per_step": ms_per_step * 1e3,
        "kv_tokens_per_s": world * run.tokens * args.steps / (elapsed_ms * 1e-3),
        "hbm_frac_of_" + peak_kind: value / world / peak,
        "e2e": {"value": world * run.kv_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * run.launches_per_step,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "kernel": run.kernel,
                     "traffic": traffic_per_launch(spec) if type(run) is DecodeRun else None},
        "clocks": clocks.summary(),
    }
    if isinstance(run, BifurcatedRun):
        extra["logical_kv_tokens_per_s"] = world * spec.n_samples * (spec.prefix_len + statistics.mean(run.lens)) * \
            args.steps / (elapsed_ms * 1e-3)
    if world == 1 and not args.no_cpu_baseline and type(run) is DecodeRun:
        G = spec.n_q_heads // spec.n_kv_heads
        sec = oracle_sample_seconds(spec, 0, list(range(G)))
        rows = spec.batch * spec.n_q_heads
        cpu_val = spec.kv_bytes / (sec / G * rows) / 1e9
        extra["cpu_baseline"] = {"value": cpu_val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"the {G} query heads of KV head 0 over all {spec.seqlens[0]} tokens took "
                                           f"{sec:.2f} s; step time = that / {G} x {rows} rows"}
    rec = make_record(value=value, n_gpus=world, steps=args.steps, warmup=args.warmup, ms_per_step=ms_per_step,
                      spec=spec, dtype="bf16", extra=extra)
    if rank == 0:
        print(json.dumps(rec), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    workloads = {**synth.decode_configs(), **synth.capture_configs(), **synth.bifurcated_configs(),
                 **synth.multi_query_configs(), **synth.paged_configs()}
    ap.add_argument("--workload", default="long_1m", choices=sorted(workloads))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    spec = workloads[args.workload]
    if args.impl == "reference":
        if isinstance(spec, synth.BifurcatedSpec):
            raise SystemExit("the reference arm times the decode workloads")
        run_reference(args, spec)
    else:
        run_gpu(args, spec)


if __name__ == "__main__":
    main()
