"""The bench's multi-rank host logic on CPU: two gloo ranks take the same collective steps,
the timed value is the max over ranks, and only rank 0 prints (replicas: no data-path
collective)."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import bench

    assert bench.dist_env() == (rank, world, rank)
    bench.barrier(world)
    got = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    bench.barrier(world)
    q.put((rank, got))
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_reference_arm_rank1_prints_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_record_fields():
    sys.path.insert(0, ROOT)
    import bench
    import synth

    spec = synth.decode_configs()["long_1m"]
    rec = bench.make_record(metric=bench.METRIC, unit=bench.UNIT, value=1.0, n_gpus=2, steps=3, warmup=3,
                            ms_per_step=0.5, spec=spec, dtype="bf16", extra={"gpu_launches": 3})
    for key in ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "gpu_launches"]:
        assert key in rec
    assert rec["scaling"] == "weak" and rec["config"]["workload"] == "long_1m"
    json.dumps(rec)


def test_record_config_of_every_workload():
    sys.path.insert(0, ROOT)
    import bench

    for name, spec in bench.all_workloads().items():
        cfg = bench.workload_config(spec, 1)
        assert cfg["workload"] == name and cfg["kv_bytes_per_step"] == spec.kv_bytes
        assert ("no flush" in cfg["l2"]) == (spec.kv_bytes > 2 * 126e6)


def test_reference_arm_runs_full_steps_on_the_host():
    """The reference arm times the oracle on every row of each step, threaded over rows."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    assert r.returncode == 0, r.stderr
    rec = json.loads(r.stdout.strip().splitlines()[-1])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["gpu_launches"] == 0
    assert "all 1 (sequence, query head) rows" in rec["cpu_baseline"]["sample"]
    assert rec["cpu_baseline"]["cores"] == 1 and rec["cpu_baseline"]["host_cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_capture_follows_its_kernel_family(monkeypatch):
    """A committed DRAM-traffic capture is attached only to the kernel family it was taken on,
    scaled by K/V bytes for another workload of that family, and dropped once its kernel's
    sources differ from the ones it was taken from."""
    import bench

    recorded = {}
    for fam, (name, _) in bench.TRAFFIC.items():
        with open(os.path.join(ROOT, "profiles", name)) as fh:
            recorded[fam] = json.load(fh)["kernel_hash"]
    # Sources as they were when each capture was taken: the captures count.
    hashes = {tuple(src): recorded[fam] for fam, (_, src) in bench.TRAFFIC.items()}
    monkeypatch.setattr(bench, "kernel_hash", lambda sources: hashes[tuple(sources)])
    specs = bench.all_workloads()
    split = bench.traffic_per_launch(specs["long_1m"], "split")
    tc = bench.traffic_per_launch(specs["long_1m_g8"], "tc_decode")
    assert isinstance(split, int) and isinstance(tc, int)
    kv = specs["long_1m"].kv_bytes
    assert kv <= split <= 1.01 * kv and kv <= tc <= 1.01 * kv
    quarter = bench.traffic_per_launch(specs["long_256k"], "split")
    assert abs(quarter - split / 4) < 0.01 * split  # reads scale with the K/V bytes
    assert bench.traffic_per_launch(specs["long_1m"], "paged") is None
    # Sources changed since: no traffic figure.
    monkeypatch.setattr(bench, "kernel_hash", lambda sources: "0" * 16)
    assert bench.traffic_per_launch(specs["long_1m"], "split") is None


def test_clock_sampler_edges_without_nvml():
    """Without NVML the sampler reports why, and the bench still gets a summary."""
    sys.path.insert(0, ROOT)
    import bench

    c = bench.ClockSampler(0)
    c.err = "nvml: not available"
    c.start()
    c.stop()
    assert c.summary()["reasons"] == ["nvml: not available"] and c.summary()["samples"] == 0
    c = bench.ClockSampler(0)
    c.max_mhz = 1965
    c.samples = [(1.0, 1965, 0), (2.0, 1800, 0x4), (3.5, 1965, 0)]
    c.window = [1.0005, 3.4995]
    s = c.summary()
    assert s["samples"] == 3 and s["reasons"] == ["sw_power_cap"] and s["sm_mhz"] == 1965


def _sharded_rank(rank, world, port, q):
    """One CPU rank of the sharded decode: the oracle stands in for the GPU decode and merge
    (test infrastructure), so what runs here is the library's sharding plan and exchange."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import oracle
    import synth
    from exact_long_context_split_b200.sharded import decode_sharded, shard_bounds

    sp = synth.DecodeSpec("sharded", [37, 5, 1, 300], 8, 2, 16, dtype="f32", seed=12)
    inp = synth.make_decode_inputs(sp)
    Hkv, D = 2, 16
    shard_lens, ks, vs, off = [], [], [], 0
    for S in sp.seqlens:
        t0, t1 = shard_bounds(S, world, rank)
        shard_lens.append(t1 - t0)
        ks.append(inp["k"][off:off + Hkv * S * D].reshape(Hkv, S, D)[:, t0:t1].reshape(-1))
        vs.append(inp["v"][off:off + Hkv * S * D].reshape(Hkv, S, D)[:, t0:t1].reshape(-1))
        off += Hkv * S * D

    def decode(dtype, qq, k, v, lens, Hq, Hkv_, D_, scale, out, lse):
        o, l = oracle.decode_attention(qq, k, v, lens, Hq, Hkv_, D_, scale, dtype=dtype)
        out.copy_(torch.from_numpy(o.reshape(-1)))
        lse.copy_(torch.from_numpy(l.reshape(-1)))

    def merge(outs, lses, n, rows, D_, out, lse):
        o = outs.numpy().reshape(n, rows, D_)
        l = lses.numpy().reshape(n, rows)
        res = [oracle.merge_shard_results(o[:, r], l[:, r]) for r in range(rows)]
        out.view(-1).copy_(torch.from_numpy(np.stack([x[0] for x in res]).reshape(-1)))
        lse.view(-1).copy_(torch.tensor([x[1] for x in res], dtype=torch.float64))

    out = torch.empty(sp.batch, 8, D)
    lse = torch.empty(sp.batch, 8)
    decode_sharded(inp["q"], np.concatenate(ks), np.concatenate(vs), shard_lens, 8, Hkv, D, sp.scale, out, lse,
                   dtype="f32", decode=decode, merge=merge)
    ref_out, ref_lse = oracle.decode_attention(inp["q"], inp["k"], inp["v"], sp.seqlens, 8, Hkv, D, sp.scale,
                                               dtype="f32")
    err = float(np.max(np.abs(out.numpy() - ref_out)))
    lerr = float(np.max(np.abs(lse.numpy() - ref_lse)))
    q.put((rank, err, lerr, shard_lens))
    dist.destroy_process_group()


def test_sharded_decode_exchange_gloo():
    """Two and three CPU ranks, each holding a contiguous slice of every sequence (one sequence
    shorter than the rank count), exchange and merge to the unsharded result."""
    for world in (2, 3):
        ctx = mp.get_context("spawn")
        q = ctx.Queue()
        port = _free_port()
        procs = [ctx.Process(target=_sharded_rank, args=(r, world, port, q)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = sorted(q.get(timeout=5) for _ in range(world))
        assert sum(r[3][2] for r in res) == 1  # the 1-token sequence lives on one rank only
        for rank, err, lerr, _ in res:
            assert err < 1e-5 and lerr < 1e-5, (world, rank, err, lerr)
