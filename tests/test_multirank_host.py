"""The N>1 plumbing of bench.py, run as world-size-2 gloo ranks on the CPU.

The attention path has no exchange step, so N ranks run N independent replicas; what must hold
across ranks is the rendezvous, the max-over-ranks timing, the whole-job aggregation (units of
all ranks over the slowest rank's time) and that only rank 0 runs and prints the oracle arm.
"""
import io
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        args = types.SimpleNamespace(impl="reference", gpus=world, steps=1, warmup=0)
        w, r, local = bench.dist_setup(args)
        assert (w, r, local) == (world, rank, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(w)
        m = bench.dist_max(10.0 * rank + 1.0, w)          # per-rank "milliseconds"
        agg = bench.aggregate_throughput(3.0e9, w, m)      # units per rank, slowest rank's ms
        out = ""
        if rank != 0:
            buf = io.StringIO()
            with redirect_stdout(buf):
                rc = bench.run_reference(args, w, r)      # must return at once, silently
            assert rc == 0
            out = buf.getvalue()
        bench.barrier(w)
        q.put((rank, m, agg, out))
    except BaseException as e:                             # reported to the parent
        q.put((rank, "error", repr(e), ""))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_aggregate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, m, agg, out in res:
        assert m != "error", agg
        assert m == 11.0                                   # max over ranks of {1, 11}
        assert abs(agg - 2 * 3.0e9 / 11.0e-3) <= 1e-6 * agg
        assert out == ""                                   # rank 1 printed nothing


def test_aggregate_is_units_of_all_ranks_over_slowest_time():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_throughput(5.0, 1, 1000.0) == 5.0
    assert bench.aggregate_throughput(5.0, 4, 2000.0) == 10.0


def test_reference_arm_line_has_the_contract_keys(monkeypatch, capsys):
    """Rank 0 of `bench.py --impl reference` prints one JSON line with the bench keys, the
    oracle's cpu_baseline and an e2e object with no host-device traffic (a tiny sample here)."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    import torch
    from mea_workloads import alibi_slope_values, make_qkv

    def tiny(_target):
        q, k, v = make_qkv([40, 24], [40, 24], 32, 8, 128, torch.bfloat16, 7)
        return (q, k, v, [40, 24], alibi_slope_values(32).double(), 0.088), \
            bench.fwd_flops([40, 24], 32, 128), "tiny sample"
    monkeypatch.setattr(bench, "oracle_sample", tiny)
    args = types.SimpleNamespace(impl="reference", gpus=1, steps=2, warmup=1,
                                 decode_requests=64)
    assert bench.run_reference(args, 1, 0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["config"] == bench.step_config(args, 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
