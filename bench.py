"""Benchmark: packed causal GQA + ALiBi prefill (attention fwd TFLOP/s) and split-KV decode
(decode KV GB/s) on B200, through the C ABI.

One step = one forward over the packed-causal workload (bf16, 32/8 heads, D=128, 32768 tokens in
segments drawn U[64, 4096]) followed by one split-KV decode over the decode workload (64 requests
x 1 token, KV lengths U[512, 32768], 64/8 heads, D=128). ``value`` is the forward's useful
TFLOP/s (4*Lq*Lk*D per head per segment, causal counted as half); the decode's GB/s (K+V bytes
read once, plus q and out) is in ``decode``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--part all|fwd|decode] [--no-e2e] [--no-cpu-baseline]

Multi-GPU: the path has no exchange step, so N ranks run N independent replicas (one per GPU,
``scaling: weak``); timings are the max over ranks.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (packed causal GQA+ALiBi) and decode KV GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--part", default="all",
                    choices=["all", "fwd", "decode", "bwd", "long", "d256"],
                    help="all = the timed step (forward + decode) plus the backward measured "
                         "on its own; bwd = the backward alone; long / d256 = the "
                         "16384-token prefill at head dim 128 / 256 alone (for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-paged", dest="paged", action="store_false",
                    help="skip the paged-cache decode measurement")
    ap.add_argument("--no-fp8", dest="fp8", action="store_false",
                    help="skip the FP8 forward measurement")
    ap.add_argument("--no-long", dest="long", action="store_false",
                    help="skip the long-context (16384-token) prefill measurement")
    ap.add_argument("--no-d256", dest="d256", action="store_false",
                    help="skip the head-dim-256 long prefill measurement")
    ap.add_argument("--paged-block-size", type=int, default=16,
                    help="slots per cache block of the paged decode measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--decode-requests", type=int, default=64,
                    help="use only the first N requests of the decode workload (profiling)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "memory_efficient_attention_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ workload accounting
def fwd_flops(seqlens, hq, d):
    # causal counted as half of 4*L*L*D per head
    return sum(2.0 * L * L * d * hq for L in seqlens)


def decode_bytes(kv_lens, hkv, d, n_req, hq, elem=2):
    kv = sum(kv_lens) * hkv * d * elem * 2
    return kv + 2 * n_req * hq * d * elem


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.dev = device_index

    def start(self):
        try:
            import torch
            uuid = None
            try:
                uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
            except Exception:
                pass
            self.path = os.path.join("/tmp", f"mea_clocks_{os.getpid()}.csv")
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            cmd = ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                   "-lms", "100", "-i", uuid if uuid else str(self.dev)]
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, p in zip(names, parts[5:9]):
                    if p.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def _collective_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def dist_max(x: float, world: int) -> float:
    """The maximum of x over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_collective_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    """All ranks meet, then this rank's device is drained."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def aggregate_throughput(units_per_rank: float, world: int, ms_max_over_ranks: float) -> float:
    """Whole-job throughput of independent replicas: the units all ranks processed divided by
    the slowest rank's time (units per second)."""
    return world * units_per_rank / (ms_max_over_ranks * 1e-3)


def step_config(args, world):
    """The `config` of the timed step (shared by both arms)."""
    from mea_workloads import workload
    w2, w4 = workload(2), workload(4)
    return {"workload": ("packed causal GQA+ALiBi prefill (bf16, 32 q / 8 kv heads, D=128, "
                         f"{w2.total_q} tokens in {len(w2.seqlens_q)} segments U[64,4096]) + "
                         "split-KV decode (bf16, 64 requests x 1 token, KV U[512,32768], "
                         "64 q / 8 kv heads, D=128)"),
            "prefill_seqlens": w2.seqlens_q,
            "decode_total_kv_tokens": sum(w4.seqlens_k[:max(1, args.decode_requests)]),
            "l2": "inputs larger than L2 (q 268 MB; K+V 4.3 GB), no flush",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample(target_flops: float):
    """Leading segments of the packed workload (all 32 heads) until the useful FLOPs reach the
    target; returns (inputs, flops, description)."""
    import torch
    from mea_workloads import alibi_slope_values, make_qkv, workload
    w = workload(2)
    segs, fl = [], 0.0
    for L in w.seqlens_q:
        segs.append(L)
        fl += fwd_flops([L], 32, 128)
        if fl >= target_flops:
            break
    q, k, v = make_qkv(segs, segs, 32, 8, 128, torch.bfloat16, w.seed)
    desc = (f"oracle (float64, torch CPU) on the first {len(segs)} segments {segs} of the "
            f"packed workload, all 32 heads, causal + ALiBi")
    return (q, k, v, segs, alibi_slope_values(32).double(), w.scale), fl, desc


def time_oracle(sample):
    import torch
    import oracle
    from mea_workloads import cu_seqlens
    q, k, v, segs, slopes, scale = sample
    cu = cu_seqlens(segs).tolist()
    t0 = time.perf_counter()
    oracle.attention(q, k, v, cu, cu, scale, True, slopes)
    return time.perf_counter() - t0


def cpu_cores():
    import torch
    return torch.get_num_threads()


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    sample, fl, desc = oracle_sample(4.0e10)
    for _ in range(args.warmup):
        time_oracle(sample)
    tot = 0.0
    for _ in range(args.steps):
        tot += time_oracle(sample)
    val = fl * args.steps / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": step_config(args, world),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    import torch
    import memory_efficient_attention_b200 as mea
    from mea_workloads import alibi_slope_values, cu_seqlens, workload

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    pk, peak_src = peaks()
    do_fwd = args.part in ("all", "fwd")
    do_dec = args.part in ("all", "decode")
    do_bwd = args.part in ("all", "bwd")
    do_long = args.part == "long" or (do_fwd and args.long)
    do_d256 = args.part == "d256" or (do_fwd and args.d256)

    w2, w4 = workload(2), workload(4)
    g = torch.Generator(device=dev)
    # ---- forward inputs (packed causal GQA + ALiBi)
    if do_fwd or do_bwd:
        g.manual_seed(w2.seed)
        tq = w2.total_q
        q = torch.randn((tq, 32, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        k = torch.randn((tq, 8, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        v = torch.randn((tq, 8, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        cu = cu_seqlens(w2.seqlens_q).to(dev)
        slopes = alibi_slope_values(32).to(dev)
        out = torch.empty_like(q)
        lse = torch.empty((32, tq), dtype=torch.float32, device=dev)
        max_q = max(w2.seqlens_q)
        flops = fwd_flops(w2.seqlens_q, 32, 128)

        def fwd():
            mea.attention_packed(q, k, v, cu, cu, max_q, causal=True, alibi_slopes=slopes,
                                 scale=w2.scale, out=out, lse=lse)
    # ---- decode inputs
    if do_dec:
        g.manual_seed(w4.seed)
        lk = w4.seqlens_k[:max(1, args.decode_requests)]
        tk = sum(lk)
        n_req = len(lk)
        dq = torch.randn((n_req, 64, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        dk = torch.empty((tk, 8, 128), dtype=torch.bfloat16, device=dev)
        dv = torch.empty((tk, 8, 128), dtype=torch.bfloat16, device=dev)
        for buf in (dk, dv):  # fill in slices to bound the fp32 temporary
            step = 1 << 17
            for i in range(0, tk, step):
                n = min(step, tk - i)
                buf[i:i + n] = torch.randn((n, 8, 128), generator=g, device=dev).bfloat16()
        dcu = cu_seqlens(lk).to(dev)
        dout = torch.empty_like(dq)
        dlse = torch.empty((64, n_req), dtype=torch.float32, device=dev)
        ws = torch.empty(mea.decode_workspace_size(n_req, tk, 64, 8, 128, 0), dtype=torch.uint8,
                         device=dev)
        dbytes = decode_bytes(lk, 8, 128, n_req, 64)
        max_k = max(lk)

        def dec():
            mea.decode_splitkv(dq, dk, dv, dcu, max_k, scale=w4.scale, workspace=ws, out=dout,
                               lse=dlse)

        # The same keys/values in a paged cache of 16-slot blocks (blocks in a shuffled order).
        pbs = args.paged_block_size
        nblk = [-(-x // pbs) for x in lk]
        pperm = torch.randperm(sum(nblk), generator=g, device=dev).to(torch.int32)
        ptable = torch.zeros((n_req, max(nblk)), dtype=torch.int32, device=dev)
        pkc = torch.zeros((sum(nblk), pbs, 8, 128), dtype=torch.bfloat16, device=dev)
        pvc = torch.zeros_like(pkc)
        nxt, off = 0, 0
        for b, length in enumerate(lk):
            ids = pperm[nxt:nxt + nblk[b]]
            ptable[b, :nblk[b]] = ids
            full = length // pbs
            if full:
                pkc[ids[:full].long()] = dk[off:off + full * pbs].view(full, pbs, 8, 128)
                pvc[ids[:full].long()] = dv[off:off + full * pbs].view(full, pbs, 8, 128)
            rem = length - full * pbs
            if rem:
                pkc[int(ids[full]), :rem] = dk[off + full * pbs:off + length]
                pvc[int(ids[full]), :rem] = dv[off + full * pbs:off + length]
            nxt += nblk[b]
            off += length
        pws = torch.empty(mea.decode_workspace_size(n_req, sum(nblk) * pbs, 64, 8, 128, 0),
                          dtype=torch.uint8, device=dev)
        pout = torch.empty_like(dq)
        plse = torch.empty_like(dlse)

        def dec_paged():
            mea.decode_paged(dq, pkc, pvc, ptable, dcu, max_k, scale=w4.scale, workspace=pws,
                             out=pout, lse=plse)

    launches_per_step = (1 if do_fwd else 0) + (2 if do_dec else 0)
    for _ in range(args.warmup):
        if do_fwd:
            fwd()
        if do_dec:
            dec()
    torch.cuda.synchronize()
    code = mea.device_error()
    if code:
        raise RuntimeError(f"device error word {code:#x} during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        if do_fwd:
            fwd()
        ev[i][1].record(stream)
        if do_dec:
            dec()
        ev[i][2].record(stream)
    t_end.record(stream)
    barrier(world)
    clk = clocks.stop()
    total_ms = dist_max(t_start.elapsed_time(t_end), world)
    fwd_ms = dist_max(sum(e[0].elapsed_time(e[1]) for e in ev), world) / args.steps
    dec_ms = dist_max(sum(e[1].elapsed_time(e[2]) for e in ev), world) / args.steps
    code = mea.device_error()
    if code:
        raise RuntimeError(f"device error word {code:#x} during the timed region")

    # ---- paged-cache decode of the same requests, timed on its own right after the decode
    # steps (not part of the step; run after the tensor-heavy forward loops instead, its
    # 16-slot stages, bound by the TMA's box rate, measured about 13 % lower)
    paged_obj = None
    if do_dec and args.paged:
        for _ in range(args.warmup):
            dec_paged()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            dec_paged()
        b.record(stream)
        barrier(world)
        pms = dist_max(a.elapsed_time(b), world) / args.steps
        code = mea.device_error()
        if code:
            raise RuntimeError(f"device error word {code:#x} during the paged decode")
        pgbs = dbytes / (pms * 1e-3) / 1e9
        hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        paged_obj = {"metric": f"paged decode KV GB/s ({pbs}-slot blocks, shuffled)",
                     "value": aggregate_throughput(dbytes, world, pms) / 1e9, "unit": "GB/s",
                     "ms_per_call": pms, "block_size": pbs,
                     "roofline": {"bound": "hbm", "achieved": pgbs, "peak": hbm, "unit": "GB/s",
                                  "frac": pgbs / hbm,
                                  "traffic": traffic_for("mea_decode_split_kernel_paged")
                                  if pbs == 16 else None,
                                  "peak_kind": "HBM copy",
                                  "kernel": "decode_split<paged> + lse_merge",
                                  "bytes_per_call": dbytes}}

    # ---- end to end through the public API with host buffers (pinned), copies inside
    e2e = None
    if not args.no_e2e and (do_fwd or do_dec):
        h2d = d2h = 0
        e2e_fwd_ms = e2e_dec_ms = 0.0
        n_e2e = max(1, args.e2e_steps)
        if do_fwd:
            hq_, hk_, hv_ = (t.cpu().pin_memory() for t in (q, k, v))
            hcu, hsl = cu.cpu().pin_memory(), slopes.cpu().pin_memory()
            hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
            hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
            h2d += sum(t.numel() * t.element_size() for t in (hq_, hk_, hv_, hcu, hsl))
            d2h += hout.numel() * hout.element_size() + hlse.numel() * 4

            def fwd_e2e():
                dq_, dk_, dv_ = (t.to(dev, non_blocking=True) for t in (hq_, hk_, hv_))
                dcu_, dsl_ = hcu.to(dev, non_blocking=True), hsl.to(dev, non_blocking=True)
                o, l_ = mea.attention_packed(dq_, dk_, dv_, dcu_, dcu_, max_q, causal=True,
                                             alibi_slopes=dsl_, scale=w2.scale)
                hout.copy_(o, non_blocking=True)
                hlse.copy_(l_, non_blocking=True)
            fwd_e2e()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n_e2e):
                fwd_e2e()
            b.record(stream)
            torch.cuda.synchronize()
            e2e_fwd_ms = dist_max(a.elapsed_time(b), world) / n_e2e
            del hq_, hk_, hv_
        if do_dec:
            hdq = dq.cpu().pin_memory()
            hdk = dk.cpu().pin_memory()
            hdv = dv.cpu().pin_memory()
            hdcu = dcu.cpu().pin_memory()
            hdo = torch.empty(dout.shape, dtype=dout.dtype).pin_memory()
            hdl = torch.empty(dlse.shape, dtype=dlse.dtype).pin_memory()
            h2d += sum(t.numel() * t.element_size() for t in (hdq, hdk, hdv, hdcu))
            d2h += hdo.numel() * hdo.element_size() + hdl.numel() * 4
            del dk, dv
            torch.cuda.empty_cache()

            def dec_e2e():
                q_, k_, v_ = (t.to(dev, non_blocking=True) for t in (hdq, hdk, hdv))
                c_ = hdcu.to(dev, non_blocking=True)
                o, l_ = mea.decode_splitkv(q_, k_, v_, c_, max_k, scale=w4.scale, workspace=ws)
                hdo.copy_(o, non_blocking=True)
                hdl.copy_(l_, non_blocking=True)
            dec_e2e()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n_e2e):
                dec_e2e()
            b.record(stream)
            torch.cuda.synchronize()
            e2e_dec_ms = dist_max(a.elapsed_time(b), world) / n_e2e
        e2e = {"h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e}
        if do_fwd:
            e2e.update({"value": aggregate_throughput(flops, world, e2e_fwd_ms) / 1e12,
                        "unit": "TFLOP/s",
                        "fwd_ms": e2e_fwd_ms})
        if do_dec:
            e2e.update({"decode_value": aggregate_throughput(dbytes, world, e2e_dec_ms) / 1e9,
                        "decode_unit": "GB/s", "decode_ms": e2e_dec_ms})
            if not do_fwd:
                e2e.update({"value": e2e["decode_value"], "unit": "GB/s"})

    # ---- FP8 forward on the packed prefill workload (e4m3 q/k/v), timed on its own
    fp8_obj = None
    if do_fwd and args.fp8:
        q8 = (q.float() * 2.0).to(torch.float8_e4m3fn)
        k8 = (k.float() * 4.0).to(torch.float8_e4m3fn)
        v8 = (v.float() * 0.5).to(torch.float8_e4m3fn)
        out8 = torch.empty_like(q)
        lse8 = torch.empty_like(lse)

        def fwd8():
            mea.attention_packed_fp8(q8, k8, v8, cu, cu, max_q, causal=True, alibi_slopes=slopes,
                                     scale=w2.scale, q_descale=0.5, k_descale=0.25,
                                     v_descale=2.0, out=out8, lse=lse8)
        for _ in range(args.warmup):
            fwd8()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fwd8()
        b.record(stream)
        barrier(world)
        f8ms = dist_max(a.elapsed_time(b), world) / args.steps
        code = mea.device_error()
        if code:
            raise RuntimeError(f"device error word {code:#x} during the FP8 forward")
        f8tf = flops / (f8ms * 1e-3) / 1e12
        peak8 = 2.0 * pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        fp8_obj = {"metric": "attention fwd TFLOP/s, e4m3 inputs (packed causal GQA+ALiBi)",
                   "value": aggregate_throughput(flops, world, f8ms) / 1e12, "unit": "TFLOP/s",
                   "ms_per_call": f8ms, "dtype": "e4m3 in, bf16 out",
                   "roofline": {"bound": "tensor", "achieved": f8tf, "peak": peak8,
                                "unit": "TFLOP/s", "frac": f8tf / peak8,
                                "traffic": traffic_for("mea_fwd_sm100_kernel_e4m3"),
                                "peak_kind": "fp8 = bf16 burst x 2 (nominal ratio)",
                                "kernel": "mea_fwd_sm100_kernel<…, e4m3>"}}

    # ---- long-context causal prefill (16384 tokens, GQA 64/8, no ALiBi), timed on its own
    long_obj = None
    if do_long:
        w3 = workload(3)
        g.manual_seed(w3.seed)
        t3 = w3.seqlens_q[0]
        q3 = torch.randn((t3, 64, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        k3 = torch.randn((t3, 8, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        v3 = torch.randn((t3, 8, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        cu3 = cu_seqlens(w3.seqlens_q).to(dev)
        out3 = torch.empty_like(q3)
        lse3 = torch.empty((64, t3), dtype=torch.float32, device=dev)
        flops3 = fwd_flops(w3.seqlens_q, 64, 128)

        def fwd3():
            mea.attention_packed(q3, k3, v3, cu3, cu3, t3, causal=True, scale=w3.scale,
                                 out=out3, lse=lse3)
        for _ in range(args.warmup):
            fwd3()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fwd3()
        b.record(stream)
        barrier(world)
        l3ms = dist_max(a.elapsed_time(b), world) / args.steps
        code = mea.device_error()
        if code:
            raise RuntimeError(f"device error word {code:#x} during the long prefill")
        l3tf = flops3 / (l3ms * 1e-3) / 1e12
        peak3 = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        long_obj = {"metric": "attention fwd TFLOP/s (causal prefill, 16384 tokens, GQA 64/8, "
                              "D=128, bf16)",
                    "value": aggregate_throughput(flops3, world, l3ms) / 1e12,
                    "unit": "TFLOP/s", "ms_per_call": l3ms,
                    "roofline": {"bound": "tensor", "achieved": l3tf, "peak": peak3,
                                 "unit": "TFLOP/s", "frac": l3tf / peak3,
                                 "traffic": traffic_for("mea_fwd_sm100_kernel_long"),
                                 "peak_kind": "bf16 burst",
                                 "kernel": "mea_fwd_sm100_kernel<128, bf16, causal>",
                                 "flops_per_launch": flops3}}
        del q3, k3, v3, out3, lse3

    # ---- the same long prefill at head dim 256 (the 256-wide kernel), timed on its own
    d256_obj = None
    if do_d256:
        w3 = workload(3)
        g.manual_seed(w3.seed + 256)
        t3 = w3.seqlens_q[0]
        q5 = torch.randn((t3, 64, 256), generator=g, device=dev, dtype=torch.float32).bfloat16()
        k5 = torch.randn((t3, 8, 256), generator=g, device=dev, dtype=torch.float32).bfloat16()
        v5 = torch.randn((t3, 8, 256), generator=g, device=dev, dtype=torch.float32).bfloat16()
        cu5 = cu_seqlens(w3.seqlens_q).to(dev)
        out5 = torch.empty_like(q5)
        lse5 = torch.empty((64, t3), dtype=torch.float32, device=dev)
        flops5 = fwd_flops(w3.seqlens_q, 64, 256)

        def fwd5():
            mea.attention_packed(q5, k5, v5, cu5, cu5, t3, causal=True, scale=1.0 / 16,
                                 out=out5, lse=lse5)
        for _ in range(args.warmup):
            fwd5()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n5 = max(1, args.steps // 4)
        a.record(stream)
        for _ in range(n5):
            fwd5()
        b.record(stream)
        barrier(world)
        d5ms = dist_max(a.elapsed_time(b), world) / n5
        code = mea.device_error()
        if code:
            raise RuntimeError(f"device error word {code:#x} during the D=256 prefill")
        d5tf = flops5 / (d5ms * 1e-3) / 1e12
        peak5 = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        d256_obj = {"metric": "attention fwd TFLOP/s (causal prefill, 16384 tokens, GQA 64/8, "
                              "D=256, bf16)",
                    "value": aggregate_throughput(flops5, world, d5ms) / 1e12,
                    "unit": "TFLOP/s", "ms_per_call": d5ms, "calls": n5,
                    "roofline": {"bound": "tensor", "achieved": d5tf, "peak": peak5,
                                 "unit": "TFLOP/s", "frac": d5tf / peak5,
                                 "traffic": traffic_for("mea_fwd256_sm100_kernel"),
                                 "peak_kind": "bf16 burst",
                                 "kernel": "mea_fwd256_sm100_kernel<bf16, causal>",
                                 "flops_per_launch": flops5}}
        del q5, k5, v5, out5, lse5

    # ---- backward on the packed prefill workload, timed on its own (not part of the step)
    bwd_obj = None
    if do_bwd:
        g.manual_seed(w2.seed + 1)
        gout = torch.randn((tq, 32, 128), generator=g, device=dev, dtype=torch.float32).bfloat16()
        gdq, gdk, gdv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = torch.empty(mea.backward_workspace_size(tq, 32), dtype=torch.uint8, device=dev)
        fwd_b = mea.attention_packed(q, k, v, cu, cu, max_q, causal=True, alibi_slopes=slopes,
                                     scale=w2.scale)

        def bwd():
            mea.attention_packed_backward(q, k, v, fwd_b[0], fwd_b[1], gout, cu, cu, max_q, max_q,
                                          causal=True, alibi_slopes=slopes, scale=w2.scale,
                                          workspace=bws, dq=gdq, dk=gdk, dv=gdv)
        for _ in range(args.warmup):
            bwd()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            bwd()
        b.record(stream)
        barrier(world)
        bwd_ms = dist_max(a.elapsed_time(b), world) / args.steps
        code = mea.device_error()
        if code:
            raise RuntimeError(f"device error word {code:#x} during the backward")
        # Peak memory of one forward + backward call pair: nothing is allocated by the library.
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        alloc0 = torch.cuda.memory_allocated(dev)
        mea.attention_packed(q, k, v, cu, cu, max_q, causal=True, alibi_slopes=slopes,
                             scale=w2.scale, out=fwd_b[0], lse=fwd_b[1])
        bwd()
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info(dev)
        mem_obj = {"device_bytes_allocated_by_calls": int(free0 - free1),
                   "torch_peak_growth_bytes": int(torch.cuda.max_memory_allocated(dev) - alloc0),
                   "backward_workspace_bytes": int(bws.numel()),
                   "largest_segment": max(w2.seqlens_q),
                   "score_matrix_bytes_if_materialised": 4 * max(w2.seqlens_q) ** 2 * 32}
        bflops = 2.5 * fwd_flops(w2.seqlens_q, 32, 128)
        btf = bflops / (bwd_ms * 1e-3) / 1e12
        peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        bwd_obj = {"metric": "attention bwd TFLOP/s (packed causal GQA+ALiBi)",
                   "value": aggregate_throughput(bflops, world, bwd_ms) / 1e12,
                   "unit": "TFLOP/s", "ms_per_call": bwd_ms, "flops_per_call": bflops,
                   "launches_per_call": 3,
                   "roofline": {"bound": "tensor", "achieved": btf, "peak": peak,
                                "unit": "TFLOP/s", "frac": btf / peak,
                                "traffic": traffic_for("mea_backward_call"),
                                "peak_kind": "bf16 burst",
                                "kernel": "bwd_pre + bwd_dkdv_tc + bwd_dq_tc"},
                   "memory": mem_obj}

    if rank != 0:
        return 0
    if args.part in ("long", "d256"):
        obj = long_obj if args.part == "long" else d256_obj
        line = {"metric": obj["metric"], "value": obj["value"], "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": obj["ms_per_call"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": obj["metric"]}, "roofline": obj["roofline"],
                "gpu_launches": args.steps}
        print(json.dumps(_compact(line)))
        return 0

    line = {"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
    line["config"] = step_config(args, world)
    if do_fwd:
        fwd_tf = flops / (fwd_ms * 1e-3) / 1e12
        line.update({"value": aggregate_throughput(flops, world, fwd_ms) / 1e12,
                     "unit": "TFLOP/s"})
        peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        line["roofline"] = {"bound": "tensor", "achieved": fwd_tf, "peak": peak,
                            "unit": "TFLOP/s", "frac": fwd_tf / peak,
                            "traffic": traffic_for("mea_fwd_sm100_kernel"),
                            "peak_kind": f"dense bf16 burst, {peak_src}",
                            "kernel": "mea_fwd_sm100_kernel", "ms_per_launch": fwd_ms,
                            "flops_per_launch": flops}
    if do_dec:
        gbs = dbytes / (dec_ms * 1e-3) / 1e9
        hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        dec_obj = {"metric": "decode KV GB/s",
                   "value": aggregate_throughput(dbytes, world, dec_ms) / 1e9, "unit": "GB/s",
                   "ms_per_call": dec_ms,
                   "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                "frac": gbs / hbm,
                                "traffic": traffic_for("mea_decode_split_kernel"),
                                "peak_kind": f"HBM copy, {peak_src}",
                                "kernel": "mea_decode_split_kernel + mea_lse_merge_kernel",
                                "bytes_per_call": dbytes}}
        if not do_fwd:
            line.update({"value": dec_obj["value"], "unit": "GB/s",
                         "roofline": dec_obj["roofline"]})
    if bwd_obj is not None and not do_fwd and not do_dec:
        line.update({"value": bwd_obj["value"], "unit": "TFLOP/s",
                     "roofline": bwd_obj["roofline"], "ms_per_step": bwd_obj["ms_per_call"]})
        line["metric"] = bwd_obj["metric"]
    line["clocks"] = clk
    line["gpu_launches"] = launches_per_step * args.steps
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and do_fwd and world == 1:
        sample, fl, desc = oracle_sample(5.0e11)
        dt = time_oracle(sample)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": desc, "seconds": dt}
    # The extra measurements come last, the decode (the step's second metric) at the very end,
    # so that a reader keeping only the tail of the line still has it.
    for key, obj in (("fp8_forward", fp8_obj), ("paged_decode", paged_obj),
                     ("backward", bwd_obj), ("prefill_d256", d256_obj),
                     ("long_prefill", long_obj)):
        if obj is not None:
            line[key] = obj
    if do_dec:
        line["decode"] = dec_obj
    print(json.dumps(_compact(line)))
    return 0


def _compact(obj):
    """Floats rounded to 5 significant digits (the line stays short; timings are not that
    precise anyway)."""
    if isinstance(obj, float):
        return float(f"{obj:.5g}") if math.isfinite(obj) else obj
    if isinstance(obj, dict):
        return {k: _compact(v) for k, v in obj.items()}
    if isinstance(obj, list):
        return [_compact(v) for v in obj]
    return obj


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
    else:
        rc = run_ours(args, world, rank, local)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
