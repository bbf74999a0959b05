"""Benchmark: retained-mass block-sparse attention on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
                    [--split problems|heads]

A step is one calibrate-then-reuse cycle of the 720p workload (the default config,
Wan-14B-like: B=1, 40 heads, D=128, 21x45x80 tokens padded to 24x48x80, 64-token blocks):
    calibration  tile_permute(Q, K) -> block_mass -> topp_select(0.99)
    10 x reuse   tile_permute(Q_r, K_r, V_r) -> bsattn_fwd(frozen lists) -> inverse permute
                 (--layout raster: bsattn_fwd_raster, the permutation fused into the
                 forward's loads and stores; the e4m3 workload always takes
                 tile_permute_quant_e4m3 x3 -> bsattn_fwd -> inverse)
on seeded synthetic inputs already resident in HBM (Q/K/V of 774 MB each, far above L2).
--config wan14b_720p_local runs the same shape with spatially local attention (~66% of
the block pairs kept at 0.99); --config wan14b_720p_fp8 the e4m3 operands; both also
take 10 reuse calls per step (--reuse overrides).

value  = executed attention TFLOP/s of the whole step (a step rate): FLOPs of the kept
         blocks of the 10 reuse calls (4 * 64 * 64 * D per kept (query block, kv block)
         pair) divided by the device time of the whole cycle, calibration included, max
         over ranks.
fwd    = the same FLOPs over the forward launches alone (CUDA events on the launch
         stream) -> roofline of the dominant kernel.
e2e    = the same metric through the public API with inputs copied from pinned host
         memory and outputs copied back inside the timed region.
--impl reference times the CPU oracle (the only other implementation of the method) on
a bounded sample of the same workload: the inputs are drawn once, each step times the
oracle's masked attention on its own sampled query rows and CSR, and the rows per step are
sized from a short probe so that all steps together take about REF_BUDGET_S seconds
(16 to --cpu-sample-rows rows a step).  The main line's cpu_baseline times
--cpu-sample-rows rows once.

With N > 1 ranks (one per GPU) the path needs no exchange step: --split problems (the
default) gives every rank an independent problem of the workload's size (weak scaling);
--split heads gives rank r the heads [r*Hh/N, (r+1)*Hh/N) of one problem (strong scaling;
Hh must divide by N).  The process group carries only the timing barrier, the
max-over-ranks reduction of the timed region and the sum of the ranks' executed work.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="wan14b_720p")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--reuse", type=int, default=None, help="reuse calls per step (default: the workload's)")
    ap.add_argument("--tau", type=float, default=0.99)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layout", default="tiles", choices=["raster", "tiles"],
                    help="bf16 reuse calls: permute + tile-major forward (the faster, measured), "
                         "or the fused raster forward")
    ap.add_argument("--cpu-sample-rows", type=int, default=256)
    ap.add_argument("--clock-log", default=None,
                    help="CSV of the nvidia-smi clock samples ({rank} is replaced); default /tmp")
    ap.add_argument("--split", default="problems", choices=["problems", "heads"],
                    help="N > 1: an independent problem per rank, or the heads of one problem "
                         "divided over the ranks")
    return ap.parse_args(argv)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16 tensor peak (NVIDIA's figure without 2:4 sparsity)


def head_range(rank: int, world: int, heads: int):
    """Heads [h0, h1) of one problem owned by `rank` when the heads are split over `world`
    ranks (equal shares; the head count must divide by the rank count)."""
    if heads % world:
        raise ValueError(f"{heads} heads do not divide over {world} ranks")
    n = heads // world
    return rank * n, (rank + 1) * n


def measured_traffic(fp8: bool, raster: bool):
    """DRAM bytes per forward launch of the variant the bench times, from the committed ncu
    summary (bf16: the recorded full-size capture; e4m3: the 8-head capture scaled to 40
    heads; raster: the recorded full-size capture), or None when the kernel sources have
    changed since it was taken."""
    import hashlib
    import re
    name = "bsattn_fwd_raster_wan14b_720p_dram.md" if raster else "bsattn_fwd_wan14b_720p_dram.md"
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    key = "traffic_bytes_per_launch_e4m3" if fp8 else "traffic_bytes_per_launch"
    m = re.search(key + r":\s*(\d+)", text)
    if not m:
        return None
    csrc = os.path.join(ROOT, "block_sparse_attention_25_b200", "csrc")
    for name in ("attn_fwd.cu", "bsa_common.cuh"):
        h = re.search(r"source_sha256 " + re.escape(name) + r":\s*([0-9a-f]{64})", text)
        cur = hashlib.sha256(open(os.path.join(csrc, name), "rb").read()).hexdigest()
        if not h or h.group(1) != cur:
            return None
    return int(m.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    def __init__(self, gpu_index: int, path: str):
        self.path = path
        self.proc = None
        try:
            self.f = open(path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 active=parts[4], hw=parts[5], hwt=parts[6], swt=parts[7],
                                 pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 300] or rows
        sms = sorted(r["sm"] for r in load)
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": sms[len(sms) // 2], "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


def dist_setup(args):
    """One process per GPU: NCCL when CUDA is available (the device of LOCAL_RANK), gloo on
    a host without GPUs (the CPU tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(x: float, pg) -> float:
    if pg is None:
        return x
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, pg) -> float:
    if pg is None:
        return x
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ============================================================================ ours
def run_ours(args, world, rank, local, pg):
    import torch

    import block_sparse_attention_25_b200 as bsa
    from block_sparse_attention_25_b200 import build, synth

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl_full = synth.WORKLOADS[args.config]
    n_reuse = args.reuse if args.reuse is not None else max(wl_full.redraws, 1)
    heads = args.split == "heads" and world > 1
    if heads:
        # rank's share of one problem: its heads of the same draws
        h0, h1 = head_range(rank, world, wl_full.heads)
        wl = wl_full.scaled(heads=h1 - h0)
        draw_wl = wl_full

        def mine(qkv):
            return tuple(x[:, :, h0:h1].contiguous() for x in qkv)
    else:
        wl = wl_full
        draw_wl = wl_full.scaled(seed=wl_full.seed + 7919 * rank)  # independent problem per rank

        def mine(qkv):
            return qkv
    s = bsa.Shape.of(wl)
    fp8 = wl.fp8
    raster = not fp8 and args.layout == "raster"

    # ---- inputs resident in HBM: the calibration draw and n_reuse correlated re-draws
    draws = [mine(synth.draw_qkv(draw_wl, device=dev))]
    for r in range(1, n_reuse + 1):
        draws.append(mine(synth.redraw_qkv(draw_wl, r, device=dev)))
    torch.cuda.synchronize()

    tiled = (s.batch, s.heads, s.Np, s.head_dim)
    qt = torch.empty(tiled, dtype=torch.bfloat16, device=dev)
    kt = torch.empty_like(qt)
    vt = torch.empty_like(qt)
    if fp8:
        q8 = torch.empty(tiled, dtype=torch.uint8, device=dev)
        k8, v8 = torch.empty_like(q8), torch.empty_like(q8)
        sc = [torch.empty((s.batch, s.heads, s.Np // 64), dtype=torch.float32, device=dev)
              for _ in range(3)]
    out_t = torch.empty_like(qt)
    out_r = [torch.empty((s.batch, s.S, s.heads, s.head_dim), dtype=torch.bfloat16, device=dev)
             for _ in range(n_reuse)]
    mass = torch.empty((s.batch, s.heads, s.n_qb, s.n_kb), dtype=torch.float32, device=dev)
    row_ptr = torch.empty(s.rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(s.rows * s.n_kb, dtype=torch.int32, device=dev)
    ws_m = bsa.new_workspace(s, bsa.OP_BLOCK_MASS, dev)
    ws_t = bsa.new_workspace(s, bsa.OP_TOPP_SELECT, dev)
    ws_f = bsa.new_workspace(s, bsa.OP_FWD, dev)
    stream = torch.cuda.current_stream()
    fwd_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_reuse)] for _ in range(args.steps)]
    cur = {"step": 0}
    cal_ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    launches_per_step = 0

    def step(time_fwd: bool):
        nonlocal launches_per_step
        n = 0
        q0, k0, _ = draws[0]
        cal_ev[0].record(stream)
        bsa.tile_permute(q0, s, out=qt)
        bsa.tile_permute(k0, s, out=kt)
        bsa.block_mass(qt, kt, s, out=mass, ws=ws_m)
        bsa.topp_select(mass, s, args.tau, ws=ws_t, row_ptr=row_ptr, col_idx=col_idx)
        cal_ev[1].record(stream)
        n += 2 + 1 + 3
        for r in range(n_reuse):
            q, k, v = draws[r + 1]
            if fp8:
                bsa.tile_permute_quant_e4m3(q, s, out=q8, scales=sc[0])
                bsa.tile_permute_quant_e4m3(k, s, out=k8, scales=sc[1])
                bsa.tile_permute_quant_e4m3(v, s, out=v8, scales=sc[2])
                if time_fwd:
                    fwd_ev[cur["step"]][r][0].record(stream)
                bsa.bsattn_fwd(q8, k8, v8, row_ptr, col_idx, s, scales=sc, out=out_t, ws=ws_f)
            elif raster:
                if time_fwd:
                    fwd_ev[cur["step"]][r][0].record(stream)
                bsa.bsattn_fwd_raster(q, k, v, row_ptr, col_idx, s, out=out_r[r], ws=ws_f)
                if time_fwd:
                    fwd_ev[cur["step"]][r][1].record(stream)
                n += 1 + s.batch  # schedule + one forward launch per batch
                continue
            else:
                bsa.tile_permute(q, s, out=qt)
                bsa.tile_permute(k, s, out=kt)
                bsa.tile_permute(v, s, out=vt)
                if time_fwd:
                    fwd_ev[cur["step"]][r][0].record(stream)
                bsa.bsattn_fwd(qt, kt, vt, row_ptr, col_idx, s, out=out_t, ws=ws_f)
            if time_fwd:
                fwd_ev[cur["step"]][r][1].record(stream)
            bsa.tile_permute(out_t, s, inverse=True, out=out_r[r])
            n += 3 + 2 + 1
        launches_per_step = n

    # warm-up
    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    for w in (ws_m, ws_t, ws_f):
        st = bsa.device_status(w)
        if st != 0:
            raise RuntimeError(f"device status {st} after warm-up: {bsa.device_status_words(w)}")

    # executed FLOPs of one reuse call: kept pairs * 4 * q_block * 64 * D
    from block_sparse_attention_25_b200.microbench import schedule_work
    work = schedule_work(row_ptr, col_idx, s)
    nnz = int(row_ptr[-1].item())
    kept_frac = nnz / float(s.rows * s.n_kb)
    flops_call = 4.0 * nnz * s.q_block * 64 * s.head_dim
    dense_flops_call = 4.0 * s.rows * s.n_kb * s.q_block * 64 * s.head_dim

    # timed region
    clk_path = (args.clock_log.replace("{rank}", str(rank)) if args.clock_log
                else f"/tmp/bsa_clocks_{rank}.csv")
    clk = ClockSampler(local, clk_path)
    barrier(pg)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        cur["step"] = i
        step(True)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(pg)
    clocks = clk.stop()
    # every bsattn_fwd launch of the timed region (CUDA events on the launch stream)
    fwd_ms = [a.elapsed_time(b) for evs in fwd_ev for a, b in evs]
    cal_ms = cal_ev[0].elapsed_time(cal_ev[1])
    elapsed_ms = t0.elapsed_time(t1)
    elapsed_ms = max_over_ranks(elapsed_ms, pg)
    for w in (ws_m, ws_t, ws_f):
        st = bsa.device_status(w)
        if st != 0:
            raise RuntimeError(f"device status {st} after timing: {bsa.device_status_words(w)}")

    ms_step = elapsed_ms / args.steps
    # every rank's executed FLOPs (a rank's problem, or its share of one problem's heads)
    total_flops = sum_over_ranks(flops_call * n_reuse * args.steps, pg)
    value = total_flops / (elapsed_ms * 1e-3) / 1e12
    fwd_avg_ms = sum(fwd_ms) / len(fwd_ms)
    fwd_tflops = flops_call / (fwd_avg_ms * 1e-3) / 1e12
    pk = peaks()
    peak = pk["bf16_sus"] * (2.0 if fp8 else 1.0)
    peak_note = ("sustained bf16 of " + pk["source"]) + (" x2 (fp8 nominal ratio)" if fp8 else "")

    # ---- end to end through the public API, host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, bsa, s, draws, n_reuse, row_ptr, col_idx, flops_call, dev, stream,
                      fp8, raster, pg, world)

    result = {
        "metric": "bsattn_fwd ms/call & executed TFLOPS at 99% retained mass, % of bf16 peak",
        "value": round(value, 2),
        "unit": f"TFLOP/s (executed, kept blocks; step rate: calibration + {n_reuse} reuse calls)",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "strong" if heads else "weak",
        "vs_baseline": None,
        "dtype": "e4m3" if fp8 else "bf16",
        "data": "synthetic (seeded 3D random-Fourier-feature Q/K/V + noise, correlated re-draws)",
        "config": {
            "workload": wl.name,
            "grid": f"{wl.T}x{wl.H}x{wl.W} padded {wl.Tp}x{wl.Hp}x{wl.Wp}",
            "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
            "q_block": wl.q_block, "kv_block": 64, "tokens": wl.S, "slots": wl.Np,
            "threshold": args.tau, "reuse_calls_per_step": n_reuse,
            "layout": "raster (permutation fused into the forward)" if raster
                      else "tile-major (separate permutation launches)",
            "kept_fraction": round(kept_frac, 5),
            "bsattn_fwd_ms_per_call": round(fwd_avg_ms, 3),
            "bsattn_fwd_tflops": round(fwd_tflops, 2),
            "bsattn_fwd_pct_of_peak": round(100.0 * fwd_tflops / peak, 2),
            "bsattn_fwd_pct_of_peak_note": "of the sustained measured peak (" + peak_note + ")",
            "bsattn_fwd_pct_of_burst_peak": round(
                100.0 * fwd_tflops / (pk["bf16"] * (2.0 if fp8 else 1.0)), 2),
            "bsattn_fwd_pct_of_nominal_peak": round(
                100.0 * fwd_tflops / (NOMINAL_BF16_TFLOPS * (2.0 if fp8 else 1.0)), 2),
            "pairs_kept": work["kept_pairs"],
            "pairs_computed": work["computed_pairs"],
            "computed_over_kept": work["computed_over_kept"],
            "dense_equivalent_tflops": round(dense_flops_call / (fwd_avg_ms * 1e-3) / 1e12, 2),
            "calibration_ms": round(cal_ms, 3),
            "executed_tflop_per_call": round(flops_call / 1e12, 3),
            "l2": "inputs larger than L2 (774 MB per tensor); no flush needed",
            "parallelism": (f"heads of one problem split over {world} GPUs ({wl.heads} each)"
                            if heads else f"independent problem per GPU x{world}"),
        },
        "roofline": {
            "bound": "tensor", "achieved": round(fwd_tflops, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(fwd_tflops / peak, 4),
            "traffic": (measured_traffic(fp8, raster)
                        if wl.name in (synth.WORKLOADS["wan14b_720p"].name,
                                       synth.WORKLOADS["wan14b_720p_fp8"].name) else None),
            "traffic_unit": ("bytes per launch (dram read + write; an 8-head ncu capture x 5)"
                             if fp8 else
                             "bytes per launch (dram read + write, one full-size ncu capture)"),
            "kernel": (f"bsattn_fwd_kernel<{s.head_dim},false,false,true> (raster layout)" if raster
                       else f"bsattn_fwd_kernel<{s.head_dim},{'true' if fp8 else 'false'},false,false>"),
            "peak_source": peak_note,
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    return result


def run_e2e(args, bsa, s, draws, n_reuse, row_ptr, col_idx, flops_call, dev, stream, fp8, fused,
            pg, world):
    """Same cycle through the public API, every input copied in from pinned host memory and
    every output copied back, inside the timed region.  The copies run on two copy streams
    and overlap the compute: the inputs of the next call land in the second of two device
    buffer sets while the current call runs, and each output is read back while the next
    call computes (events order every reuse of a buffer)."""
    import torch
    def pinned_copy(x):
        h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        h.copy_(x)
        return h

    host = [tuple(pinned_copy(x) for x in d) for d in draws]
    out_host = [torch.empty((s.batch, s.S, s.heads, s.head_dim), dtype=torch.bfloat16).pin_memory()
                for _ in range(n_reuse)]
    raster = draws[0][0]
    sets = [tuple(torch.empty_like(raster) for _ in range(3)) for _ in range(2)]
    outs = [torch.empty_like(raster) for _ in range(2)]
    tiled = (s.batch, s.heads, s.Np, s.head_dim)
    qt = torch.empty(tiled, dtype=torch.bfloat16, device=dev)
    kt, vt, ot = torch.empty_like(qt), torch.empty_like(qt), torch.empty_like(qt)
    mass = torch.empty((s.batch, s.heads, s.n_qb, s.n_kb), dtype=torch.float32, device=dev)
    rp = torch.empty_like(row_ptr)
    ci = torch.empty_like(col_idx)
    ws_m = bsa.new_workspace(s, bsa.OP_BLOCK_MASS, dev)
    ws_t = bsa.new_workspace(s, bsa.OP_TOPP_SELECT, dev)
    ws_f = bsa.new_workspace(s, bsa.OP_FWD, dev)
    if fp8:
        q8 = torch.empty(tiled, dtype=torch.uint8, device=dev)
        k8, v8 = torch.empty_like(q8), torch.empty_like(q8)
        sc = [torch.empty((s.batch, s.heads, s.Np // 64), dtype=torch.float32, device=dev)
              for _ in range(3)]
    up = torch.cuda.Stream(device=dev)    # host -> device
    down = torch.cuda.Stream(device=dev)  # device -> host
    ev = lambda: torch.cuda.Event()       # noqa: E731
    # per buffer set / output buffer: the event after which it may be overwritten
    state = {"g": 0, "set_free": [None, None], "out_free": [None, None], "in": {}}
    counts = {"h2d": 0, "d2h": 0}
    # one step = the calibration call (job 0: q, k) and n_reuse reuse calls (jobs 1..n)
    jobs = [0] + list(range(1, n_reuse + 1))

    def issue_copy(g, job):
        st = g % 2
        if state["set_free"][st] is not None:
            up.wait_event(state["set_free"][st])      # the set's previous call has read it
        with torch.cuda.stream(up):
            n_in = 2 if job == 0 else 3
            for dst, src in zip(sets[st][:n_in], host[job][:n_in]):
                dst.copy_(src, non_blocking=True)
            e = ev()
            e.record(up)
        state["in"][g] = e
        counts["h2d"] += n_in * raster.numel() * 2

    def compute(g, job):
        st = g % 2
        dq, dk, dv = sets[st]
        stream.wait_event(state["in"].pop(g))
        if job == 0:
            bsa.tile_permute(dq, s, out=qt)
            bsa.tile_permute(dk, s, out=kt)
            e = ev()
            e.record(stream)
            state["set_free"][st] = e
            bsa.block_mass(qt, kt, s, out=mass, ws=ws_m)
            bsa.topp_select(mass, s, args.tau, ws=ws_t, row_ptr=rp, col_idx=ci)
            return
        if fused:  # the forward reads the raster set and writes the output buffer directly
            if state["out_free"][st] is not None:
                stream.wait_event(state["out_free"][st])
            bsa.bsattn_fwd_raster(dq, dk, dv, rp, ci, s, out=outs[st], ws=ws_f)
            e = ev()
            e.record(stream)
            state["set_free"][st] = e
            down.wait_event(e)
            with torch.cuda.stream(down):
                out_host[job - 1].copy_(outs[st], non_blocking=True)
                e = ev()
                e.record(down)
            state["out_free"][st] = e
            counts["d2h"] += raster.numel() * 2
            return
        if fp8:
            bsa.tile_permute_quant_e4m3(dq, s, out=q8, scales=sc[0])
            bsa.tile_permute_quant_e4m3(dk, s, out=k8, scales=sc[1])
            bsa.tile_permute_quant_e4m3(dv, s, out=v8, scales=sc[2])
        else:
            bsa.tile_permute(dq, s, out=qt)
            bsa.tile_permute(dk, s, out=kt)
            bsa.tile_permute(dv, s, out=vt)
        e = ev()
        e.record(stream)
        state["set_free"][st] = e
        if fp8:
            bsa.bsattn_fwd(q8, k8, v8, rp, ci, s, scales=sc, out=ot, ws=ws_f)
        else:
            bsa.bsattn_fwd(qt, kt, vt, rp, ci, s, out=ot, ws=ws_f)
        if state["out_free"][st] is not None:
            stream.wait_event(state["out_free"][st])   # the buffer's last output was read back
        bsa.tile_permute(ot, s, inverse=True, out=outs[st])
        done = ev()
        done.record(stream)
        down.wait_event(done)
        with torch.cuda.stream(down):
            out_host[job - 1].copy_(outs[st], non_blocking=True)
            e = ev()
            e.record(down)
        state["out_free"][st] = e
        counts["d2h"] += raster.numel() * 2

    def run(steps):
        seq = [job for _ in range(steps) for job in jobs]
        g0 = state["g"]
        issue_copy(g0, seq[0])
        for i, job in enumerate(seq):
            if i + 1 < len(seq):
                issue_copy(g0 + i + 1, seq[i + 1])
            compute(g0 + i, job)
        state["g"] = g0 + len(seq)
        for e in state["out_free"]:
            if e is not None:
                stream.wait_event(e)                   # every read-back inside the region

    run(1)
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 3))
    barrier(pg)
    torch.cuda.synchronize()
    counts["h2d"] = counts["d2h"] = 0
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    down.wait_event(a)
    run(steps)
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), pg)
    val = sum_over_ranks(flops_call * n_reuse * steps, pg) / (ms * 1e-3) / 1e12
    return {"value": round(val, 2), "unit": "TFLOP/s (executed, kept blocks)",
            "h2d_bytes_per_step": counts["h2d"] // steps, "d2h_bytes_per_step": counts["d2h"] // steps,
            "steps": steps, "ms_per_step": round(ms / steps, 3),
            "copies": "pinned host memory, two copy streams overlapping the compute"}


# ============================================================================ CPU oracle
# Seconds of oracle work the reference arm's timed steps take together (about).
REF_BUDGET_S = 120.0


def oracle_inputs(wl):
    """Seeded synthetic inputs of the workload for the oracle, drawn and permuted once on
    the host: two heads of Q, K and V in tile-major float64 (the rows are sampled from
    them; a head's cost per row does not depend on the head count)."""
    import torch

    from block_sparse_attention_25_b200 import synth
    from oracle import bsa_oracle as O

    g = O.Grid(wl.T, wl.H, wl.W, wl.Tp, wl.Hp, wl.Wp)
    heads = 2
    q, k, v = synth.draw_qkv(wl.scaled(heads=heads), device="cpu")
    qt, kt, vt = (O.permute_forward(x.to(torch.float64).numpy(), g) for x in (q, k, v))
    return dict(wl=wl, g=g, heads=heads, qkv=(qt, kt, vt))


def oracle_rows(inp, n_rows: int, seed: int = 0):
    """Time the oracle's masked attention on n_rows sampled query rows (a seeded CSR at the
    workload's kept fraction).  Returns (executed FLOPs, seconds, description)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from block_sparse_attention_25_b200 import synth
    from oracle import bsa_oracle as O

    wl, g, heads = inp["wl"], inp["g"], inp["heads"]
    qt, kt, vt = inp["qkv"]
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    rp, ci = synth.draw_keep_csr(heads * n_qb, n_kb, wl.nominal_kept, seed=seed)
    rp, ci = rp.numpy(), ci.numpy()
    valid = O.valid_slots(g)
    rng = np.random.default_rng(seed)
    cand = np.nonzero(valid)[0]
    n_rows = min(n_rows, cand.size)
    rows = [(0, int(rng.integers(0, heads)), int(p)) for p in rng.choice(cand, n_rows, replace=False)]
    flops = 0.0
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        for (b, h, p) in rows:
            O.masked_attention_query(qt, kt, vt, g, b, h, p, wl.q_block, 64, rp, ci,
                                     1.0 / math.sqrt(wl.head_dim))
            r = h * n_qb + p // wl.q_block
            blocks = ci[rp[r]:rp[r + 1]]
            nk = int(sum(valid[j * 64:(j + 1) * 64].sum() for j in blocks))
            flops += 4.0 * wl.head_dim * nk
        dt = time.perf_counter() - t
    desc = (f"oracle masked attention (numpy fp64, 1 thread) on {n_rows} sampled query rows of "
            f"{wl.name} with a seeded CSR at {wl.nominal_kept} kept; TFLOP/s = executed FLOPs of those rows / time")
    return flops, dt, desc


def oracle_sample(wl, n_rows: int, seed: int = 0):
    """oracle_rows on freshly drawn inputs (the main line's CPU baseline)."""
    return oracle_rows(oracle_inputs(wl), n_rows, seed)


def oracle_units(wl, seed: int = 0):
    """Per-unit times of the oracle's other steps on the workload (one head drawn on the
    host, one thread), each with its unit count per call and a labelled extrapolation to
    one call: a query-block row of masses, a top-p row, one tensor-head of the permute."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_limits

    from block_sparse_attention_25_b200 import synth
    from oracle import bsa_oracle as O

    g = O.Grid(wl.T, wl.H, wl.W, wl.Tp, wl.Hp, wl.Wp)
    q, k, _ = synth.draw_qkv(wl.scaled(heads=1), device="cpu")
    n_qb, n_kb = wl.Np // wl.q_block, wl.Np // 64
    rows_per_call = wl.batch * wl.heads * n_qb
    out = {}

    def unit(seconds, per_call, what):
        return {"unit": what, "ms_per_unit": round(1e3 * seconds, 3), "units_per_call": per_call,
                "extrapolated_call_s": round(seconds * per_call, 1)}

    with threadpool_limits(limits=1):
        t = time.perf_counter()
        qt = O.permute_forward(q.to(torch.float64).numpy(), g)
        out["tile_permute"] = unit(time.perf_counter() - t, 3 * wl.batch * wl.heads,
                                   "one tensor of one head")
        kt = O.permute_forward(k.to(torch.float64).numpy(), g)
        rng = np.random.default_rng(seed)
        pick = rng.choice(n_qb, 2, replace=False)
        t = time.perf_counter()
        for i in pick:
            O.block_mass_row(qt, kt, g, 0, 0, int(i), wl.q_block, 64, 1.0 / math.sqrt(wl.head_dim))
        out["block_mass"] = unit((time.perf_counter() - t) / len(pick), rows_per_call,
                                 "one query-block row of masses")
        m = synth.draw_mass_rows(100, n_kb, seed=seed).double().numpy()
        t = time.perf_counter()
        for r in m:
            O.topp_select_row(r, np.float32(0.99))
        out["topp_select"] = unit((time.perf_counter() - t) / len(m), rows_per_call, "one row")
    return out


def run_reference(args, world, rank, pg):
    from block_sparse_attention_25_b200 import synth
    wl = synth.WORKLOADS[args.config]
    if rank != 0:
        return None
    # inputs drawn once; each step samples its own rows and CSR.  Rows per step: as many as
    # fit REF_BUDGET_S over all steps at the rate of an 8-row probe (at least 16, at most
    # --cpu-sample-rows), so the run stays within a few minutes for any --steps.
    inp = oracle_inputs(wl)
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_rows(inp, 4, seed=100_000)
    _, t_probe, _ = oracle_rows(inp, 8, seed=100_001)
    per_row = max(t_probe / 8, 1e-6)
    n_rows = int(min(args.cpu_sample_rows,
                     max(16, REF_BUDGET_S / max(1, args.steps) / per_row)))
    tot_f = tot_t = 0.0
    desc = ""
    for i in range(args.steps):
        f, t, desc = oracle_rows(inp, n_rows, seed=i)
        tot_f += f
        tot_t += t
    val = tot_f / tot_t / 1e12
    return {
        "impl": "reference",
        "metric": "bsattn_fwd ms/call & executed TFLOPS at 99% retained mass, % of bf16 peak",
        "value": val, "unit": "TFLOP/s (executed, kept blocks)", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name,
                   "grid": f"{wl.T}x{wl.H}x{wl.W} padded {wl.Tp}x{wl.Hp}x{wl.Wp}",
                   "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
                   "q_block": wl.q_block, "kv_block": 64, "tokens": wl.S, "slots": wl.Np,
                   "threshold": args.tau},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s (executed, kept blocks)", "cores": 1,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s (executed, kept blocks)", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world, rank, local, pg = dist_setup(args)
    if args.impl == "reference":
        res = run_reference(args, world, rank, pg)
        if rank == 0:
            print(json.dumps(res), flush=True)
        if pg is not None:
            pg.destroy_process_group()
        return
    res = run_ours(args, world, rank, local, pg)
    if rank == 0:
        from block_sparse_attention_25_b200 import synth
        wl = synth.WORKLOADS[args.config]
        res["cpu_baseline"] = None
        if world == 1:  # the oracle baseline is taken at N = 1 only
            f, t, desc = oracle_sample(wl, args.cpu_sample_rows)
            n_q = wl.batch * wl.heads * wl.S
            units = oracle_units(wl)
            units["attention"] = {"unit": "one query row", "ms_per_unit": round(1e3 * t / args.cpu_sample_rows, 3),
                                  "units_per_call": n_q,
                                  "extrapolated_call_s": round(t / args.cpu_sample_rows * n_q, 1)}
            res["cpu_baseline"] = {"value": f / t / 1e12, "unit": "TFLOP/s (executed, kept blocks)",
                                   "cores": 1, "kind": "oracle", "sample": desc,
                                   "seconds": round(t, 2),
                                   "units": units,
                                   "units_note": "per-unit oracle times; extrapolated_call_s is an "
                                                 "extrapolation to one full call, not a measurement"}
        print(json.dumps(res), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
