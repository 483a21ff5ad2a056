"""Benchmark of the VBQ mixed-bit GEMV on B200: achieved HBM GB/s against the measured copy peak.

Default workload: the seven linears of one 9B-shaped decoder layer at batch 1 (q, k, v, o 4096x4096; gate, up
4096->14336; down 14336->4096), with widths drawn from the VBQ paper's allocation (about 69% 1-bit groups,
1.85 mean bits). One step runs all seven GEMVs. Four distinct seeded copies of the layer (about 260 MB, more
than the 126 MB L2) are used in rotation, so every step streams its weights from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--impl vbq|reference]

Under torchrun (N > 1) every rank runs an independent replica on its own GPU. The path has no cross-GPU
exchange. Time is the max over ranks, and the value is the bytes of all ranks divided by that time.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import vbq_synth as S  # noqa: E402

METRIC = "mixed-bit GEMV achieved HBM GB/s (% of B200 peak); decode-step µs at 1 GPU"
UNIT = "GB/s"
NAMES = ("q", "k", "v", "o", "gate", "up", "down")
GROUPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))   # projections that share their input, fused
WORKLOAD = "9B-shaped decoder-layer linears (q,k,v,o 4096x4096; gate,up 4096->14336; down 14336->4096)"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------------ setup
def layer_matrices(copy: int):
    return [S.make_matrix(4, n, *S.CFG4_SHAPES[n], layer=copy) for n in NAMES]


def blob_bytes_of(m, R):
    from decode_vbq_gemv_b200 import vbq
    return vbq.vbq_packed_size(m.N, m.K, R, m.widths)


def cpu_baseline(B: int, budget_s: float = 12.0, matrices=None):
    """Times the fp64 oracle (as it stands) on a bounded sample of the workload: the first `rows` rows of each
    of the seven linears, growing the sample until it takes about `budget_s` seconds or covers every row."""
    from oracle import oracle as O
    from decode_vbq_gemv_b200 import vbq
    mats = matrices or layer_matrices(0)
    threads = os.cpu_count() or 1
    xs = [S.make_x(4, m.name, B, m.K) for m in mats]
    full = [vbq.vbq_packed_size(m.N, m.K, 1024, m.widths) for m in mats]
    rows = 64
    while True:
        t0 = time.perf_counter()
        nbytes = 0.0
        for m, x, fb in zip(mats, xs, full):
            r = min(rows, m.N)
            O.matvec(m.widths[:r], m.scales[:r], m.codes[:r], x, threads)
            nbytes += fb * r / m.N + B * m.K * 2 + B * r * 4
        dt = time.perf_counter() - t0
        if dt > budget_s / 4 or rows >= max(m.N for m in mats):
            break
        rows *= 4
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle on the first {rows} rows of each of the 7 linears, batch {B} "
                      f"({dt:.2f} s); GB/s scaled from those rows' share of the packed bytes"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def allreduce_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------------------ arms
def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    from oracle import oracle as O
    mats = layer_matrices(0)
    xs = [S.make_x(4, m.name, args.batch, m.K) for m in mats]
    full = [blob_bytes_of(m, 1024) for m in mats]
    rows = args.ref_rows
    threads = os.cpu_count() or 1

    def step():
        nb = 0.0
        for m, x, fb in zip(mats, xs, full):
            O.matvec(m.widths[:rows], m.scales[:rows], m.codes[:rows], x, threads)
            nb += fb * rows / m.N + args.batch * m.K * 2 + args.batch * rows * 4
        return nb

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    nb = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    val = nb / dt / 1e9
    sample = f"fp64 oracle, first {rows} rows of each of the 7 linears per step, batch {args.batch}"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD + f", sampled rows ({rows} per linear)",
                                            "batch": args.batch},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_vbq(args):
    import torch
    from decode_vbq_gemv_b200 import vbq
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, R = args.batch, args.tile_rows

    # A step is one pass over the layer's seven linears, as launch groups. Fused (default): q/k/v share their
    # input and run as one launch, so do gate/up; o and down run alone (4 launches). --no-fuse: 7 launches.
    groups = [("q",), ("k",), ("v",), ("o",), ("gate",), ("up",), ("down",)] if args.no_fuse else GROUPS
    flags = 0 if args.no_overlap else vbq.VBQ_LAUNCH_OVERLAP

    class Group:
        pass

    layers = []   # per copy: list of Group
    for cp in range(args.copies):
        by_name = {m.name: m for m in layer_matrices(cp)}
        lin = []
        for names in groups:
            g = Group()
            g.name = "_".join(names)
            ms = [by_name[n] for n in names]
            g.mats = []
            g.R = R if R > 0 else vbq.suggest_tile_rows(sum(m.N for m in ms), ms[0].K,
                                                         torch.cuda.get_device_properties(dev).multi_processor_count)
            for m in ms:
                blob, _ = vbq.vbq_pack(m.N, m.K, g.R, m.widths, m.scales, m.codes)
                g.mats.append(vbq.DeviceMatrix(blob, dev, max_batch=B))
                del blob
            g.fused = vbq.FusedMatrices(g.mats, max_batch=B) if len(ms) > 1 else None
            xb = S.make_x(4, names[0], B, ms[0].K, layer=cp)
            g.xh = torch.from_numpy(xb.astype(np.int16)).view(torch.bfloat16).pin_memory()
            g.xd = g.xh.to(dev)
            g.yd = [torch.empty((B, m.N), dtype=torch.float32, device=dev) for m in ms]
            g.yh = [torch.empty((B, m.N), dtype=torch.float32).pin_memory() for m in ms]
            g.nbytes = sum(mt.nbytes for mt in g.mats) + B * ms[0].K * 2 + sum(B * m.N * 4 for m in ms)
            g.h = None
            g.x_from_device = False
            lin.append(g)
        # The MLP runs as a chain: the fused gate/up launch writes h = silu(gate) * up (bf16) through its SwiGLU
        # epilogue straight into the down projection's input.
        names = [g.name for g in lin]
        if not args.no_fuse and "gate_up" in names and "down" in names:
            gu, dn = lin[names.index("gate_up")], lin[names.index("down")]
            gu.h = dn.xd
            gu.nbytes += dn.xd.numel() * 2
            dn.x_from_device = True
        layers.append(lin)
    step_bytes = [sum(g.nbytes for g in lin) for lin in layers]

    def launch(g, st):
        if g.h is not None:
            g.fused.swiglu(g.xd, g.yd, g.h, flags, st)
        elif g.fused is not None:
            g.fused.matmul(g.xd, g.yd, flags, st)
        else:
            mat = g.mats[0]
            vbq.vbq_gemm_skinny_ex(mat.desc, mat.blob, g.xd, B, g.yd[0], mat.workspaces[B], flags, st)

    # One CUDA graph per layer copy, so that the timed region has no host launch gaps: device-resident step
    # and end-to-end step (pinned x -> device, the launches, y -> pinned host).
    stream = torch.cuda.Stream(dev)
    graphs, graphs_e2e = [], []
    with torch.cuda.stream(stream):
        for lin in layers:
            for g in lin:
                launch(g, stream)
        torch.cuda.synchronize()
        for lin in layers:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for g in lin:
                    launch(g, stream)
            graphs.append(gr)
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=stream):
                for g in lin:
                    if not g.x_from_device:
                        g.xd.copy_(g.xh, non_blocking=True)
                    launch(g, stream)
                    for yd, yh in zip(g.yd, g.yh):
                        yh.copy_(yd, non_blocking=True)
            graphs_e2e.append(g2)
    torch.cuda.synchronize()
    launches_per_step = len(groups)

    def timed(gs):
        for i in range(args.warmup):
            gs[i % args.copies].replay()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(args.steps):
                gs[i % args.copies].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return e0.elapsed_time(e1)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms = timed(graphs)
    clocks = sampler.stop()
    total_bytes = sum(step_bytes[i % args.copies] for i in range(args.steps))
    ms_max = allreduce_max(ms, world)
    value = total_bytes * world / (ms_max / 1e3) / 1e9
    launch_ms = ms / (args.steps * launches_per_step)
    launch_bytes = total_bytes / (args.steps * launches_per_step)

    # Per-launch-group kernel time: one graph of `reps` launches of that group, timed alone (copy 0).
    per_shape = {}
    reps = 20
    for g in layers[0]:
        with torch.cuda.stream(stream):
            gl = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gl, stream=stream):
                for _ in range(reps):
                    launch(g, stream)
            gl.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gl.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        per_shape[g.name] = {"us": us, "GBps": g.nbytes / (us / 1e6) / 1e9, "note": "same launch repeated (L2-warm)"}

    # End to end through host buffers.
    h2d = sum(g.xh.numel() * 2 for g in layers[0] if not g.x_from_device)
    d2h = sum(sum(y.numel() * 4 for y in g.yh) for g in layers[0])
    e2e_ms = allreduce_max(timed(graphs_e2e), world)
    e2e_val = total_bytes * world / (e2e_ms / 1e3) / 1e9
    n_launches = args.steps * launches_per_step

    if rank == 0:
        peak, peak_kind = peaks()
        achieved = launch_bytes / (launch_ms / 1e3) / 1e9
        cpu = cpu_baseline(B, args.cpu_budget) if (world == 1 and args.cpu_budget > 0) else None
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": B,
                       "tile_rows": {g.name: g.R for g in layers[0]},
                       "launch": ("plain" if args.no_overlap else "programmatic dependent launch (VBQ_LAUNCH_OVERLAP)")
                                 + ("; one launch per linear" if args.no_fuse
                                    else "; q/k/v fused (vbq_gemm_skinny_multi); gate/up fused with the SwiGLU "
                                         "epilogue (vbq_gemm_swiglu) writing the down projection's input; "
                                         "4 launches per layer"),
                       "weights": "seeded synthetic VBQ groups: P(1,2,4,8 bit) = (0.69,0.16,0.09,0.06), fp16 "
                                  "scales U(0.01,0.1), uniform codes; x ~ N(0,1) bf16",
                       "l2": f"inputs larger than L2: {args.copies} distinct layer copies in rotation "
                             f"({sum(step_bytes) / 1e6:.0f} MB of weights)",
                       "parallelism": f"replicas x{world}"},
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "peak_kind": peak_kind,
                         "kernel": f"vbq_kernel<{B}>",
                         "algorithmic_bytes_per_launch": launch_bytes, "avg_launch_us": launch_ms * 1e3},
            "per_launch_group": per_shape,
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": n_launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--batch", type=int, default=1, choices=(1, 2, 4, 8, 16))
    ap.add_argument("--impl", default="vbq", choices=("vbq", "reference"))
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--tile-rows", type=int, default=0,
                    help="tile rows for packing; 0: per launch group, vbq.suggest_tile_rows")
    ap.add_argument("--no-fuse", action="store_true",
                    help="one launch per linear instead of fusing the projections that share their input")
    ap.add_argument("--no-overlap", action="store_true",
                    help="plain launches instead of programmatic dependent launch between the linears")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds for the CPU-oracle baseline (0: skip)")
    ap.add_argument("--ref-rows", type=int, default=256, help="rows per linear per step for --impl reference")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_vbq(args)


if __name__ == "__main__":
    main()
