"""Benchmark of the VBQ mixed-bit GEMV on B200: achieved HBM GB/s against the measured copy peak, and the
decode-step time.

Default workload: every linear of one batch-1 decode step of a 9B-shaped decoder (32 layers of q, k, v, o
4096x4096, gate, up 4096->14336 and down 14336->4096, then the LM head 4096->32000), with seeded synthetic
weights drawn from the VBQ paper's allocation (about 69% 1-bit groups and 1.85 mean bits in the layers, the
first block's MLP at 2.5 bits, the head at about 1.09 bits). The 2.1 GB of packed weights are about 17 times
the 126 MB L2, so every step streams them from HBM. One step is one token: 129 launches (per layer q/k/v
fused, o, gate/up fused with the SwiGLU epilogue feeding down's input, down; then the head).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--layers L] [--impl vbq|reference]
                    [--workload step|recipe|cfg4|pad512]

Other workloads: ``recipe`` is the same step under the paper's fixed deployment recipe (one width per
projection); ``cfg4`` times each 9B-shaped linear alone at batch 1..16; ``pad512`` compares an 8960-wide MLP
packed as is with its zero-padded 9216-wide form.

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
WORKLOAD = ("9B-shaped decode step: 32 layers of q,k,v,o 4096x4096, gate,up 4096->14336, down 14336->4096, "
            "plus the LM head 4096->32000")
SYNTH_CFG = 5   # seed family of the full decode-step stack in vbq_synth
RECIPE_CFG = 6  # seed family of the fixed-recipe stack (one width per projection, tiered LM head)
L2_BYTES = 126e6

# DRAM traffic of the kernel from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, cold L2) of the
# first five launches of `python bench.py --layers 1 --steps 3 --warmup 3 --cpu-budget 0`: layer 0's four launch
# groups and the LM head at batch 1, fused, with the tile rows below. The line reports it per launch, scaled to
# this step's algorithmic bytes per launch (traffic grows in proportion: the five launches span 4.5 to 41 MB, each
# at 0.999 to 1.019 times its algorithmic bytes), and only while the kernel source and the tile rows are the
# captured ones.
NCU_TRAFFIC = {"kernel_source_sha256": "cb7e1ff88cc5a332dfc239051f8e484ef24cadff79c3c4922100cc8b11ef8fd9",
               "tile_rows": {"q_k_v": 512, "o": 256, "gate_up": 1024, "down": 512, "head": 1024},
               "dram_bytes": 102416384, "algorithmic_bytes": 102225376, "launches": 5}


def kernel_source_sha256() -> str:
    """SHA-256 of the device code of the kernel source: the part of gemv.cu before its host-side launch-plan section,
    with comments and blank lines removed, so that neither a comment edit nor a host-only change (argument checks,
    plan queries) voids a DRAM-traffic capture. Tile rows, which do change the traffic, are checked separately.
    (A // or /* inside a string literal would be cut too; the kernel source has none.)"""
    import hashlib
    import re
    with open(os.path.join(ROOT, "decode_vbq_gemv_b200", "csrc", "gemv.cu")) as f:
        src = f.read()
    marker = "// " + "-" * 90 + " launch plan"
    if marker in src:
        src = src[:src.index(marker)]
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()


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
def step_matrices(layer: int, recipe: bool = False):
    """The seven linears of decoder layer `layer`: the paper's allocation (layer 0's MLP at the first-block mix),
    or the fixed deployment recipe (one width per projection)."""
    return S.cfg6_recipe_layer(layer) if recipe else S.cfg5_layer(layer)


def head_matrix(recipe: bool = False):
    return S.cfg6_recipe_head() if recipe else S.cfg5_head()


def sample_matrices(with_head: bool = True):
    """What the CPU oracle samples: layer 0's seven linears and the LM head."""
    return step_matrices(0) + ([S.cfg5_head()] if with_head else [])


def blob_bytes_of(m, R):
    from decode_vbq_gemv_b200 import vbq
    return vbq.vbq_packed_size(m.N, m.K, R, m.widths)


def cpu_baseline(B: int, budget_s: float = 12.0, matrices=None):
    """Times the fp64 oracle (as it stands) on a bounded sample of the workload: the first `rows` rows of each
    sampled linear, growing the sample until it takes about `budget_s` seconds or covers every row."""
    from oracle import oracle as O
    from decode_vbq_gemv_b200 import vbq
    mats = matrices or sample_matrices()
    threads = os.cpu_count() or 1
    xs = [S.make_x(SYNTH_CFG, m.name, B, m.K) for m in mats]
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
            "sample": f"fp64 oracle on the first {rows} rows of each of layer 0's 7 linears and the LM head, "
                      f"batch {B} ({dt:.2f} s); GB/s scaled from those rows' share of the packed bytes"}


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
    """The largest v over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbps(bytes_per_step: float, steps: int, world: int, ms_max: float) -> float:
    """Aggregate throughput of `world` replicas that each move `bytes_per_step` per step for `steps` steps, over
    the slowest rank's time."""
    return bytes_per_step * steps * world / (ms_max / 1e3) / 1e9


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------------------ arms
def run_reference(args):
    # The oracle arm runs on rank 0's host cores alone and needs no process group: the other ranks exit at once.
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from oracle import oracle as O
    mats = sample_matrices()
    xs = [S.make_x(SYNTH_CFG, m.name, args.batch, m.K) for m in mats]
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
    sample = (f"fp64 oracle, first {rows} rows of each of layer 0's 7 linears and the LM head per step, "
              f"batch {args.batch}")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD + f"; sampled rows ({rows} per linear)",
                                            "batch": args.batch},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def vbq_line(args, *, world, value, ms_max, step_bytes, weight_bytes, tile_rows, launches_per_step, t_setup,
             launch_bytes, launch_ms, traffic, per_shape, e2e_val, h2d, d2h, fp16, n_launches, clocks, cpu, peak,
             peak_kind) -> dict:
    """The GPU arm's JSON line from its measurements (no device work here)."""
    B = args.batch
    achieved = launch_bytes / (launch_ms / 1e3) / 1e9
    l2_bytes = 126e6
    workload = WORKLOAD if (args.layers == 32 and not args.no_head) else (
        f"{args.layers} of the 32 layers of the 9B-shaped decode step" + ("" if args.no_head else " plus the LM head"))
    if args.workload == "recipe":
        workload += ("; fixed deployment recipe: one width per projection (2-bit, first-block MLP 4-bit), LM head "
                     "tiered by token frequency to 1.18 mean bits")
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
        "config": {"workload": workload, "batch": B, "layers": args.layers, "lm_head": not args.no_head,
                   "us_per_token": 1e3 * ms_max / args.steps,
                   "weight_bytes_per_step": weight_bytes,
                   "tile_rows": tile_rows,
                   "launch": ("plain" if args.no_overlap else "programmatic dependent launch (VBQ_LAUNCH_OVERLAP)")
                             + ("; one launch per linear" if args.no_fuse
                                else "; q/k/v fused (vbq_gemm_skinny_multi); gate/up fused with the SwiGLU "
                                     "epilogue (vbq_gemm_swiglu) writing the down projection's input; "
                                     f"{launches_per_step} launches per step"),
                   "weights": ("seeded synthetic VBQ groups: P(1,2,4,8 bit) = (0.69,0.16,0.09,0.06), layer 0's "
                               "MLP (0.40,0.35,0.15,0.10), LM head tiered to ~1.09 bits; fp16 scales "
                               "U(0.01,0.1), uniform codes; x ~ N(0,1) bf16, one seeded x per linear")
                              if args.workload == "step" else
                              ("seeded synthetic VBQ groups under the fixed recipe: uniform 2-bit projections, 4-bit "
                               "layer-0 MLP, LM head rows 0.5/1.5/10/88% at 8/4/2/1 bits; fp16 scales U(0.01,0.1), "
                               "uniform codes; x ~ N(0,1) bf16, one seeded x per linear"),
                   "l2": (f"inputs larger than L2: {step_bytes / 1e6:.0f} MB of distinct weights streamed once per "
                          "step" if step_bytes > 2 * l2_bytes else
                          f"inputs NOT larger than L2 ({step_bytes / 1e6:.0f} MB): L2-warm, not an HBM figure"),
                   "setup_s": round(t_setup, 1),
                   "parallelism": f"replicas x{world}"},
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                     "traffic_source": (f"ncu capture of {NCU_TRAFFIC['launches']} launches (layer 0 and the LM "
                                        "head), scaled to this step's bytes per launch")
                                       if traffic is not None else None,
                     "kernel": f"vbq_kernel<{B}>",
                     "algorithmic_bytes_per_launch": launch_bytes, "avg_launch_us": launch_ms * 1e3},
        "per_launch_group": per_shape,
        "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "fp16_cublas_reference": fp16,
        "gpu_launches": n_launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }


def run_vbq(args):
    import concurrent.futures as cf
    import torch
    from decode_vbq_gemv_b200 import vbq
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, R = args.batch, args.tile_rows
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    # A step is one token: per layer the seven linears as launch groups, then the LM head. Fused (default): q/k/v
    # share their input and run as one launch, so do gate/up; o and down run alone (4 launches per layer).
    # --no-fuse: 7 launches per layer.
    groups = [("q",), ("k",), ("v",), ("o",), ("gate",), ("up",), ("down",)] if args.no_fuse else GROUPS

    def tile_rows(ms):
        return R if R > 0 else vbq.suggest_tile_rows(sum(m.N for m in ms), ms[0].K, sms)

    recipe = args.workload == "recipe"
    xcfg = RECIPE_CFG if recipe else SYNTH_CFG

    def prepare(layer):
        """Host side of one layer (or the head, layer -1): seeded matrices, packed; logical arrays dropped."""
        mats = [head_matrix(recipe)] if layer < 0 else step_matrices(layer, recipe)
        by_name = {m.name: m for m in mats}
        out = []
        for names in ([("head",)] if layer < 0 else groups):
            ms = [by_name[n] for n in names]
            rt = tile_rows(ms)
            blobs = [vbq.vbq_pack(m.N, m.K, rt, m.widths, m.scales, m.codes)[0] for m in ms]
            x = S.make_x(xcfg, names[0], B, ms[0].K, layer=max(layer, 0))
            out.append((names, rt, [(m.N, m.K) for m in ms], blobs, x))
        return layer, out

    class Group:
        pass

    def upload(layer, prepared):
        lin = []
        for names, rt, shapes, blobs, xb in prepared:
            g = Group()
            g.name = ("head" if layer < 0 else f"L{layer}.") + ("" if layer < 0 else "_".join(names))
            g.R = rt
            g.shapes = shapes
            g.mats = [vbq.DeviceMatrix(bl, dev, max_batch=B) for bl in blobs]
            g.fused = vbq.FusedMatrices(g.mats, max_batch=B) if len(g.mats) > 1 else None
            g.xb = xb
            g.K = shapes[0][1]
            g.nbytes = sum(mt.nbytes for mt in g.mats) + B * g.K * 2 + sum(B * N * 4 for N, _ in shapes)
            g.h = None
            g.x_from_device = False
            lin.append(g)
        # The MLP runs as a chain: the fused gate/up launch writes h = silu(gate) * up (bf16) through its SwiGLU
        # epilogue straight into the down projection's input.
        names = [g.name.split(".")[-1] for g in lin]
        if "gate_up" in names and "down" in names:
            gu, dn = lin[names.index("gate_up")], lin[names.index("down")]
            dn.x_from_device = True
            gu.h_of = dn
            gu.nbytes += B * dn.K * 2
        return lin

    # Host preparation runs on a few threads (the packer and most of the generator release the GIL); device
    # uploads stay on this thread, in layer order.
    order = list(range(args.layers)) + ([-1] if not args.no_head else [])
    step = []
    t_setup = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=min(4, os.cpu_count() or 1)) as pool:
        for layer, prepared in pool.map(prepare, order):
            step.extend(upload(layer, prepared))
    # Activations and outputs live in one device buffer each, so that the end-to-end step moves them with one
    # copy per direction from and to one pinned host buffer each. A down projection's input is the SwiGLU output
    # of its gate/up launch, produced on the device: it has a buffer of its own and is not copied.
    x_off, n_x = {}, 0
    for i, g in enumerate(step):
        if not g.x_from_device:
            x_off[i] = n_x
            n_x += B * g.K
    n_y = sum(B * N for g in step for N, _ in g.shapes)
    X_h = torch.empty(n_x, dtype=torch.bfloat16).pin_memory()
    X_d = torch.empty(n_x, dtype=torch.bfloat16, device=dev)
    Y_h = torch.empty(n_y, dtype=torch.float32).pin_memory()
    Y_d = torch.empty(n_y, dtype=torch.float32, device=dev)
    yo = 0
    for i, g in enumerate(step):
        if g.x_from_device:
            g.xd = torch.empty((B, g.K), dtype=torch.bfloat16, device=dev)
        else:
            o = x_off[i]
            X_h[o:o + B * g.K].copy_(torch.from_numpy(g.xb.astype(np.int16).reshape(-1)).view(torch.bfloat16))
            g.xd = X_d[o:o + B * g.K].view(B, g.K)
        g.yd = []
        for N, _ in g.shapes:
            g.yd.append(Y_d[yo:yo + B * N].view(B, N))
            yo += B * N
        del g.xb
    for g in step:
        if hasattr(g, "h_of"):
            g.h = g.h_of.xd
    X_d.copy_(X_h)
    t_setup = time.perf_counter() - t_setup
    step_bytes = sum(g.nbytes for g in step)
    flags = 0 if args.no_overlap else vbq.VBQ_LAUNCH_OVERLAP

    def launch(g, st):
        if g.h is not None:
            g.fused.swiglu(g.xd, g.yd, g.h, flags, st)
        elif g.fused is not None:
            g.fused.matmul(g.xd, g.yd, flags, st)
        else:
            mat = g.mats[0]
            vbq.vbq_gemm_skinny_ex(mat.desc, mat.blob, g.xd, B, g.yd[0], mat.workspaces[B], flags, st)

    # One CUDA graph per step, so that the timed region has no host launch gaps: the device-resident step and
    # the end-to-end step (each linear's x from pinned host memory to the device, the launches, every y back).
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for g in step:
            launch(g, stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for g in step:
                launch(g, stream)
        graph_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_e2e, stream=stream):
            X_d.copy_(X_h, non_blocking=True)
            for g in step:
                launch(g, stream)
            Y_h.copy_(Y_d, non_blocking=True)
    torch.cuda.synchronize()
    launches_per_step = len(step)

    def timed(gr):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                gr.replay()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                gr.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return e0.elapsed_time(e1)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms = timed(graph)
    clocks = sampler.stop()
    ms_max = allreduce_max(ms, world)
    value = whole_job_gbps(step_bytes, args.steps, world, ms_max)
    launch_ms = ms / (args.steps * launches_per_step)
    launch_bytes = step_bytes / launches_per_step

    # Per launch group of one representative layer (layer 1 when there is one: layer 0's MLP uses the first-block
    # mix) and the head: one graph of `reps` launches of that group alone, L2-warm.
    rep_layer = "L1." if args.layers > 1 else "L0."
    per_shape = {}
    reps = 20
    for g in step:
        if not (g.name.startswith(rep_layer) or g.name == "head"):
            continue
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
    h2d = X_h.numel() * 2
    d2h = Y_h.numel() * 4
    e2e_ms = allreduce_max(timed(graph_e2e), world)
    e2e_val = whole_job_gbps(step_bytes, args.steps, world, e2e_ms)
    n_launches = args.steps * launches_per_step

    # Reference point: the same linears as dense FP16 weights through cuBLAS (torch.matmul, one launch per linear),
    # captured in one CUDA graph per step and timed the same way. Weights and activations are random on the device.
    fp16 = None
    if not args.no_fp16_ref:
        shapes = [sh for g in step for sh in g.shapes]
        Ws = [torch.empty((N, K), dtype=torch.float16, device=dev).normal_(0.0, 0.02) for N, K in shapes]
        xs = [torch.randn((B, K), dtype=torch.float16, device=dev) for _, K in shapes]
        ys = [torch.empty((B, N), dtype=torch.float16, device=dev) for N, _ in shapes]
        with torch.cuda.stream(stream):
            for W, xx, yy in zip(Ws, xs, ys):
                torch.matmul(xx, W.t(), out=yy)
            torch.cuda.synchronize()
            g16 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g16, stream=stream):
                for W, xx, yy in zip(Ws, xs, ys):
                    torch.matmul(xx, W.t(), out=yy)
        torch.cuda.synchronize()
        ms16 = allreduce_max(timed(g16), world)
        b16 = sum(N * K * 2 + B * K * 2 + B * N * 2 for N, K in shapes)
        fp16 = {"value": whole_job_gbps(b16, args.steps, world, ms16), "unit": UNIT,
                "us_per_token": 1e3 * ms16 / args.steps, "weight_bytes_per_step": sum(N * K * 2 for N, K in shapes),
                "launch": f"torch.matmul (cuBLAS), {len(shapes)} launches per step in one CUDA graph",
                "vbq_speedup": ms16 / ms_max}
        del g16, Ws, xs, ys
        torch.cuda.empty_cache()

    traffic = None
    if (B == 1 and not args.no_fuse and {g.name.split(".")[-1]: g.R for g in step} == NCU_TRAFFIC["tile_rows"]
            and kernel_source_sha256() == NCU_TRAFFIC["kernel_source_sha256"]):
        traffic = launch_bytes * NCU_TRAFFIC["dram_bytes"] / NCU_TRAFFIC["algorithmic_bytes"]

    # Batch sweep (outside the timed step): the 14336x4096 gate linear alone at batch 1-16, streaming from HBM, so
    # that the step's JSON line also carries the skinny-GEMM batch sizes.
    sweep = None
    if not args.no_batch_sweep:
        speak, _ = peaks()
        res, _ = rotation_sweep(args, dev, stream, sms, speak, "gate", (1, 2, 4, 8, 16))
        sweep = {"workload": "gate 14336x4096 alone at each batch size, >= 4x L2 of distinct copies in rotation, "
                             "best of 3 graph replays",
                 "results": {k: {"us": round(v["us"], 2), "GBps": round(v["GBps"], 1), "frac": round(v["frac"], 4),
                                 "status": v["status"]} for k, v in res.items()}}
    if rank == 0:
        peak, peak_kind = peaks()
        cpu = cpu_baseline(B, args.cpu_budget) if (world == 1 and args.cpu_budget > 0) else None
        line = vbq_line(args, world=world, value=value, ms_max=ms_max, step_bytes=step_bytes,
                        weight_bytes=sum(sum(mt.nbytes for mt in g.mats) for g in step),
                        tile_rows={g.name.split(".")[-1]: g.R for g in step}, launches_per_step=launches_per_step,
                        t_setup=t_setup, launch_bytes=launch_bytes, launch_ms=launch_ms, traffic=traffic,
                        per_shape=per_shape, e2e_val=e2e_val, h2d=h2d, d2h=d2h, fp16=fp16, n_launches=n_launches,
                        clocks=clocks, cpu=cpu, peak=peak, peak_kind=peak_kind)
        line["batch_sweep"] = sweep
        print(json.dumps(line), flush=True)
    del graph, graph_e2e
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


# ------------------------------------------------------------------------------------------- config 4
CFG4 = (("q", 4096, 4096), ("gate", 14336, 4096), ("down", 4096, 14336))


def rotation_sweep(args, dev, stream, sms, peak, name, batches):
    """One config-4 matrix timed alone at each batch size: M distinct device copies of the packed matrix, together
    at least 4x the L2, launched round-robin in one CUDA graph (chained by programmatic dependent launch), so every
    launch streams its weights from HBM; time per launch = replay time / M, the best of three replays after
    warm-up. Returns ({"name NxK B=b": {...}}, launches)."""
    import torch
    from decode_vbq_gemv_b200 import vbq
    N, K = dict((n, (a, b)) for n, a, b in CFG4)[name]
    m = S.cfg4((name,))[0]
    R = args.tile_rows if args.tile_rows > 0 else vbq.suggest_tile_rows(N, K, sms)
    blob, desc = vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)
    stride = (blob.size + 255) // 256 * 256
    M = max(2, int(np.ceil(4 * L2_BYTES / stride)))
    copies = torch.empty(M * stride, dtype=torch.uint8, device=dev)
    first = torch.from_numpy(blob).to(dev)
    for c in range(M):
        copies[c * stride:c * stride + blob.size].copy_(first)
    del first
    results, n_launches = {}, 0
    for B in batches:
        ws_bytes = vbq.vbq_workspace_size(desc, B)
        ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        x = torch.from_numpy(S.make_x(4, name, B, K).astype(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty((B, N), dtype=torch.float32, device=dev)
        flags = 0 if args.no_overlap else vbq.VBQ_LAUNCH_OVERLAP
        with torch.cuda.stream(stream):
            def run_all():
                for c in range(M):
                    vbq.vbq_gemm_skinny_ex(desc, copies[c * stride:c * stride + blob.size], x, B, y, ws, flags,
                                           stream)
            run_all()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run_all()
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize()
            best = None
            for _ in range(3):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                t = e0.elapsed_time(e1) / M
                best = t if best is None else min(best, t)
            n_launches += 3 * M   # the timed replays
        status = int(ws[ws_bytes - 4:ws_bytes].cpu().numpy().view(np.uint32)[0]) if ws_bytes >= 4 else 0
        nbytes = blob.size + B * K * 2 + B * N * 4
        gbps = nbytes / (best / 1e3) / 1e9
        results[f"{name} {N}x{K} B={B}"] = {"us": best * 1e3, "GBps": gbps, "frac": gbps / peak, "tile_rows": R,
                                            "copies": M, "status": status}
        del g, ws
    del copies
    torch.cuda.empty_cache()
    return results, n_launches


def run_cfg4(args):
    """The 9B-shaped single linears (q/k/v/o 4096x4096, gate/up 4096->14336, down 14336->4096) at batch 1, 2, 4,
    8 and 16, each timed alone: M distinct device copies of the packed matrix, together at least 4x the L2, are
    launched round-robin in one CUDA graph (chained by programmatic dependent launch), so every launch streams its
    weights from HBM; time per launch = replay time / M, the best of three replays after warm-up. The headline
    value is the batch-1 GB/s of the two 15.7 MB MLP matrices (their mean); every (matrix, batch) is in `cfg4`."""
    import torch
    from decode_vbq_gemv_b200 import vbq
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak, peak_kind = peaks()
    stream = torch.cuda.Stream(dev)
    batches = (1, 2, 4, 8, 16) if args.batch == 1 else (args.batch,)
    results, n_launches, t_setup = {}, 0, time.perf_counter()
    sampler = ClockSampler(local)
    sampler.start()
    for name, N, K in CFG4:
        if args.matrices and name not in args.matrices.split(","):
            continue
        res, nl = rotation_sweep(args, dev, stream, sms, peak, name, batches)
        results.update(res)
        n_launches += nl
    clocks = sampler.stop()
    t_setup = time.perf_counter() - t_setup
    head = [results[f"{n} {N}x{K} B=1"]["GBps"] for n, N, K in CFG4
            if n in ("gate", "down") and f"{n} {N}x{K} B=1" in results] or [results[k]["GBps"] for k in results]
    value = float(np.mean(head))
    if rank == 0:
        line = {"metric": METRIC, "value": value * world, "unit": UNIT, "n_gpus": world, "steps": 3,
                "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
                "config": {"workload": "9B-shaped single linears (q 4096x4096, gate 4096->14336, down 14336->4096), "
                                       "each alone with >= 4x L2 of distinct copies in rotation",
                           "batch": list(batches), "l2": "inputs larger than L2: copies in rotation",
                           "parallelism": f"replicas x{world}"},
                "pct_of_peak": 100.0 * value / peak,
                "roofline": {"bound": "hbm", "achieved": value, "peak": peak, "unit": "GB/s", "frac": value / peak,
                             "traffic": None, "peak_kind": peak_kind,
                             "kernel": "vbq_kernel<B> (CUDA-core units at batch 1, 2, 4; mma.sync units at 8, 16)"},
                "cfg4": results, "gpu_launches": n_launches, "clocks": clocks, "setup_s": round(t_setup, 1),
                "e2e": None, "cpu_baseline": None}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


def run_pad512(args):
    """The 8960-wide MLP (gate/up 8960x1536 with the fused SwiGLU epilogue, then down 1536x8960 on h), packed as
    is and zero-padded to an intermediate width of 9216 (a multiple of 512), at batch 1 and 16 (or --batch). Each
    form is timed like cfg4: M distinct device copies of its three blobs, together at least 4x the L2, run
    round-robin in one CUDA graph; time per MLP = replay time / M, the best of three replays. GB/s counts the
    blobs, x, both y, h and the down output of the logical (unpadded) problem for both forms, so the padded form
    pays for its extra bytes."""
    import torch
    from decode_vbq_gemv_b200 import vbq
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak, peak_kind = peaks()
    stream = torch.cuda.Stream(dev)
    batches = (1, 16) if args.batch == 1 else (args.batch,)
    gm, um, dm = S.cfg7_mlp()
    I, H, I_pad = gm.N, gm.K, 9216
    R = args.tile_rows if args.tile_rows > 0 else vbq.suggest_tile_rows(I, H, sms)
    Rd = args.tile_rows if args.tile_rows > 0 else vbq.suggest_tile_rows(H, I, sms)
    results, n_launches, t_setup = {}, 0, time.perf_counter()
    sampler = ClockSampler(local)
    sampler.start()
    for pad in (False, True):
        if pad:
            packed = [vbq.vbq_pack_padded(m.N, m.K, R, m.widths, m.scales, m.codes, I_pad, H) for m in (gm, um)]
            packed.append(vbq.vbq_pack_padded(dm.N, dm.K, Rd, dm.widths, dm.scales, dm.codes, H, I_pad))
        else:
            packed = [vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes) for m in (gm, um)]
            packed.append(vbq.vbq_pack(dm.N, dm.K, Rd, dm.widths, dm.scales, dm.codes))
        blobs, descs = [b for b, _ in packed], [d for _, d in packed]
        strides = [(b.size + 255) // 256 * 256 for b in blobs]
        unit = sum(strides)
        M = max(2, int(np.ceil(4 * L2_BYTES / unit)))
        copies = torch.empty(M * unit, dtype=torch.uint8, device=dev)
        offs = [0, strides[0], strides[0] + strides[1]]
        for i, b in enumerate(blobs):
            src = torch.from_numpy(b).to(dev)
            for c in range(M):
                copies[c * unit + offs[i]:c * unit + offs[i] + b.size].copy_(src)
        Np = descs[0].N
        for B in batches:
            ws_gu = torch.zeros(vbq.vbq_workspace_size_swiglu(descs[0], descs[1], B), dtype=torch.uint8, device=dev)
            ws_d = torch.zeros(max(vbq.vbq_workspace_size(descs[2], B), 16), dtype=torch.uint8, device=dev)
            x = torch.from_numpy(S.make_x(7, "gate", B, H).astype(np.int16)).view(torch.bfloat16).to(dev)
            yg = torch.empty((B, Np), dtype=torch.float32, device=dev)
            yu = torch.empty((B, Np), dtype=torch.float32, device=dev)
            h = torch.empty((B, Np), dtype=torch.bfloat16, device=dev)
            yd = torch.empty((B, H), dtype=torch.float32, device=dev)
            flags = 0 if args.no_overlap else vbq.VBQ_LAUNCH_OVERLAP

            def blob(c, i):
                return copies[c * unit + offs[i]:c * unit + offs[i] + blobs[i].size]

            with torch.cuda.stream(stream):
                def run_all():
                    for c in range(M):
                        vbq.vbq_gemm_swiglu(descs[0], descs[1], blob(c, 0), blob(c, 1), x, B, yg, yu, h, ws_gu,
                                            flags, stream)
                        vbq.vbq_gemm_skinny_ex(descs[2], blob(c, 2), h, B, yd, ws_d, flags, stream)
                run_all()
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    run_all()
                for _ in range(args.warmup):
                    g.replay()
                torch.cuda.synchronize()
                best = None
                for _ in range(3):
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                    torch.cuda.synchronize()
                    t = e0.elapsed_time(e1) / M
                    best = t if best is None else min(best, t)
                n_launches += 2 * 3 * M   # the timed replays
            logical_bytes = sum(vbq.vbq_packed_size(m.N, m.K, r, m.widths) for m, r in ((gm, R), (um, R), (dm, Rd)))
            nbytes = logical_bytes + B * H * 2 + 2 * B * I * 4 + B * I * 2 + B * I * 2 + B * H * 4
            gbps = nbytes / (best / 1e3) / 1e9
            results[f"{'padded to 9216' if pad else 'unpadded 8960'} B={B}"] = {
                "us": best * 1e3, "GBps": gbps, "frac": gbps / peak, "blob_bytes": int(sum(b.size for b in blobs)),
                "copies": M, "tile_rows": [R, Rd]}
            del g, ws_gu, ws_d
        del copies
        torch.cuda.empty_cache()
    clocks = sampler.stop()
    t_setup = time.perf_counter() - t_setup
    value = results["unpadded 8960 B=1"]["GBps"] if 1 in batches else next(iter(results.values()))["GBps"]
    if rank == 0:
        line = {"metric": METRIC, "value": value * world, "unit": UNIT, "n_gpus": world, "steps": 3,
                "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
                "config": {"workload": "8960-wide MLP (gate/up 8960x1536 + SwiGLU, down 1536x8960), unpadded and "
                                       "zero-padded to 9216, >= 4x L2 of distinct copies in rotation",
                           "batch": list(batches), "l2": "inputs larger than L2: copies in rotation",
                           "parallelism": f"replicas x{world}"},
                "roofline": {"bound": "hbm", "achieved": value, "peak": peak, "unit": "GB/s", "frac": value / peak,
                             "traffic": None, "peak_kind": peak_kind, "kernel": "vbq_kernel<B>"},
                "pad512": results, "gpu_launches": n_launches, "clocks": clocks, "setup_s": round(t_setup, 1),
                "e2e": None, "cpu_baseline": None}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


def make_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--batch", type=int, default=1, choices=(1, 2, 4, 8, 16))
    ap.add_argument("--impl", default="vbq", choices=("vbq", "reference"))
    ap.add_argument("--workload", default="step", choices=("step", "recipe", "cfg4", "pad512"),
                    help="step: the 9B-shaped decode step at the paper's allocation (default); recipe: the same step "
                         "under the fixed deployment recipe; cfg4: each 9B-shaped linear alone at batch 1..16, "
                         "rotating copies larger than L2; pad512: an 8960-wide MLP unpadded and zero-padded to "
                         "9216")
    ap.add_argument("--layers", type=int, default=32, help="decoder layers in the step (1..32)")
    ap.add_argument("--no-head", action="store_true", help="leave the LM head out of the step")
    ap.add_argument("--no-fp16-ref", action="store_true",
                    help="skip the dense FP16 cuBLAS reference point (same shapes, same timing)")
    ap.add_argument("--tile-rows", type=int, default=0,
                    help="tile rows for packing; 0: per launch group, vbq.suggest_tile_rows")
    ap.add_argument("--no-fuse", action="store_true",
                    help="one launch per linear instead of fusing the projections that share their input")
    ap.add_argument("--no-overlap", action="store_true",
                    help="plain launches instead of programmatic dependent launch between the linears")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds for the CPU-oracle baseline (0: skip)")
    ap.add_argument("--ref-rows", type=int, default=256, help="rows per linear per step for --impl reference")
    ap.add_argument("--no-batch-sweep", action="store_true",
                    help="step workloads: skip the batch 1-16 sweep of the 14336x4096 linear after the timed step")
    ap.add_argument("--matrices", default="",
                    help="cfg4 only: comma-separated subset of q, gate, down (default: all three)")
    return ap


def main():
    ap = make_parser()
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if not 1 <= args.layers <= 32:
        ap.error("--layers must be in 1..32")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "cfg4":
        run_cfg4(args)
    elif args.workload == "pad512":
        run_pad512(args)
    else:
        run_vbq(args)


if __name__ == "__main__":
    main()
