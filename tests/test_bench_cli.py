"""The bench's command-line contract, checked on the host: the oracle arm's JSON line, its rank handling and the
argument checks. The GPU arm runs only on a device."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=timeout, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "4"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "32 layers" in d["config"]["workload"] and "LM head" in d["config"]["workload"]


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "4"],
             {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_argument_checks():
    for bad in (["--warmup", "2"], ["--layers", "0"], ["--layers", "33"], ["--batch", "3"]):
        r = _run(bad, timeout=120)
        assert r.returncode == 2, (bad, r.stderr)


def _replica_rank(rank, world, port, times, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms_max = bench.allreduce_max(times[rank], world)
        out[rank] = (ms_max, bench.whole_job_gbps(1e9, 10, world, ms_max))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_replica_timing_is_the_slowest_rank_over_gloo():
    """The N > 1 host logic on CPU (gloo, 2 ranks): every rank sees the slowest rank's time, and the whole-job
    value counts both ranks' bytes over that time."""
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    times = [120.0, 200.0]
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_replica_rank, args=(2, port, times, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    for rank in (0, 1):
        ms_max, gbps = res[rank]
        assert ms_max == 200.0
        assert abs(gbps - 1e9 * 10 * 2 / 0.2 / 1e9) < 1e-9


def test_kernel_source_hash_ignores_comments_only():
    """The bench keys its ncu traffic capture to the device code of the kernel source (the part before the
    host-side launch-plan section): comment, blank-line and host-only edits keep the key, any device-code edit
    changes it."""
    import hashlib
    import re
    sys.path.insert(0, ROOT)
    import bench

    def key(src):
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        return hashlib.sha256("\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip()).encode()).hexdigest()

    with open(os.path.join(ROOT, "decode_vbq_gemv_b200", "csrc", "gemv.cu")) as f:
        src = f.read()
    marker = "// " + "-" * 90 + " launch plan"
    assert src.count(marker) == 1
    device = src[:src.index(marker)]
    assert "__global__" in device and "__global__" not in src[src.index(marker):]
    assert bench.kernel_source_sha256() == key(device)
    assert key("// note\nint a;\n\n/* block\n comment */ int b;  // tail\n") == key("int a;\n int b;\n")
    assert key("int a = 1;\n") != key("int a = 2;\n")


def test_gpu_arm_line_has_the_contract_keys():
    """The GPU arm's JSON line, built from stand-in measurements (no device): every contract key, a roofline
    whose achieved bytes per launch over the average launch time matches frac x peak, and valid JSON."""
    sys.path.insert(0, ROOT)
    import bench
    args = bench.make_parser().parse_args([])
    line = bench.vbq_line(
        args, world=1, value=690.0, ms_max=310.0, step_bytes=2.1286e9, weight_bytes=2.1219e9,
        tile_rows={"q_k_v": 224, "o": 512, "gate_up": 224, "down": 224, "head": 224}, launches_per_step=129,
        t_setup=9.0, launch_bytes=16.5e6, launch_ms=0.024, traffic=16.53e6, per_shape={}, e2e_val=340.0,
        h2d=794624, d2h=6419456, fp16={"value": 4100.0}, n_launches=12900,
        clocks={"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
        cpu={"value": 0.18, "unit": "GB/s", "cores": 16, "kind": "oracle", "sample": "s"},
        peak=6551.0, peak_kind="measured")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
                "cpu_baseline"):
        assert key in line, key
    assert line["steps"] == 100 and line["warmup"] == 5 and line["n_gpus"] == 1 and line["scaling"] == "weak"
    assert "32 layers" in line["config"]["workload"] and line["config"]["us_per_token"] == 3100.0
    r = line["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert abs(r["achieved"] - 16.5e6 / 0.024e-3 / 1e9) < 1e-6 and abs(r["frac"] * r["peak"] - r["achieved"]) < 1e-6
    assert set(line["e2e"]) == {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert "inputs larger than L2" in line["config"]["l2"]
    json.loads(json.dumps(line))
