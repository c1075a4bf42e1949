"""Benchmark of the DualQuant hot path on B200.

One step = one full-model dual-scale solve of the Llama-3.1-8B-shaped layer set (32 blocks x
q/k/v/o/gate/up/down, 6.98e9 bf16 weights, NVFP4, 16 BCD iterations) through
dq_solve_batched, followed by the activation rescale + NVFP4 quantization of an 8192 x 4096
activation with the column scales of that step's block-0 k_proj (dq_act_quant).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--split]

The JSON line also carries, measured in the same run on one GPU: the activation quantizer
alone (NVFP4 and INT4 g=128, calls back to back over inputs larger than L2 and one call behind
an L2 flush, SQNR with and without c), the Llama-3.2-1B-shaped MXFP4 and Llama-2-7B-shaped
MXINT4 layer sets in their own shapes, and the convergence of block 0 of the three layer sets
(the Q-change trace and the normalised MSE).

Other measurements (same JSON conventions): --fmt/--update/--qchange (other formats and the
ablation modes of the headline step), --act (the activation quantizer alone), --gemm (the
W4A4 GEMM consumer), --cpu-plan (the CPU oracle over the configurations' samples).

Multi-GPU (torchrun): by default every rank solves its own layer set (different seeds; weak
scaling); with --split the ranks share ONE layer set, matrices assigned by element count
(strong scaling, full-model solve time = the slowest rank). No collective on the data path;
timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "BCD weight elems×iters/s and full-model solve s; % of B200 HBM roofline"
UNIT = "elem*iter/s"
CFG_ID = 3
FMT_SPECS = {"NVFP4": ("NVFP4", 16), "MXFP4": ("MXFP4", 32), "MXINT4": ("MXINT4", 32),
             "INT4": ("INT4", 128), "INT4_G64": ("INT4", 64), "INT8": ("INT8", 128),
             "MXINT8": ("MXINT8", 32)}

KERNEL_SOURCES = ("dq_solve.cu", "dq_solve_kernel.cuh", "dq_device.cuh", "dq_internal.h")
PROFILE_JSON = os.path.join(ROOT, "profiles", "solve_kernel_8b_nvfp4.json")


def solve_bytes_per_elem(fmt: str, T: int, esize: int = 2) -> float:
    """Algorithmic bytes per weight element of one solve-kernel run: W read and the block-scale
    state read and written at its encoded width in every iteration, the codes written once."""
    kind, B = FMT_SPECS[fmt]
    scb = 2 if kind in ("INT4", "INT8") else 1
    code = 1.0 if kind in ("INT8", "MXINT8") else 0.5
    return T * (esize + 2.0 * scb / B) + code


def prepass_bytes_per_elem(fmt: str, esize: int = 2) -> float:
    """The NVFP4 tensor-scale pre-pass reads W once; the other formats have none."""
    return float(esize) if FMT_SPECS[fmt][0] == "NVFP4" else 0.0


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "calibration_free_dual_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_solve_kernel():
    """The ncu figures of the solve kernel (profiles/solve_kernel_8b_nvfp4.json), or {} when
    the kernel's sources have changed since that capture."""
    if not os.path.exists(PROFILE_JSON):
        return {}
    with open(PROFILE_JSON) as fh:
        d = json.load(fh)
    return d if d.get("source_sha256_16") == kernel_source_hash() else {}


def workload_name(count: int, elems: int, T: int, fmt: str = "NVFP4", update: str = "both",
                  qchange: bool = False) -> str:
    extra = ""
    if update != "both":
        extra += ", %s-scale updates only" % ("row" if update == "row" else "column")
    if qchange:
        extra += ", with the Q-change trace"
    return ("Llama-3.1-8B-shaped layer set (%d matrices, %.3e bf16 weights per GPU), %s, %d "
            "BCD iterations%s + activation rescale/%s quant 8192x4096"
            % (count, elems, fmt, T, extra, fmt))


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--blocks", type=int, default=None,
                    help="solve only the first B blocks (profiling runs; not a bench value)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fmt", default="NVFP4",
                    choices=["NVFP4", "MXFP4", "MXINT4", "INT4", "INT4_G64", "INT8", "MXINT8"],
                    help="format of the solve and the activation quantization (default: the "
                         "headline NVFP4 workload)")
    ap.add_argument("--update", default="both", choices=["both", "row", "col"],
                    help="ablation: update both scales (the method), only r or only c")
    ap.add_argument("--qchange", action="store_true",
                    help="also record the per-iteration Q-change trace")
    ap.add_argument("--gemm", action="store_true",
                    help="time the W4A4 GEMM consumer instead: the 7 projections of block 0 "
                         "(solved in NVFP4) against --gemm-tokens activation rows")
    ap.add_argument("--gemm-tokens", type=int, default=8192)
    ap.add_argument("--split", action="store_true",
                    help="multi-GPU: split one layer set over the ranks by matrix (strong "
                         "scaling) instead of one layer set per rank")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the activation, 1B/7B layer-set and convergence records")
    ap.add_argument("--cpu-plan", action="store_true",
                    help="run the CPU oracle over the configurations' samples instead")
    ap.add_argument("--act", action="store_true",
                    help="time the activation rescale + quantization alone instead: 8192 x "
                         "4096 bf16 activations with a k_proj's c, NVFP4 and INT4 g=128, L2 "
                         "flushed before every call; SQNR with and without c")
    return ap.parse_args()


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------------- distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        # short enough that ranks waiting on a lost peer end with an error well before any
        # outer limit; long enough for the per-rank input generation before the first barrier
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=240))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------- CPU oracle
_ORACLE_FMT = {"NVFP4": ("NVFP4", 16), "MXFP4": ("MXFP4", 32), "MXINT4": ("MXINT4", 32),
               "INT4": ("INT4", 128), "INT4_G64": ("INT4", 64), "INT8": ("INT8", 128),
               "MXINT8": ("MXINT8", 32)}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def host_ram_gb() -> float:
    try:
        return os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES") / 1e9
    except (ValueError, OSError, AttributeError):  # pragma: no cover
        return 16.0


def oracle_pool_size(n_tasks: int, gb_per_worker: float = 3.0) -> int:
    """Workers for the oracle: min(host cores, host RAM / gb_per_worker, tasks)."""
    return max(1, min(host_cores(), int(host_ram_gb() // gb_per_worker), n_tasks))


def run_oracle_tasks(tasks, workers: int) -> dict:
    """Oracle solves over a pool of `workers` processes (oracle/pool.py, run as its own
    program: the workers import only NumPy and the oracle, never torch or CUDA)."""
    from oracle import pool
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "tasks.npz")
        pool.save_tasks(path, tasks)
        # one thread per worker process: the pool is the parallelism
        env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1",
                   MKL_NUM_THREADS="1")
        r = subprocess.run([sys.executable, "-m", "oracle.pool", path, str(workers)],
                           cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                           text=True, check=True)
    return json.loads(r.stdout.strip().splitlines()[-1])


def oracle_task(W, fmt: str, iters: int, amax=None, update: str = "both"):
    kind, group = _ORACLE_FMT[fmt]
    return (W, kind, group, iters, amax if kind == "NVFP4" else None, update)


def cpu_sample(mats, fmt: str, iters: int, cols: int, per_matrix: int, update="both"):
    """The oracle as it stands on the host cores: the first `per_matrix` strips of `cols`
    columns of each matrix (each solved with its whole matrix's amax), over a process pool."""
    tasks = []
    for W in mats:
        amax = float(np.max(np.abs(W)))
        for k in range(per_matrix):
            tasks.append(oracle_task(np.ascontiguousarray(W[:, k * cols:(k + 1) * cols]), fmt,
                                     iters, amax, update))
    return run_oracle_tasks(tasks, oracle_pool_size(len(tasks)))


def block0_host(cfg):
    """Block 0 of a layer set drawn on the host (binary64 copies of the bf16 weights)."""
    return [wl.weight_host(cfg, b, p).float().numpy().astype(np.float64)
            for b, p, _, _ in cfg.layer_set() if b == 0]


CPU_SAMPLE_COLS, CPU_SAMPLE_STRIPS = 64, 2


def cpu_baseline_record(fmt: str = "NVFP4", update: str = "both") -> dict:
    """Bounded sample of the headline workload: block 0's seven projections of the 8B layer
    set, two 64-column strips each, 16 iterations, over a pool of min(cores, RAM / 3 GB)
    workers; plus the single-core rate on the 512 x 512 fp32 INT4 tile."""
    cfg = wl.CONFIGS[CFG_ID]
    r = cpu_sample(block0_host(cfg), fmt, cfg.iters, CPU_SAMPLE_COLS, CPU_SAMPLE_STRIPS, update)
    c1 = wl.CONFIGS[1]
    W1 = wl.weight_host(c1, 0, 0).numpy().astype(np.float64)
    r1 = run_oracle_tasks([oracle_task(W1, "INT4", c1.iters)], 1)
    return {"value": r["work"] / r["wall_s"], "unit": UNIT, "cores": r["workers"],
            "kind": "oracle",
            "sample": "block 0 of the 8B layer set, 7 projections x %d strips of %d columns "
                      "(%d oracle solves, %.3g elem*iter), %s, %d iterations, %d worker "
                      "processes (host: %d cores); %.2f s wall, %.1f s of CPU work"
                      % (CPU_SAMPLE_STRIPS, CPU_SAMPLE_COLS, r["tasks"], r["work"], fmt,
                         cfg.iters, r["workers"], host_cores(), r["wall_s"], r["cpu_s"]),
            "per_core_value": r["work"] / r["cpu_s"],
            "single_core_512x512_int4": {"value": r1["work"] / r1["wall_s"], "unit": UNIT,
                                         "seconds": r1["wall_s"]}}


def run_reference(args, world, rank):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload."""
    if rank != 0:
        return
    cfg = wl.CONFIGS[CFG_ID]
    mats = block0_host(cfg)
    desc = ("block 0 of the 8B layer set, 7 projections x %d strips of %d columns, NVFP4, "
            "16 iterations, over a process pool" % (CPU_SAMPLE_STRIPS, CPU_SAMPLE_COLS))
    for _ in range(args.warmup):
        cpu_sample(mats, "NVFP4", cfg.iters, CPU_SAMPLE_COLS, CPU_SAMPLE_STRIPS)
    works, walls, P = 0, 0.0, 1
    for _ in range(args.steps):
        r = cpu_sample(mats, "NVFP4", cfg.iters, CPU_SAMPLE_COLS, CPU_SAMPLE_STRIPS)
        works += r["work"]
        walls += r["wall_s"]
        P = r["workers"]
    value = works / walls
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * walls / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(len(cfg.layer_set()), cfg.elements(), cfg.iters),
                   "sample": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": P, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_cpu_plan(args):
    """The CPU baseline plan: the single-core rate on the 512 x 512 tile; the whole 512 x 512
    tile, 1B layer set and activation workload; blocks {0, L/2, L-1} of the 8B and 7B layer
    sets (all seven projections), each over a process pool, wall times measured."""
    from oracle import formats as F
    from oracle import solver as S
    from oracle.actquant import act_quant as ora_act
    out = {"host_cores": host_cores(), "host_ram_gb": round(host_ram_gb(), 1)}
    t_all = time.perf_counter()
    c1 = wl.CONFIGS[1]
    W1 = wl.weight_host(c1, 0, 0).numpy().astype(np.float64)
    r1 = run_oracle_tasks([oracle_task(W1, "INT4", c1.iters)], 1)
    out["config1_single_core"] = {"elem_iter_per_s": r1["work"] / r1["wall_s"],
                                  "seconds": r1["wall_s"]}
    for cid, sample in ((2, False), (3, True), (4, True)):
        cfg = wl.CONFIGS[cid]
        L = cfg.blocks
        keep = sorted({0, L // 2, L - 1}) if sample else list(range(L))
        layer = [e for e in cfg.layer_set() if e[0] in keep]
        tasks = []
        for b, p, m, n in layer:
            W = wl.weight_host(cfg, b, p).float().numpy().astype(np.float64)
            amax = float(np.max(np.abs(W)))
            for j in range(0, n, 512):
                tasks.append(oracle_task(np.ascontiguousarray(W[:, j:j + 512]), cfg.fmt.kind,
                                         cfg.iters, amax))
        r = run_oracle_tasks(tasks, oracle_pool_size(len(tasks)))
        elems = sum(m * n for _, _, m, n in layer)
        rec = {"matrices": len(layer), "elements": elems, "workers": r["workers"],
               "wall_s": r["wall_s"], "cpu_s": r["cpu_s"],
               "elem_iter_per_s": r["work"] / r["wall_s"], "measured": True}
        if sample:
            rec["blocks"] = keep
            rec["full_set_wall_s_extrapolated"] = r["wall_s"] * cfg.elements() / elems
        out["config%d" % cid] = rec
    # activation workload: its k_proj solve and both quantizations
    Wk = wl.weight_host(wl.ACT_KPROJ, 0, 1).float().numpy().astype(np.float64)
    X = wl.act_host().float().numpy()
    t0 = time.perf_counter()
    c = S.solve(Wk, F.make_format("MXFP4"), wl.ACT_KPROJ.iters)["c"]
    for kind, g in (("NVFP4", 16), ("INT4", 128)):
        ora_act(X, F.make_format(kind, g), c)
    out["config5"] = {"wall_s": time.perf_counter() - t0, "workers": 1,
                      "what": "MXFP4 k_proj solve (1024 x 4096, 16 iterations) + NVFP4 and "
                              "INT4 g=128 quantization of 8192 x 4096"}
    out["config1_full"] = {"wall_s": out["config1_single_core"]["seconds"], "workers": 1,
                           "what": "the whole 512 x 512 tile is one solve"}
    out["total_wall_s"] = time.perf_counter() - t_all
    print(json.dumps({"cpu_plan": out}), flush=True)


# --------------------------------------------------------------------------- our path
class KernelTimer:
    """CUDA events recorded by the library around each solve-kernel launch (on the launch
    stream), for `cap` launches."""

    def __init__(self, lib, stream, cap: int):
        self.lib, self.cap = lib, cap
        self.ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
        self.ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
        for e in self.ev_s + self.ev_e:
            e.record(stream)                    # creates the underlying cudaEvent
        self.arr_s = (ctypes.c_void_p * cap)(*[e.cuda_event for e in self.ev_s])
        self.arr_e = (ctypes.c_void_p * cap)(*[e.cuda_event for e in self.ev_e])
        self.used = 0

    def __enter__(self):
        self.lib.dq_set_timing_events(self.arr_s, self.arr_e, self.cap)
        return self

    def __exit__(self, *exc):
        self.used = self.lib.dq_timing_events_used()
        self.lib.dq_set_timing_events(None, None, 0)

    def ms(self) -> float:
        return sum(a.elapsed_time(b) for a, b in zip(self.ev_s[:self.used], self.ev_e[:self.used]))


def _mats(Ws, outs):
    from calibration_free_dual_b200 import _lib
    arr = (_lib.dq_matrix * len(Ws))()
    for i, (W, o) in enumerate(zip(Ws, outs)):
        arr[i] = _lib.dq_matrix(W.data_ptr(), W.shape[0], W.shape[1], W.stride(0), None,
                                None, o["q_packed"].data_ptr(), o["r"].data_ptr(),
                                o["c"].data_ptr(), o["block_scales"].data_ptr(),
                                o["tensor_scale"].data_ptr(), o["mse"].data_ptr())
    return arr


def hbm_roofline(bytes_total: float, ms: float, peaks, peak_src, **extra) -> dict:
    gbs = bytes_total / (ms * 1e-3) / 1e9 if ms > 0 else None
    hbm = float(peaks["hbm_gbs"])
    d = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
         "frac": gbs / hbm if gbs else None,
         "peak_source": "%s copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" % peak_src
         if peak_src == "measured" else "fallback 6650 GB/s"}
    d.update(extra)
    return d


def convergence(mse: np.ndarray, qchange: np.ndarray) -> dict:
    """The pages' convergence figures for one matrix: the relative change of Q-hat at the
    last iteration (Figure 2 (a)), the first iteration whose normalised-MSE drop is under 1%
    (Figure 2 (b)), and single-scale over final MSE."""
    drop = (mse[:-1] - mse[1:]) / np.maximum(mse[:-1], 1e-300)
    below = [t + 1 for t in range(len(drop)) if drop[t] < 0.01]
    return {"qchange_last": float(qchange[-1]), "qchange_max": float(np.max(qchange)),
            "first_iter_drop_below_1pct": below[0] if below else None,
            "mse0_over_mseT": float(mse[0] / mse[-1]) if mse[-1] > 0 else None}


def block0_convergence(dq, cfg, dev, fmt_name) -> dict:
    """Q-change and MSE traces of block 0 of a layer set (solved once with the trace on)."""
    layer = [e for e in cfg.layer_set() if e[0] == 0]
    Ws = [wl.weight_device(cfg, b, p, device=dev) for b, p, _, _ in layer]
    outs = dq.solve_batched(Ws, fmt_name, cfg.iters, qchange=True)
    res = {}
    for (b, p, m, n), o in zip(layer, outs):
        res[wl.PROJ[p]] = convergence(o["mse"].cpu().numpy(), o["qchange"].cpu().numpy())
    del Ws, outs
    return res


def time_layer_set(dq, lib, cfg, fmt_name, dev, steps, warmup, rank=0, stream=None):
    """One dq_solve_batched over a whole layer set per step: (ms per step, solve-kernel ms per
    step, elements, launches per step)."""
    from calibration_free_dual_b200 import _lib
    stream = stream or torch.cuda.current_stream(dev)
    layer = cfg.layer_set()
    Ws = [wl.weight_device(cfg, b, p, device=dev, seed_offset=rank) for b, p, _, _ in layer]
    f = dq.fmt_of(fmt_name)
    T = cfg.iters
    outs = [dq.api.solve_outputs(W.shape[0], W.shape[1], f, T, dev) for W in Ws]
    count = len(Ws)
    ms_ = (ctypes.c_int64 * count)(*[W.shape[0] for W in Ws])
    ns_ = (ctypes.c_int64 * count)(*[W.shape[1] for W in Ws])
    need = lib.dq_solve_workspace_bytes(count, ms_, ns_, f, T)
    ws = torch.empty((need,), dtype=torch.uint8, device=dev)
    mats = _mats(Ws, outs)
    sp = ctypes.c_void_p(stream.cuda_stream)

    def step():
        st = lib.dq_solve_batched(mats, count, _lib.DQ_BF16, f, T, ctypes.c_void_p(ws.data_ptr()),
                                  need, sp)
        if st != 0:
            raise dq.DQError(st, "dq_solve_batched")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    per_step = sum((g + 63) // 64 for g in _group_sizes(layer))
    timer = KernelTimer(lib, stream, per_step * steps)
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with timer:
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if dq.last_device_error() != 0:
        raise RuntimeError("device error while timing %s" % cfg.name)
    elems = sum(W.numel() for W in Ws)
    res = (t0.elapsed_time(t1) / steps, timer.ms() / steps, elems, per_step)
    del Ws, outs, ws
    torch.cuda.empty_cache()
    return res


def config_record(dq, lib, cid, dev, steps, warmup, peaks, peak_src) -> dict:
    """A layer set in its own shapes and format: throughput, full-model solve seconds, the
    solve kernel's HBM fraction on the algorithmic bytes, block-0 convergence."""
    cfg = wl.CONFIGS[cid]
    fmt_name = cfg.fmt.kind
    ms, kms, elems, per_step = time_layer_set(dq, lib, cfg, fmt_name, dev, steps, warmup)
    bpe = solve_bytes_per_elem(fmt_name, cfg.iters)
    return {"workload": "%s (%d matrices, %.3e bf16 weights), %s, %d BCD iterations"
                        % (cfg.name, len(cfg.layer_set()), elems, fmt_name, cfg.iters),
            "value": elems * cfg.iters / (ms * 1e-3), "unit": UNIT,
            "full_model_solve_s": ms * 1e-3, "solve_kernel_ms": kms,
            "roofline": hbm_roofline(bpe * elems, kms, peaks, peak_src, kernel="solve_kernel",
                                     bytes_per_elem=bpe, traffic=None),
            "convergence_block0": block0_convergence(dq, cfg, dev, fmt_name)}


ACT_BYTES_PER_ELEM = {"NVFP4": 2.0 + 0.5 + 1.0 / 16, "INT4": 2.0 + 0.5 + 2.0 / 128}


def act_call_prepared(dq, lib, X, fmt, c):
    """A dq_act_quant call with its outputs and workspace allocated beforehand: the returned
    function enqueues the call through the C ABI alone (no allocation, a few microseconds of
    host work), so a timed region around it sees the device time."""
    from calibration_free_dual_b200 import _lib
    f = dq.fmt_of(fmt)
    T, n = X.shape
    out = dq.act_quant(X, fmt, c)                       # allocates the outputs once
    ws = out["_workspace"]
    p = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else 0)
    args = (p(X), _lib.DQ_BF16 if X.dtype == torch.bfloat16 else _lib.DQ_F32, T, n,
            X.stride(0), p(c), f, p(out["x_packed"]), p(out["scales"]), p(out["tensor_scale"]),
            p(ws), ws.numel())

    def call(stream):
        st = lib.dq_act_quant(*args, ctypes.c_void_p(stream.cuda_stream))
        if st != 0:
            raise dq.DQError(st, "dq_act_quant")
        return out
    return call




ACT_ROTATE = 4          # distinct activation inputs cycled by the back-to-back timing


def act_timings(dq, lib, X, c, fmt, dev, steps, warmup, world):
    """Device time of dq_act_quant on X (through the C ABI, preallocated outputs), two ways:

    - streamed: `steps` calls back to back between one pair of events, cycling over
      ACT_ROTATE copies of X with their own outputs (together larger than the 126 MB L2, so
      no call finds its input in L2), after an L2 flush; time per call = total / steps. This
      is the throughput of a stream of calls, the figure the roofline divides.
    - isolated: one call per event pair, L2 flushed before it (256 MB written, then 256 MB
      read, so no dirty lines are left to write back inside the call) and a 1 ms GPU-side
      wait so that the host has enqueued the call; this adds the launch and event latency
      (about 6 us on an empty kernel) to every call.

    Returns (streamed ms, isolated ms, outputs of one call, kernel launches counted)."""
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    flush_r = torch.ones((64 << 20,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    Xs = [X] + [X.clone() for _ in range(ACT_ROTATE - 1)]
    calls = [act_call_prepared(dq, lib, Xi, fmt, c) for Xi in Xs]
    for _ in range(max(warmup, 1)):
        for call in calls:
            call(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    l0 = lib.dq_kernel_launches()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush.fill_(1)
    flush_r.amax()
    torch.cuda._sleep(2_000_000)
    e0.record(stream)
    for i in range(steps):
        out = calls[i % ACT_ROTATE](stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    streamed = e0.elapsed_time(e1) / steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        flush.fill_(1)
        flush_r.amax()
        torch.cuda._sleep(2_000_000)
        a.record(stream)
        calls[0](stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    launches = lib.dq_kernel_launches() - l0
    if dq.last_device_error() != 0:
        raise RuntimeError("device error during the activation timing")
    isolated = sum(a.elapsed_time(b) for a, b in evs) / steps
    del flush, flush_r, Xs, calls
    return reduce_max(streamed, world), reduce_max(isolated, world), out, launches


def act_timing_text(steps: int) -> str:
    return ("device time per call over %d calls back to back through the C ABI (preallocated "
            "outputs), cycling over %d copies of X (268 MB, larger than L2); isolated: one "
            "call behind an L2 flush (256 MB written, then read) and a 1 ms GPU-side wait"
            % (steps, ACT_ROTATE))


def act_record(dq, lib, X, c, dev, steps, warmup, world, peaks, peak_src) -> dict:
    """dq_act_quant alone on the activation workload (8192 x 4096 bf16) with column scales c,
    NVFP4 and INT4 g=128: device time per call (streamed and isolated, see act_timings), the
    HBM fraction on the algorithmic bytes, and the SQNR of the decoded activation with and
    without c."""
    T, n = X.shape
    res = {}
    launches = 0
    for fmt in ("NVFP4", "INT4"):
        ms, ms_iso, out, nl = act_timings(dq, lib, X, c, fmt, dev, steps, warmup, world)
        launches += nl
        sq = {"with_c": _sqnr(X.float() * c, _act_decode(dq, out, fmt, T, n))}
        out0 = dq.act_quant(X, fmt, None)
        sq["without_c"] = _sqnr(X.float(), _act_decode(dq, out0, fmt, T, n))
        res[fmt] = {"us_per_call": ms * 1e3, "us_per_call_isolated": ms_iso * 1e3,
                    "elems_per_s": world * T * n / (ms * 1e-3), "sqnr_db": sq,
                    "roofline": hbm_roofline(ACT_BYTES_PER_ELEM[fmt] * T * n, ms, peaks,
                                             peak_src, bytes_per_elem=ACT_BYTES_PER_ELEM[fmt],
                                             traffic=None)}
    return {"workload": "activations 8192 x 4096 bf16 (N(0,1), 6 channels x50) times the "
                        "step's block-0 k_proj c",
            "timing": act_timing_text(steps),
            "formats": res, "gpu_launches": int(launches)}


def run_ours(args, world, rank, local):
    import calibration_free_dual_b200 as dq
    from calibration_free_dual_b200 import _lib
    from calibration_free_dual_b200.shard import assign, loads

    dev = torch.device("cuda", local)
    cfg = wl.CONFIGS[CFG_ID]
    full_layer = cfg.layer_set()
    if args.blocks is not None:
        full_layer = [e for e in full_layer if e[0] < args.blocks]
    T = cfg.iters
    fmt = dq.fmt_of(args.fmt)
    headline = args.fmt == "NVFP4" and args.update == "both" and not args.qchange
    stream = torch.cuda.current_stream(dev)
    split = bool(args.split)          # (one rank: the whole layer set, the same work either way)
    if split:
        # one layer set shared by the ranks, matrices assigned by element count
        sizes = [m * n for _, _, m, n in full_layer]
        parts = assign(sizes, world)
        layer = [full_layer[i] for i in parts[rank]]
        seed_offset = 0
    else:
        layer = full_layer
        seed_offset = rank

    # inputs (device-generated, seeded per rank) and preallocated outputs
    Ws = [wl.weight_device(cfg, b, p, device=dev, seed_offset=seed_offset)
          for b, p, _, _ in layer]
    X = wl.act_device(device=dev)
    outs = [dq.api.solve_outputs(W.shape[0], W.shape[1], fmt, T, dev) for W in Ws]
    count = len(Ws)
    ms = (ctypes.c_int64 * count)(*[W.shape[0] for W in Ws])
    ns = (ctypes.c_int64 * count)(*[W.shape[1] for W in Ws])
    lib = _lib.get()
    opts = None
    if not headline and (args.update != "both" or args.qchange):
        qtraces = [torch.empty((T + 1,), dtype=torch.float64, device=dev) for _ in Ws]
        qptrs = (ctypes.c_void_p * count)(*[q.data_ptr() for q in qtraces]) if args.qchange \
            else None
        opts = _lib.dq_solve_options(dq.api.UPDATES[args.update], qptrs)
    ws_bytes = lib.dq_solve_workspace_bytes_ex(count, ms, ns, fmt, T,
                                               ctypes.byref(opts) if opts else None)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    act_proto = dq.api.solve_outputs(X.shape[0], X.shape[1], fmt, 0, dev)
    act_out = dict(x_packed=act_proto["q_packed"], scales=act_proto["block_scales"],
                   tensor_scale=act_proto["tensor_scale"])
    act_ws = torch.empty((lib.dq_act_quant_workspace_bytes(X.shape[0], X.shape[1], fmt),),
                         dtype=torch.uint8, device=dev)
    # the activation's column scales: this rank's first k_proj (block 0's when it has it)
    k0 = next((i for i, (b, p, _, _) in enumerate(layer) if p == 1),
              0 if layer else None)

    def mats_for(Wlist, olist=None):
        return _mats(Wlist, outs if olist is None else olist)

    mats = mats_for(Ws)

    def solve_call(mats_arr, n_mats, strm):
        sp = ctypes.c_void_p(strm.cuda_stream)
        if n_mats == 0:
            return
        if opts is None:
            st = lib.dq_solve_batched(mats_arr, n_mats, _lib.DQ_BF16, fmt, T,
                                      ctypes.c_void_p(ws.data_ptr()), ws_bytes, sp)
        else:
            st = lib.dq_solve_batched_ex(mats_arr, n_mats, _lib.DQ_BF16, fmt, T,
                                         ctypes.byref(opts), ctypes.c_void_p(ws.data_ptr()),
                                         ws_bytes, sp)
        if st != 0:
            raise dq.DQError(st, "dq_solve_batched")

    c_act = outs[k0]["c"] if k0 is not None else None

    def act_call(Xin, strm):
        st = lib.dq_act_quant(ctypes.c_void_p(Xin.data_ptr()), _lib.DQ_BF16, Xin.shape[0],
                              Xin.shape[1], Xin.stride(0),
                              ctypes.c_void_p(c_act.data_ptr() if c_act is not None else 0),
                              fmt, ctypes.c_void_p(act_out["x_packed"].data_ptr()),
                              ctypes.c_void_p(act_out["scales"].data_ptr()),
                              ctypes.c_void_p(act_out["tensor_scale"].data_ptr()),
                              ctypes.c_void_p(act_ws.data_ptr()), act_ws.numel(),
                              ctypes.c_void_p(strm.cuda_stream))
        if st != 0:
            raise dq.DQError(st, "dq_act_quant")

    def step(mats_arr, Xin):
        solve_call(mats_arr, count, stream)
        act_call(Xin, stream)

    elems = sum(W.numel() for W in Ws)
    elems_job = sum(m * n for _, _, m, n in full_layer) if split else world * elems
    for _ in range(args.warmup):
        step(mats, X)
    torch.cuda.synchronize(dev)
    if dq.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # per-launch events for the solve kernel over the timed region
    per_step = sum((g + 63) // 64 for g in _group_sizes(layer))   # launches per step
    timer = KernelTimer(lib, stream, max(1, per_step * args.steps))
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = lib.dq_kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with timer:
        t0.record(stream)
        for _ in range(args.steps):
            step(mats, X)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    launches = lib.dq_kernel_launches() - launches0
    barrier(world)
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_total = reduce_max(ms_total, world)
    if dq.last_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    kern_ms = timer.ms()

    ms_step = ms_total / args.steps
    value = elems_job * T / (ms_step * 1e-3)

    peaks, peak_src = _peaks()
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    # the solve kernel against HBM on the algorithmic bytes (W and the block-scale state
    # every iteration, the codes once): what a per-iteration streaming solve would move
    bpe = solve_bytes_per_elem(args.fmt, T)
    prof = profiled_solve_kernel() if headline else {}
    traffic = None
    if prof.get("dram_bytes_per_elem_solve") is not None:
        traffic = prof["dram_bytes_per_elem_solve"] * elems / max(per_step, 1)
    kms_step = kern_ms / args.steps
    roof = hbm_roofline(bpe * elems, kms_step, peaks, peak_src, traffic=traffic,
                        kernel="solve_kernel", bytes_per_elem=bpe,
                        kernel_ms_per_step=kms_step, launches_timed=timer.used,
                        traffic_unit="DRAM bytes per solve launch (ncu capture of the same "
                                     "kernel source, layer-set average), null if the kernel "
                                     "changed since",
                        note="achieved = the algorithmic bytes of a per-iteration streaming "
                             "solve (W and the block-scale state every iteration, the codes "
                             "once) over the kernel time; the kernel itself reads W from HBM "
                             "about once per solve (dram_gbs_measured)")
    if traffic is not None:
        roof["dram_gbs_measured"] = traffic * per_step / (kms_step * 1e-3) / 1e9
    act_bpe = ACT_BYTES_PER_ELEM.get(args.fmt if args.fmt != "INT4_G64" else "INT4")
    act_elems = X.numel()
    step_bytes = (bpe + prepass_bytes_per_elem(args.fmt)) * elems + (act_bpe or 0) * act_elems
    roof_step = hbm_roofline(step_bytes, ms_total / args.steps, peaks, peak_src,
                             bytes_per_elem=bpe + prepass_bytes_per_elem(args.fmt),
                             includes="solve kernel, NVFP4 tensor-scale pre-pass, trace "
                                      "finalisation and the activation quantization",
                             per_gpu=True)
    issue = None
    if prof.get("inst_per_elem_pass") is not None:
        warp_inst = prof["inst_per_elem_pass"] / 32.0 * elems * T
        ach = warp_inst / (kms_step * 1e-3)
        pk = 148 * 4 * sm_max * 1e6
        issue = {"bound": "issue", "inst_per_elem_pass": prof["inst_per_elem_pass"],
                 "achieved": ach, "peak": pk, "unit": "warp-instructions/s", "frac": ach / pk,
                 "peak_source": "148 SMs x 4 schedulers x %.0f MHz, one instruction per "
                                "scheduler per cycle; instruction count from ncu" % sm_max}

    # ------------------------------------------------------------------ end to end
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, world, dev, Ws, X, outs, act_out, solve_call, act_call, mats_for,
                      layer, elems, T, elems_job)

    # ------------------------------------------------------------------ extra records
    extra = {}
    if world == 1 and headline and not args.no_extra:
        extra["act"] = act_record(dq, lib, X, c_act, dev, args.steps, args.warmup, world,
                                  peaks, peak_src)
        conv3 = block0_convergence(dq, cfg, dev, "NVFP4")
        del Ws, outs, mats, ws
        torch.cuda.empty_cache()
        extra["configs"] = {"1B_MXFP4": config_record(dq, lib, 2, dev, args.steps,
                                                      args.warmup, peaks, peak_src),
                            "7B_MXINT4": config_record(dq, lib, 4, dev, args.steps,
                                                       args.warmup, peaks, peak_src)}
        extra["configs"]["8B_NVFP4"] = {"convergence_block0": conv3}

    # ------------------------------------------------------------------ CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_record(args.fmt, args.update)

    if rank == 0:
        cfgd = {"workload": workload_name(len(full_layer), sum(m * n for _, _, m, n in full_layer),
                                          T, args.fmt, args.update, args.qchange),
                "full_model_solve_s": ms_step * 1e-3,
                "l2": "inputs larger than L2 (%.1f GB of weights per step)" % (elems * 2 / 1e9),
                "blocks": args.blocks if args.blocks is not None else cfg.blocks}
        if split:
            cfgd["parallelism"] = "one layer set split over %d GPUs by matrix" % world
            cfgd["elements_per_rank"] = loads([m * n for _, _, m, n in full_layer], parts)
        else:
            cfgd["parallelism"] = "one layer set per GPU (weak)"
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if split else "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": cfgd,
            "roofline": roof,
            "roofline_step": roof_step,
            "roofline_issue": issue,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)


def _group_sizes(layer):
    sizes = {}
    order = []
    for _, _, m, n in layer:
        if (m, n) not in sizes:
            sizes[(m, n)] = 0
            order.append((m, n))
        sizes[(m, n)] += 1
    return [sizes[k] for k in order]


def run_e2e(args, world, dev, Ws, X, outs, act_out, solve_call, act_call, mats_for, layer,
            elems, T, elems_job):
    """The same step through the public API from pinned host buffers, results read back to
    pinned host buffers, pipelined the way a user streams a model: one dq_solve_batched per
    block of the layer set on the compute stream, while a copy stream brings in the next
    blocks' weights and another takes the finished blocks' outputs back."""
    host_W = [torch.empty(W.shape, dtype=W.dtype, pin_memory=True) for W in Ws]
    for h, W in zip(host_W, Ws):
        h.copy_(W)
    host_X = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
    host_X.copy_(X)
    dev_W = [torch.empty_like(W) for W in Ws]
    dev_X = torch.empty_like(X)
    keys = ("q_packed", "block_scales", "c", "tensor_scale", "mse")
    host_out = [{k: torch.empty(o[k].shape, dtype=o[k].dtype, pin_memory=True) for k in keys}
                for o in outs]
    host_act = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                for k, v in act_out.items()}
    h2d = sum(h.numel() * h.element_size() for h in host_W) + host_X.numel() * host_X.element_size()
    d2h = sum(o[k].numel() * o[k].element_size() for o in outs for k in keys) + \
        sum(v.numel() * v.element_size() for v in act_out.values())
    blocks = sorted({b for b, _, _, _ in layer})
    chunks = [[i for i, (b, _, _, _) in enumerate(layer) if b == blk] for blk in blocks]
    chunk_mats = [mats_for([dev_W[i] for i in idx], [outs[i] for i in idx]) for idx in chunks]
    comp = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)

    def e2e_step():
        start = torch.cuda.Event()
        start.record(comp)
        s_in.wait_event(start)
        s_out.wait_event(start)
        ev_in = []
        with torch.cuda.stream(s_in):
            dev_X.copy_(host_X, non_blocking=True)
            for idx in chunks:
                for i in idx:
                    dev_W[i].copy_(host_W[i], non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                ev_in.append(e)
        for ci, idx in enumerate(chunks):
            comp.wait_event(ev_in[ci])
            solve_call(chunk_mats[ci], len(idx), comp)
            if ci == 0:
                act_call(dev_X, comp)
            done = torch.cuda.Event()
            done.record(comp)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                for i in idx:
                    for k in keys:
                        host_out[i][k].copy_(outs[i][k], non_blocking=True)
                if ci == 0:
                    for k, v in act_out.items():
                        host_act[k].copy_(v, non_blocking=True)
        end = torch.cuda.Event()
        end.record(s_out)
        comp.wait_event(end)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    for _ in range(args.steps):
        e2e_step()
    b.record(comp)
    torch.cuda.synchronize(dev)
    ms = reduce_max(a.elapsed_time(b), world) / args.steps
    return {"value": elems_job * T / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipeline": "per block: H2D, dq_solve_batched and D2H on three streams"}


def run_gemm(args, world, rank, local):
    """W4A4 GEMM on the solver's and the activation quantizer's NVFP4 outputs: the 7
    projections of the 8B layer set's block 0 against T activation rows each."""
    import calibration_free_dual_b200 as dq
    from calibration_free_dual_b200 import _lib
    dev = torch.device("cuda", local)
    cfg = wl.CONFIGS[CFG_ID]
    layer = [e for e in cfg.layer_set() if e[0] == 0]
    T = args.gemm_tokens
    Ws = [wl.weight_device(cfg, b, p, device=dev, seed_offset=rank) for b, p, _, _ in layer]
    sols = dq.solve_batched(Ws, "NVFP4", cfg.iters)
    g = torch.Generator(device=dev)
    g.manual_seed(77 + rank)
    acts, Xs = [], []
    for W, sol in zip(Ws, sols):
        X = torch.randn((T, W.shape[1]), generator=g, device=dev).to(torch.bfloat16)
        Xs.append(X)
        acts.append(dq.act_quant(X, "NVFP4", sol["c"]))
    lib = _lib.get()
    shapes = [(T, W.shape[0], W.shape[1]) for W in Ws]
    need = max(lib.dq_w4a4_gemm_workspace_bytes(t, n, k) for t, n, k in shapes)
    ws = torch.empty((need,), dtype=torch.uint8, device=dev)
    ys = [torch.empty((t, n), dtype=torch.float32, device=dev) for t, n, _ in shapes]
    stream = torch.cuda.current_stream(dev)
    sptr = ctypes.c_void_p(stream.cuda_stream)
    f = dq.fmt_of("NVFP4")
    p = lambda t: ctypes.c_void_p(t.data_ptr())

    def step():
        for (t, n, k), a, sol, y in zip(shapes, acts, sols, ys):
            st = lib.dq_w4a4_gemm(p(a["x_packed"]), p(a["scales"]), p(a["tensor_scale"]), t,
                                  p(sol["q_packed"]), p(sol["block_scales"]),
                                  p(sol["tensor_scale"]), n, k, f, p(y), n, p(ws), need, sptr)
            if st != 0:
                raise dq.DQError(st, "dq_w4a4_gemm")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    cap = 7 * args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(cap)]
    for e in ev_s + ev_e:
        e.record(stream)
    arr_s = (ctypes.c_void_p * cap)(*[e.cuda_event for e in ev_s])
    arr_e = (ctypes.c_void_p * cap)(*[e.cuda_event for e in ev_e])
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = lib.dq_kernel_launches()
    lib.dq_set_timing_events(arr_s, arr_e, cap)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    used = lib.dq_timing_events_used()
    lib.dq_set_timing_events(None, None, 0)
    launches = lib.dq_kernel_launches() - launches0
    barrier(world)
    clk = clocks.stop()
    if dq.last_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    ms_total = reduce_max(t0.elapsed_time(t1), world)
    kern_ms = sum(a.elapsed_time(b) for a, b in zip(ev_s[:used], ev_e[:used]))
    flop = 2.0 * sum(t * n * k for t, n, k in shapes)

    # the same layers from the unquantized activations: dq_w4a4_linear (fl32(X * c) quantized
    # straight into the tensor core's layouts, the weight's scale factors re-laid, the GEMM)
    need_lin = max(lib.dq_w4a4_linear_workspace_bytes(t, n, k, f) for t, n, k in shapes)
    wsl = torch.empty((need_lin,), dtype=torch.uint8, device=dev)

    def lin_step():
        for (t, n, k), X, sol, y in zip(shapes, Xs, sols, ys):
            st = lib.dq_w4a4_linear(p(X), 1, t, k, k, p(sol["c"]), p(sol["q_packed"]),
                                    p(sol["block_scales"]), p(sol["tensor_scale"]), n, f, p(y),
                                    n, p(wsl), need_lin, sptr)
            if st != 0:
                raise dq.DQError(st, "dq_w4a4_linear")

    for _ in range(args.warmup):
        lin_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    l0 = torch.cuda.Event(enable_timing=True)
    l1 = torch.cuda.Event(enable_timing=True)
    l0.record(stream)
    for _ in range(args.steps):
        lin_step()
    l1.record(stream)
    torch.cuda.synchronize(dev)
    if dq.last_device_error() != 0:
        raise RuntimeError("device error during the timed linear region")
    lin_ms = reduce_max(l0.elapsed_time(l1), world) / args.steps
    ms_step = ms_total / args.steps
    peaks, peak_src = _peaks()
    fp4_peak = float(peaks["bf16_tflops"]) * 4.0          # dense FP4 / BF16 = 9 / 2.25
    achieved = flop * args.steps / (kern_ms * 1e-3) / 1e12
    if rank == 0:
        line = {
            "metric": "W4A4 GEMM TFLOP/s (NVFP4 operands from the solver and dq_act_quant)",
            "value": world * flop / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (fp32 accumulate)", "data": "synthetic",
            "config": {"workload": "block-0 projections of the Llama-3.1-8B-shaped layer set "
                                   "(7 GEMMs, %d tokens each, K = 4096 / 14336)" % T,
                       "step": "7 dq_w4a4_gemm calls (each: scale-factor re-layout + GEMM)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": achieved / fp4_peak, "traffic": None,
                         "peak_source": "measured bf16 %.1f TF/s (%s) x 4, the nominal dense "
                                        "FP4/BF16 ratio" % (float(peaks["bf16_tflops"]),
                                                            peak_src),
                         "kernel": "w4a4_gemm_kernel (the scale-factor re-layout launches "
                                   "are outside this figure, inside ms_per_step)",
                         "kernel_ms_per_step": kern_ms / args.steps},
            "linear": {"ms_per_step": lin_ms,
                       "value": world * flop / (lin_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "step": "7 dq_w4a4_linear calls from bf16 X and c (activation "
                               "quantized into the tensor core's layouts, weight scale "
                               "factors re-laid, GEMM); timed after the GEMM region"},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def _act_decode(dq, out, fmt, T, n):
    """Decoded activation d * q (binary32) from dq_act_quant's outputs, with the library's
    own codecs on the device."""
    from calibration_free_dual_b200 import _lib
    xp = out["x_packed"]
    nib = torch.stack((xp & 0xF, xp >> 4), dim=2).reshape(T, n).contiguous()
    if fmt == "NVFP4":
        q = dq.decode(nib, _lib.DQ_CODEC_E2M1)
        d = dq.decode(out["scales"], _lib.DQ_CODEC_E4M3) * out["tensor_scale"][0]
        B = 16
    else:
        q = dq.decode(nib, _lib.DQ_CODEC_INT4)
        d = dq.decode(out["scales"], _lib.DQ_CODEC_BF16)
        B = 128
    return d.repeat_interleave(B, dim=1) * q


def _sqnr(xt, xhat):
    xt = xt.double()
    err = ((xt - xhat.double()) ** 2).sum().item()
    sig = (xt * xt).sum().item()
    return float("inf") if err == 0.0 else 10.0 * math.log10(sig / err)


def run_act(args, world, rank, local):
    """dq_act_quant alone on the activation workload: 8192 tokens x 4096 bf16 channels
    (N(0,1), six channels x50) rescaled by the c of a 1024 x 4096 k_proj (Student-t(4),
    std 0.02, 1% columns x8, MXFP4, 16 iterations), quantized to NVFP4 and INT4 g=128."""
    import calibration_free_dual_b200 as dq
    from calibration_free_dual_b200 import _lib
    dev = torch.device("cuda", local)
    Wk = wl.weight_device(wl.ACT_KPROJ, 0, 1, device=dev, seed_offset=rank)
    c = dq.solve(Wk, "MXFP4", wl.ACT_KPROJ.iters)["c"]
    X = wl.act_device(seed=wl.ACT_SEED + rank, device=dev)
    lib = _lib.get()
    peaks, peak_src = _peaks()
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    rec = act_record(dq, lib, X, c, dev, args.steps, args.warmup, world, peaks, peak_src)
    clk = clocks.stop()
    if rank == 0:
        head = rec["formats"]["NVFP4"]
        line = {
            "metric": "activation rescale+quantize elements/s",
            "value": head["elems_per_s"], "unit": "elem/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["us_per_call"] / 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "activations 8192 x 4096 bf16 (N(0,1), 6 channels x50) "
                                   "times a k_proj's c (1024 x 4096, MXFP4 solve), NVFP4 "
                                   "(amax pass + quantization pass); INT4 g=128 alongside",
                       "l2": "inputs larger than L2 (%d copies of X cycled); the isolated "
                             "figure flushes L2 before each call" % ACT_ROTATE,
                       "timed": rec["timing"]},
            "roofline": dict(head["roofline"], kernel="act_amax_kernel + act_quant_kernel"),
            "formats": rec["formats"], "gpu_launches": rec["gpu_launches"], "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.cpu_plan:
            if rank == 0:
                run_cpu_plan(args)
        elif args.gemm:
            run_gemm(args, world, rank, local)
        elif args.act:
            run_act(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
