"""Throughput of the InternVL visual-token compression hot path on B200.

Default workload (``flash_2b_13tiles``): one step = one ivc_flash_compress over
one image of 12 tiles + thumbnail (T = 13 tiles of [32, 32, 1024] bf16,
InternVL3.5-2B-Flash dims): pixel_shuffle 0.5 -> mlp1 and 0.25 -> mlp2 for
every tile, the ViR router (CrossAttentionPooling, Gating, quantile + absolute
threshold) and compaction to 64/256 rows per tile.

``--workload`` selects another configuration (``workloads.WORKLOADS``): the
batched 4B-Flash flow (``flash_4b_batched``, one step = one
ivc_flash_compress over 16 images), or a connector alone (``single_tile_2b``,
``connector_14b_832tiles``, ``connector_38b_416tiles``: one step = one
ivc_ps_project at factor 0.5 over the whole batch).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ivc|reference]
                    [--workload NAME]

Prints one JSON line (rank 0). Metric: tiles per second (whole job). Inputs
are resident in HBM; L2 is flushed (512 MiB write) between timed steps, each
step timed with CUDA events on the launching stream; max over ranks. With
N > 1 every rank processes its own batch (weights replicated, no data-path
collective): weak scaling. ``--impl reference`` times the fp64 CPU oracle on
a bounded per-step sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ViT tiles/sec through ps+MLP connector & ViR router; % of bf16 tensor/HBM peak"
UNIT = "tiles/s"
DEFAULT_WORKLOAD = "flash_2b_13tiles"
WORKLOAD_NAMES = ("single_tile_2b", "flash_2b_13tiles", "flash_4b_batched",
                  "connector_14b_832tiles", "connector_38b_416tiles")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_ROLES = ("mlp1.fc1", "mlp1.fc2", "mlp2.fc1", "mlp2.fc2", "mlp2.fc3")


# ----------------------------------------------------------------- helpers (CPU-testable)
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity when world == 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(kernel, workload=DEFAULT_WORKLOAD):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    capture (profiles/traffic.json), or None once the sources it was built
    from have changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("workload", DEFAULT_WORKLOAD) != workload:
        return None
    e = d.get("kernels", {}).get(kernel)
    if e is None:
        return None
    for rel, digest in d.get("sources_sha256", {}).items():
        fp = os.path.join(ROOT, rel)
        if not os.path.exists(fp) or hashlib.sha256(open(fp, "rb").read()).hexdigest() != digest:
            return None
    return e["dram_bytes_read"] + e["dram_bytes_write"]


def algorithmic(w, T):
    """Algorithmic FLOPs / bytes per step of each kernel role for T tiles of
    workload w (a role with several launches per step is divided by them).

    FLOPs count 2 per multiply-add of the literal method; bytes count each
    operand read once and each result written once."""
    C, H, M2, D, G = w.C, w.H, w.mlp2_mid, w.D, w.gate_hidden
    r256, r64, tok = T * 256, T * 64, T * 1024
    bf, f32 = 2, 4
    f = {
        "mlp1.fc1": (2.0 * r256 * 4 * C * H, bf * (tok * C + 4 * C * H + r256 * H)),
        "mlp1.fc2": (2.0 * r256 * H * H, bf * (r256 * H + H * H + r256 * H)),
        "mlp2.fc1": (2.0 * r64 * 16 * C * M2, bf * (tok * C + 16 * C * M2 + r64 * M2)),
        "mlp2.fc2": (2.0 * r64 * M2 * H, bf * (r64 * M2 + M2 * H + r64 * H)),
        "mlp2.fc3": (2.0 * r64 * H * H, bf * (r64 * H + H * H + r64 * H)),
        "pool.kv": (2.0 * tok * D * 8 * D, bf * (tok * D + 8 * D * D) + f32 * tok * 8 * D),
        # folded pooling, 4 layer launches per step: scores X u^T (u split in
        # 2x16 rows) and weighted sums p X (p split in 2x16 rows)
        "pool.scores": (4 * 2.0 * tok * D * 32, 4 * (bf * (tok * D + T * 32 * D) + f32 * tok * 32)),
        "pool.wsum": (4 * 2.0 * T * 32 * 1024 * D,
                      4 * (bf * (tok * D + T * 32 * 1024) + f32 * T * 32 * D)),
        # the same two contractions in one pass over x per layer (single-pass
        # form): x and u read once, the merged weighted sums written
        "pool.attend": (4 * 2.0 * 2 * tok * D * 32,
                        4 * (bf * (tok * D + T * 32 * D) + f32 * T * 16 * D)),
        "pool.attention": (4 * 4.0 * tok * D, 4 * f32 * tok * 2 * D),  # literal pooling
        "ps_stats": (3.0 * tok * C, bf * tok * C + f32 * 2 * (r256 + r64)),
        # compaction reads and writes the kept rows (all-256 upper bound here;
        # the bench prices it with the step's actual mask)
        "compact": (0.0, bf * 2 * r256 * H),
        "route": (0.0, f32 * 2 * T),
    }
    return f


def router_bytes(w, T):
    """Algorithmic bytes of the whole folded router for T tiles: the features
    once, every pooling and gating weight and bias once, the gates written."""
    D, G = w.D, w.gate_hidden
    pool_w = 4 * (4 * D * D + 4 * D) + D          # Wq/Wk/Wv/Wo + biases x 4 layers, query
    gate_w = 4 * (2 * D * G + G + 3 * D) + 2 * D + 2  # W1/W2, b1/b2, LN gamma/beta x 4, head
    return 2.0 * T * 1024 * w.C + 2.0 * (pool_w + gate_w) + 4.0 * 2 * T


def connector_roles(w):
    return GEMM_ROLES if w.path == "flash" else GEMM_ROLES[:2]


def image_gen(rank: int, workload: str = DEFAULT_WORKLOAD, n_images=None):
    import workloads as W
    return W.make(workload, seed_offset=1000 * rank, n_images=n_images)


class ClockSampler:
    """nvidia-smi clocks/throttle reasons, sampled every 50 ms while running.

    Each sample carries its timestamp, so the summary separates the samples
    taken inside the timed region from those of the whole loaded window
    (the untimed preheat and warm-up steps right before it, and the timed
    steps)."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    @staticmethod
    def parse(lines):
        """Rows of (epoch seconds, sm MHz, max MHz, power W or None, reasons)."""
        out = []
        for line in lines:
            p = [v.strip() for v in line.split(",")]
            if len(p) < 10 or not p[2].replace(".", "").isdigit():
                continue
            try:
                ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            pw = float(p[4]) if p[4].replace(".", "").isdigit() else None
            reasons = {ClockSampler.REASONS[i] for i in range(4) if p[6 + i].lower() == "active"}
            out.append((ts, float(p[2]), float(p[3]), pw, reasons))
        return out

    @staticmethod
    def summarise(rows, t0, t1):
        """Clock summary of the samples in [t0, t1] (the loaded window) and
        the count of those inside the timed region's own bounds, if given."""
        win = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [r[1] for r in win]
        pw = [r[3] for r in win if r[3] is not None]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": win[0][2],
                "sm_mhz_min": min(sm), "reasons": sorted(set().union(*[r[4] for r in win])),
                "samples": len(win), "power_w_max": max(pw) if pw else None}

    def summary(self, t0, t1, timed=None):
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                rows = self.parse(f)
            os.unlink(self.path)
        s = self.summarise(rows, t0, t1)
        s["window"] = "preheat + warm-up + timed steps (GPU loaded throughout)"
        if timed is not None:
            s["samples_in_timed"] = sum(1 for r in rows if timed[0] <= r[0] <= timed[1])
        return s


def thread_count() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ----------------------------------------------------------------- oracle (CPU) legs
def _oracle_params(inp):
    import oracle as O
    if "_m1_64" not in inp:
        inp["_m1_64"] = O.to64(inp["mlp1"])
        if "mlp2" in inp:
            inp["_m2_64"] = O.to64(inp["mlp2"])
            inp["_r_64"] = O.to64(inp["router"])


def oracle_sample(inp, tile: int, frac: float):
    """The oracle's whole path for `frac` of one tile: mlp1 on the first
    256*frac shuffled rows and, on the flash workloads, mlp2 on the first
    64*frac, pooling over the first 1024*frac tokens, gating, routing of the
    one-tile group and the compaction offsets. Returns the tiles processed
    (= frac)."""
    import numpy as np

    import oracle as O
    _oracle_params(inp)
    x = O.to64(inp["x"][tile:tile + 1])
    n256, n64, ntok = max(1, round(256 * frac)), max(1, round(64 * frac)), max(1, round(1024 * frac))
    P = O.pixel_shuffle(x, 0.5)[0, :n256]
    m1 = inp["_m1_64"]
    O.mlp(P, m1["ln_g"], m1["ln_b"], m1["W"], m1["b"])
    if "mlp2" not in inp:
        return frac
    Q = O.pixel_shuffle_quarter(x)[0, :n64]
    m2 = inp["_m2_64"]
    O.mlp(Q, m2["ln_g"], m2["ln_b"], m2["W"], m2["b"])
    X = x.reshape(1, 1024, -1)[:, :ntok]
    pooled = O.cross_attention_pooling(X, np.array([ntok]), inp["_r_64"])
    gate = O.gating(pooled, inp["_r_64"])
    mask = O.route(gate[:, 0], np.array([0, 1]))
    O.compaction_offsets(mask)
    return frac


def cpu_sample_plan(inp):
    """What the CPU baseline runs: whole images (routing couples the tiles of
    an image) up to at least 8 tiles on the flash workloads, the whole image
    when it has at most 16 tiles; 8 seeded tiles of a connector workload."""
    import numpy as np
    T = inp["T"]
    w = inp["workload"]
    if w.path == "flash":
        offs = inp["image_offsets"].numpy()
        if T <= 16:
            return "images", len(offs) - 1
        n = 1
        while n < len(offs) - 1 and offs[n] < 8:
            n += 1
        return "images", n
    k = min(8, T)
    rng = np.random.default_rng(2024)
    return "tiles", sorted(rng.choice(T, k, replace=False).tolist())


def cpu_baseline(inp):
    """The oracle, as it stands, on the sample cpu_sample_plan picks; the
    value is tiles processed per second of host time."""
    import oracle as O
    _oracle_params(inp)
    kind, what = cpu_sample_plan(inp)
    t0 = time.perf_counter()
    if kind == "images":
        offs = inp["image_offsets"].numpy()
        n_t = int(offs[what])
        O.flash_compress(O.to64(inp["x"][:n_t]), inp["valid_len"].numpy()[:n_t], offs[:what + 1],
                         inp["_m1_64"], inp["_m2_64"], inp["_r_64"])
        desc = (f"the first {what} image(s), {n_t} tiles, whole path (fp64)" if n_t < inp["T"]
                else f"one full batch of {n_t} tiles, whole path (fp64)")
    else:
        n_t = len(what)
        O.ps_project(O.to64(inp["x"][what]), 0.5, inp["_m1_64"])
        desc = f"{n_t} seeded tiles of {inp['T']} (ps 0.5 + mlp1, fp64), rate scales linearly in T"
    dt = time.perf_counter() - t0
    return {"value": n_t / dt, "unit": UNIT, "cores": thread_count(), "kind": "oracle",
            "sample": f"{desc}, {dt:.1f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = image_gen(0, args.workload)
    w, T = inp["workload"], inp["T"]
    t0 = time.perf_counter()
    oracle_sample(inp, 0, 1.0)
    t_tile = time.perf_counter() - t0
    budget = 150.0
    frac = 1.0
    while frac > 1.0 / 256 and (args.steps + args.warmup) * t_tile * frac > budget:
        frac /= 2
    for i in range(args.warmup):
        oracle_sample(inp, i % T, frac)
    units, dt = 0.0, 0.0
    for i in range(args.steps):
        t0 = time.perf_counter()
        units += oracle_sample(inp, i % T, frac)
        dt += time.perf_counter() - t0
    value = units / dt
    path = "whole path" if w.path == "flash" else "ps 0.5 + mlp1"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "tiles": T, "C": w.C, "H": w.H},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thread_count(), "kind": "oracle",
                             "sample": f"per step {frac:g} of one tile (rows/tokens subsampled), "
                                       f"{path} in fp64"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU leg
class Problem:
    """Device-resident inputs, outputs and the one call a step makes."""

    def __init__(self, ivc, inp, dev, routed):
        import torch
        self.ivc, self.inp, self.dev, self.routed = ivc, inp, dev, routed
        w, T = inp["workload"], inp["T"]
        self.w, self.T = w, T
        self.flash = w.path == "flash"
        self.x = inp["x"].to(dev)
        self.m1 = ivc.Mlp(inp["mlp1"], dev).fold()
        if self.flash:
            self.vl = inp["valid_len"].to(dev)
            self.offs = inp["image_offsets"].to(dev)
            self.m2 = ivc.Mlp(inp["mlp2"], dev).fold()
            self.r = ivc.Router(inp["router"], device=dev)
            self.ws = ivc.new_workspace(
                ivc.workspace_size(ivc.OP_FLASH, T, w.C, self.m1, self.m2, self.r), dev)
            self.bufs = {"gate": torch.empty(T, 2, dtype=torch.float32, device=dev),
                         "mask": torch.empty(T, dtype=torch.uint8, device=dev),
                         "offsets": torch.empty(T + 1, dtype=torch.int32, device=dev),
                         "total": torch.empty(1, dtype=torch.int32, device=dev)}
        else:
            self.ws = ivc.new_workspace(ivc.workspace_size(ivc.OP_PS_HALF, T, w.C, self.m1), dev)
            self.bufs = {}
        self.out = torch.empty(T * 256, w.H, dtype=torch.bfloat16, device=dev)

    def call(self, x=None, vl=None, offs=None, out=None, ws=None, bufs=None):
        x = self.x if x is None else x
        out = self.out if out is None else out
        ws = self.ws if ws is None else ws
        if self.flash:
            self.ivc.flash_compress(x, self.vl if vl is None else vl,
                                    self.offs if offs is None else offs, self.m1, self.m2, self.r,
                                    out=out, workspace=ws, bufs=self.bufs if bufs is None else bufs,
                                    routed=self.routed)
        else:
            self.ivc.ps_project(x, 0.5, self.m1, out=out, workspace=ws)

    def inputs(self):
        """The per-step inputs a user copies in (name -> device tensor)."""
        d = {"x": self.x}
        if self.flash:
            d.update({"vl": self.vl, "offs": self.offs})
        return d


def run_ivc(args):
    import torch

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    import vlm_visual_token_b200 as ivc

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    inp = image_gen(rank, args.workload)
    routed = args.flow == "routed"
    P = Problem(ivc, inp, dev, routed)
    w, T = P.w, P.T
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    step = P.call

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    assert ivc.device_status(P.ws) == 0
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        graph = g
    except Exception:
        graph = None
    run = graph.replay if graph is not None else step

    with ClockSampler(local) as clk:
        t_load0 = time.time()
        # untimed preheat (at least a second of the same loaded loop) so that
        # the clock sampler sees the GPU under this load right up to the
        # timed steps, however short those are
        t_end = time.perf_counter() + 1.0
        while time.perf_counter() < t_end:
            for _ in range(8):
                flush.zero_()
                run()
            torch.cuda.synchronize()
        for _ in range(args.warmup):
            flush.zero_()
            run()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        t_timed0 = time.time()
        t_wall = time.perf_counter()
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            run()
            b.record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
        t_timed1 = time.time()
        time.sleep(0.1)  # let the sampler write its last row
    barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = reduce_max(sum(step_ms), world, dev)
    value = world * T * args.steps / (total_ms / 1e3)
    clocks = clk.summary(t_load0, t_timed1, (t_timed0, t_timed1))
    if ivc.device_status(P.ws) != 0:
        raise RuntimeError("device status word set during the timed steps")

    def graph_ms(fn, reps=50):
        g = torch.cuda.CUDAGraph()
        fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            fn()
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        del g
        return tot / reps

    peaks, src = load_peaks()
    parts = {}
    if P.flash:
        # ---- the two halves of the step alone (CUDA graphs, L2 flushed): the
        # router (ivc_vir_route) and the connector (both ivc_ps_project calls)
        ws_r = ivc.new_workspace(ivc.workspace_size(ivc.OP_VIR_ROUTE, T, w.C, r=P.r), dev)
        y256 = torch.empty(T * 256, w.H, dtype=torch.bfloat16, device=dev)
        y64 = torch.empty(T * 64, w.H, dtype=torch.bfloat16, device=dev)
        ws_1 = ivc.new_workspace(ivc.workspace_size(ivc.OP_PS_HALF, T, w.C, P.m1), dev)
        ws_2 = ivc.new_workspace(ivc.workspace_size(ivc.OP_PS_QUARTER, T, w.C, P.m2), dev)
        parts = {
            "router_ms": graph_ms(lambda: ivc.vir_route(P.x, P.vl, P.offs, P.r, workspace=ws_r)),
            "connector_ms": graph_ms(lambda: (ivc.ps_project(P.x, 0.5, P.m1, out=y256, workspace=ws_1),
                                              ivc.ps_project(P.x, 0.25, P.m2, out=y64,
                                                             workspace=ws_2))),
        }
        del ws_r, ws_1, ws_2, y256, y64

    # ---- traced pass: per-kernel device time of the same steps (eager launches)
    n_trace = min(args.steps, 50)
    ivc.trace_reset()
    ivc.trace_enable(True)
    for _ in range(n_trace):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ivc.trace_enable(False)
    trace = ivc.trace_report()
    ivc.trace_reset()
    launches_per_step = sum(v["launches"] for v in trace.values()) / n_trace
    per_step_ms = {k: v["ms"] / n_trace for k, v in trace.items()}
    trace_total = sum(per_step_ms.values())
    alg = algorithmic(w, T)
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained", burst)
    # every connector Linear against the dense bf16 peak: the burst figure,
    # since each runs for well under a second inside a short step
    gemm = {}
    for k in connector_roles(w):
        if k in trace and trace[k]["launches"] > 0:
            us = 1e3 * trace[k]["ms"] / trace[k]["launches"]
            fl = alg[k][0] / (trace[k]["launches"] / n_trace)
            tf = fl / (us * 1e-6) / 1e12
            gemm[k] = {"gflop_per_launch": fl / 1e9, "us_per_launch": us, "tflops": tf,
                       "frac": tf / burst, "frac_vs_sustained": tf / sustained}
    # all connector Linears in one persistent launch: priced as their sum
    if "connector.graph" in trace and trace["connector.graph"]["launches"] > 0:
        k = "connector.graph"
        us = 1e3 * trace[k]["ms"] / trace[k]["launches"]
        fl = sum(alg[r][0] for r in connector_roles(w)) / (trace[k]["launches"] / n_trace)
        tf = fl / (us * 1e-6) / 1e12
        gemm[k] = {"gflop_per_launch": fl / 1e9, "us_per_launch": us, "tflops": tf,
                   "frac": tf / burst, "frac_vs_sustained": tf / sustained,
                   "linears": list(connector_roles(w))}
    # dominant kernel: the connector contraction with the largest traced time.
    # (Inside the step the router's launches wait for SMs the GEMMs hold, so
    # their traced times include that wait; by device time in the ncu launch
    # list the connector GEMMs dominate.) The HBM-bound kernels are reported
    # on their own below.
    dom = max(gemm, key=lambda k: per_step_ms[k])
    roof = {"bound": "tensor", "achieved": gemm[dom]["tflops"], "peak": burst, "unit": "TFLOP/s",
            "frac": gemm[dom]["frac"], "traffic": kernel_traffic(dom, w.name), "kernel": dom,
            "peak_source": f"{src} bf16_tflops (burst)",
            "frac_vs_sustained": gemm[dom]["frac_vs_sustained"],
            "duration": "traced pass (events around each launch, 50 eager steps after the timed "
                        "region)"}
    if not P.flash and trace[dom]["launches"] == n_trace:
        # one stream, one launch of the dominant kernel per step: its duration
        # inside the timed region is the timed step less the other kernels'
        # traced times (under the power cap the clock differs between the two
        # passes, so the timed region is the one that counts)
        others_ms = sum(v for k, v in per_step_ms.items() if k != dom)
        us_timed = (total_ms / args.steps - others_ms) * 1e3
        fl = gemm[dom]["gflop_per_launch"] * 1e9
        tf = fl / (us_timed * 1e-6) / 1e12
        roof.update({"achieved": tf, "frac": tf / burst, "frac_vs_sustained": tf / sustained,
                     "achieved_traced": gemm[dom]["tflops"], "us_per_launch_timed": us_timed,
                     "duration": "timed region: mean step (CUDA events) less the other kernels' "
                                 "traced device time"})
    # the HBM-bound kernels: algorithmic bytes per launch / traced launch time
    hbm = {}
    kept_rows = int(P.bufs["offsets"][-1].item()) if P.flash else T * 256
    for k in ("ps_stats", "compact", "pool.attend"):
        if k in trace and trace[k]["launches"] > 0:
            us = 1e3 * trace[k]["ms"] / trace[k]["launches"]
            b_launch = alg[k][1] / (trace[k]["launches"] / n_trace)
            if k == "compact":
                b_launch = 2.0 * 2 * kept_rows * w.H
            gbs = b_launch / (us * 1e-6) / 1e9
            hbm[k] = {"bytes_per_launch": b_launch, "us_per_launch": us, "achieved": gbs,
                      "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"]}
    router_roof = None
    if P.flash and not routed:
        rb = router_bytes(w, T)
        gbs = rb / (parts["router_ms"] * 1e-3) / 1e9
        router_roof = {"bound": "hbm", "bytes": rb, "us": parts["router_ms"] * 1e3,
                       "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": gbs / peaks["hbm_gbs"],
                       "note": "ivc_vir_route alone (CUDA graph, L2 flushed); bytes = x once + "
                               "pooling and gating weights once"}
    # whole-step roofline: algorithmic FLOPs at the dense bf16 peak vs bytes at HBM peak.
    conn = sum(alg[k][0] for k in connector_roles(w))
    if P.flash:
        # F_literal counts the method as the pages state it (K/V projections
        # of all tokens); F_folded is what the folded pooling has to compute.
        gate_f = 2.0 * T * (8 * w.D * w.gate_hidden + 2 * w.D)
        F = conn + alg["pool.kv"][0] + alg["pool.attention"][0] + gate_f + 2.0 * T * 8 * w.D * w.D
        F_folded = (conn + alg["pool.scores"][0] + alg["pool.wsum"][0] + gate_f +
                    2.0 * T * 16 * w.D * w.D)
        B_alg = 2 * (T * 1024 * w.C) + 2 * (4 * w.C * w.H + w.H * w.H + 16 * w.C * w.mlp2_mid +
                                            w.mlp2_mid * w.H + w.H * w.H + 16 * w.D * w.D +
                                            8 * w.D * w.gate_hidden) + 2 * T * 256 * w.H
    else:
        F = F_folded = conn
        B_alg = 2 * (T * 1024 * w.C) + 2 * (4 * w.C * w.H + w.H * w.H) + 2 * T * 256 * w.H
    t_roof = max(F / (burst * 1e12), B_alg / (peaks["hbm_gbs"] * 1e9))
    t_roof_f = max(F_folded / (burst * 1e12), B_alg / (peaks["hbm_gbs"] * 1e9))
    meas = total_ms / args.steps / 1e3
    step_roofline = {"flops_literal": F, "flops_folded": F_folded, "bytes": B_alg,
                     "roofline_us_literal": t_roof * 1e6, "roofline_us_folded": t_roof_f * 1e6,
                     "measured_us": meas * 1e6, "frac_vs_literal": t_roof / meas,
                     "frac_vs_folded": t_roof_f / meas,
                     "peak_source": f"{src} bf16_tflops (burst), hbm_gbs"}
    if routed:
        # router-first: only the selected path of each tile is computed
        k = int(P.bufs["mask"].sum().item())
        m1f = (alg["mlp1.fc1"][0] + alg["mlp1.fc2"][0]) * (T - k) / T
        m2f = (alg["mlp2.fc1"][0] + alg["mlp2.fc2"][0] + alg["mlp2.fc3"][0]) * k / T
        F_routed = F_folded - conn + m1f + m2f
        B_routed = B_alg - 2 * T * 256 * w.H + 2 * (256 * (T - k) + 64 * k) * w.H
        t_roof_r = max(F_routed / (burst * 1e12), B_routed / (peaks["hbm_gbs"] * 1e9))
        step_roofline.update({"compressed_tiles": k, "flops_routed": F_routed,
                              "bytes_routed": B_routed, "roofline_us_routed": t_roof_r * 1e6,
                              "frac_vs_routed": t_roof_r / meas})

    e2e = run_e2e(args, P, run, world, dev, barrier)

    fn_name = ("ivc_flash_compress_routed" if routed else "ivc_flash_compress") if P.flash \
        else "ivc_ps_project (factor 0.5)"
    launch_desc = (f"CUDA graph of one {fn_name}" if graph is not None else f"eager {fn_name}")
    run = None
    graph = None
    barrier()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    config = {"workload": w.name, "tiles_per_step": T, "C": w.C, "H": w.H}
    if P.flash:
        config.update({"mlp2_mid": w.mlp2_mid, "pool_heads": w.D // 64,
                       "gate_hidden": w.gate_hidden, "images": int(inp["image_offsets"].numel() - 1),
                       "flow": ("router first, each tile through its selected path" if routed
                                else "both paths for every tile, then compaction")})
    else:
        config["flow"] = "pixel_shuffle 0.5 + mlp1 (LayerNorm, Linear, GELU, Linear)"
    config.update({"l2": "flushed between steps (512 MiB write, outside the timed events)",
                   "launch": launch_desc,
                   "parallelism": f"replicas x{world}, one batch per GPU, no collective"})
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config, "roofline": roof, "gemm": gemm, "step_roofline": step_roofline,
            "hbm_kernels": hbm, "kernels_ms_per_step": {k: round(v, 5) for k, v in per_step_ms.items()},
            "traced_ms_per_step": trace_total, "clocks": clocks, "e2e": e2e,
            "gpu_launches": int(round(launches_per_step * args.steps)), "wall_s_timed": t_wall}
    if parts:
        line["parts_graph_ms"] = parts
    if router_roof:
        line["router_roofline"] = router_roof
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, P, run, world, dev, barrier):
    """The same metric end to end through the public API with host buffers:
    every step copies its inputs in from pinned host memory and its results
    out. First with a host sync per step, then pipelined over buffer sets on
    their own streams, as a streaming user would run it."""
    import torch
    w, T, ivc = P.w, P.T, P.ivc
    host_in = {k: v.cpu().pin_memory() for k, v in P.inputs().items()}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    out_bytes = T * 256 * w.H * 2
    small_bytes = sum(v.numel() * v.element_size() for v in P.bufs.values())
    big = h2d + out_bytes > (1 << 30)
    e2e_steps = min(args.steps, 10 if big else 100)
    n_sets = 2 if big else 3
    hout = torch.empty(T * 256, w.H, dtype=torch.bfloat16).pin_memory()
    hsmall = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in P.bufs.items()}
    d2h_rows = 0
    dev_in = P.inputs()
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        for k, v in dev_in.items():
            v.copy_(host_in[k], non_blocking=True)
        run()
        if P.flash:
            for k in P.bufs:
                hsmall[k].copy_(P.bufs[k], non_blocking=True)
            torch.cuda.current_stream().synchronize()
            rows = int(hsmall["total"][0])
        else:
            rows = T * 256
        hout[:rows].copy_(P.out[:rows], non_blocking=True)
        torch.cuda.current_stream().synchronize()
        d2h_rows += rows * w.H * 2
    e2e_s = reduce_max(time.perf_counter() - t0, world, dev)
    e2e_sync = {"value": world * T * e2e_steps / e2e_s, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": small_bytes + d2h_rows // e2e_steps, "steps": e2e_steps,
                "timing": "wall clock, host sync per step" +
                          (" (the row count read before the row copy)" if P.flash else "")}
    del hout

    sets = []
    for i in range(n_sets):
        st = torch.cuda.Stream(device=dev)
        e = {"st": st, "in": {k: torch.empty_like(v) for k, v in dev_in.items()},
             "out": torch.empty_like(P.out),
             "bufs": {k: torch.empty_like(v) for k, v in P.bufs.items()},
             "ws": ivc.new_workspace(P.ws.numel(), dev),
             "hout": torch.empty(T * 256, w.H, dtype=torch.bfloat16).pin_memory(),
             "hsmall": {k: torch.empty(v.shape, dtype=v.dtype).pin_memory()
                        for k, v in P.bufs.items()}}
        st.wait_stream(torch.cuda.current_stream())

        def call(e=e):
            P.call(x=e["in"]["x"], vl=e["in"].get("vl"), offs=e["in"].get("offs"), out=e["out"],
                   ws=e["ws"], bufs=e["bufs"])
        with torch.cuda.stream(st):
            for k, v in dev_in.items():
                e["in"][k].copy_(v)
            for _ in range(2):
                call()
        st.synchronize()
        e["g"] = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e["g"], stream=st):
            call()
        sets.append(e)
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for i in range(e2e_steps):
        e = sets[i % n_sets]
        with torch.cuda.stream(e["st"]):
            for k, v in e["in"].items():
                v.copy_(host_in[k], non_blocking=True)
            e["g"].replay()
            for k in P.bufs:
                e["hsmall"][k].copy_(e["bufs"][k], non_blocking=True)
            e["hout"].copy_(e["out"], non_blocking=True)
    torch.cuda.synchronize()
    e2e_p = reduce_max(time.perf_counter() - t0, world, dev)
    if P.flash:
        last = sets[(e2e_steps - 1) % n_sets]
        if int(last["hsmall"]["total"][0]) != int(P.bufs["total"].item()):
            raise RuntimeError("pipelined end-to-end run returned a different row count")
    e2e = {"value": world * T * e2e_steps / e2e_p, "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": small_bytes + out_bytes, "steps": e2e_steps,
           "timing": f"wall clock over all steps; {n_sets} streams, inputs copied in and "
                     "results (small outputs and the whole row capacity) copied out every step",
           "synchronous": e2e_sync}
    for e in sets:
        del e["g"]
    return e2e


def run_op(args):
    """One entry point alone on the bench image (profiling aid: a short,
    eager run whose kernels ncu can pick out by launch index)."""
    import torch

    import vlm_visual_token_b200 as ivc
    torch.cuda.set_device(0)
    inp = image_gen(0, args.workload, args.images)
    w, T = inp["workload"], inp["T"]
    if w.path != "flash" and args.op not in ("ps_half",):
        raise SystemExit(f"--op {args.op} needs a flash workload; {w.name} has mlp1 only")
    x = inp["x"].cuda()
    vl, offs = inp["valid_len"].cuda(), inp["image_offsets"].cuda()
    if args.op == "assemble":
        # the image's rows into a prompt: 64 text tokens, 13 x 256 placeholders,
        # 32 text tokens; a vocabulary of the Qwen3 size (151,936 x H table)
        m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
        r = ivc.Router(inp["router"])
        fres = ivc.flash_compress(x, vl, offs, m1, m2, r)
        V, img = 151936, 151667
        g = torch.Generator(device="cuda").manual_seed(3)
        table = (0.02 * torch.randn(V, w.H, device="cuda", generator=g)).to(torch.bfloat16)
        text = torch.randint(0, img, (96,), device="cuda", generator=g, dtype=torch.int32)
        ids = torch.cat([text[:64], torch.full((256 * T,), img, dtype=torch.int32, device="cuda"),
                         text[64:]])
        soffs = torch.tensor([0, ids.numel()], dtype=torch.int32, device="cuda")
        ws_a = ivc.new_workspace(ivc.lib().ivc_assemble_workspace_size(ids.numel()))
        aout = None

        def fn():
            nonlocal aout
            aout = ivc.assemble_sequence(ids, soffs, img, table, fres["out"], fres["mask"],
                                         fres["offsets"], workspace=ws_a, out=aout)
    elif args.op in ("flash_dual", "flash_routed"):
        m1, m2 = ivc.Mlp(inp["mlp1"]).fold(), ivc.Mlp(inp["mlp2"]).fold()
        r = ivc.Router(inp["router"])
        fn = lambda: ivc.flash_compress(x, vl, offs, m1, m2, r, routed=args.op == "flash_routed")
    elif args.op in ("ps_half", "ps_quarter"):
        m = ivc.Mlp(inp["mlp1" if args.op == "ps_half" else "mlp2"]).fold()
        scale = 0.5 if args.op == "ps_half" else 0.25
        fn = lambda: ivc.ps_project(x, scale, m)
    else:
        r = ivc.Router(inp["router"], pool_mode=1 if args.op == "route_literal" else 0)
        fn = lambda: ivc.vir_route(x, vl, offs, r)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        g.replay()
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / args.steps
    line = {"op": args.op, "workload": w.name, "tiles": T, "ms_per_call": ms,
            "tiles_per_s": T / (ms / 1e3), "timing": "CUDA graph, back to back, no L2 flush"}
    if args.op == "assemble":
        n = int(aout["seq_offsets"][-1].item())
        moved = 2.0 * n * w.H * 2  # each kept row read once and written once
        line.update({"prompt_tokens": int(ids.numel()), "kept_tokens": n,
                     "bytes_per_call": moved, "achieved_gbs": moved / (ms / 1e3) / 1e9})
    if args.trace:
        ivc.trace_reset()
        ivc.trace_enable(True)
        for _ in range(args.steps):
            fn()
        torch.cuda.synchronize()
        ivc.trace_enable(False)
        tr = ivc.trace_report()
        ivc.trace_reset()
        line["traced_us_per_launch"] = {k: round(1e3 * v["ms"] / v["launches"], 2)
                                        for k, v in tr.items()}
        line["traced_launches_per_call"] = {k: v["launches"] // args.steps for k, v in tr.items()}
    print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ivc", "reference"], default="ivc")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=WORKLOAD_NAMES, default=DEFAULT_WORKLOAD,
                    help="configuration to run (default: the 13-tile 2B-Flash image)")
    ap.add_argument("--flow", choices=["dual", "routed"], default="dual",
                    help="dual: ivc_flash_compress (both paths, then compaction); "
                         "routed: ivc_flash_compress_routed (router first)")
    ap.add_argument("--op", choices=["flash", "flash_dual", "flash_routed", "ps_half",
                                     "ps_quarter", "route", "route_literal", "assemble"],
                    default="flash", help="profiling aid: time one entry point alone "
                                          "(flash = the full benchmark)")
    ap.add_argument("--trace", action="store_true",
                    help="with --op: also report per-kernel device times (event-bracketed)")
    ap.add_argument("--images", type=int, default=None,
                    help="with --op: only the workload's first N images (small profiling cases)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.op != "flash":
        return run_op(args)
    if args.flow == "routed" and args.workload not in WORKLOAD_NAMES[1:3]:
        ap.error("--flow routed needs a flash workload")
    return run_ivc(args)


if __name__ == "__main__":
    sys.exit(main())
