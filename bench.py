"""Benchmark: LUT-GEMM microseconds per matmul and achieved HBM GB/s at batch 1.

One step is one pass over the linears of an OPT-175B-shaped decoder layer
(QKV 36864x12288, out-proj 12288x12288, FC1 49152x12288, FC2 12288x49152) with
q = 3 BCQ planes, g = 128, batch 1: four lutgemm_run calls.  Weights are
synthetic (uniform random sign bits, |N(0, 0.02)| fp16 scales, x ~ N(0, 1)),
drawn by bcq_synth; the step's working set (765 MB) is far larger than the
126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lutgemm|reference]

N > 1 runs under torchrun: every rank runs its own layer (independent weights,
no data-path collective: weak scaling); the timed region is bracketed by a
barrier and device synchronisation and its length is the max over ranks.
"--parallel rows|inputs|paired" instead splits one matrix (OPT-175B FC1, FC2,
or the FC1 -> FC2 block) over the ranks with an NCCL exchange (strong scaling).
"--impl reference" times the FP64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).

Other workloads (one JSON line each, same timing rules):
    --workload tc     the same linears at batch 256 (--tc-batch) through
                      lutgemm_run with LUTGEMM_ALLOW_TENSOR_CORES (tensor-core
                      path, K splits where the library's model picks them);
                      --tc-direct calls lutgemm_run_tc instead
    --workload fit    BCQ fitting of FP16 weights (--fit-grid: variable grid)
    --workload sweep  every configured shape and batch: lookup kernel, tensor
                      cores and the library's choice, against both floors
    --workload mixed  mixed 2/4/16-bit storage (lutgemm_run_mixed) on the
                      LLaMA-70B-shaped linears: 2-plane blocks, --mixed-hi of
                      them at 4 planes, --mixed-outliers fp16 outliers
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

if __name__ != "__mp_main__":
    # A process the CPU baseline spawns re-imports this file under that name
    # and only runs _oracle_job: it needs neither torch nor the library.
    import torch  # noqa: E402

    import bcq_synth as S  # noqa: E402
    from weight_only_quantized_bcq_b200.roofline import algorithmic_bytes  # noqa: E402

METRIC = "LUT-GEMM µs/matmul and achieved HBM GB/s (fraction of B200 peak) at batch 1"
WORKLOAD = "opt175b_layer"
DATASHEET_GBS = 8000.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


KERNEL_SOURCES = ("lutgemm_common.cuh", "lutgemm_run.cuh")


def _code_hash(files) -> str:
    """Hash of CUDA sources with their comments removed: the ncu counters in
    profiles/ are tied to the code, and an edit of comments alone keeps them."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_quantized_bcq_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        text = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(f.encode() + text.encode())
    return h.hexdigest()[:16]


def _kernel_hash() -> str:
    """Hash of the code that defines lut_gemm_kernel (ncu counters are tied to it)."""
    return _code_hash(KERNEL_SOURCES)


def _traffic(kernel_hash: str, names):
    """Mean DRAM bytes per launch over the step's linears, from the committed ncu
    summary; null unless it was taken on this kernel source and covers every linear."""
    path = os.path.join(ROOT, "profiles", "lut_gemm_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    per = d.get("per_shape_bytes", {})
    if d.get("kernel_hash") != kernel_hash or not all(n in per for n in names):
        return None
    return sum(per[n] for n in names) / len(names)


class ClockSampler:
    """SM clock and clock-event reasons read through NVML every millisecond while
    the timed region runs (reads only; no GPU setting is touched)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, torch_index: int, period_s: float = 0.001):
        self.torch_index = torch_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def _handle(self, nv):
        try:
            uuid = str(torch.cuda.get_device_properties(self.torch_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.torch_index)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nvml = nv
            self.h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._loop, daemon=True)
            self._thread.start()
        except Exception:
            self._nvml = None
        return self

    def _loop(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((float(mhz), int(mask)))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return None
        nv = self._nvml or __import__("pynvml")
        reasons = set()
        for _, mask in self.samples:
            for name, const in self.REASONS:
                if mask & int(getattr(nv, const, 0)):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml, 1 ms"}


# ---------------------------------------------------------------------------
# Workload
# ---------------------------------------------------------------------------
def make_layer(q: int, batch: int, seed: int, device, only=None, scales="packed"):
    """Packed planes, scales and inputs of the four linears, resident on `device`.

    With scales="packed" the [q][n/g][m] scales are reordered once, at load
    time, into the unit-major layout that lutgemm_run reads with
    LUTGEMM_SCALES_PACKED (same bytes for g = 128).

    The step's inputs x and outputs y of all linears sit in one buffer each
    (host: pinned; device), each linear's x and y a view into it, so the end
    to end step moves them with one copy each way."""
    from weight_only_quantized_bcq_b200 import lutgemm
    w = S.WORKLOADS[WORKLOAD]
    gen = S.generator(seed)
    shapes = [sh for sh in w.shapes if not only or sh.name == only]
    xs = sum(batch * sh.n for sh in shapes)
    ys = sum(batch * sh.m for sh in shapes)
    io = {"x_host": torch.empty(xs, dtype=torch.float16).pin_memory(),
          "x": torch.empty(xs, dtype=torch.float16, device=device),
          "y_host": torch.empty(ys, dtype=torch.float32).pin_memory(),
          "y": torch.empty(ys, dtype=torch.float32, device=device)}
    mats = []
    xo = yo = 0
    for sh in shapes:
        nbytes = lutgemm.packed_bytes(q, sh.m, sh.n)
        packed_host = S.draw_random_bytes(gen, nbytes)
        alpha_host = S.draw_alpha(gen, q, sh.m, sh.n, w.g, w.alpha_sigma)
        packed = packed_host.to(device)
        alpha = alpha_host.to(device)
        if scales == "packed":
            alpha = lutgemm.pack_scales(alpha, sh.m, sh.n, w.g)
        x_host = io["x_host"][xo: xo + batch * sh.n].view(batch, sh.n)
        x_host.copy_(S.draw_x(gen, batch, sh.n))
        mats.append({
            "name": sh.name, "m": sh.m, "n": sh.n, "packed": packed, "alpha": alpha,
            "packed_host": packed_host, "alpha_host": alpha_host,
            "scales_packed": scales == "packed", "launches": 1 + (sh.n > 1024),
            "x_host": x_host, "x": io["x"][xo: xo + batch * sh.n].view(batch, sh.n),
            "y": io["y"][yo: yo + batch * sh.m].view(batch, sh.m),
            "y_host": io["y_host"][yo: yo + batch * sh.m].view(batch, sh.m),
            "ws": lutgemm.new_workspace(sh.m, sh.n, batch, q, w.g, device=device),
            "bytes": algorithmic_bytes(sh.m, sh.n, q, w.g, batch),
        })
        xo += batch * sh.n
        yo += batch * sh.m
    io["x"].copy_(io["x_host"])
    return mats, w.g, io


def max_over_ranks(dist, v: float, device) -> float:
    """Largest v over all ranks (every rank gets it); v itself without a process group."""
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(step_bytes: int, steps: int, world: int, region_ms: float) -> float:
    """Whole-job throughput: every rank's bytes over the slowest rank's time (weak scaling)."""
    return step_bytes * steps * world / (region_ms * 1e-3) / 1e9


def rank_seed(rank: int) -> int:
    """Seed of rank `rank`'s layer: every rank draws its own weights and inputs."""
    return S.WORKLOADS[WORKLOAD].seed + 1000 * rank


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_lutgemm(args):
    from weight_only_quantized_bcq_b200 import lutgemm
    world, rank, local = _dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist
    q, batch = args.q, args.batch
    mats, g, io = make_layer(q, batch, seed=rank_seed(rank), device=device, only=args.only, scales=args.scales)
    # All work goes on one non-default stream (a CUDA graph cannot be captured
    # on the legacy default stream); it is made current so torch's copies use it.
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)

    def step(events=None):
        for i, mt in enumerate(mats):
            if events is not None:
                events[i][0].record(stream)
            lutgemm.run(mt["packed"], mt["alpha"], mt["x"], mt["m"], mt["n"], q, g, y=mt["y"],
                        workspace=mt["ws"], scales_packed=mt["scales_packed"], stream=stream)
            if events is not None:
                events[i][1].record(stream)

    def e2e_step():
        io["x"].copy_(io["x_host"], non_blocking=True)
        for mt in mats:
            lutgemm.run(mt["packed"], mt["alpha"], mt["x"], mt["m"], mt["n"], q, g, y=mt["y"],
                        workspace=mt["ws"], scales_packed=mt["scales_packed"], stream=stream)
        io["y_host"].copy_(io["y"], non_blocking=True)

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()

    # Device-resident timing: K steps back to back (consecutive launches
    # overlap their ramps by programmatic dependent launch), with CUDA events
    # on the launching stream around the whole region.  By default the steps
    # are replayed from a CUDA graph of G steps (the launches of a decode
    # step, captured once as a serving runtime would), K/G replays.
    per_graph = 0
    graph = None
    if args.graph_steps > 0:
        per_graph = args.graph_steps if args.steps % args.graph_steps == 0 else 1
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(per_graph):
                step()
        graph.replay()  # untimed: uploads the graph and runs its steps once
        barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        barrier()
        t0.record(stream)
        if graph is not None:
            for _ in range(args.steps // per_graph):
                graph.replay()
        else:
            for _ in range(args.steps):
                step()
        t1.record(stream)
        barrier()
    region_ms = max_over_ranks(pg, t0.elapsed_time(t1), device)
    if graph is not None:
        del graph
    # The outputs of the last timed step, kept for the parity check against
    # the oracle (outside the timed region).
    y_timed = io["y"].cpu().clone()

    # Per-linear times: a separate pass with events around every launch (the
    # events serialise the launches, so these are isolated kernel times).
    per_launch = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
                   for _ in mats] for _ in range(args.steps)]
    for k in range(args.steps):
        step(per_launch[k])
    barrier()
    launch_ms = [[per_launch[k][i][0].elapsed_time(per_launch[k][i][1]) for i in range(len(mats))]
                 for k in range(args.steps)]

    # End to end through the public API: per step, pinned x -> device, the four
    # runs, y -> pinned host; all inside the timed region.
    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1), device)

    step_bytes = sum(mt["bytes"] for mt in mats)
    value = aggregate_gbs(step_bytes, args.steps, world, region_ms)
    e2e_gbs = aggregate_gbs(step_bytes, args.steps, world, e2e_ms)
    # The region holds the lookup launches and the split-K reduces chained
    # behind them; a chained launch's own duration cannot be separated without
    # serialising the stream, so the whole region is charged to lut_gemm_kernel
    # (a lower bound on its rate).
    achieved = step_bytes * args.steps / (region_ms * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    khash = _kernel_hash()
    us_per = {mt["name"]: 1e3 * statistics.median([launch_ms[k][i] for k in range(args.steps)])
              for i, mt in enumerate(mats)}
    gbs_per = {mt["name"]: mt["bytes"] / (us_per[mt["name"]] * 1e-6) / 1e9 for mt in mats}

    if rank == 0:
        out = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(region_ms / args.steps, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": {
                "workload": "OPT-175B decoder-layer linears (QKV 36864x12288, out 12288x12288, "
                            f"FC1 49152x12288, FC2 12288x49152), BCQ q={q}, g={g}, batch {batch}",
                "q": q, "g": g, "batch": batch,
                "bytes_per_step": step_bytes,
                "l2": "no flush: each step streams 765 MB (> 126 MB L2) of distinct weights",
                "scales": ("unit-major, reordered once at load time (lutgemm_pack_scales)"
                           if args.scales == "packed" else "[q][n/g][m]"),
                "launch": (f"CUDA graph of {per_graph} steps, replayed {args.steps // per_graph} times"
                           if per_graph else "eager launches"),
                "parallelism": "replicas" if world == 1 else f"replicas{world} (one layer per GPU)",
                "only": args.only,
            },
            "us_per_matmul": {k: round(v, 2) for k, v in us_per.items()},
            "us_per_matmul_note": "median of isolated launches (events around each launch)",
            "gbs_per_matmul": {k: round(v, 1) for k, v in gbs_per.items()},
            "frac_of_datasheet_8tbs": round(value / world / DATASHEET_GBS, 4),
            "roofline": {
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": _traffic(khash, [mt["name"] for mt in mats]),
                "peak_kind": peak_kind, "kernel": "lut_gemm_kernel", "kernel_hash": khash,
            },
            "e2e": {"value": round(e2e_gbs, 1), "unit": "GB/s",
                    "h2d_bytes_per_step": io["x_host"].numel() * 2,
                    "d2h_bytes_per_step": io["y_host"].numel() * 4,
                    "copies_per_step": "one H2D of all x, one D2H of all y (pinned host buffers)"},
            # Per lutgemm_run: the lookup kernel, plus the split-K reduce when n > 1024.
            "gpu_launches": sum(mt["launches"] for mt in mats) * args.steps,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"], out["parity"] = cpu_baseline_and_parity(mats, q, g, batch, args.cpu_rows,
                                                                         y_timed, io)
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


# ---------------------------------------------------------------------------
# The FP64 oracle on the host cores, on a bounded sample of the same workload.
# ---------------------------------------------------------------------------
def _oracle_job(args):
    """One piece of CPU-baseline work: the oracle's product (unpack the signs,
    dequantise in FP64, matmul) on the row tiles of one packed sub-buffer.
    Runs in the bench process or in a spawned one (which has no torch)."""
    from oracle import bcq_oracle as O
    sub, q, m_sub, n, alpha_rows, x, g = args
    t = time.perf_counter()
    y = O.bcq_matmul(x, O.unpack_bcq(sub, q, m_sub, n), alpha_rows, g)
    return y, time.perf_counter() - t


def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


class OraclePool:
    """A pool of `cores` spawned processes running _oracle_job (spawned, not
    forked: a child forked from a process that has used CUDA can hang).  One
    trivial job per worker starts them all before any timing."""

    def __init__(self, cores: int):
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        import numpy as np
        self.cores = cores
        self.ex = ProcessPoolExecutor(max_workers=cores, mp_context=mp.get_context("spawn"))
        tiny = (np.zeros(4096, dtype=np.uint8), 1, 32, 1024, np.zeros((1, 8, 32), dtype=np.float16),
                np.zeros((1, 1024), dtype=np.float16), 128)
        list(self.ex.map(_oracle_job, [tiny] * cores))

    def run(self, jobs):
        """Wall seconds for all jobs on the pool, and their outputs."""
        t = time.perf_counter()
        res = list(self.ex.map(_oracle_job, jobs))
        return time.perf_counter() - t, [r[0] for r in res]

    def close(self):
        self.ex.shutdown()


def _tile_job(packed_host, alpha_host, x, q, m, n, g, tiles):
    """Job arguments for the row tiles `tiles` of one linear, and the rows they cover."""
    import numpy as np
    ns, mt = -(-n // 1024), -(-m // 32)
    blocks = packed_host.numpy().reshape(ns, mt, q * 4096)
    sub = np.ascontiguousarray(blocks[:, tiles]).reshape(-1)
    rows = (32 * np.asarray(tiles)[:, None] + np.arange(32)[None, :]).reshape(-1)
    rows = rows[rows < m]
    return (sub, q, rows.size, n, np.ascontiguousarray(alpha_host.numpy()[:, :, rows]), x, g), rows


def cpu_baseline_and_parity(mats, q: int, g: int, batch: int, rows: int, y_timed, io):
    """The oracle on sampled row tiles of the bench's own weights and inputs.

    1 thread: `rows` rows (whole 32-row tiles, the first and last tile
    included) of each linear, timed, and the outputs compared with the
    timed region's last y (the parity field).  All host cores: a pool of
    spawned processes, one tile per job, about four tiles per core."""
    import numpy as np
    from threadpoolctl import threadpool_limits
    from tests._tol import compare
    rng = np.random.default_rng(7)
    k = max(2, rows // 32)
    jobs, picks = [], []
    for mt_ in mats:
        mtiles = -(-mt_["m"] // 32)
        inner = rng.choice(np.arange(1, mtiles - 1), size=min(k - 2, mtiles - 2), replace=False)
        tiles = np.unique(np.r_[0, mtiles - 1, inner])
        job, r = _tile_job(mt_["packed_host"], mt_["alpha_host"], mt_["x_host"].numpy(), q, mt_["m"], mt_["n"],
                           g, tiles)
        jobs.append(job)
        picks.append(r)
    with threadpool_limits(limits=1):
        res = [_oracle_job(j) for j in jobs]
    secs1 = sum(t for _, t in res)
    bytes1 = sum(algorithmic_bytes(j[2], j[3], q, g, batch) for j in jobs)
    # Parity of the timed step's outputs on the sampled rows.
    per, ok_all, yo = {}, True, 0
    y_all = y_timed.numpy()
    for mt_, (y_ref, _), r, job in zip(mats, res, picks, jobs):
        got = y_all[yo: yo + batch * mt_["m"]].reshape(batch, mt_["m"])[:, r]
        ok, st = compare(got, y_ref, job[4], job[5], mt_["n"])
        per[mt_["name"]] = {"rows": int(r.size), "rel_l2": st["rel_l2"],
                            "max_abs_over_bound": round(st["max_abs_over_bound"], 5)}
        ok_all = ok_all and ok
        yo += batch * mt_["m"]
    parity = {"ok": bool(ok_all), "per_linear": per,
              "what": "the last graph-replayed step's y against the FP64 oracle on the sampled rows "
                      "(rel-L2 <= 1e-3 and per-output max-abs bound)"}
    # All host cores: one tile per job, about four per core, spread over the linears.
    cores = min(_host_cores(), 64)
    pool = OraclePool(cores)
    try:
        per_lin = max(1, -(-4 * cores // len(mats)))
        jobs_all = []
        for mt_ in mats:
            mtiles = -(-mt_["m"] // 32)
            for t in rng.choice(mtiles, size=min(per_lin, mtiles), replace=False):
                jobs_all.append(_tile_job(mt_["packed_host"], mt_["alpha_host"], mt_["x_host"].numpy(), q, mt_["m"],
                                          mt_["n"], g, [int(t)])[0])
        wall, _ = pool.run(jobs_all)
    finally:
        pool.close()
    bytes_all = sum(algorithmic_bytes(j[2], j[3], q, g, batch) for j in jobs_all)
    base = {"value": round(bytes_all / wall / 1e9, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "seconds": round(wall, 2), "host_cores": _host_cores(), "cpu_model": _cpu_model(),
            "sample": f"{len(jobs_all)} row tiles (32 rows each) of the 4 layer linears of this run's weights "
                      f"and x (q={q}, g={g}, batch {batch}), one tile per job on {cores} spawned processes: "
                      "oracle unpack + FP64 dequantise + matmul",
            "single_thread": {"value": round(bytes1 / secs1 / 1e9, 6), "cores": 1, "seconds": round(secs1, 2),
                              "sample": f"{sum(r.size for r in picks)} rows ({k} tiles of each linear, first "
                                        "and last included), one thread"}}
    return base, parity
def _oracle_sample(q: int, batch: int, rows_per_matrix: int, seed: int):
    """Timed oracle work on `rows_per_matrix` sampled rows of each of the four linears.

    Returns (seconds, algorithmic bytes of the sampled rows)."""
    import numpy as np
    from oracle import bcq_oracle as O
    w = S.WORKLOADS[WORKLOAD]
    rng = np.random.default_rng(seed)
    secs, nbytes = 0.0, 0
    for sh in w.shapes:
        gen = S.generator(seed * 31 + sh.m)
        mt = -(-sh.m // 32)
        # Only the row tiles the sample touches are drawn: rows 32*R + l.
        tiles = np.sort(rng.choice(mt, size=max(1, rows_per_matrix // 32), replace=False))
        m_s = 32 * tiles.size
        packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m_s, sh.n)).numpy()
        alpha = S.draw_alpha(gen, q, m_s, sh.n, w.g, w.alpha_sigma).numpy()
        x = S.draw_x(gen, batch, sh.n).numpy()
        t = time.perf_counter()
        signs = O.unpack_bcq(packed, q, m_s, sh.n)
        y = O.bcq_matmul(x, signs, alpha, w.g)
        secs += time.perf_counter() - t
        assert np.all(np.isfinite(y))
        nbytes += algorithmic_bytes(m_s, sh.n, q, w.g, batch)
    return secs, nbytes


def _random_tile_jobs(q: int, batch: int, n_tiles: int, seed: int):
    """Oracle jobs of one random 32-row tile each, spread over the 4 layer
    linears, drawn on the CPU with the workload's distributions."""
    w = S.WORKLOADS[WORKLOAD]
    jobs = []
    for t in range(n_tiles):
        sh = w.shapes[t % len(w.shapes)]
        gen = S.generator(seed * 7919 + t)
        packed = S.draw_random_bytes(gen, -(-sh.n // 1024) * q * 4096).numpy()   # one row tile, every slice
        alpha = S.draw_alpha(gen, q, 32, sh.n, w.g, w.alpha_sigma).numpy()
        x = S.draw_x(gen, batch, sh.n).numpy()
        jobs.append((packed, q, 32, sh.n, alpha, x, w.g))
    return jobs


def run_reference(args):
    """The reference arm: the FP64 oracle as it stands on the host cores (a
    pool of spawned processes, one 32-row tile per job, one job per core and
    step), on random tiles of the same four linears."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return
    q, batch = args.q, args.batch
    g = S.WORKLOADS[WORKLOAD].g
    from threadpoolctl import threadpool_limits
    cores = min(_host_cores(), 64)
    nb = lambda jobs: sum(algorithmic_bytes(j[2], j[3], q, g, batch) for j in jobs)
    pool = OraclePool(cores)
    try:
        for k in range(args.warmup):
            pool.run(_random_tile_jobs(q, batch, cores, seed=100 + k))
        secs, nbytes = 0.0, 0
        for k in range(args.steps):
            jobs = _random_tile_jobs(q, batch, cores, seed=200 + k)
            wall, _ = pool.run(jobs)
            secs += wall
            nbytes += nb(jobs)
    finally:
        pool.close()
    one = _random_tile_jobs(q, batch, 4, seed=999)
    with threadpool_limits(limits=1):
        secs1 = sum(_oracle_job(j)[1] for j in one)
    value = nbytes / secs / 1e9
    sample = (f"{cores} random 32-row tiles of the 4 layer linears per step (q={q}, g={g}, batch {batch}), one "
              f"tile per job on {cores} spawned processes: oracle unpack + FP64 dequantise + matmul")
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "OPT-175B decoder-layer linears (QKV 36864x12288, out 12288x12288, "
                               f"FC1 49152x12288, FC2 12288x49152), BCQ q={q}, g={g}, batch {batch}",
                   "q": q, "g": g, "batch": batch, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "host_cores": _host_cores(), "cpu_model": _cpu_model(),
                         "single_thread": {"value": round(nb(one) / secs1 / 1e9, 6), "cores": 1,
                                           "seconds": round(secs1, 2),
                                           "sample": "one random tile of each linear, one thread"}},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# BCQ fitting (the step that produces the weights): FP16 W -> signs + scales.
# ---------------------------------------------------------------------------
FIT_METRIC = "BCQ fit throughput: FP16 weights fitted per second (greedy + alternating least squares)"


def _fit_profile(kernel_hash: str, variant: str):
    """Warp instructions (and DRAM bytes) per weight of fit_bcq_kernel, plain or
    grid, from the committed ncu summary (null unless taken on this kernel source)."""
    try:
        with open(os.path.join(ROOT, "profiles", "fit_bcq_instructions.json")) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    return d.get(variant) if d.get("kernel_hash") == kernel_hash else None


def _fit_hash() -> str:
    return _code_hash(("fit.cu",))


def run_fit(args):
    from weight_only_quantized_bcq_b200 import lutgemm
    world, rank, local = _dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)
    m, n, q, g, iters = args.fit_m, args.fit_n, args.q, args.fit_g, args.fit_iters
    w_host = S.draw_weights(S.generator(rank_seed(rank)), m, n, 0.02).pin_memory()
    w = w_host.to(device)
    signs = torch.empty((q, m, n), dtype=torch.int8, device=device)
    alpha = torch.empty((q, n // g, m), dtype=torch.float16, device=device)
    offset = torch.empty((n // g, m), dtype=torch.float32, device=device)
    lib = lutgemm.lib()
    import ctypes

    def fit_once(src):
        if args.fit_grid:
            st = lib.lutgemm_fit_bcq_grid(ctypes.c_void_p(src.data_ptr()), q, m, n, g, iters,
                                          ctypes.c_void_p(signs.data_ptr()), ctypes.c_void_p(alpha.data_ptr()),
                                          ctypes.c_void_p(offset.data_ptr()), None,
                                          ctypes.c_void_p(stream.cuda_stream))
        else:
            st = lib.lutgemm_fit_bcq(ctypes.c_void_p(src.data_ptr()), q, m, n, g, iters,
                                     ctypes.c_void_p(signs.data_ptr()), ctypes.c_void_p(alpha.data_ptr()), None,
                                     ctypes.c_void_p(stream.cuda_stream))
        if st != 0:
            raise RuntimeError(lutgemm.status_string(st))

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        fit_once(w)
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        barrier()
        t0.record(stream)
        for _ in range(args.steps):
            fit_once(w)
        t1.record(stream)
        barrier()
    region_ms = max_over_ranks(pg, t0.elapsed_time(t1), device)
    # End to end: W from pinned host memory in, signs and scales back out, per step.
    s_host = torch.empty(signs.shape, dtype=torch.int8).pin_memory()
    a_host = torch.empty(alpha.shape, dtype=torch.float16).pin_memory()
    o_host = torch.empty(offset.shape, dtype=torch.float32).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        w.copy_(w_host, non_blocking=True)
        fit_once(w)
        s_host.copy_(signs, non_blocking=True)
        a_host.copy_(alpha, non_blocking=True)
        if args.fit_grid:
            o_host.copy_(offset, non_blocking=True)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1), device)
    weights = m * n
    value = weights * args.steps * world / (region_ms * 1e-3) / 1e9
    e2e = weights * args.steps * world / (e2e_ms * 1e-3) / 1e9
    if rank == 0:
        sm = torch.cuda.get_device_properties(device).multi_processor_count
        clk = clocks.summary()
        variant = "grid" if args.fit_grid else "plain"
        prof = _fit_profile(_fit_hash(), variant)
        # Issue-slot roofline: 4 schedulers per SM, one warp instruction each per clock.
        peak = 4 * sm * (clk["sm_mhz"] or 1965.0) * 1e6 / 1e9
        roof = {"bound": "alu", "unit": "G warp-inst/s", "peak": round(peak, 1), "peak_kind":
                "derived: 4 issue slots x SMs x median SM clock under load", "kernel": "fit_bcq_kernel",
                "kernel_hash": _fit_hash(), "traffic": None}
        if prof:
            ach = prof["warp_inst_per_weight"] * weights * args.steps / (region_ms * 1e-3) / 1e9
            roof.update({"achieved": round(ach, 1), "frac": round(ach / peak, 4),
                         "traffic": prof.get("dram_bytes_per_weight", 0) * weights or None})
        else:
            roof.update({"achieved": None, "frac": None})
        out = {
            "metric": FIT_METRIC, "value": round(value, 2), "unit": "Gweights/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(region_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": (f"BCQ fit of FP16 W {m}x{n} ~ N(0, 0.02): q={q}, g={g}, {iters} rounds"
                                    + (", variable grid (planes + one constant per group)" if args.fit_grid
                                       else "")),
                       "m": m, "n": n, "q": q, "g": g, "iters": iters, "grid": bool(args.fit_grid),
                       "l2": f"no flush: W is {2 * m * n / 1e6:.0f} MB (> 126 MB L2)",
                       "parallelism": "replicas" if world == 1 else f"replicas{world}"},
            "roofline": roof,
            "e2e": {"value": round(e2e, 2), "unit": "Gweights/s", "h2d_bytes_per_step": 2 * m * n,
                    "d2h_bytes_per_step": q * m * n + 2 * q * (n // g) * m
                    + (4 * (n // g) * m if args.fit_grid else 0)},
            "gpu_launches": args.steps,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_fit_baseline(q, g, iters, n, args.fit_cpu_rows, args.fit_grid)
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def cpu_fit_baseline(q: int, g: int, iters: int, n: int, rows: int, grid: bool = False):
    from threadpoolctl import threadpool_limits
    from oracle import bcq_oracle as O
    w = S.draw_weights(S.generator(77), rows, n, 0.02).numpy()
    fit = O.fit_bcq_grid if grid else O.fit_bcq
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        fit(w, q, g, iters)
        secs = time.perf_counter() - t
    return {"value": round(rows * n / secs / 1e9, 6), "unit": "Gweights/s", "cores": 1, "kind": "oracle",
            "seconds": round(secs, 2),
            "sample": f"{rows} rows x {n} of the same W distribution, oracle {fit.__name__} (FP64), one thread"}


# ---------------------------------------------------------------------------
# Large-batch path on the tensor cores (lutgemm_run_tc): the layer's linears at
# a prompt-phase batch.  One plane product per weight and batch column is two
# flops; the tensor cores execute q of them per weight (one per plane), which
# is the work this path's roofline counts.
# ---------------------------------------------------------------------------
TC_METRIC = ("BCQ tensor-core path (lutgemm_run with LUTGEMM_ALLOW_TENSOR_CORES): plane TFLOP/s "
             "(2*q*m*n*batch per matmul) over the OPT-175B layer's linears at prompt-phase batch")
TC_SOURCES = ("tc_gemm.cu",)


def _tc_hash() -> str:
    return _code_hash(TC_SOURCES)


def _tc_peak():
    """Dense fp16/bf16 tensor peak: measured (fp16 runs at the bf16 rate), the
    sustained figure since the timed region is seconds of back-to-back launches."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1400.0, 1590.0, "fallback"


def _tc_traffic(kernel_hash: str, names, batch: int):
    path = os.path.join(ROOT, "profiles", "tc_gemm_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    per = d.get("per_shape_bytes", {})
    if d.get("kernel_hash") != kernel_hash or d.get("batch") != batch or not all(n in per for n in names):
        return None
    return sum(per[n] for n in names) / len(names)


def run_tc(args):
    from weight_only_quantized_bcq_b200 import lutgemm
    world, rank, local = _dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist
    q, batch = args.q, args.tc_batch
    w = S.WORKLOADS[WORKLOAD]
    g = w.g
    gen = S.generator(rank_seed(rank))
    # All linears' x and y in one buffer each (views per linear): one copy each way per e2e step.
    xs, ys = sum(batch * sh.n for sh in w.shapes), sum(batch * sh.m for sh in w.shapes)
    io = {"x_host": torch.empty(xs, dtype=torch.float16).pin_memory(),
          "x": torch.empty(xs, dtype=torch.float16, device=device),
          "y_host": torch.empty(ys, dtype=torch.float32).pin_memory(),
          "y": torch.empty(ys, dtype=torch.float32, device=device)}
    mats = []
    xo = yo = 0
    for sh in w.shapes:
        x_host = io["x_host"][xo: xo + batch * sh.n].view(batch, sh.n)
        x_host.copy_(S.draw_x(gen, batch, sh.n))
        mats.append({"name": sh.name, "m": sh.m, "n": sh.n,
                     "packed": S.draw_random_bytes(gen, lutgemm.packed_bytes(q, sh.m, sh.n)).to(device),
                     "alpha": S.draw_alpha(gen, q, sh.m, sh.n, g, w.alpha_sigma).to(device),
                     "x_host": x_host, "x": io["x"][xo: xo + batch * sh.n].view(batch, sh.n),
                     "y": io["y"][yo: yo + batch * sh.m].view(batch, sh.m),
                     "y_host": io["y_host"][yo: yo + batch * sh.m].view(batch, sh.m),
                     "ws": None if args.tc_direct else lutgemm.new_workspace(sh.m, sh.n, batch, q, g, device=device)})
        xo += batch * sh.n
        yo += batch * sh.m
    io["x"].copy_(io["x_host"])
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)

    def one(mt):
        # The library's tensor-core path as a caller gets it: lutgemm_run with
        # the tensor cores allowed (its cost model picks K splits for short
        # matrices); --tc-direct calls lutgemm_run_tc (one split) instead.
        if args.tc_direct:
            lutgemm.run_tc(mt["packed"], mt["alpha"], mt["x"], mt["m"], mt["n"], q, g, y=mt["y"], stream=stream)
        else:
            lutgemm.run(mt["packed"], mt["alpha"], mt["x"], mt["m"], mt["n"], q, g, y=mt["y"], workspace=mt["ws"],
                        allow_tensor_cores=True, stream=stream)

    def step(events=None):
        for i, mt in enumerate(mats):
            if events is not None:
                events[i][0].record(stream)
            one(mt)
            if events is not None:
                events[i][1].record(stream)

    def e2e_step():
        io["x"].copy_(io["x_host"], non_blocking=True)
        for mt in mats:
            one(mt)
        io["y_host"].copy_(io["y"], non_blocking=True)

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        barrier()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        barrier()
    region_ms = max_over_ranks(pg, t0.elapsed_time(t1), device)
    per_launch = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
                   for _ in mats] for _ in range(args.steps)]
    for k in range(args.steps):
        step(per_launch[k])
    barrier()
    us_per = {mt["name"]: 1e3 * statistics.median(per_launch[k][i][0].elapsed_time(per_launch[k][i][1])
                                                  for k in range(args.steps))
              for i, mt in enumerate(mats)}
    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1), device)

    flops = {mt["name"]: 2 * q * mt["m"] * mt["n"] * batch for mt in mats}
    step_flops = sum(flops.values())
    value = step_flops * args.steps * world / (region_ms * 1e-3) / 1e12
    e2e = step_flops * args.steps * world / (e2e_ms * 1e-3) / 1e12
    # The region holds the tensor-core launches and, where K is split, their
    # reduces: the whole region is charged to tc_gemm_kernel (a lower bound on
    # its rate).
    achieved = step_flops * args.steps / (region_ms * 1e-3) / 1e12
    peak, peak_burst, peak_kind = _tc_peak()
    khash = _tc_hash()
    if rank == 0:
        clk = clocks.summary()
        out = {
            "metric": TC_METRIC, "value": round(value, 1), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(region_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {
                "workload": "OPT-175B decoder-layer linears (QKV 36864x12288, out 12288x12288, "
                            f"FC1 49152x12288, FC2 12288x49152), BCQ q={q}, g={g}, batch {batch}, tensor cores",
                "q": q, "g": g, "batch": batch,
                "l2": "no flush: each step streams 765 MB (> 126 MB L2) of distinct weights",
                "parallelism": "replicas" if world == 1 else f"replicas{world} (one layer per GPU)",
            },
            "us_per_matmul": {k: round(v, 1) for k, v in us_per.items()},
            "us_per_matmul_note": "median of isolated launches (events around each launch)",
            "tflops_per_matmul": {k: round(flops[k] / (us_per[k] * 1e-6) / 1e12, 1) for k in us_per},
            "dense_equivalent_tflops": round(value / q, 1),
            "dense_equivalent_note": "2*m*n*batch per matmul: the flops of the same product on dequantised weights",
            "roofline": {
                "bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": _tc_traffic(khash, list(flops), batch),
                "peak_kind": f"{peak_kind} bf16 sustained (fp16 dense rate = bf16); burst {peak_burst}",
                "frac_of_burst": round(achieved / peak_burst, 4),
                "kernel": "tc_gemm_kernel", "kernel_hash": khash,
            },
            "e2e": {"value": round(e2e, 1), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": io["x_host"].numel() * 2,
                    "d2h_bytes_per_step": io["y_host"].numel() * 4,
                    "copies_per_step": "one H2D of all x, one D2H of all y (pinned host buffers)"},
            "gpu_launches": args.steps * sum(1 + (0 if args.tc_direct else int(tc_splits(mt["m"], mt["n"], batch, q) > 1))
                                             for mt in mats),
            "gpu_launches_note": "tc_gemm_kernel per matmul, plus the split-K reduce where the library splits K",
            "clocks": clk,
        }
        out["config"]["call"] = "lutgemm_run_tc" if args.tc_direct else "lutgemm_run + LUTGEMM_ALLOW_TENSOR_CORES"
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_tc_baseline(q, batch, args.tc_cpu_rows)
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def tc_splits(m: int, n: int, batch: int, q: int) -> int:
    """K splits of lutgemm_run's tensor-core plan on this device (for launch counting)."""
    from weight_only_quantized_bcq_b200 import lutgemm
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return lutgemm.tc_plan(m, n, batch, q, sms)


def cpu_tc_baseline(q: int, batch: int, rows: int):
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        secs, _ = _oracle_sample(q, batch, rows, seed=11)
    fl = sum(2 * q * (32 * max(1, rows // 32)) * sh.n * batch for sh in S.WORKLOADS[WORKLOAD].shapes)
    return {"value": round(fl / secs / 1e12, 8), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "seconds": round(secs, 2),
            "sample": f"{32 * max(1, rows // 32)} rows of each of the 4 layer linears (q={q}, g=128, batch {batch}): "
                      "oracle unpack + FP64 dequantise + matmul, one thread; plane flops 2*q*rows*n*batch"}


# ---------------------------------------------------------------------------
# Config sweep: isolated and back-to-back time of every parity config shape
# (OPT-175B linears at batch 1..32, LLaMA-70B linears at batch 1..8), one
# JSON line each, against both rooflines (HBM and shared-memory lookups).
# ---------------------------------------------------------------------------
SWEEP = [("opt175b_qkv", 36864, 12288, 3, 128, (1, 2, 4, 8, 16, 32)),
         ("opt175b_fc1", 49152, 12288, 3, 128, (1, 2, 4, 8, 16, 32)),
         ("opt175b_fc2", 12288, 49152, 3, 128, (1, 2, 4, 8, 16, 32)),
         ("llama70b_qkvo", 8192, 8192, 2, 64, (1, 2, 4, 8)),
         ("llama70b_up", 28672, 8192, 2, 64, (1, 2, 4, 8)),
         ("llama70b_down", 8192, 28672, 2, 64, (1, 2, 4, 8))]


def _graph_us(fn, calls: int, stream, replays: int = 3) -> float:
    """Microseconds per call of fn(0), fn(1), ..., fn(calls-1) captured in one
    CUDA graph and replayed back to back: the device time of consecutive
    launches, with no host launch overhead between them."""
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(calls):
            fn(i)
    graph.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(replays):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    del graph
    return t0.elapsed_time(t1) * 1e3 / (calls * replays)


def run_sweep(args):
    from weight_only_quantized_bcq_b200 import lutgemm
    torch.cuda.set_device(0)
    peak, _ = _peaks()
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    for name, m, n, q, g, batches in SWEEP:
        gen = S.generator(3)
        reps = 3   # distinct weight copies: consecutive launches miss L2
        bufs = [S.draw_random_bytes(gen, lutgemm.packed_bytes(q, m, n)).cuda() for _ in range(reps)]
        alpha = S.draw_alpha(gen, q, m, n, g, 0.02).cuda()
        packed_scales = g % 128 == 0 or g == 64
        scales = lutgemm.pack_scales(alpha, m, n, g) if packed_scales else alpha
        for b in batches:
            x = S.draw_x(gen, b, n).cuda()
            ws = lutgemm.new_workspace(m, n, b, q, g)
            y = torch.empty((b, m), device="cuda")

            def run(i):
                lutgemm.run(bufs[i % reps], scales, x, m, n, q, g, y=y, workspace=ws,
                            scales_packed=packed_scales, stream=stream)
            for i in range(max(3, args.warmup)):
                run(i)
            torch.cuda.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(21)]
            for i, (a_, b_) in enumerate(ev):
                a_.record(stream)
                run(i)
                b_.record(stream)
            torch.cuda.synchronize()
            iso = statistics.median(a_.elapsed_time(b_) for a_, b_ in ev) * 1e3
            b2b = _graph_us(run, 30, stream)
            nbytes = algorithmic_bytes(m, n, q, g, b)
            # Lookups: q*m*n/8 table reads per batch column; one conflict-free
            # wavefront (32 reads) per clock per SM at the measured clock.
            lookups = q * m * n // 8 * b
            smem_floor = lookups / 32 / sm / 1.965e3
            line = {"config": name, "m": m, "n": n, "q": q, "g": g, "batch": b,
                    "scales": "unit-major" if packed_scales else "[q][n/g][m]",
                    "us_isolated": round(iso, 1), "us_back_to_back": round(b2b, 1),
                    "note": "isolated: events around one eager launch (includes launch latency); back to back: "
                            "30 launches in a CUDA graph, three weight copies in turn",
                    "gbs_back_to_back": round(nbytes / (b2b * 1e-6) / 1e9, 1),
                    "hbm_floor_us": round(nbytes / (peak * 1e3), 1),
                    "smem_floor_us": round(smem_floor, 1),
                    "frac_of_binding_floor": round(max(nbytes / (peak * 1e3), smem_floor) / b2b, 3)}
            if b >= 8 and n % 128 == 0 and g % 64 == 0:
                # The same product on the tensor cores (lutgemm_run_tc), back to back.
                def run_tc(i):
                    lutgemm.run_tc(bufs[i % reps], alpha, x, m, n, q, g, y=y, stream=stream)
                for i in range(3):
                    run_tc(i)
                line["us_tensor_cores_back_to_back"] = round(_graph_us(run_tc, 30, stream), 1)
                # lutgemm_run with LUTGEMM_ALLOW_TENSOR_CORES: the library's own choice
                # (lookups, or tensor cores with K splits and the reduce).
                def run_auto(i):
                    lutgemm.run(bufs[i % reps], alpha, x, m, n, q, g, y=y, workspace=ws, allow_tensor_cores=True,
                                stream=stream)
                for i in range(3):
                    run_auto(i)
                line["us_auto_back_to_back"] = round(_graph_us(run_auto, 30, stream), 1)
            print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# One matrix split over the ranks (--parallel): OPT-175B FC1 by rows with an
# all-gather, FC2 by inputs with an all-reduce, or the FC1 -> FC2 block with
# FC1 by rows and FC2 by inputs and one all-reduce.  Total work is fixed as N
# grows (strong scaling).  The exchange is NCCL (torch.distributed); every
# kernel reads only its own GPU's memory.
# ---------------------------------------------------------------------------
PARALLEL_SHAPES = {"fc1": (49152, 12288), "fc2": (12288, 49152)}


def parallel_plans(mode: str, q: int, g: int, world: int, rank: int, shapes=None):
    """The shard plans of this rank for a --parallel mode: rows (FC1), inputs
    (FC2) or paired (FC1 by rows, then FC2 by inputs over the same range)."""
    from weight_only_quantized_bcq_b200 import sharded as T
    shp = shapes or PARALLEL_SHAPES
    (m1, n1), (m2, n2) = shp["fc1"], shp["fc2"]
    if mode == "rows":
        return [T.plan_rows(m1, n1, q, g, world, rank)]
    if mode == "inputs":
        return [T.plan_inputs(m2, n2, q, g, world, rank)]
    if mode == "paired":
        assert n2 == m1
        return list(T.plan_paired(m1, n1, m2, q, g, world, rank))
    raise ValueError(mode)


def parallel_bytes(plans, batch: int):
    """(algorithmic bytes of the whole matrices, of this rank's shards) per step."""
    whole = sum(algorithmic_bytes(p.m, p.n, p.q, p.g, batch) for p in plans)
    mine = sum(algorithmic_bytes(p.local_m, p.local_n, p.q, p.g, batch) for p in plans)
    return whole, mine


def parallel_step(mode: str, lins, x):
    """One step of a --parallel mode: the shard products and their exchange."""
    from weight_only_quantized_bcq_b200 import sharded as T
    if mode == "paired":
        return T.paired_block(lins[0], lins[1], x)
    return lins[0](x)


def run_parallel(args):
    import datetime
    import torch.distributed as dist
    from weight_only_quantized_bcq_b200 import lutgemm
    from weight_only_quantized_bcq_b200 import sharded as T
    world, rank, local = _dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if "MASTER_ADDR" not in os.environ:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT="29533")
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120),
                            device_id=device)
    q, batch, g = args.q, args.batch, S.WORKLOADS[WORKLOAD].g
    plans = parallel_plans(args.parallel, q, g, world, rank)
    gen = S.generator(rank_seed(rank))
    lins = []
    for p in plans:
        packed = S.draw_random_bytes(gen, lutgemm.packed_bytes(q, p.local_m, p.local_n)).to(device)
        alpha = S.draw_alpha(gen, q, p.local_m, p.local_n, g, 0.02).to(device)
        lins.append(T.ShardedLinear.from_packed(p, packed, alpha, batch=batch))
    # Every rank draws the same x (same seed): the input the matrix multiplies.
    n_in = plans[0].n
    x_host = S.draw_x(S.generator(77), batch, n_in).pin_memory()
    x = x_host.to(device)
    x_in = T.take_input_slice(plans[0], x) if args.parallel == "inputs" else x
    stream = torch.cuda.current_stream()

    def barrier():
        torch.cuda.synchronize()
        dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, steps):
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            fn()
        t1.record(stream)
        barrier()
        return max_over_ranks(dist, t0.elapsed_time(t1), device)

    for _ in range(args.warmup):
        parallel_step(args.parallel, lins, x_in)
    # The step as a CUDA graph (shard products and the NCCL collective), so
    # the host's launch overhead is not timed; --graph-steps 0: eager.
    graph = None
    if args.graph_steps > 0:
        side = torch.cuda.Stream(device=device)
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            y_graph = parallel_step(args.parallel, lins, x_in)
        stream.wait_stream(side)
        graph.replay()
        barrier()
    step_fn = graph.replay if graph is not None else (lambda: parallel_step(args.parallel, lins, x_in))
    with ClockSampler(torch.cuda.current_device()) as clocks:
        region_ms = timed(step_fn, args.steps)
    y = y_graph if graph is not None else parallel_step(args.parallel, lins, x_in)

    # The products alone (no exchange), to give the collective's share.
    def products_only():
        if args.parallel == "paired":
            h = lins[0].local_product(x_in)
            lins[1].local_product(h.to(torch.float16))
        else:
            lins[0].local_product(x_in if args.parallel == "rows" else x_in)
    prod_ms = timed(products_only, args.steps)
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()

    def e2e_step():
        x.copy_(x_host, non_blocking=True)
        xi = T.take_input_slice(plans[0], x) if args.parallel == "inputs" else x
        y_host.copy_(parallel_step(args.parallel, lins, xi), non_blocking=True)
    e2e_ms = timed(e2e_step, args.steps)

    if graph is not None:
        del graph          # a graph holding NCCL work is released before the group is destroyed
    whole, mine = parallel_bytes(plans, batch)
    value = whole * args.steps / (region_ms * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    if rank == 0:
        names = {"rows": "OPT-175B FC1 (49152x12288) split by rows, all-gather of y",
                 "inputs": "OPT-175B FC2 (12288x49152) split by inputs, all-reduce of y",
                 "paired": "OPT-175B FC1 -> FC2 block, FC1 by rows and FC2 by inputs, one all-reduce"}
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(region_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": names[args.parallel] + f", BCQ q={q}, g={g}, batch {batch}", "q": q, "g": g,
                       "batch": batch, "parallelism": f"tp{world} ({args.parallel})",
                       "bytes_per_step_whole": whole, "bytes_per_step_rank0": mine,
                       "l2": "no flush: every step streams each shard's weights once; a shard below 126 MB "
                             "may stay in L2 at large N",
                       "launch": ("each step a CUDA graph replay (shard products + NCCL collective)"
                                  if args.graph_steps > 0 else "eager launches") +
                                 "; collectives by torch.distributed (NCCL)"},
            "products_ms_per_step": round(prod_ms / args.steps, 5),
            "collective_share": round(max(0.0, 1.0 - prod_ms / region_ms), 4),
            "roofline": {"bound": "hbm", "achieved": round(mine * args.steps / (region_ms * 1e-3) / 1e9, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(mine * args.steps / (region_ms * 1e-3) / 1e9 / peak, 4), "traffic": None,
                         "peak_kind": peak_kind, "kernel": "lut_gemm_kernel (one rank's shards, exchange included)"},
            "e2e": {"value": round(whole * args.steps / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                    "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": y_host.numel() * 4},
            "gpu_launches": args.steps * sum(1 + (p.local_n > 1024) for p in plans),
            "gpu_launches_note": "lookup kernel and split-K reduce per shard product; NCCL kernels not counted",
            "clocks": clocks.summary(),
        }
        print(json.dumps(out), flush=True)
    dist.barrier()
    dist.destroy_process_group()


# ---------------------------------------------------------------------------
# Mixed storage (2/4/16-bit in one matrix): the LLaMA-70B-shaped linears with
# 2-plane blocks, a fraction of 4-plane blocks and sparse fp16 outliers,
# through lutgemm_run_mixed.
# ---------------------------------------------------------------------------
MIXED_METRIC = "Mixed 2/4/16-bit LUT-GEMM (lutgemm_run_mixed): achieved HBM GB/s at batch 1"
MIXED_SHAPES = (("llama70b_qkvo", 8192, 8192), ("llama70b_up", 28672, 8192), ("llama70b_down", 8192, 28672))


def _mixed_layer(q_max, g, batch, frac_hi, density, seed, device, reps, packed_scales=True):
    from weight_only_quantized_bcq_b200 import lutgemm
    from weight_only_quantized_bcq_b200.roofline import mixed_algorithmic_bytes
    gen = S.generator(seed)
    mats = []
    for name, m, n in MIXED_SHAPES:
        bp = S.draw_block_planes(gen, m, n, frac_hi, lo=2, hi=q_max)
        boff_h = lutgemm.mixed_offsets(bp, q_max, m, n)
        nbytes = int(boff_h[-1]) * 4096
        copies_h = [S.draw_random_bytes(gen, nbytes) for _ in range(reps)]
        alpha_h = S.draw_alpha(gen, q_max, m, n, g, 0.03)
        x_h = S.draw_x(gen, batch, n, outlier_frac=0.001).pin_memory()
        rp, col, val = S.draw_outliers(gen, m, n, density)
        optr, oent = lutgemm.pack_outliers(rp, col, val, m, n)
        boff_d = boff_h.to(device)
        alpha_d = alpha_h.to(device)
        if packed_scales:
            alpha_d = lutgemm.pack_scales_mixed(alpha_d, boff_d, m, n, g)
        mats.append({"name": name, "m": m, "n": n, "bp": bp, "boff": boff_d,
                     "copies": [c.to(device) for c in copies_h], "packed_host": copies_h[-1],
                     "alpha": alpha_d, "alpha_host": alpha_h, "x_host": x_h, "x": x_h.to(device),
                     "outliers_host": (rp, col, val), "optr": optr.to(device), "oent": oent.to(device),
                     "y": torch.empty((batch, m), dtype=torch.float32, device=device),
                     "y_host": torch.empty((batch, m), dtype=torch.float32).pin_memory(),
                     "ws": lutgemm.new_workspace(m, n, batch, q_max, g, device=device),
                     "bytes": mixed_algorithmic_bytes(bp.numpy(), m, n, g, batch, col.numel()),
                     "nnz": col.numel(), "avg_planes": float(bp.float().mean())})
    return mats


def run_mixed_workload(args):
    from weight_only_quantized_bcq_b200 import lutgemm
    world, rank, local = _dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist
    q_max, g, batch = 4, 64, args.batch
    reps = 2      # weight copies used in turn: consecutive steps miss L2
    packed_scales = args.scales == "packed"
    mats = _mixed_layer(q_max, g, batch, args.mixed_hi, args.mixed_outliers, rank_seed(rank), device, reps,
                        packed_scales)
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)

    def one(mt, k):
        lutgemm.run_mixed(mt["copies"][k % reps], mt["boff"], mt["alpha"], mt["x"], mt["m"], mt["n"], q_max, g,
                          optr=mt["optr"], oent=mt["oent"], y=mt["y"], workspace=mt["ws"],
                          scales_packed=packed_scales, stream=stream)

    def step(k, events=None):
        for i, mt in enumerate(mats):
            if events is not None:
                events[i][0].record(stream)
            one(mt, k)
            if events is not None:
                events[i][1].record(stream)

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    for k in range(args.warmup):
        step(k)
    barrier()
    # The timed steps are replays of a CUDA graph of `per_graph` steps (the
    # weight copies alternate inside it), as in the layer bench.
    per_graph = args.graph_steps if args.graph_steps > 0 and args.steps % args.graph_steps == 0 else 0
    graph = None
    if per_graph:
        if per_graph % reps:
            per_graph = reps * max(1, per_graph // reps)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for k in range(per_graph):
                step(k)
        graph.replay()
        barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_steps = args.steps if not per_graph else (args.steps // per_graph) * per_graph
    with ClockSampler(torch.cuda.current_device()) as clocks:
        barrier()
        t0.record(stream)
        if graph is not None:
            for _ in range(n_steps // per_graph):
                graph.replay()
        else:
            for k in range(n_steps):
                step(k)
        t1.record(stream)
        barrier()
    region_ms = max_over_ranks(pg, t0.elapsed_time(t1), device)
    if graph is not None:
        del graph
    k_last = (per_graph - 1) if per_graph else (n_steps - 1)
    y_timed = [mt["y"].cpu().clone() for mt in mats]
    b2b_us = {mt["name"]: _graph_us(lambda i, mt=mt: one(mt, i), 10, stream) for mt in mats}
    status = [lutgemm.workspace_status(mt["ws"]) for mt in mats]
    ev = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in mats]
          for _ in range(args.steps)]
    for k in range(args.steps):
        step(k, ev[k])
    barrier()
    us_per = {mt["name"]: 1e3 * statistics.median(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps))
              for i, mt in enumerate(mats)}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for k in range(args.steps):
        for mt in mats:
            mt["x"].copy_(mt["x_host"], non_blocking=True)
        step(k)
        for mt in mats:
            mt["y_host"].copy_(mt["y"], non_blocking=True)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1), device)
    step_bytes = sum(mt["bytes"] for mt in mats)
    value = step_bytes * n_steps * world / (region_ms * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    if rank == 0:
        out = {
            "metric": MIXED_METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": n_steps, "warmup": args.warmup, "ms_per_step": round(region_ms / n_steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "LLaMA-70B-shaped linears (8192x8192, 28672x8192, 8192x28672), mixed storage: "
                                   f"2-plane blocks, {args.mixed_hi:.3f} of blocks at 4 planes, "
                                   f"{100 * args.mixed_outliers:.2f}% fp16 outliers, g={g}, batch {batch}",
                       "q_max": q_max, "g": g, "batch": batch, "frac_4plane_blocks": args.mixed_hi,
                       "outlier_density": args.mixed_outliers, "bytes_per_step": step_bytes,
                       "scales": ("unit-major mixed layout, reordered once at load time (lutgemm_pack_scales_mixed)"
                                  if packed_scales else "[q_max][n/g][m]"),
                       "avg_planes": {mt["name"]: round(mt["avg_planes"], 3) for mt in mats},
                       "l2": f"two weight copies used in turn: {2 * step_bytes / 1e6:.0f} MB between reuses "
                             "(> 126 MB L2)",
                       "parallelism": "replicas" if world == 1 else f"replicas{world}"},
            "us_per_matmul": {k: round(v, 2) for k, v in us_per.items()},
            "us_per_matmul_note": "median of isolated launches (events around each eager launch)",
            "us_per_matmul_back_to_back": {k: round(v, 2) for k, v in b2b_us.items()},
            "gbs_per_matmul_back_to_back": {mt["name"]: round(mt["bytes"] / (b2b_us[mt["name"]] * 1e-6) / 1e9, 1)
                                            for mt in mats},
            "hbm_floor_us": {mt["name"]: round(mt["bytes"] / (peak * 1e3), 2) for mt in mats},
            "roofline": {"bound": "hbm", "achieved": round(step_bytes * n_steps / (region_ms * 1e-3) / 1e9, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(step_bytes * n_steps / (region_ms * 1e-3) / 1e9 / peak, 4),
                         "traffic": None, "peak_kind": peak_kind, "kernel": "lut_gemm_kernel (mixed)"},
            "e2e": {"value": round(step_bytes * args.steps * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                    "h2d_bytes_per_step": sum(mt["x_host"].numel() * 2 for mt in mats),
                    "d2h_bytes_per_step": sum(mt["y_host"].numel() * 4 for mt in mats)},
            "gpu_launches": n_steps * sum(1 + (mt["n"] > 1024) for mt in mats),
            "gpu_launches_note": "lookup kernel and split-K reduce per call",
            "device_status": status,
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"], out["parity"] = cpu_mixed_baseline(mats, q_max, g, batch, y_timed, k_last % reps)
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def cpu_mixed_baseline(mats, q_max, g, batch, y_timed, copy_index):
    """The oracle on 8 row tiles of each linear (first and last included) of
    the copy the last timed step used, one thread: its rate, and the timed
    outputs compared with it on those rows."""
    import numpy as np
    from threadpoolctl import threadpool_limits
    from oracle import bcq_oracle as O
    from tests._tol import compare
    rng = np.random.default_rng(3)
    secs, nbytes, per, ok_all = 0.0, 0, {}, True
    for mt_, y in zip(mats, y_timed):
        mtiles = -(-mt_["m"] // 32)
        tiles = np.unique(np.r_[0, mtiles - 1, rng.choice(mtiles, 6, replace=False)])
        packed = mt_["copies"][copy_index].cpu().numpy()
        outl = tuple(t.numpy() for t in mt_["outliers_host"])
        with threadpool_limits(limits=1):
            t = time.perf_counter()
            y_ref, rows = O.mixed_matmul_tiles(mt_["x_host"].numpy(), packed, mt_["bp"].numpy(),
                                               mt_["alpha_host"].numpy(), g, mt_["m"], mt_["n"], tiles, outl)
            secs += time.perf_counter() - t
        a = mt_["alpha_host"].numpy().astype(np.float64)[:, :, rows].copy()
        bp = mt_["bp"].numpy()
        for G in range(mt_["n"] // g):
            for ti, R in enumerate(tiles):
                a[bp[(G * g) // 1024, R]:, G, 32 * ti: 32 * ti + 32] = 0.0
        ok, st = compare(y.numpy()[:, rows], y_ref, a, mt_["x_host"].numpy(), mt_["n"])
        per[mt_["name"]] = {"rows": int(rows.size), "rel_l2": st["rel_l2"],
                            "max_abs_over_bound": round(st["max_abs_over_bound"], 5)}
        ok_all = ok_all and ok
        frac = rows.size / mt_["m"]
        nbytes += int(mt_["bytes"] * frac)
    base = {"value": round(nbytes / secs / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": round(secs, 2), "cpu_model": _cpu_model(),
            "sample": "8 row tiles of each linear of this run's weights: oracle unpack of each block, FP64 "
                      "mixed dequantise + outliers + matmul, one thread"}
    return base, {"ok": bool(ok_all), "per_linear": per,
                  "what": "the last timed step's y against the FP64 oracle on the sampled rows"}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["lutgemm", "reference"], default="lutgemm")
    ap.add_argument("--q", type=int, default=3)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--cpu-rows", type=int, default=512, help="rows per linear in the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph-steps", type=int, default=10,
                    help="steps per captured CUDA graph in the timed region (0: eager launches)")
    ap.add_argument("--scales", choices=["packed", "raw"], default="packed",
                    help="scale layout lutgemm_run reads (packed: unit-major, reordered at load time)")
    ap.add_argument("--only", choices=[sh.name for sh in S.WORKLOADS[WORKLOAD].shapes], default=None,
                    help="time one linear of the layer only (profiling)")
    ap.add_argument("--parallel", choices=["rows", "inputs", "paired"], default=None,
                    help="split one matrix over the --gpus ranks (strong scaling, NCCL exchange)")
    ap.add_argument("--mixed-hi", type=float, default=0.125, help="mixed workload: fraction of 4-plane blocks")
    ap.add_argument("--mixed-outliers", type=float, default=0.005, help="mixed workload: fp16 outlier density")
    ap.add_argument("--workload", choices=["layer", "fit", "sweep", "tc", "mixed"], default="layer",
                    help="layer: the LUT-GEMM step (default); fit: BCQ fitting of FP16 weights; "
                         "sweep: every parity config shape and batch, one line each; "
                         "tc: the layer's linears at a large batch on the tensor-core path")
    ap.add_argument("--tc-batch", type=int, default=256)
    ap.add_argument("--tc-direct", action="store_true",
                    help="tc workload: call lutgemm_run_tc (one K split) instead of lutgemm_run with the tensor cores allowed")
    ap.add_argument("--tc-cpu-rows", type=int, default=128, help="rows per linear in the tc CPU baseline sample")
    ap.add_argument("--fit-m", type=int, default=49152)
    ap.add_argument("--fit-n", type=int, default=12288)
    ap.add_argument("--fit-g", type=int, default=128)
    ap.add_argument("--fit-iters", type=int, default=3)
    ap.add_argument("--fit-cpu-rows", type=int, default=384, help="rows of the CPU baseline fit sample")
    ap.add_argument("--fit-grid", action="store_true",
                    help="fit the variable grid (planes + one constant per group) instead of plain BCQ")
    args = ap.parse_args()
    # At least three untimed warm-up steps, whatever the caller asks for.
    args.warmup = max(3, args.warmup)
    if args.parallel is not None and args.impl == "lutgemm":
        run_parallel(args)
    elif args.workload == "sweep":
        run_sweep(args)
    elif args.workload == "mixed":
        run_mixed_workload(args)
    elif args.workload == "tc":
        if args.impl == "reference":
            world, rank, _ = _dist_env()
            if rank == 0:
                r = cpu_tc_baseline(args.q, args.tc_batch, args.tc_cpu_rows)
                print(json.dumps({"impl": "reference", "metric": TC_METRIC, "value": r["value"],
                                  "unit": "TFLOP/s", "n_gpus": world, "steps": 1, "warmup": 0,
                                  "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                                  "dtype": "f64", "data": "synthetic", "cpu_baseline": r,
                                  "e2e": {"value": r["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0}}), flush=True)
        else:
            run_tc(args)
    elif args.workload == "fit":
        if args.impl == "reference":
            world, rank, _ = _dist_env()
            if rank == 0:
                r = cpu_fit_baseline(args.q, args.fit_g, args.fit_iters, args.fit_n, args.fit_cpu_rows, args.fit_grid)
                print(json.dumps({"impl": "reference", "metric": FIT_METRIC, "value": r["value"],
                                  "unit": "Gweights/s", "n_gpus": world, "steps": 1, "warmup": 0,
                                  "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                                  "dtype": "f64", "data": "synthetic", "cpu_baseline": r,
                                  "e2e": {"value": r["value"], "unit": "Gweights/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0}}), flush=True)
        else:
            run_fit(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_lutgemm(args)


if __name__ == "__main__":
    main()
