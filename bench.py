"""Benchmark of the W4A16 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Workloads (synthetic, seeded; see weight_only_int4_06_b200/synth.py):
  decode       (default) single-token decode through 7B-class layers: M=1,
               (K,N) in (4096,4096), (4096,12288), (4096,11008), (11008,4096); one step = one
               w4_gemm per shape
  small_batch  M in {4,8,16,32} x 70B-class (K,N); one step = every (M, shape) once
  prefill      M in {512,2048,4096} x (K,N) in (4096,11008), (4096,4096), (8192,28672)
  quantize     w4_quantize_pack of the four 7B-class weight matrices
  awq          awq_scale_search on X_calib [65536,4096], W [4096,4096], 20 alphas

Timing: every step is captured once in a CUDA graph; W warm-up steps run first, then exactly K
steps are timed with CUDA events on the launching stream between barriers and device
synchronisations.  Weight-streaming workloads cycle through enough distinct weight buffers that
the bytes touched between two uses of a buffer exceed 3x the L2 size, so every step reads HBM.
Under torchrun every rank runs its own replica (no collective on the data path) and the
reported time is the maximum over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_int4_06_b200 import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------- DRAM-traffic records
# An ncu capture (dram__bytes_read.sum, dram__bytes_write.sum per launch) of one step of a workload
# is summed into profiles/traffic_<workload>.json together with a digest of the kernel's sources;
# the roofline line reports that traffic only while the digest still matches, so a kernel edited
# after the capture reports none.
KERNEL_SOURCES = {
    "decode": ["weight_only_int4_06_b200/csrc/decode_stream.cu", "weight_only_int4_06_b200/csrc/sm100.cuh",
               "weight_only_int4_06_b200/csrc/common.cuh"],
    "prefill": ["weight_only_int4_06_b200/csrc/gemm_tc.cu", "weight_only_int4_06_b200/csrc/sm100.cuh",
                "weight_only_int4_06_b200/csrc/common.cuh"],
}

_COMMENT = re.compile(r"/\*.*?\*/|//[^\n]*", re.S)


def code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed: what the compiler sees."""
    return " ".join(_COMMENT.sub(" ", text).split())


def source_digest(workload: str) -> str:
    """Digest of the kernel sources' code (comments and layout excluded)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[workload]:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + code_only(fh.read()).encode())
    return h.hexdigest()


def traffic_record_path(workload: str) -> str:
    return os.path.join(ROOT, "profiles", f"traffic_{workload}.json")


def load_traffic(workload: str):
    """DRAM bytes per step, or None (no record, or the kernel sources changed since)."""
    try:
        with open(traffic_record_path(workload)) as f:
            rec = json.load(f)
        if rec.get("source_sha256") != source_digest(workload):
            return None
        return int(rec["dram_bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


def gemm_bytes(M, K, N):
    """Algorithmic HBM bytes of one w4_gemm: packed W, fp16 scales, u8 zeros, X and Y."""
    return N * K // 2 + N * (K // 128) * 3 + 2 * M * K + 2 * M * N


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"w4_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        load = [v for v in sm if smax and v > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------- distributed
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------- workloads
def decode_cases():
    return [(1, K, N) for (K, N) in synth.DECODE_7B_SHAPES], 2, "decode GEMV, 7B-class layer shapes"


def small_batch_cases():
    return ([(M, K, N) for (K, N) in synth.SMALL_BATCH_70B_SHAPES for M in synth.SMALL_BATCH_MS], 3,
            "small-batch decode, 70B-class shapes")


def prefill_cases():
    return ([(M, K, N) for (K, N) in synth.PREFILL_SHAPES for M in synth.PREFILL_MS], 4,
            "prefill, compute-bound")


def gemm_launches(M, K, N, variant=0, scales=None, zeros=None):
    """Kernel launches of one w4_gemm call, as the library's own dispatch decides them."""
    from weight_only_int4_06_b200 import w4a16 as B
    return B.w4_gemm_plan(M, N, K, 128, variant, scales, zeros)[1]


class GemmWorkload:
    """Device-resident inputs for a list of (M, K, N) layers, with rotating weight copies."""

    def __init__(self, cases, case_id, l2_bytes, variant=0):
        import torch
        from weight_only_int4_06_b200 import w4a16 as B
        self.B = B
        self.variant = variant
        self.cases = cases
        # Weight copies per layer: the step rotates through n_sets copies of every layer (more than
        # 3x L2 between two uses of a copy); a layer timed alone rotates through its own copies,
        # at least 3x L2 of that layer's weights.
        step_w = sum(N * K // 2 + N * (K // 128) * 3 for (M, K, N) in cases)
        self.n_sets = max(1, min(16, int(np.ceil(3 * l2_bytes / max(step_w, 1))) + 1))
        self.layers = []
        for (M, K, N) in cases:
            X, W = synth.layer_case(case_id, M, K, N)
            Xd = torch.from_numpy(X).cuda()
            Wd = torch.from_numpy(W).cuda()
            packed, scales, zeros = B.w4_quantize_pack(Wd)
            copies = [(packed, scales, zeros)]
            layer_w = N * K // 2 + N * (K // 128) * 3
            n_layer = max(self.n_sets, min(64, int(np.ceil(3 * l2_bytes / layer_w)) + 1))
            for c in range(1, n_layer):
                copies.append((packed.clone(), scales.clone(), zeros.clone()))
            del Wd
            Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
            need = B.w4_gemm_workspace_size(M, N, K)
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
            self.layers.append(dict(M=M, K=K, N=N, X=Xd, Xh=torch.from_numpy(X).pin_memory(),
                                    Yh=torch.empty((M, N), dtype=torch.float16).pin_memory(),
                                    xs=torch.empty((M, K), dtype=torch.float16, device="cuda"),
                                    copies=copies, Y=Y, ws=ws))
        torch.cuda.synchronize()
        self.bytes_per_step = sum(gemm_bytes(M, K, N) for (M, K, N) in cases)
        self.flops_per_step = sum(2 * M * K * N for (M, K, N) in cases)
        self.launches_per_step = sum(gemm_launches(M, K, N, variant, L["copies"][0][1], L["copies"][0][2])
                                     for (M, K, N), L in zip(cases, self.layers))
        self.host_calls = None  # prepared w4_gemm_host_batch calls, built on first use
        self.host_graphs = None  # their CUDA graphs
        self.host_path_note = None

    def run_step(self, step, only=None):
        for i, L in enumerate(self.layers):
            if only is not None and i != only:
                continue
            copies = L["copies"] if only is not None else L["copies"][:self.n_sets]
            p, sc, z = copies[step % len(copies)]
            self.B.w4_gemm(L["X"], p, sc, z, out=L["Y"], workspace=L["ws"], variant=self.variant)

    def run_step_host(self, step):
        """The same step through the public API with host (pinned) activations and results: the
        w4_gemm_host_batch call (every layer's X in one host-to-device copy, the layers' GEMMs,
        every Y in one device-to-host copy), prepared once per weight set as a serving loop over
        fixed buffers would and captured as a CUDA graph (HostGemmBatch.capture) that each step
        replays; the copies move the host buffers' current contents at every replay.  The step
        ends when the stream has drained (the results are then readable on the host, in the
        batch's pinned result buffer: `HostGemmBatch.y(i)` views it)."""
        import torch
        if self.host_calls is None:
            try:
                self.host_calls, self.host_graphs = [], []
                for c in range(self.n_sets):
                    b = self.B.HostGemmBatch([L["copies"][c] for L in self.layers],
                                             [(L["M"], L["K"], L["N"]) for L in self.layers],
                                             workspace=self.layers[0]["ws"], variant=self.variant)
                    for i, L in enumerate(self.layers):
                        b.x(i).copy_(L["Xh"])
                    self.host_calls.append(b)
                    self.host_graphs.append(b.capture())
            except Exception as e:  # the per-layer C call instead
                self.host_calls, self.host_graphs = [], []
                self.host_path_note = f"batched call unavailable ({type(e).__name__}: {e}); per-layer w4_gemm_host"
        if self.host_calls:
            c = step % self.n_sets
            b = self.host_calls[c]
            self.host_graphs[c].replay()
            torch.cuda.current_stream().synchronize()
            return b
        s = step % self.n_sets
        for L in self.layers:
            p, sc, z = L["copies"][s]
            self.B.w4_gemm_host(L["Xh"], p, sc, z, L["Yh"], L["xs"], L["Y"], workspace=L["ws"])
        torch.cuda.current_stream().synchronize()
        return [L["Yh"] for L in self.layers]

    def h2d_d2h_bytes(self):
        return (sum(2 * M * K for (M, K, N) in self.cases), sum(2 * M * N for (M, K, N) in self.cases))


def capture(fn, n_steps, first_step=0):
    import torch
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(n_steps):
                fn(first_step + i)
    torch.cuda.current_stream().wait_stream(s)
    return g


def time_graph(g, world, stream=None):
    import torch
    barrier(world)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream() if stream is None else stream
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)  # ms


class L2Flush:
    """Writes a buffer of twice the L2 size, evicting whatever the previous replay left there."""

    def __init__(self, l2_bytes):
        import torch
        self.buf = torch.empty(max(1, int(2 * l2_bytes) // 4), dtype=torch.int32, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


def time_graph_median(g, world, replays, flush=None):
    """Median over `replays` replays of the graph's CUDA-event time (ms), each replay bracketed by a
    barrier and device synchronisations (time_graph), the L2 flushed before each replay outside
    the timed region; then the maximum of the ranks' medians."""
    times = []
    for _ in range(replays):
        if flush is not None:
            flush()
        times.append(time_graph(g, world))
    return max_over_ranks(statistics.median(times), world), times


def oracle_cpu_baseline(cases, case_id, budget_s=20.0):
    """The CPU oracle as it stands, on a bounded sample of the same step."""
    import oracle
    t_total = 0.0
    done = 0
    per_case = []
    for (M, K, N) in cases:
        X, W = synth.layer_case(case_id, M, K, N)
        p, s, z = oracle.quantize_pack(W)
        Msub = min(M, 16)
        t0 = time.perf_counter()
        oracle.gemm(X[:Msub], p, s, z)
        dt = time.perf_counter() - t0
        per_case.append((M, K, N, Msub, dt))
        t_total += dt * (M / Msub)
        done += 1
        if t_total > budget_s:
            break
    frac = done / len(cases)
    cores = len(os.sched_getaffinity(0))
    return {"value_us_per_step": t_total / frac * 1e6, "cores": cores,
            "sample": (f"{done} of {len(cases)} layers of one step"
                       + (", activation rows capped at 16 and scaled by M/16" if any(c[0] > 16 for c in cases) else "")
                       + "; oracle = numpy dequantise + fp64 matmul (OpenBLAS threads)")}


def layer_rows(wl, world, reps, peaks, compute_bound, flush=None, replays=5):
    """Per-layer device time, one layer at a time: a graph of `reps` calls of that layer (rotating
    weight sets), median of `replays` replays."""
    rows = []
    for i, L in enumerate(wl.layers):
        # every call of the graph uses a different copy of the layer's weights (cold L2)
        n = max(reps, len(L["copies"]))
        gi = capture(lambda s, i=i: wl.run_step(s, only=i), n, 0)
        gi.replay()
        t = time_graph_median(gi, world, replays, flush)[0] / n
        b = gemm_bytes(L["M"], L["K"], L["N"])
        fl = 2 * L["M"] * L["K"] * L["N"]
        r = {"M": L["M"], "K": L["K"], "N": L["N"], "us": round(t * 1e3, 3),
             "GBps": round(b / (t * 1e-3) / 1e9, 1), "TFLOPs": round(fl / (t * 1e-3) / 1e12, 2)}
        if compute_bound:
            r["tensor_frac"] = round(fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 3)
        else:
            r["hbm_frac"] = round(b / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)
        rows.append(r)
        del gi
    return rows


def run_gemm_bench(args, rank, world, local, kind, with_extras=True):
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    cases, case_id, desc = {"decode": decode_cases, "small_batch": small_batch_cases,
                            "prefill": prefill_cases}[kind]()
    compute_bound = kind == "prefill"
    peaks = load_peaks()
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    # Decode-time weights are resident and never rewritten between calls: declare them static so
    # each GEMM may start streaming its weights while the previous kernel drains.
    variant = B.FLAG_WEIGHTS_STATIC
    wl = GemmWorkload(cases, case_id, l2, variant=variant)
    K_steps, W_steps = args.steps, args.warmup

    for i in range(2):
        wl.run_step(i)
    torch.cuda.synchronize()
    g_warm = capture(wl.run_step, W_steps, 0)
    g_timed = capture(wl.run_step, K_steps, W_steps)
    g_warm.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
        t_end = time.time() + 1.0
        while time.time() < t_end:   # keep the GPU busy while the sampler settles
            g_warm.replay()
        torch.cuda.synchronize()
    flush = L2Flush(l2)
    ms, replay_ms = time_graph_median(g_timed, world, args.replays, flush)
    clocks = sampler.stop() if sampler else None
    ms_per_step = ms / K_steps
    del g_timed, g_warm

    # the same step with plain stream-ordered launches (no early weight streaming)
    wl.variant = 0
    g_plain = capture(wl.run_step, K_steps, 0)
    g_plain.replay()
    ms_plain = time_graph_median(g_plain, world, max(3, args.replays // 4), flush)[0] / K_steps
    del g_plain
    wl.variant = variant

    per_layer = layer_rows(wl, world, max(W_steps, 20), peaks, compute_bound, flush)

    # end to end through the public API with host buffers (pinned X in, Y out, every step)
    h2d, d2h = wl.h2d_d2h_bytes()
    e2e_steps = 50
    # warm-up: prepares the batch calls and replays every weight set's graph twice (a graph's
    # first launch uploads it)
    for i in range(max(W_steps, 3) + 2 * wl.n_sets):
        wl.run_step_host(i)
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        wl.run_step_host(i)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)

    if compute_bound:
        achieved = wl.flops_per_step / (ms_per_step * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": load_traffic("prefill"),
                "peak_note": "dense bf16 burst (fp16 dense rate is the same on B200)"}
        kern = "tc_gemm_kernel<DEQ> (tcgen05 + TMEM + TMA)"
    else:
        achieved = wl.bytes_per_step / (ms_per_step * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": load_traffic("decode") if kind == "decode" else None}
        kern = ("decode_stream_kernel<MT> (one full-SM CTA per SM, TMA ring of 32 KB stages, mma.sync, "
                "metadata by bulk copy)"
                if kind == "decode" else
                "w4_gemm per shape: decode_stream_kernel in launches of <= 8 rows (K cut into slices of "
                "4096 + splitk_reduce where the rows would leave a shallow ring), the tcgen05 GEMM at "
                "M = 32 on wide layers")
    roof["traffic_unit"] = "DRAM bytes per step (ncu, see profiles/)"
    roof["peak_source"] = peaks["source"]
    roof["kernel"] = kern
    roof["algorithmic_bytes_per_step"] = wl.bytes_per_step
    roof["algorithmic_flops_per_step"] = wl.flops_per_step

    out = {
        "metric": "W4A16 GEMM us & % roofline (HBM GB/s at M<=16, TFLOP/s at M>=512)",
        "value": round(ms_per_step * 1e3, 3),
        "unit": "us/step",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_steps,
        "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": desc, "layers": [list(c) for c in cases], "group": 128,
                   "weights_static_flag": True,
                   "l2": f"cold: {wl.n_sets} rotating weight-buffer sets, >=3x L2 between reuses",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roof,
        "plain_launch_us_per_step": round(ms_plain * 1e3, 3),
        "layers": per_layer,
        "timing": {"replays": len(replay_ms), "statistic": "median of replays, each exactly K steps",
                   "replay_us_per_step_min_max": [round(min(replay_ms) / K_steps * 1e3, 3),
                                                  round(max(replay_ms) / K_steps * 1e3, 3)],
                   "l2": "flushed (2x L2 write) before every replay, outside the timed region"},
        "e2e": {"value": round(e2e_ms * 1e3, 3), "unit": "us/step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": wl.host_path_note or ("one w4_gemm_host_batch call per step (all layers' X in one "
                                              "pinned host-to-device copy, the GEMMs, all Y in one "
                                              "device-to-host copy), prepared once per weight set "
                                              "(HostGemmBatch) and replayed as a CUDA graph; pinned buffers moved by "
                                              "SM copy kernels chained to the GEMMs; one stream synchronisation per "
                                              "step")},
        "gpu_launches": wl.launches_per_step * K_steps,
        "clocks": clocks,
    }
    del wl
    torch.cuda.empty_cache()
    if with_extras and not args.no_rows:
        out["rows"] = other_rows(args, world, peaks, l2)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_cpu_baseline(cases, case_id)
        out["cpu_baseline"] = {"value": round(cb["value_us_per_step"], 1), "unit": "us/step",
                               "cores": cb["cores"], "kind": "oracle", "sample": cb["sample"]}
    return out


def bench_quantize(world, peaks, l2, reps=10):
    """w4_quantize_pack on the four 7B-class weight matrices, rotating copies (cold L2)."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    res = []
    for (K, N) in synth.DECODE_7B_SHAPES:
        _, W = synth.layer_case(2, 1, K, N)
        Wd = torch.from_numpy(W).cuda()
        n_sets = max(2, int(np.ceil(3 * l2 / (W.nbytes))) + 1)
        Ws = [Wd] + [Wd.clone() for _ in range(n_sets - 1)]
        outs = [B.w4_quantize_pack(w) for w in Ws]
        G = K // 128
        L = B.lib()
        stream = B._stream(None)

        def step(i):
            w = Ws[i % n_sets]
            p, s, z = outs[i % n_sets]
            L.w4_quantize_pack(B._dev(w, torch.float16, "W"), N, K, 128, None,
                               B.ctypes.c_void_p(p.data_ptr()), B.ctypes.c_void_p(s.data_ptr()),
                               B.ctypes.c_void_p(z.data_ptr()), B._stream(None))
        step(0)
        g = capture(step, reps, 0)
        g.replay()
        t = max_over_ranks(time_graph(g, world) / reps, world)
        byts = N * K * 2 + N * K // 2 + N * G * 3
        res.append({"K": K, "N": N, "us": round(t * 1e3, 2), "GBps": round(byts / (t * 1e-3) / 1e9, 1),
                    "hbm_frac": round(byts / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)})
        del g, Ws, outs, Wd
        _ = stream
    torch.cuda.empty_cache()
    return {"kernel": "quantize_pack_kernel", "bound": "hbm", "layers": res}


def _time_awq_search(world, search, Xd, Wd, ws, reps):
    """Min over reps of one search call's CUDA-event time (ms), max over ranks."""
    import torch
    search(Xd, Wd, 20, workspace=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        search(Xd, Wd, 20, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return max_over_ranks(min(times), world)


def bench_awq(world, peaks, case, reps=2):
    """awq_scale_search on X_calib [65536, 4096], W [4096, 4096], 20 alphas."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    X, W = case
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    T, K = X.shape
    N = W.shape[0]
    ws = torch.empty(B.awq_workspace_size(T, N, K, 128, 20), dtype=torch.uint8, device="cuda")
    t = _time_awq_search(world, B.awq_scale_search, Xd, Wd, ws, reps)
    flops = 20 * 2 * T * K * N
    tf = flops / (t * 1e-3) / 1e12
    del Xd, Wd, ws
    torch.cuda.empty_cache()
    return {"kernel": "colabs + 20 x (awq_fakequant + tc_gemm_kernel<SSE>) + finalize",
            "T": T, "K": K, "N": N, "n_alpha": 20, "ms": round(t, 3), "TFLOPs": round(tf, 1),
            "bound": "tensor", "tensor_frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 3),
            "flops": flops}


def bench_awq_gram(world, peaks, case, reps=3):
    """awq_scale_search_gram on the same calibration layer: G = X^T X once, then 20 K x K forms."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    X, W = case
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    T, K = X.shape
    N = W.shape[0]
    ws = torch.empty(B.awq_gram_workspace_size(T, N, K, 128, 20), dtype=torch.uint8, device="cuda")
    t = _time_awq_search(world, B.awq_scale_search_gram, Xd, Wd, ws, reps)
    flops = 2 * T * K * K + 20 * 2 * N * K * K  # Gram + one quadratic-form GEMM per alpha
    tf = flops / (t * 1e-3) / 1e12
    # executed: G is formed as its 256 x 256 tiles on and below the diagonal
    nt = (K + 255) // 256
    executed = 2 * T * K * K * (nt * (nt + 1) // 2) / (nt * nt) + 20 * 2 * N * K * K
    tf_exec = executed / (t * 1e-3) / 1e12
    del Xd, Wd, ws
    torch.cuda.empty_cache()
    return {"kernel": "transpose + 16 x (tc_gemm_kernel<f32 out, lower-triangle tiles> + fp64 add) + scale + "
                      "20 x (fakequant + tc_gemm_kernel<quadratic form>) + finalize",
            "T": T, "K": K, "N": N, "n_alpha": 20, "ms": round(t, 3), "TFLOPs": round(tf, 1),
            "bound": "tensor", "tensor_frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 3),
            "flops": flops, "flops_executed": int(executed),
            "tensor_frac_sustained_executed": round(tf_exec / peaks["bf16_tflops_sustained"], 3)}


def bench_gptq(world, peaks, reps=2):
    """gptq_quantize on the calibration layer's 4096-row subsample, K = N = 4096 (fp64 CUDA cores)."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    X, W = synth.awq_case()
    Xs = torch.from_numpy(np.ascontiguousarray(X[synth.awq_subsample_rows()])).cuda()
    Wd = torch.from_numpy(W).cuda()
    T, K = Xs.shape
    N = Wd.shape[0]
    ws = torch.empty(B.gptq_workspace_size(T, N, K), dtype=torch.uint8, device="cuda")
    B.gptq_quantize(Xs, Wd, workspace=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        B.gptq_quantize(Xs, Wd, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    t = max_over_ranks(min(times), world)
    flops = 2 * T * K * K + 2 * K ** 3 // 3 + N * K * K  # H, Cholesky + inverse, sweep updates (fp64)
    del Xs, Wd, ws
    torch.cuda.empty_cache()
    return {"kernel": "gptq_gram + blocked Cholesky/inverse + 32 x (sweep + trailing), fp64", "T": T, "K": K,
            "N": N, "ms": round(t, 3), "TFLOPs_fp64": round(flops / (t * 1e-3) / 1e12, 2), "flops": flops,
            "bound": "fp64 FMA"}


def bench_wb_gemm(world, peaks, reps=20):
    """wb_gemm (dequantise to fp16 + tcgen05 GEMM) for 3-bit g128 and 2-bit g64 at M = 1 and 2048."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    K = N = 4096
    _, W = synth.layer_case(6, 1, K, N)
    Wd = torch.from_numpy(W).cuda()
    ws = torch.empty(N * K * 2, dtype=torch.uint8, device="cuda")
    res = []
    for bits, group in ((3, 128), (2, 64)):
        p, s, z = B.w4_quantize_pack_bits(Wd, bits, group)
        for M in (1, 2048):
            X, _ = synth.layer_case(6, M, K, 8)
            Xd = torch.from_numpy(X).cuda()
            B.wb_gemm(Xd, p, s, z, bits, group, ws)
            g = capture(lambda i: B.wb_gemm(Xd, p, s, z, bits, group, ws), reps, 0)
            g.replay()
            t = max_over_ranks(time_graph(g, world) / reps, world)
            byts = N * K * bits // 8 + 3 * N * (K // group) + 2 * M * K + 2 * M * N  # algorithmic (b/8 B/weight)
            r = {"bits": bits, "group": group, "M": M, "K": K, "N": N, "us": round(t * 1e3, 2),
                 "hbm_frac_of_algorithmic": round(byts / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}
            if M > 1:
                r["tensor_frac"] = round(2 * M * N * K / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 3)
            res.append(r)
            del g
    del Wd, ws
    torch.cuda.empty_cache()
    return {"kernel": "M <= 8: wb_gemv_kernel (fused: bit stream read once, codes dequantised in registers, "
                      "fp32 CUDA-core sums); larger M: dequant_bits_kernel + tc_gemm_kernel<fp16 B> (two passes "
                      "through an fp16 workspace)", "layers": res}


FP32_FMA_PER_CLK_PER_SM = 128     # B200 SM: 4 partitions x 32 fp32 FMA lanes
B200_SMS, B200_MAX_SM_MHZ = 148, 1965


def bench_awq_clip(world, peaks, case, reps=3, n_ratios=10):
    """awq_clip_search on X_calib [65536, 4096], W [4096, 4096], 10 ratios, with an AWQ scale."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    X, W = case
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    T, K = X.shape
    N = W.shape[0]
    a = torch.ones(K, dtype=torch.float32, device="cuda")
    ws = torch.empty(B.awq_clip_workspace_size(T, N, K, 128, n_ratios), dtype=torch.uint8, device="cuda")
    B.awq_clip_search(Xd, Wd, a, n_ratios, workspace=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        B.awq_clip_search(Xd, Wd, a, n_ratios, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    t = max_over_ranks(min(times), world)
    G = K // 128
    flops = 2 * T * K * 128 + N * G * n_ratios * 2 * 128 * 128  # Gram blocks + quadratic forms
    tf = flops / (t * 1e-3) / 1e12
    peak = 2 * FP32_FMA_PER_CLK_PER_SM * B200_SMS * B200_MAX_SM_MHZ * 1e6 / 1e12
    del Xd, Wd, ws
    torch.cuda.empty_cache()
    return {"kernel": "gram_partial + gram_reduce + clip_kernel (fp32 CUDA cores)",
            "T": T, "K": K, "N": N, "n_ratios": n_ratios, "ms": round(t, 3), "TFLOPs": round(tf, 2),
            "bound": "alu", "peak_tflops": round(peak, 1),
            "peak_note": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x 1965 MHz (unit counts and max clock)",
            "alu_frac": round(tf / peak, 3), "flops": flops}


def _small_batch_row(world, peaks, l2):
    """Config-3 shapes one at a time: M in {4, 8, 16, 32} x the 70B-class (K, N)."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    cases = small_batch_cases()[0]
    wl = GemmWorkload(cases, 3, l2, variant=B.FLAG_WEIGHTS_STATIC)
    wl.run_step(0)
    torch.cuda.synchronize()
    flush = L2Flush(l2)
    layers = layer_rows(wl, world, 10, peaks, False, flush)
    for r, (M, K, N), L in zip(layers, cases, wl.layers):
        fam, n = B.w4_gemm_plan(M, N, K, 128, 0, L["copies"][0][1], L["copies"][0][2])
        r["family"] = {B.VARIANT_GEMV: "gemv", B.VARIANT_SKINNY: "skinny", B.VARIANT_TC: "tc"}.get(fam, str(fam))
        r["launches"] = n
    del wl, flush
    torch.cuda.empty_cache()
    return {"kernel": "w4_gemm (per-shape family: decode_stream_kernel in launches of <= 8 rows, K cut "
                      "into slices of 4096 + splitk_reduce where the rows would leave a shallow ring; the "
                      "tcgen05 GEMM where its tiles fill the SMs)", "bound": "hbm", "layers": layers}


def _prefill_row(world, peaks, l2):
    import torch
    pre = GemmWorkload(prefill_cases()[0], 4, l2)
    pre.run_step(0)
    torch.cuda.synchronize()
    row = {"kernel": "tc_gemm_kernel<DEQ>", "bound": "tensor", "layers": layer_rows(pre, world, 10, peaks, True)}
    del pre
    torch.cuda.empty_cache()
    return row


def other_rows(args, world, peaks, l2):
    """The rows besides the headline.  On one GPU a row that fails is reported as {"error": ...}
    and the others still run; with several ranks an error propagates (the ranks' collective steps
    must stay in step)."""
    import torch
    rows = {}

    def row(name, fn):
        if world > 1:
            rows[name] = fn()
            return
        try:
            rows[name] = fn()
        except Exception as e:  # keep the headline line and the other rows
            rows[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
            try:
                torch.cuda.synchronize()
                torch.cuda.empty_cache()
            except Exception:
                pass

    row("small_batch", lambda: _small_batch_row(world, peaks, l2))
    row("quantize", lambda: bench_quantize(world, peaks, l2))
    row("prefill", lambda: _prefill_row(world, peaks, l2))
    case = synth.awq_case()
    row("awq", lambda: bench_awq(world, peaks, case))
    row("awq_gram", lambda: bench_awq_gram(world, peaks, case))
    if "ms" in rows["awq"] and "ms" in rows["awq_gram"]:
        rows["awq_gram"]["speedup_vs_direct"] = round(rows["awq"]["ms"] / rows["awq_gram"]["ms"], 2)
    row("awq_clip", lambda: bench_awq_clip(world, peaks, case))
    row("gptq", lambda: bench_gptq(world, peaks))
    row("wb_gemm", lambda: bench_wb_gemm(world, peaks))
    return rows


def run_dispatch(args):
    """Every kernel family that can serve each decode and small-batch shape, timed alone (cold L2,
    median of replays), next to the family w4_gemm picks: the measurement behind the dispatch."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    l2 = getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "L2_cache_size", 126 * 2 ** 20)
    flush = L2Flush(l2)
    peaks = load_peaks()
    names = {B.VARIANT_GEMV: "gemv", B.VARIANT_SKINNY: "skinny", B.VARIANT_TC: "tc"}
    shapes = decode_cases()[0] + small_batch_cases()[0]
    table = []
    for (M, K, N) in shapes:
        X, W = synth.layer_case(3, M, K, N)
        Xd = torch.from_numpy(X).cuda()
        p, sc, z = B.w4_quantize_pack(torch.from_numpy(W).cuda())
        layer_w = N * K // 2 + N * (K // 128) * 3
        n = max(8, min(64, int(np.ceil(3 * l2 / layer_w)) + 1))
        copies = [(p, sc, z)] + [(p.clone(), sc.clone(), z.clone()) for _ in range(n - 1)]
        Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        row = {"M": M, "K": K, "N": N, "auto": names.get(B.w4_gemm_plan(M, N, K, 128, 0, sc, z)[0])}
        for fam in (B.VARIANT_GEMV, B.VARIANT_SKINNY, B.VARIANT_TC):
            try:
                B.w4_gemm_plan(M, N, K, 128, fam, sc, z)
            except B.W4Error:
                row[names[fam]] = None
                continue
            var = fam | B.FLAG_WEIGHTS_STATIC

            def step(i, var=var):
                pp, ss, zz = copies[i % n]
                B.w4_gemm(Xd, pp, ss, zz, out=Y, variant=var)
            step(0)
            torch.cuda.synchronize()
            g = capture(step, n, 0)
            g.replay()
            t = time_graph_median(g, 1, 3, flush)[0] / n
            row[names[fam]] = {"us": round(t * 1e3, 3),
                               "hbm_frac": round(gemm_bytes(M, K, N) / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}
            del g
        timed = {k: v["us"] for k, v in row.items() if isinstance(v, dict)}
        row["fastest"] = min(timed, key=timed.get) if timed else None
        table.append(row)
        del copies, Xd, Y
        torch.cuda.empty_cache()
    return {"workload": "dispatch table: decode and small-batch shapes x kernel family", "table": table,
            "peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"]}


def run_profile_case(args):
    """A short, self-checking run for ncu captures (no timing): the workload's layers with one
    weight copy each (ncu flushes the caches between its passes), `args.profile_only` steps, then
    the device status.  Workloads: decode, small_batch, prefill (w4_gemm per layer), awq / awq_gram
    (the scale search on the calibration layer's 16384-row subsample), quantize (w4_quantize_pack of
    the decode layers' weights), awq_clip (the clip search, 10 ratios, on the same subsample)."""
    import torch
    from weight_only_int4_06_b200 import w4a16 as B
    steps = max(1, args.profile_only)
    kind = args.workload
    if kind in ("awq", "awq_gram", "awq_clip"):
        X, W = synth.awq_case()
        Xd = torch.from_numpy(X[:16384].copy()).cuda()
        Wd = torch.from_numpy(W).cuda()
        for _ in range(steps):
            if kind == "awq_clip":
                B.awq_clip_search(Xd, Wd, None, 10)
            else:
                (B.awq_scale_search if kind == "awq" else B.awq_scale_search_gram)(Xd, Wd, 20)
    elif kind == "quantize":
        Ws = [torch.from_numpy(synth.layer_case(2, 1, K, N)[1]).cuda() for (K, N) in synth.DECODE_7B_SHAPES]
        for _ in range(steps):
            for Wd in Ws:
                B.w4_quantize_pack(Wd)
    else:
        cases, case_id, _ = {"decode": decode_cases, "small_batch": small_batch_cases,
                             "prefill": prefill_cases}[kind]()
        layers = []
        for (M, K, N) in cases:
            X, W = synth.layer_case(case_id, M, K, N)
            layers.append((torch.from_numpy(X).cuda(), *B.w4_quantize_pack(torch.from_numpy(W).cuda())))
        for _ in range(steps):
            for (Xd, p, sc, z) in layers:
                B.w4_gemm(Xd, p, sc, z, variant=B.FLAG_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    st = B.w4_check_device_status()
    assert st == 0, B.STATUS_NAMES.get(st, st)
    return {"profile_case": kind, "steps": steps, "status": "ok"}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle timed on a bounded sample of the same workload."""
    if rank != 0:
        return None
    kind = args.workload
    cases, case_id, desc = {"decode": decode_cases, "small_batch": small_batch_cases,
                            "prefill": prefill_cases}.get(kind, decode_cases)()
    vals = []
    cb = None
    for _ in range(args.warmup + args.steps):
        cb = oracle_cpu_baseline(cases, case_id, budget_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)))
        vals.append(cb["value_us_per_step"])
    v = statistics.median(vals[args.warmup:]) if len(vals) > args.warmup else vals[-1]
    return {
        "impl": "reference",
        "metric": "W4A16 GEMM us & % roofline (HBM GB/s at M<=16, TFLOP/s at M>=512)",
        "value": round(v, 1), "unit": "us/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(v / 1e3, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": desc, "layers": [list(c) for c in cases], "group": 128},
        "cpu_baseline": {"value": round(v, 1), "unit": "us/step", "cores": cb["cores"],
                         "kind": "oracle", "sample": cb["sample"]},
        "e2e": {"value": round(v, 1), "unit": "us/step", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "small_batch", "prefill", "dispatch", "awq", "awq_gram", "awq_clip",
                             "quantize"])
    ap.add_argument("--profile-only", type=int, default=0, metavar="S",
                    help="run S untimed steps of the workload for an ncu capture, check the status, exit")
    ap.add_argument("--replays", type=int, default=20,
                    help="graph replays of the K timed steps; the median is reported (>= 20 by default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the secondary rows (quantize, prefill, awq) in the JSON line")
    ap.add_argument("--extra-rows", action="store_true",
                    help="accepted for compatibility: GPTQ and the other-width matmul are in the default line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    elif args.profile_only:
        out = run_profile_case(args) if rank == 0 else None
    elif args.workload == "dispatch":
        out = run_dispatch(args) if rank == 0 else None
    elif args.workload in ("awq", "awq_gram", "awq_clip", "quantize"):
        raise SystemExit(f"--workload {args.workload} is a profiling case only: add --profile-only S")
    else:
        out = run_gemm_bench(args, rank, world, local, args.workload)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
