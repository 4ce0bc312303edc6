#!/usr/bin/env python
"""Benchmark of the NVFP4 block-scaled GEMM hot path on B200.

Metric: NVFP4 GEMM TFLOP/s (whole step) and the fraction of the B200 roofline per
M x N x K. Workload (default): the attention-projection sweep N=768, K=6144,
M in {16, 64, 256, 1024}, A ~ N(0,1) fp32 activations, B ~ N(0,0.02) weights quantised
once to NVFP4 outside the timed region. One step = for every M: per-tensor global scale
of A, alpha = 1/(gsA gsB), NVFP4 quantisation of A, block-scaled GEMM -> bf16.

Timing: the step is captured as a CUDA graph of its eight kernels, nothing else, so each
kernel launches early behind the one before it (programmatic dependent launch). A second
graph with event-record nodes between the kernels is replayed afterwards, untimed, for the
per-shape breakdown (`per_shape`; the event nodes cost each kernel its early launch).
Inputs are larger than L2: 8 independent input sets of the sweep (activations, weights,
outputs; 41 MiB each, 327 MiB in all, "layers" with different seeds) are replayed in
rotation, so each step's data was last touched 7 steps (about 286 MiB) earlier and comes
from HBM. W warm-up replays, then exactly K steps back to back between one pair of CUDA
events (whole rotations from one graph of all 8 sets, the remainder from single-set
graphs), bracketed by a barrier and a device synchronise; step time = event time / K, max
over ranks. --flush instead flushes L2 before every step (a 512 MB write, then a 256 MB
read, which also evicts kernel code and tensor maps) and brackets each replay on its own,
the flush outside. SM clocks and throttle reasons are polled through NVML during the timed
bracket.

e2e: the same metric through the public Python API called eagerly per step, with the
activations copied from pinned host memory and the outputs copied back inside the timed
region. The input copies run on a second stream into two alternating device buffers, so a
step's copy overlaps the previous step's kernels; the outputs are checked against the graph's.

context (rank 0, after the timed step, --no-context skips it): the compute-bound 8192^3 GEMM
against the FP4 tensor peak, and 512 x 2048 x 6144 beside a bf16 torch matmul of that shape,
both with the tiled scale layout.

--impl reference: the CPU oracle as it stands (test infrastructure), on a bounded sample
of the same workload per step, on this machine's host cores.

Multi-GPU (torchrun, --gpus N): independent replicas, one per GPU ("weak" scaling); the
path has no exchange step on one GPU's worth of work, so no collective is used on the
data path.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

N_ATTN, K_ATTN, M_SWEEP = 768, 6144, (16, 64, 256, 1024)
FLUSH_BYTES = 512 << 20
CLEAN_BYTES = 256 << 20
FP4_PER_BF16 = 4.0     # nominal dense FP4 / BF16 tensor throughput ratio on B200 (9 / 2.25 PF)


# ------------------------------------------------------------------ environment

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(flops_per_rank: float, step_ms_max: float, world: int) -> float:
    """TFLOP/s of the whole job: every rank's work over the slowest rank's step time."""
    return flops_per_rank * world / (step_ms_max * 1e-3) / 1e12


# DRAM traffic of the GEMM launches of one sweep (M = 16, 64, 256, 1024; tiled scales), from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, cold L2; the bf16 outputs stay in
# L2 within a launch): 2802432 + 2954240 + 3596544 + 6251008 bytes; the capture command and its table are
# in the committed ncu summary of these launches under profiles/. Valid only for the kernel
# sources it was taken on (hash below); reported as null otherwise.
GEMM_TRAFFIC_BYTES = 2802432 + 2954240 + 3596544 + 6251008
GEMM_TRAFFIC_SOURCES = ("gemm_kernel.cuh", "gemm.cu", "ptx.cuh", "internal.h")
GEMM_TRAFFIC_SHA = "9dbe30d4e3215f45"


def _code_hash(files) -> str:
    """sha256 (16 hex digits) of the sources with their comments removed: it changes when
    the code the counters were taken on changes, not when a comment does."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "nvfp4_block_scaled_08_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def gemm_traffic():
    """The captured traffic, or None once the GEMM code differs from the captured one."""
    return GEMM_TRAFFIC_BYTES if _code_hash(GEMM_TRAFFIC_SOURCES) == GEMM_TRAFFIC_SHA else None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML in a background thread."""

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self._marks = []
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self._physical_index(device_index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    @staticmethod
    def _physical_index(i):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[i])
            except Exception:
                return i
        return i

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self):
        self._marks.append(time.perf_counter())

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        nv = self.nv
        t0, t1 = (self._marks + [0, 0])[:2] if len(self._marks) >= 2 else (0, float("inf"))
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(inside) < 3:
            inside = self.samples
            window = "timed+warmup"
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
        }
        seen = set()
        for _, _, r in inside:
            for k, bit in names.items():
                if r & bit:
                    seen.add(k)
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(seen), "samples": len(inside), "window": window}


# ------------------------------------------------------------------ roofline model

def gemm_bytes(M, N, K):
    """Algorithmic HBM bytes of one GEMM: packed operands + scales once, bf16 out once."""
    return (M + N) * K * (0.5 + 1.0 / 16.0) + 2.0 * M * N


def quant_bytes(M, K):
    """Algorithmic HBM bytes of quantising an fp32 [M, K]: read once, codes + scales out."""
    return M * K * (4.0 + 0.5 + 1.0 / 16.0)


def roofline_us(flops, nbytes, peaks):
    p_fp4 = peaks["bf16_tflops"] * FP4_PER_BF16 * 1e12
    bw = peaks["hbm_gbs"] * 1e9
    t_tc, t_mem = flops / p_fp4, nbytes / bw
    return max(t_tc, t_mem) * 1e6, ("tensor" if t_tc >= t_mem else "hbm")


# ------------------------------------------------------------------ our implementation

class AttnSweep:
    """Resident inputs, outputs and workspaces of the attention-projection sweep."""

    def __init__(self, dev, rank, set_index=0, tiled=True):
        import nvfp4_block_scaled_08_b200 as nv
        from nvfp4_block_scaled_08_b200 import workloads
        self.nv = nv
        self.dev = dev
        cases = workloads.attn_proj_cases()
        # set 0 is the canonical seeded case; the other sets (other "layers") differ only in
        # their seeds
        b = cases[0].b() if set_index == 0 else workloads.normal(
            N_ATTN, K_ATTN, 0.02, cases[0].seed + 1 + 7919 * set_index)   # same weights for every M
        bd = b.to(dev)
        self.gsB = nv.global_scale(bd)
        self.Bq, self.sfB = nv.quantize(bd, self.gsB)
        self.tiled = tiled
        if tiled:                   # weights' scales re-laid out once, outside any timing
            self.sfB = nv.sf_tile(self.sfB)
        del bd
        self.items = []
        for c in cases:
            a_cpu = c.a() if set_index == 0 else workloads.normal(c.M, K_ATTN, 1.0, c.seed + 7919 * set_index)
            it = {
                "M": c.M, "a_cpu": a_cpu.pin_memory(),
                "a": a_cpu.to(dev),
                "gs": torch.empty(1, dtype=torch.float32, device=dev),
                "alpha": torch.empty(1, dtype=torch.float32, device=dev),
                "q": torch.empty(c.M, K_ATTN // 2, dtype=torch.uint8, device=dev),
                "sf": torch.empty(nv.sf_bytes(c.M, K_ATTN, tiled), dtype=torch.uint8, device=dev),
                "out": torch.empty(c.M, N_ATTN, dtype=torch.bfloat16, device=dev),
                "out_host": torch.empty(c.M, N_ATTN, dtype=torch.bfloat16).pin_memory(),
                "ws": nv.make_workspace(c.M, N_ATTN, K_ATTN, dev),
            }
            self.items.append(it)
        self.flops = sum(2 * it["M"] * N_ATTN * K_ATTN for it in self.items)
        self.launches_per_step = 2 * len(self.items)   # fused quantize, gemm

    def step_one(self, it, stream=None):
        """One M of the step: activations (fp32, resident) -> codes, scales, alpha -> bf16 out."""
        self.run_one(it, stream)
        self.gemm_one(it, stream)

    def run_one(self, it, stream=None, a=None):
        # global scale + alpha + NVFP4 quantisation of the activations: one launch
        self.nv.quantize_dynamic(it["a"] if a is None else a, gs_other=self.gsB, gs=it["gs"], q=it["q"],
                                 sf=it["sf"], alpha_out=it["alpha"], stream=stream, tiled=self.tiled)

    def gemm_one(self, it, stream=None):
        self.nv.gemm(it["q"], it["sf"], self.Bq, self.sfB, it["alpha"], out=it["out"],
                     workspace=it["ws"], stream=stream, tiled=self.tiled)

    def capture(self):
        """Two CUDA graphs of the whole step: `graph`, the timed one, holds only the kernels
        (so each GEMM keeps its programmatic dependency on the quantiser before it); `graph_ev`
        adds event nodes around each kernel for the per-shape breakdown."""
        self.ev = []
        for it in self.items:
            self.ev.append([torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)])
        # run once eagerly so every lazily-initialised resource exists before capture
        for it in self.items:
            self.run_one(it)
            self.gemm_one(it)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for it in self.items:
                self.run_one(it)
                self.gemm_one(it)
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge):
            for it, ev in zip(self.items, self.ev):
                ev[0].record()
                self.run_one(it)
                ev[1].record()
                self.gemm_one(it)
                ev[2].record()
        self.graph, self.graph_ev = g, ge
        return g

    def setup_e2e(self):
        """A second device buffer for every activation tensor, and the events that order the
        host copies (on their own stream) against the quantiser that reads them."""
        for it in self.items:
            it["a_dev"] = [it["a"], torch.empty_like(it["a"])]
            it["ready"] = [torch.cuda.Event(), torch.cuda.Event()]
            it["consumed"] = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_step(self, step, stream, copy_stream):
        """One step through the public API with host buffers. Every M's fp32 activations are
        copied from pinned host memory on `copy_stream` into one of two device buffers
        (alternating by step, so that the copy overlaps the previous step's kernels), then
        quantised and multiplied on `stream`, and the bf16 output is copied back to pinned
        host memory on `stream`."""
        b = step & 1
        for it in self.items:
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(it["consumed"][b])     # step - 2 has read this buffer
                it["a_dev"][b].copy_(it["a_cpu"], non_blocking=True)
                it["ready"][b].record(copy_stream)
            stream.wait_event(it["ready"][b])
            self.run_one(it, stream, a=it["a_dev"][b])
            it["consumed"][b].record(stream)
            self.gemm_one(it, stream)
            it["out_host"].copy_(it["out"], non_blocking=True)

    @property
    def h2d_bytes(self):
        return sum(it["a_cpu"].numel() * 4 for it in self.items)

    @property
    def d2h_bytes(self):
        return sum(it["out"].numel() * 2 for it in self.items)


def graph_time_us(fn, reps: int, iters: int = 5) -> float:
    """Median device time of one call, from CUDA graphs of `reps` back-to-back calls."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    ts = []
    for _ in range(iters):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        e.synchronize()
        ts.append(s.elapsed_time(e) * 1e3 / reps)
    del g
    return statistics.median(ts)


def context_gemms(dev, peaks):
    """Context outside the timed step, from the compute-bound configurations: the 8192^3
    NVFP4 GEMM (uniform(-1, 1) inputs, quantised on the device) against the FP4 tensor peak,
    and the 512 x 2048 x 6144 NVFP4 GEMM beside a bf16 torch matmul of the same shape."""
    import nvfp4_block_scaled_08_b200 as nv
    from nvfp4_block_scaled_08_b200 import workloads
    p_fp4 = peaks["bf16_tflops"] * FP4_PER_BF16
    out = {}
    for c in workloads.plateau_cases():
        if c.name not in ("square_8192", "ratio_512x2048x6144"):
            continue
        a, b = c.a().to(dev), c.b().to(dev)
        gsa, gsb = nv.global_scale(a), nv.global_scale(b)
        qa, sa = nv.quantize(a, gsa)
        qb, sb = nv.quantize(b, gsb)
        sa, sb = nv.sf_tile(sa), nv.sf_tile(sb)
        al = nv.alpha(gsa, gsb)
        o = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)
        ws = nv.make_workspace(c.M, c.N, c.K, dev)
        us = graph_time_us(lambda: nv.gemm(qa, sa, qb, sb, al, out=o, workspace=ws, tiled=True),
                           reps=5 if c.M >= 8192 else 20)
        tf = c.flops / (us * 1e-6) / 1e12
        item = {"M": c.M, "N": c.N, "K": c.K, "us": round(us, 2), "tflops": round(tf, 1),
                "frac_of_fp4_peak": round(tf / p_fp4, 4),
                "fp4_peak_tflops": round(p_fp4, 1), "peak_source": "measured bf16 burst x 4"}
        if c.name.startswith("ratio"):
            ab, bb = a.to(torch.bfloat16), b.to(torch.bfloat16)
            ub = graph_time_us(lambda: torch.matmul(ab, bb.t()), reps=20)
            item["bf16_torch_us"] = round(ub, 2)
            item["fp4_over_bf16"] = round(ub / us, 3)
            del ab, bb
        out[c.name] = item
        del a, b, qa, sa, qb, sb, o, ws
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    nsets = 1 if args.flush else args.sets
    sets = [AttnSweep(dev, rank, i, args.sf_layout == "tiled") for i in range(nsets)]
    graphs = [sw.capture() for sw in sets]
    sweep = sets[0]
    # one graph of a whole rotation (every set once, in order: eight "layers"), so that
    # consecutive steps are not separated by graph launches; single-set graphs cover the rest
    rotation = torch.cuda.CUDAGraph()
    with torch.cuda.graph(rotation):
        for sw in sets:
            for it in sw.items:
                sw.step_one(it)
    stream = torch.cuda.current_stream()
    if args.flush:
        flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        clean = torch.ones(CLEAN_BYTES // 4, dtype=torch.float32, device=dev)

    def before_step():
        if args.flush:
            # write a buffer 4x the L2, then read another 2x the L2: the step starts with
            # nothing cached (data, kernel code and tensor maps alike) and no dirty lines
            flush.zero_()
            torch.sum(clean)

    clocks = ClockSampler(local)
    clocks.start()
    if args.flush:
        for i in range(args.warmup):
            before_step()
            graphs[i % nsets].replay()
    else:                                  # W steps, from the same graphs as the timed ones
        for _ in range(args.warmup // nsets):
            rotation.replay()
        for i in range(args.warmup % nsets):
            graphs[i].replay()
    torch.cuda.synchronize()

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    quant_ms = [0.0] * len(sweep.items)
    gemm_ms = [0.0] * len(sweep.items)
    total_ms = 0.0
    barrier(world)
    clocks.mark()
    if args.flush:
        # the flush before each step stays outside the timing: one bracket per step
        for i in range(args.steps):
            before_step()
            start.record(stream)
            graphs[i % nsets].replay()
            end.record(stream)
            end.synchronize()
            total_ms += start.elapsed_time(end)
    else:
        # K steps back to back (each set was last touched nsets - 1 steps earlier), one
        # bracket around all of them: whole rotations, then single sets
        start.record(stream)
        for _ in range(args.steps // nsets):
            rotation.replay()
        for i in range(args.steps % nsets):
            graphs[i].replay()
        end.record(stream)
        end.synchronize()
        total_ms = start.elapsed_time(end)
    barrier(world)
    clocks.mark()
    clocks.stop()
    # per-shape breakdown, untimed pass: the same step with event nodes between the kernels
    # (they cost each GEMM its early launch, so this pass runs slower than the timed one)
    nbreak = min(args.steps, 100)
    for i in range(nbreak):
        k = i % nsets
        before_step()
        sets[k].graph_ev.replay()
        torch.cuda.synchronize()
        for j, ev in enumerate(sets[k].ev):
            quant_ms[j] += ev[0].elapsed_time(ev[1]) / nbreak
            gemm_ms[j] += ev[1].elapsed_time(ev[2]) / nbreak
    step_ms = total_ms / args.steps
    set_bytes = sum(it["a"].numel() * 4 + it["q"].numel() + it["sf"].numel() + it["out"].numel() * 2
                    for it in sweep.items) + sweep.Bq.numel() + sweep.sfB.numel()

    step_ms = max_over_ranks(step_ms, world)
    value = whole_job_value(sweep.flops, step_ms, world)

    # e2e through the public API with host buffers; its outputs must equal the graph's
    golden = [it["out"].cpu() for it in sweep.items]    # set 0's outputs from its last replay
    sweep.setup_e2e()
    copy_stream = torch.cuda.Stream(device=dev)
    e2e_start = torch.cuda.Event(enable_timing=True)
    e2e_end = torch.cuda.Event(enable_timing=True)
    nwarm = max(2, min(args.warmup, 4))
    for i in range(nwarm):
        sweep.e2e_step(i, stream, copy_stream)
    barrier(world)
    e2e_start.record(stream)
    copy_stream.wait_event(e2e_start)       # no timed copy starts before the bracket
    for i in range(args.steps):
        sweep.e2e_step(nwarm + i, stream, copy_stream)
    e2e_end.record(stream)
    barrier(world)
    torch.cuda.synchronize()
    e2e_match = all(torch.equal(it["out_host"], g) for it, g in zip(sweep.items, golden))
    e2e_ms = max_over_ranks(e2e_start.elapsed_time(e2e_end) / args.steps, world)
    e2e_value = whole_job_value(sweep.flops, e2e_ms, world)

    # roofline: per shape, and for the dominant kernel family
    per_shape = []
    tot_gemm_us = tot_quant_us = tot_gemm_bytes = tot_quant_bytes = 0.0
    for it, qm, gm in zip(sweep.items, quant_ms, gemm_ms):
        M = it["M"]
        fl = 2.0 * M * N_ATTN * K_ATTN
        by = gemm_bytes(M, N_ATTN, K_ATTN)
        r_us, bound = roofline_us(fl, by, peaks)
        per_shape.append({
            "M": M, "N": N_ATTN, "K": K_ATTN, "gemm_us": round(gm * 1e3, 3),
            "gemm_tflops": round(fl / (gm * 1e-3) / 1e12, 1),
            "roofline_us": round(r_us, 3), "bound": bound, "frac": round(r_us / (gm * 1e3), 4),
            "quantize_us": round(qm * 1e3, 3),
            "quantize_gbs": round(quant_bytes(M, K_ATTN) / (qm * 1e-3) / 1e9, 1),
        })
        tot_gemm_us += gm * 1e3
        tot_quant_us += qm * 1e3
        tot_gemm_bytes += by
        tot_quant_bytes += quant_bytes(M, K_ATTN)
    gemm_dominant = tot_gemm_us >= tot_quant_us
    if gemm_dominant:
        achieved = tot_gemm_bytes / (tot_gemm_us * 1e-6) / 1e9
        kernel = "nvfp4_gemm_kernel (all M of the sweep)"
        units = f"{tot_gemm_bytes:.0f} algorithmic bytes per sweep of 4 launches"
    else:
        achieved = tot_quant_bytes / (tot_quant_us * 1e-6) / 1e9
        kernel = "quantize_dynamic_kernel (all M of the sweep)"
        units = f"{tot_quant_bytes:.0f} algorithmic bytes per sweep"
    roof = {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": gemm_traffic() if gemm_dominant else None, "per": units,
            "peak_source": f"{peaks['source']} hbm_gbs (burst copy)"}

    line = {
        "metric": "NVFP4 GEMM TFLOPS and % of B200 FP4/HBM roofline per M x N x K",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3/16) -> fp32 acc -> bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
        "config": {"workload": "attn_proj_sweep N=768 K=6144 M={16,64,256,1024}",
                   "scales": f"{args.sf_layout} layout (both operands)",
                   "step": "per M: quantize_dynamic(A fp32: global scale, alpha, codes) + gemm; one CUDA graph",
                   "timing": ("one event pair per step, L2 flush before each (outside the pair)" if args.flush
                              else f"{args.steps} steps back to back between one event pair (graphs of "
                                   f"{nsets}-set rotations, then single sets)"),
                   "l2": ("flushed before every timed step (512 MB write, then 256 MB read)" if args.flush else
                          f"inputs larger than L2: {nsets} independent input sets of {set_bytes / 2**20:.0f} MiB "
                          f"(activations, weights, outputs) in rotation, {nsets * set_bytes / 2**20:.0f} MiB "
                          "in all, so each set was last touched nsets-1 steps ago"),
                   "parallelism": f"replicas x{world}"},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": sweep.h2d_bytes, "d2h_bytes_per_step": sweep.d2h_bytes,
                "ms_per_step": round(e2e_ms, 5),
                "how": ("eager public-API calls per step; pinned host A copied in on a second stream "
                        "into double-buffered device inputs (overlapping the previous step's kernels), "
                        "bf16 out copied back every step"),
                "outputs_match_graph": e2e_match},
        "gpu_launches": sweep.launches_per_step * args.steps,
        "roofline": roof,
        "per_shape": per_shape,
        "gemm_only_tflops": round(sweep.flops / (tot_gemm_us * 1e-6) / 1e12, 1),
        "clocks": clocks.summary(),
    }
    if rank == 0 and not args.no_context:
        line["context"] = context_gemms(dev, peaks)
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    for sw in sets:
        sw.graph = sw.graph_ev = None
    del rotation
    del graphs
    return line


# ------------------------------------------------------------------ the oracle (CPU)

class OracleSweep:
    """The oracle on a bounded sample of the sweep: for every M, the first r rows of A (global
    scale over the full A). Inputs, the weights' quantisation and dequantisation (the weights
    are static, as in the GPU step) and a calibration pass are prepared once, outside any
    timing. Each pass runs the oracle's quantisation of the A sample, its dequantisation and
    the oracle's product of the dequantised operands (oracle.gemm is exactly that composition;
    calling it would dequantise the 768 x 6144 weights again on every call, a fixed cost that
    would swamp small samples)."""

    def __init__(self):
        import oracle
        from nvfp4_block_scaled_08_b200 import workloads
        self.oracle = oracle
        cases = workloads.attn_proj_cases()
        self.Ms = [c.M for c in cases]
        b = cases[0].b().numpy()
        self.gb = oracle.global_scale(b)
        qb, sb = oracle.quantize(b, self.gb)
        self.deq_b = oracle.dequantize(qb, sb)
        self.a_all = [c.a().numpy() for c in cases]
        self.threads = os.cpu_count() or 1
        self.used_threads = 1
        t0 = time.perf_counter()
        self.one_pass([min(64, m) for m in self.Ms])
        self.per_row = (time.perf_counter() - t0) / sum(min(64, m) for m in self.Ms)

    def one_pass(self, rows, split=None):
        """One pass over the row sample; adds the quantise and GEMM seconds to split[0], [1]."""
        o = self.oracle
        f = 0.0
        for a, r in zip(self.a_all, rows):
            t0 = time.perf_counter()
            ga = o.global_scale(a)
            qa, sa = o.quantize(a[:r], ga)
            t1 = time.perf_counter()
            o.gemm_dequantized(o.dequantize(qa, sa), self.deq_b, o.alpha(ga, self.gb), threads=self.threads)
            t2 = time.perf_counter()
            self.used_threads = max(self.used_threads, min(r, self.threads))   # rows split over threads
            if split is not None:
                split[0] += t1 - t0
                split[1] += t2 - t1
            f += 2.0 * r * N_ATTN * K_ATTN
        return f

    def run(self, budget_s: float):
        """Passes over a row sample sized so that they take about budget_s (at least one
        pass). Returns (flops, seconds, threads, description)."""
        frac = min(1.0, budget_s / max(self.per_row * sum(self.Ms), 1e-9))
        rows = [max(1, int(round(m * frac))) for m in self.Ms]
        flops, passes = 0.0, 0
        self.split = [0.0, 0.0]
        self.used_threads = 1
        t0 = time.perf_counter()
        while True:
            flops += self.one_pass(rows, self.split)
            passes += 1
            if time.perf_counter() - t0 >= 0.8 * budget_s:
                break
        dt = time.perf_counter() - t0
        sample = (f"attn_proj sweep, first {rows} rows of M={list(M_SWEEP)} (global scale over the "
                  f"full A), N=768, K=6144, {passes} pass(es); weights quantised and dequantised "
                  f"outside timing; GEMM on up to {self.used_threads} threads (one per row), "
                  f"quantisation on one")
        return flops, dt, self.used_threads, sample


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(budget_s: float):
    sweep = OracleSweep()
    flops, dt, threads, sample = sweep.run(budget_s)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle", "sample": sample, "seconds": round(dt, 2),
            "quantize_seconds": round(sweep.split[0], 3), "gemm_seconds": round(sweep.split[1], 3),
            "cpu_model": cpu_model()}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    # every step a bounded sample, so that warm-up + K steps take about two minutes
    per_step = max(0.02, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    sweep = OracleSweep()
    for _ in range(args.warmup):
        sweep.run(per_step)
    tot_f = tot_t = tot_q = tot_g = 0.0
    info = None
    for _ in range(args.steps):
        f, t, th, sample = sweep.run(per_step)
        tot_f += f
        tot_t += t
        tot_q += sweep.split[0]
        tot_g += sweep.split[1]
        info = (th, sample)
    value = tot_f / tot_t / 1e12
    return {
        "impl": "reference",
        "metric": "NVFP4 GEMM TFLOPS and % of B200 FP4/HBM roofline per M x N x K",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded)",
        "config": {"workload": "attn_proj_sweep N=768 K=6144 M={16,64,256,1024}",
                   "note": "CPU oracle (test infrastructure) on a bounded row sample per step"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": info[0],
                         "kind": "oracle", "sample": info[1], "quantize_seconds": round(tot_q, 3),
                         "gemm_seconds": round(tot_g, 3), "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sf-layout", choices=["tiled", "linear"], default="tiled",
                    help="scale layout of both GEMM operands in the sweep (tiled: the layout the "
                         "tensor cores read, fetched without a re-layout step)")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the compute-bound context GEMMs reported after the timed step")
    ap.add_argument("--sets", type=int, default=8,
                    help="independent input sets rotated between steps (together larger than L2)")
    ap.add_argument("--flush", action="store_true",
                    help="flush L2 before every step instead of rotating input sets")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        # CPU only: rank 0 times the oracle, the other ranks exit without work
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        line = run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
