"""Benchmark of the CSA2 decode layer step on B200: Reindex mode at 1M context (batch 128, a pool of
2000 blocks x 8 positions, Top-512, 16 heads x 128 + a 128-token window).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One JSON line on rank 0. `value` is whole-job queries/s with inputs resident in HBM, timed with
CUDA events (max over ranks); `e2e` is the same through the C ABI with the step's inputs copied
from pinned host memory and its outputs copied back inside the timed region. `roofline` reports the
dominant kernel (the Reindex indexer) against the measured HBM copy bandwidth. `cpu_baseline` times
the CPU oracle on a bounded sample. With --gpus N > 1 (torchrun), every rank runs its own batch of
sequences (data parallel, no collective in the data path: weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode queries/s at 1M ctx; HBM GB/s as % of 8 TB/s roofline"
UNIT = "queries/s"
DEFAULT_WORKLOAD = "reindex_b128_n1m"


# ---------------------------------------------------------------------------------------------
# algorithmic bytes (reads of what the step must read, writes of what it must write; no scratch)
# ---------------------------------------------------------------------------------------------
def algorithmic_bytes(wl):
    """Per query: dict kernel -> bytes. Entry sizes: FP4 main row 128 + 16 B, indexer row 128 + 16 B,
    window row 256 B (FP8)."""
    k, win = wl.k, wl.win
    if wl.mode == "latent":
        # the pages' own shape: k selected latent entries (256 B codes + 32 B scales), the window rows
        # (512 B), the query and the output (64 heads x 512, bf16) and the indices, per row
        return {"append": 0, "index": 0, "attend": k * 288 + win * 512 + 2 * (64 * 512 * 2) + k * 4}
    if wl.mode == "latent_index":
        # the pages' own indexer: every visible MXFP4 key (64 B codes + 4 B scales), the query
        # (hi x 128 bf16), its position and the selected indices, per row
        return {"append": 0, "index": wl.context * 68 + wl.hi * 128 * 2 + 8 + k * 4, "attend": 0}
    q, out, iq, idx = 16 * 128 * 2, 16 * 128 * 2, 4 * 64 * 2, k * 4
    attend = k * 144 + win * 256 + q + idx + out
    if wl.mode == "reindex":
        index = wl.pool_blocks * wl.bs * 144 + wl.pool_blocks * 4 + 4 + iq + idx
        append = 256 * 2 + 256
    elif wl.mode == "full":
        index = wl.context * 144 + iq + idx + (wl.pool_blocks * 4 + 4 if wl.pool_blocks else 0)
        append = 3 * 256 * 2 + 144 * 2 + 256
    elif wl.mode == "minimal":
        index = 0
        append = 256 * 2 + 256
    elif wl.mode == "draft":
        # the tq rows of a sequence share one pass over its visible indexer keys: per row, 1/tq of it
        index = wl.context * 144 / wl.tq + iq + idx
        append = 3 * 256 * 2 + 144 * 2 + 256
    else:
        # prefill chunk: the chunk's rows share one pass over the visible indexer keys
        index = wl.context * 144 / wl.tq + iq + idx
        append = 3 * 256 * 2 + 144 * 2 + 256
    return {"append": append, "index": index, "attend": attend}


L2_BYTES = 126 * 1024 * 1024


def latent_flops(wl):
    """Tensor work of one latent row: S^T = L Q^T and O^T = L^T P^T over k + win keys, 64 heads and
    512 channels (2 flops per multiply-add)."""
    return 2 * 2 * 64 * 512 * (wl.k + wl.win)


def tensor_core_index(wl):
    """Several rows per sequence at a context of 8,192 or more (and k <= 1024) take the tensor-core
    filter of index_mma.cu."""
    return wl.mode in ("prefill", "draft") and wl.context >= 8192 and wl.k <= 1024


def kernels_per_step(wl):
    """Kernels one step launches: append 1; index: 3 for decode rows (zero + score + select); for
    several rows per sequence 6 on the tensor-core path (prep, sampled pass, threshold, filter, final
    selection, and the exact scan, which returns at once when no row was handed back), else 1;
    attention 1."""
    if wl.mode == "latent":
        return 1
    if wl.mode == "latent_index":
        return 3
    if wl.mode == "minimal":
        return 2
    if wl.mode in ("full", "reindex"):
        return 5
    return 8 if tensor_core_index(wl) else 3


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def fp4_tensor_peak():
    """Dense FP4 tensor TFLOP/s: the measured bf16 GEMM burst figure times the nominal FP4 : bf16
    ratio (9 : 2.25 PFLOP/s dense = 4)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return 4.0 * float(d["bf16_tflops"]), "measured bf16 burst x 4"
    return 4.0 * 1590.0, "fallback bf16 1.59 PFLOP/s x 4"


def bf16_peak():
    """Dense bf16 (= fp16) tensor TFLOP/s: the measured cuBLAS burst figure, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured bf16 burst"
    return 1590.0, "fallback bf16 1.59 PFLOP/s"


def kernel_source_hash(name):
    src = os.path.join(ROOT, "compressed_sparse_attention_append_b200", "csrc", name)
    with open(src, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel_file, workload):
    """Per-launch DRAM bytes of a kernel from profiles/traffic.txt, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    h = kernel_source_hash(kernel_file)
    with open(p) as f:
        for line in f:
            parts = line.split("#")[0].split()
            if len(parts) == 4 and parts[0] == kernel_file and parts[1] == workload and parts[2] == h:
                return int(parts[3])
    return None


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples go to $CSA2_CLOCKS_DIR when set (kept for inspection), else a temp dir
        d = os.environ.get("CSA2_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, f"csa2_clocks_rank{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv",
                                          "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if not self.proc or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9 or not c[1].split()[0].isdigit():
                    continue
                sm.append(int(c[1].split()[0]))
                mx = int(c[2].split()[0])
                for n, v in zip(names, c[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# NVML clock-event reason bits (nvmlClocksEventReason*), by the names the clock record uses
NVML_REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                ("sw_power_cap", 0x4))


def nvml_clock_summary(samples, window, max_mhz):
    """Median SM clock and the union of reasons over the (time, sm_mhz, reason_bits) samples that
    fall inside window = (t0, t1); None when no sample does."""
    t0, t1 = window
    inside = [s for s in samples if t0 is not None and t1 is not None and t0 <= s[0] <= t1]
    if not inside:
        return None
    sm = sorted(s[1] for s in inside)
    bits = 0
    for s in inside:
        bits |= s[2]
    return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max_mhz,
            "reasons": sorted(n for n, b in NVML_REASONS if bits & b), "samples": len(inside)}


def nvml_sample_loop(nv, handle, period, out, stop=lambda: False):
    """Writes one line "time sm_mhz reason_bits" per NVML reading of the SM clock and the
    clock-event reasons to the open file `out`, every `period` seconds, until stop() is true.
    Time is time.monotonic(), the same clock in every process of the host. Reads only."""
    reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
        nv.nvmlDeviceGetCurrentClocksThrottleReasons
    while not stop():
        t = time.monotonic()
        sm = int(nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM))
        bits = int(reasons(handle))
        out.write(f"{t:.6f} {sm} {bits}\n")
        out.flush()
        time.sleep(period)


def nvml_sampler_main(uuid, bus, period, path):
    """Body of the sampler process: the NVML device with this UUID (else this PCI address); the
    file gets "max <MHz>" first, then nvml_sample_loop's lines until the process is ended."""
    import pynvml

    pynvml.nvmlInit()
    try:
        h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
    except Exception:
        h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
    with open(path, "w") as f:
        f.write(f"max {int(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))}\n")
        f.flush()
        nvml_sample_loop(pynvml, h, period, f)


def read_nvml_samples(path):
    """(samples [(time, sm_mhz, reason_bits)], max_mhz) from a sampler file; complete lines only."""
    samples, mx = [], None
    try:
        with open(path) as f:
            for line in f:
                c = line.split()
                if not line.endswith("\n"):
                    break
                try:
                    if len(c) == 2 and c[0] == "max":
                        mx = int(c[1])
                    elif len(c) == 3:
                        samples.append((float(c[0]), int(c[1]), int(c[2])))
                except ValueError:
                    continue
    except OSError:
        pass
    return samples, mx


class NvmlClocks:
    """SM clock and clock-event reasons of one GPU, read through NVML about every `period` seconds
    by a separate process (so that sampling takes nothing from the process that launches the
    kernels); summary() keeps the samples taken between mark_start() and mark_end(). The timed
    region of a decode step lasts milliseconds, far below nvidia-smi's sampling period, so this is
    the record that can see inside it. Reads only: no clock or setting is changed."""

    def __init__(self, ident=None, period=0.001, path=None, start_timeout=10.0):
        self.ident, self.period, self.start_timeout = ident, period, start_timeout
        d = os.environ.get("CSA2_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = path or os.path.join(d, f"csa2_nvml_{os.getpid()}.txt")
        self.proc = None
        self.window = [None, None]

    @classmethod
    def for_device(cls, device, **kw):
        """Sampler of the NVML device that is CUDA device `device` (matched by UUID, else by PCI
        address); one that records nothing when the device properties are unavailable."""
        try:
            import torch

            p = torch.cuda.get_device_properties(device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return cls(("GPU-" + str(p.uuid), bus), **kw)
        except Exception:
            return cls(None, **kw)

    def __enter__(self):
        if self.ident is None:
            return self
        try:
            if os.path.exists(self.path):
                os.remove(self.path)
            code = (f"import sys; sys.path.insert(0, {ROOT!r}); import bench; "
                    f"bench.nvml_sampler_main({self.ident[0]!r}, {self.ident[1]!r}, {self.period!r}, {self.path!r})")
            self.proc = subprocess.Popen([sys.executable, "-c", code], stdout=subprocess.DEVNULL,
                                         stderr=subprocess.DEVNULL)
            t0 = time.monotonic()
            while time.monotonic() - t0 < self.start_timeout and self.proc.poll() is None:
                if len(read_nvml_samples(self.path)[0]) >= 2:
                    break
                time.sleep(0.02)
        except Exception:
            self.proc = None
        return self

    def mark_start(self):
        self.window[0] = time.monotonic()

    def mark_end(self):
        self.window[1] = time.monotonic()

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self._summary = self.summary()
        if not os.environ.get("CSA2_CLOCKS_DIR"):
            try:
                os.remove(self.path)  # kept only where the samples were asked for
            except OSError:
                pass

    def summary(self):
        if getattr(self, "_summary", None) is not None:
            return self._summary
        samples, mx = read_nvml_samples(self.path)
        return nvml_clock_summary(samples, tuple(self.window), mx)


def clocks_record(nvml, smi):
    """The clocks object of the JSON line: NVML samples inside the timed region when there are any,
    else nvidia-smi's samples around it; both sources' sample counts are given."""
    s = smi.summary()
    n = nvml.summary()
    if n is None:
        return dict(s, source="nvidia-smi -lms 100 around the timed region")
    return dict(n, source="NVML every ~1 ms from the launch of the timed region to its end", smi_samples=s.get("samples", 0),
                smi_sm_mhz=s.get("sm_mhz"), smi_reasons=s.get("reasons"))


# ---------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------------------------
def oracle_sample(wl_name, budget_s=12.0, context=None, seqs=(0, 1)):
    """Times the CPU oracle on whole decode steps of sampled sequences of the workload (their caches are
    built first, untimed); returns (queries/s, description, threads)."""
    import oracle
    from oracle import workload as OW

    oracle.build()
    wl = OW.workload(wl_name, context)
    seqs = list(seqs)
    built = [OW.build_sequence(wl, b) for b in seqs]
    rows = [0] if wl.mode == "prefill" else None
    per_step = 1 if wl.mode == "prefill" else wl.tq  # queries one oracle step answers
    n = 0
    t0 = time.perf_counter()
    while True:
        for c, inp in built:
            OW.run_step(c, wl, inp, rows=rows)
            n += per_step
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    what = {"prefill": "prefill query rows (one row per step)",
            "draft": f"query rows of whole multi-token decode steps ({wl.tq} rows per step)"}.get(wl.mode,
                                                                                             "whole decode steps")
    desc = (f"{n} {what} of {wl_name} (sequences {seqs} repeated, cache resident in host memory), "
            f"single-threaded C oracle, fp64, {el:.1f} s")
    return n / el, desc, 1


def _oracle_worker(job):
    wl_name, budget_s, context, seq = job
    v, _, _ = oracle_sample(wl_name, budget_s, context, seqs=(seq,))
    return v


def oracle_sample_all_cores(wl_name, budget_s=12.0, context=None, max_procs=16):
    """The same oracle, one process per host core (at most max_procs: each holds one sequence's
    dense cache), each timing its own sequence; returns (queries/s summed over the processes,
    description, processes). Processes are spawned, never forked from a process that used CUDA."""
    import multiprocessing as mp

    procs = max(1, min(os.cpu_count() or 1, max_procs))
    jobs = [(wl_name, budget_s, context, i) for i in range(procs)]
    with mp.get_context("spawn").Pool(procs) as pool:
        rates = pool.map(_oracle_worker, jobs)
    desc = (f"{procs} processes on {os.cpu_count()} host cores, each timing whole steps of its own sequence of "
            f"{wl_name} for {budget_s:.0f} s (single-threaded C oracle, fp64); rates summed")
    return sum(rates), desc, procs


# ---------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------
def shard_offset(rank, batch):
    """Weak scaling: rank r owns sequences r*batch .. r*batch+batch-1 of the global batch."""
    return rank * batch


def reduce_max(value, device, world):
    """The largest of the ranks' values (every rank calls it, in the same order)."""
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(units_per_rank_step, world, steps, ms_max):
    """Units all ranks processed per second, timed by the slowest rank."""
    return units_per_rank_step * world * steps / (ms_max / 1e3)


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import workloads as W
    from workloads import gpu as G

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    wl = W.WORKLOADS[args.workload]
    B = args.batch or wl.batch
    step = G.build(args.workload, batch=B, seq_offset=shard_offset(rank, B), context=args.context or None)
    wl = step.wl
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    kern = ("append", "index", "attend")
    ev = {k: [] for k in kern}
    # a step that reads less than the L2 holds is timed step by step with L2 flushed in between
    step_read = sum(algorithmic_bytes(wl).values()) * B * wl.tq
    flush = step_read < L2_BYTES
    scrub = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    step_ev = []

    def hook(name, phase):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        if phase == 0:
            ev[name].append([e, None])
        else:
            ev[name][-1][1] = e

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the clock samplers start before the warm-up, so that they are running when the timed region is
    with Clocks(local) as clk, NvmlClocks.for_device(dev) as nclk:
        for _ in range(args.warmup):
            step.run()
        barrier()
        # ---- timed region: K steps, per-kernel events on the launching stream ----
        torch.cuda._sleep(int(2e7))  # lets the host enqueue the K steps ahead of the GPU
        nclk.mark_start()
        start.record(stream)
        for _ in range(args.steps):
            if flush:
                scrub.zero_()  # writes twice the L2: the step reads its inputs from HBM
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            step.run()  # the composed entry point (its kernels overlap through programmatic launch)
            if flush:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(stream)
                step_ev.append((e0, e1))
        end.record(stream)
        barrier()
        nclk.mark_end()
        # per-kernel times: the same K steps as separate entry points with events between them
        torch.cuda._sleep(int(2e7))
        for _ in range(args.steps):
            if flush:
                scrub.zero_()
            step.run_parts(hook)
        barrier()
    ms = sum(a.elapsed_time(b) for a, b in step_ev) if flush else start.elapsed_time(end)
    kms = {k: sum(a.elapsed_time(b) for a, b in v) / max(1, len(v)) for k, v in ev.items()}
    ms_max = reduce_max(ms, dev, world)
    value = weak_value(B * wl.tq, world, args.steps, ms_max)
    launches = args.steps * kernels_per_step(wl)
    if wl.mode == "minimal":
        kms.pop("index", None)
    if wl.mode == "latent":
        kms.pop("index", None)
        kms.pop("append", None)
    if wl.mode == "latent_index":
        kms.pop("attend", None)
        kms.pop("append", None)

    # ---- end to end: host inputs -> C ABI call -> host outputs ----
    e2e = run_e2e(step, args, world, barrier)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peak, peak_kind = measured_peaks()
    ab = algorithmic_bytes(wl)
    # every kernel of the step against the HBM roofline (algorithmic bytes / its event time)
    per_kernel = {}
    tpeak, tpeak_kind = fp4_tensor_peak()
    # the prefill chunk's index step is a contraction: rows x visible positions x 256 channels
    p0 = wl.context - wl.tq
    macs = 256.0 * (wl.tq * p0 + wl.tq * (wl.tq + 1) / 2.0) * B
    for k, t_ms in kms.items():
        if t_ms <= 0:
            continue
        if wl.mode == "latent":
            # both contractions (S^T = L Q^T and O^T = L^T P^T) on fp16 tensor cores, next to the bytes
            nbytes = ab[k] * B
            flops = latent_flops(wl) * B
            per_kernel[k] = {"algorithmic_bytes_per_launch": int(nbytes), "ms_per_launch": round(t_ms, 5),
                             "achieved_gbs": round(nbytes / (t_ms / 1e3) / 1e9, 1),
                             "frac": round(nbytes / (t_ms / 1e3) / 1e9 / peak, 4),
                             "flops_per_launch": flops, "achieved_tflops": round(flops / (t_ms / 1e3) / 1e12, 1),
                             "tensor_frac_of_bf16_peak": round(flops / (t_ms / 1e3) / 1e12 / bf16_peak()[0], 4)}
        elif wl.mode == "prefill" and k == "index":
            tf = 2.0 * macs / (t_ms / 1e3) / 1e12
            per_kernel[k] = {"bound": "tensor", "flops_per_launch": 2.0 * macs, "ms_per_launch": round(t_ms, 5),
                             "achieved_tflops": round(tf, 1), "frac": round(tf / tpeak, 4)}
        elif ab.get(k):
            nbytes = ab[k] * B * wl.tq
            per_kernel[k] = {"algorithmic_bytes_per_launch": int(round(nbytes)), "ms_per_launch": round(t_ms, 5),
                             "achieved_gbs": round(nbytes / (t_ms / 1e3) / 1e9, 1),
                             "frac": round(nbytes / (t_ms / 1e3) / 1e9 / peak, 4)}
    dom = "attend" if wl.mode in ("minimal", "latent") else "index"
    mma_kernels = ("mma_prep_kernel + mma_score_kernel (sampled pass) + mma_tau_kernel + mma_score_kernel "
                   "(tensor-core filter) + mma_final_kernel + index_kernel (rows handed back)")
    if wl.mode == "prefill":
        dom_bytes = None
        dom_file, dom_kernels = "index_mma.cu", mma_kernels
    elif wl.mode == "draft":
        dom_bytes = int(round(ab[dom] * B * wl.tq))
        dom_file, dom_kernels = ("index_mma.cu", mma_kernels) if tensor_core_index(wl) else ("index.cu", "index_kernel")
    else:
        dom_bytes = ab[dom] * B
        # decode rows: the index step is zero_kernel + score_kernel + select_kernel (index_decode.cu)
        if wl.mode == "latent_index":
            dom_file, dom_kernels = "latent_index.cu", "mxfp4_kernel + lat_index_score_kernel + lat_index_select_kernel"
        elif dom == "index":
            dom_file, dom_kernels = "index_decode.cu", "zero_kernel + score_kernel + select_kernel"
        elif wl.mode == "latent":
            dom_file, dom_kernels = "latent.cu", "latent_attend_kernel"
        else:
            dom_file, dom_kernels = "attend.cu", "attend_kernel"
    dur_s = kms[dom] / 1e3
    if wl.mode == "prefill":
        # block-scaled FP4 MMA of every visible (row, position) pair of the chunk: 2 x rows x visible
        # positions x 256 channels of FP4 tensor work per index step, against the dense FP4 peak
        achieved = 2.0 * macs / dur_s / 1e12
        roof = {"kernel": dom, "kernels": dom_kernels, "bound": "tensor", "achieved": round(achieved, 1),
                "peak": round(tpeak, 1), "unit": "TFLOP/s", "frac": round(achieved / tpeak, 4),
                "peak_kind": tpeak_kind, "traffic": None, "flops_per_launch": 2.0 * macs,
                "ms_per_launch": round(kms[dom], 5)}
    else:
        achieved = dom_bytes / dur_s / 1e9
        roof = {"kernel": dom, "kernels": dom_kernels, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_kind": f"of {peak_kind}",
                "traffic": ncu_traffic(dom_file, args.workload), "algorithmic_bytes_per_launch": dom_bytes,
                "ms_per_launch": round(kms[dom], 5)}
    step_bytes = sum(ab.values()) * B * wl.tq
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic (seeded bf16 from an Irwin-Hall(12) near-Gaussian, sigma 1: |x| <= 6, so the +-26 clip "
                "of the workload statement never engages)",
        "config": {"workload": args.workload + (f"@ctx{wl.context}" if args.context else ""), "mode": wl.mode,
                   "batch_per_gpu": B, "query_rows_per_sequence": wl.tq, "context": wl.context,
                   "pool_blocks": wl.pool_blocks, "topk": wl.k, "query_heads": wl.hq, "head_dim": wl.d,
                   "indexer": ("none in the step (inherited selection)" if wl.mode == "latent" else
                               f"{wl.hi} heads x 128 over one MXFP4 key per entry, ReLU scores"
                               if wl.mode == "latent_index" else "4 heads x 64, FP4"),
                   "kv_cache": ("one 512-channel latent per entry (K = V), E2M1 + E4M3/16, window FP8 x 512"
                                if wl.mode == "latent" else
                                "MXFP4 indexer key only (E2M1 + E8M0/32, 68 B per entry)"
                                if wl.mode == "latent_index" else "E2M1 + E4M3/16 (FP4), window FP8"),
                   "window": wl.win, "parallelism": f"dp{world}",
                   "l2": (f"L2 flushed between timed steps (a step reads {step_bytes / 1e6:.0f} MB, less than the L2)"
                          if flush else f"inputs larger than L2 ({step_bytes / 1e6:.0f} MB read per step)"),
                   "step_hbm_gbs": round(step_bytes / (ms_max / args.steps / 1e3) / 1e9, 1),
                   "accumulate": "fp32 attention, exact fp64 index scores"},
        "kernel_ms": {k: round(v, 5) for k, v in kms.items()},
        "roofline": roof,
        "rooflines": per_kernel,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks_record(nclk, clk),
    }
    if world == 1 and not args.no_cpu_baseline:
        v, desc, cores = oracle_sample(args.workload, budget_s=args.cpu_budget, context=args.context or None)
        line["cpu_baseline"] = {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
        v, desc, cores = oracle_sample_all_cores(args.workload, budget_s=args.cpu_budget, context=args.context or None)
        line["cpu_baseline_all_cores"] = {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                                          "sample": desc}
    print(json.dumps(line), flush=True)


def pack(tensors, device, pinned=False):
    """One byte buffer holding every tensor of `tensors` (256-byte aligned slots) and views into it
    with the tensors' shapes and dtypes; the views are filled with the tensors' values."""
    import torch

    offs, off = {}, 0
    for n, t in tensors.items():
        offs[n] = off
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(max(off, 256), dtype=torch.uint8, device=device, pin_memory=pinned)
    views = {}
    for n, t in tensors.items():
        nb = t.numel() * t.element_size()
        v = buf[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape)
        v.copy_(t)
        views[n] = v
    return buf, views


def run_e2e(step, args, world, barrier):
    """The step through the public entry point with its inputs copied from pinned host memory and its
    outputs copied back inside the timed region, as a serving loop runs it: the inputs of a step live
    in one pinned host buffer and one device buffer (one cudaMemcpyAsync per direction), and so do the
    outputs. Two slots of device buffers alternate, and each copy direction has a stream of its own,
    so that a step's host-to-device copy overlaps the previous step's compute and its device-to-host
    copy the next step's. The timed region ends after the last step's outputs reached the host."""
    import torch

    wl = step.wl
    if wl.mode == "prefill":
        names_in = ["kv", "idx_k", "swa_kv", "idx_q", "q"]
    else:
        names_in = [n for n in ("pos", "qpos", "swa_kv", "idx_q", "q", "pool", "pool_n", "kv", "idx_k", "idx")
                    if n in step.inputs]
    names_out = [n for n in ("out", "idx") if n in step.outputs and not (n == "idx" and wl.mode == "minimal")]
    dev = step.inputs[names_in[0]].device
    slots = []
    for _ in range(2):
        d_in, v_in = pack({n: step.inputs[n] for n in names_in}, dev)
        d_out, v_out = pack({n: step.outputs[n] for n in names_out}, dev)
        h_out = torch.empty(d_out.numel(), dtype=torch.uint8, pin_memory=True)
        slots.append((d_in, v_in, d_out, v_out, h_out))
    h_in, _ = pack({n: step.inputs[n].cpu() for n in names_in}, "cpu", pinned=True)
    saved_in, saved_out = dict(step.inputs), dict(step.outputs)
    h2d = sum(step.inputs[n].numel() * step.inputs[n].element_size() for n in names_in)
    d2h = sum(step.outputs[n].numel() * step.outputs[n].element_size() for n in names_out)
    stream = torch.cuda.current_stream()
    # one stream per copy direction: a step's host-to-device copy must not queue behind the
    # previous step's device-to-host copy (which waits for that step's compute)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "done", "out")}
    K = max(1, args.steps)

    def steps(n, first):
        for i in range(n):
            sl = i % 2
            d_in, v_in, d_out, v_out, h_out = slots[sl]
            with torch.cuda.stream(up):
                if i >= 2 or not first:
                    up.wait_event(ev["done"][sl])  # the step two back has read this slot's inputs
                d_in.copy_(h_in, non_blocking=True)
                ev["in"][sl].record(up)
            stream.wait_event(ev["in"][sl])
            if i >= 2 or not first:
                stream.wait_event(ev["out"][sl])  # and its outputs have reached the host
            step.inputs.update(v_in)
            step.outputs.update(v_out)
            step.run()
            ev["done"][sl].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev["done"][sl])
                h_out.copy_(d_out, non_blocking=True)
                ev["out"][sl].record(down)
        last = (n - 1) % 2
        stream.wait_event(ev["out"][last])
        if n >= 2:
            stream.wait_event(ev["out"][1 - last])

    try:
        steps(2, True)
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(2e7))
        s.record(stream)
        up.wait_event(s)
        down.wait_event(s)
        steps(K, False)
        e.record(stream)
        barrier()
    finally:
        step.inputs.clear()
        step.inputs.update(saved_in)
        step.outputs.clear()
        step.outputs.update(saved_out)
    ms = reduce_max(s.elapsed_time(e), "cuda", world)
    v = weak_value(step.batch * wl.tq, world, K, ms)
    return {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / K, 5), "call": e2e_call(wl.mode),
            "copies": "one cudaMemcpyAsync host->device and one device->host per step (packed pinned buffers, "
                      "two slots, one stream per copy direction, overlapping the neighbouring steps' compute)"}


def e2e_call(mode):
    """The public entry point(s) one end-to-end step goes through."""
    if mode == "latent":
        return "csa2_latent_attend"
    if mode == "latent_index":
        return "csa2_latent_index_topk"
    if mode == "prefill":
        return "csa2_prefill_chunk"
    if mode == "draft":
        return "csa2_quantize_append + csa2_index_topk_full + csa2_sparse_attend (tq rows)"
    return f"csa2_decode_{mode}"


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    v, desc, cores = oracle_sample_all_cores(args.workload, budget_s=per_step * max(1, args.steps),
                                             context=args.context or None)
    line = {"metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload},
            "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=0, help="sequences per GPU (default: the workload's)")
    ap.add_argument("--context", type=int, default=0, help="context override (profiling small cases)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
