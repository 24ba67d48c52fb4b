"""Benchmark of the paged-KV decode step on B200.

One step = the whole hot path on one batch: copy-on-write block copies (when
the workload has them), slot of every appended token, scatter of the new K/V
rows, decode attention (plus the log-sum-exp reduce when a context spans
several partitions). The step is captured once in a CUDA graph (the launch
path of a serving decode loop) and replayed; every replay is bracketed by
timing events recorded inside the graph. Before every timed step a 512 MiB
buffer is written and then read back, which evicts the 126 MB L2 without
leaving dirty lines whose write-back would land in the timed step, so the KV
bytes come from HBM.

By default one run times the decode workloads 3, 2, 4 and 5 in turn. The
JSON line's top level is the first of them (the Llama2-13B-shaped
mixed-length batch); the others sit under "workloads", each with its own
roofline, end-to-end figure, clocks and CPU baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1..5 | --workloads 3,2,4,5]
                    [--impl ours|reference]
    python bench.py --prefill 1..3      (paged prefill: TFLOP/s against the tensor peak)

Under torchrun each rank runs its own independently seeded batch of the same
shape (sequences are independent; there is no exchange step), and rank 0
prints one JSON line with the slowest rank's times.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = ("paged decode attention KV GB/s (% of B200 HBM peak) and decode tokens/s, 1 GPU")
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 512 << 20


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("pa_decode.cuh", "pa_device.cuh", "pa_cache_ops.cuh")
PREFILL_SOURCES = ("pa_prefill.cuh", "pa_decode.cuh", "pa_device.cuh")


def code_tokens(src: str) -> str:
    """C++ source without its comments, whitespace runs collapsed to one
    space (string and character literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(names=DECODE_SOURCES) -> str:
    """Hash of the device code (kernels and their helpers; not the host-side
    launch logic), so a recorded ncu traffic figure is dropped when a kernel
    changes. Comments and layout do not count."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "pagedattention_paged_kv_decode_b200", "csrc")
    for name in names:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, record: str = "decode_dram_traffic.json", names=DECODE_SOURCES):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", record)
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get(workload)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash(names):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """Clock and throttle-reason samples while the timed region runs: NVML
    read about every millisecond (queries only; nothing is set), else
    nvidia-smi every 200 ms. Rows keep nvidia-smi's field order."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None
        self.source = "nvidia-smi"
        self._stop = threading.Event()

    def _start_nvml(self) -> bool:
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = (nv.nvmlDeviceGetHandleByUUID(self.gpu) if self.gpu.startswith(("GPU-", "MIG-"))
                 else nv.nvmlDeviceGetHandleByIndex(int(self.gpu)))
            max_sm = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            bits = (nv.nvmlClocksThrottleReasonHwSlowdown, nv.nvmlClocksThrottleReasonHwThermalSlowdown,
                    nv.nvmlClocksThrottleReasonSwThermalSlowdown, nv.nvmlClocksThrottleReasonSwPowerCap)
            reasons(h)
        except Exception:
            return False

        def loop():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    r = reasons(h)
                except Exception:
                    break
                self.rows.append((time.time(), ["", str(self.gpu), str(sm), str(max_sm), "", hex(r)] +
                                  ["Active" if r & bit else "Not Active" for bit in bits]))
                self._stop.wait(0.001)
            try:
                nv.nvmlShutdown()
            except Exception:
                pass

        self.source = "nvml"
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        return True

    def start(self):
        if self._start_nvml():
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        self._stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        # nvidia-smi's 200 ms period may put no sample inside a short timed
        # region, so it takes a quarter second on either side; NVML samples
        # are taken inside the region only (the nearest one if none is)
        slack = 0.25 if self.source == "nvidia-smi" else 0.0
        rows = [r for t, r in self.rows if t0 - slack <= t <= t1 + slack]
        if not rows and self.rows:
            rows = ([r for _, r in self.rows] if self.source == "nvidia-smi" else
                    [min(self.rows, key=lambda tr: min(abs(tr[0] - t0), abs(tr[0] - t1)))[1]])
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 6 + i and r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "source": self.source}


# ----------------------------------------------------------------- our arm

class PackedInputs:
    """The per-step inputs of a step packed back to back (256-byte aligned)
    in one device buffer and one pinned host buffer, so that the end-to-end
    path moves them with a single host-to-device copy. The device tensors
    the step (and its CUDA graph) uses are views into the device buffer."""

    def __init__(self, torch, tensors: dict, device):
        offs, off = {}, 0
        for k, t in tensors.items():
            nbytes = t.numel() * t.element_size()
            offs[k] = (off, nbytes)
            off = (off + nbytes + 255) // 256 * 256
        self.dev = torch.empty(max(off, 256), dtype=torch.uint8, device=device)
        self.host = torch.empty(max(off, 256), dtype=torch.uint8).pin_memory()
        self.views = {}
        for k, t in tensors.items():
            o, nb = offs[k]
            v = self.dev[o:o + nb].view(t.dtype).view(t.shape)
            v.copy_(t)
            self.host[o:o + nb].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
            self.views[k] = v
        self.nbytes = int(self.host.numel())

    def upload(self):
        self.dev.copy_(self.host, non_blocking=True)



def slowest_rank(times, dist=None, device=None):
    """Max over ranks of each per-rank mean time (the only collective: timing)."""
    import torch
    t = torch.tensor([float(x) for x in times], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def aggregate_gbs(world: int, bytes_per_rank: int, ms: float) -> float:
    """Whole-job throughput: every rank processed its own batch in <= ms."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


HEADLINE_WORKLOAD = 3
DEFAULT_WORKLOADS = "3,2,4,5"   # headline first; the others are reported beside it


def decode_arithmetic(w) -> str:
    """The arithmetic the decode kernel does for this cache type."""
    return ("fp32 sums of exact products of the fp16 query with keys decoded exactly from E4M3 "
            "codes to fp16; softmax weights rounded to fp16 for the exact products with the "
            "decoded values, summed in fp32" if w.kv_dtype == "e4m3" else
            "fp32 sums of exact fp16 x fp16 products (query x key); softmax weights rounded to "
            "fp16 for the exact products with the values, summed in fp32")


def empty_graph_ms(torch, stream, steps: int) -> float:
    """Floor of the event timing: one tiny kernel captured in a graph between
    two timing events, replayed like a step (mean over `steps` replays)."""
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    x = torch.zeros(1, dtype=torch.int32, device=stream.device)
    with torch.cuda.stream(stream):
        x.add_(1)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            ev[0].record()
            x.add_(1)
            ev[1].record()
        ts = []
        for i in range(3 + steps):
            g.replay()
            stream.synchronize()
            if i >= 3:
                ts.append(ev[0].elapsed_time(ev[1]))
    del g
    return statistics.mean(ts)


def read_floor_ms(torch, stream, nbytes: int, evict, steps: int) -> float:
    """Reference for the decode's byte rate: a plain reduction (torch's
    sum) over nbytes of fp16 in one contiguous buffer, captured in a graph
    between two timing events and replayed after the same L2 eviction as a
    step (mean over `steps` replays). It reads the same number of bytes as
    the decode's K/V stream with no gather, no block table and no softmax."""
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    buf = torch.ones(max(nbytes // 2, 1), dtype=torch.float16, device=stream.device)
    res = torch.zeros((), dtype=torch.float32, device=stream.device)
    with torch.cuda.stream(stream):
        res.copy_(buf.sum(dtype=torch.float32))
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            ev[0].record()
            res.copy_(buf.sum(dtype=torch.float32))
            ev[1].record()
        ts = []
        for i in range(3 + steps):
            evict()
            g.replay()
            stream.synchronize()
            if i >= 3:
                ts.append(ev[0].elapsed_time(ev[1]))
    del g, buf
    return statistics.mean(ts)


def measure_decode(args, wid, rank, world, local_rank, dist, cpu_seconds, with_swap):
    """One decode workload: build, capture the step in a CUDA graph, time it
    (and its end-to-end form from pinned host buffers), and return the
    result dict on rank 0 (None elsewhere). Every rank takes the same
    collective steps in the same order."""
    import torch
    import pagedattention_paged_kv_decode_b200 as pk

    dev = torch.device("cuda", local_rank)
    w = W.named(wid, seed=W.rank_seed(1000 + wid, rank), num_seqs=args.num_seqs or None)
    dw = W.to_device(w, dev, encode=pk.load_cache)
    S = w.num_seqs
    bound = w.max_blocks_per_seq * w.block_size  # host-side bound: table capacity, no sync
    launch = None
    if args.launch:
        launch = dict(zip(("partition_size", "heads_per_cta", "warps_per_head", "stages"),
                          (int(x) for x in args.launch.split(","))))
    shared = bool(w.shared_blocks) and not args.no_shared_prefix and not args.unfused
    cfg = pk.choose_config(dw.key_cache, S, bound, launch)
    parts = -(-bound // cfg["partition_size"])
    launches_per_step = ((3 if args.unfused else 1) + (1 if w.cow_pairs.size else 0)
                         + (1 if parts > 1 else 0))
    if shared:   # prefix kernel + decode of the private parts + reduce
        launches_per_step = 3 + (1 if w.cow_pairs.size else 0)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)

    stream = torch.cuda.Stream(dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
    packed = PackedInputs(torch, {k: getattr(dw, k) for k in ("query", "new_key", "new_value", "block_tables",
                                                               "context_lens", "cow_pairs")}, dev)
    for k, v in packed.views.items():
        setattr(dw, k, v)

    def step():
        ev[0].record()
        if w.cow_pairs.size:
            pk.copy_blocks(dw.key_cache, dw.value_cache, dw.cow_pairs)
        if args.unfused:
            pk.slot_mapping(dw.block_tables, dw.context_lens, dw.key_cache, out=dw.slots)
            pk.kv_cache_write(dw.new_key, dw.new_value, dw.key_cache, dw.value_cache, dw.slots,
                              w.k_scale, w.v_scale)
            ev[1].record()
            pk.paged_attention_decode(dw.out, dw.query, dw.key_cache, dw.value_cache,
                                      dw.block_tables, dw.context_lens, w.scale, w.k_scale,
                                      w.v_scale, max_context_len=bound)
        elif shared:
            ev[1].record()
            pk.paged_attention_decode_shared_prefix(dw.out, dw.query, dw.key_cache, dw.value_cache,
                                                    dw.block_tables, dw.context_lens,
                                                    w.shared_blocks, w.scale, w.k_scale, w.v_scale,
                                                    new_key=dw.new_key, new_value=dw.new_value,
                                                    max_context_len=bound, slot_mapping=dw.slots,
                                                    config=launch)
        else:
            ev[1].record()
            pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value,
                                             dw.key_cache, dw.value_cache, dw.block_tables,
                                             dw.context_lens, w.scale, w.k_scale, w.v_scale,
                                             max_context_len=bound, slot_mapping=dw.slots,
                                             config=launch)
        ev[2].record()

    with torch.cuda.stream(stream):
        for _ in range(3):          # un-captured warm-up: sizes the split workspace, sets attributes
            step()
        stream.synchronize()
        assert pk.check_status(stream) == 0
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        stream.synchronize()

        def evict_l2():
            # Write a buffer 4x the L2, then read it back: the read pass evicts
            # the written lines (their write-back happens here, outside the timed
            # step) and leaves L2 holding clean lines of the flush buffer only.
            flush.fill_(1)
            flush_sink.copy_(flush.view(torch.int64).sum())

        def timed_step():
            evict_l2()
            graph.replay()
            stream.synchronize()
            return ev[0].elapsed_time(ev[2]), ev[1].elapsed_time(ev[2])

        for _ in range(max(3, args.warmup)):
            timed_step()

        visible = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
        sampler = ClockSampler(visible[local_rank] if len(visible) > local_rank and visible[local_rank]
                               else str(local_rank))
        sampler.start()
        time.sleep(0.3)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        step_ms, dec_ms = [], []
        for _ in range(args.steps):
            a, b = timed_step()
            step_ms.append(a)
            dec_ms.append(b)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        t1 = time.time()
        sampler.stop()
        assert pk.check_status(stream) == 0

        # ------------------------------------------------ end to end (host buffers)
        # One graph holds the whole end-to-end step: the copy of the packed
        # per-step inputs from pinned host memory, the step's launches and the
        # copy of the output back to pinned host memory (one submission, as a
        # serving loop replays it).
        host_out = torch.empty(dw.out.shape, dtype=dw.out.dtype).pin_memory()
        e2e_start = torch.cuda.Event(enable_timing=True)
        e2e_end = torch.cuda.Event(enable_timing=True)
        h2d = packed.nbytes
        d2h = host_out.numel() * host_out.element_size()
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph, stream=stream):
            packed.upload()
            step()
            host_out.copy_(dw.out, non_blocking=True)
        stream.synchronize()
        e2e_ms = []
        e2e_warm = max(20, args.warmup)  # untimed: the first replays of a new graph with host copies run slow
        for i in range(e2e_warm + args.steps):
            evict_l2()
            e2e_start.record()
            e2e_graph.replay()
            e2e_end.record()
            stream.synchronize()
            if i >= e2e_warm:
                e2e_ms.append(e2e_start.elapsed_time(e2e_end))

        # ------------------------------------------------ swap to/from pinned host memory
        swap = measure_swap(pk, dw, stream, torch) if with_swap else None
        floor = empty_graph_ms(torch, stream, max(20, args.steps))
        read_ms = read_floor_ms(torch, stream, w.unique_kv_bytes(), evict_l2, max(20, args.steps))

    step_t, dec_t, e2e_t, floor_t, read_t = slowest_rank(
        [statistics.mean(step_ms), statistics.mean(dec_ms), statistics.mean(e2e_ms), floor, read_ms], dist, dev)
    clocks = sampler.summary(t0, t1)
    del graph, e2e_graph
    del dw, flush, packed
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    kv = w.kv_bytes()
    peak, peak_kind = hbm_peak()
    dec_bytes = w.decode_bytes() if args.unfused else W.fused_step_bytes(w)
    achieved = dec_bytes / (dec_t * 1e-3) / 1e9
    value = aggregate_gbs(world, kv, step_t)
    roofline = {
        "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
        "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
        "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
        "traffic": recorded_traffic(w.name),
        "kernel": ("paged_prefix_kernel + paged_decode_kernel (fused append) + lse_reduce_kernel"
                   if shared else "paged_decode_kernel" + ("" if args.unfused else " (fused append)")
                   + (" + lse_reduce_kernel" if parts > 1 else "")),
        "algorithmic_bytes_per_launch": dec_bytes,
    }
    if w.shared_blocks:
        uniq = dec_bytes - kv + w.unique_kv_bytes()
        roofline.update(
            unique_bytes_per_launch=uniq,
            unique_achieved=round(uniq / (dec_t * 1e-3) / 1e9, 2),
            unique_frac=round(uniq / (dec_t * 1e-3) / 1e9 / peak, 4),
            note="algorithmic bytes count the shared prefix once per sequence (logical); the unique "
                 "figures count each distinct cache row once")
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "ms_per_step": round(step_t, 5),
        "dtype": "f32",
        "arithmetic": decode_arithmetic(w),
        "kv_dtype": w.kv_dtype,
        "config": {
            "workload": w.name, "num_seqs": S, "num_heads": w.num_heads,
            "head_size": w.head_size, "block_size": w.block_size, "kv_dtype": w.kv_dtype,
            "num_blocks": w.num_blocks, "mean_context": round(float(w.context_lens.mean()), 1),
            "max_context": w.max_context_len, "kv_bytes_per_step": kv,
            "launch": cfg, "parallelism": f"replicas x{world} (independent batches, no collective)",
            "l2": "before every timed step a 512 MiB buffer is written then read (L2 is 126 MB): "
                  "no step data and no dirty lines left in L2",
            "step": "CUDA graph: " + ("copy_blocks, " if w.cow_pairs.size else "")
                    + ("slot_mapping, kv_cache_write, paged_attention_decode" if args.unfused
                       else ("paged_attention_decode_shared_prefix (prefix kernel over the "
                             f"{w.shared_blocks} shared blocks + fused append/decode of the rest "
                             "+ lse reduce)") if shared
                       else "paged_attention_decode_append (slot + K/V store + decode in one launch)")
                    + (" (+lse reduce)" if parts > 1 and not shared else ""),
        },
        "tokens_per_s": round(world * S / (step_t * 1e-3), 1),
        "hbm_pct_of_nominal_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "hbm_pct_of_measured": round(100 * value / world / peak, 2),
        "decode_ms": round(dec_t, 5),
        "decode_kv_gbs": round(kv / (dec_t * 1e-3) / 1e9, 2),
        "empty_graph_ms": round(floor_t, 5),
        "plain_read": {"ms": round(read_t, 5), "bytes": w.unique_kv_bytes(),
                       "gbs": round(w.unique_kv_bytes() / (read_t * 1e-3) / 1e9, 2),
                       "what": "torch sum over one contiguous fp16 buffer of the step's distinct K/V bytes, "
                               "same graph, events and L2 eviction (a reference rate for this size, not our kernel)"},
        "roofline": roofline,
        "e2e": {"value": round(aggregate_gbs(world, kv, e2e_t), 2), "unit": "GB/s",
                "ms_per_step": round(e2e_t, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "one CUDA graph per step: pinned host inputs (one packed buffer) -> one copy to the "
                        "device -> the step's launches -> output to pinned host"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if swap is not None:
        res["swap_blocks"] = swap
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_both(w, cpu_seconds)
    return res


def run_ours(args, rank, world, local_rank):
    import torch

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    ids = [args.workload] if args.workload else [int(x) for x in args.workloads.split(",")]
    results = []
    for i, wid in enumerate(ids):
        secs = args.cpu_seconds if i == 0 else max(1.0, args.cpu_seconds / 3)
        results.append(measure_decode(args, wid, rank, world, local_rank, dist, secs, with_swap=(i == 0)))
    if dist:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps(assemble_line(results, args, world)), flush=True)


def assemble_line(results, args, world):
    """The JSON line: the first workload's result at the top level (the
    contract's keys first), the others under "workloads" by name."""
    head = results[0]
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "data": "synthetic (seeded numpy PCG64; no dataset)",
    }
    line.update({k: v for k, v in head.items() if k not in line})
    if len(results) > 1:
        line["workloads"] = {r["config"]["workload"]: {k: v for k, v in r.items() if k != "metric"}
                             for r in results[1:]}
        line["gpu_launches_all_workloads"] = sum(r["gpu_launches"] for r in results)
    return line


def measure_swap(pk, dw, stream, torch, n_blocks: int = 256, reps: int = 5):
    """Block swap between the device pool and a pinned host pool (the pages'
    --swap-space), outside the timed decode steps: GB/s of K+V moved out
    (device -> host) and in (host -> device), n_blocks blocks per call."""
    kc, vc = dw.key_cache, dw.value_cache
    n = min(n_blocks, kc.shape[0])
    hk = torch.empty((n,) + tuple(kc.shape[1:]), dtype=kc.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    pairs_out = torch.stack([torch.arange(n), torch.arange(n)], 1).to(torch.int32).to(kc.device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    res = {}
    for name, call in (("out", lambda: pk.swap_blocks(hk, hv, kc, vc, pairs_out)),
                       ("in", lambda: pk.swap_blocks(kc, vc, hk, hv, pairs_out))):
        call()
        ts = []
        for _ in range(reps):
            e0.record()
            call()
            e1.record()
            stream.synchronize()
            ts.append(e0.elapsed_time(e1))
        nbytes = 2 * n * kc[0].numel() * kc.element_size()
        res[f"{name}_gbs"] = round(nbytes / (statistics.mean(ts) * 1e-3) / 1e9, 2)
    assert pk.check_status(stream) == 0
    res.update(blocks=n, bytes_per_call=2 * n * kc[0].numel() * kc.element_size(),
               host="pinned host pool read/written by the swap kernel over the host link")
    return res


# ------------------------------------------------------------- CPU oracle

class OracleState:
    """Host pools of a workload for the oracle, built once (and, for E4M3,
    encoded block by block as sampled sequences first need them)."""

    def __init__(self, w):
        self.pk, self.pv = w.pool_host()
        if w.kv_dtype == "e4m3":
            self.kc = np.zeros(self.pk.shape, np.uint8)
            self.vc = np.zeros(self.pv.shape, np.uint8)
            self.encoded = np.zeros(w.num_blocks, bool)
        else:
            self.kc, self.vc = self.pk, self.pv
            self.encoded = None


def _encode_blocks(w, state: "OracleState", seqs) -> None:
    """E4M3 pools: encode (with the oracle's cache write) the blocks of the
    given sequences that are not encoded yet. Outside every timed region."""
    import oracle
    if w.kv_dtype != "e4m3":
        return
    bt = w.block_tables[np.asarray(seqs)]
    blocks = np.unique(bt[bt >= 0])
    blocks = blocks[~state.encoded[blocks]].astype(np.int64)
    if blocks.size:
        slots = (blocks[:, None] * w.block_size + np.arange(w.block_size)).reshape(-1).astype(np.int32)
        oracle.kv_cache_write(state.pk[blocks].reshape(-1, w.num_heads, w.head_size),
                              state.pv[blocks].reshape(-1, w.num_heads, w.head_size), state.kc, state.vc,
                              slots, w.k_scale, w.v_scale)
        state.encoded[blocks] = True


def _oracle_steps(w, state: "OracleState", seqs, threads) -> None:
    """The oracle's decode step for the given sequences (all heads each):
    copy-on-write pairs, slots, cache write, attention."""
    import oracle
    seqs = np.asarray(seqs)
    kc, vc, ctx = state.kc, state.vc, w.context_lens
    if w.cow_pairs.size:
        oracle.copy_blocks(kc, vc, w.cow_pairs[seqs])
    slot = oracle.slot_mapping(w.block_tables[seqs], ctx[seqs], w.block_size)
    oracle.kv_cache_write(w.new_key[seqs], w.new_value[seqs], kc, vc, slot, w.k_scale, w.v_scale)
    pairs = np.stack([np.repeat(seqs, w.num_heads), np.tile(np.arange(w.num_heads), seqs.size)],
                     1).astype(np.int32)
    oracle.paged_attention(w.query, kc, vc, w.block_tables, ctx, w.scale, w.k_scale, w.v_scale,
                           seq_head=pairs, threads=threads)


def cpu_baseline(w, seconds: float, state: "OracleState | None" = None, start: int = 0,
                 threads: int | None = None):
    """The oracle on this host: whole decode steps of a bounded, seeded sample
    of the workload's sequences (all heads of each; at least one call).
    threads=None: one sequence per call on one thread. threads=n (0: every
    core): calls of enough sequences to give each thread two (sequence,
    head) pairs, spread over n OpenMP threads. Building the host pools (and,
    for E4M3, encoding the sampled sequences' blocks) happens outside the
    timed region. Returns the same GB/s metric."""
    import oracle
    order = np.random.default_rng(0).permutation(w.num_seqs)
    state = state or OracleState(w)
    cores = 1 if threads is None else (threads or oracle.max_threads())
    per_call = 1 if threads is None else max(1, -(-2 * cores // w.num_heads))
    done_bytes, elapsed, n, calls = 0, 0.0, 0, 0
    while elapsed < seconds and calls < 100000:
        seqs = [int(order[(start + n + k) % w.num_seqs]) for k in range(per_call)]
        _encode_blocks(w, state, seqs)
        t = time.perf_counter()
        _oracle_steps(w, state, seqs, threads)
        elapsed += time.perf_counter() - t
        done_bytes += sum(int(w.context_lens[s]) for s in seqs) * w.num_heads * w.head_size * w.elem_bytes * 2
        n += per_call
        calls += 1
    how = ("single-thread fp64" if threads is None else
           f"fp64, (sequence, head) pairs over {cores} OpenMP threads, {per_call} sequences per call")
    return {"value": round(done_bytes / elapsed / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{n} sequences (all {w.num_heads} heads each) of {w.name}, one decode step "
                      f"each (copy-on-write, slot, cache write, attention): {elapsed:.1f} s, {how}"}


def cpu_baseline_both(w, seconds: float) -> dict:
    """The multi-core oracle (every host core) as the baseline, with the
    single-thread figure beside it; each leg takes about `seconds`."""
    state = OracleState(w)
    single = cpu_baseline(w, seconds, state)
    multi = cpu_baseline(w, seconds, state, threads=0)
    multi["single_thread"] = {k: single[k] for k in ("value", "cores", "sample")}
    multi["host_cpu_count"] = os.cpu_count()
    return multi


# ------------------------------------------------------------ paged prefill

PREFILL_METRIC = "paged prefill attention TFLOP/s (causal, over the block table), 1 GPU"


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            rec = json.load(f)
        return float(rec["bf16_tflops"]), float(rec["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def run_prefill(args, rank, world, local_rank):
    """One prefill step = slots of the chunk's tokens, their K/V scattered into
    the cache, causal attention of the chunk over the block table. Same
    capture, L2 eviction, timing, clock and end-to-end rules as the decode."""
    import torch
    import pagedattention_paged_kv_decode_b200 as pk

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = W.prefill_named(args.prefill, seed=W.rank_seed(2000 + args.prefill, rank))
    dp = W.prefill_to_device(w, dev)
    mql = int(w.chunk_lens.max(initial=0))
    tc = w.head_size in (64, 128) and w.scale > 0  # the library's choice of prefill kernel
    T = w.total_q
    n_write = -(-T // 65535)  # the library launches the cache write in slices of 65535 tokens
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)
    stream = torch.cuda.Stream(dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
    packed = PackedInputs(torch, {k: getattr(dp, k) for k in ("query", "new_key", "new_value", "query_start",
                                                               "block_tables", "context_lens")}, dev)
    for k, v in packed.views.items():
        setattr(dp, k, v)

    def step():
        ev[0].record()
        pk.prefill_slot_mapping(dp.query_start, dp.block_tables, dp.context_lens, dp.key_cache, mql,
                                out=dp.slots)
        pk.kv_cache_write(dp.new_key, dp.new_value, dp.key_cache, dp.value_cache, dp.slots)
        ev[1].record()
        pk.paged_prefill(dp.out, dp.query, dp.query_start, dp.key_cache, dp.value_cache, dp.block_tables,
                         dp.context_lens, mql, w.scale)
        ev[2].record()

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
        stream.synchronize()
        assert pk.check_status(stream) == 0
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        stream.synchronize()

        def evict_l2():
            flush.fill_(1)
            flush_sink.copy_(flush.view(torch.int64).sum())

        def timed_step():
            evict_l2()
            graph.replay()
            stream.synchronize()
            return ev[0].elapsed_time(ev[2]), ev[1].elapsed_time(ev[2])

        for _ in range(max(3, args.warmup)):
            timed_step()
        visible = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
        sampler = ClockSampler(visible[local_rank] if len(visible) > local_rank and visible[local_rank]
                               else str(local_rank))
        sampler.start()
        time.sleep(0.3)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        step_ms, att_ms = [], []
        for _ in range(args.steps):
            a, b = timed_step()
            step_ms.append(a)
            att_ms.append(b)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        t1 = time.time()
        sampler.stop()
        assert pk.check_status(stream) == 0

        host_out = torch.empty(dp.out.shape, dtype=dp.out.dtype).pin_memory()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h2d = packed.nbytes
        d2h = host_out.numel() * host_out.element_size()
        e2e_graph = torch.cuda.CUDAGraph()  # inputs in, the step, output out: one replay per step
        with torch.cuda.graph(e2e_graph, stream=stream):
            packed.upload()
            step()
            host_out.copy_(dp.out, non_blocking=True)
        stream.synchronize()
        e2e_ms = []
        e2e_warm = max(20, args.warmup)  # untimed: the first replays of a new graph with host copies run slow
        for i in range(e2e_warm + min(args.steps, 200)):
            evict_l2()
            e0.record()
            e2e_graph.replay()
            e1.record()
            stream.synchronize()
            if i >= e2e_warm:
                e2e_ms.append(e0.elapsed_time(e1))

    step_t, att_t, e2e_t = slowest_rank([statistics.mean(step_ms), statistics.mean(att_ms),
                                         statistics.mean(e2e_ms)], dist, dev)
    clocks = sampler.summary(t0, t1)
    del graph, e2e_graph
    if dist:
        dist.destroy_process_group()
    if rank != 0:
        return
    flops = w.flops()
    peak, peak_sust, kind = tensor_peak()
    achieved = flops / (att_t * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC,
        "value": round(world * flops / (step_t * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_t, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded numpy PCG64; no dataset)",
        "config": {
            "workload": w.name, "num_seqs": w.num_seqs, "num_heads": w.num_heads,
            "head_size": w.head_size, "block_size": w.block_size, "kv_dtype": "f16",
            "total_q": T, "context_lens": [int(x) for x in w.context_lens],
            "chunk_lens": [int(x) for x in w.chunk_lens], "flops_per_step": flops,
            "parallelism": f"replicas x{world} (independent batches, no collective)",
            "l2": "before every timed step a 512 MiB buffer is written then read (L2 is 126 MB)",
            "step": "CUDA graph: prefill_slot_mapping, kv_cache_write, paged_prefill",
        },
        "tokens_per_s": round(world * T / (step_t * 1e-3), 1),
        "prefill_ms": round(att_t, 5),
        "roofline": {
            "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_kind": f"{kind} dense bf16 GEMM, burst (fp16 runs at the same nominal rate); "
                         f"sustained {peak_sust}",
            "traffic": recorded_traffic(w.name, "prefill_dram_traffic.json", PREFILL_SOURCES) if tc else None,
            "kernel": "paged_prefill_tc_kernel" if tc else "paged_prefill_kernel (mma.sync)",
            "algorithmic_flops_per_launch": flops,
            "io_bytes_per_launch": w.io_bytes(),
        },
        "e2e": {"value": round(world * flops / (e2e_t * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_t, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "one CUDA graph per step: pinned host inputs (one packed buffer) -> one copy to the "
                        "device -> the step's launches -> output to pinned host"},
        "gpu_launches": (2 + n_write) * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)


_PREFILL_POOLS: dict = {}


def cpu_baseline_prefill(w, seconds: float, seed: int = 0):
    """The oracle, single-threaded, on a seeded sample of (row, head) pairs of
    the prefill workload (at least one; the pools and the chunk's cache write
    are built once, outside the timed region); TFLOP/s of the sampled pairs."""
    import oracle
    if w.name not in _PREFILL_POOLS:
        kc, vc = w.pool_host()
        slots = oracle.prefill_slot_mapping(w.query_start, w.block_tables, w.context_lens, w.block_size)
        oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
        _PREFILL_POOLS.clear()
        _PREFILL_POOLS[w.name] = (kc, vc)
    kc, vc = _PREFILL_POOLS[w.name]
    rng = np.random.default_rng(seed)
    pos = w.positions()
    done, elapsed, n = 0, 0.0, 0
    while elapsed < seconds and n < 100000:
        r = int(rng.integers(0, w.total_q))
        h = int(rng.integers(0, w.num_heads))
        t = time.perf_counter()
        oracle.paged_prefill(w.query, w.query_start, kc, vc, w.block_tables, w.context_lens, w.scale,
                             row_head=np.array([[r, h]], np.int32))
        elapsed += time.perf_counter() - t
        done += 4 * w.head_size * (int(pos[r]) + 1)
        n += 1
    return {"value": round(done / elapsed / 1e12, 8), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} random (row, head) pairs of {w.name}: {elapsed:.1f} s, single-thread fp64"}


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: rank 0 only, same metric and unit.
    The whole run is bounded by --cpu-seconds of oracle time spread over the
    steps (each step at least one sequence, or one (row, head) pair for a
    prefill), with the host pools built once."""
    if rank != 0:
        return
    if args.prefill:
        run_reference_prefill(args, world)
        return
    w = W.named(args.workload or int(args.workloads.split(",")[0]))
    per_step = args.cpu_seconds / max(1, args.steps + args.warmup)
    state = OracleState(w)
    vals, cores = [], 1
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(w, per_step, state, start=i, threads=0)
        cores = r["cores"]
        if i >= args.warmup:
            vals.append(r["value"])
    v = statistics.mean(vals)
    kv = w.kv_bytes()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(kv / (v * 1e9) * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64; no dataset)",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_heads": w.num_heads,
                   "head_size": w.head_size, "block_size": w.block_size, "kv_dtype": w.kv_dtype},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {per_step:.3f} s (at least one call) of whole-sequence "
                                   f"oracle steps, fp64, (sequence, head) pairs over {cores} OpenMP threads"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_prefill(args, world):
    w = W.prefill_named(args.prefill)
    per_step = args.cpu_seconds / max(1, args.steps + args.warmup)
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline_prefill(w, per_step, seed=i)
        if i >= args.warmup:
            vals.append(r["value"])
    v = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": PREFILL_METRIC, "value": round(v, 8), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(w.flops() / (v * 1e12) * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64; no dataset)",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "num_heads": w.num_heads,
                   "head_size": w.head_size, "block_size": w.block_size, "kv_dtype": "f16"},
        "cpu_baseline": {"value": round(v, 8), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: {per_step:.3f} s (at least one (row, head) pair) of "
                                   "random (row, head) pairs, single-thread fp64"},
        "e2e": {"value": round(v, 8), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", type=int, default=0, choices=[0, 1, 2, 3, 4, 5],
                    help="time one decode workload only (default: the --workloads list)")
    ap.add_argument("--workloads", default=DEFAULT_WORKLOADS,
                    help="decode workloads timed in one run; the first is the headline")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="batch size of the decode workloads (default: each workload's own); a smaller "
                         "batch of the same recipe keeps a profiler capture small")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-shared-prefix", action="store_true",
                    help="decode a shared-prefix workload without the prefix kernel")
    ap.add_argument("--unfused", action="store_true",
                    help="slot mapping, cache write and decode as three launches")
    ap.add_argument("--launch", default="",
                    help="decode launch shape partition_size,heads_per_cta,warps_per_head,stages")
    ap.add_argument("--prefill", type=int, default=0, choices=[0, 1, 2, 3],
                    help="time a paged prefill workload (1 tiny, 2 long prompts, 3 chunked) instead")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE {world}; using WORLD_SIZE", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.prefill:
        run_prefill(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
