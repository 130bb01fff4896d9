"""Benchmark of the MLA attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the workload's whole hot path through the C ABI
(attention kernel, split-KV combine, and for the sparse workload the mask
compaction first) over one batch of synthetic inputs resident in HBM. Between
timed steps L2 is flushed by writing a 256 MiB buffer and then reading another
(outside the timed events), so a step starts from a cold L2 with no dirty lines
of the flush left to write back. Each step is timed with CUDA events on the
launching stream; with N ranks every rank runs its own replica of the batch (weak
scaling, no collective on the data path) and the time is the max over ranks.
`--gpus N` without a launcher starts the N ranks itself (torch.distributed.run on
127.0.0.1, one process per GPU).

Printed (rank 0): one JSON line. Its headline (`value`, `roofline`, `e2e`,
`cpu_baseline`) is the V3 batched decode workload, timed over exactly K steps:
whole-job KV-cache GB/s, us/call, the roofline of the dominant kernel, an
end-to-end figure through the same C ABI with host buffers (pinned host -> device
copies of the inputs and device -> host copy of the output inside the timed
region), the oracle's CPU throughput on a bounded sample, SM clocks sampled during
the timed passes, and the launch count. `configs` holds the same measurement for
every other workload of the benchmark definition (tiny decode, V2-Lite decode,
prefill chunk, sparse q8_0 decode), each in the same process.

Kernel times: the step time comes from a pass with only the two events around each
step (events between the launches of a step would serialise them); per-kernel
times come from a second pass of the same steps with the library's per-launch
events. A roofline takes the dominant kernel's time from the second pass, capped at
the step time of the first (a kernel cannot take longer than the step holding it;
the passes may run at different clocks), and for a step of one kernel it is the
step time itself. The median SM clock of each pass is recorded.

--impl reference times the fp64 CPU oracle as the reference arm (there is no
runnable reference implementation of this path), on a bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_flash_attention_attn_b200 import workloads as W  # noqa: E402

METRIC = ("MLA attention µs/call & KV-cache GB/s (DK576/DV512), "
          "% of HBM/tensor roofline")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
DEFAULT_WORKLOAD = "v3_batched_decode"


# ----------------------------------------------------------------------------- accounting
def algorithmic(w, kept_cells=None, wuv=False, mask_gather=False):
    if isinstance(w, W.HeadsWorkload):
        return algorithmic_heads(w)
    return algorithmic_mla(w, kept_cells, wuv, mask_gather)


def algorithmic_mla(w, kept_cells=None, wuv=False, mask_gather=False):
    """Algorithmic bytes and flops of one step, split partials excluded.

    bytes = cache rows attended x row bytes + Q + mask cells read + output;
    flops = 2 * n_head * (576 + 512) per (query row, attended key). With the fused
    value up-projection (wuv) the output is 128 wide and the step also reads the
    weights (n_head x 512 x 128 f16) and does 2 x 512 x 128 flops per query row.
    A sparse step reads its mask row and writes then reads the index list; with the
    mask gather there is no list: the mask rows are read once."""
    dk = w.q.shape[-1]  # 576, or 512 for the DK = DV = 512 head shape
    row_bytes = 2 * dk if w.kv_type == W.KV_F16 else W.Q8_ROW_BYTES
    if kept_cells is None:
        keep = ~np.isneginf(w.mask) if w.mask is not None else None
        kept_cells = []
        for b in range(w.n_seq):
            L = int(w.kv_len[b])
            if keep is None:
                kept_cells.append([L] * w.n_q)
            else:
                kept_cells.append([int(keep[b, t, :L].sum()) for t in range(w.n_q)])
    rows_attended = 0  # distinct cache rows read per sequence
    pairs = 0          # (query token, attended key) pairs
    mask_bytes = 0
    for b in range(w.n_seq):
        rows_attended += max(kept_cells[b])
        pairs += sum(kept_cells[b])
        mask_bytes += w.n_q * int(w.kv_len[b]) * 2 if w.mask is not None else 0
    if w.sparse and not mask_gather:
        mask_bytes = w.n_seq * w.n_kv * 2 + rows_attended * 4 * 2  # mask read + idx write/read
    q_bytes = w.q.size * 2
    out_bytes = w.n_seq * w.n_q * w.n_head * (128 if wuv else 512) * 4
    kv_bytes = rows_attended * row_bytes
    flops = 2.0 * w.n_head * (dk + 512) * pairs
    if wuv:
        out_bytes += w.n_head * 512 * 128 * 2
        flops += 2.0 * 512 * 128 * w.n_seq * w.n_q * w.n_head
    return {"kv_bytes": kv_bytes, "bytes": kv_bytes + q_bytes + mask_bytes + out_bytes,
            "flops": flops}


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture
# of this same bench command (profiles/ gives the command and the figures), keyed by a
# hash of the kernel sources the capture ran. Any change to those sources makes the
# figure stale, and the roofline then reports traffic as null.
MEASURED_TRAFFIC = {
    "v3_batched_decode": {"source": "a3f8efe4f21d1aa1", "bytes": 164443392},
    "prefill_chunk": {"source": "a3f8efe4f21d1aa1", "bytes": 203976704},
    "sparse_q8_decode": {"source": "a3f8efe4f21d1aa1", "bytes": 19130880},
}


def kernel_source_hash():
    import hashlib
    src = os.path.join(ROOT, "mla_flash_attention_attn_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(src)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(f.encode())
            with open(os.path.join(src, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def workload_name(args):
    """The workload as the step runs it: the cache geometry plus the fused options."""
    return (args.workload + ("+wuv" if args.wuv else "")
            + (f"+split_kv{args.split_kv}" if getattr(args, "split_kv", 0) > 1 else "")
            + ("+no_kv_len" if getattr(args, "no_kv_len", False) else "")
            + ("+mask_gather" if args.mask_gather else "")
            + ("+dk512" if args.head_dim == 512 else ""))  # heads_* names carry their shape


HEADS_WORKLOADS = {"heads_prefill": W.heads_prefill, "heads_decode": W.heads_decode}


def algorithmic_heads(w):
    """Algorithmic bytes and flops of one step of the DK = 192 / DV = 128 head shape:
    bytes = K and V rows attended (every KV head: 384 + 256 bytes per cell) + Q + mask
    cells read + output; flops = 2 * n_head * (192 + 128) per (query token, kept key)."""
    keep = ~np.isneginf(w.mask) if w.mask is not None else None
    rows_attended = pairs = mask_bytes = 0
    for b in range(w.n_seq):
        L = int(w.kv_len[b])
        kept = [L] * w.n_q if keep is None else [int(keep[b, t, :L].sum()) for t in range(w.n_q)]
        rows_attended += max(kept)
        pairs += sum(kept)
        mask_bytes += w.n_q * L * 2 if w.mask is not None else 0
    kv_bytes = rows_attended * w.n_kv_head * (192 + 128) * 2
    out_bytes = w.n_seq * w.n_q * w.n_head * 128 * 4
    return {"kv_bytes": kv_bytes, "bytes": kv_bytes + w.q.size * 2 + mask_bytes + out_bytes,
            "flops": 2.0 * w.n_head * (192 + 128) * pairs}


def make_workload(args):
    """The named workload; with --head-dim 512 the same one with the 64 RoPE columns
    of q and of the cache dropped (the DK = DV = 512 head shape, f16 cache); the heads_*
    workloads are the DK = 192 / DV = 128 head shape."""
    if args.workload in HEADS_WORKLOADS:
        return HEADS_WORKLOADS[args.workload]()
    w = W.make(args.workload)
    if args.head_dim == 512:
        if w.kv_type != W.KV_F16:
            raise SystemExit("--head-dim 512 takes an f16-cache workload")
        w.q = np.ascontiguousarray(w.q[..., :512])
        w.kcache = np.ascontiguousarray(w.kcache[..., :512])
    return w


def measured_traffic(workload):
    m = MEASURED_TRAFFIC.get(workload)
    if m is None or m["source"] != kernel_source_hash():
        return None
    return m["bytes"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed passes run.
    Each sample is tagged with the pass that was running (set_label), so every pass can
    report its own median clock."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.002):
        self.index = index
        self.period = period
        self.samples = []  # (label, MHz)
        self.reasons = set()
        self.max_mhz = None
        self.label = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False

    def set_label(self, label):
        """Samples from now on belong to `label` (None: not a timed pass; not kept)."""
        self.label = label

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            label = self.label
            if label is not None:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    self.samples.append((label, mhz))
                    for bit, name in self.REASONS.items():
                        if mask & bit and bit != 0x1:
                            self.reasons.add(name)
                except Exception:  # noqa: BLE001
                    pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def median(self, prefix=None):
        xs = [m for lab, m in self.samples if prefix is None or lab.startswith(prefix)]
        return float(statistics.median(xs)) if xs else None

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": self.median(), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- GPU arm
class Step:
    """Device-resident inputs and the hot path of one workload."""

    def __init__(self, w, torch, binding, wuv=False, mask_gather=False, lengths=True):
        self.w = w
        self.torch = torch
        self.b = binding
        dev = torch.device("cuda")
        self.q = torch.from_numpy(w.q).to(dev)
        self.k = torch.from_numpy(w.kcache).to(dev)
        self.mask = torch.from_numpy(w.mask).to(dev) if w.mask is not None else None
        # with the fused value up-projection the step's result is the 128-wide projection
        self.wv = torch.from_numpy(W.wv_random(n_head=w.n_head)).to(dev) if wuv else None
        self.out = torch.empty(w.q.shape[:3] + ((128 if wuv else 512),), dtype=torch.float32,
                               device=dev)
        # without lengths the mask alone says which cells (and tiles) are kept
        self.kv_len = [int(x) for x in w.kv_len] if lengths else None
        self.idx = self.cnt = None
        if w.sparse and not mask_gather:
            # the step starts from the mask row: compaction, then attention over the kept rows
            self.idx = torch.empty((w.n_seq, w.n_kv), dtype=torch.int32, device=dev)
            self.cnt = torch.zeros((w.n_seq,), dtype=torch.int32, device=dev)
            self.cws = torch.zeros(binding.mla_compact_workspace_size(w.n_seq, w.n_kv),
                                   dtype=torch.uint8, device=dev)
        self.args, self._keep = binding.make_args(
            self.q, self.k, w.kv_type, self.mask, None if wuv else self.out, w.scale,
            kv_len=self.kv_len, idx=self.idx, idx_count=self.cnt, wv=self.wv,
            out_proj=self.out if wuv else None, mask_gather=mask_gather)
        need = binding.mla_fa_workspace_size(self.args)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        self.ws_used = need > 0

    def inputs(self):
        """(device tensor, host array) of every input a step reads."""
        ins = [(self.q, self.w.q), (self.k, self.w.kcache)]
        return ins + ([(self.mask, self.w.mask)] if self.mask is not None else [])

    def run(self, stream=None):
        if self.idx is not None:
            self.b.mla_compact_mask_ex(self.mask[:, 0, :], self.idx, self.cnt, self.cws, stream)
        self.b.mla_fa_forward_ex(self.args, self.ws if self.ws_used else None, stream)


class HeadsStep:
    """Device-resident inputs and the hot path of the DK = 192 / DV = 128 head shape."""

    def __init__(self, w, torch, binding):
        self.w = w
        self.b = binding
        dev = torch.device("cuda")
        self.q = torch.from_numpy(w.q).to(dev)
        self.k = torch.from_numpy(w.k).to(dev)
        self.v = torch.from_numpy(w.v).to(dev)
        self.mask = torch.from_numpy(w.mask).to(dev) if w.mask is not None else None
        self.out = torch.empty(w.q.shape[:3] + (128,), dtype=torch.float32, device=dev)
        self.args, self._keep = binding.make_heads_args(self.q, self.k, self.v, self.mask,
                                                        self.out, w.scale,
                                                        [int(x) for x in w.kv_len])
        need = binding.mla_fa_workspace_size(self.args)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        self.ws_used = need > 0

    def inputs(self):
        """(device tensor, host array) of every input a step reads."""
        ins = [(self.q, self.w.q), (self.k, self.w.k), (self.v, self.w.v)]
        return ins + ([(self.mask, self.w.mask)] if self.mask is not None else [])

    def run(self, stream=None):
        self.b.mla_fa_forward_ex(self.args, self.ws if self.ws_used else None, stream)


class SplitKVStep:
    """The ranks' calls of a split-KV decode (the cache split into `parts` ranges), made
    one after another on one GPU: each attends over its range with each row's lse,
    writing O and lse into its slice of the packed buffer the all-gather would fill,
    and the merge (mla_fa_combine_strided) combines them. The all-gather itself is not
    part of this step (one GPU)."""

    def __init__(self, w, torch, binding, parts):
        from mla_flash_attention_attn_b200 import split_kv

        self.w = w
        self.b = binding
        dev = torch.device("cuda")
        self.q = torch.from_numpy(w.q).to(dev)
        self.rows = w.n_seq * w.n_q * w.n_head
        self.packed = torch.empty((parts, binding.packed_width(self.rows)), dtype=torch.float32,
                                  device=dev)
        self.out = torch.empty((self.rows, 512), dtype=torch.float32, device=dev)
        self.shards = []
        for r, (lo, hi) in enumerate(split_kv.shard_bounds(w.n_kv, parts)):
            k = torch.from_numpy(np.ascontiguousarray(w.kcache[:, lo:hi])).to(dev)
            m = torch.from_numpy(np.ascontiguousarray(w.mask[:, :, lo:hi])).to(dev)
            o = self.packed[r, : self.rows * 512].view(w.n_seq, w.n_q, w.n_head, 512)
            lse = self.packed[r, self.rows * 512:].view(w.n_seq, w.n_q, w.n_head)
            args, keep = binding.make_args(self.q, k, w.kv_type, m, o, w.scale,
                                           kv_len=split_kv.shard_lengths(w.kv_len, lo, hi),
                                           out_lse=lse)
            need = binding.mla_fa_workspace_size(args)
            ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
            self.shards.append((args, keep, ws, k, m))

    def inputs(self):
        return [(self.q, self.w.q)]

    def run(self, stream=None):
        for args, _, ws, _, _ in self.shards:
            self.b.mla_fa_forward_ex(args, ws, stream)
        self.b.combine_packed(self.packed, self.rows, out=self.out, stream=stream)


def config_of(w, name, world):
    """The workload's description as it appears in both arms' JSON lines."""
    heads = isinstance(w, W.HeadsWorkload)
    extra = {"n_kv_head": w.n_kv_head, "v_head_dim": 128} if heads else {}
    return {"workload": name, "n_seq": w.n_seq, "n_q": w.n_q, "n_head": w.n_head,
            "n_kv": w.n_kv, "head_dim": int(w.q.shape[-1]), **extra,
            "kv_type": "q8_0" if (not heads and w.kv_type) else "f16",
            "kv_len": [int(x) for x in w.kv_len][:16],
            "parallelism": f"replicas x{world}",
            "l2": "flushed between timed steps (256 MiB written, then 256 MiB read; outside "
                  "the events)"}


def roofline_of(kacc, kernel_ms, peaks, peak_kind, traffic):
    """Roofline of the dominant kernel: algorithmic bytes (or flops) per launch over its
    time, against the measured peak of the binding roof."""
    tensor_bound = kacc["flops"] / kacc["bytes"] > peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        achieved = kacc["flops"] / (kernel_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    else:
        achieved = kacc["bytes"] / (kernel_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["traffic"] = traffic
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else \
        "fallback (profiling recipe)"
    return roof


def measure(args, w, name, torch, binding, clocks, world, steps, headline=False):
    """Time `steps` steps of workload w (after args.warmup untimed ones), then the same
    steps again with per-kernel events. Returns the measurement and the Step."""
    acc = algorithmic(w, wuv=args.wuv, mask_gather=args.mask_gather)
    if isinstance(w, W.HeadsWorkload):
        step = HeadsStep(w, torch, binding)
    elif getattr(args, "split_kv", 0) > 1:
        step = SplitKVStep(w, torch, binding, args.split_kv)
    else:
        step = Step(w, torch, binding, wuv=args.wuv, mask_gather=args.mask_gather,
                    lengths=not getattr(args, "no_kv_len", False))
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def l2_flush():
        # write a buffer larger than L2, then read another one: the dirty lines of the
        # write are written back here, outside the timed region, so that every timed step
        # starts from an L2 that holds none of its data and owes no write-back
        flush.fill_(1.0)
        flush_rd.sum()

    for _ in range(args.warmup):
        l2_flush()
        step.run()
    torch.cuda.synchronize()
    if binding.mla_get_device_status() != 0:
        raise RuntimeError(f"{name}: device status after warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    # pass 1: nothing but the two events around each step (per-kernel events between the
    # launches would serialise them: the combine is a programmatic dependent of the
    # forward kernel)
    clocks.set_label(f"{name}/step")
    for i in range(steps):
        l2_flush()
        starts[i].record(stream)
        step.run()
        stops[i].record(stream)
    torch.cuda.synchronize()
    # pass 2: per-kernel device times with the library's per-launch events
    clocks.set_label(f"{name}/kernels")
    binding.mla_profile_begin()
    for i in range(steps):
        l2_flush()
        step.run()
    torch.cuda.synchronize()
    prof = binding.mla_profile_end()
    clocks.set_label(None)
    barrier(world)
    torch.cuda.synchronize()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, stops)]
    ms_per_step = max_over_ranks(sum(step_ms), world) / steps
    status = binding.mla_get_device_status()
    if status != 0:
        raise RuntimeError(f"{name}: device status {binding.mla_status_string(status)}")
    del flush, flush_rd

    peaks, peak_kind = load_peaks()
    dom = max((k for k in prof if k.startswith("mla_fwd")), key=lambda k: prof[k][1])
    launches, dom_ms = prof.get(dom, (0, 0.0))
    dom_prof_ms = dom_ms / max(launches, 1)
    per_step_launches = sum(v[0] for v in prof.values()) / steps
    # the kernel's time in a step: its own events (all its launches of the step: the
    # emulated split-KV step launches it once per cache range), capped at the step that
    # holds it; a step of one kernel is that kernel
    dom_step_ms = dom_ms / steps
    kernel_ms = ms_per_step if per_step_launches <= 1 else min(dom_step_ms, ms_per_step)
    # the roofline is the dominant (attention) kernel's: its own algorithmic bytes and
    # flops, which leave out the W_UV weights and projection of a --wuv step (the
    # combine does those)
    kacc = algorithmic(w, mask_gather=args.mask_gather) if args.wuv else acc
    roof = roofline_of(kacc, kernel_ms, peaks, peak_kind, measured_traffic(
        name + ("+wuv" if args.wuv else "") + ("+mask_gather" if args.mask_gather else "")
        + ("+dk512" if args.head_dim == 512 else "")))
    roof["kernel"] = dom
    roof["kernel_us"] = round(kernel_ms * 1e3, 3)
    roof["kernel_launches_per_step"] = round(launches / steps, 3)
    roof["kernel_avg_us_events"] = round(dom_prof_ms * 1e3, 3)
    roof["algorithmic_bytes_per_launch"] = kacc["bytes"]
    roof["algorithmic_flops_per_launch"] = kacc["flops"]
    res = {
        "us_per_call": round(ms_per_step * 1e3, 3),
        "ms_per_step": round(ms_per_step, 6),
        "kv_gbs": round(acc["kv_bytes"] * world / (ms_per_step * 1e-3) / 1e9, 2),
        "tokens_per_s": round(w.n_seq * w.n_q * world / (ms_per_step * 1e-3), 1),
        "steps": steps,
        "roofline": roof,
        "kernels": {k: {"launches": v[0], "avg_us": round(1e3 * v[1] / max(v[0], 1), 3)}
                    for k, v in prof.items()},
        "gpu_launches": int(sum(v[0] for v in prof.values())),
        "clocks_mhz": {"step_pass": clocks.median(f"{name}/step"),
                       "kernel_pass": clocks.median(f"{name}/kernels")},
    }
    return res, acc, step


def gpu_arm(args, rank, world):
    import torch

    from mla_flash_attention_attn_b200 import binding

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    binding.load()
    others = [] if (args.only or args.wuv or args.mask_gather or args.head_dim != 576 or
                    args.no_kv_len or args.split_kv > 1) else \
        [n for n in W.WORKLOAD_ORDER if n != args.workload]
    with ClockSampler(torch.cuda.current_device()) as clocks:
        w = make_workload(args)
        head, acc, step = measure(args, w, args.workload, torch, binding, clocks, world,
                                  args.steps, headline=True)
        if args.traffic is not None:
            head["roofline"]["traffic"] = args.traffic
        # ---- end to end through the same C ABI with host buffers
        e2e = None
        if not args.no_e2e:
            e2e = e2e_measure(args, w, step, torch, binding, acc, world)
        del step
        torch.cuda.empty_cache()
        cfgs = {}
        for name in others:
            wo = W.make(name)
            # a short step gets the requested step count; a long one (the prefill chunk)
            # enough steps for the clock sampler to see it under load
            n = args.steps if name != "prefill_chunk" else max(args.steps, args.prefill_steps)
            r, acc_o, st = measure(args, wo, name, torch, binding, clocks, world, n)
            r["config"] = config_of(wo, name, world)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                r["cpu_baseline"] = oracle_throughput(wo, acc_o, args.cpu_budget_configs_s)
            cfgs[name] = r
            del st
            torch.cuda.empty_cache()

    result = {
        "metric": METRIC,
        "value": head["kv_gbs"],
        "unit": "GB/s",
        "us_per_call": head["us_per_call"],
        "tokens_per_s": head["tokens_per_s"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic (seeded PCG64; DeepSeek-V3/V2-Lite cache geometry, random values)",
        "config": config_of(w, workload_name(args), world),
        "roofline": head["roofline"],
        "e2e": e2e,
        "gpu_launches": head["gpu_launches"],
        "kernels": head["kernels"],
        "kernel_times": "per-launch CUDA events in a second pass of the same steps, capped at "
                        "the step time",
        "clocks": clocks.summary(),
        "clocks_mhz_by_pass": head["clocks_mhz"],
        "configs": cfgs,
        "impl": "ours",
    }
    return result, w


def e2e_measure(args, w, step, torch, binding, acc, world):
    """Same hot path, with the inputs copied from pinned host memory each step and the
    output copied back, all inside the CUDA-event timed region."""
    pairs = [(dev_t, torch.from_numpy(host).pin_memory()) for dev_t, host in step.inputs()]
    hout = torch.empty(step.out.shape, dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()
    n = max(1, min(args.steps, args.e2e_steps))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for i in range(n + 1):
        s, e = ev[i - 1] if i else (None, None)
        if s is not None:
            s.record(stream)
        for dev_t, host_t in pairs:
            dev_t.copy_(host_t, non_blocking=True)
        step.run()
        hout.copy_(step.out, non_blocking=True)
        if e is not None:
            e.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in ev), world) / n
    h2d = sum(h.numel() * h.element_size() for _, h in pairs)
    return {"value": round(acc["kv_bytes"] * world / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "us_per_call": round(ms * 1e3, 2), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(hout.numel() * 4), "steps": n}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_throughput(w, acc, budget_s):
    """Time the oracle on a bounded sample of query rows; scale to the metric's unit."""
    import oracle

    rows_total = w.n_seq * w.n_q * w.n_head
    # rows per second estimate from one small probe, then a sample sized to the budget
    t0 = time.perf_counter()
    _oracle_rows(oracle, w, 1)
    per_row = max(time.perf_counter() - t0, 1e-4)
    n = int(min(rows_total, max(oracle.max_threads(), budget_s / per_row * oracle.max_threads())))
    t0 = time.perf_counter()
    _oracle_rows(oracle, w, n)
    dt = time.perf_counter() - t0
    full_s = dt * rows_total / n
    return {"value": round(acc["kv_bytes"] / full_s / 1e9, 6), "unit": "GB/s",
            "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n} of {rows_total} query rows, {dt:.1f} s on the host; "
                      f"time scaled by rows to the full step",
            "us_per_call_equiv": round(full_s * 1e6, 1)}


def _oracle_rows(oracle, w, n):
    """Compute n query rows spread over the sequences (sparse: over the kept indices;
    the 192 / 128 head shape: whole tokens, every head)."""
    if isinstance(w, W.HeadsWorkload):
        toks = max(1, n // w.n_head)
        per_seq = max(1, toks // w.n_seq)
        for b in range(w.n_seq):
            L = int(w.kv_len[b])
            for t in np.linspace(0, w.n_q - 1, min(per_seq, w.n_q)).astype(int):
                oracle.attention_heads(w.q[b, t:t + 1], w.k[b, :L], w.v[b, :L],
                                       w.mask[b, t:t + 1, :L] if w.mask is not None else None,
                                       w.scale)
        return
    per_seq = max(1, n // w.n_seq)
    done = 0
    for b in range(w.n_seq):
        if done >= n:
            break
        k = min(per_seq, n - done, w.n_q * w.n_head)
        rows = np.linspace(0, w.n_q * w.n_head - 1, k).astype(np.int32)
        mask = w.mask[b] if w.mask is not None else None
        idx = None
        if w.sparse:
            idx = oracle.compact(w.mask[b, 0])
        oracle.attention(w.q[b], w.kcache[b], w.kv_type, mask, w.scale, rows=rows, idx=idx)
        done += k


def reference_arm(args, rank, world):
    """The oracle as the reference arm: each step computes a bounded sample of the step's
    rows on the host cores; the per-step time is scaled by rows to the full step."""
    if rank != 0:
        return None
    import oracle

    w = W.make(args.workload)
    acc = algorithmic(w)
    rows_total = w.n_seq * w.n_q * w.n_head
    per_step_budget = max(0.5, args.ref_budget_s / max(1, args.steps + args.warmup))
    t0 = time.perf_counter()
    _oracle_rows(oracle, w, 1)
    per_row = max(time.perf_counter() - t0, 1e-4)
    n = int(min(rows_total, max(1, per_step_budget / per_row * oracle.max_threads())))
    for _ in range(args.warmup):
        _oracle_rows(oracle, w, max(1, n // 8))
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_rows(oracle, w, n)
        times.append((time.perf_counter() - t0) * rows_total / n)
    ms = 1e3 * sum(times) / len(times)
    value = acc["kv_bytes"] / (ms * 1e-3) / 1e9
    cpu = {"value": round(value, 6), "unit": "GB/s", "cores": oracle.max_threads(),
           "kind": "oracle",
           "sample": f"{n} of {rows_total} query rows per step, time scaled by rows"}
    return {
        "metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded PCG64)",
        "config": config_of(w, args.workload, world),
        "impl": "reference", "cpu_baseline": cpu,
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- ranks
def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def init_ranks(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        backend = "nccl" if (torch.cuda.is_available() and args.impl == "ours") else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def free_port():
    import socket

    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def launch_ranks(n, argv):
    """Run this same command as n ranks under torch.distributed.run on 127.0.0.1 (one
    process per GPU) and return its exit status."""
    import subprocess

    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=W.WORKLOAD_ORDER + list(HEADS_WORKLOADS))
    ap.add_argument("--only", action="store_true",
                    help="time the --workload alone (no per-config measurements)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--wuv", action="store_true",
                    help="fuse the value up-projection W_UV (synthetic f16 weights) into the "
                         "step; the result is the 128-wide projection")
    ap.add_argument("--mask-gather", action="store_true",
                    help="masked workloads: sparse attention straight from the mask (the "
                         "compaction fused into the attention kernel, no index list)")
    ap.add_argument("--head-dim", type=int, default=576, choices=[576, 512, 192],
                    help="512: the DK = DV = 512 head shape (the workload without its RoPE "
                         "columns; f16 cache); 192: the DK = 192 / DV = 128 head shape (a K "
                         "and a V per KV head; the heads_prefill workload unless a heads_* "
                         "workload is named)")
    ap.add_argument("--no-kv-len", action="store_true",
                    help="pass no host lengths: the kept tiles come from the mask alone "
                         "(scanned on the device)")
    ap.add_argument("--split-kv", type=int, default=0,
                    help="R >= 2: the calls of a split-KV decode over R cache ranges, made one "
                         "after another on this GPU (R shard forwards with the lse, then the "
                         "merge of the packed parts; the all-gather between GPUs is left out)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--prefill-steps", type=int, default=60,
                    help="least number of timed steps of the prefill chunk in `configs`")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--cpu-budget-configs-s", type=float, default=3.0)
    ap.add_argument("--ref-budget-s", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the dominant kernel, if captured")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.wuv and args.impl == "reference":
        ap.error("--wuv applies to --impl ours (the oracle arm times the attention only)")
    if args.head_dim != 576 and args.impl == "reference":
        ap.error("--head-dim applies to --impl ours")
    if args.mask_gather and args.impl == "reference":
        ap.error("--mask-gather applies to --impl ours (the oracle arm runs the unfused chain)")
    if args.wuv:
        args.no_cpu_baseline = True  # the oracle baseline times the attention only
    if args.split_kv > 1 and (args.impl == "reference" or args.wuv or args.mask_gather or
                              args.head_dim != 576 or args.workload in HEADS_WORKLOADS or
                              args.gpus > 1):
        ap.error("--split-kv emulates the ranks on one GPU, for the MLA decode workloads")
    if args.split_kv > 1:
        args.no_e2e = True  # the emulated ranks' step reads shards no host copy would fill
    if args.head_dim == 192 and args.workload not in HEADS_WORKLOADS:
        args.workload = "heads_prefill"
    if args.workload in HEADS_WORKLOADS:
        if args.impl == "reference":
            ap.error("the reference arm times the MLA workloads")
        if args.wuv or args.mask_gather:
            ap.error("the 192 / 128 head shape takes neither --wuv nor --mask-gather")
        args.head_dim = 192
    if "WORLD_SIZE" not in os.environ:
        if args.gpus > 1:
            # one process per GPU: start the ranks under the launcher
            sys.exit(launch_ranks(args.gpus, argv))
    elif int(os.environ["WORLD_SIZE"]) != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started {os.environ['WORLD_SIZE']} ranks")
    rank, world = init_ranks(args)
    try:
        if args.impl == "reference":
            res = reference_arm(args, rank, world)
        else:
            res, w = gpu_arm(args, rank, world)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = oracle_throughput(w, algorithmic(w), args.cpu_budget_s)
            elif rank == 0:
                res["cpu_baseline"] = None
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
