#!/usr/bin/env python3
"""Benchmark of the paged decode step on B200: tokens/s and KV-cache GB/s.

One step = the whole hot path for one decode step of one layer over a batch:
K1 (pa_reshape_and_cache: each sequence's new K/V into its slot), then K2 (+K3)
(pa_decode: attention over every sequence's paged context, split partitions
merged).  The slot resolution a1 (host allocator) is timed separately and
reported as ``a1_us``.  One new token per sequence per step: tokens/s =
num_seqs / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama7b]
    python bench.py --impl reference ...      # the fp64 CPU oracle on host cores

Under torchrun (N > 1) every rank runs an independent replica of the workload on
its own GPU (the decode path has no exchange step), time is the max over ranks,
and the value is the sum of all ranks' tokens over that time (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention tokens/s and KV-cache HBM GB/s (fraction of ~8 TB/s) on 1 B200"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "paged_decode_llama7b.md")
GQA_PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "paged_decode_gqa70b.md")
# ncu summaries that give roofline.traffic, by workload (+fp8 for the e4m3 cache)
TRAFFIC_SUMMARIES = {"llama7b": PROFILE_SUMMARY, "gqa70b": GQA_PROFILE_SUMMARY,
                     "llama13b": os.path.join(ROOT, "profiles", "paged_decode_llama13b.md"),
                     "llama7b+fp8": os.path.join(ROOT, "profiles", "paged_decode_fp8_llama7b.md"),
                     "gqa70b+fp8": os.path.join(ROOT, "profiles", "paged_decode_fp8_gqa70b.md")}
SHARED_PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "shared_prefix_beam.md")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="llama7b")
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--partition-tokens", type=int, default=0)
    p.add_argument("--num-seqs", type=int, default=None, help="truncate the batch (smaller profiling case)")
    p.add_argument("--kv-dtype", default="native", choices=["native", "fp8"],
                   help="fp8: the cache is stored as E4M3 codes (pa_reshape_and_cache_fp8 / pa_decode_fp8)")
    p.add_argument("--shared-prefix", default="auto", choices=["auto", "off"],
                   help="auto: sequences sharing prompt blocks (the beam workload) run through "
                        "pa_decode_shared_prefix; off: plain pa_decode")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-detail-workloads", action="store_true",
                   help="skip the 13B append loop, gqa70b and beam entries of detail.workloads")
    p.add_argument("--row", default="decode", choices=["decode", "copy_blocks", "swap", "prefill"],
                   help="decode: the hot path (default); copy_blocks: copy-on-write block copies alone; "
                        "swap: swap-out / swap-in of blocks to pinned host memory")
    return p.parse_args()


# ------------------------------------------------------------------ helpers

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity on one rank).

    Every rank of a replica run times its own copy of the workload; the job's time
    is the slowest rank's.
    """
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(world, tokens_per_step, ms_per_step):
    """Whole-job tokens/s: every rank decodes tokens_per_step tokens per step."""
    return world * tokens_per_step / (ms_per_step / 1e3)


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(paths):
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(units_now: int, workload: str, summary=PROFILE_SUMMARY):
    """DRAM bytes per launch of the decode kernels from a committed ncu summary,
    scaled to this launch's (unique) tokens; None when the summary is missing, was
    taken on another workload (bytes per token depend on the head counts), or one
    of the sources the profiled kernels are built from (the summary's `sources`)
    has changed since the counters were taken."""
    try:
        fields = {}
        with open(summary) as f:
            for line in f:
                if line.startswith("- ") and ": " in line:
                    k, v = line[2:].split(": ", 1)
                    fields[k.strip()] = v.strip().strip("`")
        sources = [os.path.join(ROOT, "paged_kv_cache_374_b200", "csrc", n.strip())
                   for n in fields["sources"].split(",")]
        if fields.get("workload") != workload or fields.get("source_sha256_16") != source_digest(sources):
            return None
        per_token = float(fields["dram_bytes_per_launch"]) / float(fields["tokens_per_launch"])
        return per_token * units_now
    except Exception:
        return None


class ClockSampler:
    """SM clock and clock-event reasons during a timed region.  Read through NVML by
    a thread every 0.2 ms from entry to exit (the timed regions here are a few
    milliseconds long, so this puts dozens of samples under load); where NVML is not
    usable, nvidia-smi every 200 ms around the region instead.  Only reads: no
    setting of the GPU is changed."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits reported by name
    NVML_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.lines = []
        self.proc = None
        self.nvml = None
        self.samples = []  # (sm MHz, reason bits) from NVML
        self.max_mhz = None
        self.stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id) if self.gpu_id.startswith("GPU-")
                 else pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_id)))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.nvml = (pynvml, h)
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _poll(self):
        pynvml, h = self.nvml
        while not self.stop.is_set():
            try:
                self.samples.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                     int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
            except Exception:
                return
            time.sleep(0.0002)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.nvml:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:
                pass
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        if self.samples:
            sm = [c for c, _ in self.samples]
            reasons = sorted({name for _, bits in self.samples for b, name in self.NVML_BITS.items() if bits & b})
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(sm), "source": "nvml, during the timed region"}
        rows = []
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, fl in enumerate(flags) if fl.lower() == "active"})
        sm = [r[0] for r in rows]
        loaded = [x for x in sm if x >= 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi, around the timed region"}


def gpu_uuid(torch, device):
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else f"GPU-{u}"
    except Exception:
        return str(device.index or 0)


# --------------------------------------------------------------- workload

FP8_INV_SCALE = 32.0  # fp8 caches: stored value = code / 32 (N(0,1) values use codes up to ~150)


def build_step(name, device, partition_tokens, num_seqs=None, kv_dtype="native", shared=False):
    """Tables from the library's allocator, one step's slots via a1, tensors on
    the device.  Returns a dict of everything the timed loop needs."""
    import torch
    from paged_kv_cache_374_b200 import binding as pa
    from paged_kv_cache_374_b200 import workloads as wk

    wl = wk.make_workload(name, num_seqs=num_seqs)
    spec = wl.spec
    bs = spec.block_size
    alloc = pa.BlockAllocator(wl.num_blocks, wl.pool_order)
    s = spec.num_seqs
    stored = (wl.context_lens - 1).astype(np.int32)
    tables = np.full((s, wl.max_blocks_per_seq), -1, dtype=np.int32)
    have = np.zeros(s, dtype=np.int64)
    if spec.prefix_tokens:
        npre = pa.pa_num_required_blocks(spec.prefix_tokens, bs)
        prefix = alloc.alloc_n(npre)
        for i in range(s):
            tables[i, :npre] = alloc.fork(prefix)
        have[:] = npre
    for i in range(s):
        n = pa.pa_num_required_blocks(int(stored[i]), bs) - int(have[i])
        tables[i, have[i]:have[i] + n] = alloc.alloc_n(n)
    lens = stored.copy()
    t0 = time.perf_counter()
    slots = alloc.append_slots(tables, lens, bs)
    a1_us = (time.perf_counter() - t0) * 1e6
    t = wk.make_tensors(wl, device=device)
    if kv_dtype == "fp8":
        import torch
        for key in ("k_cache", "v_cache"):
            t[key] = (t[key].float() * FP8_INV_SCALE).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    ws_bytes = pa.pa_decode_workspace_size(s, spec.num_heads, spec.num_kv_heads, spec.head_dim, bs,
                                           wl.max_blocks_per_seq, partition_tokens)
    ptok = partition_tokens or pa.pa_decode_partition_tokens(s, spec.num_heads, spec.num_kv_heads, spec.head_dim, bs,
                                                             wl.max_blocks_per_seq)
    groups = None
    if shared and kv_dtype == "native":
        groups = pa.pa_find_shared_prefixes(tables, lens, bs, ptok)
        if groups.num_groups == 0:
            groups = None
    d = dict(
        wl=wl, spec=spec, alloc=alloc, tables_h=tables, lens_h=lens, slots_h=slots, a1_us=a1_us,
        tables=torch.from_numpy(tables).to(device), lens=torch.from_numpy(lens).to(device),
        slots=torch.from_numpy(slots).to(device), out=torch.empty_like(t["q"]),
        workspace=torch.zeros(max(ws_bytes, 1), dtype=torch.uint8, device=device), ws_bytes=ws_bytes,
        partition_tokens=partition_tokens, ptok=ptok, groups=groups,
        group_dev=groups.to(device) if groups is not None else None, **t)
    return d


def algorithmic_bytes(st, lens=None):
    """Bytes K2+K3 must move per step: every sequence's K and V rows once (shared
    prefix blocks once), q in and out back, the table entries read, the lengths,
    and the partials written by K2 and read by K3.  ``lens``: the step's context
    lengths (default: the step the workload was built for)."""
    spec = st["spec"]
    lens = (st["lens_h"] if lens is None else lens).astype(np.int64)
    e = 2                                  # q and out elements
    ec = st["k_cache"].element_size()      # cache elements (1 for fp8 codes)
    hk, d, h, s, bs = spec.num_kv_heads, spec.head_dim, spec.num_heads, spec.num_seqs, spec.block_size
    row = 2 * hk * d * ec  # K and V of one token, all kv heads
    if spec.prefix_tokens:
        unique_tokens = spec.prefix_tokens + int(np.sum(lens - spec.prefix_tokens))
    else:
        unique_tokens = int(np.sum(lens))
    logical_tokens = int(np.sum(lens))
    ptok = st["ptok"]
    nparts = np.where(lens > ptok, -(-lens // ptok), 0)
    partials = int(np.sum(nparts)) * h * (d + 2) * 4 * 2
    meta = int(np.sum(-(-lens // bs))) * 4 + 4 * s
    qo = 2 * s * h * d * e
    return {"unique": unique_tokens * row + qo + meta + partials,
            "logical": logical_tokens * row + qo + meta + partials,
            "unique_tokens": unique_tokens, "k1": 2 * s * hk * d * (e + ec) + 8 * s}


def static_config(wl, args, world):
    spec = wl.spec
    lens = wl.context_lens.astype(np.int64)
    kv = int(np.sum(lens)) * 2 * spec.num_kv_heads * spec.head_dim * 2
    return {
        "workload": f"{spec.name}: {spec.description}",
        "num_seqs": spec.num_seqs, "num_heads": spec.num_heads, "num_kv_heads": spec.num_kv_heads,
        "head_dim": spec.head_dim, "block_size": spec.block_size, "seed": spec.seed,
        "mean_context": float(np.mean(lens)),
        "partition_tokens": args.partition_tokens or "auto",
        "l2": "no flush: the paged cache read per step (%.2f GB) is far larger than the 126 MB L2" % (kv / 1e9),
        "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
    }


# --------------------------------------------------------------- native arm

class Ops:
    """K1 and K2+K3 of one built workload, through the binding, on one stream."""

    def __init__(self, st, stream, fp8):
        from paged_kv_cache_374_b200 import binding as pa
        self.pa, self.st, self.stream, self.fp8 = pa, st, stream, fp8
        self.ks = self.vs = 1.0 / FP8_INV_SCALE

    def k1(self, k, v, slots):
        st, pa = self.st, self.pa
        if self.fp8:
            pa.pa_reshape_and_cache_fp8(k, v, slots, st["k_cache"], st["v_cache"], self.ks, self.vs,
                                        stream=self.stream)
        else:
            pa.pa_reshape_and_cache(k, v, slots, st["k_cache"], st["v_cache"], stream=self.stream)

    def k2(self, q, tables, lens, groups=None, out=None):
        st, pa, spec = self.st, self.pa, self.st["spec"]
        g = st["groups"]
        out = st["out"] if out is None else out
        if g is not None:
            start, offs, mem = groups if groups is not None else st["group_dev"]
            pa.pa_decode_shared_prefix(q, st["k_cache"], st["v_cache"], tables, lens, spec.scale, spec.num_kv_heads,
                                       out, start, offs, mem, g.num_groups, g.max_group_size,
                                       g.max_shared_tokens, workspace=st["workspace"],
                                       partition_tokens=st["partition_tokens"], stream=self.stream)
        elif self.fp8:
            pa.pa_decode_fp8(q, st["k_cache"], st["v_cache"], tables, lens, spec.scale, self.ks, self.vs,
                             spec.num_kv_heads, out, workspace=st["workspace"],
                             partition_tokens=st["partition_tokens"], stream=self.stream)
        else:
            pa.pa_decode(q, st["k_cache"], st["v_cache"], tables, lens, spec.scale, spec.num_kv_heads, out,
                         workspace=st["workspace"], partition_tokens=st["partition_tokens"], stream=self.stream)

    @property
    def fused(self):
        """One call per step: pa_decode_step(_fp8), or pa_decode_step_shared_prefix
        with shared-prefix groups."""
        return True

    def step(self, k, v, slots, q, tables, lens, groups=None, out=None):
        if self.fused:
            st = self.st
            out = st["out"] if out is None else out
            g = st["groups"]
            if g is not None:
                start, offs, mem = groups if groups is not None else st["group_dev"]
                self.pa.pa_decode_step_shared_prefix(k, v, slots, q, st["k_cache"], st["v_cache"], tables, lens,
                                                     st["spec"].scale, st["spec"].num_kv_heads, out, start, offs, mem,
                                                     g.num_groups, g.max_group_size, g.max_shared_tokens,
                                                     workspace=st["workspace"],
                                                     partition_tokens=st["partition_tokens"], stream=self.stream)
            elif self.fp8:
                self.pa.pa_decode_step_fp8(k, v, slots, q, st["k_cache"], st["v_cache"], tables, lens,
                                           st["spec"].scale, self.ks, self.vs, st["spec"].num_kv_heads, out,
                                           workspace=st["workspace"], partition_tokens=st["partition_tokens"],
                                           stream=self.stream)
            else:
                self.pa.pa_decode_step(k, v, slots, q, st["k_cache"], st["v_cache"], tables, lens, st["spec"].scale,
                                       st["spec"].num_kv_heads, out, workspace=st["workspace"],
                                       partition_tokens=st["partition_tokens"], stream=self.stream)
        else:
            self.k1(k, v, slots)
            self.k2(q, tables, lens, groups, out)

    def resident_step(self):
        st = self.st
        self.step(st["k"], st["v"], st["slots"], st["q"], st["tables"], st["lens"])

    def launches_per_step(self):
        st = self.st
        nparts_max = -(-int(st["wl"].max_blocks_per_seq * st["spec"].block_size) // st["ptok"])
        return 2 + (1 if nparts_max > 1 else 0) + (1 if st["groups"] is not None else 0)


def _events(torch, n):
    return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]


def time_device_steps(torch, ops, device, steps, warmup, barrier, clocks=True):
    """W untimed steps, then exactly `steps` steps on resident inputs, bracketed by
    a barrier and a synchronize on both sides, with clocks sampled meanwhile.  A
    fused step (one pa_decode_step call) carries no events inside the region: its
    launches run back to back and the region's events give their mean duration.
    Otherwise K2+K3 carry their own events on the launching stream."""
    st, stream = ops.st, ops.stream
    for _ in range(max(3, warmup)):
        ops.resident_step()
    barrier()
    k2_ev = None if ops.fused else _events(torch, steps)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_uuid(torch, device)) if clocks else None
    if sampler:
        sampler.__enter__()
    barrier()
    start.record(stream)
    for i in range(steps):
        if k2_ev is None:
            ops.resident_step()
        else:
            ops.k1(st["k"], st["v"], st["slots"])
            k2_ev[i][0].record(stream)
            ops.k2(st["q"], st["tables"], st["lens"])
            k2_ev[i][1].record(stream)
    stop.record(stream)
    barrier()
    if sampler:
        sampler.__exit__(None, None, None)
    elapsed = start.elapsed_time(stop)
    return {"elapsed_ms": elapsed,
            "k2_ms": statistics.mean(a.elapsed_time(b) for a, b in k2_ev) if k2_ev else None,
            "clocks": sampler.summary() if sampler else None}


def time_alone(torch, ops, barrier, which, n=200):
    """K1 alone or K2+K3 alone (outside any timed region), mean event time per call."""
    st = ops.st
    ev = _events(torch, n)
    for a, b in ev:
        a.record(ops.stream)
        if which == "k1":
            ops.k1(st["k"], st["v"], st["slots"])
        else:
            ops.k2(st["q"], st["tables"], st["lens"])
        b.record(ops.stream)
    barrier()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def time_e2e_repeated(torch, ops, device, steps, barrier, clocks=True):
    """e2e through the binding, two steps in flight: step i+1's inputs go H2D from
    pinned host memory on a copy stream while step i computes, and each step's
    output goes D2H on a third stream.  Every step still copies all of its own
    inputs and reads back its own result inside the timed region."""
    from paged_kv_cache_374_b200 import binding as pa
    st, stream, spec = ops.st, ops.stream, ops.st["spec"]
    nbuf = 2
    names = ("q", "k", "v", "slots", "tables", "lens")
    offs, h2d = {}, 0
    for n in names:                       # one staging buffer: 256-byte aligned fields
        offs[n] = h2d
        h2d += -(-st[n].numel() * st[n].element_size() // 256) * 256
    host_buf = torch.empty(h2d, dtype=torch.uint8).pin_memory()
    for n in names:
        nb = st[n].numel() * st[n].element_size()
        host_buf[offs[n]:offs[n] + nb].copy_(st[n].cpu().contiguous().view(-1).view(torch.uint8))
    dev_buf = [torch.empty(h2d, dtype=torch.uint8, device=device) for _ in range(nbuf)]
    dev_in = [{n: dev_buf[b][offs[n]:offs[n] + st[n].numel() * st[n].element_size()].view(st[n].dtype)
               .view(st[n].shape) for n in names} for b in range(nbuf)]
    out_d = [torch.empty_like(st["out"]) for _ in range(nbuf)]
    out_h = [torch.empty(st["out"].shape, dtype=st["out"].dtype).pin_memory() for _ in range(nbuf)]
    d2h = out_h[0].numel() * out_h[0].element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]     # set b's inputs are on the device
    ev_used = [torch.cuda.Event() for _ in range(nbuf)]   # K1/K2 of set b are done (inputs read, out_d[b] written)
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]    # out_d[b] is back on the host

    grp_dev = grp_h = None
    n1 = spec.num_seqs + 1
    if st["groups"] is not None:  # the grouping is redone from the host tables every step: one int32 buffer of
        grp_dev = [torch.empty(3 * n1, dtype=torch.int32, device=device) for _ in range(nbuf)]  # seq_start |
        grp_h = [torch.zeros(3 * n1, dtype=torch.int32).pin_memory() for _ in range(nbuf)]     # offsets | members
        h2d += 4 * 3 * n1

    def e2e_step(i):
        b = i % nbuf
        groups = None
        if grp_dev is not None:
            g = pa.pa_find_shared_prefixes(st["tables_h"], st["lens_h"], spec.block_size, st["ptok"])
            ev_in[b].synchronize()                     # the copy that last read grp_h[b] is done
            hv = grp_h[b].numpy()
            groups = []
            for part, arr in enumerate((g.seq_start, g.group_offsets, g.group_members)):
                hv[part * n1:part * n1 + len(arr)] = arr
                groups.append(grp_dev[b][part * n1:part * n1 + len(arr)])
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(ev_used[b])          # the step two back has finished with set b
            dev_buf[b].copy_(host_buf, non_blocking=True)
            if grp_dev is not None:
                grp_dev[b].copy_(grp_h[b], non_blocking=True)
            ev_in[b].record(h2d_stream)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])                   # out_d[b] of the step two back is on the host
        ops.step(dev_in[b]["k"], dev_in[b]["v"], dev_in[b]["slots"], dev_in[b]["q"], dev_in[b]["tables"],
                 dev_in[b]["lens"], groups, out=out_d[b])
        ev_used[b].record(stream)
        d2h_stream.wait_event(ev_used[b])
        with torch.cuda.stream(d2h_stream):
            out_h[b].copy_(out_d[b], non_blocking=True)
            ev_out[b].record(d2h_stream)

    for i in range(3):
        e2e_step(i)
    barrier()
    sampler = ClockSampler(gpu_uuid(torch, device)) if clocks else None
    if sampler:
        sampler.__enter__()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)
    for i in range(steps):
        e2e_step(i)
    stream.wait_event(ev_out[(steps - 1) % nbuf])  # the last read-back (the D2H stream runs in order)
    e1.record(stream)
    barrier()
    if sampler:
        sampler.__exit__(None, None, None)
    # the pipelined steps compute what the device-timed ones did (same inputs, same cache slots)
    matches = bool(torch.equal(out_h[(steps - 1) % nbuf], st["out"].cpu()))
    return {"e2e_ms": e0.elapsed_time(e1) / steps, "h2d": h2d, "d2h": d2h, "matches": matches,
            "clocks": sampler.summary() if sampler else None}


def roofline_traffic(st, workload, fp8, ab):
    key = workload + ("+fp8" if fp8 else "")
    if st["groups"] is not None:
        return profiled_traffic(ab["unique_tokens"], workload, SHARED_PROFILE_SUMMARY)
    return profiled_traffic(ab["unique_tokens"], key, TRAFFIC_SUMMARIES.get(key, PROFILE_SUMMARY))


def roofline_leg(ops, ab, t, steps):
    """(bytes, ms) of the kernel sequence the roofline is taken on: the whole fused
    step (K1 + K2 + K3: the write's bytes too, and the region's mean per step), or
    K2+K3 alone with their per-step events."""
    if ops.fused:
        return ab["unique"] + ab["k1"], t["elapsed_ms"] / steps
    return ab["unique"], t["k2_ms"]


def roofline_kernel(ops):
    if ops.fused and ops.st["groups"] is not None:
        return ("reshape_and_cache_kernel + shared-prefix kernel + paged_decode_kernel + paged_decode_merge_kernel "
                "(one pa_decode_step_shared_prefix call: the prefix kernel a programmatic dependent of K1)")
    if ops.fused:
        call = "pa_decode_step_fp8" if ops.fp8 else "pa_decode_step"
        return ("reshape_and_cache_kernel + paged_decode_kernel + paged_decode_merge_kernel (one %s call: K2 a "
                "programmatic dependent of K1)" % call)
    return "paged_decode_kernel + paged_decode_merge_kernel (timed together: one pa_decode call)"


def steps_for(torch, ops, target_s, lo=200, hi=40000):
    """Steps that fill about target_s of device time (from a 20-step probe)."""
    st, stream = ops.st, ops.stream
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(20):
        ops.resident_step()
    b.record(stream)
    torch.cuda.synchronize()
    per = a.elapsed_time(b) / 20 / 1e3
    return int(min(hi, max(lo, target_s / max(per, 1e-7))))


def measure_repeated(torch, name, device, args, target_s=0.8, shared=True):
    """One detail entry: the workload's step repeated on resident inputs for about
    target_s, its K2+K3 against the roofline, and an e2e over as many steps."""
    st = build_step(name, device, args.partition_tokens, shared=shared)
    ops = Ops(st, torch.cuda.current_stream(device), False)
    barrier = lambda: torch.cuda.synchronize(device)
    for _ in range(5):
        ops.resident_step()
    steps = steps_for(torch, ops, target_s)
    t = time_device_steps(torch, ops, device, steps, 5, barrier)
    e = time_e2e_repeated(torch, ops, device, steps, barrier)
    k2k3_ms = time_alone(torch, ops, barrier, "k2k3")
    ab = algorithmic_bytes(st)
    peak, _ = measured_hbm_peak()
    nbytes, ms = roofline_leg(ops, ab, t, steps)
    gbs = nbytes / (ms / 1e3) / 1e9
    spec = st["spec"]
    res = {"workload": f"{spec.name}: {spec.description}", "steps": steps,
           "tokens_per_s": round(spec.num_seqs / (t["elapsed_ms"] / steps / 1e3), 1),
           "ms_per_step": round(t["elapsed_ms"] / steps, 5), "k2k3_us_alone": round(k2k3_ms * 1e3, 2),
           "roofline_kernel": roofline_kernel(ops), "bytes_per_step": nbytes, "kv_gbs": round(gbs, 1),
           "frac": round(gbs / peak, 4), "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
           "traffic": roofline_traffic(st, name, False, ab), "clocks": t["clocks"],
           "e2e_tokens_per_s": round(spec.num_seqs / (e["e2e_ms"] / 1e3), 1), "e2e_output_matches": e["matches"],
           "e2e_clocks": e["clocks"]}
    if st["groups"] is not None:
        res["path"] = "pa_decode_shared_prefix: %d group(s), %d shared tokens" % (st["groups"].num_groups,
                                                                                  st["groups"].max_shared_tokens)
    del st, ops
    torch.cuda.empty_cache()
    return res


def measure_append_loop(torch, name, device, args, target_s=0.8):
    """The workload as its configuration states it: `spec.steps` consecutive decode
    steps, each appending one token per sequence.  Every step runs a1 on the host
    (pa_append_slots: a new block at each block boundary), K1 into the step's slots
    and K2+K3 over the grown tables and lengths.

    Device leg: the steps' tables, lengths and slots are resolved by a1 up front and
    resident in HBM; each pass runs the spec.steps steps in order (K2+K3 timed with
    events, each step against its own algorithmic bytes); passes repeat for about
    target_s.  e2e leg: each pass starts from the same allocator state (rebuilt
    outside the timed region) and every step runs a1 on the host, copies that
    step's inputs (q, k, v, the grown tables, lengths and slots) H2D from pinned
    memory, runs K1 + K2+K3 and reads the output back, two steps in flight."""
    from paged_kv_cache_374_b200 import binding as pa
    st = build_step(name, device, args.partition_tokens, shared=False)
    spec, wl = st["spec"], st["wl"]
    bs, S, nsteps = spec.block_size, spec.num_seqs, spec.steps
    stream = torch.cuda.current_stream(device)
    ops = Ops(st, stream, False)

    def fresh_state():
        """Allocator and host tables/lengths before step 1 (every pass starts here)."""
        alloc = pa.BlockAllocator(wl.num_blocks, wl.pool_order)
        tables = np.full((S, wl.max_blocks_per_seq), -1, dtype=np.int32)
        stored = (wl.context_lens - 1).astype(np.int32)
        for i in range(S):
            n = pa.pa_num_required_blocks(int(stored[i]), bs)
            tables[i, :n] = alloc.alloc_n(n)
        return alloc, tables, stored.copy()

    alloc, tables, lens = fresh_state()
    per_step, a1_us = [], []
    for _ in range(nsteps):
        t0 = time.perf_counter()
        slots = alloc.append_slots(tables, lens, bs)
        a1_us.append((time.perf_counter() - t0) * 1e6)
        per_step.append((tables.copy(), lens.copy(), slots.copy()))
    new_blocks = int(np.sum(per_step[-1][0] >= 0) - np.sum(per_step[0][0] >= 0))
    dev_steps = [tuple(torch.from_numpy(x).to(device) for x in s) for s in per_step]
    step_bytes = [algorithmic_bytes(st, lens=s[1])["unique"] + (algorithmic_bytes(st)["k1"] if ops.fused else 0)
                  for s in per_step]
    del alloc

    def run_pass(ev=None):
        for i, (tb, ln, sl) in enumerate(dev_steps):
            if ops.fused:                 # events around the one call of the step
                if ev is not None:
                    ev[i][0].record(stream)
                ops.step(st["k"], st["v"], sl, st["q"], tb, ln)
            else:                         # events around K2+K3
                ops.k1(st["k"], st["v"], sl)
                if ev is not None:
                    ev[i][0].record(stream)
                ops.k2(st["q"], tb, ln)
            if ev is not None:
                ev[i][1].record(stream)

    for _ in range(3):
        run_pass()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    run_pass()
    b.record(stream)
    torch.cuda.synchronize(device)
    passes = int(min(400, max(3, target_s / max(a.elapsed_time(b) / 1e3, 1e-6))))
    evs = [_events(torch, nsteps) for _ in range(passes)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_uuid(torch, device))
    sampler.__enter__()
    torch.cuda.synchronize(device)
    start.record(stream)
    for p in range(passes):
        run_pass(evs[p])
    stop.record(stream)
    torch.cuda.synchronize(device)
    sampler.__exit__(None, None, None)
    total_ms = start.elapsed_time(stop)
    k2_ms = np.array([[e0.elapsed_time(e1) for e0, e1 in ev] for ev in evs]).mean(axis=0)  # per step
    peak, _ = measured_hbm_peak()
    gbs_steps = [by / (ms / 1e3) / 1e9 for by, ms in zip(step_bytes, k2_ms)]
    gbs = sum(step_bytes) / (float(np.sum(k2_ms)) / 1e3) / 1e9
    ref_out = st["out"].clone()   # output of the last step of the last pass

    # e2e: a1 on the host, the step's inputs H2D, K1 + K2+K3, the output D2H
    nbuf = 2
    sizes = {"q": st["q"], "k": st["k"], "v": st["v"]}
    mb = wl.max_blocks_per_seq
    fixed = {n: t.numel() * t.element_size() for n, t in sizes.items()}
    layout, off = {}, 0
    for n, nb in list(fixed.items()) + [("tables", S * mb * 4), ("lens", S * 4), ("slots", S * 8)]:
        layout[n] = (off, nb)
        off += -(-nb // 256) * 256
    h2d = off
    host = [torch.empty(h2d, dtype=torch.uint8).pin_memory() for _ in range(nbuf)]
    for hb in host:
        for n, t in sizes.items():
            o, nb = layout[n]
            hb[o:o + nb].copy_(t.cpu().contiguous().view(-1).view(torch.uint8))
    dev_buf = [torch.empty(h2d, dtype=torch.uint8, device=device) for _ in range(nbuf)]

    def view(b, n, dtype, shape):
        o, nb = layout[n]
        return dev_buf[b][o:o + nb].view(dtype).view(shape)
    dev_in = [{"q": view(b, "q", st["q"].dtype, st["q"].shape), "k": view(b, "k", st["k"].dtype, st["k"].shape),
               "v": view(b, "v", st["v"].dtype, st["v"].shape), "tables": view(b, "tables", torch.int32, (S, mb)),
               "lens": view(b, "lens", torch.int32, (S,)), "slots": view(b, "slots", torch.int64, (S,))}
              for b in range(nbuf)]
    out_d = [torch.empty_like(st["out"]) for _ in range(nbuf)]
    out_h = [torch.empty(st["out"].shape, dtype=st["out"].dtype).pin_memory() for _ in range(nbuf)]
    d2h = out_h[0].numel() * out_h[0].element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_used = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e_pass(alloc, tables, lens):
        for i in range(nsteps):
            b = i % nbuf
            slots = alloc.append_slots(tables, lens, bs)       # a1 on the host
            ev_in[b].synchronize()                            # the copy that last read host[b] is done
            hv = host[b].numpy()
            for n, arr in (("tables", tables), ("lens", lens), ("slots", slots)):
                o, nb = layout[n]
                hv[o:o + nb] = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
            with torch.cuda.stream(h2d_stream):
                h2d_stream.wait_event(ev_used[b])
                dev_buf[b].copy_(host[b], non_blocking=True)
                ev_in[b].record(h2d_stream)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])
            ops.step(dev_in[b]["k"], dev_in[b]["v"], dev_in[b]["slots"], dev_in[b]["q"], dev_in[b]["tables"],
                     dev_in[b]["lens"], out=out_d[b])
            ev_used[b].record(stream)
            d2h_stream.wait_event(ev_used[b])
            with torch.cuda.stream(d2h_stream):
                out_h[b].copy_(out_d[b], non_blocking=True)
                ev_out[b].record(d2h_stream)

    e2e_ms, matches = 0.0, True
    e_sampler = ClockSampler(gpu_uuid(torch, device))
    e_sampler.__enter__()
    for p in range(passes + 1):                  # the first pass is a warm-up
        state = fresh_state()                    # outside the timed region
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d_stream.wait_event(e0)
        e2e_pass(*state)
        stream.wait_event(ev_out[(nsteps - 1) % nbuf])
        e1.record(stream)
        torch.cuda.synchronize(device)
        if p:
            e2e_ms += e0.elapsed_time(e1)
        # every pass re-derives the device leg's tables and slots step for step
        matches &= bool(np.array_equal(state[1], per_step[-1][0]) and np.array_equal(state[2], per_step[-1][1]))
    e_sampler.__exit__(None, None, None)
    matches &= bool(torch.equal(out_h[(nsteps - 1) % nbuf], ref_out.cpu()))
    res = {"workload": f"{spec.name}: {spec.description}", "steps_per_pass": nsteps, "passes": passes,
           "new_blocks_per_pass": new_blocks,
           "tokens_per_s": round(S * nsteps * passes / (total_ms / 1e3), 1),
           "ms_per_step": round(total_ms / (nsteps * passes), 5),
           "roofline_kernel": roofline_kernel(ops), "roofline_us_per_step": round(float(np.mean(k2_ms)) * 1e3, 2),
           "roofline_us_first_last": [round(float(k2_ms[0]) * 1e3, 2), round(float(k2_ms[-1]) * 1e3, 2)],
           "bytes_per_pass": int(sum(step_bytes)), "kv_gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
           "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
           # DRAM bytes per step from the ncu summary, scaled to the loop's mean context tokens per step
           "traffic": profiled_traffic(float(np.mean([np.sum(ps[1]) for ps in per_step])), spec.name,
                                       TRAFFIC_SUMMARIES.get(spec.name, PROFILE_SUMMARY)),
           "kv_gbs_min_max_step": [round(min(gbs_steps), 1), round(max(gbs_steps), 1)],
           "a1_us_mean": round(float(np.mean(a1_us)), 1), "clocks": sampler.summary(),
           "e2e_tokens_per_s": round(S * nsteps * passes / (e2e_ms / 1e3), 1),
           "e2e_h2d_bytes_per_step": h2d, "e2e_d2h_bytes_per_step": d2h, "e2e_output_matches": matches,
           "e2e_clocks": e_sampler.summary()}
    del st, ops, dev_steps
    torch.cuda.empty_cache()
    return res


def run_native(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    st = build_step(args.workload, device, args.partition_tokens, args.num_seqs, args.kv_dtype,
                    shared=args.shared_prefix == "auto")
    fp8 = args.kv_dtype == "fp8"
    spec = st["spec"]
    stream = torch.cuda.current_stream(device)
    ops = Ops(st, stream, fp8)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)

    t = time_device_steps(torch, ops, device, args.steps, args.warmup, barrier, clocks=not args.no_clocks)
    (elapsed_ms,) = max_over_ranks([t["elapsed_ms"]], dist if world > 1 else None, device)
    k1_ms = time_alone(torch, ops, barrier, "k1")
    k2_ms = t["k2_ms"] if t["k2_ms"] is not None else time_alone(torch, ops, barrier, "k2k3")
    e = time_e2e_repeated(torch, ops, device, args.steps, barrier, clocks=not args.no_clocks)
    (e2e_ms,) = max_over_ranks([e["e2e_ms"]], dist if world > 1 else None, device)

    ab = algorithmic_bytes(st)
    ms_per_step = elapsed_ms / args.steps
    tokens_per_step = spec.num_seqs
    value = job_throughput(world, tokens_per_step, ms_per_step)
    peak, peak_kind = measured_hbm_peak()
    roof_bytes, roof_ms = roofline_leg(ops, ab, dict(t, elapsed_ms=elapsed_ms), args.steps)
    achieved = roof_bytes / (roof_ms / 1e3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": spec.dtype + ("+e4m3 cache" if fp8 else ""),
        "data": "synthetic",
        "config": dict(static_config(st["wl"], args, world), **({"kv_cache": "fp8 e4m3, scale 1/32"} if fp8 else {}),
                       **({"shared_prefix": "pa_decode_shared_prefix: %d group(s), %d shared tokens" % (
                           st["groups"].num_groups, st["groups"].max_shared_tokens)} if st["groups"] is not None
                          else {})),
        "detail": {
            "kv_gbs": round(achieved, 1), "frac_of_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "kv_bytes_per_step": ab["unique"], "logical_kv_bytes_per_step": ab["logical"],
            "k1_bytes_per_step": ab["k1"], "roofline_bytes_per_step": roof_bytes,
            "k1_us_alone": round(k1_ms * 1e3, 2), "k2k3_us" + ("_alone" if ops.fused else ""): round(k2_ms * 1e3, 2),
            "k2k3_gbs_alone" if ops.fused else "k2k3_gbs": round(ab["unique"] / (k2_ms / 1e3) / 1e9, 1),
            "a1_us": round(st["a1_us"], 1),
            "e2e_ms_per_step": round(e2e_ms, 4), "e2e_output_matches": e["matches"],
        },
        "roofline": {
            "kernel": roofline_kernel(ops),
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "peak_kind": (peak_kind + ": a device copy, which reads and writes; this kernel almost only reads, "
                          "so it can pass 1.0 (frac_of_nominal is against 8 TB/s)"),
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "traffic": roofline_traffic(st, args.workload, fp8, ab),
        },
        "e2e": {"value": round(job_throughput(world, tokens_per_step, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"], "clocks": e["clocks"]},
        "gpu_launches": args.steps * ops.launches_per_step(),
        "clocks": t["clocks"],
    }
    del ops, st
    torch.cuda.empty_cache()
    if (world == 1 and not args.no_detail_workloads and not fp8 and args.num_seqs is None
            and args.workload == "llama7b"):
        # the other configurations, each with its own clocks: 13B as its 32-step
        # append loop, GQA long context, and the beam batch's shared prefix
        result["detail"]["workloads"] = {
            "llama13b": measure_append_loop(torch, "llama13b", device, args),
            "gqa70b": measure_repeated(torch, "gqa70b", device, args),
            "beam": measure_repeated(torch, "beam", device, args, shared=args.shared_prefix == "auto"),
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.workload, budget_s=12.0)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ------------------------------------------------------------ oracle timing

def oracle_sample(name, max_pairs=None):
    """Host inputs for the first sequences of a workload (same lengths as the full
    workload's first sequences), drawn on the CPU."""
    import torch
    from paged_kv_cache_374_b200 import workloads as wk
    from oracle.block_pool import BlockPoolModel
    import oracle as oracle_pkg

    full = wk.make_workload(name)
    n = min(full.spec.num_seqs, 4)
    wl = wk.make_workload(name, num_seqs=n)
    spec = wl.spec
    bs = spec.block_size
    pool = BlockPoolModel(wl.num_blocks, wl.pool_order)
    tables = np.full((n, wl.max_blocks_per_seq), -1, dtype=np.int32)
    for i in range(n):
        k = -(-int(wl.context_lens[i]) // bs)
        tables[i, :k] = pool.allocate_n(k)
    t = wk.make_tensors(wl, device="cpu")
    to_bits = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    q, kc, vc = to_bits(t["q"]), to_bits(t["k_cache"]), to_bits(t["v_cache"])
    o = oracle_pkg.get()
    dt = 0 if spec.dtype == "f16" else 1
    lens = wl.context_lens.copy()
    slots = o.slot_mapping(tables, lens, bs)
    kn, vn = to_bits(t["k"]), to_bits(t["v"])
    return dict(o=o, q=q, kc=kc, vc=vc, tables=tables, lens=lens, slots=slots, k=kn, v=vn, spec=spec, dt=dt)


def time_oracle_pairs(smp, pairs, nthreads):
    o = smp["o"]
    t0 = time.perf_counter()
    o.reshape_and_cache(smp["k"], smp["v"], smp["slots"], smp["kc"], smp["vc"])
    o.decode(smp["q"], smp["kc"], smp["vc"], smp["tables"], smp["lens"], smp["spec"].scale, smp["dt"],
             pairs=pairs, nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_baseline(name, budget_s=12.0):
    """The oracle as it stands on this host's cores, on a bounded sample: every
    (sequence, head) pair of the workload's first sequences, K1 + fp64 decode,
    repeated until about `budget_s` of wall time has passed."""
    smp = oracle_sample(name)
    spec = smp["spec"]
    nthreads = os.cpu_count() or 1
    pairs = np.array([(s, h) for s in range(len(smp["lens"])) for h in range(spec.num_heads)], dtype=np.int32)
    reps, total = 0, 0.0
    while total < budget_s:
        total += time_oracle_pairs(smp, pairs, nthreads)
        reps += 1
    tokens = reps * len(smp["lens"])
    return {"value": round(tokens / total, 3), "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"all {spec.num_heads} heads of the first {len(smp['lens'])} sequences of {name} "
                      f"(mean context {float(np.mean(smp['lens'])):.0f}), K1 + fp64 decode, repeated {reps} "
                      f"times in {total:.1f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    smp = oracle_sample(args.workload)
    spec = smp["spec"]
    nthreads = os.cpu_count() or 1
    all_pairs = np.array([(s, h) for s in range(len(smp["lens"])) for h in range(spec.num_heads)], dtype=np.int32)
    probe = all_pairs[:nthreads]
    per_pair = time_oracle_pairs(smp, probe, nthreads) / len(probe) * nthreads
    # size each step so that warmup + steps take about two minutes in all
    per_step_s = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(len(all_pairs), max(1, per_step_s * nthreads / max(per_pair, 1e-9))))
    pairs = all_pairs[:n]
    for _ in range(args.warmup):
        time_oracle_pairs(smp, pairs, nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time_oracle_pairs(smp, pairs, nthreads)
    total = time.perf_counter() - t0
    tokens = args.steps * n / spec.num_heads
    value = tokens / total
    sample = (f"each step: {n} (sequence, head) pairs of the first {len(smp['lens'])} sequences of "
              f"{args.workload}, K1 + fp64 decode")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": static_config(__import__("paged_kv_cache_374_b200.workloads", fromlist=["x"]).make_workload(
            args.workload), args, world),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_copy_blocks(args):
    """Copy-on-write block copies: 512 (src, dst) pairs of the beam workload's blocks
    (block size 64, 32 kv heads, head_dim 128, fp16: 512 KiB per block per cache),
    i.e. 512 MiB read + 512 MiB written per call, timed with CUDA events."""
    import torch
    from paged_kv_cache_374_b200 import binding as pa
    nb, bs, hk, d, n = 1536, 64, 32, 128, 512
    kc = torch.empty(nb, bs, hk, d, dtype=torch.float16, device="cuda").normal_()
    vc = torch.empty_like(kc).normal_()
    g = torch.Generator().manual_seed(5)
    perm = torch.randperm(nb, generator=g)
    pairs = torch.stack([perm[:n], perm[n:2 * n]], dim=1).to(torch.int32).cuda()
    for _ in range(max(3, args.warmup)):
        pa.pa_copy_blocks(kc, vc, pairs)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = min(args.steps, 200)
    e0.record()
    for _ in range(steps):
        pa.pa_copy_blocks(kc, vc, pairs)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    moved = 2 * 2 * n * bs * hk * d * 2
    peak, kind = measured_hbm_peak()
    gbs = moved / (ms / 1e3) / 1e9
    print(json.dumps({"row": "copy_blocks", "metric": "copy-on-write block copy GB/s (read + write)",
                      "value": round(gbs, 1), "unit": "GB/s", "ms_per_call": round(ms, 4), "pairs": n,
                      "bytes_per_call": moved, "frac_of_copy_peak": round(gbs / peak, 4), "peak_kind": kind,
                      "steps": steps}), flush=True)


def run_swap(args):
    """Swap-out (device -> pinned host) and swap-in (host -> device) of 256 blocks of
    the 7B layer geometry (block size 16, 32 kv heads, head_dim 128, fp16: 128 KiB
    per block per cache, 64 MiB per call), timed with CUDA events."""
    import torch
    from paged_kv_cache_374_b200 import binding as pa
    nd, nh, bs, hk, d, n = 1024, 512, 16, 32, 128, 256
    kc = torch.empty(nd, bs, hk, d, dtype=torch.float16, device="cuda").normal_()
    vc = torch.empty_like(kc).normal_()
    kh = torch.zeros(nh, bs, hk, d, dtype=torch.float16).pin_memory()
    vh = torch.zeros_like(kh).pin_memory()
    g = torch.Generator().manual_seed(6)
    pairs = torch.stack([torch.randperm(nd, generator=g)[:n], torch.randperm(nh, generator=g)[:n]], 1)
    out_pairs = pairs.to(torch.int32).cuda()
    in_pairs = pairs.flip(1).contiguous().to(torch.int32).cuda()
    moved = 2 * n * bs * hk * d * 2
    res = {}
    for name, fn in (("swap_out", lambda: pa.pa_swap_blocks(kc, vc, kh, vh, out_pairs)),
                     ("swap_in", lambda: pa.pa_swap_blocks(kh, vh, kc, vc, in_pairs))):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = min(args.steps, 50)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        res[name] = {"GB/s": round(moved / (ms / 1e3) / 1e9, 2), "ms_per_call": round(ms, 4)}
    print(json.dumps({"row": "swap", "metric": "swap-out / swap-in GB/s over the host link",
                      "bytes_per_call": moved, "blocks_per_call": n, **res}), flush=True)


def run_prefill(args):
    """Paged prefill at the 7B layer shape (32 heads, head_dim 128, block size 16,
    fp16): (a) 8 whole 2048-token prompts, (b) 8 chunks of 512 tokens after 3584
    cached ones.  Attention FLOPs = 4 * d * H * (attended tokens summed over rows)."""
    import torch
    from paged_kv_cache_374_b200 import binding as pa
    h = hk = 32
    d, bs = 128, 16
    peak = 1713.1
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
    except Exception:
        pass
    res = {}
    for name, prior, chunk in (("prompt_2048", 0, 2048), ("chunk_512_after_3584", 3584, 512)):
        s = 8
        L = prior + chunk
        nblk = L // bs
        nb = s * nblk + 8
        g = torch.Generator(device="cuda").manual_seed(7)
        kc = torch.randn(nb, bs, hk, d, generator=g, device="cuda").to(torch.float16)
        vc = torch.randn(nb, bs, hk, d, generator=g, device="cuda").to(torch.float16)
        perm = torch.randperm(nb, generator=torch.Generator().manual_seed(8))[: s * nblk]
        tables = perm.view(s, nblk).to(torch.int32).cuda()
        lens = torch.full((s,), L, dtype=torch.int32, device="cuda")
        qs = (torch.arange(s + 1, dtype=torch.int32) * chunk).cuda()
        q = torch.randn(s * chunk, h, d, generator=g, device="cuda").to(torch.float16)
        out = torch.empty_like(q)
        call = lambda: pa.pa_prefill(q, kc, vc, tables, lens, qs, 1 / math.sqrt(d), hk, out, chunk)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = min(args.steps, 50)
        e0.record()
        for _ in range(steps):
            call()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        attended = s * sum(prior + i + 1 for i in range(chunk))
        flops = 4 * d * h * attended
        tf = flops / (ms / 1e3) / 1e12
        res[name] = {"TFLOP/s": round(tf, 1), "ms_per_call": round(ms, 4), "tokens_per_s": round(s * chunk / ms * 1e3),
                     "frac_of_bf16_peak": round(tf / peak, 4)}
    print(json.dumps({"row": "prefill", "metric": "paged prefill attention TFLOP/s (7B layer shape, fp16)",
                      "peak_tflops": peak, **res}), flush=True)


def main():
    args = parse()
    if args.row == "prefill":
        run_prefill(args)
        return
    if args.row == "copy_blocks":
        run_copy_blocks(args)
        return
    if args.row == "swap":
        run_swap(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
