#!/usr/bin/env python
"""Throughput of the LTX-2 joint audio-video block attention on B200.

One step = the whole attention set of one DiT block (video self, audio self with
the key-padding mask, v2a, a2v) over one batch of synthetic bf16 N(0,1) inputs,
run back to back on one stream through the C ABI (libltxattn.so).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on a sample
    python bench.py --workload qk_prologue   # the QK-norm + rotary prologue alone (GB/s)
    python bench.py --workload na3d_decoder  # 3-D neighbourhood attention, decoder-size grid

Prints one JSON line (rank 0).  ``value`` is the whole-job TFLOP/s (algorithmic
FLOPs of all ranks / max-over-ranks device time); the timed region holds exactly
K steps between barriers and device synchronisations, timed with CUDA events on
the launching stream.  Multi-GPU runs are independent replicas (the attention of
one block has no exchange step), hence weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s and µs/call per config; % of B200 dense-BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per launch of the dominant kernel from an ncu capture, keyed by
# the hash of the sources that make up that kernel; reported as null once they change.
KERNEL_SOURCES = {
    "video_self": ("joint_audio_video_flash_b200/csrc/attn_fwd_pair.cuh",
                   "joint_audio_video_flash_b200/csrc/attn_fwd_pp.cuh",
                   "joint_audio_video_flash_b200/csrc/attn_fwd.cuh",
                   "joint_audio_video_flash_b200/csrc/sm100_ptx.cuh"),
    "na3d_decoder": ("joint_audio_video_flash_b200/csrc/na3d_fwd.cuh",
                     "joint_audio_video_flash_b200/csrc/attn_fwd.cuh",
                     "joint_audio_video_flash_b200/csrc/sm100_ptx.cuh"),
    "qk_prologue": ("joint_audio_video_flash_b200/csrc/qk_prologue.cuh",
                    "joint_audio_video_flash_b200/csrc/sm100_ptx.cuh"),
}
TRAFFIC = {
    "video_self": {"src": "7c8cf86aca84f424", "bytes_per_token": (201.467392e6 + 47.959040e6) / 8192,
                   "note": "ncu_small capture (B1 8192 tokens), scaled linearly by tokens"},
    "qk_prologue": {"src": "75b060c4d34193c3", "bytes": 511.267584e6 + 446.194176e6,
                    "note": "full launch, B2 x 15360 x 32 x 128, q and k"},
    "na3d_decoder": {"src": "7986839b9164a1e4", "bytes": 802.395136e6 + 248.623104e6,
                     "note": "full launch, 16x34x60 grid, 3x7x7 window, 32x128"},
}


def kernel_label(c, num_sms: int = 148, grouped: bool = False) -> str:
    """Name of the kernel the library's host dispatch picks for a call (report label only),
    from the library's own plan (``ltxattn_forward_plan``, host only)."""
    from joint_audio_video_flash_b200 import ltxattn
    kt = -(-c.kv_valid_len // 128)
    if grouped and c.head_dim == 64 and kt == 1:
        return "ltx_attn_fwd_a2v (persistent, per-unit K/V, grouped launch)"
    kernel, _ = ltxattn.forward_plan(c.q_len, c.kv_len, c.kv_valid_len, c.batch, c.heads,
                                     c.head_dim, 0, num_sms)
    d = c.head_dim
    return {
        ltxattn.KERNEL_A2V: "ltx_attn_fwd_a2v (persistent, per-unit K/V)",
        ltxattn.KERNEL_SHORT_KV:
            f"ltx_attn_fwd_skv<{d}, {2 if d == 64 else kt}> (persistent, K/V resident)",
        ltxattn.KERNEL_ONE_TILE_DUAL: "ltx_attn_fwd<64, 1 S buffer> (two CTAs per SM)",
        ltxattn.KERNEL_PAIR: "ltx_attn_fwd_pair (CTA pairs, cta_group::2, four query tiles per pair)",
        ltxattn.KERNEL_TWO_TILES: f"ltx_attn_fwd_pp<{d}> (two 128-row query tiles per CTA)",
        ltxattn.KERNEL_ONE_TILE: f"ltx_attn_fwd<{d}>",
    }[kernel]


GROUP_MAX = 4  # calls per launch of the grouped kernel


def launch_items(calls, grouped: bool = True):
    """The step's API calls, as lists of indices into `calls`: the calls the library can
    group (head_dim 64, every valid key in one 128-key tile: a2v and audio self-attention)
    go together through forward_grouped when there are at least two; every other call is one
    forward.  Order: each item where its first call stands."""
    elig = [i for i, c in enumerate(calls) if c.head_dim == 64 and c.kv_valid_len <= 128]
    if not grouped or len(elig) < 2:
        return [[i] for i in range(len(calls))]
    items = []
    for i in range(len(calls)):
        if i not in elig:
            items.append([i])
        elif i == elig[0]:
            items.append(list(elig))
    return items


def group_base(item, member_us):
    """The member of a grouped launch whose own launch takes longest: the base of the split."""
    return max(item, key=lambda i: statistics.median(member_us[("alone", i)]))


def group_share(item, i, member_us, groups):
    """Per-step times of call i's share of its grouped launch, from the interleaved loop: every
    member but the base gets what it adds (the group minus the group without it, step by
    step), the base the rest (the group minus the others' additions), so that the shares add
    up to the group."""
    group = member_us[("group", groups.index(item))]
    added = {x: [g - w for g, w in zip(group, member_us[("without", x)])] for x in item}
    base = group_base(item, member_us)
    if i != base:
        return added[i]
    return [g - sum(added[x][s] for x in item if x != base) for s, g in enumerate(group)]


def item_launches(item, splits):
    """Kernel launches of one launch item (a grouped item: one per GROUP_MAX calls)."""
    if len(item) > 1:
        return -(-len(item) // GROUP_MAX)
    return 1 if splits[item[0]] == 1 else 2


def kernel_source_hash(kernel: str = "video_self") -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_per_launch(kernel: str):
    """ncu DRAM bytes per launch of `kernel`, or None when its sources changed since."""
    tr = TRAFFIC.get(kernel)
    if tr is None or tr["src"] != kernel_source_hash(kernel):
        return None
    return tr.get("bytes")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.file.flush()
        with open(self.file.name) as f:
            lines = [ln.strip() for ln in f if ln.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2]))
                smax.append(float(parts[3]))
            except ValueError:
                continue
            for n, flag in zip(names, parts[6:10]):
                if flag.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


class NvmlClockTrace:
    """The SM clock read through NVML (read-only queries) every `period_s` on a host thread,
    each reading stamped with the host wall clock, so that per-call device times can be put
    beside the clock they ran at (nvidia-smi's 200 ms samples are coarser than one call)."""

    def __init__(self, uuid: str | None, period_s: float = 0.002):
        self.uuid, self.period_s = uuid, period_s
        self.samples = []  # (wall time s, SM MHz)
        self._stop = None
        self._thread = None
        self.max_mhz = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                except Exception:
                    break
                self.samples.append((time.time(), float(mhz)))
                self._stop.wait(self.period_s)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def mhz_during(self, t0: float, t1: float):
        """Mean SM MHz of the readings in [t0, t1], else the reading nearest to the middle."""
        if not self.samples:
            return None
        inside = [m for t, m in self.samples if t0 <= t <= t1]
        if inside:
            return sum(inside) / len(inside)
        mid = 0.5 * (t0 + t1)
        return min(self.samples, key=lambda tm: abs(tm[0] - mid))[1]


def clock_normalised(us, wall, trace):
    """Per-call times at the maximum SM clock: t x (MHz the call ran at / max MHz), with the
    calls binned by clock.  `us` and `wall` ([start, end] host seconds) are per call."""
    if trace is None or not trace.samples or not trace.max_mhz:
        return None
    mhz = [trace.mhz_during(a, b) for a, b in wall]
    norm = [t * f / trace.max_mhz for t, f in zip(us, mhz)]
    bins = {}
    for t, f in zip(us, mhz):
        lo = int(f // 100) * 100
        bins.setdefault(lo, []).append(t)
    return {"us_median_at_max_clock": statistics.median(norm),
            "us_p10_at_max_clock": pct(norm, 0.1), "us_p90_at_max_clock": pct(norm, 0.9),
            "mhz_median": statistics.median(mhz), "mhz_min": min(mhz), "mhz_max_seen": max(mhz),
            "sm_max_mhz": trace.max_mhz, "nvml_samples": len(trace.samples),
            "by_clock": [{"mhz": [lo, lo + 100], "calls": len(v), "us_median": statistics.median(v)}
                         for lo, v in sorted(bins.items())]}


def pct(xs, f):
    s = sorted(xs)
    return s[min(len(s) - 1, max(0, int(f * len(s))))]


def device_uuid(dev):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None


# --------------------------------------------------------------------------- oracle sample
def oracle_sample(calls, fraction: float, seed: int):
    """Time the fp64 oracle on ``fraction`` of every call's query rows (same mix of work)."""
    import torch

    from joint_audio_video_flash_b200 import synth
    from oracle import oracle
    flops = 0.0
    secs = 0.0
    rows_total = 0
    g = torch.Generator().manual_seed(seed)
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                                 q_valid=c.q_valid, kv_valid=c.kv_valid_len)
        n_rows = c.batch * c.q_valid * c.heads
        take = max(1, int(round(n_rows * fraction)))
        # real (unpadded) query rows only, sampled uniformly
        pick = torch.randperm(n_rows, generator=g)[:take]
        h = pick % c.heads
        bi = pick // c.heads
        i = bi % c.q_valid
        b = bi // c.q_valid
        rows = ((b * c.q_len + i) * c.heads + h).numpy()
        t0 = time.perf_counter()
        oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len, rows=rows)
        secs += time.perf_counter() - t0
        flops += 4.0 * take * c.kv_valid_len * c.head_dim
        rows_total += take
    return flops, secs, rows_total


def cpu_baseline(calls, target_s: float, seed: int = 0):
    from oracle import oracle
    oracle.build()
    total = sum(c.flops for c in calls)
    # calibrate on a small sample, then size the measured sample to ~target_s
    f0 = min(1.0, 2e9 / total)
    fl, s, _ = oracle_sample(calls, f0, seed)
    rate = fl / max(s, 1e-9)
    frac = min(1.0, max(f0, target_s * rate / total))
    fl, s, rows = oracle_sample(calls, frac, seed + 1)
    return {"value": fl / s / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{rows} query rows ({frac:.4%} of every call's real rows, same work mix), "
                      f"{fl:.3e} FLOP in {s:.1f} s, fp64, OpenMP over rows"}


# --------------------------------------------------------------------------- per-config table
# Every workload of the attention set (the block768 set is the headline line itself) and the
# next rows' workloads, each timed on its own, with parity against the oracle on sampled rows
# computed after its timed loop.
PER_CONFIG_ATTENTION = ("tiny", "video15360_b1", "audio_stream", "longclip", "text_xattn")
L2_FLUSH_BYTES = 256 << 20  # written before every timed call: L2 (126 MB) holds no input


def parity_stats(got, ref):
    """max-abs, relative L2 and cosine of a GPU result against the fp64 oracle."""
    import numpy as np
    g = np.asarray(got, dtype=np.float64).reshape(ref.shape)
    d = g - ref
    nr = float(np.linalg.norm(ref))
    return {"max_abs": float(np.abs(d).max()),
            "rel_l2": float(np.linalg.norm(d) / nr) if nr else None,
            "cos": float((g * ref).sum() / (np.linalg.norm(g) * nr)) if nr else None,
            "finite": bool(np.all(np.isfinite(g)))}


def attention_parity(c, q, k, v, out_dev, seed):
    """The oracle on every row of a small call, else on sampled rows: 2 seeded rows of every
    (batch, head) and the last 16 real rows of the last head (the ragged tail)."""
    import torch

    from joint_audio_video_flash_b200 import synth
    from oracle import oracle
    n_rows = c.batch * c.q_len * c.heads
    rows = None
    if n_rows * c.kv_valid_len > 4e6:
        r = synth.sample_rows(c.batch, c.q_len, c.heads, 2, seed=seed, full_heads=())
        i = torch.arange(max(0, c.q_valid - 16), c.q_valid)
        tail = ((c.batch - 1) * c.q_len + i) * c.heads + (c.heads - 1)
        rows = torch.unique(torch.cat([r, tail]))
    ref = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len,
                           rows=None if rows is None else rows.numpy())
    got = out_dev.cpu().to(torch.float64)
    got = got.numpy() if rows is None else got.reshape(-1, c.head_dim)[rows].numpy()
    st = parity_stats(got, ref)
    st["rows"] = int(n_rows if rows is None else len(rows))
    return st


def call_roofline(flops, nbytes, us, peaks):
    """TFLOP/s, GB/s and the fraction of the binding measured peak (by arithmetic intensity
    against the ridge of the measured bf16 burst peak and HBM bandwidth)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tfl = flops / (us * 1e-6) / 1e12
    gbs = nbytes / (us * 1e-6) / 1e9
    tensor = flops / nbytes > burst * 1e12 / (hbm * 1e9)
    return {"tflops": tfl, "frac_bf16_peak": tfl / burst, "gbs": gbs, "frac_hbm": gbs / hbm,
            "bound": "tensor" if tensor else "hbm",
            "frac_of_bound": tfl / burst if tensor else gbs / hbm}


def timed_calls(fns, steps, warmup, stream, flush):
    """Runs every fn of `fns` once per step, each bracketed by CUDA events on `stream` after an
    L2 flush (outside the events); returns per-fn lists of µs and of host-wall intervals."""
    import torch
    for _ in range(warmup):
        for f in fns:
            f()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in fns] for _ in range(steps)]
    e0 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    wall0 = time.time()
    e0.record(stream)
    for s in range(steps):
        for i, f in enumerate(fns):
            if flush is not None:
                flush.zero_()
            ev[s][i][0].record(stream)
            f()
            ev[s][i][1].record(stream)
    torch.cuda.synchronize()
    us = [[ev[s][i][0].elapsed_time(ev[s][i][1]) * 1e3 for s in range(steps)]
          for i in range(len(fns))]
    wall = [[(wall0 + e0.elapsed_time(ev[s][i][0]) * 1e-3, wall0 + e0.elapsed_time(ev[s][i][1]) * 1e-3)
             for s in range(steps)] for i in range(len(fns))]
    return us, wall


def dist_stats(us):
    return {"us_median": statistics.median(us), "us_p10": pct(us, 0.1), "us_p90": pct(us, 0.9)}


def measure_attention_config(name, steps, warmup, peaks, dev, stream, flush, trace):
    import torch

    from joint_audio_video_flash_b200 import ltxattn, synth, workloads
    desc, calls = workloads.configs()[name]
    host, ins, outs = [], [], []
    for c in calls:
        trip = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                              q_valid=c.q_valid, kv_valid=c.kv_valid_len)
        host.append(trip)
        ins.append(tuple(t.to(dev) for t in trip))
        outs.append(torch.empty_like(ins[-1][0]))

    def fn(i):
        c = calls[i]
        return lambda: ltxattn.forward(*ins[i], outs[i], kv_valid_len=c.kv_valid_len,
                                       scale=c.scale)

    us, wall = timed_calls([fn(i) for i in range(len(calls))], steps, warmup, stream, flush)
    ltxattn.check()
    out = {"description": desc, "steps": steps, "l2": "flushed before every call", "calls": {}}
    tot_us = 0.0
    for i, c in enumerate(calls):
        d = dist_stats(us[i])
        d.update(call_roofline(c.flops, c.bytes, d["us_median"], peaks))
        d["shape"] = (f"B{c.batch} Lq{c.q_len} Lkv{c.kv_len} valid{c.kv_valid_len} "
                      f"H{c.heads} D{c.head_dim}")
        d["kernel"] = kernel_label(c)
        if c.flops / c.bytes > 1000:  # tensor-bound calls: the clock decides their time
            d["clock"] = clock_normalised(us[i], wall[i], trace)
        d["parity"] = attention_parity(c, *host[i], outs[i], seed=c.seed)
        out["calls"][c.name] = d
        tot_us += d["us_median"]
    flops = sum(c.flops for c in calls)
    out.update({"us_sum_of_medians": tot_us, "tflops": flops / (tot_us * 1e-6) / 1e12})
    del ins, outs
    torch.cuda.empty_cache()
    return out


def measure_prologue_config(steps, warmup, peaks, dev, stream):
    import torch

    from joint_audio_video_flash_b200 import ltxattn, synth
    from oracle import qk_prologue as qp
    b, l, h, d = PROLOGUE_SHAPE
    host = synth.make_qk_prologue_inputs(b, l, h, d, seed=PROLOGUE_SEED)
    dq, dk, dwq, dwk, dcos, dsin = (t.to(dev) for t in host)
    qo, ko = torch.empty_like(dq), torch.empty_like(dk)
    us, _ = timed_calls([lambda: ltxattn.qk_norm_rope(dq, dk, dwq, dwk, dcos, dsin, qo, ko)],
                        steps, warmup, stream, None)
    nbytes = prologue_step_bytes()
    r = dist_stats(us[0])
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    r.update({"gbs": nbytes / (r["us_median"] * 1e-6) / 1e9, "bound": "hbm",
              "l2": "inputs larger than L2", "steps": steps,
              "kernel": "ltx_qk_norm_rope<4, 4, 2>", "description": prologue_config(1)["description"]})
    r["frac_hbm"] = r["gbs"] / hbm
    # parity: the first 256 and the last 64 tokens of every batch element, q and k
    q, k, wq, wk, cos, sin = host
    worst = None
    for sl in (slice(0, 256), slice(l - 64, l)):
        for x, w, o in ((q, wq, qo), (k, wk, ko)):
            st = parity_stats(o[:, sl].cpu().to(torch.float64).numpy(),
                              qp.rms_norm_rope(x[:, sl], w, cos[sl], sin[sl], 1e-6))
            if worst is None or st["rel_l2"] > worst["rel_l2"]:
                worst = st
    worst["rows"] = "tokens 0..255 and the last 64 of both batch elements, q and k (worst part)"
    r["parity"] = worst
    del dq, dk, qo, ko
    torch.cuda.empty_cache()
    return r


def measure_na3d_config(steps, warmup, peaks, dev, stream):
    import numpy as np
    import torch

    from joint_audio_video_flash_b200 import ltxattn, synth
    from oracle import na3d as na
    grid, window, heads, d, b = NA_GRID, NA_WINDOW, NA_HEADS, NA_D, NA_BATCH
    n = grid[0] * grid[1] * grid[2]
    q, k, v = synth.make_qkv(b, n, n, heads, d, seed=NA_SEED)
    dq, dk, dv = (t.to(dev) for t in (q, k, v))
    out = torch.empty_like(dq)
    us, _ = timed_calls([lambda: ltxattn.na3d_forward(dq, dk, dv, grid, window, out)],
                        steps, warmup, stream, None)
    ltxattn.check()
    r = dist_stats(us[0])
    flops = na3d_step_flops()
    issued = na_issued_flops(grid, window, b, heads, d)
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tfl = flops / (r["us_median"] * 1e-6) / 1e12
    r.update({"tflops": tfl, "frac_bf16_peak": tfl / burst, "bound": "tensor",
              "issued_tflops": issued / (r["us_median"] * 1e-6) / 1e12, "density": flops / issued,
              "l2": "inputs larger than L2", "steps": steps,
              "description": na3d_config(1)["description"]})
    # parity on 192 tokens: the grid's corners and edges and seeded interior tokens
    g = np.random.default_rng(NA_SEED)
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(n - 64, n),
                                     g.integers(0, n, 64)]))
    ref = na.na3d(q, k, v, grid, window, d ** -0.5, rows=rows)
    got = out.cpu().to(torch.float64)[:, torch.as_tensor(rows)].numpy()
    r["parity"] = parity_stats(got, ref)
    r["parity"]["rows"] = f"{len(rows)} tokens x {heads} heads"
    del dq, dk, dv, out
    torch.cuda.empty_cache()
    return r


def per_config_table(args, peaks, dev, stream):
    import torch
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    table = {}
    with NvmlClockTrace(device_uuid(dev)) as trace:
        for name in PER_CONFIG_ATTENTION:
            table[name] = measure_attention_config(name, args.per_config_steps, 3, peaks, dev,
                                                   stream, flush, trace)
        table["qk_prologue"] = measure_prologue_config(args.per_config_steps, 3, peaks, dev,
                                                       stream)
        table["na3d_decoder"] = measure_na3d_config(args.per_config_steps, 3, peaks, dev, stream)
    del flush
    torch.cuda.empty_cache()
    return table


# --------------------------------------------------------------------------- dist
def dist_setup(n_gpus: int, backend: str = "nccl", timeout_s: float = 120.0):
    """Process group for N replicas (one process per GPU; torchrun's env variables).

    Only the barrier and the max-over-ranks timing use it: every (batch, head) of every call
    is independent, so there is no data-path collective.  `backend` "gloo" runs the same
    host logic on CPU processes (tests).
    """
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if backend == "nccl":
        import torch
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest x over all ranks (the job's time is its slowest replica's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(step_flops: float, steps: int, world: int, total_ms: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the max-over-ranks device time."""
    return step_flops * steps * world / (total_ms * 1e-3) / 1e12


# --------------------------------------------------------------------------- main arms
def run_reference(args):
    from joint_audio_video_flash_b200 import workloads
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    desc, calls = workloads.configs()[args.workload]
    from oracle import oracle
    oracle.build()
    total = sum(c.flops for c in calls)
    per_step_s = max(2.0, args.reference_budget_s / (args.steps + args.warmup))
    f0 = min(1.0, 1e9 / total)
    fl, s, _ = oracle_sample(calls, f0, 0)
    frac = min(1.0, max(f0, per_step_s * (fl / max(s, 1e-9)) / total))
    for w in range(args.warmup):
        oracle_sample(calls, f0, 100 + w)
    flops = secs = 0.0
    rows = 0
    for st in range(args.steps):
        a, b, r = oracle_sample(calls, frac, 1000 + st)
        flops += a
        secs += b
        rows += r
    value = flops / secs / 1e12
    sample = (f"{rows} query rows over {args.steps} steps ({frac:.4%} of every call's real rows "
              f"per step, same work mix), fp64 oracle, OpenMP over rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "description": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ltxattn(args):
    import torch

    from joint_audio_video_flash_b200 import build, ltxattn, synth, workloads

    world, rank, local = dist_setup(args.gpus)
    build.build()
    ltxattn.create()
    desc, calls = workloads.configs()[args.workload]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    host, dev_in, outs, splits = [], [], [], []
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                                 q_valid=c.q_valid, kv_valid=c.kv_valid_len)
        host.append((q, k, v))
        dev_in.append(tuple(t.to(dev) for t in (q, k, v)))
        outs.append(torch.empty_like(dev_in[-1][0]))

    items = launch_items(calls, grouped=not args.no_group)
    splits = [1] * len(calls)

    def launch(item):
        if len(item) > 1:  # one forward_grouped: a2v and audio self-attention share a launch
            ltxattn.forward_grouped([dict(q=dev_in[i][0], k=dev_in[i][1], v=dev_in[i][2],
                                          out=outs[i], kv_valid_len=calls[i].kv_valid_len,
                                          scale=calls[i].scale) for i in item])
            return
        i = item[0]
        _, splits[i] = ltxattn.forward(*dev_in[i], outs[i], kv_valid_len=calls[i].kv_valid_len,
                                       scale=calls[i].scale, return_splits=True)

    def step(events=None):
        for j, item in enumerate(items):
            if events is not None:
                events[j][0].record(stream)
            launch(item)
            if events is not None:
                events[j][1].record(stream)

    if args.once:  # one launch set, no timing: the command the Nsight Compute captures run
        step()
        torch.cuda.synchronize()
        ltxattn.check()
        print(json.dumps({"workload": args.workload, "once": True, "splits": splits,
                          "items": items}))
        return
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    ltxattn.check()

    per_item = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in items] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    with ClockSampler(uuid) as clocks, NvmlClockTrace(uuid) as trace:
        barrier(world)
        torch.cuda.synchronize()
        wall0 = time.time()
        t_start.record(stream)
        for s in range(args.steps):
            step(per_item[s])
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ltxattn.check()
    total_ms = t_start.elapsed_time(t_end)
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    step_flops = sum(c.flops for c in calls)
    value = whole_job_tflops(step_flops, args.steps, world, total_ms)

    item_us, item_wall = [], []
    for j in range(len(items)):
        item_us.append([per_item[s][j][0].elapsed_time(per_item[s][j][1]) * 1e3
                        for s in range(args.steps)])
        item_wall.append([(wall0 + t_start.elapsed_time(per_item[s][j][0]) * 1e-3,
                           wall0 + t_start.elapsed_time(per_item[s][j][1]) * 1e-3)
                          for s in range(args.steps)])
    launches_per_step = sum(item_launches(it, splits) for it in items)

    # ---- the members of a grouped launch, timed once more (outside the timed region, L2
    # flushed before every call, interleaved so that all see the same clocks): the whole
    # group, each member alone through forward (its own launch and kernel), and the group
    # without it through forward_grouped, so that the group's time splits into what each
    # member adds to the shared launch
    item_of = {i: j for j, it in enumerate(items) for i in it}
    member_us = {}
    groups = [it for it in items if len(it) > 1]
    if groups:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        fns, keys = [], []
        for gi, it in enumerate(groups):
            fns.append(lambda it=it: launch(it))
            keys.append(("group", gi))
            for i in it:
                fns.append(lambda i=i: ltxattn.forward(*dev_in[i], outs[i],
                                                       kv_valid_len=calls[i].kv_valid_len,
                                                       scale=calls[i].scale))
                keys.append(("alone", i))
                rest = [x for x in it if x != i]
                fns.append(lambda rest=rest: launch(rest) if len(rest) > 1 else
                           ltxattn.forward_grouped([dict(
                               q=dev_in[rest[0]][0], k=dev_in[rest[0]][1], v=dev_in[rest[0]][2],
                               out=outs[rest[0]], kv_valid_len=calls[rest[0]].kv_valid_len,
                               scale=calls[rest[0]].scale)]))
                keys.append(("without", i))
        us_m, _ = timed_calls(fns, args.steps, 3, stream, flush)
        ltxattn.check()
        member_us = dict(zip(keys, us_m))
        del flush
        step()  # outs hold the timed configuration's results again (checked below)
        torch.cuda.synchronize()

    # ---- end to end through the public API with host buffers.  Every step uploads all
    # inputs from pinned host memory and downloads every output; uploads run on one copy
    # stream and downloads on another (PCIe is full duplex), each launch item waits for
    # its own uploads, and an upload into a device buffer waits for the previous step's
    # kernel that read it.
    pinned = [tuple(t.pin_memory() for t in trip) for trip in host]
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    h2d = sum(t.numel() * t.element_size() for trip in pinned for t in trip)
    d2h = sum(o.numel() * o.element_size() for o in host_out)
    e2e_steps = max(1, min(args.steps, 5))
    up_stream = torch.cuda.Stream(device=dev)
    down_stream = torch.cuda.Stream(device=dev)
    consumed = [None] * len(items)  # event: item j's kernels of the previous step finished
    drained = [None] * len(calls)   # event: call i's output of the previous step downloaded

    def e2e_step():
        for j, item in enumerate(items):
            with torch.cuda.stream(up_stream):
                if consumed[j] is not None:
                    up_stream.wait_event(consumed[j])
                for i in item:
                    for d_t, h_t in zip(dev_in[i], pinned[i]):
                        d_t.copy_(h_t, non_blocking=True)
                uploaded = torch.cuda.Event()
                uploaded.record(up_stream)
            stream.wait_event(uploaded)
            for i in item:
                if drained[i] is not None:
                    stream.wait_event(drained[i])
            launch(item)
            done = torch.cuda.Event()
            done.record(stream)
            consumed[j] = done
            with torch.cuda.stream(down_stream):
                down_stream.wait_event(done)
                for i in item:
                    host_out[i].copy_(outs[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(down_stream)
                for i in item:
                    drained[i] = ev

    e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    up_stream.wait_event(e0)  # no copy of the timed steps starts before the start event
    for _ in range(e2e_steps):
        e2e_step()
    # the timed region ends when the last download has landed
    for ev in drained:
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ltxattn.check()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = whole_job_tflops(step_flops, e2e_steps, world, e2e_ms)

    peaks, peak_src = load_peaks()
    # dominant kernel: the call with the most FLOPs.  Its bound follows from its arithmetic
    # intensity against the measured ridge point.  For a tensor-bound call the denominator
    # is the burst GEMM peak while the SM clock held near its maximum during the timed
    # region (the sustained figure was measured at the power-capped clock), else the
    # sustained one.
    vi = max(range(len(calls)), key=lambda i: calls[i].flops)
    assert items[item_of[vi]] == [vi], "the dominant call runs on its own launch"
    v_us = statistics.mean(item_us[item_of[vi]])
    clk = clocks.summary()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    at_max = bool(clk.get("sm_mhz") is not None and clk.get("sm_max_mhz")
                  and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"])
    tflops_peak = burst if at_max else sustained
    tr = TRAFFIC.get(calls[vi].name)
    traffic = None
    if tr is not None and tr["src"] == kernel_source_hash("video_self"):
        traffic = tr["bytes_per_token"] * calls[vi].batch * calls[vi].q_len
    if calls[vi].flops / calls[vi].bytes > tflops_peak * 1e12 / (hbm * 1e9):
        achieved = calls[vi].flops / (v_us * 1e-6) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tflops_peak,
                    "unit": "TFLOP/s", "frac": achieved / tflops_peak,
                    "frac_of_sustained_peak": achieved / sustained,
                    "peak_source": f"{peak_src} " + (
                        "bf16_tflops (burst; SM clock at max during the timed region)"
                        if at_max else "bf16_tflops_sustained")}
    else:
        achieved = calls[vi].bytes / (v_us * 1e-6) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "peak_source": f"{peak_src} hbm_gbs"}
    roofline.update({"traffic": traffic, "kernel": kernel_label(calls[vi]),
                     "call": calls[vi].name, "algorithmic_flops": calls[vi].flops,
                     "algorithmic_bytes": calls[vi].bytes})

    per_call_out = {}
    for i, c in enumerate(calls):
        j = item_of[i]
        grouped = len(items[j]) > 1
        us_list = group_share(items[j], i, member_us, groups) if grouped else item_us[j]
        entry = dist_stats(us_list)
        added = grouped and group_base(items[j], member_us) != i
        # a member that rides in another call's launch adds too little time for a throughput
        # figure to mean anything: its roofline fields are left out
        if not added:
            entry.update(call_roofline(c.flops, c.bytes, entry["us_median"], peaks))
        entry.update({
            "shape": f"B{c.batch} Lq{c.q_len} Lkv{c.kv_len} valid{c.kv_valid_len} "
                     f"H{c.heads} D{c.head_dim}",
            "splits": splits[i],
            "kernel": kernel_label(c, grouped=True) if grouped else kernel_label(c)})
        if grouped:
            # us_* above: this call's share of the grouped launch (group_share); measured in
            # the interleaved loop after the timed step, L2 flushed before every call
            group_alone = statistics.median(member_us[("group", groups.index(items[j]))])
            without = statistics.median(member_us[("without", i)])
            entry["group"] = {
                "members": [calls[x].name for x in items[j]],
                "share": "base" if group_base(items[j], member_us) == i else "added",
                "us_median_in_step": statistics.median(item_us[j]),  # the timed step
                "us_median": group_alone,
                "us_without_this_call": without,
                "us_added_by_this_call": group_alone - without,
                # the call on a launch of its own (its own kernel choice)
                "us_median_own_launch": statistics.median(member_us[("alone", i)]),
                "kernel_own_launch": kernel_label(c)}
        if c.flops / c.bytes > 1000:  # tensor-bound: time beside the SM clock it ran at
            entry["clock"] = clock_normalised(item_us[j], item_wall[j], trace)
        if rank == 0 and not args.no_parity:  # the oracle on sampled rows, after the timing
            entry["parity"] = attention_parity(c, *host[i], outs[i], seed=c.seed)
        per_call_out[c.name] = entry

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": desc,
                   "l2": "inputs larger than L2 (video q/k/v alone exceed 126 MB per step)",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "per_call": per_call_out,
        "launch_items": [[calls[i].name for i in it] for it in items],
    }
    if rank == 0 and world == 1 and not args.no_per_config and args.workload == "block768":
        del dev_in, pinned
        torch.cuda.empty_cache()
        line["per_config"] = per_config_table(args, peaks, dev, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(calls, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


PROLOGUE_SHAPE, PROLOGUE_SEED = (2, 15360, 32, 128), 21  # batch, tokens, heads, head_dim
PROLOGUE_METRIC = "qk norm + rotary prologue GB/s"
NA_GRID, NA_WINDOW, NA_HEADS, NA_D, NA_BATCH, NA_SEED = (16, 34, 60), (3, 7, 7), 32, 128, 1, 77
NA_METRIC = "3-D neighbourhood attention TFLOP/s (neighbourhood FLOPs)"


def prologue_config(world):
    return {"workload": "qk_prologue",
            "description": "queries and keys of the video stream, B2 x 15360 tokens x "
                           "32 heads x 128: RMSNorm over heads*dim, rotary on channel "
                           "pairs (a reading; see the header)",
            "l2": "inputs larger than L2 (q and k are 252 MB each)",
            "parallelism": f"replicas x{world}"}


def prologue_step_bytes():
    b, l, h, d = PROLOGUE_SHAPE
    # q and k read and written once (bf16); weights and tables are 0.1 %
    return 4.0 * b * l * h * d * 2 + 2 * h * d * 2 + 2 * l * (d // 2) * 4


def prologue_oracle_time(inputs, seconds, start=0, block=512):
    """Runs the fp64 oracle over token blocks from `start` for about `seconds`; returns
    (tokens done, seconds)."""
    from oracle import qk_prologue as qp
    q, k, wq, wk, cos, sin = inputs
    l = q.shape[1]
    done, secs = 0, 0.0
    while done < l and secs < seconds:
        a = (start + done) % l
        sl = slice(a, min(l, a + block))
        t_start = time.perf_counter()
        qp.rms_norm_rope(q[:, sl], wq, cos[sl], sin[sl], 1e-6)
        qp.rms_norm_rope(k[:, sl], wk, cos[sl], sin[sl], 1e-6)
        secs += time.perf_counter() - t_start
        done += sl.stop - sl.start
    return done, secs


def na3d_config(world):
    return {"workload": "na3d_decoder",
            "description": "grid 16 x 34 x 60 tokens (960x544x121 at 16x16 patches and "
                           "8-frame compression, a reading), window 3 x 7 x 7, "
                           "32 heads x 128, batch 1",
            "l2": "inputs larger than L2 (q, k, v 267 MB each)",
            "parallelism": f"replicas x{world}"}


def na3d_step_flops():
    n = NA_GRID[0] * NA_GRID[1] * NA_GRID[2]
    vol = NA_WINDOW[0] * NA_WINDOW[1] * NA_WINDOW[2]
    # every query against its neighbourhood: QK and PV, 2 FLOP a multiply-add
    return 4.0 * NA_BATCH * NA_HEADS * n * vol * NA_D


def na3d_oracle_time(q, k, v, seconds, start=0, chunk=512):
    """Runs the fp64 oracle over query-token chunks from `start` for about `seconds`;
    returns (tokens done, seconds)."""
    import numpy as np

    from oracle import na3d as na
    n = q.shape[1]
    done, secs = 0, 0.0
    while secs < seconds and done < n:
        a = (start + done) % n
        rows = np.arange(a, min(n, a + chunk))
        t_start = time.perf_counter()
        na.na3d(q, k, v, NA_GRID, NA_WINDOW, NA_D ** -0.5, rows=rows)
        secs += time.perf_counter() - t_start
        done += len(rows)
    return done, secs


def run_reference_other(args):
    """Reference arm of the prologue and neighbourhood workloads: their fp64 oracles, timed
    on a bounded sample per step (CPU only; rank 0 alone)."""
    from joint_audio_video_flash_b200 import synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    per_step_s = max(1.0, args.reference_budget_s / (args.steps + args.warmup))
    if args.workload == "qk_prologue":
        b, l, h, d = PROLOGUE_SHAPE
        inputs = synth.make_qk_prologue_inputs(b, l, h, d, seed=PROLOGUE_SEED)
        run = lambda st: prologue_oracle_time(inputs, per_step_s, start=st * 4096)  # noqa: E731
        total, per_token, metric, unit, config = l, prologue_step_bytes() / l / 1e9, \
            PROLOGUE_METRIC, "GB/s", prologue_config(world)
        what = "token blocks of 512, both batch elements, q and k; numpy fp64, one core"
    else:
        n = NA_GRID[0] * NA_GRID[1] * NA_GRID[2]
        q, k, v = synth.make_qkv(NA_BATCH, n, n, NA_HEADS, NA_D, seed=NA_SEED)
        run = lambda st: na3d_oracle_time(q, k, v, per_step_s, start=st * 4096)  # noqa: E731
        total, per_token, metric, unit, config = n, na3d_step_flops() / n / 1e12, \
            NA_METRIC, "TFLOP/s", na3d_config(world)
        what = "query-token chunks of 512, all 32 heads; numpy fp64, one core"
    for w in range(args.warmup):
        run(100 + w)
    done = secs = 0.0
    for st in range(args.steps):
        a, b_ = run(st)
        done += a
        secs += b_
    value = per_token * done / secs
    sample = f"{int(done)} of {total} tokens per workload pass over {args.steps} steps: {what}"
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
        "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_prologue(args):
    """The QK-norm + rotary prologue at the video stream's size (HBM-bound streaming kernel)."""
    import torch

    from joint_audio_video_flash_b200 import build, ltxattn, synth
    world, rank, local = dist_setup(args.gpus)
    build.build()
    b, l, h, d = PROLOGUE_SHAPE
    q, k, wq, wk, cos, sin = synth.make_qk_prologue_inputs(b, l, h, d, seed=PROLOGUE_SEED)
    dev = torch.device("cuda", local)
    dq, dk, dwq, dwk, dcos, dsin = (t.to(dev) for t in (q, k, wq, wk, cos, sin))
    qo, ko = torch.empty_like(dq), torch.empty_like(dk)
    stream = torch.cuda.current_stream()

    def step():
        ltxattn.qk_norm_rope(dq, dk, dwq, dwk, dcos, dsin, qo, ko)

    if args.once:  # one launch, no timing: the command the Nsight Compute captures run
        step()
        torch.cuda.synchronize()
        print(json.dumps({"workload": args.workload, "once": True}))
        return
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    with ClockSampler(uuid) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    step_bytes = prologue_step_bytes()
    value = step_bytes * args.steps * world / (total_ms * 1e-3) / 1e9
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # end to end through the same call: every step uploads q and k from pinned host memory
    # and downloads both outputs.  Each batch element is its own piece: uploads run on one
    # copy stream and downloads on another (PCIe is full duplex), a piece's kernel waits
    # for its upload, and an upload into a device buffer waits for the kernel that last
    # read it.
    hq, hk = q.pin_memory(), k.pin_memory()
    oq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    ok_ = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    up_stream, down_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    consumed, drained = [None] * b, [None] * b

    def e2e_step():
        for i in range(b):
            with torch.cuda.stream(up_stream):
                if consumed[i] is not None:
                    up_stream.wait_event(consumed[i])
                dq[i].copy_(hq[i], non_blocking=True)
                dk[i].copy_(hk[i], non_blocking=True)
                uploaded = torch.cuda.Event()
                uploaded.record(up_stream)
            stream.wait_event(uploaded)
            if drained[i] is not None:
                stream.wait_event(drained[i])
            ltxattn.qk_norm_rope(dq[i:i + 1], dk[i:i + 1], dwq, dwk, dcos, dsin, qo[i:i + 1],
                                 ko[i:i + 1])
            done = torch.cuda.Event()
            done.record(stream)
            consumed[i] = done
            with torch.cuda.stream(down_stream):
                down_stream.wait_event(done)
                oq[i].copy_(qo[i], non_blocking=True)
                ok_[i].copy_(ko[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(down_stream)
                drained[i] = ev

    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    up_stream.wait_event(e0)  # no copy of the timed steps starts before the start event
    for _ in range(e2e_steps):
        e2e_step()
    for ev in drained:  # the timed region ends when the last download has landed
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    line = {
        "metric": PROLOGUE_METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": prologue_config(world),
        "roofline": {"bound": "hbm", "achieved": value, "peak": hbm, "unit": "GB/s",
                     "frac": value / hbm, "traffic": traffic_per_launch("qk_prologue"),
                     "kernel": "ltx_qk_norm_rope<4, 4, 2>",
                     "algorithmic_bytes": step_bytes, "peak_source": f"{peak_src} hbm_gbs"},
        "e2e": {"value": step_bytes * e2e_steps * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": 2 * q.numel() * 2, "d2h_bytes_per_step": 2 * q.numel() * 2},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    line["e2e"]["steps"] = e2e_steps
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, secs = prologue_oracle_time((q, k, wq, wk, cos, sin), args.cpu_seconds)
        line["cpu_baseline"] = {"value": step_bytes * (done / l) / secs / 1e9, "unit": "GB/s",
                                "cores": 1, "kind": "oracle",
                                "sample": f"token positions 0..{done - 1} of {l} in blocks of "
                                          f"512, both batch elements, q and k; numpy fp64, "
                                          f"{secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# (query brick, key tile) pairs the library is built for, as t x y x x
def na_key_tiles(grid, window, with_shape=False):
    """Key tiles the neighbourhood kernel multiplies per (batch, head), from the library's own
    plan (``ltxattn_na3d_plan``, host only).  With with_shape, also the query brick and key
    tile shapes."""
    from joint_audio_video_flash_b200 import ltxattn
    brick, tile, tiles = ltxattn.na3d_plan(grid, window)
    return (tiles, brick, tile) if with_shape else tiles


def na_issued_flops(grid, window, b, heads, d):
    """FLOPs of the tiles the tensor cores multiply: QK^T and PV of every 128-query x
    (keys per tile) tile."""
    tiles, _, kb = na_key_tiles(grid, window, with_shape=True)
    return tiles * b * heads * 4.0 * 128 * (kb[0] * kb[1] * kb[2]) * d


def na_kernel_label(grid, window, d):
    _, qb, kb = na_key_tiles(grid, window, with_shape=True)
    return f"ltx_na3d_fwd<{d}, query {qb[0]}x{qb[1]}x{qb[2]}, keys {kb[0]}x{kb[1]}x{kb[2]}>"


def run_na3d(args):
    """3-D neighbourhood attention over the decoder-size grid (tensor-core kernel)."""
    import torch

    from joint_audio_video_flash_b200 import build, ltxattn, synth
    world, rank, local = dist_setup(args.gpus)
    build.build()
    ltxattn.create()
    grid, window, heads, d, b = NA_GRID, NA_WINDOW, NA_HEADS, NA_D, NA_BATCH
    n = grid[0] * grid[1] * grid[2]
    q, k, v = synth.make_qkv(b, n, n, heads, d, seed=NA_SEED)
    dev = torch.device("cuda", local)
    dq, dk, dv = (t.to(dev) for t in (q, k, v))
    out = torch.empty_like(dq)
    stream = torch.cuda.current_stream()

    def step():
        ltxattn.na3d_forward(dq, dk, dv, grid, window, out)

    if args.once:  # one launch, no timing: the command the Nsight Compute captures run
        step()
        torch.cuda.synchronize()
        ltxattn.check()
        print(json.dumps({"workload": args.workload, "once": True}))
        return
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    ltxattn.check()
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ltxattn.check()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    step_flops = na3d_step_flops()
    value = whole_job_tflops(step_flops, args.steps, world, total_ms)
    issued = na_issued_flops(grid, window, b, heads, d)  # the tiles the tensor cores multiply
    issued_tflops = whole_job_tflops(issued, args.steps, world, total_ms)
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # end to end: q, k, v up from pinned host memory and the output down, every step
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ltxattn.check()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    line = {
        "metric": NA_METRIC, "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": na3d_config(world),
        "roofline": {"bound": "tensor", "achieved": value, "peak": burst, "unit": "TFLOP/s",
                     "frac": value / burst, "traffic": traffic_per_launch("na3d_decoder"),
                     "kernel": na_kernel_label(grid, window, d),
                     "issued_tflops": issued_tflops, "issued_frac": issued_tflops / burst,
                     "density": step_flops / issued,
                     "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "e2e": {"value": whole_job_tflops(step_flops, e2e_steps, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": q.numel() * 2,
                "steps": e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, secs = na3d_oracle_time(q, k, v, args.cpu_seconds)
        line["cpu_baseline"] = {"value": step_flops * (done / n) / secs / 1e12, "unit": "TFLOP/s",
                                "cores": 1, "kind": "oracle",
                                "sample": f"tokens 0..{done - 1} of {n}, all 32 heads; numpy "
                                          f"fp64, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


CP_SEQ, CP_AUDIO, CP_AUDIO_VALID, CP_SEED = 27280, 256, 252, 91
CP_METRIC = "context-parallel attention TFLOP/s (video self + v2a, long clip)"


def cp_config(world):
    return {"workload": "cp_longclip",
            "description": "long clip 1280x704x241: video self-attention over 27280 tokens "
                           "(B2, 32x128) with the sequence sharded over the ranks, and v2a "
                           "(audio 252->256 queries, 32x64) over the sharded video keys; "
                           "K/V shards broadcast per source rank, partials merged through "
                           "their softmax statistics",
            "l2": "inputs larger than L2", "parallelism": f"cp{world} (sequence sharded)"}


def cp_step_flops():
    b, h = 2, 32
    return 4.0 * b * h * 128 * CP_SEQ * CP_SEQ + 4.0 * b * h * 64 * CP_AUDIO_VALID * CP_SEQ


def run_cp(args):
    """Context-parallel attention (the row built on ltxattn_forward_partial and
    ltxattn_combine) at the long-clip size.  Strong scaling: every step is the whole problem,
    shared by the ranks; with one GPU the process group has one rank (NCCL all the same)."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    from joint_audio_video_flash_b200 import build, cp, ltxattn, synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world == 1:
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    else:
        dist_setup(args.gpus)
    build.build()
    ltxattn.create()
    b, h, d, da = 2, 32, 128, 64
    ls = cp.shard_len(CP_SEQ, world)
    lo, hi = rank * ls, min(CP_SEQ, (rank + 1) * ls)

    def shard(t):
        out = torch.zeros((t.shape[0], ls, *t.shape[2:]), dtype=t.dtype)
        if hi > lo:
            out[:, :hi - lo] = t[:, lo:hi]
        return out

    # every rank draws the whole problem from the same seeds and keeps its shard
    vq, vk, vv = synth.make_qkv(b, CP_SEQ, CP_SEQ, h, d, seed=CP_SEED)
    aq, _, _ = synth.make_qkv(b, CP_AUDIO, 1, h, da, seed=CP_SEED + 1, q_valid=CP_AUDIO_VALID)
    _, xk, xv = synth.make_qkv(b, 1, CP_SEQ, h, da, seed=CP_SEED + 2)
    host = [shard(vq), shard(vk), shard(vv), aq, shard(xk), shard(xv)]
    dq, dk, dv, daq, dxk, dxv = (t.to(dev) for t in host)
    stream = torch.cuda.current_stream()
    outs = {}

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        outs["self"] = cp.self_attention(dq, dk, dv, CP_SEQ, None)
        if ev is not None:
            ev[1].record(stream)
        outs["v2a"] = cp.cross_attention(daq, dxk, dxv, CP_SEQ, None)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ltxattn.check()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = device_uuid(dev)
    with ClockSampler(uuid) as clocks:
        dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for s_ in range(args.steps):
            step(evs[s_])
        t1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
    ltxattn.check()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    self_us = [e[0].elapsed_time(e[1]) * 1e3 for e in evs]
    v2a_us = [e[1].elapsed_time(e[2]) * 1e3 for e in evs]
    step_flops = cp_step_flops()
    value = step_flops * args.steps / (total_ms * 1e-3) / 1e12
    # the dominant kernels: this rank's partials over every shard (tensor-bound)
    own_flops = 4.0 * b * h * d * max(0, hi - lo) * CP_SEQ
    t_self = statistics.median(self_us)
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = own_flops / (t_self * 1e-6) / 1e12
    # end to end: this rank's shards up from pinned host memory, both results down
    pinned = [t.pin_memory() for t in host]
    dsts = [dq, dk, dv, daq, dxk, dxv]
    h_self = torch.empty((b, ls, h, d), dtype=torch.bfloat16, pin_memory=True)
    h_v2a = torch.empty((b, CP_AUDIO, h, da), dtype=torch.bfloat16, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        for dst, src in zip(dsts, pinned):
            dst.copy_(src, non_blocking=True)
        step()
        h_self.copy_(outs["self"], non_blocking=True)
        h_v2a.copy_(outs["v2a"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    line = {
        "metric": CP_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cp_config(world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                     "frac": achieved / burst, "traffic": None,
                     "kernel": "ltx_attn_fwd_pp<128, split> over every shard + ltx_attn_combine",
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "note": "this rank's video self-attention (partials, exchange waits and "
                             "merge) timed with CUDA events"},
        "per_call": {"video_self_cp": dist_stats(self_us), "v2a_cp": dist_stats(v2a_us)},
        "e2e": {"value": step_flops * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host),
                "d2h_bytes_per_step": h_self.numel() * 2 + h_v2a.numel() * 2,
                "steps": e2e_steps},
        "gpu_launches": None,
        "clocks": clocks.summary(),
    }
    # launches per step: one partial per non-empty shard + the merge, and v2a's partial + merge
    n_shards = sum(1 for r in range(world) if cp.shard_valid(CP_SEQ, world, r) > 0)
    line["gpu_launches"] = (n_shards + 1 + (1 if hi > lo else 0) + 1) * args.steps
    if rank == 0 and not args.no_parity:
        from oracle import oracle
        rows_s = synth.sample_rows(b, ls, h, 2, seed=CP_SEED, full_heads=())
        bi, rem = rows_s // (ls * h), rows_s % (ls * h)
        i, hh = rem // h, rem % h
        keep = (lo + i) < hi
        rows_s, bi, i, hh = rows_s[keep], bi[keep], i[keep], hh[keep]
        full_rows = ((bi * CP_SEQ + lo + i) * h + hh).numpy()
        ref = oracle.attention(vq, vk, vv, d ** -0.5, rows=full_rows)
        got = outs["self"].cpu().to(torch.float64).reshape(-1, d)[rows_s].numpy()
        par = {"video_self_cp": parity_stats(got, ref)}
        ref2 = oracle.attention(aq, xk, xv, da ** -0.5)
        par["v2a_cp"] = parity_stats(outs["v2a"].cpu().to(torch.float64).numpy(), ref2)
        line["parity"] = par
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from joint_audio_video_flash_b200 import workloads
        calls = [c for c in workloads.configs()["longclip"][1] if c.name in ("video_self", "v2a")]
        line["cpu_baseline"] = cpu_baseline(calls, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ltxattn", "reference"], default="ltxattn")
    ap.add_argument("--workload", default="block768")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-budget-s", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-config table (every other workload, timed on its own)")
    ap.add_argument("--no-parity", action="store_true",
                    help="skip the oracle comparison of the timed outputs")
    ap.add_argument("--per-config-steps", type=int, default=10)
    ap.add_argument("--no-group", action="store_true",
                    help="launch a2v and audio self-attention separately (forward per call) "
                         "instead of through one forward_grouped")
    ap.add_argument("--once", action="store_true",
                    help="run each call of the workload once and exit (profiling)")
    ap.add_argument("--cp", action="store_true",
                    help="context-parallel attention at the long-clip size (sequence sharded "
                         "over the ranks; strong scaling)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.cp and args.impl != "reference":
        run_cp(args)
        return
    if args.cp:
        args.workload = "longclip"
    if args.workload in ("qk_prologue", "na3d_decoder") and args.impl == "reference":
        run_reference_other(args)
    elif args.workload == "qk_prologue":
        run_prologue(args)
    elif args.workload == "na3d_decoder":
        run_na3d(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ltxattn(args)


if __name__ == "__main__":
    main()
