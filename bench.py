"""Benchmark of the PR-Sink per-block step on B200.

One step = one block of a 480x480 stream through 40 attention layers (heads 40 x 128): the
fingerprint and pose retrieval with the dynamic-sink fill of every layer, then per layer the 3
denoising passes and the Clean KV Update pass (KV append into ring slot b mod 3 + PR-Sink
attention over ref 900 + static 2700 + dynamic 2700 + 3 x 2700 ring = 14400 keys), then the bank
update.  By default (``--path fused``) each pass is one prsink_attention_fused launch, which
stores the pass's K/V into the ring slot itself, after one rotation pass per layer and block
(prsink_rotate_sinks); ``--path unfused`` launches the append and prsink_attention separately.  The bank (M = 5) is filled during the first 20 blocks, which run untimed before the
warm-up; the timed blocks are the steady state after it is frozen.

Metric: blocks/s per 40-head layer (layer-blocks per second of the whole job), with the
attention TFLOP/s and its fraction of the measured dense bf16 peak.  Inputs are synthetic
(N(0,1) bf16 Q/K/V, clustered synthetic poses); per-layer caches are 295 MB and 40 layers are
cycled, so every launch reads from HBM (the working set is far above the 126 MB L2).

At one GPU the line also carries sub-records: each kernel timed alone (KV append, the 40-layer
dynamic-sink fill, attention at the 3024-query layouts, attention on rotating and on repeated
inputs) and a 300-block stream from block 0 (bank written during the first 20 blocks, then
frozen), end to end on the device.

``--gpus N`` runs one process per GPU (started here through torch.distributed.run when no
launcher did).  ``--partition heads`` (default) splits the 40 heads of every cache and bank
entry over the ranks, as the pages' Ulysses layout does, with the pose decisions replicated:
one stream, strong scaling.  ``--partition replicas`` runs an independent stream per rank
(weak scaling).  No collective is on the data path either way.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
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

METRIC = "PR-Sink attention TFLOPS (% of bf16 peak) and blocks/s per 40-head layer at 1 B200"
UNIT = "layer-blocks/s"
PASSES = 4          # 3 denoising passes + the Clean KV Update pass
M_BANK = 5
WRITE_BLOCKS = 20


def max_over_ranks(x: float, device, world: int) -> float:
    """Max of a per-rank timing over all ranks (the job takes as long as its slowest rank); the
    identity on one rank.  `device` is where the reduction tensor lives (cuda for NCCL, cpu for
    gloo)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(n_layers: int, steps: int, streams: int, seconds: float) -> float:
    """Layer-blocks per second of the whole job: each of `streams` independent streams (one per
    rank for replicas, one for the whole job when the heads are split) runs `steps` blocks of
    `n_layers` layers, and the job's time is the slowest rank's."""
    return n_layers * steps * streams / seconds


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def _profiled_traffic(src_rel: str, profile_rel: str):
    """DRAM bytes per launch (read + write) recorded from an ncu capture in ``profiles/``, or
    None when the kernel's sources (its .cu file and the shared device header) have changed
    since that capture (sha256 mismatch)."""
    import hashlib
    try:
        h = hashlib.sha256()
        for rel in (src_rel, KERNEL_HEADER):
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        digest = h.hexdigest()
        with open(os.path.join(ROOT, profile_rel)) as f:
            text = f.read()
    except OSError:
        return None
    rec_hash = rec_bytes = None
    for line in text.splitlines():
        if line.startswith("kernel source sha256"):
            rec_hash = line.split(":", 1)[1].strip()
        elif line.startswith("DRAM bytes per launch (read + write):"):
            rec_bytes = int(line.split(":", 1)[1].strip())
    return rec_bytes if rec_hash == digest else None


KERNEL_HEADER = "pose_retrieved_kv_b200/csrc/prsink_internal.cuh"
ATTN_SRC = "pose_retrieved_kv_b200/csrc/attention_sm100.cu"
ATTN_PROFILE = "profiles/attention_480x480.md"
FUSED_PROFILE = "profiles/attention_fused_480x480.md"
APPEND_SRC = "pose_retrieved_kv_b200/csrc/kv_copy.cu"
APPEND_PROFILE = "profiles/append_480x480.md"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, pw, smax, reasons = [], [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[3]))
            except ValueError:
                pass
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        loaded = [v for v in sm if v > 0.5 * smax] or sm
        rec = {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
               "reasons": sorted(reasons), "samples": len(sm)}
        if pw:
            rec["power_w"] = statistics.median(pw)    # board power draw, median of the samples
        return rec


# ------------------------------------------------------------------------------------------
# kernels timed alone
# ------------------------------------------------------------------------------------------

def time_launches(launch, warmup: int, steps: int):
    """Device times (ms) of ``launch(i)`` after ``warmup`` untimed launches: the average launch
    duration in a steady stream of ``steps`` back-to-back launches (one CUDA event pair around
    all of them), and each launch's own duration (an event pair per launch, which adds each
    launch's start-up gap; used for min and max).  A device-side sleep is queued ahead of the
    timed launches so that the host has enqueued them all before the first one starts."""
    import torch
    for i in range(warmup):
        launch(i)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e6 + 2e5 * steps))
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    b0.record()
    for i in range(steps):
        launch(warmup + i)
    b1.record()
    torch.cuda.synchronize()
    avg = b0.elapsed_time(b1) / steps
    ev = []
    torch.cuda._sleep(int(2e6 + 4e5 * steps))
    for i in range(steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        launch(warmup + steps + i)
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    return avg, [a.elapsed_time(b) for a, b in ev]


def _summary(ms, work, unit, peak, peak_source):
    avg, each = ms
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    ach = work / (avg / 1e3) / scale
    return {"avg_ms": round(avg, 4), "min_ms": round(min(each), 4), "max_ms": round(max(each), 4),
            "launches": len(each), "achieved": round(ach, 1), "unit": unit, "peak": peak,
            "frac": round(ach / peak, 4), "peak_source": peak_source,
            "timing": "avg: back-to-back launches between one event pair; min/max: one event "
                      "pair per launch"}


def attention_alone(name: str, warmup: int, steps: int, repeat: bool = False, nbuf: int = 2,
                    split: bool = False, heads: int = None):
    """One attention call at a workload's full size (block 1000, every slot valid), timed
    alone.  ``repeat`` = the same inputs every launch; otherwise ``nbuf`` input sets (each
    larger than L2) alternate.  ``split``: prsink_attention_split (the last wave's units split
    over the key range).  ``heads``: fewer heads than the workload's (an L2-resident case)."""
    import torch

    import pose_retrieved_kv_b200 as P
    import synth

    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    if heads is not None:
        cfg["n_heads"] = heads
    lay = P.make_layout(**cfg)
    _, lblk, _, T = P.prsink_layout_tokens(lay)
    H, d = cfg["n_heads"], cfg["head_dim"]
    n = 1 if repeat else nbuf
    q = [synth.normal_bf16((lblk, H, d), 5 + i, 0).cuda() for i in range(n)]
    k = [synth.normal_bf16((H, T, d), 5 + i, 1).cuda() for i in range(n)]
    v = [synth.normal_bf16((H, T, d), 5 + i, 2).cuda() for i in range(n)]
    out = torch.empty((lblk, H, d), dtype=torch.bfloat16, device="cuda")
    nbytes = P.prsink_attention_scratch_bytes(lay) if split else 0
    scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda") if nbytes else None
    if split:
        def launch(i):
            P.prsink_attention_split(lay, q[i % n], k[i % n], v[i % n], out, scratch)
    else:
        def launch(i):
            P.prsink_attention(lay, q[i % n], k[i % n], v[i % n], out)
    ms = time_launches(launch, warmup, steps)
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout")
    peaks = _peaks()
    rec = _summary(ms, 4.0 * lblk * T * d * H, "TFLOP/s", peaks["bf16"],
                   f"{peaks['source']} bf16_tflops (burst)")
    rec.update(queries=lblk, keys=T, gflop=round(4.0 * lblk * T * d * H / 1e9, 1),
               scratch_bytes=nbytes,
               inputs="repeated" if repeat else f"{n} sets of {(lblk + 2 * T) * H * d * 2 / 1e6:.0f} MB alternating")
    return rec


def fused_alone(name: str, warmup: int, steps: int, split: bool = False):
    """prsink_attention_fused (append folded in, sinks read pre-rotated) and the rotation pass
    prsink_rotate_sinks, each timed alone at a workload's full size on two alternating input
    sets (each larger than L2).  ``split``: the last wave split over the key range, as the
    stream runs it when the plan calls for it (prsink_attention_fused_split)."""
    import torch

    import pose_retrieved_kv_b200 as P
    import synth

    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    lay = P.make_layout(**cfg)
    _, lblk, _, T = P.prsink_layout_tokens(lay)
    H, d = cfg["n_heads"], cfg["head_dim"]
    sets = []
    for i in range(2):
        k = synth.normal_bf16((H, T, d), 5 + i, 1).cuda()
        kr = torch.empty_like(k)
        P.prsink_rotate_sinks(lay, k, kr, 0xFFFF)
        sets.append(dict(q=synth.normal_bf16((lblk, H, d), 5 + i, 0).cuda(), k=k,
                         v=synth.normal_bf16((H, T, d), 5 + i, 2).cuda(), kr=kr,
                         kn=synth.normal_bf16((lblk, H, d), 5 + i, 3).cuda(),
                         vn=synth.normal_bf16((lblk, H, d), 5 + i, 4).cuda()))
    out = torch.empty((lblk, H, d), dtype=torch.bfloat16, device="cuda")
    n_scr = P.prsink_attention_scratch_bytes(lay) if split else 0
    scratch = torch.empty(n_scr, dtype=torch.uint8, device="cuda") if n_scr > 0 else None

    def fused(i):
        x = sets[i % 2]
        P.prsink_attention_fused(lay, x["q"], x["kn"], x["vn"], x["kr"], x["k"], x["v"], out,
                                 scratch=scratch)

    ring = ((1 << cfg["ring_slots"]) - 1) << P.SLOT_RING0

    def rotate(i):
        x = sets[i % 2]
        P.prsink_rotate_sinks(lay, x["k"], x["kr"], ring)

    ms_f = time_launches(fused, warmup, steps)
    ms_r = time_launches(rotate, warmup, steps)
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout")
    peaks = _peaks()
    rec = _summary(ms_f, 4.0 * lblk * T * d * H, "TFLOP/s", peaks["bf16"],
                   f"{peaks['source']} bf16_tflops (burst)")
    n_rot = (cfg["ring_slots"] - 1) * lblk * H             # the two older ring slots
    rot = _summary(ms_r, 2.0 * n_rot * d * 2, "GB/s", peaks["hbm"], f"{peaks['source']} hbm_gbs")
    rot["rows_per_call"] = n_rot
    rec.update(queries=lblk, keys=T, scratch_bytes=n_scr,
               note="includes the raw store of the block into its ring slot (the append); "
                    "sinks read from the rotated copy")
    return rec, rot


def append_alone(name: str, warmup: int, steps: int):
    """prsink_kv_append of one block into a ring slot, timed alone: six source blocks and two
    caches rotate, so consecutive launches touch different memory."""
    import torch

    import pose_retrieved_kv_b200 as P
    import synth

    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    lay = P.make_layout(**cfg)
    _, lblk, _, T = P.prsink_layout_tokens(lay)
    H, d = cfg["n_heads"], cfg["head_dim"]
    nbuf = 6
    src = [synth.normal_bf16((lblk, H, d), 5 + i, 0).cuda() for i in range(nbuf)]
    k = [torch.zeros((H, T, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    v = [torch.zeros((H, T, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def launch(i):
        j = i % nbuf
        P.prsink_kv_append(lay, src[j], src[(j + 3) % nbuf], k[i % 2], v[i % 2],
                           P.SLOT_RING0 + (i // 2) % 3)

    ms = time_launches(launch, warmup, steps)
    peaks = _peaks()
    work = 2.0 * 2 * lblk * H * d * 2          # K and V, read + written
    rec = _summary(ms, work, "GB/s", peaks["hbm"], f"{peaks['source']} hbm_gbs")
    rec.update(bytes_per_launch=int(work), inputs=f"{nbuf} source blocks x 2 caches rotating")
    return rec


def dynfill_alone(st, warmup: int, steps: int):
    """The dynamic-sink fill of every layer of a stream (prsink_retrieve with the copy), timed
    alone on the stream's own 40-layer cache and bank: the query fingerprint alternates between
    two bank entries, so every call moves a different entry's K/V of all layers."""
    import torch

    import pose_retrieved_kv_b200 as P

    lay = st.layout()
    count = int(st.bank_count.item())
    if count < 2:
        return None
    phis = [st.bank_phi[j].clone() for j in range(2)]
    r = torch.zeros(1, dtype=torch.int32, device=st.bank_phi.device)
    sc = torch.zeros(1, dtype=torch.float32, device=st.bank_phi.device)
    cp = torch.zeros(1, dtype=torch.int32, device=st.bank_phi.device)
    dyn = torch.full((1,), -1, dtype=torch.int64, device=st.bank_phi.device)

    def launch(i):
        P.prsink_retrieve(lay, phis[i % 2], st.bank_phi, st.bank_src, st.bank_count, st.M,
                          -10, r, sc, cp, dyn, st.bank_kv, st.cache_kv, st.n_layers)

    ms = time_launches(launch, warmup, steps)
    if int(cp.item()) != 1:
        raise RuntimeError("the dynamic fill did not copy on the last call")
    peaks = _peaks()
    work = 2.0 * 2 * st.L_blk * st.cfg["n_heads"] * st.cfg["head_dim"] * 2 * st.n_layers
    rec = _summary(ms, work, "GB/s", peaks["hbm"], f"{peaks['source']} hbm_gbs")
    rec.update(layers=st.n_layers, bytes_per_call=int(work),
               note="one call = the retrieval kernel + the predicated copy of every layer")
    return rec


def kernel_records(st, args):
    """Sub-records of the one-GPU line: every kernel the benchmark spec's targets name, timed alone."""
    w, k = 3, 20
    rec = {"append_480x480": append_alone("480x480", w, 50),
           "dynfill_40_layers": dynfill_alone(st, w, 10),
           "attention_480x480_rotating": attention_alone("480x480", w, k),
           "attention_480x480_repeat": attention_alone("480x480", w, k, repeat=True)}
    for name in ("384x672", "384x672_r4", "672x384"):
        rec[f"attention_{name}"] = attention_alone(name, w, k)
        rec[f"attention_{name}_split"] = attention_alone(name, w, k, split=True)
    # hot against cold L2 at 13 heads (143 units: one wave of 148 SMs): 105 MB of Q/K/V stay
    # resident when repeated; three alternating sets (315 MB) do not
    rec["attention_480x480_13heads_hot_l2"] = attention_alone("480x480", w, k, repeat=True,
                                                              heads=13)
    rec["attention_480x480_13heads_cold_l2"] = attention_alone("480x480", w, k, nbuf=3, heads=13)
    rec["attention_fused_480x480"], rec["rotate_ring_slots_480x480"] = fused_alone("480x480", w, k)
    for name in ("384x672", "384x672_r4", "672x384"):
        rec[f"attention_fused_{name}_split"] = fused_alone(name, w, k, split=True)[0]
    rec["note"] = ("attention: burst bf16 peak (a kernel timed alone); 'rotating' alternates "
                   "two input sets of 322 MB, 'repeat' reuses one (K/V of 295 MB exceed the "
                   "126 MB L2 either way); the 13-head pair compares L2-resident inputs (hot) "
                   "with three alternating sets (cold)")
    return rec


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------

def _inputs(args, cfg_full, rank, world, dev):
    """Per-pass Q/K/V pool, ref K/V per layer and poses of this rank.  With the head partition
    every rank draws the whole job's inputs (same seeds) and keeps its heads; replicas draw
    their own."""
    import synth
    from pose_retrieved_kv_b200 import shard

    split = args.partition == "heads" and world > 1
    seed0 = 0 if split else 1000 * rank
    H, d = cfg_full["n_heads"], cfg_full["head_dim"]
    lf = cfg_full["grid_h"] * cfg_full["grid_w"]
    lblk, lref = lf * cfg_full["frames_per_block"], lf * cfg_full["ref_frames"]

    def mine(x):
        return shard.shard_tokens(x, world, rank) if split else x

    qkv = [[mine(synth.normal_bf16((lblk, H, d), 100 + seed0 + i, j)).to(dev) for j in range(3)]
           for i in range(args.pool)]
    ref = [mine(synth.normal_bf16((lref, H, d), 7 + seed0 + layer, 1)).to(dev)
           for layer in range(args.layers)]
    return qkv, ref, 11 + (0 if split else rank)


def _block(st, P, b, kp_dev, ok_dev, qkv, out, events=None, stream=None):
    """One block of the stream: retrieval + dynamic fill, per layer 3 denoising passes and the
    Clean KV Update pass (append + attention), bank update.  Fused streams run each pass as one
    prsink_attention_fused launch (after the layer's once-per-block rotation pass).  ``events``
    collects the attention launch of every pass (the fused launch includes the append)."""
    import torch
    st.begin_block(kp_dev[b], ok_dev[b])
    i = 0
    pool = len(qkv)
    for layer in range(st.n_layers):
        st.prepare_layer(layer)
        for p in range(PASSES):
            q, kn, vn = qkv[(b * st.n_layers * PASSES + i) % pool]
            i += 1
            lay = st.layout()
            k, v = st.kv(layer)
            if not st.fused:
                P.prsink_kv_append(lay, kn, vn, k, v, P.SLOT_RING0 + st.b % st.R)
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            if st.fused:
                P.prsink_attention_fused(lay, q, kn, vn, st.k_rot[layer], k, v, out, None,
                                         st.dyn_src, scratch=st.scratch)
            elif st.scratch is not None:
                P.prsink_attention_split(lay, q, k, v, out, st.scratch, None, st.dyn_src)
            else:
                P.prsink_attention(lay, q, k, v, out, None, st.dyn_src)
            if events is not None:
                e1.record(stream)
                events.append((e0, e1))
            if p == PASSES - 1 and st.b == 0:
                P.prsink_kv_append(lay, kn, vn, k, v, P.SLOT_STATIC)
                if st.fused:
                    st.mark_written(layer, P.SLOT_STATIC)
    st.end_block()


def step_record(cfg, fused: bool, qkv, ref, kp_dev, ok_dev, dev, steps: int = 5,
                warmup: int = 3):
    """The per-block step on a stream of its own with the given path (fused: one
    prsink_attention_fused launch per pass after a rotation pass per layer and block; unfused:
    append + prsink_attention), timed in the steady state after the bank was filled."""
    import torch

    import pose_retrieved_kv_b200 as P

    n_layers = len(ref)
    st = P.PRSinkStream(cfg, n_layers=n_layers, M=M_BANK, write_blocks=WRITE_BLOCKS, device=dev,
                        fused=fused)
    for layer in range(n_layers):
        st.set_ref(layer, ref[layer], ref[layer])
    lblk, T, H, d = st.L_blk, st.T, cfg["n_heads"], cfg["head_dim"]
    out = torch.empty((lblk, H, d), dtype=torch.bfloat16, device=dev)
    for b in range(WRITE_BLOCKS + warmup):
        _block(st, P, b, kp_dev, ok_dev, qkv, out)
    ev = []
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(steps):
        _block(st, P, WRITE_BLOCKS + warmup + k, kp_dev, ok_dev, qkv, out, ev)
    t1.record()
    torch.cuda.synchronize()
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout")
    ms = t0.elapsed_time(t1) / steps
    attn = statistics.mean(a.elapsed_time(b) for a, b in ev)
    tf = 4.0 * lblk * T * d * H / (attn / 1e3) / 1e12
    peaks = _peaks()
    del st
    torch.cuda.empty_cache()
    return {"path": "fused" if fused else "unfused", "ms_per_step": round(ms, 3),
            "layer_blocks_per_s": round(n_layers * 1e3 / ms, 3),
            "attention_avg_ms": round(attn, 4), "attention_tflops": round(tf, 1),
            "frac_of_bf16_sustained": round(tf / peaks["bf16_sustained"], 4),
            "note": "fused: the timed launch includes the append; the rotation pass (once per "
                    "layer and block) is in ms_per_step only"}


def run_stream(st, P, kp_dev, ok_dev, qkv, out, n_blocks, dev):
    """A whole stream from block 0 (bank written during the first blocks, then frozen),
    timed on the device with the inputs resident; counts the dynamic fills and bank writes on
    the device."""
    import torch
    st.reset()
    fills = torch.zeros(1, dtype=torch.int32, device=dev)
    writes = torch.zeros(1, dtype=torch.int32, device=dev)
    n0 = P.prsink_launch_count()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for b in range(n_blocks):
        _block(st, P, b, kp_dev, ok_dev, qkv, out)
        fills += st.copied
        writes += (st.action >= 0).to(torch.int32)
    t1.record()
    torch.cuda.synchronize()
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout in the stream")
    s = t0.elapsed_time(t1) / 1e3
    return {"blocks": n_blocks, "layers": st.n_layers, "seconds": round(s, 3),
            "blocks_per_s": round(n_blocks / s, 3),
            "layer_blocks_per_s": round(n_blocks * st.n_layers / s, 3),
            "dynamic_fills": int(fills.item()), "bank_writes": int(writes.item()),
            "gpu_launches": int(P.prsink_launch_count() - n0),
            "inputs": "resident in HBM; poses from 12 recurring clusters (sigma 0.03), 5 % "
                      "failed frames; bank M = 5 written during the first 20 blocks"}


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import pose_retrieved_kv_b200 as P
    import synth
    from pose_retrieved_kv_b200 import shard

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream_only = args.config == "stream300"
    cfg_full = synth.preset("480x480" if stream_only else args.config)
    split = args.partition == "heads" and world > 1
    cfg = shard.shard_config(cfg_full, world, rank) if split else cfg_full
    n_layers = args.layers
    H, d = cfg["n_heads"], cfg["head_dim"]
    st = P.PRSinkStream(cfg, n_layers=n_layers, M=M_BANK, write_blocks=WRITE_BLOCKS, device=dev,
                        fused=args.path == "fused")
    lblk, T = st.L_blk, st.T
    qkv, ref, pose_seed = _inputs(args, cfg_full, rank, world, dev)
    for layer in range(n_layers):
        st.set_ref(layer, ref[layer], ref[layer])
    n_blocks = max(WRITE_BLOCKS + args.warmup + args.steps + 2, args.stream_blocks)
    kp_all, ok_all, _ = synth.pose_stream(pose_seed, n_blocks)
    kp_dev = torch.from_numpy(np.ascontiguousarray(kp_all[:, :, :62, :])).to(dev)
    ok_dev = torch.from_numpy(ok_all).to(dev)
    out = torch.empty((lblk, H, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    streams = 1 if split else world             # independent streams in the job

    if stream_only:
        if world > 1:
            dist.barrier()
        rec = run_stream(st, P, kp_dev, ok_dev, qkv, out, args.stream_blocks, dev)
        s = max_over_ranks(rec["seconds"], dev, world)
        if rank != 0:
            return None
        return {"metric": METRIC, "value": round(n_layers * args.stream_blocks * streams / s, 3),
                "unit": UNIT, "n_gpus": world, "steps": args.stream_blocks, "warmup": 0,
                "ms_per_step": round(1e3 * s / args.stream_blocks, 3), "higher_is_better": True,
                "scaling": "strong" if split else "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "gpu_launches": rec["gpu_launches"],
                "config": {"workload": f"{args.stream_blocks}-block stream at 480x480 from "
                                       "block 0, 40 layers x 4 passes per block",
                           "parallelism": _parallelism(args, world)},
                "stream": rec}

    attn_events = []
    for b in range(WRITE_BLOCKS + args.warmup):          # bank fill + warm-up, untimed
        _block(st, P, b, kp_dev, ok_dev, qkv, out)
    torch.cuda.synchronize()
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout during warm-up")

    clocks = ClockSampler(local_rank)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = P.prsink_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        _block(st, P, WRITE_BLOCKS + args.warmup + k, kp_dev, ok_dev, qkv, out, attn_events,
               stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = P.prsink_launch_count() - n0
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout in the timed region")
    attn_ms = [a.elapsed_time(b) for a, b in attn_events]
    ms = max_over_ranks(ms, dev, world)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, st, qkv, kp_all, ok_all, dev, world, streams)
    extras = stream_rec = None
    if world == 1 and not args.no_extras:
        extras = kernel_records(st, args)
        extras["step_other_path"] = step_record(cfg, args.path != "fused", qkv, ref, kp_dev,
                                                ok_dev, dev)
        stream_rec = run_stream(st, P, kp_dev, ok_dev, qkv, out, args.stream_blocks, dev)

    if rank != 0:
        return None
    peaks = _peaks()
    prof = FUSED_PROFILE if args.path == "fused" else ATTN_PROFILE
    value = job_throughput(n_layers, args.steps, streams, ms / 1e3)
    flops = 4.0 * lblk * T * d * H                      # QK^T + PV, steady state: all keys valid
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = flops / (attn_avg_ms / 1e3) / 1e12
    peak = peaks["bf16_sustained"]
    res = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3),
        "higher_is_better": True, "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (N(0,1) bf16 Q/K/V, clustered synthetic poses; no weights needed)",
        "config": {"workload": _workload(args.config, n_layers),
                   "path": args.path,
                   "heads": cfg_full["n_heads"], "heads_per_gpu": H, "head_dim": d,
                   "queries": lblk, "keys": T, "ring_slots": cfg["ring_slots"],
                   "layers": n_layers, "bank": M_BANK,
                   "l2": "inputs larger than L2 (295 MB cache per layer, layers cycled)",
                   "parallelism": _parallelism(args, world)},
        "attention": {"avg_ms": round(attn_avg_ms, 4), "tflops": round(achieved, 1),
                      "frac_of_bf16_peak": round(achieved / peak, 4),
                      "launches_timed": len(attn_ms), "rank": 0},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": (_profiled_traffic(ATTN_SRC, prof)
                                 if args.config == "480x480" and H == 40 else None),
                     "traffic_source": f"{prof}: ncu dram__bytes_read.sum + "
                                       "dram__bytes_write.sum, bytes per launch",
                     "kernel": ("prsink_attention_kernel (fused: the pass's append included)"
                                if args.path == "fused" else "prsink_attention_kernel"),
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if e2e is not None:
        res["e2e"] = e2e
    if extras is not None:
        res["kernels"] = extras
    if stream_rec is not None:
        res["stream300"] = stream_rec
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(args, cfg)
    return res


def _workload(config: str, n_layers: int) -> str:
    return (f"per-block step {config}: {n_layers} layers x ({PASSES - 1} denoise + 1 clean) x "
            "(append + PR-Sink attention), retrieval + dynamic fill, bank update")


def _parallelism(args, world):
    if world == 1:
        return "single GPU"
    if args.partition == "heads":
        return f"heads split over {world} GPUs (one stream; pose decisions replicated)"
    return f"replica x{world} (independent streams)"


def run_kernel_only(args, local_rank: int):
    """Time one kernel alone (``--only attention|append|dynfill``) at the workload's sizes
    (for profiling: one process, few launches)."""
    import torch

    import pose_retrieved_kv_b200 as P
    import synth

    torch.cuda.set_device(local_rank)
    if args.only == "attention":
        rec = attention_alone(args.config, args.warmup, args.steps)
        rec["traffic"] = (_profiled_traffic(ATTN_SRC, ATTN_PROFILE)
                          if args.config == "480x480" else None)
    elif args.only == "split":
        rec = attention_alone(args.config, args.warmup, args.steps, split=True)
    elif args.only in ("fused", "rotate"):
        fused, rot = fused_alone(args.config, args.warmup, args.steps)
        rec = fused if args.only == "fused" else rot
        if args.only == "fused":
            rec["traffic"] = (_profiled_traffic(ATTN_SRC, FUSED_PROFILE)
                              if args.config == "480x480" else None)
    elif args.only == "append":
        rec = append_alone(args.config, args.warmup, args.steps)
        rec["traffic"] = (_profiled_traffic(APPEND_SRC, APPEND_PROFILE)
                          if args.config == "480x480" else None)
    else:
        cfg = synth.preset(args.config)
        st = P.PRSinkStream(cfg, n_layers=args.layers, M=M_BANK, write_blocks=WRITE_BLOCKS,
                            device=torch.device("cuda", local_rank))
        g = torch.Generator().manual_seed(11)
        st.bank_phi.copy_(torch.nn.functional.normalize(
            torch.randn(M_BANK, P.FP_DIM, generator=g, dtype=torch.float64), dim=1).float())
        st.bank_src.copy_(torch.arange(M_BANK))
        st.bank_count.fill_(M_BANK)
        st.bank_kv.view(-1)[::4099] = 1.0
        rec = dynfill_alone(st, args.warmup, args.steps)
    return {"kernel": args.only, "config": args.config, **rec}


def run_e2e(args, st, qkv, kp_all, ok_all, dev, world, streams):
    """Same step through the public API with pinned HOST inputs and outputs: every step copies
    its poses and per-pass Q/K/V from the host and reads every attention output back.  Copies
    run on their own streams, overlapped with compute through double buffering.  Timed with
    CUDA events from the first copy to the last read-back, max over ranks."""
    import torch
    import torch.distributed as dist

    import pose_retrieved_kv_b200 as P

    n_layers, pool = st.n_layers, len(qkv)
    lblk = st.L_blk
    H, d = st.cfg["n_heads"], st.cfg["head_dim"]
    host_in = [[t.cpu().pin_memory() for t in s] for s in qkv]
    host_out = [torch.empty((lblk, H, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    kp_h = torch.from_numpy(np.ascontiguousarray(kp_all[:, :, :62, :])).pin_memory()
    ok_h = torch.from_numpy(ok_all).pin_memory()
    stage = [[torch.empty((lblk, H, d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
             for _ in range(2)]
    outs = [torch.empty((lblk, H, d), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    kp_d = torch.empty((3, 62, 3), dtype=torch.float32, device=dev)
    ok_d = torch.empty(3, dtype=torch.uint8, device=dev)
    comp = torch.cuda.current_stream(dev)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]
    for e in in_free + out_free:
        e.record(comp)
    bytes_in = bytes_out = 0
    first = WRITE_BLOCKS + args.warmup + args.steps
    n_blocks = kp_all.shape[0]

    def block(b):
        nonlocal bytes_in, bytes_out
        bb = b % n_blocks
        with torch.cuda.stream(h2d):
            kp_d.copy_(kp_h[bb], non_blocking=True)
            ok_d.copy_(ok_h[bb], non_blocking=True)
        comp.wait_stream(h2d)
        bytes_in += kp_d.numel() * 4 + 3
        st.begin_block(kp_d, ok_d)
        i = 0
        for layer in range(n_layers):
            for p in range(PASSES):
                j = i & 1
                src = host_in[(b * n_layers * PASSES + i) % pool]
                h2d.wait_event(in_free[j])
                with torch.cuda.stream(h2d):
                    for t, h in zip(stage[j], src):
                        t.copy_(h, non_blocking=True)
                    in_ready[j].record(h2d)
                bytes_in += 3 * lblk * H * d * 2
                comp.wait_event(in_ready[j])
                comp.wait_event(out_free[j])
                q, kn, vn = stage[j]
                st.layer_pass(layer, q, kn, vn, outs[j], clean=(p == PASSES - 1))
                in_free[j].record(comp)
                out_ready[j].record(comp)
                d2h.wait_event(out_ready[j])
                with torch.cuda.stream(d2h):
                    host_out[j].copy_(outs[j], non_blocking=True)
                    out_free[j].record(d2h)
                bytes_out += lblk * H * d * 2
                i += 1
        st.end_block()

    for k in range(2):
        block(first + k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    bytes_in = bytes_out = 0
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    h2d.wait_event(t0)
    for k in range(args.steps):
        block(first + 2 + k)
    comp.wait_stream(h2d)
    comp.wait_stream(d2h)
    t1.record(comp)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    el = max_over_ranks(t0.elapsed_time(t1) / 1e3, dev, world)
    if P.prsink_sync_status() != P.PRSINK_OK:
        raise RuntimeError("device status reported a timeout in the e2e run")
    return {"value": round(job_throughput(n_layers, args.steps, streams, el), 3), "unit": UNIT,
            "h2d_bytes_per_step": bytes_in // args.steps,
            "d2h_bytes_per_step": bytes_out // args.steps}


# ------------------------------------------------------------------------------------------
# CPU oracle (baseline only)
# ------------------------------------------------------------------------------------------

def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample_seconds_per_layer_block(cfg, heads: int, seed: int = 0):
    """Time the oracle on ``heads`` heads of one attention pass plus one append, and scale to
    one layer-block (all heads, 4 passes)."""
    import oracle
    import synth

    s = oracle.layout_sizes(cfg)
    H, d = cfg["n_heads"], cfg["head_dim"]
    sub = dict(cfg, n_heads=heads, block_index=1000, valid_mask=0xFF)
    q = synth.normal_bf16((s["L_blk"], heads, d), seed, 0).double().numpy()
    k = synth.normal_bf16((heads, s["T"], d), seed, 1).double().numpy()
    v = synth.normal_bf16((heads, s["T"], d), seed, 2).double().numpy()
    kn = synth.normal_bf16((s["L_blk"], heads, d), seed, 3).double().numpy()
    t0 = time.perf_counter()
    k2, v2 = oracle.kv_append(sub, kn, kn, k, v, oracle.SLOT_RING0)
    oracle.attention(sub, q, k2, v2)
    el = time.perf_counter() - t0
    return el * (H / heads) * PASSES, el


def cpu_baseline(args, cfg):
    heads = args.baseline_heads
    per_lb, el = oracle_sample_seconds_per_layer_block(cfg, heads)
    return {"value": round(1.0 / per_lb, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"{heads} of {cfg['n_heads']} heads, 1 pass (append + attention, all "
                      f"{oracle_rows(cfg)} queries x {oracle_keys(cfg)} keys) in {el:.1f} s, "
                      f"scaled x{cfg['n_heads'] // heads} heads x{PASSES} passes"}


def oracle_rows(cfg):
    return cfg["frames_per_block"] * cfg["grid_h"] * cfg["grid_w"]


def oracle_keys(cfg):
    lf = cfg["grid_h"] * cfg["grid_w"]
    return lf * cfg["ref_frames"] + (2 + cfg["ring_slots"]) * cfg["frames_per_block"] * lf


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import synth
    cfg = synth.preset(args.config)
    heads = args.cpu_heads
    for _ in range(args.warmup):
        oracle_sample_seconds_per_layer_block(cfg, 1)
    per = []
    t0 = time.perf_counter()
    for k in range(args.steps):
        per.append(oracle_sample_seconds_per_layer_block(cfg, heads, seed=k)[0])
    wall = time.perf_counter() - t0
    value = 1.0 / statistics.mean(per)
    cb = {"value": round(value, 6), "unit": UNIT, "cores": _cores(), "kind": "oracle",
          "sample": f"each step: {heads} of {cfg['n_heads']} heads, 1 pass, scaled to one "
                    f"layer-block (x{cfg['n_heads'] // heads} heads x{PASSES} passes)"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * wall / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (N(0,1) bf16 Q/K/V)",
            "config": {"workload": _workload(args.config, args.layers),
                       "parallelism": "cpu (float64 oracle, rank 0 only)",
                       "sampled": f"{heads} of {cfg['n_heads']} heads of one pass per step, "
                                  "scaled to the layer-block"},
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _launch_ranks(args) -> int:
    """Start ``--gpus`` processes through torch.distributed.run (one per GPU, rendezvous on
    127.0.0.1) running this script with the same arguments; returns their exit status."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="480x480",
                    choices=["480x480", "384x672", "384x672_r4", "672x384", "stream300"])
    ap.add_argument("--path", choices=["fused", "unfused"], default="fused",
                    help="fused: each pass is one prsink_attention_fused launch (append folded "
                         "in, sinks pre-rotated once per layer and block)")
    ap.add_argument("--partition", choices=["heads", "replicas"], default="heads",
                    help="N > 1: split the heads of one stream, or one stream per GPU")
    ap.add_argument("--layers", type=int, default=40)
    ap.add_argument("--pool", type=int, default=8)
    ap.add_argument("--stream-blocks", type=int, default=300)
    ap.add_argument("--cpu-heads", type=int, default=4,
                    help="heads per step of the CPU oracle in --impl reference")
    ap.add_argument("--baseline-heads", type=int, default=40,
                    help="heads of the CPU oracle sample in the cpu_baseline leg (~10-30 s)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the kernel sub-records and the 300-block stream")
    ap.add_argument("--only", choices=["attention", "append", "dynfill", "fused", "rotate",
                                       "split"], default=None,
                    help="time one kernel alone at the workload's sizes (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(_launch_ranks(args))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but the launcher started {world} "
                         "ranks\n")
        sys.exit(2)
    if args.only:
        if world > 1:
            ap.error("--only times one kernel on one GPU")
        res = run_kernel_only(args, local_rank)
    elif args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        import torch.distributed as dist
        if world > 1:
            import datetime
            import torch
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        try:
            res = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
