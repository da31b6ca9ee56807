"""Benchmark of the rolling-window attention layer hot path on B200.

One step = one pass of the layer's hot path on the paper-shaped denoise
workload: fused 3D-RoPE attention of 23,400 query tokens over 32,760 context
tokens (12 heads, d = 128, bf16; RoPE on Q and K inside the kernel) plus the
per-layer ring KV-cache update that inserts 5 frames (30x52 tokens, 12 heads)
into a 21-slot ring.  Inputs are seeded N(0,1) bf16 draws resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Under torchrun with N > 1 every rank runs an
independent replica of the same step (the path has no exchange step), the
timed region is bracketed by a barrier + synchronize and the max over ranks is
reported.  ``--impl reference`` times the CPU oracle on this host instead.

Besides the step, the line reports (each measured with CUDA events on the
launching stream): the attention call alone against the dense bf16 peak,
ring inserts in steady state (back-to-back inserts whose destinations exceed
the 126 MB L2), standalone RoPE, the rolling-cache and two-pass attention
variants, and the 30-layer rolling sweep (rotated insert + Q-only attention,
Lk 9,360 -> 32,760).

``--profile-case NAME`` runs only W + K launches of one call on the bench
workload, with no timing and no JSON (the command the ncu summaries under
profiles/ were captured with).
"""

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

METRIC = "fused-RoPE attention TFLOP/s @23.4k×32.8k (% bf16 peak); KV update GB/s"
H, D = 12, 128
GRID_H, GRID_W = 30, 52
F = GRID_H * GRID_W
LQ, LK = 15 * F, 21 * F
Q_T0, K_T0 = 6, 0
RING_SLOTS, RING_INSERT = 21, 5
ATTN_FLOPS = 4.0 * LQ * LK * D * H                 # QK^T and PV, visible pairs only (no mask)
RING_BYTES = 2 * 2 * RING_INSERT * F * H * D * 2    # (K and V) x (read + write)
ROPE_BYTES = 2 * (LQ + LK) * H * D * 2               # Q and K rows, read + write
SEED = 1002
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0


def workload_config(n_gpus):
    return {
        "workload": "denoise_30x52_h12_q23400_k32760 + ring_21x1560x12_insert5",
        "Lq": LQ, "Lk": LK, "heads": H, "head_dim": D, "frame_grid": [GRID_H, GRID_W],
        "rope": "3D t/h/w pairs 22/21/21 theta 1e4, fused on Q and K",
        "mask": "none", "ring": {"slots": RING_SLOTS, "insert_frames": RING_INSERT},
        "global_batch": n_gpus, "seq_len": LQ, "parallelism": f"replicas x{n_gpus}",
        "l2": "no flush: each step reads 273 MB of attention operands and moves 96 MB in the ring update, "
              "both above the 126 MB L2",
    }


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"bf16": j.get("bf16_tflops", 1590.0), "bf16_sustained": j.get("bf16_tflops_sustained", 1400.0),
                "hbm": j.get("hbm_gbs", 6650.0), "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
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
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def make_inputs(device):
    import torch
    from rolling_kv_cache_rope_b200.synth import bf16_normal_bits

    def dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)

    qb = bf16_normal_bits(SEED, (LQ, H, D))
    kb = bf16_normal_bits(SEED + 100, (LK, H, D))
    vb = bf16_normal_bits(SEED + 200, (LK, H, D))
    knb = bf16_normal_bits(SEED + 300, (RING_INSERT * F, H, D))
    vnb = bf16_normal_bits(SEED + 400, (RING_INSERT * F, H, D))
    host = {"q": qb, "k": kb, "v": vb, "k_new": knb, "v_new": vnb}
    devt = {k: dev(v) for k, v in host.items()}
    return host, devt


ORACLE_ROWS = 2048   # query rows of one head per oracle sample


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def cpu_baseline(host, head=0, rows=ORACLE_ROWS):
    """Time the float64 oracle on a bounded sample of the step's attention:
    ``rows`` query rows (evenly spaced over the 23,400) of one head over all
    32,760 keys, including the fp64 RoPE of that head's keys and of the rows.
    The oracle's cost per (query, key) pair does not depend on which head, so
    the rate stands for the whole call."""
    import oracle
    rows_idx = np.linspace(0, LQ - 1, rows).astype(np.int64)
    sl = slice(head, head + 1)
    t0 = time.perf_counter()
    oracle.fused_attention_ref(oracle.bf16_bits_to_f64(host["q"][:, sl]), oracle.bf16_bits_to_f64(host["k"][:, sl]),
                               oracle.bf16_bits_to_f64(host["v"][:, sl]), scale=1 / math.sqrt(D), grid_h=GRID_H,
                               grid_w=GRID_W, rope_q=True, rope_k=True, q_t0=Q_T0, k_t0=K_T0, rows=rows_idx)
    dt = time.perf_counter() - t0
    flops = 4.0 * rows * LK * D
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(oracle_threads()), "kind": "oracle",
            "sample": f"{rows} of {LQ} query rows of head {head} over all {LK} keys, incl. fp64 RoPE of that "
                      f"head's keys and rows; {dt:.2f} s"}


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, rank 0 only.  Each step
    is the cpu_baseline sample (2,048 query rows of one head over all keys,
    the head cycling with the step)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
    host = {"q": bf16_normal_bits(SEED, (LQ, H, D)), "k": bf16_normal_bits(SEED + 100, (LK, H, D)),
            "v": bf16_normal_bits(SEED + 200, (LK, H, D))}
    for i in range(args.warmup):
        cpu_baseline(host, head=i % H)
    t0 = time.perf_counter()
    vals = [cpu_baseline(host, head=i % H) for i in range(args.steps)]
    dt = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = value
    cb["sample"] = (f"per step {ORACLE_ROWS} of {LQ} query rows of one head (cycling over the {H} heads) over all "
                    f"{LK} keys, incl. fp64 RoPE of that head's keys and rows")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.gpus), "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))
    return 0


def max_over_ranks(ms, world, device):
    """The largest of the ranks' device-timed milliseconds (every rank calls
    this at the same point; world == 1 returns ms unchanged)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    tt = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def ring_steady_state(rkv, ring, rope, srcs, rotated, device, reps=5):
    """Back-to-back inserts whose destinations exceed L2: 4 inserts of 5
    frames into 20 distinct slots of the 21-slot ring (383 MB written, 192 MB
    read from 4 distinct source sets), after a 512 MB write that evicts the
    previous group from L2.  Returns the mean time of one insert in ms."""
    import torch
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    times = []
    for rep in range(reps + 1):
        ring.c.head, ring.c.count = 0, 0
        flush.fill_(rep & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i, (k_new, v_new) in enumerate(srcs):
            if rotated:
                rkv.kvcache_ring_update_rope(ring, k_new, v_new, 1 + RING_INSERT * i, rope, RING_INSERT)
            else:
                rkv.kvcache_ring_update(ring, k_new, v_new, RING_INSERT)
        e1.record(stream)
        torch.cuda.synchronize()
        if rep > 0:                       # the first group warms up
            times.append(e0.elapsed_time(e1) / len(srcs))
    rkv.rkv_ring_status()
    del flush
    return statistics.mean(times)


def copy_steady_state(srcs, device, reps=5):
    """Context for the ring inserts' HBM fraction: torch's own device copy of
    the same bytes, timed the same way (four back-to-back copies of 5 frames
    of K and V into distinct buffers after a 512 MB L2 flush).  Returns the
    mean time of one (K + V) copy in ms."""
    import torch
    stream = torch.cuda.current_stream()
    dsts = [(torch.empty_like(k), torch.empty_like(v)) for k, v in srcs]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    times = []
    for rep in range(reps + 1):
        flush.fill_(rep & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for (k, v), (kd, vd) in zip(srcs, dsts):
            kd.copy_(k)
            vd.copy_(v)
        e1.record(stream)
        torch.cuda.synchronize()
        if rep > 0:
            times.append(e0.elapsed_time(e1) / len(srcs))
    del flush, dsts
    return statistics.mean(times)


SWEEP_LAYERS, SWEEP_STEPS = 30, 8


def sweep_bench(rkv, rope, device, ws):
    """The rolling sweep of the pages' window: 30 layers, each with its own
    21-slot ring (one frame seeded), 8 window steps; per step and layer one
    rotated insert of 5 frames and one attention call of the 23,400-token
    query window over the ring's valid frames (K already rotated, Q rotated in
    the kernel, no mask; Lk = 6, 11, 16, 21, 21, 21, 21, 21 frames).  Inputs
    of each step are seeded N(0,1) draws made on the device (shared by the
    layers).  Returns a dict of measured figures."""
    import torch
    stream = torch.cuda.current_stream()
    rings = [rkv.KVRing(RING_SLOTS, F, H, D, device=device) for _ in range(SWEEP_LAYERS)]
    inputs = []
    for st in range(SWEEP_STEPS + 1):
        gen = torch.Generator(device=device).manual_seed(4000 + st)
        n = 1 if st == 0 else RING_INSERT
        q = None if st == 0 else torch.randn((LQ, H, D), generator=gen, device=device).to(torch.bfloat16)
        k = torch.randn((n * F, H, D), generator=gen, device=device).to(torch.bfloat16)
        v = torch.randn((n * F, H, D), generator=gen, device=device).to(torch.bfloat16)
        inputs.append((q, k, v))
    o = torch.empty((LQ, H, D), dtype=torch.bfloat16, device=device)

    def run(evs=None):
        for r in rings:
            r.c.head, r.c.count = 0, 0
            rkv.kvcache_ring_update_rope(r, inputs[0][1], inputs[0][2], 0, rope, 1)
        lk = []
        for st in range(SWEEP_STEPS):
            q, k_new, v_new = inputs[st + 1]
            t_new = 1 + RING_INSERT * st
            for li, r in enumerate(rings):
                if evs is not None:
                    evs[st][li][0].record(stream)
                rkv.kvcache_ring_update_rope(r, k_new, v_new, t_new, rope, RING_INSERT)
                if evs is not None:
                    evs[st][li][1].record(stream)
                Lk = r.count * F
                seq = rkv.AttnSeq(q, r.k.view(-1, H, D)[:Lk], r.v.view(-1, H, D)[:Lk], o, q_t0=t_new, rope_k=False)
                rkv.attn_fwd_varlen([seq], rope, workspace=ws)
                if evs is not None:
                    evs[st][li][2].record(stream)
            lk.append(rings[0].count)
        return lk

    run()                                  # warm-up pass (rings start empty again below)
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(SWEEP_LAYERS)]
           for _ in range(SWEEP_STEPS)]
    # seeding the rings is not part of a window step: time from the first insert
    lk = run(evs)
    torch.cuda.synchronize()
    total = evs[0][0][0].elapsed_time(evs[-1][-1][2])
    rkv.rkv_attn_status(ws)
    rkv.rkv_ring_status()
    ins = [evs[s][li][0].elapsed_time(evs[s][li][1]) for s in range(SWEEP_STEPS) for li in range(SWEEP_LAYERS)]
    att = [evs[s][li][1].elapsed_time(evs[s][li][2]) for s in range(SWEEP_STEPS) for li in range(SWEEP_LAYERS)]
    flops = sum(4.0 * LQ * c * F * D * H for c in lk) * SWEEP_LAYERS
    ins_bytes = RING_BYTES * SWEEP_LAYERS * SWEEP_STEPS
    del rings, inputs, o
    return {
        "workload": "rolling_sweep_30layers_8steps: ring 21x1560x12x128 per layer, insert 5 roped frames, "
                    "attention q23400 over k9360..32760 (Q-only RoPE)",
        "ms_per_window_step": total / SWEEP_STEPS, "ms_total": total, "lk_frames": lk,
        "insert_rope": {"value": ins_bytes / (sum(ins) * 1e-3) / 1e9, "unit": "GB/s",
                        "avg_us": statistics.mean(ins) * 1e3, "calls": len(ins)},
        "attention": {"value": flops / (sum(att) * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "avg_ms": statistics.mean(att), "calls": len(att), "flops": flops},
        "launches": SWEEP_LAYERS * SWEEP_STEPS * 3,   # rotated insert, attention, merge of split tail units
    }


def sweep_cpu_baseline(host):
    """The oracle on a sample of the sweep: one rotated 5-frame insert into a
    21-slot oracle ring (fp64 RoPE of the keys, bf16 rounding, copy), in GB/s
    of the insert's algorithmic bytes."""
    import oracle
    ring = oracle.RingRef(RING_SLOTS)
    kb = host["k_new"]
    vb = host["v_new"]
    t0 = time.perf_counter()
    kr = oracle.f64_to_bf16_bits(oracle.rope3d_ref(oracle.bf16_bits_to_f64(kb), 1, GRID_H, GRID_W))
    ring.insert([(kr[i * F:(i + 1) * F], vb[i * F:(i + 1) * F], 1 + i) for i in range(RING_INSERT)])
    dt = time.perf_counter() - t0
    return {"value": RING_BYTES / dt / 1e9, "unit": "GB/s", "cores": int(oracle_threads()), "kind": "oracle",
            "sample": f"one rotated insert of {RING_INSERT} frames into a {RING_SLOTS}-slot oracle ring; {dt:.2f} s"}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from rolling_kv_cache_rope_b200 import rkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=device, timeout=__import__("datetime").timedelta(seconds=120))

    host, t = make_inputs(device)
    rope = rkv.make_rope(GRID_H, GRID_W)
    o = torch.empty((LQ, H, D), dtype=torch.bfloat16, device=device)
    ring = rkv.KVRing(RING_SLOTS, F, H, D, device=device)
    ws = torch.zeros(rkv.attn_fwd_varlen_workspace_size(1, H, D), dtype=torch.uint8, device=device)
    seq = rkv.AttnSeq(t["q"], t["k"], t["v"], o, q_t0=Q_T0, k_t0=K_T0)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rkv.attn_fwd_varlen([seq], rope, workspace=ws)
        if ev is not None:
            ev[1].record(stream)
        rkv.kvcache_ring_update(ring, t["k_new"], t["v_new"], RING_INSERT)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    rkv.rkv_attn_status(ws)
    total_ms = start.elapsed_time(end)
    attn_ms = [e[0].elapsed_time(e[1]) for e in evs]
    ring_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = max_over_ranks(total_ms, world, device)

    # end to end through the public API with host buffers: every step copies
    # its inputs (Q, K, V, new K/V frames) from pinned host memory, runs the
    # two calls and copies O back.  Steps are pipelined the way a serving loop
    # would run them: two device buffer sets, uploads on a copy stream and
    # downloads on another, so step i's copies overlap step i-1's kernels.
    pinned = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory() for k, v in host.items()}
    o_host = [torch.empty((LQ, H, D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    sets = [t, {k: torch.empty_like(v) for k, v in t.items()}]
    outs = [o, torch.empty_like(o)]
    seqs = [seq, rkv.AttnSeq(sets[1]["q"], sets[1]["k"], sets[1]["v"], outs[1], q_t0=Q_T0, k_t0=K_T0)]
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "comp", "d2h")}
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_run(n_steps, start_ev=None, end_ev=None):
        if start_ev is not None:
            start_ev.record(stream)
            up.wait_event(start_ev)
            down.wait_event(start_ev)
        for i in range(n_steps):
            b = i % 2
            if i >= 2:
                up.wait_event(ev["comp"][b])           # the kernels of step i-2 have read set b
            with torch.cuda.stream(up):
                for k in ("q", "k", "v", "k_new", "v_new"):
                    sets[b][k].copy_(pinned[k], non_blocking=True)
                ev["h2d"][b].record(up)
            stream.wait_event(ev["h2d"][b])
            if i >= 2:
                stream.wait_event(ev["d2h"][b])         # O of step i-2 has left the device
            rkv.attn_fwd_varlen([seqs[b]], rope, workspace=ws)
            rkv.kvcache_ring_update(ring, sets[b]["k_new"], sets[b]["v_new"], RING_INSERT)
            ev["comp"][b].record(stream)
            down.wait_event(ev["comp"][b])
            with torch.cuda.stream(down):
                o_host[b].copy_(outs[b], non_blocking=True)
                ev["d2h"][b].record(down)
        for b in range(min(2, n_steps)):
            stream.wait_event(ev["d2h"][b])
        if end_ev is not None:
            end_ev.record(stream)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    if world > 1:
        dist.barrier()
    h2d = sum(v.nbytes for v in host.values())
    d2h = LQ * H * D * 2
    del sets[1], outs[1], seqs[1]

    # standalone 3D-RoPE of the step's Q and K (out of place); 345 MB per call
    # pair, above the L2, so no flush is needed between calls
    yq, yk = torch.empty_like(t["q"]), torch.empty_like(t["k"])
    for _ in range(3):
        rkv.rope3d_apply(t["q"], yq, t0=Q_T0, rope=rope)
        rkv.rope3d_apply(t["k"], yk, t0=K_T0, rope=rope)
    rope_iters = 20
    rope_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(rope_iters)]
    torch.cuda.synchronize()
    for i in range(rope_iters):
        rope_ev[i][0].record(stream)
        rkv.rope3d_apply(t["q"], yq, t0=Q_T0, rope=rope)
        rkv.rope3d_apply(t["k"], yk, t0=K_T0, rope=rope)
        rope_ev[i][1].record(stream)
    torch.cuda.synchronize()
    rope_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in rope_ev)
    # the same Q and K in one rope3d_apply_batch call (one launch)
    pair = [(t["q"], yq, Q_T0), (t["k"], yk, K_T0)]
    for _ in range(3):
        rkv.rope3d_apply_batch(pair, rope=rope)
    torch.cuda.synchronize()
    for i in range(rope_iters):
        rope_ev[i][0].record(stream)
        rkv.rope3d_apply_batch(pair, rope=rope)
        rope_ev[i][1].record(stream)
    torch.cuda.synchronize()
    rope_batch_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in rope_ev)
    del yq, yk, pair

    # ring inserts in steady state (destinations above L2), plain and rotated
    gen = torch.Generator(device=device).manual_seed(SEED + 500)
    srcs = [(torch.randn((RING_INSERT * F, H, D), generator=gen, device=device).to(torch.bfloat16),
             torch.randn((RING_INSERT * F, H, D), generator=gen, device=device).to(torch.bfloat16))
            for _ in range(4)]
    ring_plain_ms = ring_steady_state(rkv, ring, rope, srcs, False, device)
    ring_rope_ms = ring_steady_state(rkv, ring, rope, srcs, True, device)
    copy_ms = copy_steady_state(srcs, device)
    del srcs

    def time_attn(seqs_, rope_=rope, iters=5):
        for _ in range(3):
            rkv.attn_fwd_varlen(seqs_, rope_, workspace=ws)
        evs_ = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
        torch.cuda.synchronize()
        for i in range(iters):
            evs_[i][0].record(stream)
            rkv.attn_fwd_varlen(seqs_, rope_, workspace=ws)
            evs_[i][1].record(stream)
        torch.cuda.synchronize()
        rkv.rkv_attn_status(ws)
        return statistics.mean(e[0].elapsed_time(e[1]) for e in evs_)

    # the rolling-cache pass: keys already rotated (as the rotated ring insert
    # stores them), only Q rotated in-kernel, same sizes as the step
    seq_qonly = rkv.AttnSeq(t["q"], t["k"], t["v"], o, q_t0=Q_T0, k_t0=K_T0, rope_k=False)
    qonly_ms = time_attn([seq_qonly])
    # the batched two-pass launch: the denoise pass and a 5-frame cache-update
    # pass over the same 21-frame context, both frame-block-causal (blocks of
    # 3 frames, query frames bottom-right aligned); FLOPs of visible pairs only
    q_cache = torch.randn((5 * F, H, D), generator=gen, device=device).to(torch.bfloat16)
    o_cache = torch.empty_like(q_cache)
    two_pass = [rkv.AttnSeq(t["q"], t["k"], t["v"], o, q_t0=Q_T0, k_t0=K_T0, block_frames=3,
                            q_frame_offset=LK // F - LQ // F),
                 rkv.AttnSeq(q_cache, t["k"], t["v"], o_cache, q_t0=16, k_t0=K_T0, block_frames=3,
                             q_frame_offset=16)]

    def visible_pairs(q_frames, off, k_frames, block=3):
        return sum(F * F for qf in range(q_frames) for kf in range(k_frames) if kf // block <= (off + qf) // block)

    two_pass_flops = 4.0 * D * H * (visible_pairs(LQ // F, LK // F - LQ // F, LK // F) + visible_pairs(5, 16, LK // F))
    two_pass_ms = time_attn(two_pass)
    del q_cache, o_cache, two_pass

    # the other RoPE reading: rotate-half pairs
    rope_half = rkv.make_rope(GRID_H, GRID_W, layout="half")
    half_attn_ms = time_attn([rkv.AttnSeq(t["q"], t["k"], t["v"], o, q_t0=Q_T0, k_t0=K_T0)], rope_half)
    yq, yk = torch.empty_like(t["q"]), torch.empty_like(t["k"])
    hv = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(5)]
    for i in range(5):
        hv[i][0].record(stream)
        rkv.rope3d_apply(t["q"], yq, t0=Q_T0, rope=rope_half)
        rkv.rope3d_apply(t["k"], yk, t0=K_T0, rope=rope_half)
        hv[i][1].record(stream)
    torch.cuda.synchronize()
    half_rope_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in hv[1:])
    del yq, yk

    sweep = sweep_bench(rkv, rope, device, ws) if not args.no_sweep else None

    # kernels per step: attention, the merge of split tail units when the
    # persistent grid's last wave is at most half full (same rule as the
    # library, one CTA pair per two SMs), and the ring update
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    clusters, units = sms // 2, -(-LQ // 512) * H
    rest = units % clusters
    split = units > clusters and rest > 0 and 2 * rest <= clusters and ws.numel() > 256
    launches_per_step = 3 if split else 2

    if rank == 0:
        peaks = measured_peaks()
        ms_per_step = total_ms / args.steps
        value = world * ATTN_FLOPS / (ms_per_step * 1e-3) / 1e12
        attn_avg = statistics.mean(attn_ms)
        ring_avg = statistics.mean(ring_ms)
        achieved = ATTN_FLOPS / (attn_avg * 1e-3) / 1e12

        def gbs(ms):
            return RING_BYTES / (ms * 1e-3) / 1e9

        traffic = load_traffic()
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(world),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16"], "traffic": traffic,
                         "peak_kind": f"bf16 dense cuBLAS burst ({peaks['source']}): the attention call is timed "
                                      f"on its own for {attn_avg * args.steps:.0f} ms in total",
                         "frac_of_nominal_2250": achieved / NOMINAL_BF16_TFLOPS,
                         "frac_of_sustained": achieved / peaks["bf16_sustained"],
                         "kernel": "attn_fwd_kernel (+ attn_combine_kernel)", "avg_ms": attn_avg,
                         "flops_per_launch": ATTN_FLOPS,
                         "algorithmic_bytes_per_launch": (2 * LQ + 2 * LK) * H * D * 2},
            "kv_update": {"value": gbs(ring_avg), "unit": "GB/s", "avg_us": ring_avg * 1e3,
                          "bytes_per_call": RING_BYTES, "frac_of_measured_hbm": gbs(ring_avg) / peaks["hbm"],
                          "frac_of_nominal_8000": gbs(ring_avg) / NOMINAL_HBM_GBS,
                          "what": "kvcache_ring_update in the step (after the attention call, no flush)"},
            "kv_update_steady": {"value": gbs(ring_plain_ms), "unit": "GB/s", "avg_us": ring_plain_ms * 1e3,
                                 "frac_of_measured_hbm": gbs(ring_plain_ms) / peaks["hbm"],
                                 "frac_of_nominal_8000": gbs(ring_plain_ms) / NOMINAL_HBM_GBS,
                                 "frac_of_same_size_copy": copy_ms / ring_plain_ms,
                                 "what": "kvcache_ring_update: 4 back-to-back inserts of 5 frames into 20 distinct "
                                         "slots (383 MB written, above L2), after a 512 MB L2 flush; per insert"},
            "kv_update_rope": {"value": gbs(ring_rope_ms), "unit": "GB/s", "avg_us": ring_rope_ms * 1e3,
                               "bytes_per_call": RING_BYTES,
                               "frac_of_measured_hbm": gbs(ring_rope_ms) / peaks["hbm"],
                               "frac_of_nominal_8000": gbs(ring_rope_ms) / NOMINAL_HBM_GBS,
                               "frac_of_same_size_copy": copy_ms / ring_rope_ms,
                               "what": "kvcache_ring_update_rope (raw K rotated on the way in), steady state as "
                                       "kv_update_steady; per insert"},
            "copy_reference": {"value": gbs(copy_ms), "unit": "GB/s", "avg_us": copy_ms * 1e3,
                               "what": "torch device copy of the same bytes as one ring insert (5 frames of K and V), "
                                       "steady state as kv_update_steady: the practical copy rate at this size "
                                       "(the measured HBM peak comes from a 2 GB copy)"},
            "rope3d": {"value": ROPE_BYTES / (rope_ms * 1e-3) / 1e9, "unit": "GB/s", "avg_us": rope_ms * 1e3,
                       "bytes_per_call": ROPE_BYTES, "what": "rope3d_apply of Q (23,400 rows) + K (32,760 rows)",
                       "frac_of_measured_hbm": ROPE_BYTES / (rope_ms * 1e-3) / 1e9 / peaks["hbm"]},
            "rope3d_batched": {"value": ROPE_BYTES / (rope_batch_ms * 1e-3) / 1e9, "unit": "GB/s",
                               "avg_us": rope_batch_ms * 1e3, "bytes_per_call": ROPE_BYTES,
                               "what": "rope3d_apply_batch of the same Q and K: one launch",
                               "frac_of_measured_hbm": ROPE_BYTES / (rope_batch_ms * 1e-3) / 1e9 / peaks["hbm"]},
            "attn_k_prerotated": {"value": ATTN_FLOPS / (qonly_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                                  "avg_ms": qonly_ms, "what": "same attention with K already rotated "
                                                              "(rolling-cache pass: Q-only RoPE in-kernel)",
                                  "frac_of_nominal_2250": ATTN_FLOPS / (qonly_ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS},
            "two_pass": {"value": two_pass_flops / (two_pass_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                         "avg_ms": two_pass_ms, "useful_flops": two_pass_flops,
                         "what": "one launch: denoise 23,400 + cache-update 7,800 queries over 32,760 keys, "
                                 "frame-block-causal (3 frames), RoPE on Q and K; visible pairs only"},
            "rotate_half": {"attention": ATTN_FLOPS / (half_attn_ms * 1e-3) / 1e12, "attention_unit": "TFLOP/s",
                            "rope3d": ROPE_BYTES / (half_rope_ms * 1e-3) / 1e9, "rope3d_unit": "GB/s",
                            "what": "RKV_ROPE_HALF layout (pairs j, j + 64): fused attention of the step and "
                                    "standalone RoPE of its Q and K"},
            "sweep": sweep,
            "e2e": {"value": world * ATTN_FLOPS * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / e2e_steps,
                    "steps": e2e_steps, "how": "pinned host buffers; uploads, kernels and downloads of "
                                               "consecutive steps overlap on three streams"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(host)
            if sweep is not None:
                sweep["cpu_baseline_insert"] = sweep_cpu_baseline(host)
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def profile_case(args):
    """--profile-case: W + K launches of one call on the bench workload, for
    ncu (no timing, no JSON)."""
    import torch
    from rolling_kv_cache_rope_b200 import rkv
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    _, t = make_inputs(device)
    rope = rkv.make_rope(GRID_H, GRID_W)
    o = torch.empty((LQ, H, D), dtype=torch.bfloat16, device=device)
    ws = torch.zeros(rkv.attn_fwd_varlen_workspace_size(1, H, D), dtype=torch.uint8, device=device)
    ring = rkv.KVRing(RING_SLOTS, F, H, D, device=device)
    yq, yk = torch.empty_like(t["q"]), torch.empty_like(t["k"])
    case = args.profile_case

    def once(i):
        if case == "attention":
            rkv.attn_fwd_varlen([rkv.AttnSeq(t["q"], t["k"], t["v"], o, q_t0=Q_T0, k_t0=K_T0)], rope, workspace=ws)
        elif case == "attention_qonly":
            rkv.attn_fwd_varlen([rkv.AttnSeq(t["q"], t["k"], t["v"], o, q_t0=Q_T0, k_t0=K_T0, rope_k=False)], rope,
                                workspace=ws)
        elif case == "ring":
            rkv.kvcache_ring_update(ring, t["k_new"], t["v_new"], RING_INSERT)
        elif case == "ring_rope":
            rkv.kvcache_ring_update_rope(ring, t["k_new"], t["v_new"], 1 + RING_INSERT * i, rope, RING_INSERT)
        elif case == "rope":
            rkv.rope3d_apply(t["q"], yq, t0=Q_T0, rope=rope)
            rkv.rope3d_apply(t["k"], yk, t0=K_T0, rope=rope)
        elif case == "rope_batched":
            rkv.rope3d_apply_batch([(t["q"], yq, Q_T0), (t["k"], yk, K_T0)], rope=rope)
        else:
            raise SystemExit(f"unknown --profile-case {case}")

    for i in range(args.warmup + args.steps):
        once(i)
    torch.cuda.synchronize()
    rkv.rkv_attn_status(ws)
    rkv.rkv_ring_status()
    return 0


ATTN_SOURCES = ("rolling_kv_cache_rope_b200/csrc/attn_fwd.cu", "rolling_kv_cache_rope_b200/csrc/sm100_ptx.cuh",
                "rolling_kv_cache_rope_b200/csrc/common.cuh")


def attn_source_sha256():
    """sha256 over the attention kernel's source files, in ATTN_SOURCES order."""
    import hashlib
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def load_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, or None
    when the attention kernel's sources have changed since that capture."""
    p = os.path.join(ROOT, "profiles", "attn_fwd_kernel_denoise_23400x32760.md")
    try:
        with open(p) as f:
            kv = dict(line.split(":", 1) for line in f.read().splitlines()
                      if line.startswith(("source_sha256:", "dram_bytes_per_launch:")))
        sha = attn_source_sha256()
    except (OSError, ValueError):
        return None
    if kv.get("source_sha256", "").strip() != sha:
        return None
    try:
        return int(kv["dram_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 30-layer rolling sweep measurement")
    ap.add_argument("--profile-case", choices=["attention", "attention_qonly", "ring", "ring_rope", "rope", "rope_batched"],
                    help="run only W + K launches of one call (for ncu); prints nothing")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return profile_case(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
