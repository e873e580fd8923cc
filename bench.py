#!/usr/bin/env python
"""Benchmark of the low-bit block-diffusion KV-cache hot path on B200.

One step = dkv_commit_block of one 32-token block (quantize-on-commit) +
dkv_block_attention of the next active block's queries over the committed
cache (one denoising step).  Every max(1, k_group/block) steps a cache is
rolled back with dkv_cache_truncate to its starting length, so the committed
length stays at the workload's L (+ at most k_group tokens) however many
steps run.  Inputs are seeded synthetic data from `synth`, resident in HBM
before the timed region; caches are replicated R times and used round-robin
so that the bytes touched between two uses of one cache exceed the L2.

Output: one JSON line (rank 0).  `value` = algorithmic HBM bytes of all steps
(packed cache + scales + side table + tail read by attention, Q / active
block / output, commit reads and writes) / device time of the timed region,
summed over ranks (weak scaling: each rank runs its own copy of the
workload).  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = ("block-attention HBM GB/s & % of 8 TB/s roofline; commit tokens/s (1×B200)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ accounting

def _n_prot(w: synth.Workload, L: int) -> float:
    """Expected protected positions per unit among the first L tokens."""
    return w.prot_frac * L


def attn_bytes(w: synth.Workload, L: int) -> float:
    """Algorithmic HBM bytes of one dkv_block_attention at committed length L."""
    U, d = w.B * w.Hkv, w.d
    if w.k_bits < 16:
        Lq = (L // w.k_group) * w.k_group
        nG = Lq // w.k_group
        kb = Lq * d * w.k_bits / 8 + nG * d * 4 + (nG + 1) * 4 + (L - Lq) * d * 2
        kb += _n_prot(w, Lq) * (d * 2 + 4)
    else:
        kb = L * d * 2
    vb = L * (d * w.v_bits / 8 + (d // w.v_group) * 4) if w.v_bits < 16 else L * d * 2
    io = w.B * w.Hq * w.blk * d * 2 * 2 + 2 * U * w.blk * d * 2
    return U * (kb + vb) + io


def attn_flops(w: synth.Workload, L: int) -> float:
    """QK^T and PV multiply-adds x 2 over committed + active tokens."""
    return 4.0 * w.rows * w.d * (L + w.blk) * w.B * w.Hkv


def commit_bytes(w: synth.Workload, L_before: int) -> float:
    U, d, blk = w.B * w.Hkv, w.d, w.blk
    b = 2 * blk * d * 2 + 4                                   # K, V block + mask
    b += blk * (d * w.v_bits / 8 + (d // w.v_group) * 4) if w.v_bits < 16 else blk * d * 2
    if w.k_bits < 16:
        n_tail = L_before % w.k_group
        if n_tail + blk >= w.k_group:                        # completes a group
            b += n_tail * d * 2 + w.k_group * d * w.k_bits / 8 + d * 4 + 8
            b += _n_prot(w, w.k_group) * (d * 2 + 4)
        else:
            b += blk * d * 2
    else:
        b += blk * d * 2
    return U * b


def cycle_len(w: synth.Workload) -> int:
    return max(1, w.k_group // w.blk) if w.k_bits < 16 else 1


def step_lengths(w: synth.Workload, K: int, R: int):
    """Committed length before the commit of each step k (cache k % R)."""
    C = cycle_len(w)
    pos = [0] * R
    out = []
    for k in range(K):
        r = k % R
        out.append(w.L + pos[r] * w.blk)
        pos[r] = (pos[r] + 1) % C
    return out


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record():
    """ncu DRAM traffic per launch of the dominant kernel, if the committed
    record matches the kernel source as it is now (else None)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    with open(p) as f:
        rec = json.load(f)
    out = {}
    for wl, r in rec.items():
        src = os.path.join(ROOT, r.get("source", ""))
        if not os.path.exists(src):
            continue
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if h == r.get("source_sha256_16"):
            out[wl] = r
    return out


# ------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", gpu_id, "-lms", "100"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                pw.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        busy = [s for s, p in zip(sm, pw) if p > 200.0] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(busy),
                "power_w_max": max(pw)}


# ------------------------------------------------------------ GPU arm

def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process
    group); NCCL reduces a device tensor, other backends a host tensor."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def whole_job_gbs(bytes_per_rank: float, max_ms: float, world: int) -> float:
    """Weak scaling: every rank moves bytes_per_rank; the job's time is the
    slowest rank's."""
    return world * bytes_per_rank / (max_ms / 1e3) / 1e9


def io_bytes(w: synth.Workload) -> float:
    """Q, active K/V and output bytes of one attention call."""
    return w.B * w.Hq * w.blk * w.d * 2 * 2 + 2 * w.B * w.Hkv * w.blk * w.d * 2


def run_gpu(w: synth.Workload, K: int, W: int, want_e2e=True, log=print, kernel=0,
            v_rotation=0, suffix=0, time_build=False, select_budget=0):
    import torch
    import quantized_kv_cache_dkv_b200 as dkv

    world, rank, local = _dist()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    C = cycle_len(w)
    cache_bytes = attn_bytes(w, w.L)
    R = 1 if cache_bytes >= 2 * l2 else min(8, math.ceil(3 * l2 / cache_bytes))
    unit = max(w.k_group, w.blk)
    cap = ((w.L + C * w.blk + unit - 1) // unit) * unit
    P = int(round(w.prot_frac * cap)) * 2 + 64
    cfg = dkv.make_config(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group,
                          w.v_group, P, cap)
    caches = [dkv.dkv_cache_alloc(cfg) for _ in range(R)]
    # dual cache: a suffix cache of `suffix` committed tokens per replica
    sfx = []
    if suffix:
        cap_s = ((suffix + unit - 1) // unit) * unit
        cfg_s = dkv.make_config(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group,
                                w.v_group, int(round(w.prot_frac * cap_s)) * 2 + 64, cap_s)
        sfx = [dkv.dkv_cache_alloc(cfg_s) for _ in range(R)]
    if v_rotation:
        perm, mix = synth.krpbh_params(w.seed, v_rotation)
        for c in caches:
            dkv.dkv_cache_set_v_rotation(c, perm, mix, v_rotation)
    if kernel:
        for c in caches:
            dkv.dkv_cache_set_option(c, dkv.DKV_OPT_ATTN_KERNEL, kernel)

    def up(bits):
        import numpy as np
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(
            torch.bfloat16)

    def upw(words):
        import numpy as np
        return torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).to(dev)

    t0 = time.time()
    nb = w.L // w.blk
    kept = []
    for i in range(nb):
        K_, V_, M_ = synth.block_inputs(w, i)
        Kd, Vd, Md = up(K_), up(V_), upw(M_)
        for c in caches:
            dkv.dkv_commit_block(c, Kd, Vd, Md)
        if time_build:
            kept.append((Kd, Vd, Md))
    for i in range(suffix // w.blk):
        K_, V_, M_ = synth.block_inputs(w, 100000 + i)
        Kd, Vd, Md = up(K_), up(V_), upw(M_)
        for c in sfx:
            dkv.dkv_commit_block(c, Kd, Vd, Md)
    torch.cuda.synchronize()
    t_prefill = time.time() - t0
    build = None
    if time_build:
        # The whole cache built again by its nb commits, captured in one CUDA
        # graph: rolled back to 0 first, so every replay starts from an empty
        # cache and rewrites the same state as the eager build above.
        dkv.dkv_cache_truncate(caches[0], 0)
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb):
            for Kd, Vd, Md in kept:
                dkv.dkv_commit_block(caches[0], Kd, Vd, Md)
        gb.replay()
        torch.cuda.synchronize()
        times = []
        eb0 = torch.cuda.Event(enable_timing=True)
        eb1 = torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            eb0.record()
            gb.replay()
            eb1.record()
            torch.cuda.synchronize()
            times.append(eb0.elapsed_time(eb1))
        bms = statistics.median(times)
        build = {"commits": nb, "tokens": nb * w.blk, "ms": round(bms, 4),
                 "us_per_commit": round(bms * 1e3 / nb, 3),
                 "tokens_per_s": round(w.B * nb * w.blk / (bms / 1e3), 1),
                 "method": "all commits captured in one CUDA graph; median of 3 replays "
                           "(CUDA events)"}
        del gb
        kept.clear()

    def attend(r, q, ka, va, out):
        if select_budget:
            dkv.dkv_block_attention_selected(caches[r], q, ka, va, w.softmax_scale,
                                             select_budget, out)
        elif sfx:
            dkv.dkv_block_attention_dual(caches[r], sfx[r], q, ka, va, w.softmax_scale, out)
        else:
            dkv.dkv_block_attention(caches[r], q, ka, va, w.softmax_scale, out)

    # per-step inputs: C blocks to commit, S distinct query / active blocks
    blocks = [synth.block_inputs(w, nb + c) for c in range(C)]
    host_blocks = blocks
    dblocks = [(up(a), up(b), upw(m)) for a, b, m in blocks]
    S = min(K, R * C) if K > 0 else 1
    S = max(S, 1)
    host_steps = [(synth.queries_bits(w, s),) + tuple(synth.active_block_bits(w, s))
                  for s in range(S)]
    dsteps = [(up(q), up(ka), up(va)) for q, ka, va in host_steps]
    outs = [torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device=dev)
            for _ in range(S)]

    pos = [0] * R
    launches = [0]

    def step(k):
        r = k % R
        c = pos[r]
        Kd, Vd, Md = dblocks[c]
        dkv.dkv_commit_block(caches[r], Kd, Vd, Md)
        q, ka, va = dsteps[k % S]
        attend(r, q, ka, va, outs[k % S])
        launches[0] += 1 + dkv.dkv_last_attention_plan(caches[r])[2]
        pos[r] += 1
        if pos[r] == C:  # back to the starting length (recorded; the next commit applies it)
            dkv.dkv_cache_truncate(caches[r], w.L)
            pos[r] = 0

    def finish():
        for r in range(R):
            if pos[r]:
                dkv.dkv_cache_truncate(caches[r], w.L)
                pos[r] = 0

    # warm-up (eager; at least one step per cache replica, so that every
    # handle has made its first call -- which may allocate -- before the
    # capture), then capture exactly K steps in one CUDA graph
    for k in range(max(W, R)):
        step(k)
    finish()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    launches[0] = 0
    with torch.cuda.graph(g):
        for k in range(K):
            step(k)
        finish()
    graph_launches = launches[0]
    plan = dkv.dkv_last_attention_plan(caches[0])
    g.replay()
    torch.cuda.synchronize()

    # clocks sampled over a window of back-to-back replays around the timed one
    gpu_id = str(getattr(props, "uuid", local))
    gpu_id = gpu_id if gpu_id.startswith("GPU-") or not hasattr(props, "uuid") else "GPU-" + gpu_id
    sampler = ClockSampler(gpu_id)
    t_end = time.time() + 0.6
    while time.time() < t_end:
        g.replay()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    t_end = time.time() + 0.4
    while time.time() < t_end:
        g.replay()
        torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = max_over_ranks(ms)

    Ls = step_lengths(w, K, R)
    sfx_bytes = attn_bytes(w, suffix) - io_bytes(w) if suffix else 0.0
    step_bytes = sum(attn_bytes(w, L + w.blk) + sfx_bytes + commit_bytes(w, L) for L in Ls)
    value = whole_job_gbs(step_bytes, ms, world)

    # profiling pass: device time of each kernel kind (eager launches)
    for c in caches + sfx:
        dkv.dkv_cache_set_option(c, dkv.DKV_OPT_PROFILE, 1)
    Kp = max(K, 2 * R * C)
    for k in range(Kp):
        step(k)
    finish()
    torch.cuda.synchronize()
    prof = {}
    for kind, name in ((dkv.DKV_KERNEL_ATTENTION, "attention"), (dkv.DKV_KERNEL_COMBINE, "combine"),
                       (dkv.DKV_KERNEL_COMMIT, "commit"), (dkv.DKV_KERNEL_TRUNCATE, "truncate")):
        tot, n = 0.0, 0
        for c in caches:
            a, b = dkv.dkv_profile_read(c, kind)
            tot += a
            n += b
        prof[name] = (tot, n)
    for c in caches + sfx:
        dkv.dkv_cache_set_option(c, dkv.DKV_OPT_PROFILE, 0)
    Lp = step_lengths(w, Kp, R)
    att_ms, att_n = prof["attention"]
    if select_budget:
        # one selection call = four kernels timed as attention (statistics,
        # scores, top-k, attention over the kept tokens): per-call figures
        att_n = att_n // 4
    # The timed region is a CUDA-graph replay whose kernels overlap their
    # launch with the previous kernel (programmatic dependent launch), so the
    # eager per-launch times above do not add up to its step time.  Each
    # kernel's time in the timed execution is the graph's step time times that
    # kernel's share of the eager device time.
    eager_tot = sum(v[0] for v in prof.values())
    share = {k: (v[0] / eager_tot if eager_tot > 0 else 0.0) for k, v in prof.items()}
    step_ms_graph = ms / K
    # (a dual-cache step launches the attention kernel twice: its bytes and
    # flops are those of both launches, averaged per launch below)
    att_bytes = sum(attn_bytes(w, L + w.blk) + sfx_bytes for L in Lp)
    att_flops = sum(attn_flops(w, L + w.blk) + 4.0 * w.rows * w.d * suffix * w.B * w.Hkv
                    for L in Lp)
    com_ms, com_n = prof["commit"]

    # end to end through the public API from pinned host memory
    e2e = None
    if want_e2e:
        import numpy as np
        # Three streams, two buffer sets: step k+1's inputs go up while step
        # k computes, and step k's output comes down while step k+1 computes.
        # Every step still copies its own inputs from pinned host memory and
        # reads its own result back inside the timed region.
        s_up, s_dn = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        s_cp = stream
        nb = 2
        # One step's inputs -- K, V block and protect words (commit), Q and
        # the active K, V (attention) -- packed in one pinned host buffer per
        # (block, step) pair, so each step uploads them with one copy into a
        # device buffer of the same layout (the API takes views into it).
        n_kv = w.B * w.Hkv * w.blk * w.d
        n_q = w.B * w.Hq * w.blk * w.d
        n_m = w.B * w.Hkv * (w.blk // 32)
        n_m16 = (2 * n_m + 7) // 8 * 8  # the words' int16 slots, padded to 16 bytes
        offs = [0, n_kv, 2 * n_kv, 2 * n_kv + n_m16, 2 * n_kv + n_m16 + n_q,
                3 * n_kv + n_m16 + n_q]  # int16 element offsets: K, V, M, Q, Ka, Va
        n_in = 4 * n_kv + n_m16 + n_q
        hin = {}
        for c in range(C):
            for st in range(S):
                buf = torch.empty(n_in, dtype=torch.int16)
                a_, b_, m_ = host_blocks[c]
                q_, ka_, va_ = host_steps[st]
                npb = buf.numpy()
                npb[offs[0]:offs[1]] = a_.view(np.int16).ravel()
                npb[offs[1]:offs[2]] = b_.view(np.int16).ravel()
                npb[offs[2]:offs[2] + 2 * n_m] = m_.view(np.int32).ravel().view(np.int16)
                npb[offs[3]:offs[4]] = q_.view(np.int16).ravel()
                npb[offs[4]:offs[5]] = ka_.view(np.int16).ravel()
                npb[offs[5]:] = va_.view(np.int16).ravel()
                hin[(c, st)] = buf.pin_memory()
        dIn = [torch.empty(n_in, dtype=torch.int16, device=dev) for _ in range(nb)]
        shp_kv = (w.B, w.Hkv, w.blk, w.d)
        shp_q = (w.B, w.Hq, w.blk, w.d)
        views = []
        for bf in dIn:
            views.append((bf[offs[0]:offs[1]].view(shp_kv), bf[offs[1]:offs[2]].view(shp_kv),
                          bf[offs[2]:offs[2] + 2 * n_m].view(torch.int32).view(w.B, w.Hkv, w.blk // 32),
                          bf[offs[3]:offs[4]].view(shp_q), bf[offs[4]:offs[5]].view(shp_kv),
                          bf[offs[5]:].view(shp_kv)))
        dO = [torch.empty(shp_q, dtype=torch.int16, device=dev) for _ in range(nb)]
        hout = [torch.empty(shp_q, dtype=torch.int16).pin_memory() for _ in range(nb)]
        ev_up = [torch.cuda.Event() for _ in range(nb)]     # inputs of buffer b are on the device
        ev_cp = [torch.cuda.Event() for _ in range(nb)]     # step using buffer b has computed
        ev_dn = [torch.cuda.Event() for _ in range(nb)]     # output of buffer b is on the host
        h2d = n_in * 2
        d2h = dO[0].numel() * 2
        used = [False] * nb

        def upload(k):
            b = k % nb
            with torch.cuda.stream(s_up):
                if used[b]:
                    s_up.wait_event(ev_cp[b])  # the step that read buffer b is done
                dIn[b].copy_(hin[(pos_e[k % R], k % S)], non_blocking=True)
                ev_up[b].record(s_up)

        def compute(k):
            b, r = k % nb, k % R
            s_cp.wait_event(ev_up[b])
            if used[b]:
                s_cp.wait_event(ev_dn[b])  # the previous output in dO[b] has been read back
            dK, dV, dM, dQ, dKa, dVa = views[b]
            dkv.dkv_commit_block(caches[r], dK, dV, dM)
            attend(r, dQ, dKa, dVa, dO[b])
            ev_cp[b].record(s_cp)
            pos[r] += 1
            if pos[r] == C:
                dkv.dkv_cache_truncate(caches[r], w.L)
                pos[r] = 0

        def download(k):
            b = k % nb
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(ev_cp[b])
                hout[b].copy_(dO[b], non_blocking=True)
                ev_dn[b].record(s_dn)
            used[b] = True

        pos_e = [0] * R  # block index of the next commit of each cache, for uploads

        def run(n):
            for i in range(nb):
                used[i] = False
            for r in range(R):
                pos_e[r] = pos[r]
            upload(0)
            pos_e[0 % R] = (pos_e[0 % R] + 1) % C
            for k in range(n):
                if k + 1 < n:
                    upload(k + 1)
                    pos_e[(k + 1) % R] = (pos_e[(k + 1) % R] + 1) % C
                compute(k)
                download(k)

        def join_streams():
            for st in (s_up, s_dn):
                ev = torch.cuda.Event()
                ev.record(st)
                s_cp.wait_event(ev)

        run(W)
        join_streams()
        finish()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0.record(s_cp)
        s_up.wait_stream(s_cp)
        s_dn.wait_stream(s_cp)
        run(K)
        join_streams()
        e1.record(s_cp)
        torch.cuda.synchronize()
        barrier()
        ems = e0.elapsed_time(e1)
        finish()
        ems = max_over_ranks(ems)
        e2e = {"value": whole_job_gbs(step_bytes, ems, world), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ems / K}

    for c in caches + sfx:
        dkv.dkv_cache_free(c)
    return {
        "ms": ms, "value": value, "R": R, "C": C, "cap": cap, "P": P, "plan": plan,
        "graph_launches": graph_launches, "clocks": clocks, "t_prefill_s": t_prefill,
        "att_ms": att_ms, "att_n": att_n, "att_bytes": att_bytes, "att_flops": att_flops,
        "combine_ms": prof["combine"][0], "combine_n": prof["combine"][1],
        "commit_ms": com_ms, "commit_n": com_n, "e2e": e2e, "L_mean": sum(Ls) / len(Ls) + w.blk,
        "step_bytes": step_bytes / K, "build": build, "Kp": Kp, "share": share,
        # per-launch times in the timed (graph) execution
        "att_us_graph": step_ms_graph * share["attention"] * Kp / max(att_n, 1) * 1e3,
        "commit_us_graph": step_ms_graph * share["commit"] * Kp / max(com_n, 1) * 1e3,
        "combine_us_graph": step_ms_graph * share["combine"] * Kp / max(prof["combine"][1], 1) * 1e3,
    }


TIMING_METHOD = ("step time: CUDA events around one CUDA-graph replay of the K timed steps; "
                 "per-kernel time in that execution = step time x the kernel's share of device "
                 "time in an eager pass of the same steps with CUDA events around each launch")


def roofline(w: synth.Workload, r: dict, peaks: dict, peak_kind: str, traffic):
    """Roofline of the dominant kernel (the split attention kernel), at its
    per-launch time in the timed (graph) execution."""
    avg_s = r["att_us_graph"] / 1e6
    bytes_launch = r["att_bytes"] / max(r["att_n"], 1)
    flops_launch = r["att_flops"] / max(r["att_n"], 1)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if flops_launch / bytes_launch > ridge else "hbm"
    if bound == "hbm":
        ach, peak, unit = bytes_launch / avg_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        ach, peak, unit = flops_launch / avg_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    tr = None
    if traffic and w.name in traffic:
        t = traffic[w.name]
        tr = t["traffic_bytes_per_launch"] * (bytes_launch / t["algorithmic_bytes_per_launch"]) \
            if t.get("scale_by_bytes") else t["traffic_bytes_per_launch"]
    return {"bound": bound, "achieved": round(ach, 2), "peak": peak, "unit": unit,
            "frac": round(ach / peak, 4), "traffic": tr,
            "peak_source": f"{peak_kind} ({'hbm_gbs' if bound == 'hbm' else 'bf16_tflops burst'})",
            "kernel": "attention split kernel", "avg_launch_us": round(avg_s * 1e6, 3),
            "avg_launch_us_eager": round(r["att_ms"] / max(r["att_n"], 1) * 1e3, 3),
            "share_of_step": round(r["share"]["attention"], 4),
            "algorithmic_bytes_per_launch": int(bytes_launch),
            "algorithmic_flops_per_launch": int(flops_launch),
            "hbm_gbs_at_kernel": round(bytes_launch / avg_s / 1e9, 1),
            "pct_of_8tbs_at_kernel": round(100 * bytes_launch / avg_s / 8e12, 2)}


# ------------------------------------------------------------ CPU oracle arm

def _blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w: synth.Workload, seconds: float, max_steps=None, warmup=0):
    """Time the oracle (as it stands) on sampled units of the workload: each
    step = commit of one block + one block attention, per sampled unit.
    Returns (GB/s, steps, elapsed, description)."""
    from oracle import OracleCache
    nb = w.L // w.blk
    C = cycle_len(w)
    units = [(0, 0)] if w.L >= 16384 or w.B * w.Hkv == 1 else [(0, 0), (w.B - 1, w.Hkv - 1)]
    cap = w.L + C * w.blk + max(w.k_group, w.blk)
    P = int(round(w.prot_frac * cap)) * 2 + 64
    ocs = []
    for (b, h) in units:
        oc = OracleCache(1, w.g, 1, w.d, w.blk, w.k_bits, w.v_bits, w.k_group, w.v_group, P, cap)
        for i in range(nb):
            Kb, Vb = synth.kv_block_bits(w, b, h, i)
            oc.commit(Kb[None, None], Vb[None, None],
                      synth.block_protect_words(w, b, h, i)[None, None])
        ocs.append(oc)
    blocks = {}
    for (b, h) in units:
        for c in range(C):
            Kb, Vb = synth.kv_block_bits(w, b, h, nb + c)
            blocks[(b, h, c)] = (Kb[None, None], Vb[None, None],
                                 synth.block_protect_words(w, b, h, nb + c)[None, None])
    q = synth.queries_bits(w, 0)
    ka, va = synth.active_block_bits(w.with_(B=1, Hkv=1, Hq=w.g), 0)
    U = w.B * w.Hkv
    pos = 0
    per_unit_bytes = 0.0
    steps = 0
    elapsed = 0.0
    k = 0
    while True:
        if max_steps is not None and steps >= max_steps:
            break
        if max_steps is None and elapsed >= seconds and steps > 0:
            break
        L_before = w.L + pos * w.blk
        t0 = time.perf_counter()
        for (b, h), oc in zip(units, ocs):
            oc.commit(*blocks[(b, h, pos)])
            oc.block_attention(q[b:b + 1, h * w.g:(h + 1) * w.g], ka, va, w.softmax_scale)
        dt = time.perf_counter() - t0
        pos += 1
        if pos == C:
            for oc in ocs:
                oc.truncate(w.L)
            pos = 0
        k += 1
        if k <= warmup:
            continue
        elapsed += dt
        steps += 1
        per_unit_bytes += (attn_bytes(w, L_before + w.blk) + commit_bytes(w, L_before)) / U
    gbs = per_unit_bytes * len(units) / elapsed / 1e9
    desc = (f"{len(units)} of {U} (batch, kv-head) units x {steps} steps (commit + attention), "
            f"L={w.L}; numpy/BLAS fp64")
    return gbs, steps, elapsed, desc


# ------------------------------------------------------------ main

def base_line(w, args, value, ms_per_step, world):
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
                   "L": w.L, "block": w.blk, "k_bits": w.k_bits, "v_bits": w.v_bits,
                   "k_group": w.k_group, "v_group": w.v_group, "prot_frac": w.prot_frac,
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
    }


def plan_name(w: synth.Workload, kernel: int) -> str:
    return {1: "mma.sync", 2: "tcgen05 (query-row blocks)",
            3: "tcgen05 (tokens on TMEM lanes)"}.get(kernel, str(kernel))


def kernel_fields(w: synth.Workload, r: dict) -> dict:
    """Per-kernel figures of one run: times in the timed (graph) execution
    and in the eager pass, commit rate, launch plan."""
    att_us = r["att_us_graph"]
    return {
        "attention_gbs": round(r["att_bytes"] / max(r["att_n"], 1) / (att_us / 1e6) / 1e9, 1),
        "pct_of_8tbs": round(100 * r["att_bytes"] / max(r["att_n"], 1) / (att_us / 1e6) / 8e12, 2),
        "commit_tokens_per_s": round(w.B * w.blk / (r["commit_us_graph"] / 1e6), 1)
        if r["commit_us_graph"] > 0 else None,
        "kernel_us": {"attention": round(att_us, 3), "combine": round(r["combine_us_graph"], 3),
                      "commit": round(r["commit_us_graph"], 3)},
        "kernel_us_eager": {"attention": round(r["att_ms"] / max(r["att_n"], 1) * 1e3, 3),
                            "combine": round(r["combine_ms"] / max(r["combine_n"], 1) * 1e3, 3),
                            "commit": round(r["commit_ms"] / max(r["commit_n"], 1) * 1e3, 3)},
        "attention_plan": {"kernel": plan_name(w, r["plan"][0]),
                           "splits": r["plan"][1], "launches": r["plan"][2]},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", choices=["dkv", "reference"], default="dkv")
    ap.add_argument("--workload", default="batch32", choices=list(synth.WORKLOADS),
                    help="the line's workload (default: the batch-32 decode profile, the "
                         "largest single-GPU configuration)")
    ap.add_argument("--no-sub-records", action="store_true",
                    help="skip the per-workload records of the other configurations")
    ap.add_argument("--kernel", type=int, default=0, choices=[0, 1, 2, 3],
                    help="attention kernel: 0 = library's choice, 1 = mma.sync, 2 = tcgen05 "
                         "(query-row blocks), 3 = tcgen05 with the tokens on the TMEM lanes "
                         "(32-row query groups)")
    ap.add_argument("--B", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--L", type=int, default=0, help="override the committed length (profiling)")
    ap.add_argument("--k-bits", type=int, default=0, choices=[0, 2, 3, 4, 16],
                    help="override the line's K code width (0 = the workload's)")
    ap.add_argument("--v-bits", type=int, default=0, choices=[0, 2, 3, 4, 16],
                    help="override the line's V code width (0 = the workload's)")
    ap.add_argument("--v-rotation", type=int, default=0, choices=[0, 16, 32, 64, 128],
                    help="K-RPBH rotation of V with this Hadamard block (0 = none)")
    ap.add_argument("--suffix", type=int, default=0,
                    help="dual cache: tokens in a second (suffix) cache attended with the prefix")
    ap.add_argument("--select-budget", type=int, default=0,
                    help="Q-MaskAhead selection: each step attends to this many committed tokens "
                         "per (sequence, kv-head), chosen by contribution score, plus the block")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = _dist()
    w = synth.WORKLOADS[args.workload]
    if args.B:
        w = w.with_(B=args.B)
    if args.L:
        w = w.with_(L=args.L)
    if args.k_bits:
        w = w.with_(k_bits=args.k_bits)
    if args.v_bits:
        w = w.with_(v_bits=args.v_bits)

    if args.impl == "reference":
        if rank != 0:
            return
        gbs, steps, el, desc = oracle_sample(w, 0, max_steps=args.steps, warmup=args.warmup)
        line = base_line(w, args, gbs, el / max(steps, 1) * 1e3, world)
        line["dtype"] = "f64"
        line["impl"] = "reference"
        cores = _blas_threads()
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "sample": desc}
        line["e2e"] = {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}
        print(json.dumps(line), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks, peak_kind = load_peaks()
    traffic = traffic_record()
    if args.suffix % w.blk:
        raise SystemExit("--suffix must be a multiple of the block")
    r = run_gpu(w, args.steps, args.warmup, log=lambda *a: None, kernel=args.kernel,
                v_rotation=args.v_rotation, suffix=args.suffix,
                time_build=(w.name == "longprompt"), select_budget=args.select_budget)
    line = base_line(w, args, r["value"], r["ms"] / args.steps, world)
    if args.v_rotation:
        line["config"]["v_rotation"] = f"K-RPBH, Hadamard block {args.v_rotation}"
    if args.suffix:
        line["config"]["dual_cache_suffix_tokens"] = args.suffix
    if args.select_budget:
        line["config"]["select_budget"] = args.select_budget
        line["config"]["select_bytes"] = ("the packed cache counted once per step (the scores read "
                                          "all of it); the attention kernel figures sum its two "
                                          "launches (softmax statistics over the whole cache, "
                                          "then the gathered tokens)")
    line["config"]["L2_policy"] = (f"{r['R']} cache replicas used round-robin"
                                   if r["R"] > 1 else "cache larger than L2")
    line["config"]["L_mean"] = r["L_mean"]
    line["config"]["step"] = (f"1 commit + 1 attention; truncate to L every {r['C']} steps; "
                              "timed region = one CUDA graph replay of the steps")
    line["config"]["timing"] = TIMING_METHOD
    line["roofline"] = roofline(w, r, peaks, peak_kind, traffic)
    if args.suffix or args.select_budget or args.k_bits or args.v_bits:
        # the recorded traffic is that of the plain launch at the workload's own code widths
        line["roofline"]["traffic"] = None
    line["clocks"] = r["clocks"]
    line["e2e"] = r["e2e"]
    line["gpu_launches"] = r["graph_launches"]
    line.update(kernel_fields(w, r))
    if r["build"]:
        line["build"] = r["build"]
    if not args.no_sub_records and not (args.select_budget or args.suffix or args.v_rotation):
        # every other configuration of the workload set, each with its own
        # roofline (same timing method, no end-to-end or oracle leg)
        line["workloads"] = {}
        for name in synth.WORKLOAD_ORDER:
            if name == w.name:
                continue
            ww = synth.WORKLOADS[name]
            kern = args.kernel if (args.kernel != 3 or ww.rows == 32) else 0
            rr = run_gpu(ww, args.steps, args.warmup, want_e2e=False, kernel=kern,
                         time_build=(name == "longprompt"))
            rec = {"value_gbs": round(rr["value"], 1),
                   "ms_per_step": round(rr["ms"] / args.steps, 6),
                   "config": {k: getattr(ww, k) for k in ("B", "Hq", "Hkv", "L", "k_bits",
                                                          "v_bits", "k_group", "v_group",
                                                          "prot_frac")},
                   "roofline": roofline(ww, rr, peaks, peak_kind, traffic),
                   "clocks_sm_mhz": (rr["clocks"] or {}).get("sm_mhz"),
                   "clock_reasons": (rr["clocks"] or {}).get("reasons")}
            rec.update(kernel_fields(ww, rr))
            if rr["build"]:
                rec["build"] = rr["build"]
            line["workloads"][name] = rec
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.v_rotation \
            and not args.suffix and not args.select_budget:
        gbs, steps, el, desc = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": _blas_threads(),
                                "kind": "oracle", "sample": desc}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
