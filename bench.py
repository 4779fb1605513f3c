"""Benchmark of one AsyncTLS decode step (two-level sparse attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = block score + top-K_b, label-channel token score + top-K_t, and
sparse attention with log-sum-exp merge, for all B x H_q heads of one layer,
through the C ABI of libtls.so.  Default workload: GQA, batch 8, 32/8 heads,
head_dim 128, 96k context, K_b 256, K_t 4096, r 16, bf16.  Inputs are seeded
synthetic tensors (see two_level_sparse_quest_b200/workloads.py); the step
rotates over 4 layer copies held in separate device memory, so consecutive
steps never hit the 126 MB L2 with the previous step's bytes.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
copy of the workload (independent sequences, no collective on the data path);
time is the max over ranks; value = steps of all ranks / time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode steps/sec (all heads) at 96k ctx; achieved HBM GB/s vs peak"
N_LAYERS_DEFAULT = 4
L2_BYTES = 126e6
STAGE_STEPS_MIN = 100  # steps of the separate per-stage timing pass
SMI_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# ----------------------------------------------------------------------------- bytes
def algorithmic_bytes(w) -> dict:
    """Bytes one step must touch (the method's data, not scratch):
    block summary of every block, label slab rows of the K_b * bs candidates,
    K and V rows of the K_t kept tokens, q, out (fp32), lse, and the int32
    block / token index lists (written once, read once)."""
    e = w.elem_bytes
    G = w.batch * w.n_kv_heads
    vrow = 0 if w.v_is_k_prefix else w.d_v
    parts = {
        "block_summary": G * w.n_blocks * 2 * w.d_qk * e,
        "label_slab": (G * w.k_b * w.block_size * w.n_label * e if getattr(w, "slab_bits", 0) != 8
                       else G * w.k_b * w.block_size * w.n_label + G * w.n_label * 4),  # int8 codes + scales
        "gathered_kv": G * w.k_t * (w.d_qk + vrow) * e,
        "q": w.batch * w.n_q_heads * w.d_qk * e,
        "out_lse": w.batch * w.n_q_heads * (w.d_v * 4 + 4),
        "indices": G * (w.k_b + w.k_t) * 4 * 2,
    }
    parts["total"] = sum(parts.values())
    # per stage (what each C call must read/write)
    parts["stage_block"] = parts["block_summary"] + parts["q"] + G * w.k_b * 4
    parts["stage_token"] = parts["label_slab"] + parts["q"] + G * (w.k_b + w.k_t) * 4
    # stages 1-4 in one launch (tls_select_step): the block ids go out and come back once
    parts["stage_select"] = parts["stage_block"] + parts["stage_token"] - parts["q"]
    parts["stage_attn"] = parts["gathered_kv"] + parts["q"] + parts["out_lse"] + G * w.k_t * 4
    return parts


# ----------------------------------------------------------------------------- helpers
def read_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


# the sources each stage's kernels are built from (a profile of a stage stays
# valid while these are unchanged)
STAGE_SOURCES = {
    "stage_select": ["tls_select.cu", "tls_device.cuh", "tls_internal.h"],
    "stage_attn": ["tls_attn.cu", "tls_attn_mma.cu", "tls_attn_mla_tc.cu", "tls_mma.cuh", "tls_device.cuh",
                   "tls_internal.h"],
}


def kernel_source_hash(files=None) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "two_level_sparse_quest_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def read_profile(stage: str):
    """The committed ncu summary entry of a stage (profiles/traffic.json), only
    if it was taken on the stage's kernel sources as they are now."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(stage)
    if not ent or ent.get("source_hash") != kernel_source_hash(STAGE_SOURCES.get(stage)):
        return None
    return ent


def read_traffic(stage: str):
    """DRAM traffic per launch from a committed ncu summary (null when the
    kernels changed since the counters were taken)."""
    ent = read_profile(stage)
    return ent.get("bytes_per_launch") if ent else None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
            time.sleep(0.5)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self) -> dict:
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        for ts, line in self.lines:
            if self.t0 and (ts < self.t0 or ts > (self.t1 or ts) + 0.1):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                smax.append(float(f[3]))
                power.append(float(f[4]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 f[6:10]):
                if val.lower() == "active":
                    reasons.add(name)
        med = sorted(sm)[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- ranks
def rank_workload(base, rank: int):
    """Weak scaling: rank r decodes its own independent sequences (seed offset)."""
    return base.with_(seed=base.seed + 7919 * rank)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank timing over all ranks (the job's time)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- GPU arm
class Layer:
    """One layer's resident state: KV cache, block summary, label slab, query."""

    def __init__(self, T, w, shape, K, V, seq_lens, label, q, dev):
        import torch

        self.K = K.clone()
        self.V = V.clone() if V is not None else None
        self.q = q
        edt = torch.int16 if w.dtype == 1 else torch.float32
        self.meta = torch.empty((w.batch, w.n_kv_heads, w.n_blocks, 2, w.d_qk), dtype=edt, device=dev)
        if shape.slab_bits == 8:
            self.slab = torch.empty(T.tls_slab_bytes(shape), dtype=torch.uint8, device=dev)
        else:
            self.slab = torch.empty((w.batch, w.n_kv_heads, w.ctx, w.n_label), dtype=edt, device=dev)
        T.tls_build_block_meta(shape, self.K, seq_lens, label, self.meta, self.slab)


def gpu_arm(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from two_level_sparse_quest_b200 import build as tls_build

    tls_build.build()
    from two_level_sparse_quest_b200 import tls as T
    from two_level_sparse_quest_b200 import workloads as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = W.WORKLOADS[args.workload].with_(slab_bits=args.slab_bits, block_agg=args.block_agg)
    w = rank_workload(base, rank)
    shape = T.shape_from_workload(w)
    inp = W.make_decode_inputs(w)
    # layer copies rotated through: enough that one rotation's algorithmic bytes
    # are at least twice the 126 MB L2, so no step finds its data in L2
    N_LAYERS = args.layers or max(N_LAYERS_DEFAULT, math.ceil(2 * L2_BYTES / algorithmic_bytes(w)["total"]))
    qs = W.make_query_stream(w.with_(ar_rho=0.5), steps=N_LAYERS)

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)

    K0 = up(inp.K)
    V0 = up(inp.V) if inp.V is not None else None
    seq_lens, label = up(inp.seq_lens), up(inp.label_idx)
    layers = [Layer(T, w, shape, K0, V0, seq_lens, label, up(qs[i]), dev) for i in range(N_LAYERS)]
    del K0, V0
    G = w.batch * w.n_kv_heads
    ws = torch.zeros(T.tls_workspace_size(shape), dtype=torch.uint8, device=dev)
    bidx = torch.empty((G, w.k_b), dtype=torch.int32, device=dev)
    tidx = torch.empty((G, w.k_t), dtype=torch.int32, device=dev)
    out = torch.empty((w.batch, w.n_q_heads, w.d_v), dtype=torch.float32, device=dev)
    lse = torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    def step(L, ev=None):
        """One decode step through the public call, tls_decode_step."""
        T.tls_decode_step(shape, L.q, L.meta, L.slab, label, seq_lens, L.K, L.V, bidx, tidx, out, lse, None, None,
                          ws, sh)


    def step_stages(L, ev):
        """The same step as its two calls, with CUDA events around each: the
        selection with tls_decode_step's workspace (tls_select_step_ws, the
        same launches as the selection part of tls_decode_step), then the
        attention."""
        ev[0].record(stream)
        T.tls_select_step_ws(shape, L.q, L.meta, L.slab, label, seq_lens, bidx, tidx, ws, None, None, sh)
        ev[1].record(stream)
        T.tls_sparse_attn_decode(shape, L.q, L.K, L.V, tidx, out, lse, ws, sh)
        ev[2].record(stream)

    # stages 1-4 (one cluster launch; with few groups a block-score launch
    # first), attention split, log-sum-exp merge
    groups = w.batch * w.n_kv_heads
    # tls_decode_step's launches: with few groups and >= 4 MB of summary the
    # two-phase selection adds a phase-1 launch (and, for groups of more than
    # 16 heads, a query-fold launch before it); max-over-heads adds a score
    # launch (or the two separate selection launches) before the rest
    two_phase = (w.block_agg == 0 and groups * 8 < 2 * torch.cuda.get_device_properties(dev).multi_processor_count
                 and algorithmic_bytes(w)["block_summary"] >= 4 << 20)
    launches_per_step = 3 + (1 if (two_phase or w.block_agg == 1) else 0) + (1 if two_phase and w.group > 16 else 0)
    # The clock sampler starts (and settles) before the warm-up, so that the
    # GPU does not sit idle between the warm-up and the timed region and the
    # timed steps start at the clocks the warm-up brought it to.
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    sampler = ClockSampler(int(vis[local_rank]) if local_rank < len(vis) and vis[local_rank].isdigit() else local_rank)
    if rank == 0:
        sampler.start()
    for i in range(args.warmup):
        step(layers[i % N_LAYERS])
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps, nothing else on the stream.  Kernels
    # within and across steps are chained by programmatic dependent launch.
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("t0")
    t_start.record(stream)
    for i in range(args.steps):
        step(layers[i % N_LAYERS])
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if rank == 0 else None
    ms = t_start.elapsed_time(t_end)
    ms = max_over_ranks(ms, dev)

    # ---- per-stage times, in a separate untimed pass: CUDA events around each
    # C call on every step (the events cut the launch chain at the stage
    # boundaries, which is why they stay out of the timed region).  The first
    # step of the pass is dropped.
    n_stage = max(STAGE_STEPS_MIN, min(args.steps, 1000))
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_stage + 1)]
    for i in range(n_stage + 1):
        step_stages(layers[i % N_LAYERS], sev[i])
    torch.cuda.synchronize()
    st = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])] for e in sev[1:]])
    names = ["stage_select", "stage_attn"]
    stage_ms = st.mean(axis=0)
    stage_med = np.median(st, axis=0)

    # ---- end to end through the C ABI with host buffers: every step uploads its
    # q from pinned host memory and reads its out + lse back.  The copies run on
    # their own streams, double-buffered, so step i's download and step i+1's
    # upload overlap the neighbouring steps' kernels; events order each buffer's
    # reuse.  The timed region ends after the last download.
    n_e2e = min(args.steps, 500)
    q_host = [torch.empty(L.q.shape, dtype=L.q.dtype, pin_memory=True) for L in layers]
    for i, L in enumerate(layers):
        q_host[i].copy_(L.q.cpu())
    up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    qd = [torch.empty_like(layers[0].q) for _ in range(2)]
    od = [torch.empty_like(out) for _ in range(2)]
    ld = [torch.empty_like(lse) for _ in range(2)]
    out_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    lse_host = [torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True) for _ in range(2)]
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        j, L = i % 2, layers[i % N_LAYERS]
        if i >= 2:
            up_s.wait_event(ev_comp[j])  # qd[j] is no longer read
        with torch.cuda.stream(up_s):
            qd[j].copy_(q_host[i % N_LAYERS], non_blocking=True)
        ev_up[j].record(up_s)
        stream.wait_event(ev_up[j])
        if i >= 2:
            stream.wait_event(ev_down[j])  # od[j], ld[j] are no longer read
        T.tls_decode_step(shape, qd[j], L.meta, L.slab, label, seq_lens, L.K, L.V, bidx, tidx, od[j], ld[j], None,
                          None, ws, sh)
        ev_comp[j].record(stream)
        down_s.wait_event(ev_comp[j])
        with torch.cuda.stream(down_s):
            out_host[j].copy_(od[j], non_blocking=True)
            lse_host[j].copy_(ld[j], non_blocking=True)
        ev_down[j].record(down_s)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up_s.wait_event(e0)
    for i in range(n_e2e):
        e2e_step(i)
    stream.wait_event(ev_down[(n_e2e - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h2d = layers[0].q.numel() * layers[0].q.element_size()
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()

    if rank != 0:
        return None, None
    ab = algorithmic_bytes(w)
    peaks = read_peaks()
    step_ms = ms / args.steps
    dom = int(np.argmax(stage_ms))  # the roofline's stage: the slower of the two calls
    dom_bytes = ab[names[dom]]
    achieved = dom_bytes / (stage_ms[dom] * 1e-3) / 1e9
    # a stage inside the step cannot take longer than the whole step; if the
    # separately timed stage does (it runs without the launch chain), say so
    consistent = bool(stage_ms[dom] <= step_ms * 1.05)
    if not consistent:
        print(f"warning: {names[dom]} mean {stage_ms[dom] * 1e3:.1f} us > step {step_ms * 1e3:.1f} us",
              file=sys.stderr)
    prof = read_profile(names[dom])
    res = {
        "metric": METRIC,
        "value": world * args.steps / (ms * 1e-3),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == 1 else "f32",
        "data": "synthetic: seeded Gaussian K/V with outlier channels and planted needle keys",
        "config": {
            "workload": args.workload, "batch": w.batch, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "d_qk": w.d_qk, "d_v": w.d_v, "ctx": w.ctx, "block_size": w.block_size, "k_b": w.k_b, "k_t": w.k_t,
            "n_label": w.n_label, "out_dtype": "f32", "label_slab": "int8" if w.slab_bits == 8 else "kv dtype",
            "block_agg": "max over heads" if w.block_agg == 1 else "sum over heads",
            "l2": f"inputs larger than L2: {N_LAYERS} layer copies rotated, {N_LAYERS * ab['total'] / 1e6:.0f} MB "
                  f"of algorithmic bytes per rotation (L2 126 MB)",
            "algorithmic_bytes_per_step": ab["total"],
        },
        "hbm_gbs": ab["total"] / (step_ms * 1e-3) / 1e9,
        "hbm_frac_of_measured": ab["total"] / (step_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "hbm_frac_of_8000": ab["total"] / (step_ms * 1e-3) / 1e9 / 8000.0,
        "stages_us": {n: float(v * 1e3) for n, v in zip(names, stage_ms)},
        "stages_median_us": {n: float(v * 1e3) for n, v in zip(names, stage_med)},
        "stage_timing": f"separate untimed pass of {n_stage} steps after the timed region: the step as its two "
                        f"calls (tls_select_step_ws, tls_sparse_attn_decode), CUDA events around each on every step "
                        f"(first step dropped); mean reported",
        "step_call": "tls_decode_step",
        "roofline": {
            "kernel": names[dom], "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
            "traffic": read_traffic(names[dom]), "algorithmic_bytes_per_launch": dom_bytes,
            "stage_us": float(stage_ms[dom] * 1e3), "samples": n_stage,
            "consistent_with_step": consistent,
            "cross_check": {
                "whole_step_gbs": ab["total"] / (step_ms * 1e-3) / 1e9,
                "profile_mean_us": prof.get("mean_us") if prof else None,
                "profile_frac": (dom_bytes / (prof["mean_us"] * 1e-6) / 1e9 / peaks["hbm_gbs"]
                                 if prof and prof.get("mean_us") else None),
                "profile_source": prof.get("capture") if prof else None,
            },
        },
        "e2e": {"value": world * n_e2e / (e2e_ms * 1e-3), "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    return res, inp


# ----------------------------------------------------------------------------- offload stream
def offload_arm(args):
    """The offload engine on the streaming workload (stream96k_bf16): the full KV
    lives in pinned host memory, a 2*K_b-slot block cache on the GPU.  One step:
    block top-K_b from q_t (compute stream); on a copy stream, tls_prefetch_diff
    loads the blocks of S(t) that are not resident over PCIe while the compute
    stream scores the tokens of S(t-1) and runs the paged attention (after the
    copy of step t-1).  The whole query stream is timed with CUDA events; the
    PCIe bytes per step come from an untimed replay that reads the copy counts."""
    import numpy as np
    import torch

    from two_level_sparse_quest_b200 import build as tls_build

    tls_build.build()
    from two_level_sparse_quest_b200 import tls as T
    from two_level_sparse_quest_b200 import workloads as W

    dev = torch.device("cuda", 0)
    w = W.WORKLOADS["stream96k_bf16"]
    s = T.shape_from_workload(w)
    inp = W.make_decode_inputs(w)
    qs = W.make_query_stream(w)
    steps = qs.shape[0]
    B, H, nb, bs, d = w.batch, w.n_kv_heads, w.n_blocks, w.block_size, w.d_qk
    n_slots = 2 * w.k_b

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)

    K = up(inp.K)
    sl, lab = up(inp.seq_lens), up(inp.label_idx)
    meta = torch.zeros((B, H, nb, 2, d), dtype=torch.int16, device=dev)
    slab = torch.zeros((B, H, w.ctx, w.n_label), dtype=torch.int16, device=dev)
    T.tls_build_block_meta(s, K, sl, lab, meta, slab)
    torch.cuda.synchronize()
    del K
    host_kv = torch.from_numpy(W.paged_host_kv(inp).view(np.int16)).pin_memory()
    cache = torch.zeros((B, H, n_slots, 2, bs, d), dtype=torch.int16, device=dev)
    sob = torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    bos = torch.empty((B, H, n_slots), dtype=torch.int32, device=dev)
    jobs = torch.empty((B, H, w.k_b, 2), dtype=torch.int32, device=dev)
    n_new = torch.empty((B, H), dtype=torch.int32, device=dev)
    ws = torch.zeros(T.tls_workspace_size(s), dtype=torch.uint8, device=dev)
    ring = [torch.empty((B, H, w.k_b), dtype=torch.int32, device=dev) for _ in range(3)]
    tidx = torch.empty((B, H, w.k_t), dtype=torch.int32, device=dev)
    out = torch.empty((B, w.n_q_heads, w.d_v), dtype=torch.float32, device=dev)
    lse = torch.empty((B, w.n_q_heads), dtype=torch.float32, device=dev)
    q_dev = [up(qs[t]) for t in range(steps)]
    compute = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)
    ev_sel = [torch.cuda.Event() for _ in range(2)]
    ev_copy = [torch.cuda.Event() for _ in range(2)]

    def run(count=False):
        T.tls_offload_reset(s, n_slots, sob, bos)
        copied = 0
        for t in range(steps):
            cur, prev = ring[t % 3], (ring[(t - 1) % 3] if t else None)
            T.tls_block_score_topk(s, q_dev[t], meta, sl, cur, None, ws)
            ev_sel[t % 2].record(compute)
            copy.wait_event(ev_sel[t % 2])
            T.tls_prefetch_diff(s, n_slots, host_kv, cache, sob, bos, prev, cur, n_new, jobs, stream=copy)
            ev_copy[t % 2].record(copy)
            T.tls_token_score_topk(s, q_dev[t], slab, lab, cur if t == 0 else prev, sl, tidx, None, ws)
            compute.wait_event(ev_copy[t % 2] if t == 0 else ev_copy[(t - 1) % 2])
            T.tls_sparse_attn_decode_paged(s, q_dev[t], cache, sob, n_slots, tidx, out, lse, ws)
            if count:
                torch.cuda.synchronize()
                copied += int(n_new.sum())
        compute.wait_event(ev_copy[(steps - 1) % 2])
        return copied

    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    copy.wait_event(e0)
    run()
    e1.record(compute)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    copied = run(count=True)
    block_bytes = 2 * bs * d * 2
    return {
        "metric": "offload decode steps/s (block select, PCIe prefetch of new blocks, paged attention)",
        "value": steps / (ms * 1e-3), "unit": "steps/s", "n_gpus": 1, "steps": steps,
        "ms_per_step": ms / steps, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic: seeded K/V, AR(1) query stream",
        "config": {"workload": "stream96k_bf16", "batch": B, "n_q_heads": w.n_q_heads, "n_kv_heads": H,
                   "d_qk": d, "ctx": w.ctx, "block_size": bs, "k_b": w.k_b, "k_t": w.k_t, "n_slots": n_slots,
                   "host_kv_bytes": int(host_kv.numel() * 2)},
        "pcie_bytes_per_step": copied * block_bytes / steps,
        "pcie_gbs": copied * block_bytes / (ms * 1e-3) / 1e9,
        "blocks_copied": copied, "first_step_blocks": B * H * w.k_b,
        "gpu_launches_per_step": 6,
    }


# ----------------------------------------------------------------------------- dense context
def dense_arm(args):
    """Full-attention decode of the same workload on the same GPU, for context:
    the attention kernels with every token of every sequence selected (K_t = n),
    so each step streams the whole K/V cache once.  Reports its time per step
    next to the sparse step's (measured the same way)."""
    import numpy as np
    import torch

    from two_level_sparse_quest_b200 import build as tls_build

    tls_build.build()
    from two_level_sparse_quest_b200 import tls as T
    from two_level_sparse_quest_b200 import workloads as W

    dev = torch.device("cuda", 0)
    w = W.WORKLOADS[args.workload]
    inp = W.make_decode_inputs(w)

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)

    q, K = up(inp.q), up(inp.K)
    V = up(inp.V) if inp.V is not None else None
    G = w.batch * w.n_kv_heads
    dense = T.shape_from_workload(w, k_t=w.ctx)
    all_tok = torch.arange(w.ctx, dtype=torch.int32, device=dev).repeat(G, 1).contiguous()
    ws = torch.zeros(T.tls_workspace_size(dense), dtype=torch.uint8, device=dev)
    out = torch.empty((w.batch, w.n_q_heads, w.d_v), dtype=torch.float32, device=dev)
    lse = torch.empty((w.batch, w.n_q_heads), dtype=torch.float32, device=dev)
    steps = max(3, min(args.steps, 50))
    for _ in range(3):
        T.tls_sparse_attn_decode(dense, q, K, V, all_tok, out, lse, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        T.tls_sparse_attn_decode(dense, q, K, V, all_tok, out, lse, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    kv_bytes = G * w.ctx * (w.d_qk + (0 if w.v_is_k_prefix else w.d_v)) * w.elem_bytes
    return {"metric": "dense decode attention (all tokens) per step, same kernels", "workload": args.workload,
            "dense_us_per_step": ms * 1e3, "dense_kv_bytes": kv_bytes, "dense_gbs": kv_bytes / (ms * 1e-3) / 1e9,
            "steps": steps, "input": "the whole cache is larger than L2, so no rotation is needed"}


# ----------------------------------------------------------------------------- CPU oracle
class OracleStep:
    """The fp64 oracle's decode step (stages 1-5 from the block summary on) on
    the host cores.  The step's (sequence, KV head) groups are independent, so
    each is its own oracle call on a one-group shape; a thread pool runs them
    concurrently (the oracle is C called through ctypes, which releases the
    GIL for the duration of each call).  The block summaries are built once,
    untimed, as the GPU side builds them once per KV cache."""

    def __init__(self, w, inp, threads: int):
        from concurrent.futures import ThreadPoolExecutor

        from oracle import oracle as O

        self.O, self.w, self.threads = O, w, threads
        G = w.group
        self.s = O.shape_of(w.with_(batch=1, n_kv_heads=1, n_q_heads=G))
        self.groups = []
        for b in range(w.batch):
            for g in range(w.n_kv_heads):
                self.groups.append(dict(
                    q=inp.q[b:b + 1, g * G:(g + 1) * G], K=inp.K[b:b + 1, g:g + 1],
                    V=None if inp.V is None else inp.V[b:b + 1, g:g + 1],
                    sl=inp.seq_lens[b:b + 1], label=inp.label_idx))
        self.pool = ThreadPoolExecutor(max_workers=threads)

        def meta(gr):
            gr["meta"] = O.build_meta(self.s, gr["K"], gr["sl"])

        list(self.pool.map(meta, self.groups))

    def _one(self, gr):
        self.O.decode_step(self.s, np.ascontiguousarray(gr["q"]), gr["K"], gr["V"], gr["meta"], gr["sl"], gr["label"])

    def run(self, n_groups=None, threads=True) -> float:
        """Seconds for the first n_groups groups (all by default), on the pool
        or on this thread alone."""
        todo = self.groups[:n_groups] if n_groups else self.groups
        t0 = time.perf_counter()
        if threads:
            list(self.pool.map(self._one, todo))
        else:
            for gr in todo:
                self._one(gr)
        return time.perf_counter() - t0


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_baseline(w, inp, budget_s: float) -> dict:
    """The oracle timed on all host cores on whole decode steps of the
    workload (a bounded number of them), plus one single-thread figure."""
    cores = host_cores()
    os_ = OracleStep(w, inp, cores)
    n_groups = len(os_.groups)
    # single thread: a few groups, scaled to the step (the groups are alike)
    k1 = max(1, min(n_groups, 4))
    t1 = os_.run(k1, threads=False) * n_groups / k1
    times = []
    t_all = time.time()
    while True:
        times.append(os_.run())
        if time.time() - t_all > budget_s or len(times) >= 10:
            break
    per_step = float(np.median(times))
    return {
        "value": 1.0 / per_step, "unit": "steps/s", "cores": cores, "kind": "oracle",
        "sample": f"{len(times)} whole decode step(s) of {args_workload_name(w)} (all {n_groups} (sequence, KV head) "
                  f"groups, stages 1-5 from the block summary), fp64, {cores} threads over the groups; median",
        "seconds_per_step": per_step,
        "single_thread": {"value": 1.0 / t1, "unit": "steps/s", "seconds_per_step": t1,
                          "sample": f"{k1} of {n_groups} groups on one thread, scaled x{n_groups / k1:g}"},
    }


def args_workload_name(w) -> str:
    return getattr(w, "name", "workload")


def reference_arm(args, rank, world):
    """The oracle as the reference arm: --warmup untimed and --steps timed
    decode steps of the workload on all host cores (rank 0 only).  When a
    whole step would not let the run end within a few minutes, each step is a
    fixed sample of the step's groups, scaled, and the line says so."""
    if rank != 0:
        return None
    from two_level_sparse_quest_b200 import workloads as W

    w = W.WORKLOADS[args.workload]
    inp = W.make_decode_inputs(w)
    cores = host_cores()
    os_ = OracleStep(w, inp, cores)
    n_groups = len(os_.groups)
    probe = os_.run(min(n_groups, cores))  # one round of the pool
    est_step = probe * math.ceil(n_groups / cores) if n_groups > cores else probe
    budget = 150.0
    n_sample = n_groups
    if est_step * (args.steps + args.warmup) > budget:
        n_sample = max(1, min(n_groups, int(n_groups * budget / (est_step * (args.steps + args.warmup)))))
    for _ in range(args.warmup):
        os_.run(n_sample)
    times = [os_.run(n_sample) * n_groups / n_sample for _ in range(args.steps)]
    total = float(np.sum(times))
    per_step = total / args.steps
    sample = (f"every step is the whole decode step ({n_groups} groups)" if n_sample == n_groups
              else f"every step runs {n_sample} of {n_groups} groups, scaled x{n_groups / n_sample:g}")
    cb = {"value": 1.0 / per_step, "unit": "steps/s", "cores": cores, "kind": "oracle",
          "sample": f"{args.warmup} warm-up + {args.steps} timed steps; {sample}; fp64, {cores} threads over the groups",
          "seconds_per_step": per_step}
    return {
        "metric": METRIC, "impl": "reference", "value": cb["value"], "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded Gaussian K/V with outlier channels and planted needle keys",
        "config": {"workload": args.workload, "batch": w.batch, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
                   "d_qk": w.d_qk, "d_v": w.d_v, "ctx": w.ctx, "block_size": w.block_size, "k_b": w.k_b,
                   "k_t": w.k_t, "n_label": w.n_label},
        "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "reference arm = the fp64 CPU oracle (no runnable reference implementation exists)",
    }


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="gqa96k_b8_bf16")
    ap.add_argument("--impl", default="tls", choices=["tls", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dense", action="store_true",
                    help="time full-attention decode (all tokens selected) of the workload, for context")
    ap.add_argument("--offload", action="store_true",
                    help="time the offload engine on the streaming workload instead (one JSON line of its own)")
    ap.add_argument("--block-agg", type=int, default=0, choices=[0, 1],
                    help="block score over a group's heads: 0 = the sum (the method), 1 = the maximum (variant)")
    ap.add_argument("--slab-bits", type=int, default=0, choices=[0, 8],
                    help="label slab storage: 0 = the K dtype (the method), 8 = int8 codes + per-channel scales")
    ap.add_argument("--layers", type=int, default=0,
                    help="layer copies rotated through (default: enough for twice the L2 per rotation, at least 4)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.dense:
        if rank == 0:
            print(json.dumps(dense_arm(args)), flush=True)
        return

    if args.offload:
        if rank == 0:
            print(json.dumps(offload_arm(args)), flush=True)
        return

    if args.impl == "reference":
        res = reference_arm(args, rank, world)
        if res:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res, inp = gpu_arm(args, rank, world, local_rank)
    if rank == 0 and res is not None:
        if world == 1 and not args.no_cpu_baseline:
            from two_level_sparse_quest_b200 import workloads as W

            res["cpu_baseline"] = oracle_baseline(W.WORKLOADS[args.workload], inp, budget_s=15.0)
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
