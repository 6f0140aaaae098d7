"""Benchmark of the hierarchical sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lf|reference] [--config 480p]

One step = one pass of the whole path over one synthetic chunk: (a) token compression,
(b) frame top-k and (c) block top-k through lf_select_chunk, then (d) block-sparse
attention through lf_block_sparse_attn, on inputs already resident in HBM.  The L2 cache
is flushed before every timed step, outside the step's event pair: 256 MB written, then
read back, so the timed kernels start from a cold L2 that holds no dirty lines of the
flush.  Reported: effective TFLOP/s = executed
attention FLOPs (4*d per valid query-key pair) / step time; ms per chunk; roofline of the
dominant kernel (attention, bf16 tensor cores) and of the selection (HBM); the e2e
figure through lf_forward_chunk with host buffers (pinned host -> device copy of the
chunk's Q/K/V, device -> host copy of the output inside the timed region; the KV cache is
state that stays resident); and the float64 oracle timed on the host cores on a bounded
sample.

Multi-GPU (torchrun): every rank runs its own chunk (independent video streams), no
collective on the data path; value = all ranks' FLOPs / max-over-ranks time (weak
scaling).  --impl reference times the float64 CPU oracle on the same config (rank 0 only).
"""
from __future__ import annotations

import argparse
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

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def block_lens(T, B):
    nb = -(-T // B)
    return np.array([min(B, T - b * B) for b in range(nb)], dtype=np.int64)


def executed_flops(shape, block_idx_np, cur_idx_np=None) -> int:
    """4*d per (head, query, valid key): current chunk (dense, or the kept current blocks
    of each query's block) + sinks dense, plus the tokens of the selected history blocks."""
    lens = block_lens(shape.T, shape.block)
    nb = len(lens)
    qlen = np.tile(lens, shape.n_cur_frames)                  # tokens per query block
    dense = (shape.n_cur_frames * shape.T if cur_idx_np is None else 0) + shape.n_sink * shape.T
    sel = np.zeros((shape.H, len(qlen)), dtype=np.int64)
    if shape.n_hist > 0 and block_idx_np is not None:
        sel = sel + lens[block_idx_np % nb].sum(axis=-1)
    if cur_idx_np is not None:
        sel = sel + lens[cur_idx_np % nb].sum(axis=-1)
    return int(4 * shape.d * (qlen[None, :] * (dense + sel)).sum())


def tail_split(shape, n_sm=148) -> bool:
    """Whether the attention launch splits its last, partial wave of tiles (mirrors the
    library's rule: the last wave is less than half full, and it can be cut into at least
    two key ranges of at least one key tile each)."""
    per = 2 if shape.block == 64 else 1
    nbpf = -(-shape.T // shape.block)
    nqb = shape.n_cur_frames * nbpf
    tiles = shape.H * -(-nqb // per)
    r = tiles % n_sm
    if r == 0 or 2 * r > n_sm:
        return False
    k_c = getattr(shape, "k_c", 0)
    kc = min(k_c, nqb) if k_c > 0 else 0
    nsel = (min(shape.k_f, shape.n_hist) * min(shape.k_b, nbpf)) if shape.n_hist > 0 else 0
    min_tiles = (0 if kc > 0 else -(-shape.n_cur_frames * shape.T // 128)) + \
        -(-(shape.n_sink * nbpf + kc + nsel) // per)
    return min(n_sm // r, 16, min_tiles) >= 2


def selection_launches(shape) -> int:
    """Kernels one lf_select_chunk call launches (mirrors the library's rule): pooling,
    block scores and pick when the fused path applies, else pooling, frame pooling, frame
    selection and block selection."""
    if shape.n_hist <= 0:
        return 0
    nbpf = -(-shape.T // shape.block)
    kf, kb = min(shape.k_f, shape.n_hist), min(shape.k_b, nbpf)
    fused = (shape.n_hist * nbpf <= 2048 and kf * kb <= 256 and shape.n_hist <= 256
             and nbpf <= 256)
    return 3 if fused else 4


def attn_sources_sha256() -> str:
    """Digest of the attention kernel's sources (the DRAM traffic figure taken from an ncu
    capture is reported only while the kernel is unchanged)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_46_b200", "csrc")
    for name in ("lf_attn.cuh", "lf_common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu figures of this workload
    (profiles/attn_kernel_<workload>.json), or None if there are none or the kernel's
    sources changed since they were taken."""
    path = os.path.join(ROOT, "profiles", f"attn_kernel_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        vals = json.load(f)
    if vals.get("source_sha256") != attn_sources_sha256():
        return None
    v = vals.get("dram_bytes_per_launch")
    return float(v) if v is not None else None


def max_over_ranks(x: float, device) -> float:
    """The largest value of x over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device) -> float:
    """The sum of x over all ranks (work done by the whole job)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def head_shard(H: int, world: int, rank: int):
    """Heads [h0, h1) of `rank` when H heads are split over `world` ranks: contiguous, the
    first H % world ranks one head more.  Heads are independent at every stage, so a
    sharded chunk needs no collective on the data path."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_heads(ci, h0: int, h1: int):
    """The chunk restricted to heads [h0, h1) (contiguous per-rank tensors)."""
    from dataclasses import replace
    part = lambda x: x[..., h0:h1, :].contiguous()
    return replace(ci, shape=replace(ci.shape, H=h1 - h0), q=part(ci.q), k_cur=part(ci.k_cur),
                   v_cur=part(ci.v_cur), k_cache=part(ci.k_cache), v_cache=part(ci.v_cache),
                   planted=ci.planted[h0:h1])


def weak_scaling_value(flops_per_rank: int, world: int, ms: float) -> float:
    """Whole-job TFLOP/s: every rank processed its own chunk in at most `ms`."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def selection_bytes(shape) -> int:
    return 2 * shape.H * shape.d * shape.T * (shape.n_cur_frames + shape.n_hist)


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.6)
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [l for (t, l) in self.lines if t0 - 0.15 <= t <= t1 + 0.15] or \
               [l for (_, l) in self.lines]
        return summarise_clocks(rows)


def summarise_clocks(rows):
    """Median SM clock, the highest reported maximum clock and the throttle reasons seen
    active, from nvidia-smi CSV rows in ClockSampler.Q's column order (malformed rows and
    rows without numbers are skipped)."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for l in rows:
        f = [x.strip() for x in l.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax.append(float(f[2]))
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(sm)}


CONFIG_NAMES = ("480p", "large", "rolling", "growth", "chunk1_80")


def make_workload(name, seed):
    """(chunks, description) of a benchmark workload.  A step processes every chunk of the
    list once: the 480p and large chunks alone, the rolling cache's steady-state chunk (3
    sink frames + the last 21 frames), or the 7 chunks of the growth sweep, whose (k_f,
    k_b) budgets come from the library's growth schedule (lf_cag_schedule)."""
    import lf_workloads as W
    if name == "480p":
        return [W.p480(seed)], "Self-Forcing-shaped 480p chunk: H=12 d=128 T=1560 (30x52), " \
                               "chunk 3 frames (4680 queries), 18 history frames, B=64, k_f=6, k_b=12"
    if name == "large":
        return [W.large(seed)], "large-model stress: H=40 d=128 T=1560, chunk 3, " \
                                "42 history frames, B=128, k_f=8, k_b=5"
    if name == "rolling":
        ci = None
        for ci in W.rolling(seed, n_chunks=9):
            pass
        return [ci], "rolling-cache steady state (chunk 9 of the 60-frame generation): H=12 " \
                     "d=128 T=1560, chunk 3 frames, 3 sink frames + 21 rolling history frames, " \
                     "B=64, k_f=4, k_b=6"
    if name == "growth":
        import block_sparse_attention_46_b200 as lf
        chunks = W.growth_sweep(seed)
        nbpf = -(-chunks[0].shape.T // chunks[0].shape.block)
        keep, kf, kb = lf.lf_cag_schedule(7, 2, 0.8, 0.9, [c.shape.n_hist for c in chunks],
                                          nbpf, 6)
        for c, f, b in zip(chunks, kf, kb):
            if c.shape.n_hist > 0 and (c.shape.k_f, c.shape.k_b) != (f, b):
                raise SystemExit(f"growth budget {(c.shape.k_f, c.shape.k_b)} != schedule {(f, b)}")
        return chunks, "chunk-aware growth sweep: 7 chunks of 3 frames at the 480p shape " \
                       "(H=12 d=128 T=1560, B=64), history 0,3,...,18 frames, keep ratio " \
                       "1 then mean 0.2 over chunks 2-7 (k_f, k_b from lf_cag_schedule: " + \
                       ", ".join(f"({a},{b})" for a, b in zip(kf, kb)) + ")"
    if name == "chunk1_80":
        from dataclasses import replace
        ci = W.growth_sweep(seed)[0]
        nqb = ci.shape.n_cur_frames * -(-ci.shape.T // ci.shape.block)
        k_c = nqb // 5                                       # keep 20%: 15 of 75 blocks
        return [replace(ci, shape=replace(ci.shape, k_c=k_c), name="chunk1_80")], \
            "first chunk at 80% sparsity inside the current chunk (no history): H=12 d=128 " \
            f"T=1560, chunk 3 frames, B=64, each query block keeps its own block + the " \
            f"{k_c - 1} best of the other {nqb - 1} current blocks"
    raise SystemExit(f"unknown config {name} (one of {', '.join(CONFIG_NAMES)})")


# ----------------------------------------------------------------------------- oracle
def oracle_sample(chunks, budget_s=0.0, first=0):
    """Runs the float64 oracle (a)-(d) one (chunk, head) at a time (each head of a chunk is
    an independent problem), starting at unit `first`, until `budget_s` seconds are spent
    (at least one unit): a bounded sample of the workload.  Returns (executed FLOPs of the
    sample, seconds, cores, units run)."""
    from dataclasses import replace
    from oracle import hsa64 as O
    import torch
    units = [(c, h) for c in range(len(chunks)) for h in range(chunks[c].shape.H)]
    flops, dt, n = 0, 0.0, 0
    for i in range(len(units)):
        c, h = units[(first + i) % len(units)]
        ci = chunks[c]
        s1 = replace(ci.shape, H=1)
        sl = lambda t: t[..., h:h + 1, :].contiguous()
        t0 = time.perf_counter()
        r = O.forward_chunk(s1, sl(ci.q), sl(ci.k_cur), sl(ci.v_cur), sl(ci.k_cache),
                            sl(ci.v_cache), ci.hist_slots, ci.sink_slots)
        dt += time.perf_counter() - t0
        flops += executed_flops(s1, r.get("block_idx"))
        n += 1
        if dt >= budget_s:
            break
    return flops, dt, torch.get_num_threads(), n


def oracle_single_core(chunks):
    """One head of the workload through the oracle with torch and the BLAS pools at one
    thread (the pools are restored afterwards).  Returns (FLOPs, seconds)."""
    import numpy  # noqa: F401  (loads the BLAS library so its pool can be limited)
    import torch
    from threadpoolctl import threadpool_limits
    n = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        with threadpool_limits(limits=1):
            f, dt, _, _ = oracle_sample(chunks[-1:])
    finally:
        torch.set_num_threads(n)
    return f, dt


def run_reference(args, rank, world):
    if rank != 0:
        return
    chunks, desc = make_workload(args.config, 0)
    for _ in range(min(args.warmup, 1)):
        oracle_sample(chunks)
    tot_f, tot_t, cores = 0, 0.0, 1
    for k in range(args.steps):
        f, t, cores, _ = oracle_sample(chunks, first=k)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = f"one (chunk, head) of the {args.config} workload per step ((a)-(d), float64 numpy)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": desc, "oracle_sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


METRIC = "ms/chunk & effective TFLOP/s, hierarchical sparse attn, 480p chunk shape"


# ----------------------------------------------------------------------------- GPU arm
class ChunkRun:
    """Device tensors and C-ABI calls of one chunk of a workload."""

    def __init__(self, lf, ci, dev, e4m3=False):
        import torch
        self.lf, self.ci, self.sh = lf, ci, ci.shape
        self.e4m3 = e4m3
        sh = self.sh
        nbpf, nqb, kf, kb = lf.derived(sh)
        self.t = {k: getattr(ci, k).to(dev) for k in ("q", "k_cur", "v_cur", "k_cache", "v_cache")}
        self.bidx = torch.empty(sh.H, nqb, max(kf * kb, 1), dtype=torch.int32, device=dev)
        self.kc = lf.current_blocks(sh)
        self.cidx = torch.empty(sh.H, nqb, max(self.kc, 1), dtype=torch.int32, device=dev)
        self.sws = torch.empty(max(lf.lf_select_workspace_size(sh), 256), dtype=torch.uint8,
                               device=dev)
        self.out = torch.empty_like(self.t["q"])
        self.lse = torch.empty(sh.H, self.t["q"].shape[0], device=dev)
        self.ws = torch.empty(max(lf.lf_attn_workspace_size(sh), 256), dtype=torch.uint8,
                              device=dev)
        # the one-call path (lf_forward_chunk): its own outputs and workspace
        self.out_f = torch.empty_like(self.t["q"])
        self.lse_f = torch.empty_like(self.lse)
        self.fws = torch.empty(max(lf.lf_forward_workspace_size(sh), 256), dtype=torch.uint8,
                               device=dev)
        if e4m3:
            # the cache's keys are quantised once (model state); the queries and the current
            # chunk's keys every step, with the per-head key scales of the cache and chunk
            t = self.t
            self.q8 = torch.empty(t["q"].shape, dtype=torch.uint8, device=dev)
            self.qs = torch.empty(t["q"].shape[0], sh.H, device=dev)
            self.ks = torch.empty(sh.H, device=dev)
            self.kc8 = torch.empty(t["k_cur"].shape, dtype=torch.uint8, device=dev)
            self.kh8 = torch.empty(t["k_cache"].shape, dtype=torch.uint8, device=dev)
            rows = t["k_cache"].view(-1, sh.H, sh.d)
            lf.lf_e4m3_head_scales([t["k_cur"], rows], self.ks)
            lf.lf_quantize_e4m3(rows, self.kh8.view(-1, sh.H, sh.d), head_scale=self.ks)

    def select(self):
        t = self.t
        if self.sh.n_hist > 0:
            self.lf.lf_select_chunk(self.sh, t["q"], t["k_cache"], self.ci.hist_slots, self.bidx,
                                    self.sws)
        if self.kc > 0:
            self.lf.lf_select_current(self.sh, t["q"], t["k_cur"], self.cidx, self.sws)

    def attend(self):
        t = self.t
        if self.e4m3:
            self.lf.lf_quantize_e4m3(t["q"], self.q8, row_scale=self.qs)
            self.lf.lf_quantize_e4m3(t["k_cur"], self.kc8, head_scale=self.ks)
            self.lf.lf_block_sparse_attn_e4m3(
                self.sh, self.q8, self.qs, self.kc8, t["v_cur"], self.kh8, t["v_cache"],
                self.ks, self.ci.hist_slots, self.ci.sink_slots, self.bidx, self.out, self.lse,
                self.ws, cur_idx=self.cidx if self.kc > 0 else None)
            return
        self.lf.lf_block_sparse_attn(self.sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"],
                                     t["v_cache"], self.ci.hist_slots, self.ci.sink_slots,
                                     self.bidx, self.out, self.lse, self.ws,
                                     cur_idx=self.cidx if self.kc > 0 else None)

    def forward(self):
        """Stages (a)-(d) of the chunk in one call; the attention takes the key plans the
        selection's pick kernel wrote (no plan kernel) when the current chunk is dense."""
        t = self.t
        self.lf.lf_forward_chunk(self.sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"],
                                 t["v_cache"], self.ci.hist_slots, self.ci.sink_slots,
                                 self.out_f, self.lse_f, None, self.fws)

    def forward_launches(self) -> int:
        # selection (+ the current-chunk choice) | plan unless the pick wrote the plans,
        # attn (+ merge)
        hist = self.sh.n_hist > 0
        sel = selection_launches(self.sh)
        cur = (1 if hist else 2) if self.kc > 0 else 0
        plans_ready = hist and sel == 3 and self.kc == 0
        return sel + cur + (0 if plans_ready else 1) + 1 + (1 if tail_split(self.sh) else 0)

    def flops(self) -> int:
        return executed_flops(self.sh, self.bidx.cpu().numpy(),
                              self.cidx.cpu().numpy() if self.kc > 0 else None)

    def launches(self) -> int:
        # selection kernels (+ current-chunk pooling and choice) | plan, attn (+ merge)
        return selection_launches(self.sh) + (2 if self.kc > 0 else 0) + 2 + \
            (1 if tail_split(self.sh) else 0) + (2 if self.e4m3 else 0)


def capture(fn, stream, cap):
    """fn() captured once into a CUDA graph on the side stream `cap`."""
    import torch
    g = torch.cuda.CUDAGraph()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            fn()
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    return g


def run_lf(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import block_sparse_attention_46_b200 as lf
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lf.load()
    if args.shard == "heads":
        # one workload split by heads over the ranks (strong scaling): same seed everywhere
        chunks, desc = make_workload(args.config, 0)
        split = []
        for ci in chunks:
            h0, h1 = head_shard(ci.shape.H, world, rank)
            if h1 <= h0:
                raise SystemExit(f"--shard heads needs at most H={ci.shape.H} ranks")
            split.append(shard_heads(ci, h0, h1))
        chunks = split
        desc += f"; heads split over {world} ranks"
    else:
        chunks, desc = make_workload(args.config, rank)
    runs = [ChunkRun(lf, ci, dev, e4m3=args.e4m3) for ci in chunks]
    if args.e4m3:
        desc += "; stage (d) with e4m3 queries and keys (QK^T on the FP8 tensor cores, " \
                "quantised in the step: queries per token, current keys per head) and bf16 values"
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2():
        # write 256 MB (> 126 MB of L2), then read it back: L2 ends up holding clean lines
        # of the flush buffer, so no dirty write-back is charged to the timed kernels
        flush.zero_()
        torch.sum(flush.view(torch.int64), dim=0, out=flush_sink)
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def sel_stage():
        for r in runs:
            r.select()

    def att_stage():
        for r in runs:
            r.attend()

    # The step is the one-call path, lf_forward_chunk per chunk (the e4m3 variant, which
    # has no one-call entry point, uses the stage calls).  The stage breakdown (selection,
    # attention) is timed separately through lf_select_chunk + lf_block_sparse_attn.
    use_fwd = not args.e4m3

    def fwd_stage():
        for r in runs:
            r.forward()

    # warm up eagerly, then capture each path in a CUDA graph (removes host overhead
    # between launches; the graphs replay exactly the kernels of the C-ABI calls)
    for _ in range(3):
        sel_stage()
        att_stage()
        if use_fwd:
            fwd_stage()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    g_sel, g_att = capture(sel_stage, stream, cap), capture(att_stage, stream, cap)
    g_fwd = capture(fwd_stage, stream, cap) if use_fwd else None

    def stage_step(record=False):
        if record:
            ev[0].record(stream)
        g_sel.replay()
        if record:
            ev[1].record(stream)
        g_att.replay()
        if record:
            ev[2].record(stream)

    def step(record=False):
        if not use_fwd:
            stage_step(record)
            return
        if record:
            ev[0].record(stream)
        g_fwd.replay()
        if record:
            ev[1].record(stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
        if use_fwd:
            flush_l2()
            stage_step()
    torch.cuda.synchronize()
    flops = sum(r.flops() for r in runs)
    sel_bytes = sum(selection_bytes(r.sh) for r in runs if r.sh.n_hist > 0)
    launches_per_step = sum(r.forward_launches() if use_fwd else r.launches() for r in runs)

    clocks = ClockSampler(local_rank)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    step_ms, sel_ms, att_ms = [], [], []
    for _ in range(args.steps):
        flush_l2()
        step(record=True)
        if use_fwd:
            ev[1].synchronize()
            step_ms.append(ev[0].elapsed_time(ev[1]))
        else:
            ev[2].synchronize()
            sel_ms.append(ev[0].elapsed_time(ev[1]))
            att_ms.append(ev[1].elapsed_time(ev[2]))
            step_ms.append(sel_ms[-1] + att_ms[-1])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.time()
    if use_fwd:
        # the stage breakdown, after the timed steps (same flush, same events)
        for _ in range(args.steps):
            flush_l2()
            stage_step(record=True)
            ev[2].synchronize()
            sel_ms.append(ev[0].elapsed_time(ev[1]))
            att_ms.append(ev[1].elapsed_time(ev[2]))
        torch.cuda.synchronize()
    clk = clocks.stop(t_wall0, t_wall1)
    assert lf.lf_device_status() == 0, "device status reported an error"
    if use_fwd:
        for r in runs:                 # the one-call path computes what the stage calls do
            assert torch.equal(r.out_f, r.out), "lf_forward_chunk differs from the stage calls"
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_step = total_ms / args.steps
    if args.shard == "heads":
        job_flops = sum_over_ranks(float(flops), dev)
        value = job_flops / (ms_step * 1e-3) / 1e12
    else:
        job_flops = float(world * flops)
        value = weak_scaling_value(flops, world, ms_step)

    single = len(runs) == 1 and runs[0].sh.n_hist > 0 and runs[0].kc == 0 and not args.e4m3
    inc = incremental_compression(lf, runs[0], args, stream, cap, ev, flush_l2, g_att) \
        if single else None
    abl = ablation_1d(lf, runs[0], args, stream, cap, ev, flush_l2) if single else None
    e2e = end_to_end(lf, runs, args, stream, dev, world, job_flops)

    pk, src = peaks()
    att_mean = statistics.mean(att_ms)
    sel_mean = statistics.mean(sel_ms)
    att_tflops = flops / (att_mean * 1e-3) / 1e12
    n_chunks = len(runs)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None, "dtype": "e4m3 QK^T, bf16 PV" if args.e4m3 else "bf16",
        "data": "synthetic (seeded; per-frame key centroids, planted related frames)",
        "config": {"workload": desc, "chunks_per_step": n_chunks,
                   "l2": "flushed before every timed step (256 MB written, then read back)",
                   "executed_gflop_per_step": flops / 1e9,
                   "selection_mb_per_step": sel_bytes / 1e6,
                   "ms_per_chunk": ms_step / n_chunks,
                   "step_api": ("lf_forward_chunk per chunk (the attention takes the key plans "
                                "the selection's pick kernel wrote)") if use_fwd else
                               "lf_select_chunk (+ lf_select_current) + quantisation + "
                               "lf_block_sparse_attn_e4m3",
                   "ms_selection_abc": sel_mean, "ms_attention_d": att_mean,
                   "stage_breakdown": "ms_selection_abc and ms_attention_d timed separately "
                                      "through lf_select_chunk and lf_block_sparse_attn",
                   "selection_share": sel_mean / (sel_mean + att_mean)},
        "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": att_tflops / pk["bf16_tflops"],
                     # the committed DRAM figures are the bf16 kernel's
                     "traffic": profiled_traffic(args.config)
                     if n_chunks == 1 and not args.e4m3 else None,
                     "kernel": "stage (d): plan + attn_kernel + merge (lf_block_sparse_attn)",
                     "peak_source": f"{src} bf16_tflops (burst)"},
        "e2e": e2e,
        "incremental_compression": inc,
        "ablation_1d": abl,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if sel_bytes > 0:
        sel_gbs = sel_bytes / (sel_mean * 1e-3) / 1e9
        line["roofline_selection"] = {
            "bound": "hbm", "achieved": sel_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": sel_gbs / pk["hbm_gbs"],
            "kernels": "pool_blocks + block_scores + select_pick (lf_select_chunk)",
            "peak_source": f"{src} hbm_gbs"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, dt, cores, n = oracle_sample(chunks, budget_s=10.0)
        f1, dt1 = oracle_single_core(chunks)
        line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle", "seconds": dt,
                                "sample": f"{n} (chunk, head) units of the workload in order: "
                                          f"(a)-(d) float64 numpy, head by head",
                                "single_core": {"value": f1 / dt1 / 1e12, "unit": "TFLOP/s",
                                                "seconds": dt1,
                                                "sample": "head 0 of the last chunk, one thread"}}
    if rank == 0:
        print(json.dumps(line), flush=True)


def incremental_compression(lf, r, args, stream, cap, ev, flush_l2, g_att):
    """History block means kept per cache slot (the pooled-key cache): per step the frames
    that enter the cache (three slots re-pooled here, their keys unchanged, so the
    selection is the same) are pooled and the selection reads the pooled-key cache."""
    import torch
    sh, t, ci = r.sh, r.t, r.ci
    dev = t["q"].device
    k_pool = torch.empty(lf.lf_pooled_cache_bytes(sh) // 4, dtype=torch.float32, device=dev)
    lf.lf_pool_frames(sh, t["k_cache"], sorted(set(ci.hist_slots)), k_pool)
    new_slots = list(ci.hist_slots[:sh.n_cur_frames])
    bidx_c = torch.empty_like(r.bidx)

    def sel_cached():
        lf.lf_pool_frames(sh, t["k_cache"], new_slots, k_pool)
        lf.lf_select_chunk_cached(sh, t["q"], k_pool, ci.hist_slots, bidx_c, r.sws)
    for _ in range(3):
        sel_cached()
    torch.cuda.synchronize()
    g_selc = capture(sel_cached, stream, cap)
    selc_ms, attc_ms = [], []
    for _ in range(max(3, min(args.steps, 200))):
        flush_l2()
        ev[0].record(stream)
        g_selc.replay()
        ev[1].record(stream)
        g_att.replay()
        ev[2].record(stream)
        ev[2].synchronize()
        selc_ms.append(ev[0].elapsed_time(ev[1]))
        attc_ms.append(ev[1].elapsed_time(ev[2]))
    same = bool(torch.equal(bidx_c, r.bidx))
    inc_bytes = 2 * sh.H * sh.d * sh.T * (2 * sh.n_cur_frames)      # Q + the new frames' K
    selc_mean = max_over_ranks(statistics.mean(selc_ms), dev)
    return {"ms_selection_abc": selc_mean,
            "ms_per_step": selc_mean + max_over_ranks(statistics.mean(attc_ms), dev),
            "selection_mb_per_chunk": inc_bytes / 1e6,
            "selection_gbs": inc_bytes / (selc_mean * 1e-3) / 1e9,
            "indices_equal_full_recompute": same,
            "api": "lf_pool_frames (the chunk's frames entering the cache) + "
                   "lf_select_chunk_cached, then lf_block_sparse_attn"}


def ablation_1d(lf, r, args, stream, cap, ev, flush_l2):
    """The one-dimensional ablation (no frame stage): its selection and the attention over
    the blocks it selects (the same number per query block, not clustered by frame)."""
    import torch
    sh, t, ci = r.sh, r.t, r.ci
    if sh.n_hist * -(-sh.T // sh.block) > 2048:
        return None
    dev = t["q"].device
    bidx_1d = torch.empty_like(r.bidx)
    out_1d = torch.empty_like(r.out)
    ws_1d = torch.empty_like(r.ws)

    def stages_1d():
        lf.lf_select_chunk_1d(sh, t["q"], t["k_cache"], ci.hist_slots, bidx_1d, r.sws)
        lf.lf_block_sparse_attn(sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"],
                                t["v_cache"], ci.hist_slots, ci.sink_slots, bidx_1d,
                                out_1d, None, ws_1d)
    for _ in range(3):
        stages_1d()
    torch.cuda.synchronize()
    g_1d = capture(stages_1d, stream, cap)
    ms_1d = []
    for _ in range(max(3, min(args.steps, 200))):
        flush_l2()
        ev[0].record(stream)
        g_1d.replay()
        ev[1].record(stream)
        ev[1].synchronize()
        ms_1d.append(ev[0].elapsed_time(ev[1]))
    f1d = executed_flops(sh, bidx_1d.cpu().numpy())
    m1d = max_over_ranks(statistics.mean(ms_1d), dev)
    return {"ms_per_step": m1d, "executed_gflop_per_chunk": f1d / 1e9,
            "tflops": f1d / (m1d * 1e-3) / 1e12,
            "api": "lf_select_chunk_1d + lf_block_sparse_attn"}


def end_to_end(lf, runs, args, stream, dev, world, job_flops):
    """The metric through lf_forward_chunk with host buffers: every chunk of every step
    copies its Q, K, V from pinned host memory, runs the call, and copies the output back.
    Two chunks are in flight: uploads, compute and downloads run on three streams
    (separate copy engines), with double-buffered device inputs/outputs; the KV cache is
    model state and stays resident."""
    import torch
    n = len(runs)
    hq = [{k: r.t[k].cpu().pin_memory() for k in ("q", "k_cur", "v_cur")} for r in runs]
    dq = [{k: torch.empty_like(runs[0].t[k]) for k in ("q", "k_cur", "v_cur")} for _ in range(2)]
    dout = [torch.empty_like(runs[0].out) for _ in range(2)]
    hout = [torch.empty(runs[0].out.shape, dtype=runs[0].out.dtype, pin_memory=True)
            for _ in range(2)]
    fws = torch.empty(max(lf.lf_forward_workspace_size(r.sh) for r in runs), dtype=torch.uint8,
                      device=dev)
    steps = max(4, min(args.steps, 50 // n if n > 1 else 50))
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for r in runs:
        assert r.t["q"].shape == runs[0].t["q"].shape    # one buffer shape serves every chunk

    def run(n_steps):
        for i in range(n_steps * n):
            b, c = i % 2, i % n
            r = runs[c]
            if i >= 2:
                s_in.wait_event(ev_comp[b])          # chunk i-2 has consumed these inputs
            with torch.cuda.stream(s_in):
                for k in hq[c]:
                    dq[b][k].copy_(hq[c][k], non_blocking=True)
            ev_in[b].record(s_in)
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])         # chunk i-2's output has been read back
            lf.lf_forward_chunk(r.sh, dq[b]["q"], dq[b]["k_cur"], dq[b]["v_cur"],
                                r.t["k_cache"], r.t["v_cache"], r.ci.hist_slots,
                                r.ci.sink_slots, dout[b], None, None, fws, stream=s_comp)
            ev_comp[b].record(s_comp)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                hout[b].copy_(dout[b], non_blocking=True)
            ev_out[b].record(s_out)

    run(1)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    s_in.wait_stream(stream)
    e0.record(s_in)
    run(steps)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    last = (steps * n - 1)
    same = bool(torch.equal(hout[last % 2], runs[last % n].out.cpu()))
    h2d = sum(sum(x.numel() * x.element_size() for x in h.values()) for h in hq)
    d2h = n * hout[0].numel() * hout[0].element_size()
    return {"value": job_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": "lf_forward_chunk per chunk, two chunks in flight (uploads, compute and "
                   "downloads on three streams)",
            "output_equals_device_path": same}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lf", choices=["lf", "reference"])
    ap.add_argument("--config", default="480p", choices=CONFIG_NAMES)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e4m3", action="store_true",
                    help="stage (d) with e4m3 queries and keys (lf_block_sparse_attn_e4m3)")
    ap.add_argument("--shard", default="chunks", choices=["chunks", "heads"],
                    help="chunks: one chunk per rank (weak scaling); heads: one chunk split "
                         "by heads over the ranks (strong scaling)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        args.steps = min(args.steps, 30)     # ~1 s of oracle work per step
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_lf(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
