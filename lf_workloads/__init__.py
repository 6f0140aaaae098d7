"""Seeded synthetic inputs for the hierarchical sparse attention (HSA) path.

This module is shared by the float64 oracle's tests and by the CUDA path's tests and
benchmark.  It holds shapes and random tensors only: no pooling, scoring, selection or
attention arithmetic lives here, so neither side can inherit the other's mistakes.

Workloads follow the chunk-wise autoregressive video setting of the Light Forcing pages
(480p latent frames of 30x52 = 1560 tokens, chunks of 3 latent frames, a KV cache of
earlier frames) and the rolling KV cache with sink frames of the Self Forcing and Rolling
Forcing articles.  The trained models, prompts and videos behind those pages are not
available; the tensors below stand in for their attention inputs with the same shapes
and a comparable structure (per-frame key centroids so that selection is not trivial).

Seeding: numpy ``Generator(PCG64)`` streams spawned from one ``SeedSequence(seed)`` in a
fixed order; values are drawn in float32 and rounded once to bfloat16 (round to nearest
even, by torch).  Both sides consume those bf16 bits.  ``N(0, s)`` means standard
deviation ``s``.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Iterator, List, Optional

import numpy as np
import torch

__all__ = [
    "Shape", "ChunkInputs", "tiny", "p480", "large", "random_small",
    "growth_sweep", "rolling", "GROWTH_KEEP", "GROWTH_TOPK", "CONFIGS",
]


@dataclass(frozen=True)
class Shape:
    """Plain problem sizes of one attention call (no derived quantities)."""
    H: int                 # heads
    d: int                 # head dimension
    T: int                 # tokens per latent frame
    block: int             # block size B in tokens
    n_cur_frames: int      # F_c, frames in the current chunk
    n_hist: int            # F, selectable history frames
    n_sink: int            # S_k, always-dense sink frames
    n_slots: int           # frames the KV cache tensor can hold
    k_f: int               # frames kept per query block
    k_b: int               # blocks kept per chosen frame
    scale: float           # softmax scale (1/sqrt(d))
    k_c: int = 0           # current-chunk blocks kept per query block (0: dense)


@dataclass
class ChunkInputs:
    """One attention call: current chunk Q/K/V and the KV cache with its slot lists.

    q, k_cur, v_cur: bf16 [n_cur_frames*T, H, d] (token-major, raster order per frame).
    k_cache, v_cache: bf16 [n_slots, T, H, d].
    hist_slots: cache slot of each history frame, oldest first.
    sink_slots: cache slot of each sink frame, oldest first.
    planted: int [H, n_cur_frames], history position each current frame's queries were
        drawn towards (-1 where none); used only by a soft recovery check.
    """
    shape: Shape
    q: torch.Tensor
    k_cur: torch.Tensor
    v_cur: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    hist_slots: List[int]
    sink_slots: List[int]
    planted: np.ndarray = field(default=None)
    name: str = ""


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _streams(seed: int, n: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(n)]


def _normal(g: np.random.Generator, shape, std=1.0) -> np.ndarray:
    return g.standard_normal(shape, dtype=np.float32) * np.float32(std)


def tiny_shape() -> Shape:
    return Shape(H=2, d=64, T=256, block=64, n_cur_frames=1, n_hist=4, n_sink=0,
                 n_slots=4, k_f=2, k_b=2, scale=1.0 / 8.0)


def p480_shape() -> Shape:
    return Shape(H=12, d=128, T=1560, block=64, n_cur_frames=3, n_hist=18, n_sink=0,
                 n_slots=18, k_f=6, k_b=12, scale=1.0 / float(np.sqrt(128.0)))


def large_shape() -> Shape:
    return Shape(H=40, d=128, T=1560, block=128, n_cur_frames=3, n_hist=42, n_sink=0,
                 n_slots=42, k_f=8, k_b=5, scale=1.0 / float(np.sqrt(128.0)))


def _ring_slots(n_hist: int, n_slots: int, start: int) -> List[int]:
    """Slot ids of a ring-buffer cache whose oldest frame sits at ``start``."""
    return [(start + i) % n_slots for i in range(n_hist)]


def _centroid_chunk(shape: Shape, seed: int, name: str, offset_std: float,
                    q_pull: float, plant: bool, slot_start: int = 0) -> ChunkInputs:
    """Frames with per-(head, frame) key centroids; queries optionally pulled towards one
    planted history frame per current frame."""
    H, d, T, Fc, F = shape.H, shape.d, shape.T, shape.n_cur_frames, shape.n_hist
    gq, gk, gv, gc, gp = _streams(seed, 5)
    n_frames = F + shape.n_sink + Fc
    cent = _normal(gc, (H, n_frames, d), offset_std)        # frame order: sinks, hist, cur
    planted = np.full((H, Fc), -1, dtype=np.int64)
    if plant and F > 0:
        planted = gp.integers(0, F, size=(H, Fc))
    k_cache = np.zeros((shape.n_slots, T, H, d), dtype=np.float32)
    v_cache = np.zeros((shape.n_slots, T, H, d), dtype=np.float32)
    hist_slots = _ring_slots(F, shape.n_slots - shape.n_sink, slot_start)
    hist_slots = [shape.n_sink + s for s in hist_slots]
    sink_slots = list(range(shape.n_sink))
    frame_slots = sink_slots + hist_slots
    for i, slot in enumerate(frame_slots):
        k_cache[slot] = _normal(gk, (T, H, d)) + cent[:, i, :][None, :, :]
        v_cache[slot] = _normal(gv, (T, H, d))
    k_cur = np.empty((Fc * T, H, d), dtype=np.float32)
    v_cur = np.empty((Fc * T, H, d), dtype=np.float32)
    q = np.empty((Fc * T, H, d), dtype=np.float32)
    for j in range(Fc):
        rows = slice(j * T, (j + 1) * T)
        k_cur[rows] = _normal(gk, (T, H, d)) + cent[:, len(frame_slots) + j, :][None]
        v_cur[rows] = _normal(gv, (T, H, d))
        pull = np.zeros((H, d), dtype=np.float32)
        if plant and F > 0:
            pull = q_pull * cent[np.arange(H), shape.n_sink + planted[:, j], :]
        q[rows] = _normal(gq, (T, H, d)) + pull[None]
    return ChunkInputs(shape, _bf16(q), _bf16(k_cur), _bf16(v_cur), _bf16(k_cache),
                       _bf16(v_cache), hist_slots, sink_slots, planted, name)


def tiny(seed: int = 0) -> ChunkInputs:
    """Tiny check: H=2, d=64, T=256 (16x16), 4 history frames, 1 current frame, B=64,
    k_f=2, k_b=2.  Q, K, V ~ N(0,1); K gets a per-(frame, head) offset ~ N(0, 0.5)."""
    return _centroid_chunk(tiny_shape(), seed, "tiny", 0.5, 0.0, False, slot_start=1)


def p480(seed: int = 0) -> ChunkInputs:
    """480p chunk: H=12, d=128, T=1560 (30x52), chunk of 3 frames (4680 queries),
    18 history frames (28080 keys), B=64, k_f=6, k_b=12 (half of 25 blocks).
    K = N(0,1) + c[h,f] with c ~ N(0,0.5); Q = N(0,1) + 0.5*c[h, planted frame]."""
    return _centroid_chunk(p480_shape(), seed, "480p", 0.5, 0.5, True, slot_start=5)


def large(seed: int = 0, n_hist: Optional[int] = None) -> ChunkInputs:
    """Large-model stress: H=40, d=128, T=1560, chunk 3, 42 history frames, B=128,
    k_f=8, k_b=5 (40% of 13).  Per head a basis U (16 x d, N(0, 1/16)); per (head, frame)
    coefficients a ~ N(0,1); K = a_K U + N(0,1), Q = a_Q U + N(0,1); V ~ N(0,1)."""
    shape = large_shape()
    if n_hist is not None:
        shape = replace(shape, n_hist=n_hist, n_slots=n_hist)
    H, d, T, Fc, F = shape.H, shape.d, shape.T, shape.n_cur_frames, shape.n_hist
    gq, gk, gv, gu, ga = _streams(seed, 5)
    U = _normal(gu, (H, 16, d), 1.0 / 16.0)
    k_cache = np.empty((shape.n_slots, T, H, d), dtype=np.float32)
    v_cache = np.empty((shape.n_slots, T, H, d), dtype=np.float32)
    hist_slots = _ring_slots(F, shape.n_slots, 7 % max(shape.n_slots, 1))
    for f in range(F):
        a = _normal(ga, (H, 16))
        k_cache[hist_slots[f]] = _normal(gk, (T, H, d)) + np.einsum("hr,hrd->hd", a, U)[None]
        v_cache[hist_slots[f]] = _normal(gv, (T, H, d))
    q = np.empty((Fc * T, H, d), dtype=np.float32)
    k_cur = np.empty((Fc * T, H, d), dtype=np.float32)
    v_cur = np.empty((Fc * T, H, d), dtype=np.float32)
    for j in range(Fc):
        rows = slice(j * T, (j + 1) * T)
        aq = _normal(ga, (H, 16))
        ak = _normal(ga, (H, 16))
        q[rows] = _normal(gq, (T, H, d)) + np.einsum("hr,hrd->hd", aq, U)[None]
        k_cur[rows] = _normal(gk, (T, H, d)) + np.einsum("hr,hrd->hd", ak, U)[None]
        v_cur[rows] = _normal(gv, (T, H, d))
    return ChunkInputs(shape, _bf16(q), _bf16(k_cur), _bf16(v_cur), _bf16(k_cache),
                       _bf16(v_cache), hist_slots, [], np.full((H, Fc), -1), "large")


def random_small(seed: int, H: int, d: int, T: int, block: int, n_cur_frames: int,
                 n_hist: int, n_sink: int, k_f: int, k_b: int,
                 extra_slots: int = 1, k_c: int = 0) -> ChunkInputs:
    """Small random shape for parity sweeps: centroids N(0, 0.5), planted queries, and a
    cache with spare slots (unused slots are filled too, so a wrong slot id shows)."""
    n_slots = n_hist + n_sink + extra_slots
    shape = Shape(H=H, d=d, T=T, block=block, n_cur_frames=n_cur_frames, n_hist=n_hist,
                  n_sink=n_sink, n_slots=n_slots, k_f=k_f, k_b=k_b,
                  scale=1.0 / float(np.sqrt(d)), k_c=k_c)
    ci = _centroid_chunk(shape, seed, f"rand{seed}", 0.5, 0.5, True,
                         slot_start=seed % max(n_slots - n_sink, 1))
    g = _streams(seed + 1000, 1)[0]
    used = set(ci.hist_slots) | set(ci.sink_slots)
    for s in range(n_slots):
        if s not in used:
            ci.k_cache[s] = _bf16(_normal(g, (T, H, d), 3.0))
            ci.v_cache[s] = _bf16(_normal(g, (T, H, d), 3.0))
    return ci


# Chunk-aware growth sweep: keep ratio per chunk (the input array of the growth schedule,
# s_i = s_base - alpha_i * beta with alpha_i = 1/sqrt(i), mean sparsity 80% over chunks
# 2-7 and 90% at chunk 7), and the integer (k_f, k_b) budget each ratio maps to
# (k_f = min(6, F); k_b = clamp(floor(r * F * n_bpf / k_f + 0.5), 1, n_bpf)).
GROWTH_KEEP = [1.0, 0.3633, 0.2595, 0.1976, 0.1554, 0.1242, 0.1000]
GROWTH_TOPK = [(0, 0), (3, 9), (6, 6), (6, 7), (6, 8), (6, 8), (6, 8)]


def growth_sweep(seed: int = 0) -> List[ChunkInputs]:
    """7 sequential chunks of 3 frames at the 480p shape; history grows 0, 3, ..., 18."""
    base = p480_shape()
    out = []
    for i, (kf, kb) in enumerate(GROWTH_TOPK):
        F = 3 * i
        shape = replace(base, n_hist=F, n_slots=max(F, 1), k_f=max(kf, 1), k_b=max(kb, 1))
        out.append(_centroid_chunk(shape, seed + i, f"growth{i + 1}", 0.5, 0.5, True))
    return out


def rolling(seed: int = 0, n_chunks: int = 20, window: int = 21, n_sink: int = 3,
            shape: Optional[Shape] = None) -> Iterator[ChunkInputs]:
    """Rolling-cache generation: chunks of 3 frames; sinks are the first chunk's frames;
    the cache keeps the last ``window`` non-sink frames (oldest evicted first).  Key
    centroids follow a random walk c_{f+1} = c_f + N(0, 0.1), c_0 ~ N(0, 1).
    k_f = min(4, F), k_b = 6 (25% of 25)."""
    base = shape or replace(p480_shape(), k_f=4, k_b=6)
    H, d, T, Fc = base.H, base.d, base.T, base.n_cur_frames
    n_slots = n_sink + window
    n_frames = n_chunks * Fc
    gq, gk, gv, gc, gp = _streams(seed, 5)
    steps = _normal(gc, (H, n_frames, d), 0.1)
    steps[:, 0, :] = _normal(gc, (H, d), 1.0)
    cent = np.cumsum(steps, axis=1)
    k_cache = torch.zeros((n_slots, T, H, d), dtype=torch.bfloat16)
    v_cache = torch.zeros((n_slots, T, H, d), dtype=torch.bfloat16)

    def frame_slot(f: int) -> int:
        return f if f < n_sink else n_sink + (f - n_sink) % window

    for c in range(n_chunks):
        cur = list(range(c * Fc, (c + 1) * Fc))
        sinks = [f for f in range(n_sink) if f < c * Fc]
        hist = [f for f in range(n_sink, c * Fc)][-window:]
        planted = np.full((H, Fc), -1, dtype=np.int64)
        q = np.empty((Fc * T, H, d), dtype=np.float32)
        k_cur = np.empty((Fc * T, H, d), dtype=np.float32)
        v_cur = np.empty((Fc * T, H, d), dtype=np.float32)
        for j, f in enumerate(cur):
            rows = slice(j * T, (j + 1) * T)
            k_cur[rows] = _normal(gk, (T, H, d)) + cent[:, f, :][None]
            v_cur[rows] = _normal(gv, (T, H, d))
            if hist:
                planted[:, j] = gp.integers(0, len(hist), size=H)
                pull = 0.5 * cent[np.arange(H), np.array(hist)[planted[:, j]], :]
            else:
                pull = 0.5 * cent[:, f, :]
            q[rows] = _normal(gq, (T, H, d)) + pull[None]
        shape_c = replace(base, n_hist=len(hist), n_sink=len(sinks), n_slots=n_slots,
                          k_f=min(base.k_f, max(len(hist), 1)))
        kc, vc = _bf16(k_cur), _bf16(v_cur)
        yield ChunkInputs(shape_c, _bf16(q), kc, vc, k_cache, v_cache,
                          [frame_slot(f) for f in hist], [frame_slot(f) for f in sinks],
                          planted, f"rolling{c + 1}")
        # the finished chunk enters the cache; a full window evicts its oldest frame
        for j, f in enumerate(cur):
            rows = slice(j * T, (j + 1) * T)
            k_cache[frame_slot(f)] = kc[rows]
            v_cache[frame_slot(f)] = vc[rows]


CONFIGS = {"tiny": tiny, "480p": p480, "large": large}
