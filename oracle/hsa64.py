"""Float64 CPU oracle of Light Forcing's hierarchical sparse attention (HSA).

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA path and must never be used
as a fallback for it.

It restates, step by step and in the pages' order, what the method computes:

  [LF-gist]  "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
             Attention" (gist.science explainer), section 2.2, Hierarchical Sparse
             Attention: token compression by mean pooling at block and frame granularity;
             two-stage mask selection (frames by frame-level compressed keys for each
             query block, then blocks inside the chosen frames by block-level compressed
             keys); attention computed only on the chosen frame-block pairs, at a cost
             that does not grow with the number of history frames.
  [LF-yly]   "南洋理工大学AI新突破 视频生成引擎模仿人脑高效学习" (m.youleyou.com),
             section 三 (hierarchical sparse attention): compression of the current
             queries per block and of the history keys per block and per frame; frame
             retrieval by inner-product similarity; block choice inside chosen frames;
             block-level mask fed to a sparse attention kernel.
  [SF]       Self Forcing article (rushgoaltv.com page), rolling KV cache paragraph:
             a fixed-size cache of the last L frames, oldest evicted first.
  [RF]       "南洋理工大学突破：AI实现实时流式视频生成" (163.com, Rolling Forcing),
             section 三: the first frames kept as a permanent attention anchor (sinks)
             beside the recent-frame cache.

Readings where the pages are silent (each one is listed with its reason in the design
notes): blocks are 1-D, frame-aligned runs of B tokens in raster order with a shorter
last block; a frame's pooled key is the mean over all of its tokens; scores are
unscaled dot products; top-k keeps the k largest, ties going to the lower index, and
index lists are returned ascending; k_b blocks are kept in EACH chosen frame; the current
chunk and the sink frames are always attended densely and are never candidates; the
softmax is one joint softmax over current + sink + selected keys with scale 1/sqrt(d).
Optionally (k_c > 0) the current chunk is sparse too: its keys are mean-pooled per block
like the queries, and each query block keeps its own block plus the k_c - 1 other
current-chunk blocks with the largest q_blk . k_blk (ties to the lower index).

All arithmetic is float64 on values upcast from the bf16 inputs.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

__all__ = [
    "block_bounds", "n_blocks", "compress_queries", "compress_keys", "frame_scores",
    "topk_lower_index", "select_frames", "block_scores_in_frame", "select_blocks",
    "key_set", "attention_qblock", "attention", "forward_chunk", "boundary_gap",
    "select_blocks_1d", "select_current_blocks", "current_boundary_gap", "executed_flops",
]


# ----------------------------------------------------------------------------- blocks
def n_blocks(T: int, B: int) -> int:
    """Blocks per frame: ceil(T / B)."""
    return -(-T // B)


def block_bounds(T: int, B: int) -> List[Tuple[int, int]]:
    """Token ranges [start, end) of the blocks of one frame (reading: 1-D, raster order,
    frame-aligned; the last block holds the T mod B leftover tokens)."""
    return [(b * B, min((b + 1) * B, T)) for b in range(n_blocks(T, B))]


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):          # torch tensor (bf16 on CPU)
        import torch
        return x.detach().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# ------------------------------------------------------------------ (a) compression
def compress_queries(q, T: int, B: int) -> np.ndarray:
    """[LF-gist 2.2, token compression; LF-yly 三, stage 1] Mean-pool the current chunk's
    queries per block.  q: [F_c*T, H, d] -> q_blk: [H, F_c*n_bpf, d].  Query block
    index = frame * n_bpf + block; a short last block is averaged over its true length."""
    q = _f64(q)
    n_tok, H, d = q.shape
    Fc = n_tok // T
    bounds = block_bounds(T, B)
    out = np.empty((H, Fc * len(bounds), d))
    for f in range(Fc):
        for b, (s, e) in enumerate(bounds):
            out[:, f * len(bounds) + b, :] = q[f * T + s: f * T + e].mean(axis=0)
    return out


def compress_keys(k_cache, hist_slots: Sequence[int], T: int, B: int):
    """[LF-gist 2.2, token compression; LF-yly 三, stage 1] Mean-pool the history keys per
    block and per frame.  k_cache: [n_slots, T, H, d]; hist_slots lists the cache slot of
    each history frame (oldest first).  Returns k_blk [H, F, n_bpf, d] and
    k_frm [H, F, d] (mean over all T tokens of the frame)."""
    kc = k_cache
    bounds = block_bounds(T, B)
    F = len(hist_slots)
    H, d = kc.shape[2], kc.shape[3]
    k_blk = np.empty((H, F, len(bounds), d))
    k_frm = np.empty((H, F, d))
    for f, slot in enumerate(hist_slots):
        frame = _f64(kc[slot])                       # [T, H, d]
        for b, (s, e) in enumerate(bounds):
            k_blk[:, f, b, :] = frame[s:e].mean(axis=0)
        k_frm[:, f, :] = frame.mean(axis=0)
    return k_blk, k_frm


# ------------------------------------------------------------- (b), (c) selection
def topk_lower_index(scores: Sequence[float], k: int) -> List[int]:
    """The k largest scores; equal scores go to the lower index.  Returned ascending."""
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], i))
    return sorted(order[:min(k, len(scores))])


def boundary_gap(scores: Sequence[float], k: int) -> float:
    """Relative score gap at the k-th boundary, (s_(k) - s_(k+1)) / max(|s_(k)|, 1e-30),
    with s sorted descending; +inf when every candidate is kept."""
    s = sorted((float(x) for x in scores), reverse=True)
    if k >= len(s) or k <= 0:
        return math.inf
    return (s[k - 1] - s[k]) / max(abs(s[k - 1]), 1e-30)


def frame_scores(q_blk: np.ndarray, k_frm: np.ndarray) -> np.ndarray:
    """[LF-gist 2.2, frame selection; LF-yly 三, inner-product similarity] Score of every
    history frame for every query block: sf[h, qb, f] = q_blk[h, qb] . k_frm[h, f]."""
    H, nqb, _ = q_blk.shape
    F = k_frm.shape[1]
    sf = np.empty((H, nqb, F))
    for h in range(H):
        for qb in range(nqb):
            for f in range(F):
                sf[h, qb, f] = np.dot(q_blk[h, qb], k_frm[h, f])
    return sf


def select_frames(q_blk: np.ndarray, k_frm: np.ndarray, k_f: int):
    """[LF-gist 2.2, stage 1 of mask selection] For each (head, query block) keep the
    k_f best-scoring history frames.  Returns frame_idx [H, n_qb, min(k_f, F)] (history
    positions, ascending) and the scores [H, n_qb, F]."""
    sf = frame_scores(q_blk, k_frm)
    H, nqb, F = sf.shape
    kf = min(k_f, F)
    idx = np.empty((H, nqb, kf), dtype=np.int64)
    for h in range(H):
        for qb in range(nqb):
            idx[h, qb] = topk_lower_index(list(sf[h, qb]), kf)
    return idx, sf


def block_scores_in_frame(q_vec: np.ndarray, k_blk_frame: np.ndarray) -> np.ndarray:
    """Score of each block of one frame: q_blk . k_blk[b]."""
    return np.array([np.dot(q_vec, k_blk_frame[b]) for b in range(k_blk_frame.shape[0])])


def select_blocks(q_blk: np.ndarray, k_blk: np.ndarray, frame_idx: np.ndarray, k_b: int):
    """[LF-gist 2.2, stage 2 of mask selection; LF-yly 三] Inside each chosen frame keep
    the k_b best-scoring blocks.  Global block id = f * n_bpf + b (f = history position).
    Returns block_idx [H, n_qb, kf*min(k_b, n_bpf)] ascending and the block scores
    [H, n_qb, kf, n_bpf] of the chosen frames."""
    H, nqb, kf = frame_idx.shape
    nbpf = k_blk.shape[2]
    kb = min(k_b, nbpf)
    idx = np.empty((H, nqb, kf * kb), dtype=np.int64)
    sb = np.empty((H, nqb, kf, nbpf))
    for h in range(H):
        for qb in range(nqb):
            chosen = []
            for j, f in enumerate(frame_idx[h, qb]):
                sb[h, qb, j] = block_scores_in_frame(q_blk[h, qb], k_blk[h, f])
                chosen += [int(f) * nbpf + b for b in topk_lower_index(list(sb[h, qb, j]), kb)]
            idx[h, qb] = sorted(chosen)
    return idx, sb


# --------------------------------------------------------------- (d) attention
def select_blocks_1d(q_blk: np.ndarray, k_blk: np.ndarray, k: int):
    """[LF-yly 四, the one-dimensional block-sparse ablation] No frame stage: each query
    block keeps the k best-scoring history blocks over all frames (global id f * n_bpf + b,
    equal scores to the lower id).  Returns block_idx [H, n_qb, min(k, F * n_bpf)] ascending
    and the scores of every history block [H, n_qb, F * n_bpf]."""
    H, nqb, _ = q_blk.shape
    F, nbpf = k_blk.shape[1], k_blk.shape[2]
    nb = F * nbpf
    kk = min(k, nb)
    idx = np.empty((H, nqb, kk), dtype=np.int64)
    s = np.empty((H, nqb, nb))
    for h in range(H):
        for qb in range(nqb):
            for f in range(F):
                s[h, qb, f * nbpf:(f + 1) * nbpf] = block_scores_in_frame(q_blk[h, qb], k_blk[h, f])
            idx[h, qb] = topk_lower_index(list(s[h, qb]), kk)
    return idx, s


def select_current_blocks(q_blk: np.ndarray, kc_blk: np.ndarray, k_c: int):
    """[LF-yly 一, second scenario: 80% sparsity applied to the first chunk, which has no
    history, so the sparsity reaches the current chunk's own keys; LF-gist 2.2, token
    compression and block selection by inner products.]  Reading: the current chunk's keys
    are mean-pooled per block exactly as its queries are (kc_blk = compress_queries(k_cur));
    query block qb keeps its own block qb (the diagonal) and the k_c - 1 other current
    blocks with the largest scores q_blk[h, qb] . kc_blk[h, c], equal scores to the lower
    index.  Returns cur_idx [H, n_qb, min(k_c, n_qb)] ascending and the scores
    [H, n_qb, n_qb] of every current block."""
    H, nqb, _ = q_blk.shape
    kk = min(k_c, nqb)
    idx = np.empty((H, nqb, kk), dtype=np.int64)
    sc = np.empty((H, nqb, nqb))
    for h in range(H):
        for qb in range(nqb):
            sc[h, qb] = block_scores_in_frame(q_blk[h, qb], kc_blk[h])
            others = [c for c in range(nqb) if c != qb]
            best = topk_lower_index([sc[h, qb, c] for c in others], kk - 1)
            idx[h, qb] = sorted([qb] + [others[i] for i in best])
    return idx, sc


def current_boundary_gap(scores: Sequence[float], own: int, k_c: int) -> float:
    """boundary_gap of the current-chunk choice of one query block: the own block is
    always kept, so the gap is that of the k_c - 1 best among the other blocks."""
    return boundary_gap([x for c, x in enumerate(scores) if c != own], k_c - 1)


def key_set(shape, qb_blocks: Sequence[int], cur_h: np.ndarray, cache_h: np.ndarray,
            hist_slots, sink_slots, cur_blocks=None) -> np.ndarray:
    """Keys (or values) one query block attends to, in a fixed order: the current chunk
    (every token, or with `cur_blocks` the tokens of those current-chunk blocks, block
    qb = frame * n_bpf + b), every token of every sink frame, then the tokens of the
    selected history blocks.  cur_h: [F_c*T, d] and cache_h: [n_slots, T, d] are one
    head's float64 tensors.  Returns [n_keys, d]."""
    bounds = block_bounds(shape.T, shape.block)
    nb = len(bounds)
    if cur_blocks is None:
        parts = [cur_h]
    else:
        parts = []
        for c in cur_blocks:
            f, b = divmod(int(c), nb)
            s, e = bounds[b]
            parts.append(cur_h[f * shape.T + s: f * shape.T + e])
    for slot in sink_slots:
        parts.append(cache_h[slot])
    for g in qb_blocks:
        f, b = divmod(int(g), nb)
        s, e = bounds[b]
        parts.append(cache_h[hist_slots[f], s:e])
    return np.concatenate(parts, axis=0)


def attention_qblock(q_rows: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """[LF-gist 2.2, execution] softmax(scale * q k^T) v over one key set, float64 with the
    row maximum subtracted.  Returns (O [rows, d], lse [rows], P [rows, n_keys])."""
    logits = (q_rows @ keys.T) * scale
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    P = p / l
    return P @ values, (m + np.log(l))[:, 0], P


def attention(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots,
              block_idx, heads=None, qblocks=None, cur_idx=None):
    """[LF-gist 2.2 / LF-yly 三, block-sparse attention; SF rolling cache; RF sinks]
    For each query token of query block qb, one joint softmax over the current chunk's
    keys (all of them, or with cur_idx only those of qb's kept current blocks), the sink
    frames' keys and the keys of qb's selected history blocks.
    block_idx: [H, n_qb, n_sel] global block ids (ignored when there is no history).
    cur_idx: None (dense current chunk) or [H, n_qb, n_c] current-chunk block ids.
    Returns O [F_c*T, H, d] and lse [H, F_c*T] (natural log of the scaled-logit
    normaliser); entries outside ``heads`` x ``qblocks`` are left as NaN."""
    T, B = shape.T, shape.block
    bounds = block_bounds(T, B)
    nb = len(bounds)
    qf = _f64(q)
    n_tok, H, d = qf.shape
    Fc = n_tok // T
    O = np.full((n_tok, H, d), np.nan)
    lse = np.full((H, n_tok), np.nan)
    heads = range(H) if heads is None else heads
    qblocks = range(Fc * nb) if qblocks is None else qblocks
    for h in heads:
        kcur_h, vcur_h = _f64(k_cur[:, h, :]), _f64(v_cur[:, h, :])
        kc_h, vc_h = _f64(k_cache[:, :, h, :]), _f64(v_cache[:, :, h, :])
        for qb in qblocks:
            f, b = divmod(qb, nb)
            s, e = bounds[b]
            rows = slice(f * T + s, f * T + e)
            sel = [] if len(hist_slots) == 0 else list(block_idx[h, qb])
            cur = None if cur_idx is None else list(cur_idx[h, qb])
            keys = key_set(shape, sel, kcur_h, kc_h, hist_slots, sink_slots, cur)
            vals = key_set(shape, sel, vcur_h, vc_h, hist_slots, sink_slots, cur)
            o, l, _ = attention_qblock(qf[rows, h, :], keys, vals, shape.scale)
            O[rows, h, :] = o
            lse[h, rows] = l
    return O, lse


def forward_chunk(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots):
    """(a) compress -> (b) frame top-k -> (c) block top-k -> (d) block-sparse attention.
    With shape.k_c > 0 (default 0: dense current chunk) the current chunk's blocks are
    selected too (select_current_blocks) and attended sparsely."""
    out = {}
    k_c = getattr(shape, "k_c", 0)
    if len(hist_slots) > 0 or k_c > 0:
        q_blk = compress_queries(q, shape.T, shape.block)
        out.update(q_blk=q_blk)
    if len(hist_slots) > 0:
        k_blk, k_frm = compress_keys(k_cache, hist_slots, shape.T, shape.block)
        frame_idx, sf = select_frames(q_blk, k_frm, shape.k_f)
        block_idx, sb = select_blocks(q_blk, k_blk, frame_idx, shape.k_b)
        out.update(k_blk=k_blk, k_frm=k_frm, frame_idx=frame_idx,
                   frame_scores=sf, block_idx=block_idx, block_scores=sb)
    else:
        block_idx = None
    cur_idx = None
    if k_c > 0:
        kc_blk = compress_queries(k_cur, shape.T, shape.block)
        cur_idx, sc = select_current_blocks(q_blk, kc_blk, k_c)
        out.update(kc_blk=kc_blk, cur_idx=cur_idx, cur_scores=sc)
    O, lse = attention(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots,
                       block_idx, cur_idx=cur_idx)
    out.update(O=O, lse=lse)
    return out


# ------------------------------------------------------------ algorithmic work
def executed_flops(shape, block_idx, cur_idx=None) -> int:
    """4*d per (head, query, valid key) pair: the QK^T and PV products actually needed
    (the current chunk dense, or only the kept current blocks when cur_idx is given)."""
    T, B = shape.T, shape.block
    bounds = block_bounds(T, B)
    nb = len(bounds)
    Fc = shape.n_cur_frames
    dense_keys = (Fc * T if cur_idx is None else 0) + shape.n_sink * T
    total = 0
    for h in range(shape.H):
        for qb in range(Fc * nb):
            s, e = bounds[qb % nb]
            nsel = 0
            if shape.n_hist > 0 and block_idx is not None:
                for g in block_idx[h, qb]:
                    bs, be = bounds[int(g) % nb]
                    nsel += be - bs
            if cur_idx is not None:
                for c in cur_idx[h, qb]:
                    bs, be = bounds[int(c) % nb]
                    nsel += be - bs
            total += (e - s) * (dense_keys + nsel)
    return 4 * shape.d * total
