"""Float64 CPU oracle of Light Forcing's chunk-aware growth (CAG) of the sparsity.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the library's schedule and must
never be used in its place.

  [LF-gist]  "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
             Attention" (gist.science explainer), section 2.1, chunk-aware growth: the
             sparsity of chunk i is s_i = s_base - alpha_i * beta, alpha_i following the
             noise level (proportional to 1/sqrt of it), beta tuned so that the total
             work meets a target sparsity; early chunks get low sparsity, later ones high.
  [LF-yly]   "南洋理工大学AI新突破 视频生成引擎模仿人脑高效学习" (m.youleyou.com),
             section 二: the sparsity of chunk i is a base level minus a term that falls
             as the inverse square root of the chunk's position; section 一: a dense
             first chunk followed by 80% sparsity on chunks 2-7 keeps the quality, and
             90% is the harsher setting.

Readings where the pages are silent: alpha_i = 1/sqrt(i) for chunk i (1-based); the
chunks before `first` are dense; the two unknowns (s_base, beta) are fixed by two
conditions, the mean sparsity over chunks first..n and the sparsity of the last chunk;
a chunk's keep ratio 1 - s_i becomes a budget of k_f frames and k_b blocks per frame out
of F history frames of n_bpf blocks, k_f = min(kf_max, F) and k_b the integer in
[1, n_bpf] that brings k_f * k_b / (F * n_bpf) nearest to the keep ratio (a tie takes the
larger k_b).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = ["cag_alpha", "cag_sparsity", "cag_budget", "cag_schedule"]


def cag_alpha(i: int) -> float:
    """[LF-gist 2.1; LF-yly 二] alpha_i, here 1/sqrt(i) for chunk i >= 1."""
    return 1.0 / math.sqrt(i)


def cag_sparsity(n_chunks: int, first: int, mean: float, final: float):
    """[LF-gist 2.1] s_i = s_base - alpha_i * beta for i = first..n_chunks, 0 before
    `first`.  (s_base, beta) solve the 2x2 linear system
        s_base - beta * mean_i(alpha_i) = mean,   s_base - beta * alpha_n = final.
    With a single sparse chunk the system is singular: beta = 0, s_base = final, and
    mean must equal final.  Returns (s [n_chunks], s_base, beta)."""
    if not (1 <= first <= n_chunks):
        raise ValueError("first must lie in [1, n_chunks]")
    idx = range(first, n_chunks + 1)
    if first == n_chunks:
        if abs(mean - final) > 1e-6:
            raise ValueError("one sparse chunk: mean and final sparsity must agree")
        s_base, beta = float(final), 0.0
    else:
        a_bar = float(np.mean([cag_alpha(i) for i in idx]))
        A = np.array([[1.0, -a_bar], [1.0, -cag_alpha(n_chunks)]])
        s_base, beta = (float(v) for v in np.linalg.solve(A, np.array([mean, final], float)))
    s = [0.0] * n_chunks
    for i in idx:
        s[i - 1] = s_base - cag_alpha(i) * beta
    return s, s_base, beta


def cag_budget(keep: float, F: int, n_bpf: int, kf_max: int, dense: bool) -> Tuple[int, int]:
    """Top-k budget (k_f, k_b) of a chunk with F history frames of n_bpf blocks: (0, 0)
    without history, all of it when dense, else k_f = min(kf_max, F) and k_b the integer
    of [1, n_bpf] whose fraction k_f * k_b / (F * n_bpf) lies nearest to `keep`, found by
    trying each one (a tie, up to 1e-9 of a block, takes the larger)."""
    if F <= 0:
        return 0, 0
    if dense:
        return F, n_bpf
    kf = min(kf_max, F)
    target = keep * F * n_bpf / kf           # the ideal k_b, in blocks
    best, best_err = 1, math.inf
    for kb in range(1, n_bpf + 1):
        err = abs(kb - target)
        if err <= best_err + 1e-9:
            best, best_err = kb, min(err, best_err)
    return kf, best


def cag_schedule(n_chunks: int, first: int, mean: float, final: float,
                 n_hist: Optional[Sequence[int]] = None, n_bpf: int = 1, kf_max: int = 1):
    """Keep ratio 1 - s_i per chunk (clamped to [0, 1]; 1 before `first`) and, with
    n_hist given, the (k_f, k_b) budget per chunk.  Returns (keep, budgets or None)."""
    s, _, _ = cag_sparsity(n_chunks, first, mean, final)
    keep: List[float] = []
    for i in range(1, n_chunks + 1):
        keep.append(1.0 if i < first else min(1.0, max(0.0, 1.0 - s[i - 1])))
    if n_hist is None:
        return keep, None
    budgets = [cag_budget(keep[i], int(n_hist[i]), n_bpf, kf_max, i + 1 < first)
               for i in range(n_chunks)]
    return keep, budgets
