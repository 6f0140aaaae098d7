"""Helpers shared by the GPU parity tests: run the CUDA path through the Python binding
of the C ABI, run the float64 oracle, and compare under the stated tolerances.

Tolerances (float64 oracle vs the CUDA path on the same bf16 inputs):
  * indices: bit-exact, except where the oracle's relative score gap at the k-th
    boundary is below 1e-3 (reported, not failed);
  * attention output given the oracle's block mask: max-abs <= 2e-2 and relative L2
    <= 5e-3 (bf16 output upcast);
  * pooled means: fp32 sums of at most 128 bf16 values in token order against float64,
    |err| <= 2e-6 * (1 + |x|) (a few fp32 ulps of the running sum);
  * lse: |err| <= 2e-3 (fp32 softmax statistics over up to ~1e4 keys).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_attention_46_b200 as lf
from oracle import hsa64 as O

GAP_TOL = 1e-3
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3
LSE_ABS = 2e-3


def to_dev(ci, device="cuda"):
    return {k: getattr(ci, k).to(device) for k in ("q", "k_cur", "v_cur", "k_cache", "v_cache")}


def gpu_compress(ci, t):
    sh = ci.shape
    nbpf, nqb, kf, kb = lf.derived(sh)
    dev = t["q"].device
    q_blk = torch.empty(sh.H, nqb, sh.d, device=dev)
    k_blk = torch.empty(sh.H, sh.n_hist, nbpf, sh.d, device=dev)
    k_frm = torch.empty(sh.H, sh.n_hist, sh.d, device=dev)
    lf.lf_compress(sh, t["q"], t["k_cache"], ci.hist_slots, q_blk, k_blk, k_frm)
    return q_blk, k_blk, k_frm


def gpu_select_frames(ci, q_blk, k_frm):
    sh = ci.shape
    nbpf, nqb, kf, kb = lf.derived(sh)
    fidx = torch.full((sh.H, nqb, kf), -7, dtype=torch.int32, device=q_blk.device)
    fsc = torch.empty(sh.H, nqb, sh.n_hist, device=q_blk.device)
    lf.lf_select_frames(sh, q_blk, k_frm, fidx, fsc)
    return fidx, fsc


def gpu_select_blocks(ci, q_blk, k_blk, fidx):
    sh = ci.shape
    nbpf, nqb, kf, kb = lf.derived(sh)
    bidx = torch.full((sh.H, nqb, kf * kb), -7, dtype=torch.int32, device=q_blk.device)
    bsc = torch.empty(sh.H, nqb, kf, nbpf, device=q_blk.device)
    lf.lf_select_blocks(sh, q_blk, k_blk, fidx, bidx, bsc)
    return bidx, bsc


def gpu_select_current(ci, t):
    sh = ci.shape
    nbpf, nqb, kf, kb = lf.derived(sh)
    cidx = torch.full((sh.H, nqb, lf.current_blocks(sh)), -7, dtype=torch.int32,
                      device=t["q"].device)
    lf.lf_select_current(sh, t["q"], t["k_cur"], cidx)
    return cidx


def gpu_attention(ci, t, block_idx, cur_idx=None):
    sh = ci.shape
    dev = t["q"].device
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((sh.H, t["q"].shape[0]), float("nan"), device=dev)
    bi = ci_ = None
    if sh.n_hist > 0:
        bi = torch.as_tensor(np.asarray(block_idx), dtype=torch.int32).to(dev).contiguous()
    if cur_idx is not None:
        ci_ = torch.as_tensor(np.asarray(cur_idx), dtype=torch.int32).to(dev).contiguous()
    lf.lf_block_sparse_attn(sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"], t["v_cache"],
                            ci.hist_slots, ci.sink_slots, bi, out, lse, cur_idx=ci_)
    return out, lse


def gpu_forward(ci, t, with_cur=False):
    """lf_forward_chunk; returns (out, lse, block_idx) or, with_cur, also cur_idx."""
    sh = ci.shape
    nbpf, nqb, kf, kb = lf.derived(sh)
    dev = t["q"].device
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((sh.H, t["q"].shape[0]), float("nan"), device=dev)
    bidx = torch.full((sh.H, nqb, max(kf * kb, 1)), -7, dtype=torch.int32, device=dev)
    kc = lf.current_blocks(sh)
    cidx = torch.full((sh.H, nqb, max(kc, 1)), -7, dtype=torch.int32, device=dev)
    lf.lf_forward_chunk(sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"], t["v_cache"],
                        ci.hist_slots, ci.sink_slots, out, lse,
                        bidx if sh.n_hist > 0 else None, cur_idx_out=cidx if kc > 0 else None)
    if with_cur:
        return out, lse, bidx, cidx
    return out, lse, bidx


def current_gaps(sc: np.ndarray, k_c: int) -> np.ndarray:
    """Per (h, qb): the oracle's boundary gap of the current-chunk choice."""
    H, nqb, _ = sc.shape
    return np.array([[O.current_boundary_gap(list(sc[h, q]), q, min(k_c, nqb))
                      for q in range(nqb)] for h in range(H)])


def compare_indices(gpu_idx: np.ndarray, ora_idx: np.ndarray, gaps: np.ndarray):
    """gpu/oracle index lists [..., k]; gaps [...] = oracle boundary gap of each list.
    Returns (n_mismatch_outside_near_ties, n_near_tie_lists, n_lists)."""
    g = np.asarray(gpu_idx).reshape(-1, gpu_idx.shape[-1])
    o = np.asarray(ora_idx).reshape(-1, ora_idx.shape[-1])
    gp = np.asarray(gaps).reshape(-1)
    bad = 0
    near = 0
    for i in range(g.shape[0]):
        if gp[i] < GAP_TOL:
            near += 1
            continue
        if not np.array_equal(g[i], o[i]):
            bad += 1
    return bad, near, g.shape[0]


def frame_gaps(sf: np.ndarray, k: int) -> np.ndarray:
    H, nqb, F = sf.shape
    return np.array([[O.boundary_gap(list(sf[h, q]), k) for q in range(nqb)] for h in range(H)])


def block_gaps(sb: np.ndarray, k: int) -> np.ndarray:
    """Per (h, qb): the smallest boundary gap over its chosen frames."""
    H, nqb, kf, nb = sb.shape
    out = np.empty((H, nqb))
    for h in range(H):
        for q in range(nqb):
            out[h, q] = min(O.boundary_gap(list(sb[h, q, j]), k) for j in range(kf))
    return out


def output_errors(o_gpu: torch.Tensor, o_ref: np.ndarray, rows=None):
    """max-abs and relative L2 of the bf16 output against the float64 reference."""
    g = o_gpu.float().cpu().double().numpy()
    r = o_ref
    if rows is not None:
        g, r = g[rows], r[rows]
    err = g - r
    max_abs = float(np.abs(err).max())
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(r), 1e-30))
    return max_abs, rel_l2


def assert_output_close(o_gpu, o_ref, rows=None, what=""):
    max_abs, rel_l2 = output_errors(o_gpu, o_ref, rows)
    assert np.isfinite(max_abs), f"{what}: non-finite output"
    assert max_abs <= OUT_MAX_ABS and rel_l2 <= OUT_REL_L2, \
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e}"
    return max_abs, rel_l2


def qblock_rows(T, B, qb):
    nb = -(-T // B)
    f, b = divmod(qb, nb)
    s, e = b * B, min(b * B + B, T)
    return np.arange(f * T + s, f * T + e)
