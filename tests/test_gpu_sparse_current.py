"""Sparse attention inside the current chunk (k_c > 0), through the C ABI, against the
float64 oracle on the same seeded inputs.

Each query block keeps its own block and the k_c - 1 other current-chunk blocks with the
largest pooled inner product.  Checked: the current-chunk choice of lf_select_current
(bit-exact outside near ties, relative boundary gap < 1e-3), the attention on the
oracle's lists (max-abs <= 2e-2, relative L2 <= 5e-3, lse within 2e-3), and
lf_forward_chunk end to end (its lists against the oracle's, its output against the
oracle on the lists it chose).  Shapes span ragged frame tails, an odd number of query
blocks (a tile with one query block), B = 128, sinks with and without history, k_c = 1
and k_c above the number of blocks; at full size the first chunk of the 480p workload at
80% sparsity (the youleyou article's first-chunk experiment) and the 480p chunk with
history."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import lf_workloads as W
from oracle import hsa64 as O
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

SMALL = {
    "cur_only_sinks": lambda: W.random_small(50, H=2, d=64, T=200, block=64, n_cur_frames=3,
                                             n_hist=0, n_sink=1, k_f=1, k_b=1, k_c=3),
    "cur_hist_d128": lambda: W.random_small(51, H=2, d=128, T=200, block=64, n_cur_frames=3,
                                            n_hist=4, n_sink=1, k_f=2, k_b=2, k_c=5),
    "cur_b128": lambda: W.random_small(52, H=3, d=128, T=300, block=128, n_cur_frames=2,
                                       n_hist=3, n_sink=0, k_f=2, k_b=2, k_c=2),
    "cur_all_kept": lambda: W.random_small(53, H=2, d=64, T=130, block=64, n_cur_frames=2,
                                           n_hist=2, n_sink=0, k_f=1, k_b=1, k_c=99),
    "cur_k1_T_below_B": lambda: W.random_small(54, H=1, d=128, T=40, block=64, n_cur_frames=3,
                                               n_hist=2, n_sink=0, k_f=1, k_b=1, k_c=1),
}


def _oracle_lists(ci):
    sh = ci.shape
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    kcb = O.compress_queries(ci.k_cur, sh.T, sh.block)
    cidx, sc = O.select_current_blocks(qb, kcb, sh.k_c)
    out = dict(q_blk=qb, cur_idx=cidx, cur_scores=sc, block_idx=None)
    if sh.n_hist > 0:
        kb, kf = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)
        fidx, sf = O.select_frames(qb, kf, sh.k_f)
        bidx, sb = O.select_blocks(qb, kb, fidx, sh.k_b)
        nbpf = O.n_blocks(sh.T, sh.block)
        gaps = np.minimum(G.frame_gaps(sf, min(sh.k_f, sh.n_hist)),
                          G.block_gaps(sb, min(sh.k_b, nbpf)))
        out.update(block_idx=bidx, hist_gaps=gaps)
    return out


def _check_forward(gpu_lib, ci, ref):
    sh = ci.shape
    t = G.to_dev(ci)
    out, lse, g_b, g_c = G.gpu_forward(ci, t, with_cur=True)
    torch.cuda.synchronize()
    g_c = g_c.cpu().numpy()
    bad, near, n = G.compare_indices(g_c, ref["cur_idx"], G.current_gaps(ref["cur_scores"], sh.k_c))
    assert bad == 0, f"{ci.name}: {bad}/{n} current lists differ outside near ties"
    g_b = g_b.cpu().numpy() if sh.n_hist > 0 else None
    if sh.n_hist > 0:
        bad, near, n = G.compare_indices(g_b, ref["block_idx"], ref["hist_gaps"])
        assert bad == 0, f"{ci.name}: {bad}/{n} history lists differ outside near ties"
    o_ref, lse_ref = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                 ci.hist_slots, ci.sink_slots, g_b, cur_idx=g_c)
    G.assert_output_close(out, o_ref, what=ci.name + "/forward")
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= G.LSE_ABS
    assert gpu_lib.lf_device_status() == 0
    return out


@pytest.mark.parametrize("name", list(SMALL))
def test_small_sparse_current(gpu_lib, name):
    ci = SMALL[name]()
    sh = ci.shape
    t = G.to_dev(ci)
    ref = _oracle_lists(ci)
    # the current-chunk choice alone
    g_c = G.gpu_select_current(ci, t)
    torch.cuda.synchronize()
    g_c = g_c.cpu().numpy()
    nqb = ref["cur_idx"].shape[1]
    assert g_c.shape[-1] == min(sh.k_c, nqb)
    bad, near, n = G.compare_indices(g_c, ref["cur_idx"], G.current_gaps(ref["cur_scores"], sh.k_c))
    assert bad == 0, f"{name}: {bad}/{n} current lists differ outside near ties"
    for h in range(sh.H):                     # the own block is always there
        for q in range(nqb):
            assert q in g_c[h, q]
    # attention on the oracle's lists
    o_ref, lse_ref = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                 ci.hist_slots, ci.sink_slots, ref["block_idx"],
                                 cur_idx=ref["cur_idx"])
    out, lse = G.gpu_attention(ci, t, ref["block_idx"], ref["cur_idx"])
    torch.cuda.synchronize()
    G.assert_output_close(out, o_ref, what=name)
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= G.LSE_ABS
    # end to end
    _check_forward(gpu_lib, ci, ref)


def test_first_chunk_at_80_percent_full_size(gpu_lib):
    """The 480p shape's first chunk (no history) with 15 of its 75 current blocks kept per
    query block: 80% sparsity on chunk 1."""
    ci = W.growth_sweep(0)[0]
    ci = replace(ci, shape=replace(ci.shape, k_c=15), name="chunk1_80")
    out = _check_forward(gpu_lib, ci, _oracle_lists(ci))
    out2, _, _ = G.gpu_forward(ci, G.to_dev(ci))
    assert torch.equal(out, out2)                       # deterministic


def test_480p_with_sparse_current_full_size(gpu_lib):
    ci = W.p480(0)
    ci = replace(ci, shape=replace(ci.shape, k_c=15), name="480p_cur15")
    _check_forward(gpu_lib, ci, _oracle_lists(ci))


def test_bad_current_index_is_reported_and_dropped(gpu_lib):
    ci = SMALL["cur_hist_d128"]()
    t = G.to_dev(ci)
    ref = _oracle_lists(ci)
    bad = ref["cur_idx"].copy()
    bad[0, 0, 0] = 10 ** 6                          # out of range
    gpu_lib.lf_device_status(True)
    out, _ = G.gpu_attention(ci, t, ref["block_idx"], bad)
    torch.cuda.synchronize()
    assert gpu_lib.lf_device_status(True) == 6          # LF_ERR_BAD_INDEX
