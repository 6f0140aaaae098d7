"""CUDA path (through the C ABI) against the float64 oracle on the same seeded inputs.

Small shapes are compared element by element for every stage; they span several query
and key tiles, ragged frame tails (T not a multiple of B, T < B), odd query-block counts
(a tile with one query block), sinks, no history, and k_f / k_b at or above their
limits, and the size limits (the most frames, selected blocks and tokens per frame the
library accepts).  The full-size workloads (the 480p chunk the benchmark times, the large-model
stress, a rolling-cache chunk and a growth-sweep chunk) run the exact benchmark call and
are checked on all selected indices and on every output element and lse against the
float64 oracle (evaluated on the lists the GPU chose, which may differ from the oracle's
only at near ties), plus properties that hold at any size (every row written, finite,
bit-identical on a repeated call).
"""
import numpy as np
import pytest
import torch

import lf_workloads as W
from oracle import hsa64 as O
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": lambda: W.tiny(0),
    "ragged_d64": lambda: W.random_small(1, H=2, d=64, T=200, block=64, n_cur_frames=1,
                                         n_hist=5, n_sink=0, k_f=2, k_b=2),
    "sinks_d128": lambda: W.random_small(2, H=2, d=128, T=200, block=64, n_cur_frames=3,
                                         n_hist=4, n_sink=1, k_f=3, k_b=2),
    "b128": lambda: W.random_small(3, H=3, d=128, T=300, block=128, n_cur_frames=2,
                                   n_hist=3, n_sink=0, k_f=2, k_b=2),
    "k_at_limits": lambda: W.random_small(4, H=2, d=64, T=130, block=128, n_cur_frames=1,
                                          n_hist=2, n_sink=2, k_f=5, k_b=9),
    "T_below_B_odd_tiles": lambda: W.random_small(5, H=1, d=128, T=40, block=64,
                                                  n_cur_frames=3, n_hist=6, n_sink=0,
                                                  k_f=3, k_b=1),
    "no_history": lambda: W.random_small(6, H=2, d=128, T=192, block=64, n_cur_frames=1,
                                         n_hist=0, n_sink=0, k_f=1, k_b=1),
    "sinks_only": lambda: W.random_small(7, H=2, d=64, T=160, block=64, n_cur_frames=2,
                                         n_hist=0, n_sink=3, k_f=1, k_b=1),
    "frames_1560_b64": lambda: W.random_small(8, H=2, d=128, T=1560, block=64,
                                              n_cur_frames=1, n_hist=3, n_sink=1,
                                              k_f=2, k_b=12),
    "frames_1560_b128": lambda: W.random_small(9, H=2, d=128, T=1560, block=128,
                                               n_cur_frames=1, n_hist=4, n_sink=0,
                                               k_f=2, k_b=5),
    # the size limits: n_hist + n_sink = LF_MAX_FRAMES (fused selection, 250 candidate
    # frames, 200 kept) ...
    "max_frames_fused": lambda: W.random_small(10, H=1, d=64, T=64, block=64,
                                               n_cur_frames=1, n_hist=250, n_sink=6,
                                               k_f=200, k_b=1),
    # ... 1000 selected blocks per query block, near LF_MAX_SELECTED (the separate
    # frame and block selection kernels; a 2016-entry key plan) ...
    "max_selected_unfused": lambda: W.random_small(11, H=1, d=64, T=256, block=64,
                                                   n_cur_frames=1, n_hist=252, n_sink=4,
                                                   k_f=250, k_b=4),
    # ... and T = LF_MAX_T tokens per frame
    "max_T": lambda: W.random_small(12, H=1, d=64, T=16384, block=128, n_cur_frames=1,
                                    n_hist=2, n_sink=1, k_f=2, k_b=8),
}


def _oracle_selection(ci):
    sh = ci.shape
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    kb, kf = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)
    fidx, sf = O.select_frames(qb, kf, sh.k_f)
    bidx, sb = O.select_blocks(qb, kb, fidx, sh.k_b)
    return qb, kb, kf, fidx, sf, bidx, sb


@pytest.mark.parametrize("name", list(SMALL))
def test_small_all_stages(gpu_lib, name):
    ci = SMALL[name]()
    sh = ci.shape
    t = G.to_dev(ci)
    nbpf = O.n_blocks(sh.T, sh.block)

    if sh.n_hist > 0:
        qb, kb, kf, fidx, sf, bidx, sb = _oracle_selection(ci)
        # (a) compression
        g_qb, g_kb, g_kf = G.gpu_compress(ci, t)
        for g, o in ((g_qb, qb), (g_kb, kb), (g_kf, kf)):
            gn = g.cpu().double().numpy()
            assert np.all(np.abs(gn - o) <= 2e-6 * (1 + np.abs(o))), name
        # (b) frames, on the GPU's own pooled tensors
        g_fidx, g_fsc = G.gpu_select_frames(ci, g_qb, g_kf)
        assert np.allclose(g_fsc.cpu().double().numpy(), sf, rtol=1e-4, atol=1e-4)
        kf_eff = min(sh.k_f, sh.n_hist)
        bad, near, n = G.compare_indices(g_fidx.cpu().numpy(), fidx, G.frame_gaps(sf, kf_eff))
        assert bad == 0, f"{name}: {bad}/{n} frame lists differ outside near ties"
        # (c) blocks, isolated: the GPU selector on the oracle's frame lists
        o_fidx = torch.as_tensor(fidx, dtype=torch.int32).cuda().contiguous()
        g_bidx, g_bsc = G.gpu_select_blocks(ci, g_qb, g_kb, o_fidx)
        assert np.allclose(g_bsc.cpu().double().numpy(), sb, rtol=1e-4, atol=1e-4)
        kb_eff = min(sh.k_b, nbpf)
        bad, near, n = G.compare_indices(g_bidx.cpu().numpy(), bidx, G.block_gaps(sb, kb_eff))
        assert bad == 0, f"{name}: {bad}/{n} block lists differ outside near ties"
        assert g_bidx.shape[-1] == kf_eff * kb_eff          # fixed complexity
    else:
        bidx = None

    # (d) attention on the oracle's mask
    o_ref, lse_ref = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                 ci.hist_slots, ci.sink_slots, bidx)
    out, lse = G.gpu_attention(ci, t, bidx)
    torch.cuda.synchronize()
    G.assert_output_close(out, o_ref, what=name)
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= G.LSE_ABS

    # end to end through lf_forward_chunk: its indices against the oracle's (only near ties
    # may differ), and its output on every row against the oracle evaluated on the lists
    # the GPU chose
    out2, lse2, g_b2 = G.gpu_forward(ci, t)
    torch.cuda.synchronize()
    if sh.n_hist > 0:
        g_b2 = g_b2.cpu().numpy()
        gaps = np.minimum(G.frame_gaps(sf, kf_eff), G.block_gaps(sb, kb_eff))
        bad, near, n = G.compare_indices(g_b2, bidx, gaps)
        assert bad == 0, f"{name}: {bad}/{n} forward lists differ outside near ties"
        o_fwd, lse_fwd = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                     ci.hist_slots, ci.sink_slots, g_b2)
    else:
        o_fwd, lse_fwd = o_ref, lse_ref
    G.assert_output_close(out2, o_fwd, what=name + "/forward")
    assert np.abs(lse2.cpu().double().numpy() - lse_fwd).max() <= G.LSE_ABS
    assert gpu_lib.lf_device_status() == 0


@pytest.mark.parametrize("name", [n for n in SMALL if n not in ("no_history", "sinks_only")])
def test_select_chunk_matches_oracle(gpu_lib, name):
    """(a)+(b)+(c) in one call against the oracle's two-stage selection."""
    ci = SMALL[name]()
    sh = ci.shape
    t = G.to_dev(ci)
    nbpf, nqb, kf, kb = gpu_lib.derived(sh)
    bidx = torch.full((sh.H, nqb, kf * kb), -7, dtype=torch.int32, device="cuda")
    gpu_lib.lf_select_chunk(sh, t["q"], t["k_cache"], ci.hist_slots, bidx)
    torch.cuda.synchronize()
    qb, kb_, kf_, fidx, sf, oidx, sb = _oracle_selection(ci)
    gaps = np.minimum(G.frame_gaps(sf, kf), G.block_gaps(sb, kb))
    bad, near, n = G.compare_indices(bidx.cpu().numpy(), oidx, gaps)
    assert bad == 0, f"{name}: {bad}/{n} lists differ outside near ties"
    assert gpu_lib.lf_device_status() == 0


def _full_size_check(ci, heads=None):
    """The benchmark's call on a full-size workload: every selected index against the
    oracle's (only near ties may differ), and every output element and lse of `heads`
    (all heads by default) against the float64 oracle evaluated on the lists the GPU
    chose."""
    sh = ci.shape
    t = G.to_dev(ci)
    out, lse, g_bidx = G.gpu_forward(ci, t)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    g_bidx = g_bidx.cpu().numpy()
    nbpf = O.n_blocks(sh.T, sh.block)
    if sh.n_hist > 0:
        qb, kb, kf, fidx, sf, bidx, sb = _oracle_selection(ci)
        kf_eff, kb_eff = min(sh.k_f, sh.n_hist), min(sh.k_b, nbpf)
        gaps = np.minimum(G.frame_gaps(sf, kf_eff), G.block_gaps(sb, kb_eff))
        bad, near, n = G.compare_indices(g_bidx, bidx, gaps)
        assert bad == 0, f"{ci.name}: {bad}/{n} block lists differ outside near ties ({near} near)"
    heads = list(range(sh.H)) if heads is None else list(heads)
    o_ref, lse_ref = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                 ci.hist_slots, ci.sink_slots,
                                 g_bidx if sh.n_hist > 0 else None, heads=heads)
    g = out[:, heads].float().cpu().double().numpy()
    r = o_ref[:, heads]
    err = g - r
    max_abs = float(np.abs(err).max())
    rel_l2 = float(np.linalg.norm(err) / np.linalg.norm(r))
    assert max_abs <= G.OUT_MAX_ABS and rel_l2 <= G.OUT_REL_L2, (ci.name, max_abs, rel_l2)
    # and per head (a wrong key plan in one tile must not hide in the global norm)
    for i, h in enumerate(heads):
        e_h = err[:, i]
        assert np.linalg.norm(e_h) / np.linalg.norm(r[:, i]) <= G.OUT_REL_L2, (ci.name, h)
    assert np.abs(lse[heads].cpu().double().numpy() - lse_ref[heads]).max() <= G.LSE_ABS
    return out


def test_480p_chunk_full_size(gpu_lib):
    ci = W.p480(0)
    out = _full_size_check(ci)
    # determinism: the same call again gives the same bits
    t = G.to_dev(ci)
    out2, _, _ = G.gpu_forward(ci, t)
    assert torch.equal(out, out2)
    assert gpu_lib.lf_device_status() == 0


@pytest.mark.slow
def test_large_model_full_size(gpu_lib):
    _full_size_check(W.large(0))
    assert gpu_lib.lf_device_status() == 0


def test_rolling_steady_state_chunk(gpu_lib):
    chunks = W.rolling(0, n_chunks=9)
    for ci in chunks:
        pass                           # chunk 9: 3 sinks + 21 rolling history frames
    assert ci.shape.n_sink == 3 and ci.shape.n_hist == 21
    _full_size_check(ci)
    assert gpu_lib.lf_device_status() == 0


def test_growth_sweep_chunk(gpu_lib):
    ci = W.growth_sweep(0)[2]          # chunk 3: 6 history frames, (k_f, k_b) = (6, 6)
    _full_size_check(ci)
    assert gpu_lib.lf_device_status() == 0


def test_bad_block_index_is_reported_and_dropped(gpu_lib):
    ci = W.tiny(0)
    t = G.to_dev(ci)
    sh = ci.shape
    qb, kb, kf, fidx, sf, bidx, sb = _oracle_selection(ci)
    bad = bidx.copy()
    bad[0, 0, 0] = sh.n_hist * 4 + 3          # out of range
    gpu_lib.lf_device_status(True)
    out, _ = G.gpu_attention(ci, t, bad)
    torch.cuda.synchronize()
    assert gpu_lib.lf_device_status(True) == 6          # LF_ERR_BAD_INDEX
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("name", ["ragged_d64", "sinks_d128", "b128", "frames_1560_b64", "480p"])
def test_forward_equals_stagewise_calls(gpu_lib, name):
    """lf_forward_chunk (whose selection also writes the attention key plans) gives the
    same bits as lf_select_chunk followed by lf_block_sparse_attn (whose plans are built
    from the lists by plan_kernel): lists, plans and rounding agree."""
    ci = W.p480(0) if name == "480p" else SMALL[name]()
    sh = ci.shape
    t = G.to_dev(ci)
    nbpf, nqb, kf, kb = gpu_lib.derived(sh)
    out, lse, bidx = G.gpu_forward(ci, t)
    b2 = torch.full((sh.H, nqb, kf * kb), -7, dtype=torch.int32, device="cuda")
    gpu_lib.lf_select_chunk(sh, t["q"], t["k_cache"], ci.hist_slots, b2)
    out2 = torch.full_like(out, float("nan"))
    lse2 = torch.full_like(lse, float("nan"))
    gpu_lib.lf_block_sparse_attn(sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"], t["v_cache"],
                                 ci.hist_slots, ci.sink_slots, b2, out2, lse2)
    torch.cuda.synchronize()
    assert torch.equal(bidx, b2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    assert gpu_lib.lf_device_status() == 0
