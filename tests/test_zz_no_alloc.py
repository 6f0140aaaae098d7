"""lf_block_sparse_attn_noalloc: block-sparse attention for callers that cannot allocate
device memory (no allocator or scratch hook in their host runtime, or no allocation
allowed after start-up).  It runs through the C ABI on the library's fixed scratch array
and must give the results of lf_block_sparse_attn, call after call.

Kept in a file of its own that pytest collects last; it passes alone in a fresh process
and after the other tests."""
import numpy as np
import pytest
import torch

import lf_workloads as W
from oracle import hsa64 as O
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _inputs(ci):
    sh = ci.shape
    t = G.to_dev(ci)
    bidx = None
    if sh.n_hist > 0:
        qb = O.compress_queries(ci.q, sh.T, sh.block)
        kb, kf = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)
        fidx, _ = O.select_frames(qb, kf, sh.k_f)
        b, _ = O.select_blocks(qb, kb, fidx, sh.k_b)
        bidx = torch.as_tensor(b, dtype=torch.int32).cuda().contiguous()
    return t, bidx


@pytest.mark.parametrize("make", [lambda: W.tiny(0), lambda: W.p480(0),
                                  lambda: W.random_small(3, H=3, d=128, T=300, block=128,
                                                         n_cur_frames=2, n_hist=3, n_sink=1,
                                                         k_f=2, k_b=2)])
def test_noalloc_matches_workspace_entry_point_twice(gpu_lib, make):
    """Same kernels, same inputs: the outputs and lse must be the same bits as those of
    lf_block_sparse_attn with a caller workspace, on two calls in a row (the second call
    finds the first call's contents in the shared scratch)."""
    ci = make()
    sh = ci.shape
    t, bidx = _inputs(ci)
    n = t["q"].shape[0]
    ref = torch.empty_like(t["q"])
    ref_lse = torch.empty(sh.H, n, device="cuda")
    gpu_lib.lf_block_sparse_attn(sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"], t["v_cache"],
                                 ci.hist_slots, ci.sink_slots, bidx, ref, ref_lse)
    for _ in range(2):                       # two calls in a row share the fixed scratch
        out = torch.full_like(t["q"], float("nan"))
        lse = torch.full((sh.H, n), float("nan"), device="cuda")
        gpu_lib.lf_block_sparse_attn_noalloc(sh, t["q"], t["k_cur"], t["v_cur"], t["k_cache"],
                                             t["v_cache"], ci.hist_slots, ci.sink_slots, bidx,
                                             out, lse)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), "output differs from lf_block_sparse_attn"
        assert torch.equal(lse, ref_lse), "lse differs from lf_block_sparse_attn"
    if ci.shape.H * ci.shape.T <= 1024:      # the tiny shape: also against the float64 oracle
        o_ref, lse_ref = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                     ci.hist_slots, ci.sink_slots,
                                     None if bidx is None else bidx.cpu().numpy())
        G.assert_output_close(out, o_ref, what="noalloc vs oracle")
        assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= G.LSE_ABS
    assert gpu_lib.lf_device_status() == 0


def test_noalloc_rejects_shapes_beyond_the_scratch(gpu_lib):
    cap = gpu_lib.lf_noalloc_scratch_bytes()
    big = W.Shape(H=64, d=128, T=4096, block=64, n_cur_frames=8, n_hist=8, n_sink=0,
                  n_slots=8, k_f=8, k_b=64, scale=0.088)
    assert gpu_lib.lf_attn_workspace_size(big) > cap
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    bi = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(gpu_lib.LfError) as e:
        gpu_lib.lf_block_sparse_attn_noalloc(big, x, x, x, x, x, list(range(8)), [], bi, x)
    assert e.value.code == 5                    # LF_ERR_WORKSPACE, nothing launched
