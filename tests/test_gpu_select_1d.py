"""One-dimensional block selection (the ablation without the frame stage) through the C
ABI against the float64 oracle, and the attention it feeds."""
import numpy as np
import pytest
import torch

import lf_workloads as W
from oracle import hsa64 as O
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": lambda: W.tiny(0),
    "ragged_d64": lambda: W.random_small(1, H=2, d=64, T=200, block=64, n_cur_frames=1,
                                         n_hist=5, n_sink=0, k_f=2, k_b=2),
    "sinks_b128": lambda: W.random_small(3, H=3, d=128, T=300, block=128, n_cur_frames=2,
                                         n_hist=3, n_sink=1, k_f=2, k_b=2),
    "k_at_limits": lambda: W.random_small(4, H=2, d=64, T=130, block=128, n_cur_frames=1,
                                          n_hist=2, n_sink=2, k_f=5, k_b=9),
    "480p": lambda: W.p480(0),
}


def _gaps_1d(s, k):
    H, nqb, _ = s.shape
    return np.array([[O.boundary_gap(list(s[h, q]), k) for q in range(nqb)] for h in range(H)])


@pytest.mark.parametrize("name", list(CASES))
def test_select_1d_matches_oracle(gpu_lib, name):
    ci = CASES[name]()
    sh = ci.shape
    t = G.to_dev(ci)
    nbpf, nqb, kf, kb = gpu_lib.derived(sh)
    bidx = torch.full((sh.H, nqb, kf * kb), -7, dtype=torch.int32, device="cuda")
    gpu_lib.lf_select_chunk_1d(sh, t["q"], t["k_cache"], ci.hist_slots, bidx)
    torch.cuda.synchronize()
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    kb_o, _ = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)
    oidx, s = O.select_blocks_1d(qb, kb_o, kf * kb)
    g = bidx.cpu().numpy()
    assert np.all(np.diff(g, axis=-1) > 0)                     # ascending, no repeats
    bad, near, n = G.compare_indices(g, oidx, _gaps_1d(s, kf * kb))
    assert bad == 0, f"{name}: {bad}/{n} lists differ outside near ties ({near} near)"

    # the attention kernel consumes the 1-D lists unchanged
    if name != "480p":
        o_ref, lse_ref = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                     ci.hist_slots, ci.sink_slots, g)
        out, lse = G.gpu_attention(ci, t, g)
        torch.cuda.synchronize()
        G.assert_output_close(out, o_ref, what=name + "/1d")
    assert gpu_lib.lf_device_status() == 0
