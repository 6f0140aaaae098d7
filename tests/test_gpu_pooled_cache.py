"""Pooled-key cache (incremental compression) through the C ABI: block means computed once
per cache slot by lf_pool_frames and read by lf_select_chunk_cached must select exactly
what lf_select_chunk selects (bit-identical indices), the pooled rows must equal the
oracle's block means, and refreshing only the slots a chunk wrote must keep a rolling
cache in step with full recomputation, evictions included."""
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
    "frames_1560_b64": lambda: W.random_small(8, H=2, d=128, T=1560, block=64,
                                              n_cur_frames=1, n_hist=3, n_sink=1,
                                              k_f=2, k_b=12),
    "480p": lambda: W.p480(0),
}


def _new_pool(gpu_lib, shape):
    # NaN everywhere: a row the selection reads without it having been pooled shows up
    return torch.full((gpu_lib.lf_pooled_cache_bytes(shape) // 4,), float("nan"),
                      dtype=torch.float32, device="cuda")


def _select_both(gpu_lib, ci, q, k_cache, k_pool):
    sh = ci.shape
    nbpf, nqb, kf, kb = gpu_lib.derived(sh)
    full = torch.full((sh.H, nqb, kf * kb), -7, dtype=torch.int32, device="cuda")
    cached = torch.full_like(full, -9)
    gpu_lib.lf_select_chunk(sh, q, k_cache, ci.hist_slots, full)
    gpu_lib.lf_select_chunk_cached(sh, q, k_pool, ci.hist_slots, cached)
    torch.cuda.synchronize()
    return full, cached


@pytest.mark.parametrize("name", list(CASES))
def test_cached_selection_equals_full_and_oracle(gpu_lib, name):
    ci = CASES[name]()
    sh = ci.shape
    t = G.to_dev(ci)
    nbpf, nqb, kf, kb = gpu_lib.derived(sh)
    k_pool = _new_pool(gpu_lib, sh)
    gpu_lib.lf_pool_frames(sh, t["k_cache"], sorted(set(ci.hist_slots)), k_pool)
    full, cached = _select_both(gpu_lib, ci, t["q"], t["k_cache"], k_pool)
    assert torch.equal(full, cached), name

    # the pooled rows are the block means of each history slot's keys
    kb_o, kf_o = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)   # [H, F, nbpf, d]
    kp = k_pool.view(sh.n_slots, sh.H, nbpf, sh.d).cpu().double().numpy()
    for f, slot in enumerate(ci.hist_slots):
        o = kb_o[:, f]
        assert np.all(np.abs(kp[slot] - o) <= 2e-6 * (1 + np.abs(o))), (name, f)

    # and the oracle's two-stage selection, near ties excepted
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    fidx, sf = O.select_frames(qb, kf_o, sh.k_f)
    bidx, sb = O.select_blocks(qb, kb_o, fidx, sh.k_b)
    gaps = np.minimum(G.frame_gaps(sf, kf), G.block_gaps(sb, kb))
    bad, near, n = G.compare_indices(cached.cpu().numpy(), bidx, gaps)
    assert bad == 0, f"{name}: {bad}/{n} lists differ outside near ties"
    assert gpu_lib.lf_device_status() == 0


def test_rolling_cache_refreshed_incrementally(gpu_lib):
    """Ten chunks of the rolling workload (3 sinks + 21-frame window; chunk 10 sees the
    first evictions): only the slots the previous chunk wrote are pooled again."""
    n_sink, window = 3, 21

    def frame_slot(f):
        return f if f < n_sink else n_sink + (f - n_sink) % window

    k_pool, fresh, checked = None, [], 0
    for c, ci in enumerate(W.rolling(0, n_chunks=10, window=window, n_sink=n_sink)):
        sh = ci.shape
        if k_pool is None:
            k_pool = _new_pool(gpu_lib, sh)
        k_cache = ci.k_cache.cuda()
        if fresh:
            gpu_lib.lf_pool_frames(sh, k_cache, fresh, k_pool)
        if sh.n_hist > 0:
            full, cached = _select_both(gpu_lib, ci, ci.q.cuda(), k_cache, k_pool)
            assert torch.equal(full, cached), f"chunk {c + 1}"
            checked += 1
        # this chunk's frames enter the cache once it is done
        fresh = sorted({frame_slot(f) for f in range(c * sh.n_cur_frames,
                                                     (c + 1) * sh.n_cur_frames)})
    assert checked == 8
    assert gpu_lib.lf_device_status() == 0
