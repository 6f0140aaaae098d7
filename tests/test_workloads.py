"""Seeded generators: determinism, shapes and the structure each workload promises."""
import numpy as np
import torch

import lf_workloads as W


def test_tiny_is_deterministic_and_shaped():
    a, b = W.tiny(0), W.tiny(0)
    assert torch.equal(a.q, b.q) and torch.equal(a.k_cache, b.k_cache)
    assert not torch.equal(W.tiny(1).q, a.q)
    assert a.q.dtype == torch.bfloat16 and tuple(a.q.shape) == (256, 2, 64)
    assert tuple(a.k_cache.shape) == (4, 256, 2, 64)
    assert sorted(a.hist_slots) == [0, 1, 2, 3] and a.sink_slots == []


def test_480p_shapes():
    s = W.p480_shape()
    assert (s.H, s.d, s.T, s.block, s.n_cur_frames, s.n_hist, s.k_f, s.k_b) == \
        (12, 128, 1560, 64, 3, 18, 6, 12)


def test_growth_sweep_budget_table():
    assert len(W.GROWTH_KEEP) == 7 and W.GROWTH_KEEP[0] == 1.0
    # mean sparsity over chunks 2-7 is 80%
    assert abs(np.mean([1 - r for r in W.GROWTH_KEEP[1:]]) - 0.8) < 1e-3
    # the integer budgets follow k_b = floor(r*F*n_bpf/k_f + 0.5), k_f = min(6, F)
    for i, (r, (kf, kb)) in enumerate(zip(W.GROWTH_KEEP[1:], W.GROWTH_TOPK[1:]), start=2):
        F = 3 * (i - 1)
        assert kf == min(6, F)
        assert kb == max(1, min(25, int(np.floor(r * F * 25 / kf + 0.5))))


def test_rolling_cache_slots():
    shape = W.Shape(H=1, d=8, T=4, block=2, n_cur_frames=3, n_hist=0, n_sink=0,
                    n_slots=0, k_f=4, k_b=1, scale=1.0)
    chunks = list(W.rolling(0, n_chunks=10, window=6, n_sink=3, shape=shape))
    assert chunks[0].sink_slots == [] and chunks[0].hist_slots == []
    assert chunks[1].sink_slots == [0, 1, 2] and chunks[1].hist_slots == []
    assert chunks[2].hist_slots == [3, 4, 5]
    last = chunks[9]                     # frames 27..29 current; history = frames 21..26
    assert last.hist_slots == [3 + (f - 3) % 6 for f in range(21, 27)]
    assert len(set(last.hist_slots)) == 6
