"""Chunk-aware sparsity growth (lf_cag_schedule, host only) against its closed form, the
float64 oracle, the stored growth schedule under tests/golden, and the growth-sweep
workload's keep ratios and top-k budgets."""
import json
import math
import os

import pytest

import block_sparse_attention_46_b200 as lf
import lf_workloads as W
from oracle import cag64 as C

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cag_growth_480p.json")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_46_b200 import build
    build.build()
    return lf.load()


def test_growth_golden(lib):
    """The stored 7-chunk schedule (80% mean over chunks 2-7, 90% at chunk 7)."""
    g = json.load(open(GOLDEN))
    a = g["args"]
    keep, kf, kb = lf.lf_cag_schedule(a["n_chunks"], a["first"], a["mean_sparsity"],
                                      a["final_sparsity"], a["n_hist"], n_bpf=a["n_bpf"],
                                      kf_max=a["kf_max"])
    assert keep == pytest.approx(g["keep"], abs=1e-6)        # float32 outputs
    assert [list(p) for p in zip(kf, kb)] == g["budgets"]
    # the workload's 4-decimal keep ratios and its budgets are the stored ones
    assert W.GROWTH_KEEP == [round(v, 4) for v in g["keep"]]
    assert [list(p) for p in W.GROWTH_TOPK] == g["budgets"]


@pytest.mark.parametrize("n,first,mean,final,n_bpf,kf_max",
                         [(7, 2, 0.8, 0.9, 25, 6), (20, 2, 0.8, 0.95, 25, 6),
                          (12, 3, 0.6, 0.85, 13, 4), (5, 1, 0.3, 0.2, 7, 3),
                          (9, 4, 0.9, 0.97, 100, 8)])
def test_matches_oracle(lib, n, first, mean, final, n_bpf, kf_max):
    n_hist = [min(3 * i, 21) for i in range(n)]
    keep, kf, kb = lf.lf_cag_schedule(n, first, mean, final, n_hist, n_bpf=n_bpf,
                                      kf_max=kf_max)
    keep_o, budgets_o = C.cag_schedule(n, first, mean, final, n_hist, n_bpf=n_bpf,
                                       kf_max=kf_max)
    assert keep == pytest.approx(keep_o, abs=1e-6)
    assert list(zip(kf, kb)) == budgets_o


def test_growth_sweep_schedule(lib):
    """The 480p growth sweep: chunks 2..7 sparse, mean sparsity 80%, 90% at chunk 7; the
    workload's keep ratios (4 decimals) and (k_f, k_b) budgets are reproduced."""
    n_hist = [3 * i for i in range(7)]
    keep, kf, kb = lf.lf_cag_schedule(7, 2, 0.8, 0.9, n_hist, n_bpf=25, kf_max=6)
    assert keep == pytest.approx(W.GROWTH_KEEP, abs=6e-5)
    assert list(zip(kf, kb)) == W.GROWTH_TOPK


@pytest.mark.parametrize("n,first,mean,final", [(7, 2, 0.8, 0.9), (20, 2, 0.8, 0.95),
                                                (5, 3, 0.5, 0.6), (3, 1, 0.2, 0.1)])
def test_closed_form(lib, n, first, mean, final):
    keep, _, _ = lf.lf_cag_schedule(n, first, mean, final)
    s = [1.0 - k for k in keep]
    sparse = s[first - 1:]
    assert sum(sparse) / len(sparse) == pytest.approx(mean, abs=1e-6)
    assert s[-1] == pytest.approx(final, abs=1e-6)
    assert all(k == 1.0 for k in keep[:first - 1])            # dense before `first`
    # s_i = s_base - beta / sqrt(i): s_i * sqrt(i) is affine in sqrt(i)
    beta = (s[-1] - s[first - 1]) / (1 / math.sqrt(first) - 1 / math.sqrt(n))
    for i in range(first, n + 1):
        assert s[i - 1] == pytest.approx(s[-1] + beta / math.sqrt(n) - beta / math.sqrt(i),
                                         abs=1e-6)
    # sparsity grows with the chunk index when the final level is above the mean
    if final > mean:
        assert all(a < b for a, b in zip(sparse, sparse[1:]))


def test_budgets_dense_and_clamped(lib):
    keep, kf, kb = lf.lf_cag_schedule(4, 3, 0.5, 0.5, [0, 4, 4, 2], n_bpf=13, kf_max=8)
    assert (kf[0], kb[0]) == (0, 0)                           # no history
    assert (kf[1], kb[1]) == (4, 13)                          # dense chunk before `first`
    assert kf[2] == 4 and kf[3] == 2                          # k_f = min(kf_max, F)
    assert kb[2] == math.floor(keep[2] * 4 * 13 / 4 + 0.5)
    keep, kf, kb = lf.lf_cag_schedule(2, 2, 0.0, 0.0, [5, 5], n_bpf=7, kf_max=3)
    assert keep == [1.0, 1.0] and kb[1] == 7                  # clamped to n_bpf


@pytest.mark.parametrize("args", [(0, 1, 0.5, 0.5), (3, 0, 0.5, 0.6), (3, 4, 0.5, 0.6),
                                  (3, 2, 1.0, 0.6), (3, 2, 0.5, -0.1), (3, 3, 0.5, 0.6)])
def test_invalid_arguments(lib, args):
    with pytest.raises(lf.LfError) as e:
        lf.lf_cag_schedule(*args)
    assert e.value.code == 1
