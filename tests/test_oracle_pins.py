"""Pins of the float64 oracle against facts fixed by the mathematics and by the method's
statement, not against the oracle itself.

The Light Forcing pages print no worked example of hierarchical sparse attention, so the
pins are closed forms, brute force on tiny inputs, library routines for the special cases
the method reduces to, and invariants the method's description implies:

* pooling: ramp inputs whose block and frame means are known in closed form;
* frame score linearity: a frame's pooled key is the length-weighted mean of its block
  means, so its score is the length-weighted mean of block scores;
* selection: exhaustive search over all k-subsets (maximal score sum, lexicographically
  smallest among equals) agrees with the top-k rule;
* attention: with every frame and block kept, HSA is full attention, checked against
  torch's scaled_dot_product_attention in float64; for arbitrary block lists it is SDPA
  with a token mask built from the lists by another route; zero queries give the uniform
  average of the key set's values and lse = log(|key set|); probabilities are
  non-negative and sum to one; unselected keys can be permuted or replaced freely;
* fixed complexity: the number of selected blocks does not depend on the history length;
* chunk-aware growth: the two conditions that fix (s_base, beta) hold, a two-chunk case
  solved by hand, constant sparsity when the mean and the final level agree, growth with
  the chunk index, and budgets against an exhaustive search over (k_f, k_b) pairs.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import lf_workloads as W
from oracle import cag64 as C
from oracle import hsa64 as O


# ------------------------------------------------------------------ pooling
def _ramp_inputs(T=20, B=8, H=2, d=4, F=3, Fc=2, n_slots=5):
    """q[t] = t (token index in the chunk), k in slot s at token t = 10*s + t/4.
    All values are exact in bf16 (multiples of 1/4 below 64)."""
    q = torch.zeros(Fc * T, H, d)
    for t in range(Fc * T):
        q[t] = float(t)
    kc = torch.zeros(n_slots, T, H, d)
    for s in range(n_slots):
        for t in range(T):
            kc[s, t] = 10.0 * s + t / 4.0
    return q.to(torch.bfloat16), kc.to(torch.bfloat16)


def test_block_bounds_closed_form():
    b = O.block_bounds(1560, 64)
    assert len(b) == 25 and b[-1] == (1536, 1560)          # 24 full blocks + 24 tokens
    assert all(e - s == 64 for s, e in b[:-1])
    assert sum(e - s for s, e in b) == 1560
    assert O.block_bounds(1560, 128)[-1] == (1536, 1560) and O.n_blocks(1560, 128) == 13
    assert O.block_bounds(256, 64) == [(0, 64), (64, 128), (128, 192), (192, 256)]


@pytest.mark.parametrize("T,B,blocks", [(20, 8, [(0, 8), (8, 16), (16, 20)]),   # ragged tail
                                         (24, 8, [(0, 8), (8, 16), (16, 24)]),   # exact
                                         (20, 32, [(0, 20)])])                   # T < B
def test_pooling_ramp_closed_form(T, B, blocks):
    q, kc = _ramp_inputs(T, B)
    qb = O.compress_queries(q, T, B)
    nb = len(blocks)
    # query block b of frame f covers tokens [s, e): mean token = f*T + (s + e - 1)/2
    for f in range(2):
        for b, (s, e) in enumerate(blocks):
            assert np.allclose(qb[:, f * nb + b, :], f * T + (s + e - 1) / 2.0, atol=0, rtol=0)
    slots = [3, 0, 4]
    kb, kf = O.compress_keys(kc, slots, T, B)
    assert kb.shape[2] == nb
    for f, s in enumerate(slots):
        for b, (a, e) in enumerate(blocks):
            assert np.allclose(kb[:, f, b, :], 10.0 * s + (a + e - 1) / 8.0, rtol=0, atol=1e-12)
        assert np.allclose(kf[:, f, :], 10.0 * s + (T - 1) / 8.0, rtol=0, atol=1e-12)


def test_frame_pool_is_length_weighted_block_mean():
    ci = W.random_small(3, H=2, d=16, T=100, block=32, n_cur_frames=1, n_hist=3,
                        n_sink=0, k_f=2, k_b=2)
    kb, kf = O.compress_keys(ci.k_cache, ci.hist_slots, ci.shape.T, ci.shape.block)
    lens = np.array([e - s for s, e in O.block_bounds(100, 32)], dtype=np.float64)
    lin = np.einsum("hfbd,b->hfd", kb, lens) / 100.0
    assert np.allclose(lin, kf, rtol=0, atol=1e-12)
    # so the frame score equals the length-weighted mean of block scores
    qb = O.compress_queries(ci.q, 100, 32)
    sf = O.frame_scores(qb, kf)
    sb_all = np.einsum("hqd,hfbd->hqfb", qb, kb)
    assert np.allclose(sf, np.einsum("hqfb,b->hqf", sb_all, lens) / 100.0, atol=1e-12)


# ------------------------------------------------------------------ selection
def _brute_topk(scores, k):
    """Exhaustive: the k-subset with the largest score sum; among equal sums the
    lexicographically smallest index tuple (ties to lower indices)."""
    best, best_key = None, None
    for sub in itertools.combinations(range(len(scores)), k):
        key = (-sum(scores[i] for i in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return list(best)


@pytest.mark.parametrize("seed", range(40))
def test_topk_matches_brute_force(seed):
    g = np.random.default_rng(seed)
    n = int(g.integers(1, 9))
    k = int(g.integers(1, n + 1))
    if seed % 2:
        scores = list(g.integers(-2, 3, size=n).astype(float))   # many exact ties
    else:
        scores = list(g.standard_normal(n))
    assert O.topk_lower_index(scores, k) == _brute_topk(scores, k)


def test_topk_ties_go_to_lower_index():
    assert O.topk_lower_index([1.0, 2.0, 2.0, 2.0, 0.5], 2) == [1, 2]
    assert O.topk_lower_index([5.0, 5.0, 5.0], 1) == [0]
    assert O.topk_lower_index([-1.0, -1.0, 3.0], 2) == [0, 2]
    assert O.topk_lower_index([0.0, 1.0], 5) == [0, 1]        # k >= n keeps everything


def test_boundary_gap_closed_form():
    assert O.boundary_gap([4.0, 1.0, 3.0, 2.0], 2) == pytest.approx((3.0 - 2.0) / 3.0)
    assert O.boundary_gap([1.0, 2.0], 2) == math.inf


@pytest.mark.parametrize("seed", range(6))
def test_two_stage_selection_brute_force(seed):
    """Frames, then blocks inside each chosen frame, against exhaustive search with the
    scores recomputed through a different route (reshape-mean pooling + einsum)."""
    g = np.random.default_rng(100 + seed)
    T, B = int(g.choice([40, 48, 50])), 16
    F, kf, kb = int(g.integers(2, 6)), int(g.integers(1, 3)), int(g.integers(1, 3))
    ci = W.random_small(seed, H=2, d=8, T=T, block=B, n_cur_frames=1, n_hist=F,
                        n_sink=0, k_f=kf, k_b=kb)
    qb = O.compress_queries(ci.q, T, B)
    kbk, kfr = O.compress_keys(ci.k_cache, ci.hist_slots, T, B)
    fidx, _ = O.select_frames(qb, kfr, kf)
    bidx, _ = O.select_blocks(qb, kbk, fidx, kb)

    q64 = ci.q.double().numpy()
    k64 = ci.k_cache.double().numpy()
    nb = -(-T // B)
    pad = nb * B - T
    kfr2 = np.stack([k64[s].mean(axis=0) for s in ci.hist_slots], axis=1)      # [H,F,d]
    for h in range(2):
        for qi in range(nb):
            s, e = qi * B, min(qi * B + B, T)
            qv = q64[s:e, h, :].mean(axis=0)
            fs = [float(qv @ kfr2[h, f]) for f in range(F)]
            frames = _brute_topk(fs, min(kf, F))
            assert list(fidx[h, qi]) == frames
            want = []
            for f in frames:
                fr = k64[ci.hist_slots[f], :, h, :]
                means = [fr[b * B:min(b * B + B, T)].mean(axis=0) for b in range(nb)]
                bs = [float(qv @ m) for m in means]
                want += [f * nb + b for b in _brute_topk(bs, min(kb, nb))]
            assert list(bidx[h, qi]) == sorted(want)


def test_fixed_complexity_independent_of_history_length():
    counts = set()
    for F in (3, 6, 12):
        ci = W.random_small(F, H=2, d=8, T=64, block=16, n_cur_frames=1, n_hist=F,
                            n_sink=0, k_f=2, k_b=3)
        r = O.forward_chunk(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                            ci.hist_slots, ci.sink_slots)
        counts.add(r["block_idx"].shape[-1])
        assert r["frame_idx"].shape[-1] == 2
    assert counts == {2 * 3}


def test_planted_frame_recovered():
    """Soft check: queries pulled towards one history frame usually select it."""
    ci = W.random_small(11, H=4, d=64, T=256, block=64, n_cur_frames=2, n_hist=8,
                        n_sink=0, k_f=2, k_b=2)
    qb = O.compress_queries(ci.q, 256, 64)
    _, kfr = O.compress_keys(ci.k_cache, ci.hist_slots, 256, 64)
    fidx, _ = O.select_frames(qb, kfr, 2)
    hits = [ci.planted[h, qi // 4] in fidx[h, qi] for h in range(4) for qi in range(8)]
    assert np.mean(hits) >= 0.8


# ------------------------------------------------------------------ attention
def _dense_reference_sdpa(ci):
    """torch SDPA (float64, CPU) over current + sinks + all history frames."""
    sh = ci.shape
    keys = [ci.k_cur.double()] + [ci.k_cache[s].double() for s in ci.sink_slots] + \
           [ci.k_cache[s].double() for s in ci.hist_slots]
    vals = [ci.v_cur.double()] + [ci.v_cache[s].double() for s in ci.sink_slots] + \
           [ci.v_cache[s].double() for s in ci.hist_slots]
    K = torch.cat(keys, 0).permute(1, 0, 2)[None]
    V = torch.cat(vals, 0).permute(1, 0, 2)[None]
    Q = ci.q.double().permute(1, 0, 2)[None]
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=sh.scale)
    logits = torch.einsum("hqd,hkd->hqk", Q[0], K[0]) * sh.scale
    return out[0].permute(1, 0, 2).numpy(), torch.logsumexp(logits, -1).numpy()


@pytest.mark.parametrize("T,B,F,S", [(100, 32, 3, 0), (96, 32, 2, 1), (64, 64, 1, 2)])
def test_dense_equivalence_with_sdpa(T, B, F, S):
    ci = W.random_small(T + F, H=2, d=16, T=T, block=B, n_cur_frames=2, n_hist=F,
                        n_sink=S, k_f=F, k_b=-(-T // B))
    r = O.forward_chunk(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                        ci.hist_slots, ci.sink_slots)
    o_ref, lse_ref = _dense_reference_sdpa(ci)
    assert np.allclose(r["O"], o_ref, rtol=0, atol=1e-12)
    assert np.allclose(r["lse"], lse_ref, rtol=0, atol=1e-12)


def _masked_reference_sdpa(ci, block_idx):
    """torch SDPA (float64, CPU) over current + sinks + ALL history frames with a boolean
    token mask: a history key token (frame position f, token t) is visible to a query
    token iff f * n_bpf + t // B is in the selected list of the query's block."""
    sh = ci.shape
    T, B, Fc = sh.T, sh.block, sh.n_cur_frames
    nbpf = -(-T // B)
    keys = [ci.k_cur.double()] + [ci.k_cache[s].double() for s in ci.sink_slots] + \
           [ci.k_cache[s].double() for s in ci.hist_slots]
    vals = [ci.v_cur.double()] + [ci.v_cache[s].double() for s in ci.sink_slots] + \
           [ci.v_cache[s].double() for s in ci.hist_slots]
    K = torch.cat(keys, 0).permute(1, 0, 2)
    V = torch.cat(vals, 0).permute(1, 0, 2)
    Q = ci.q.double().permute(1, 0, 2)
    n_q, n_dense = Fc * T, Fc * T + sh.n_sink * T
    tq = torch.arange(n_q)
    q_block = (tq // T) * nbpf + (tq % T) // B                       # [n_q]
    th = torch.arange(sh.n_hist * T)
    k_block = (th // T) * nbpf + (th % T) // B                       # [F*T] global block id
    mask = torch.ones(sh.H, n_q, n_dense + sh.n_hist * T, dtype=torch.bool)
    for h in range(sh.H):
        sel = torch.zeros(Fc * nbpf, sh.n_hist * nbpf, dtype=torch.bool)
        for qb in range(Fc * nbpf):
            sel[qb, torch.as_tensor(block_idx[h, qb], dtype=torch.long)] = True
        mask[h, :, n_dense:] = sel[q_block][:, k_block]
    out = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None],
                                                           attn_mask=mask[None],
                                                           scale=sh.scale)[0]
    logits = torch.einsum("hqd,hkd->hqk", Q, K) * sh.scale
    lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), -1)
    return out.permute(1, 0, 2).numpy(), lse.numpy()


@pytest.mark.parametrize("seed,T,B,F,S,nsel", [(21, 100, 32, 3, 0, 5), (22, 70, 16, 4, 1, 7),
                                               (23, 64, 64, 3, 2, 2), (24, 40, 64, 5, 0, 3)])
def test_sparse_attention_equals_masked_sdpa(seed, T, B, F, S, nsel):
    """Any block lists (here random, not the selection's) give the attention of a token
    mask built from the lists: ragged last blocks, slot indirection and the joint
    softmax over current + sinks + selected blocks are all in the mask route."""
    nbpf = -(-T // B)
    ci = W.random_small(seed, H=2, d=16, T=T, block=B, n_cur_frames=2, n_hist=F,
                        n_sink=S, k_f=1, k_b=1)
    g = np.random.default_rng(seed)
    nqb = 2 * nbpf
    bidx = np.stack([np.stack([np.sort(g.choice(F * nbpf, size=nsel, replace=False))
                               for _ in range(nqb)]) for _ in range(2)])
    o, lse = O.attention(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                         ci.hist_slots, ci.sink_slots, bidx)
    o_ref, lse_ref = _masked_reference_sdpa(ci, bidx)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_no_history_is_attention_over_current_and_sinks():
    ci = W.random_small(5, H=2, d=16, T=48, block=16, n_cur_frames=2, n_hist=0,
                        n_sink=2, k_f=1, k_b=1)
    r = O.forward_chunk(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                        ci.hist_slots, ci.sink_slots)
    o_ref, _ = _dense_reference_sdpa(ci)
    assert np.allclose(r["O"], o_ref, rtol=0, atol=1e-12)


def test_zero_queries_average_values_and_lse_counts_keys():
    """q = 0 gives equal logits: O is the plain mean of the key set's values and
    lse = log(number of keys) = log(F_c*T + S*T + sum of selected block lengths)."""
    ci = W.random_small(7, H=2, d=16, T=50, block=16, n_cur_frames=1, n_hist=4,
                        n_sink=1, k_f=2, k_b=2)
    sh = ci.shape
    r = O.forward_chunk(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                        ci.hist_slots, ci.sink_slots)
    bidx = r["block_idx"]
    zq = torch.zeros_like(ci.q)
    O0, lse0 = O.attention(sh, zq, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                           ci.hist_slots, ci.sink_slots, bidx)
    nb = 4                       # blocks of 16 over 50 tokens: 16, 16, 16, 2
    lens = [16, 16, 16, 2]
    v64 = ci.v_cache.double().numpy()
    vc64 = ci.v_cur.double().numpy()
    for h in range(2):
        for qi in range(nb):
            sel = [int(g) for g in bidx[h, qi]]
            n_keys = 50 + 50 + sum(lens[g % nb] for g in sel)
            total = vc64[:, h].sum(0) + v64[ci.sink_slots[0], :, h].sum(0)
            for g in sel:
                f, b = divmod(g, nb)
                total = total + v64[ci.hist_slots[f], b * 16:b * 16 + lens[b], h].sum(0)
            rows = slice(qi * 16, qi * 16 + lens[qi])
            assert np.allclose(O0[rows, h], total / n_keys, rtol=0, atol=1e-12)
            assert np.allclose(lse0[h, rows], math.log(n_keys), rtol=0, atol=1e-12)


def test_two_key_closed_form():
    """One query, two keys with logits 0 and x: O = (v0 + e^x v1) / (1 + e^x)."""
    q = np.array([[1.0, 0.0]])
    k = np.array([[0.0, 1.0], [2.0, 0.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0]])
    o, lse, P = O.attention_qblock(q, k, v, 0.5)
    x = 1.0
    assert np.allclose(o, [[1 / (1 + math.e ** x), math.e ** x / (1 + math.e ** x)]], atol=1e-15)
    assert np.allclose(lse, [math.log(1 + math.e ** x)], atol=1e-15)


def test_probabilities_are_a_distribution():
    g = np.random.default_rng(0)
    q, k, v = g.standard_normal((7, 32)), g.standard_normal((300, 32)) * 3, g.standard_normal((300, 32))
    _, _, P = O.attention_qblock(q, k, v, 1 / math.sqrt(32))
    assert (P >= 0).all()
    assert np.abs(P.sum(axis=1) - 1.0).max() < 1e-12


def test_unselected_blocks_do_not_matter():
    """Replacing every unselected history block (contents permuted across tokens and
    scaled) leaves O unchanged for a fixed selection; touching one selected block
    changes it."""
    ci = W.random_small(9, H=2, d=16, T=64, block=16, n_cur_frames=1, n_hist=4,
                        n_sink=0, k_f=2, k_b=2)
    sh = ci.shape
    r = O.forward_chunk(sh, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                        ci.hist_slots, ci.sink_slots)
    bidx = r["block_idx"]
    nb = 4
    for h in range(2):
        for qi in range(nb):
            sel = set(int(g) for g in bidx[h, qi])
            kc, vc = ci.k_cache.clone(), ci.v_cache.clone()
            g = torch.Generator().manual_seed(h * 10 + qi)
            for f, slot in enumerate(ci.hist_slots):
                for b in range(nb):
                    if f * nb + b not in sel:
                        perm = torch.randperm(16, generator=g) + b * 16
                        kc[slot, b * 16:(b + 1) * 16, h] = (kc[slot, perm, h].float() * 2).bfloat16()
                        vc[slot, b * 16:(b + 1) * 16, h] = (vc[slot, perm, h].float() * -3).bfloat16()
            O2, _ = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, kc, vc, ci.hist_slots,
                                ci.sink_slots, bidx, heads=[h], qblocks=[qi])
            rows = slice(qi * 16, (qi + 1) * 16)
            assert np.array_equal(O2[rows, h], r["O"][rows, h])
            f, b = divmod(min(sel), nb)
            vc[ci.hist_slots[f], b * 16, h] += 1.0
            O3, _ = O.attention(sh, ci.q, ci.k_cur, ci.v_cur, kc, vc, ci.hist_slots,
                                ci.sink_slots, bidx, heads=[h], qblocks=[qi])
            assert not np.allclose(O3[rows, h], r["O"][rows, h], rtol=0, atol=1e-9)


def test_executed_flops_counts_valid_pairs():
    """4*d per (query, key) pair; at full selection this is 4*d*Nq*(all keys)."""
    ci = W.random_small(2, H=2, d=16, T=50, block=16, n_cur_frames=2, n_hist=3,
                        n_sink=1, k_f=3, k_b=4)
    r = O.forward_chunk(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                        ci.hist_slots, ci.sink_slots)
    assert O.executed_flops(ci.shape, r["block_idx"]) == 4 * 16 * 2 * 100 * (100 + 50 + 150)


# ------------------------------------------------------------------ 1-D ablation selection
@pytest.mark.parametrize("seed", range(6))
def test_select_blocks_1d_brute_force(seed):
    """No frame stage: per query block the k-subset of ALL history blocks with the largest
    score sum (scores recomputed here as plain dot products), ties to lower ids."""
    g = np.random.default_rng(100 + seed)
    H, nqb, F, nbpf, d = 2, 3, 3, 4, 8
    q = g.standard_normal((H, nqb, d))
    kb = g.standard_normal((H, F, nbpf, d))
    if seed % 2:                       # exact ties: duplicated block keys across frames
        kb[:, 2] = kb[:, 0]
    k = int(g.integers(1, F * nbpf + 1))
    idx, s = O.select_blocks_1d(q, kb, k)
    assert idx.shape == (H, nqb, k)
    for h in range(H):
        for qq in range(nqb):
            flat = [float(np.dot(q[h, qq], kb[h, f, b])) for f in range(F) for b in range(nbpf)]
            assert np.allclose(s[h, qq], flat, rtol=0, atol=1e-12)
            assert list(idx[h, qq]) == _brute_topk(flat, k)


def test_select_blocks_1d_degenerate_and_two_stage():
    g = np.random.default_rng(7)
    q = g.standard_normal((1, 2, 4))
    kb = g.standard_normal((1, 2, 3, 4))
    idx, _ = O.select_blocks_1d(q, kb, 99)                 # k >= all blocks: every block
    assert idx.tolist() == [[list(range(6)), list(range(6))]]
    # with a single frame the frame stage is trivial: 1-D equals the two-stage selection
    kb1 = kb[:, :1]
    one_d, _ = O.select_blocks_1d(q, kb1, 2)
    two, _ = O.select_blocks(q, kb1, np.zeros((1, 2, 1), dtype=np.int64), 2)
    assert np.array_equal(one_d, two)


# ------------------------------------------------------------------ sparse current chunk
@pytest.mark.parametrize("seed", range(12))
def test_current_selection_brute_force(seed):
    """Own block always kept, plus the (k_c - 1)-subset of the other current blocks with the
    largest score sum (scores recomputed here as plain dot products), lexicographically
    smallest among equal sums; the own block is kept even when it scores lowest."""
    g = np.random.default_rng(200 + seed)
    H, nqb, d = 2, int(g.integers(1, 8)), 6
    q = g.standard_normal((H, nqb, d))
    kc = g.standard_normal((H, nqb, d))
    if seed % 3 == 1 and nqb > 2:           # exact ties between other blocks
        kc[:, 2] = kc[:, 1]
    if seed % 3 == 2:                       # small integers: many exact ties everywhere
        q = g.integers(-1, 2, size=(H, nqb, d)).astype(float)
        kc = g.integers(-1, 2, size=(H, nqb, d)).astype(float)
    k = int(g.integers(1, nqb + 2))          # also k_c > n_qb
    idx, sc = O.select_current_blocks(q, kc, k)
    kk = min(k, nqb)
    assert idx.shape == (H, nqb, kk)
    for h in range(H):
        for qq in range(nqb):
            flat = [float(np.dot(q[h, qq], kc[h, c])) for c in range(nqb)]
            assert np.allclose(sc[h, qq], flat, rtol=0, atol=1e-12)
            others = [c for c in range(nqb) if c != qq]
            best = _brute_topk([flat[c] for c in others], kk - 1) if kk > 1 else []
            assert list(idx[h, qq]) == sorted([qq] + [others[i] for i in best])


def test_current_selection_keeps_own_block_when_it_scores_lowest():
    q = np.ones((1, 3, 2))
    kc = np.array([[[-5.0, -5.0], [1.0, 0.0], [2.0, 0.0]]])     # block 0 scores -10
    idx, _ = O.select_current_blocks(q, kc, 2)
    assert idx[0].tolist() == [[0, 2], [1, 2], [1, 2]]
    assert O.current_boundary_gap([-10.0, 1.0, 2.0], 0, 2) == pytest.approx(0.5)


@pytest.mark.parametrize("T,B,F,S", [(100, 32, 3, 0), (64, 64, 2, 1)])
def test_current_all_kept_equals_dense(T, B, F, S):
    """k_c >= n_qb keeps every current block: the same result as the dense current chunk
    (the same keys in the same order) and as plain SDPA when all history is kept too."""
    nbpf = -(-T // B)
    ci = W.random_small(T + 5, H=2, d=16, T=T, block=B, n_cur_frames=2, n_hist=F,
                        n_sink=S, k_f=F, k_b=nbpf)
    dense = O.forward_chunk(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                            ci.hist_slots, ci.sink_slots)
    from dataclasses import replace
    sparse = O.forward_chunk(replace(ci.shape, k_c=2 * nbpf + 3), ci.q, ci.k_cur, ci.v_cur,
                             ci.k_cache, ci.v_cache, ci.hist_slots, ci.sink_slots)
    assert np.array_equal(sparse["O"], dense["O"]) and np.array_equal(sparse["lse"], dense["lse"])
    assert sparse["cur_idx"].tolist() == [[list(range(2 * nbpf))] * (2 * nbpf)] * 2
    o_ref, lse_ref = _dense_reference_sdpa(ci)
    assert np.allclose(sparse["O"], o_ref, rtol=0, atol=1e-12)


def _masked_reference_sdpa_cur(ci, block_idx, cur_idx):
    """SDPA with a token mask over the current chunk too: a current key token t is visible
    to a query token iff block (t // T) * n_bpf + (t % T) // B is in the query block's
    current list; sinks always; history tokens as in _masked_reference_sdpa."""
    sh = ci.shape
    T, B, Fc = sh.T, sh.block, sh.n_cur_frames
    nbpf = -(-T // B)
    keys = [ci.k_cur.double()] + [ci.k_cache[s].double() for s in ci.sink_slots] + \
           [ci.k_cache[s].double() for s in ci.hist_slots]
    vals = [ci.v_cur.double()] + [ci.v_cache[s].double() for s in ci.sink_slots] + \
           [ci.v_cache[s].double() for s in ci.hist_slots]
    K = torch.cat(keys, 0).permute(1, 0, 2)
    V = torch.cat(vals, 0).permute(1, 0, 2)
    Q = ci.q.double().permute(1, 0, 2)
    n_q, n_dense = Fc * T, Fc * T + sh.n_sink * T
    tq = torch.arange(n_q)
    q_block = (tq // T) * nbpf + (tq % T) // B
    th = torch.arange(sh.n_hist * T)
    k_block = (th // T) * nbpf + (th % T) // B
    mask = torch.ones(sh.H, n_q, n_dense + sh.n_hist * T, dtype=torch.bool)
    for h in range(sh.H):
        cur = torch.zeros(Fc * nbpf, Fc * nbpf, dtype=torch.bool)
        for qb in range(Fc * nbpf):
            cur[qb, torch.as_tensor(cur_idx[h, qb], dtype=torch.long)] = True
        mask[h, :, :n_q] = cur[q_block][:, q_block]
        if sh.n_hist > 0:
            sel = torch.zeros(Fc * nbpf, sh.n_hist * nbpf, dtype=torch.bool)
            for qb in range(Fc * nbpf):
                sel[qb, torch.as_tensor(block_idx[h, qb], dtype=torch.long)] = True
            mask[h, :, n_dense:] = sel[q_block][:, k_block]
    out = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None],
                                                           attn_mask=mask[None],
                                                           scale=sh.scale)[0]
    logits = torch.einsum("hqd,hkd->hqk", Q, K) * sh.scale
    lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), -1)
    return out.permute(1, 0, 2).numpy(), lse.numpy()


@pytest.mark.parametrize("seed,T,B,F,S,nsel,ncur", [(31, 100, 32, 3, 0, 5, 3),
                                                    (32, 70, 16, 0, 1, 0, 4),
                                                    (33, 40, 64, 4, 2, 3, 1)])
def test_sparse_current_equals_masked_sdpa(seed, T, B, F, S, nsel, ncur):
    """Any current-chunk lists (random, each holding its own block) together with any
    history lists give the attention of a token mask built from the lists."""
    nbpf = -(-T // B)
    ci = W.random_small(seed, H=2, d=16, T=T, block=B, n_cur_frames=2, n_hist=F,
                        n_sink=S, k_f=1, k_b=1)
    g = np.random.default_rng(seed)
    nqb = 2 * nbpf
    cur = np.stack([np.stack([np.sort(np.concatenate(
        [[qb], g.choice([c for c in range(nqb) if c != qb], size=min(ncur, nqb) - 1,
                        replace=False)]).astype(np.int64)) for qb in range(nqb)])
        for _ in range(2)])
    bidx = None
    if F > 0:
        bidx = np.stack([np.stack([np.sort(g.choice(F * nbpf, size=nsel, replace=False))
                                   for _ in range(nqb)]) for _ in range(2)])
    o, lse = O.attention(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                         ci.hist_slots, ci.sink_slots, bidx, cur_idx=cur)
    o_ref, lse_ref = _masked_reference_sdpa_cur(ci, bidx, cur)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_current_own_block_only_closed_form():
    """k_c = 1, no history, q = 0: every key of the own block and of the sinks has the
    same logit, so O is the plain mean of those values and lse = log(their count)."""
    ci = W.random_small(41, H=2, d=16, T=50, block=16, n_cur_frames=2, n_hist=0,
                        n_sink=1, k_f=1, k_b=1, k_c=1)
    sh = ci.shape
    zq = torch.zeros_like(ci.q)
    r = O.forward_chunk(sh, zq, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                        ci.hist_slots, ci.sink_slots)
    lens = [16, 16, 16, 2]
    vc64 = ci.v_cur.double().numpy()
    vs = ci.v_cache.double().numpy()[ci.sink_slots[0]]
    for h in range(2):
        for qb in range(8):
            f, b = divmod(qb, 4)
            rows = slice(f * 50 + b * 16, f * 50 + b * 16 + lens[b])
            assert r["cur_idx"][h, qb].tolist() == [qb]
            total = vc64[rows, h].sum(0) + vs[:, h].sum(0)
            n_keys = lens[b] + 50
            assert np.allclose(r["O"][rows, h], total / n_keys, rtol=0, atol=1e-12)
            assert np.allclose(r["lse"][h, rows], math.log(n_keys), rtol=0, atol=1e-12)


def test_executed_flops_with_sparse_current():
    """4*d per pair, with only the kept current blocks' tokens counted."""
    ci = W.random_small(42, H=1, d=16, T=50, block=16, n_cur_frames=1, n_hist=0,
                        n_sink=0, k_f=1, k_b=1)
    cur = np.array([[[0, 3], [1, 3], [0, 2], [3, 2]]])      # lists need not be sorted here
    lens = [16, 16, 16, 2]
    expect = sum(lens[qb] * sum(lens[c] for c in cur[0, qb]) for qb in range(4))
    assert O.executed_flops(ci.shape, None, cur) == 4 * 16 * expect


# ------------------------------------------------------------------ chunk-aware growth
@pytest.mark.parametrize("n,first,mean,final", [(7, 2, 0.8, 0.9), (20, 2, 0.8, 0.95),
                                                (5, 3, 0.5, 0.6), (4, 1, 0.3, 0.2)])
def test_cag_conditions_hold(n, first, mean, final):
    """The solved schedule meets both conditions and has the form base - beta/sqrt(i)."""
    s, s_base, beta = C.cag_sparsity(n, first, mean, final)
    sparse = s[first - 1:]
    assert sum(sparse) / len(sparse) == pytest.approx(mean, abs=1e-12)
    assert s[-1] == pytest.approx(final, abs=1e-12)
    assert all(v == 0.0 for v in s[:first - 1])
    for i in range(first, n + 1):
        assert s[i - 1] == pytest.approx(s_base - beta / math.sqrt(i), abs=1e-12)
    # later chunks are sparser exactly when the last chunk is above the mean
    steps = [b - a for a, b in zip(sparse, sparse[1:])]
    assert all((d > 0) == (final > mean) for d in steps)


def test_cag_two_chunks_by_hand():
    """n = 2, first = 1: (s_1 + s_2)/2 = m and s_2 = f give s_1 = 2m - f, and
    beta = (s_2 - s_1) / (1 - 1/sqrt(2))."""
    m, f = 0.5, 0.7
    s, s_base, beta = C.cag_sparsity(2, 1, m, f)
    assert s == pytest.approx([2 * m - f, f], abs=1e-12)
    assert beta == pytest.approx((f - (2 * m - f)) / (1 - 1 / math.sqrt(2)), abs=1e-12)
    assert s_base == pytest.approx(s[0] + beta, abs=1e-12)


def test_cag_constant_and_single_sparse_chunk():
    s, _, beta = C.cag_sparsity(6, 2, 0.75, 0.75)
    assert beta == pytest.approx(0.0, abs=1e-12)
    assert s[1:] == pytest.approx([0.75] * 5, abs=1e-12)
    s, _, beta = C.cag_sparsity(3, 3, 0.4, 0.4)
    assert s == [0.0, 0.0, 0.4] and beta == 0.0
    with pytest.raises(ValueError):
        C.cag_sparsity(3, 3, 0.4, 0.5)
    keep, budgets = C.cag_schedule(3, 2, 0.5, 0.5, [0, 4, 4], n_bpf=10, kf_max=2)
    assert keep == [1.0, 0.5, 0.5] and budgets[0] == (0, 0)


@pytest.mark.parametrize("F,n_bpf,kf_max", [(3, 25, 6), (18, 25, 6), (5, 13, 2), (1, 4, 8)])
def test_cag_budget_exhaustive(F, n_bpf, kf_max):
    """Over every pair k_f in [1, kf_max], k_b in [1, n_bpf], the budget keeps
    k_f = min(kf_max, F) frames and its k_b brings the kept fraction nearest to the keep
    ratio among all k_b for that k_f; it never exceeds the frame's blocks."""
    for keep in np.linspace(0.0, 1.0, 41):
        kf, kb = C.cag_budget(float(keep), F, n_bpf, kf_max, dense=False)
        assert kf == min(kf_max, F) and 1 <= kb <= n_bpf
        errs = {b: abs(kf * b / (F * n_bpf) - keep) for b in range(1, n_bpf + 1)}
        assert errs[kb] <= min(errs.values()) + 1e-12
        assert C.cag_budget(float(keep), F, n_bpf, kf_max, dense=True) == (F, n_bpf)
    assert C.cag_budget(0.5, 0, n_bpf, kf_max, dense=False) == (0, 0)
