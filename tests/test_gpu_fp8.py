"""FP8 (e4m3) variant of the attention stage, through the C ABI, against the float64 oracle.

The quantiser's codes and scales must be the oracle's bit for bit (rounding to nearest,
ties to the even code; power-of-two scales chosen by exact comparison).  The attention on
e4m3 queries and keys (QK^T on the FP8 tensor cores) must match the float64 attention of
the dequantised queries and keys with the bf16 values within the stated tolerance
(max-abs <= 2e-2, relative L2 <= 5e-3, lse within 2e-3): the products of e4m3 values are
exact and the rest of the path is the bf16 one."""
import numpy as np
import pytest
import torch
from dataclasses import replace

import lf_workloads as W
from oracle import fp8q as Q
from oracle import hsa64 as O
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _decode(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_quantiser_matches_oracle_bit_for_bit(gpu_lib):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(300, 3, 128, generator=g) * torch.exp(torch.empty(300, 3, 1).uniform_(-6, 6, generator=g))
    x[4, 1] = 0.0
    x[9, 2, :5] = torch.tensor([448.0, -464.0, 1e-30, 3.0, 2.0 ** -12])
    xb = x.to(torch.bfloat16)
    xd = xb.cuda()
    x8 = torch.empty(xd.shape, dtype=torch.uint8, device="cuda")
    rs = torch.empty(300, 3, device="cuda")
    gpu_lib.lf_quantize_e4m3(xd, x8, row_scale=rs)
    hs = torch.empty(3, device="cuda")
    gpu_lib.lf_e4m3_head_scales([xd[:100], xd[100:]], hs)
    x8h = torch.empty_like(x8)
    gpu_lib.lf_quantize_e4m3(xd, x8h, head_scale=hs)
    torch.cuda.synchronize()
    o8, os_ = Q.quantize_rows(xb)
    assert np.array_equal(rs.cpu().double().numpy(), os_)
    assert np.array_equal(_decode(x8), o8)
    o8h, osh = Q.quantize_per_head(xb)
    assert np.array_equal(hs.cpu().double().numpy(), osh)
    assert np.array_equal(_decode(x8h), o8h)


def _fp8_inputs(gpu_lib, ci):
    sh = ci.shape
    t = G.to_dev(ci)
    n = t["q"].shape[0]
    q8 = torch.empty(t["q"].shape, dtype=torch.uint8, device="cuda")
    qs = torch.empty(n, sh.H, device="cuda")
    gpu_lib.lf_quantize_e4m3(t["q"], q8, row_scale=qs)
    ks = torch.empty(sh.H, device="cuda")
    kc_rows = t["k_cache"].view(-1, sh.H, sh.d)
    gpu_lib.lf_e4m3_head_scales([t["k_cur"], kc_rows], ks)
    kc8 = torch.empty(t["k_cur"].shape, dtype=torch.uint8, device="cuda")
    kh8 = torch.empty(t["k_cache"].shape, dtype=torch.uint8, device="cuda")
    gpu_lib.lf_quantize_e4m3(t["k_cur"], kc8, head_scale=ks)
    gpu_lib.lf_quantize_e4m3(kc_rows, kh8.view(-1, sh.H, sh.d), head_scale=ks)
    torch.cuda.synchronize()
    # the oracle's own quantisation of the same bf16 inputs
    oq8, oqs = Q.quantize_rows(ci.q)
    allk = np.concatenate([O._f64(ci.k_cur), O._f64(ci.k_cache).reshape(-1, sh.H, sh.d)])
    _, oks = Q.quantize_per_head(allk)
    assert np.array_equal(qs.cpu().double().numpy(), oqs) and np.array_equal(ks.cpu().double().numpy(), oks)
    q_hat = oq8 * oqs[..., None]
    kc_hat = Q.round_e4m3(O._f64(ci.k_cur) / oks[None, :, None]) * oks[None, :, None]
    kh_hat = Q.round_e4m3(O._f64(ci.k_cache) / oks[None, None, :, None]) * oks[None, None, :, None]
    assert np.array_equal(_decode(q8), oq8)
    assert np.array_equal(_decode(kh8) * oks[None, None, :, None], kh_hat)
    return t, dict(q8=q8, qs=qs, kc8=kc8, kh8=kh8, ks=ks), (q_hat, kc_hat, kh_hat)


def _check(gpu_lib, ci, bidx, cidx=None):
    sh = ci.shape
    t, f, (q_hat, kc_hat, kh_hat) = _fp8_inputs(gpu_lib, ci)
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((sh.H, t["q"].shape[0]), float("nan"), device="cuda")
    bi = None if sh.n_hist == 0 else torch.as_tensor(bidx, dtype=torch.int32).cuda().contiguous()
    ci_ = None if cidx is None else torch.as_tensor(cidx, dtype=torch.int32).cuda().contiguous()
    gpu_lib.lf_block_sparse_attn_e4m3(sh, f["q8"], f["qs"], f["kc8"], t["v_cur"], f["kh8"],
                                      t["v_cache"], f["ks"], ci.hist_slots, ci.sink_slots, bi,
                                      out, lse, cur_idx=ci_)
    torch.cuda.synchronize()
    o_ref, lse_ref = O.attention(sh, q_hat, kc_hat, ci.v_cur, kh_hat, ci.v_cache, ci.hist_slots,
                                 ci.sink_slots, bidx, cur_idx=cidx)
    G.assert_output_close(out, o_ref, what=ci.name + "/e4m3")
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= G.LSE_ABS
    assert gpu_lib.lf_device_status() == 0
    return out


def _oracle_lists(ci):
    sh = ci.shape
    if sh.n_hist == 0:
        return None
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    kb, kf = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)
    fidx, _ = O.select_frames(qb, kf, sh.k_f)
    bidx, _ = O.select_blocks(qb, kb, fidx, sh.k_b)
    return bidx


SMALL = {
    "sinks_b64": lambda: W.random_small(2, H=2, d=128, T=200, block=64, n_cur_frames=3,
                                        n_hist=4, n_sink=1, k_f=3, k_b=2),
    "b128": lambda: W.random_small(3, H=3, d=128, T=300, block=128, n_cur_frames=2,
                                   n_hist=3, n_sink=0, k_f=2, k_b=2),
    "no_history": lambda: W.random_small(6, H=2, d=128, T=192, block=64, n_cur_frames=1,
                                         n_hist=0, n_sink=0, k_f=1, k_b=1),
    "frames_1560": lambda: W.random_small(8, H=2, d=128, T=1560, block=64, n_cur_frames=1,
                                          n_hist=3, n_sink=1, k_f=2, k_b=12),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_e4m3_attention_small(gpu_lib, name):
    ci = SMALL[name]()
    _check(gpu_lib, ci, _oracle_lists(ci))


def test_e4m3_attention_sparse_current(gpu_lib):
    ci = W.random_small(51, H=2, d=128, T=200, block=64, n_cur_frames=3, n_hist=4, n_sink=1,
                        k_f=2, k_b=2, k_c=5)
    sh = ci.shape
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    cidx, _ = O.select_current_blocks(qb, O.compress_queries(ci.k_cur, sh.T, sh.block), sh.k_c)
    _check(gpu_lib, ci, _oracle_lists(ci), cidx)


def test_e4m3_attention_480p_full_size(gpu_lib):
    ci = W.p480(0)
    out = _check(gpu_lib, ci, _oracle_lists(ci))
    assert torch.isfinite(out.float()).all()
