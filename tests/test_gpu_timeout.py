"""The bounded device waits of the attention kernel, made to run out without a GPU fault.

A test hook (lf_debug_configure) shortens the wait limit of the next launches to 20 ms and
makes the first CTA of each attention launch never arm its query barrier, so nothing ever
arrives on it.  Every wait of that CTA is bounded: it gives up, the CTA drains its copies,
frees its tensor memory and returns, and the device status word reads LF_ERR_TIMEOUT.  The
context stays usable: a normal call afterwards matches the float64 oracle and leaves the
status at LF_OK.  Nothing here faults, traps or hangs the GPU."""
import time

import numpy as np
import pytest
import torch

import lf_workloads as W
from oracle import hsa64 as O
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

LF_ERR_TIMEOUT = 4


def _oracle_lists(ci):
    sh = ci.shape
    qb = O.compress_queries(ci.q, sh.T, sh.block)
    kb, kf = O.compress_keys(ci.k_cache, ci.hist_slots, sh.T, sh.block)
    fidx, _ = O.select_frames(qb, kf, sh.k_f)
    bidx, _ = O.select_blocks(qb, kb, fidx, sh.k_b)
    return bidx


def test_stalled_wait_times_out_and_context_recovers(gpu_lib):
    ci = W.tiny(0)
    t = G.to_dev(ci)
    bidx = _oracle_lists(ci)
    assert gpu_lib.lf_device_status(True) == 0
    try:
        gpu_lib.lf_debug_configure(wait_limit_ns=20_000_000, stall=True)
        t0 = time.perf_counter()
        G.gpu_attention(ci, t, bidx)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        gpu_lib.lf_debug_configure()                  # defaults: 2 s, no stall, split on
    assert gpu_lib.lf_device_status(True) == LF_ERR_TIMEOUT
    assert dt < 1.5, f"the stalled launch took {dt:.3f} s (limit 20 ms per wait)"
    # the context is usable and the normal path is unaffected
    o_ref, lse_ref = O.attention(ci.shape, ci.q, ci.k_cur, ci.v_cur, ci.k_cache, ci.v_cache,
                                 ci.hist_slots, ci.sink_slots, bidx)
    out, lse = G.gpu_attention(ci, t, bidx)
    torch.cuda.synchronize()
    assert gpu_lib.lf_device_status(True) == 0
    G.assert_output_close(out, o_ref, what="after the timeout")
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= G.LSE_ABS

