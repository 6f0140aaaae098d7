"""Head-parallel sharding of one chunk, proven on one GPU.

Heads are independent at every stage (pooling, scores, selection, attention), so running
the library once per contiguous head range and concatenating must reproduce the call over
all heads.  With the tail split off (every query tile computed whole) the rounding of a
tile no longer depends on how many tiles a launch holds, and the outputs, lse and indices
must be the same bits.  With the default split the indices must still be the same bits
and the outputs agree within the stated tolerance.  This is the data path a multi-GPU run
uses (each rank owns a head range and needs no collective); only the device count
differs."""
import numpy as np
import pytest
import torch

import lf_workloads as W
from bench import head_shard, shard_heads
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _forward(ci):
    out, lse, bidx = G.gpu_forward(ci, G.to_dev(ci))
    torch.cuda.synchronize()
    return out, lse, bidx


@pytest.mark.parametrize("world", [2, 3, 5])
def test_head_shards_reproduce_the_whole_chunk(gpu_lib, world):
    ci = W.p480(0)
    H = ci.shape.H
    try:
        gpu_lib.lf_debug_configure(tail_split=False)
        full = _forward(ci)
        parts = []
        for r in range(world):
            h0, h1 = head_shard(H, world, r)
            parts.append((h0, h1, _forward(shard_heads(ci, h0, h1))))
    finally:
        gpu_lib.lf_debug_configure()
    for h0, h1, (o, l, b) in parts:
        assert torch.equal(o, full[0][:, h0:h1]), (world, h0, h1)
        assert torch.equal(l, full[1][h0:h1]), (world, h0, h1)
        assert torch.equal(b, full[2][h0:h1]), (world, h0, h1)
    # default decomposition: indices identical, outputs within tolerance
    full = _forward(ci)
    for r in range(world):
        h0, h1 = head_shard(H, world, r)
        o, l, b = _forward(shard_heads(ci, h0, h1))
        assert torch.equal(b, full[2][h0:h1])
        G.assert_output_close(o, full[0][:, h0:h1].float().cpu().double().numpy(),
                              what=f"shard {r}/{world}")
        assert (l - full[1][h0:h1]).abs().max().item() <= G.LSE_ABS
    assert gpu_lib.lf_device_status() == 0
