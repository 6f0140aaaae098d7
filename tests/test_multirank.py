"""The benchmark's multi-rank logic on CPU: two gloo ranks, each with its own chunk (weak
scaling, no collective on the data path); the job time is the slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"))
        dist.barrier()
        out[rank] = ms
        # every rank ran its own chunk: the whole-job value counts both
        out[2 + rank] = bench.weak_scaling_value(10 ** 12, world, ms)
        # a head-sharded chunk: the job's work is the sum of the ranks' shares
        out[4 + rank] = bench.sum_over_ranks([1.5e12, 2.5e12][rank], torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_and_count_all_work():
    world = 2
    out = mp.get_context("spawn").Array("d", 6)
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert list(out[:2]) == [5.0, 5.0]
    assert out[2] == out[3] == pytest.approx(2 * 1e12 / 5e-3 / 1e12)
    assert out[4] == out[5] == pytest.approx(4e12)


def test_single_process_is_identity():
    assert bench.max_over_ranks(7.5, torch.device("cpu")) == 7.5
    assert bench.weak_scaling_value(2 * 10 ** 12, 1, 1000.0) == pytest.approx(2.0)


def test_tail_split_rule():
    import lf_workloads as W
    assert bench.tail_split(W.p480_shape())          # 456 tiles = 3 x 148 + 12
    assert not bench.tail_split(W.large_shape())     # 1560 tiles = 10 x 148 + 80


@pytest.mark.parametrize("H,world", [(12, 1), (12, 2), (12, 5), (40, 8), (3, 3), (7, 4)])
def test_head_shards_cover_every_head_once(H, world):
    spans = [bench.head_shard(H, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == H
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))          # contiguous
    sizes = [h1 - h0 for h0, h1 in spans]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_shard_heads_is_a_head_slice():
    import lf_workloads as W
    ci = W.tiny(0)
    part = bench.shard_heads(ci, 1, 2)
    assert part.shape.H == 1 and part.shape.T == ci.shape.T
    assert torch.equal(part.q[:, 0], ci.q[:, 1])
    assert torch.equal(part.k_cache[:, :, 0], ci.k_cache[:, :, 1])
    assert part.q.is_contiguous() and part.hist_slots == ci.hist_slots


def test_oracle_timings_are_bounded_samples():
    """The CPU-baseline helpers: one (chunk, head) unit per sample without a budget, the
    torch thread count restored after the single-thread run, the FLOPs those of the units
    run; a workload of several chunks is sampled across its chunks in order."""
    import lf_workloads as W
    ci = W.tiny(0)
    n = torch.get_num_threads()
    f, dt, cores, units = bench.oracle_sample([ci])
    assert units == 1 and f > 0 and dt > 0 and cores == n
    f1, dt1 = bench.oracle_single_core([ci])
    assert f1 == f and dt1 > 0
    assert torch.get_num_threads() == n
    f_all, _, _, units_all = bench.oracle_sample([ci], budget_s=1e9)
    assert units_all == ci.shape.H and f_all == ci.shape.H * f
    ci2 = W.tiny(1)
    f2, _, _, u2 = bench.oracle_sample([ci, ci2], budget_s=1e9)
    g2, _, _, _ = bench.oracle_sample([ci2], budget_s=1e9)
    assert u2 == 2 * ci.shape.H and f2 == f_all + g2
    # starting at unit H runs the second chunk's first head
    f_b, _, _, _ = bench.oracle_sample([ci, ci2], first=ci.shape.H)
    f_c, _, _, _ = bench.oracle_sample([ci2])
    assert f_b == f_c


def test_clock_summary_from_fake_rows():
    """The clock record of the JSON line from nvidia-smi rows (a fake of its CSV output):
    median SM clock, max clock, the active throttle reasons; bad rows are skipped."""
    row = "0, {sm}, 1965, 700.5, 0x{m}, {hw}, Not Active, Not Active, {pc}"
    rows = [row.format(sm=1965, m="0", hw="Not Active", pc="Not Active"),
            row.format(sm=1800, m="4", hw="Not Active", pc="Active"),
            row.format(sm=1900, m="4", hw="Not Active", pc="Active"),
            "0, [N/A], 1965, 700, 0x0, Not Active, Not Active, Not Active, Not Active",
            "garbage"]
    out = bench.summarise_clocks(rows)
    assert out == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}
    rows.append(row.format(sm=1200, m="8", hw="Active", pc="Not Active"))
    assert bench.summarise_clocks(rows)["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.summarise_clocks([])["sm_mhz"] is None


def test_forward_launch_counts():
    """Kernels one lf_forward_chunk call launches (the benchmark's gpu_launches claim):
    selection, the current-chunk choice when it is sparse, plan_kernel unless the pick
    kernel wrote the plans, attention, and merge when the tail is split."""
    from dataclasses import replace
    import lf_workloads as W

    class Run:
        def __init__(self, sh, kc):
            self.sh, self.kc = sh, kc
    p480 = W.p480_shape()
    assert bench.ChunkRun.forward_launches(Run(p480, 0)) == 3 + 1 + 1       # tail split
    assert bench.ChunkRun.forward_launches(Run(W.large_shape(), 0)) == 3 + 1
    # sparse current chunk: its pooling shares the selection's launch, then its choice and
    # plan_kernel
    assert bench.ChunkRun.forward_launches(Run(replace(p480, k_c=15), 15)) == 3 + 1 + 1 + 1 + 1
    # first chunk (no history): query/current pooling and the choice, plan_kernel
    first = replace(p480, n_hist=0, k_c=15)
    assert bench.ChunkRun.forward_launches(Run(first, 15)) == \
        2 + 1 + 1 + (1 if bench.tail_split(first) else 0)
