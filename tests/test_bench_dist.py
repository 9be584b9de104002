"""The benchmark's multi-rank plumbing on CPU ranks (gloo, world size 2): the
barrier, the MAX reduction of the timed region, and the whole-job rate."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(dist)
        secs = 1.0 + rank  # rank 1 is the slow one
        got = bench.max_over_ranks(dist, secs, device="cpu")
        bench.barrier(dist)
        results[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, results), nprocs=2, join=True, start_method="spawn")
    assert results[0] == 2.0 and results[1] == 2.0


def test_job_rate_is_weak_scaling_aggregate():
    # 2 ranks x 68.75 GFLOP each over a slowest-rank time of 0.1 ms per step
    v = bench.job_rate(68.75e9, 2, 0.1e-3 * 10, 10, "TFLOP/s")
    assert abs(v - 2 * 687.5) < 1e-6
    assert bench.job_rate(17.18e9, 1, 3e-3, 1, "GB/s") == pytest.approx(17.18e9 / 3e-3 / 1e9)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(None, 3.5) == 3.5
    bench.barrier(None)


def test_visible_pairs_closed_forms():
    from synth import workloads as sw
    r = sw.RECIPES["dot_causal_2k_bf16"]
    assert bench.visible_pairs(r) == 2048 * 2049 // 2
    r4 = sw.RECIPES["sink_gqa_window_16k_bf16"]
    W, L = r4.window, r4.L
    assert bench.visible_pairs(r4) == W * (W + 1) // 2 + (L - W) * W
    r2 = sw.RECIPES["dot_bias10_2k_f32"]
    assert bench.visible_pairs(r2) == 2048 * 2048
    amount, unit, bound = bench.work_units(sw.RECIPES["decode_sink_gqa_128k_bf16"])
    assert (amount, unit, bound) == (32 * 8 * 131072 * 256 * 2, "GB/s", "hbm")


def test_visible_pairs_and_decode_keys_match_the_oracle_mask():
    """Work accounting of every mask kind against the oracle's visibility, by brute force."""
    import dataclasses

    import numpy as np

    from oracle import attention as orc
    from synth import workloads as sw
    base = sw.RECIPES["tiny_rbf_sink_causal_f32"]
    cases = [("none", 0, 0), ("causal", 0, 0), ("window", 7, 0), ("streaming", 7, 3), ("streaming", 5, 0),
             ("streaming", 4, 200), ("streaming", 1, 1)]
    for L, S in ((37, 37), (5, 60), (60, 20), (1, 90)):
        for mk, w, keep in cases:
            r = dataclasses.replace(base, L=L, S=S, mask_kind=mk, window=w, keep=keep)
            vis = orc.visible(np.arange(L), S, L, mk, w, keep)
            assert bench.visible_pairs(r) == int(vis.sum()), (L, S, mk, w, keep)
            if mk in ("window", "streaming"):
                assert bench.decode_keys(r) == int(vis.any(axis=0).sum()), (L, S, mk, w, keep)


def test_visible_pairs_total_with_keep_bits_and_padding():
    """Work accounting with keep bits and ragged padding equals the oracle's visibility count."""
    import dataclasses

    import numpy as np

    from oracle import attention as orc
    from synth import workloads as sw
    base = sw.RECIPES["tiny_rbf_sink_causal_f32"]
    for mk, w in (("none", 0), ("causal", 0), ("window", 9)):
        for keep, pl, pr in (("random10", 0.0, 0.0), ("none", 0.5, 0.0), ("random10", 0.3, 0.4), ("none", 0.0, 0.6)):
            r = dataclasses.replace(base, N=5, L=40, S=61, mask_kind=mk, window=w, keep_mask=keep, pad_left=pl,
                                    pad_right=pr)
            km = sw.keep_matrix(r)
            ks, ke = sw.kv_ranges(r)
            want = 0
            for n in range(r.N):
                vis = orc.padded_visible(orc.visible(np.arange(r.L), r.S, r.L, mk, w), km,
                                         None if ks is None else (ks[n], ke[n]))
                want += int(vis.sum())
            assert bench.visible_pairs_total(r) == want, (mk, keep, pl, pr)
