"""N > 1 host logic on CPU: two gloo ranks, independent instances, max-over-ranks timing.

The attention path shards by (b, h) with no data-path collective, so the only
multi-rank logic is on the host: each rank owns a distinct seeded instance, and
the step time is the max over ranks. Runs as two spawned processes on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local = [10.0 + rank * 5.0, 3.0 - rank]  # rank 1 is slower on the first, faster on the second
        got = bench.reduce_max(local, world, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed("c2", rank))
        out[rank] = (got, seeds, bench.job_throughput(1e12, world, got[0]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_seeds():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        got, seeds, tput = out[r]
        assert got == [15.0, 3.0]
        assert len(set(seeds)) == world  # independent instances
        assert tput == pytest.approx(1e12 * world / 15e-3 / 1e12)


def _shard_worker(rank, world, port, out):
    """Each rank runs the oracle (standing in for the GPU path, which needs a device) on its own
    head range of one small arrow problem, then the heads are all-gathered."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np

        import workloads as W
        from block_sparse_attention_37_b200 import sharding
        from oracle import attention as OA
        from oracle import masks as OM
        w = W.arrow_case(B=2, H=4, n_text=32, grid_hw=(4, 24), d=16, block=32, seed=3,
                         fracs=(0.5, 0.5, 0.0), with_cache=False)
        s = w["shape"]
        q, k, v = (sharding.local_heads(t, rank, world) for t in (w["q"], w["k"], w["v"]))
        modes = sharding.local_heads(torch.from_numpy(w["head_mode"]), rank, world, head_dim=0).numpy()
        wins = sharding.local_heads(torch.from_numpy(w["window"]), rank, world, head_dim=0).numpy()
        o_local = torch.empty(q.shape, dtype=torch.float64)
        for b in range(s.B):
            for h in range(q.shape[1]):
                fn = lambda r, h=h: OM.arrow_token_mask(s.N, s.n_text, s.block_q, int(modes[h]), int(wins[h]), r)
                o_local[b, h] = torch.from_numpy(OA.head_forward(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                                                 v[b, h].double().numpy(), int(modes[h]), fn,
                                                                 s.d ** -0.5))
        full = sharding.gather_heads(o_local, world)
        out[rank] = (sharding.head_range(s.H, rank, world), full.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharding_gathers_every_head():
    """Head sharding (each rank computes its contiguous head range; one all-gather per batch item)
    yields, on every rank, the output of the unsharded problem."""
    import numpy as np

    import workloads as W
    from block_sparse_attention_37_b200 import sharding
    from oracle import attention as OA
    from oracle import masks as OM
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    w = W.arrow_case(B=2, H=4, n_text=32, grid_hw=(4, 24), d=16, block=32, seed=3, fracs=(0.5, 0.5, 0.0),
                     with_cache=False)
    s = w["shape"]
    exp = np.zeros((s.B, s.H, s.N, s.d))
    for b in range(s.B):
        for h in range(s.H):
            mode, win = int(w["head_mode"][h]), int(w["window"][h])
            fn = lambda r, mode=mode, win=win: OM.arrow_token_mask(s.N, s.n_text, s.block_q, mode, win, r)
            exp[b, h] = OA.head_forward(w["q"][b, h].double().numpy(), w["k"][b, h].double().numpy(),
                                        w["v"][b, h].double().numpy(), mode, fn, s.d ** -0.5)
    assert out[0][0] == (0, 2) and out[1][0] == (2, 4)
    for r in range(world):
        np.testing.assert_array_equal(out[r][1], exp)
    with pytest.raises(ValueError):
        sharding.head_range(5, 0, 2)


def test_shard_workload_slices_every_per_head_input():
    """bench --shard heads: each rank's workload holds exactly its head range of every per-head
    input (Q, K, V, cache, mode table, windows, block bias, bias kinds) and the rest unchanged."""
    import numpy as np

    import bench
    import workloads as W
    w = W.arrow_case(B=2, H=6, n_text=32, grid_hw=(4, 8), d=16, block=32, seed=1)
    d = W.dlm_case(B=1, H=4, n_prefill=256, n_gen=128, d=16, block=64, seed=2)
    d["q"], d["k"], d["v"] = W.qkv_normal(1, 4, 384, 16, 2)
    for case, world in ((w, 3), (d, 2)):
        H = case["shape"].H
        parts = [bench.shard_workload(case, r, world) for r in range(world)]
        for r, p in enumerate(parts):
            h0, h1 = r * H // world, (r + 1) * H // world
            assert p["shape"].H == h1 - h0 and p["shape"].N == case["shape"].N
            for key in ("q", "k", "v", "cache"):
                if case.get(key) is not None:
                    assert torch.equal(p[key], case[key][:, h0:h1]) and p[key].is_contiguous()
            for key in ("head_mode", "window"):
                if key in case:
                    assert np.array_equal(p[key], case[key][h0:h1])
            if "bias" in case:
                assert torch.equal(p["bias"], case["bias"][h0:h1])
                assert p["bias_kinds"] == case["bias_kinds"][h0:h1]
        assert sum(p["shape"].H for p in parts) == H
