"""The multi-GPU host logic on CPU with two gloo ranks: each rank owns whole fold groups
of a global batch, the shards need no exchange (samples are independent by the reset),
and the benchmark's timing is the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_shard_ranges_partition_whole_fold_groups():
    for B, world, fold in [(256, 1, 1), (256, 2, 4), (256, 8, 8), (12, 4, 3), (10, 3, 2), (7, 7, 1)]:
        seen = []
        for r in range(world):
            lo, hi = bench.shard_range(B, world, r, fold)
            assert lo % fold == 0 and hi % fold == 0
            seen.extend(range(lo, hi))
        assert seen == list(range(B))


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from selective_scan_sfm_b200 import synth
        B = 8
        d = synth.make_inputs(B=B, D=6, T=9, N=4, dtype="f32", seed=3)
        lo, hi = bench.shard_range(B, world, rank, fold=2)
        f = lambda t: t[lo:hi].double().numpy()
        p = lambda t: t.double().numpy()
        y = oracle.mixer_layer(f(d["x"]), f(d["dt"]), f(d["z"]), f(d["Bm"]), f(d["Cm"]), p(d["A"]), p(d["Dskip"]),
                               p(d["dt_bias"]), p(d["conv_w"]), p(d["conv_b"]), aux_init_in=True)
        np.save(os.path.join(out_dir, "y%d.npy" % rank), y)
        t = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        np.save(os.path.join(out_dir, "t%d.npy" % rank), np.array([t]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_match_the_whole_batch(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle
    from selective_scan_sfm_b200 import synth
    d = synth.make_inputs(B=8, D=6, T=9, N=4, dtype="f32", seed=3)
    p = lambda t: t.double().numpy()
    whole = oracle.mixer_layer(p(d["x"]), p(d["dt"]), p(d["z"]), p(d["Bm"]), p(d["Cm"]), p(d["A"]), p(d["Dskip"]),
                               p(d["dt_bias"]), p(d["conv_w"]), p(d["conv_b"]), aux_init_in=True)
    parts = [np.load(tmp_path / ("y%d.npy" % r)) for r in range(world)]
    np.testing.assert_array_equal(np.concatenate(parts, axis=0), whole)
    for r in range(world):
        assert float(np.load(tmp_path / ("t%d.npy" % r))[0]) == 2.5  # every rank sees the max
