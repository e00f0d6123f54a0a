"""Row-sharded quantization across ranks, tested on CPU with gloo (world size 2).

The collective step is the all-reduce-MAX of per-rank tensor scales; the test computes each
rank's S_r with the oracle on its row shard and checks that the reduced S equals the
oracle's S of the whole tensor bit for bit, that the shards quantized with it reproduce the
whole tensor's codes, and that a non-finite element on one rank reaches every rank.  The
timing helper (slowest rank) is checked too.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import oracle as O
    from fp4_block_scaled_nvfp4_b200 import synth
    from fp4_block_scaled_nvfp4_b200.dist import max_over_ranks, reduce_global_scale

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.make("cfg3", rows=32, cols=256)
        x = O.widen_bf16(w["x"])
        shard = x[rank * 16:(rank + 1) * 16]
        s_loc, st = O.tensor_scale(shard)
        s_all = reduce_global_scale(torch.tensor([s_loc], dtype=torch.float32))
        codes = O.nvfp4_quantize(shard, "sweep_mse", S=float(s_all.item()))
        bad = shard.copy()
        if rank == 1:
            bad[3, 7] = np.nan
        s_bad_loc, _ = O.tensor_scale(bad)
        s_bad = reduce_global_scale(torch.tensor([s_bad_loc], dtype=torch.float32))
        slowest = max_over_ranks(1.5 + rank)
        # the 16-point rotated path: S of the rotated shard, reduced the same way
        s_rot_loc, _ = O.tensor_scale(O.rotate16(shard))
        s_rot = reduce_global_scale(torch.tensor([s_rot_loc], dtype=torch.float32))
        rot = O.nvfp4_quantize(shard, "sweep_mse", S=float(s_rot.item()), hadamard16=True)
        # IF6: its own tensor scale RN(amax / 1920), reduced the same way
        s6 = reduce_global_scale(torch.tensor([O.if6_tensor_scale(shard)], dtype=torch.float32))
        q6 = O.if6_quantize(shard, S=float(s6.item()))
        results[rank] = (float(s_all.item()), codes["codes"].tobytes(), codes["scales"].tobytes(),
                         float(s_bad.item()), slowest, float(s_rot.item()), rot["codes"].tobytes(),
                         rot["scales"].tobytes(), float(s6.item()), q6["codes"].tobytes(), q6["scales"].tobytes())
    finally:
        dist.destroy_process_group()


def test_sharded_scale_matches_whole_tensor():
    import oracle as O
    from fp4_block_scaled_nvfp4_b200 import synth

    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world, start_method="spawn", join=True)
    w = synth.make("cfg3", rows=32, cols=256)
    x = O.widen_bf16(w["x"])
    whole = O.nvfp4_quantize(x, "sweep_mse")
    whole_rot = O.nvfp4_quantize(x, "sweep_mse", hadamard16=True)
    whole6 = O.if6_quantize(x)
    assert whole_rot["S"] != whole["S"]
    for rank in range(world):
        s_all, c, sc, s_bad, slowest, s_rot, c_rot, sc_rot, s6, c6, sc6 = results[rank]
        assert np.float32(s6).view(np.uint32) == np.float32(whole6["S"]).view(np.uint32)
        assert c6 == whole6["codes"][rank * 16:(rank + 1) * 16].tobytes()
        assert sc6 == whole6["scales"][rank * 16:(rank + 1) * 16].tobytes()
        assert np.float32(s_rot).view(np.uint32) == np.float32(whole_rot["S"]).view(np.uint32)
        assert c_rot == whole_rot["codes"][rank * 16:(rank + 1) * 16].tobytes()
        assert sc_rot == whole_rot["scales"][rank * 16:(rank + 1) * 16].tobytes()
        assert np.float32(s_all).view(np.uint32) == np.float32(whole["S"]).view(np.uint32)
        assert c == whole["codes"][rank * 16:(rank + 1) * 16].tobytes()
        assert sc == whole["scales"][rank * 16:(rank + 1) * 16].tobytes()
        assert np.isnan(s_bad)
        assert slowest == 2.5
