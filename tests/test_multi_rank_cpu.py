"""Data-parallel path on CPU with two gloo ranks.

Calibration is the one exchange: each rank reduces its share of the calibration tokens and the shares
are combined with an all-reduce(MAX); the result must equal the single-process abs-max bit for bit.
The online path has no exchange: each rank's tokens give exactly the rows the unsharded run gives.
The per-rank arithmetic here is the oracle's (there is no GPU); the code under test is the sharding
and the collective.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_quantization_calib_b200 import dist as sqdist
from post_quantization_calib_b200 import synth


def h16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import oracle as orc
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w = synth.WORKLOADS[0]
        d = synth.group_inputs(w, 0, "cpu")
        calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], "cpu")))
        lo, hi = sqdist.shard_range(calib.shape[0] - 37, world, rank)     # uneven shares
        mine = [calib[lo:hi]]

        def absmax_fn(batch, amax):
            prev = None if amax is None else amax.numpy()
            return torch.from_numpy(orc.calibrate_absmax(h16(batch), amax=prev, accumulate=prev is not None))

        amax = sqdist.sharded_absmax(mine, absmax_fn)
        full = orc.calibrate_absmax(h16(calib[: calib.shape[0] - 37]))
        assert np.array_equal(amax.numpy(), full), "sharded calibration differs from the single-process one"

        # every rank now holds the same s and INT8 weight; each quantises and multiplies its own tokens
        aw = orc.calibrate_absmax(h16(d["weight"]))
        s, fold = orc.compute_scales(amax.numpy(), aw, w.alpha)
        wq, ws = orc.smooth_quantize_weight(h16(d["weight"]), s)
        t0, t1 = sqdist.shard_range(w.T, world, rank)
        xq, xs = orc.rmsnorm_smooth_quant(h16(d["x"][t0:t1]), fold, apply_norm=False)
        y, _ = orc.w8a8_linear(xq, xs, wq, ws, h16(d["bias"]))
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_calibration_and_token_sharding(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle as orc
    w = synth.WORKLOADS[0]
    d = synth.group_inputs(w, 0, "cpu")
    calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], "cpu")))
    amax = orc.calibrate_absmax(h16(calib[: calib.shape[0] - 37]))
    aw = orc.calibrate_absmax(h16(d["weight"]))
    s, fold = orc.compute_scales(amax, aw, w.alpha)
    wq, ws = orc.smooth_quantize_weight(h16(d["weight"]), s)
    xq, xs = orc.rmsnorm_smooth_quant(h16(d["x"]), fold, apply_norm=False)
    y, _ = orc.w8a8_linear(xq, xs, wq, ws, h16(d["bias"]))
    parts = [np.load(tmp_path / f"y{r}.npy") for r in range(world)]
    assert np.array_equal(np.concatenate(parts), y)


def test_shard_range_covers_exactly():
    for total in (0, 1, 7, 64, 1001):
        for world in (1, 2, 3, 8):
            got = [sqdist.shard_range(total, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sqdist.shard_range(10, 2, 2)


def test_allreduce_is_noop_without_group():
    t = torch.tensor([1.0, 2.0])
    assert sqdist.allreduce_max_(t) is t and t.tolist() == [1.0, 2.0]
