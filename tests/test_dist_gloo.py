"""Multi-rank host logic on CPU: two gloo ranks shard the activation rows, reduce their
shards to column sums, gather them in rank order and finish h -- which must equal h over
all rows. The column sums and the finalize here are CPU stand-ins (the oracle's column
sums and a float64 numpy combine); on GPUs they are mxq_act_sqsum and
mxq_act_sqmean_finalize."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from block_scaled_weight_b200.dist import shard_rows


def test_shard_rows_partitions_every_row():
    for total in (0, 1, 2, 7, 244449):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, rows, cols, q):
    import datetime

    import torch.distributed as dist

    from block_scaled_weight_b200 import synth
    from block_scaled_weight_b200.dist import distributed_h, shard_rows
    from oracle import oracle as orc
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        X = synth.activations(rows, cols, 11, dtype=torch.bfloat16)
        r0, r1 = shard_rows(rows, world, rank)
        X_local = X[r0:r1]

        def colsum(x):
            if x.shape[0] == 0:
                return torch.zeros(cols, dtype=torch.float64)
            return torch.from_numpy(orc.act_sqsum(x.contiguous().view(torch.int16).numpy()
                                                  .view(np.uint16)))

        def finalize(parts, total):
            acc = np.zeros(cols, np.float64)
            for p in parts.numpy():          # ascending rank order
                acc += p
            return torch.from_numpy((acc / total).astype(np.float32))

        h = distributed_h(X_local, colsum, finalize, group=None)
        q.put((rank, h.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rows,cols", [(1000, 264), (3, 16), (1, 8)])
def test_two_rank_h_equals_single_process_h(rows, cols, orc):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rows, cols, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from block_scaled_weight_b200 import synth
    X = synth.activations(rows, cols, 11, dtype=torch.bfloat16)
    ref = orc.act_sqmean(X.view(torch.int16).numpy().view(np.uint16))
    for r in range(world):
        np.testing.assert_allclose(got[r], ref, rtol=1e-12)
    assert np.array_equal(got[0], got[1])
