"""Column-parallel sharding of the layer, host side, on CPU: the column
blocks cover the output exactly once in multiples of 16, and two gloo ranks
that each compute their block (here with the oracle, since this box has no
GPU) and all-gather them reproduce the unsharded output bit for bit. Each
output column of the method depends only on X and that column of W
("The Full LLM.int8() Algorithm", Steps 1-5: the outlier set, row scales and
codes come from X alone; the column scale and codes from that column), which
is what makes the blocks exact.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("o,world", [(4096, 8), (49152, 8), (784, 3), (272, 4),
                                     (16, 4), (20480, 6)])
def test_shard_columns_cover_the_output_once(o, world):
    from mixed_precision_int8_b200.column_parallel import shard_columns, shard_width
    per = shard_width(o, world)
    assert per % 16 == 0 and per * world >= o
    seen = np.zeros(o, dtype=np.int64)
    for r in range(world):
        c0, w = shard_columns(o, world, r)
        assert c0 % 16 == 0 and w % 16 == 0 and 0 <= w <= per
        seen[c0:c0 + w] += 1
    assert (seen == 1).all()
    with pytest.raises(ValueError):
        shard_columns(o, world, world)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import oracle
    from mixed_precision_int8_b200 import workloads
    from mixed_precision_int8_b200.column_parallel import gather_columns, shard_columns
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(7)  # same inputs on every rank
        s, h, o = 24, 256, 784
        X = workloads.random_x(rng, s, h, outlier_cols=(3, 100, 255))
        W = workloads.random_w(rng, h, o)
        c0, w = shard_columns(o, world, rank)
        Wq, aw = oracle.prepare_weight(np.ascontiguousarray(W[:, c0:c0 + w]))
        block = oracle.matmul(X, Wq, aw, 6.0)
        full = gather_columns(torch.from_numpy(block), o, world)
        q.put((rank, full.numpy().view(np.uint16).tobytes()))
    finally:
        dist.destroy_process_group()


def test_gloo_ranks_gather_the_unsharded_output_bit_for_bit():
    sys.path.insert(0, ROOT)
    import oracle
    from mixed_precision_int8_b200 import workloads
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    import queue
    import time
    got, t0 = {}, time.time()
    while len(got) < 2 and time.time() - t0 < 180:
        try:
            r, b = q.get(timeout=2)
            got[r] = b
        except queue.Empty:
            assert all(p.is_alive() or p.exitcode == 0 for p in procs), "a rank failed"
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    rng = np.random.default_rng(7)
    X = workloads.random_x(rng, 24, 256, outlier_cols=(3, 100, 255))
    W = workloads.random_w(rng, 256, 784)
    Wq, aw = oracle.prepare_weight(W)
    ref = oracle.matmul(X, Wq, aw, 6.0).view(np.uint16)
    for r in range(2):
        assert np.frombuffer(got[r], dtype=np.uint16).reshape(24, 784).tolist() == ref.tolist()
