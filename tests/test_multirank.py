"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2): each
rank decodes its own batch (weak scaling, distinct seeds, no collective on the data
path), and the reported time is the max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    from long_context_decode_02_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sh = bench.rank_shape(synth.CONFIGS[2], rank)
        q1 = synth.queries(sh.replace(batch=1, n_tokens=64), 0, 0)
        mx = bench.max_over_ranks(1.5 + rank)
        bench.barrier()
        q.put((rank, sh.seed, float(q1.float().sum()), mx))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = [r[1] for r in res]
    assert len(set(seeds)) == world                  # independent batches per rank
    assert res[0][2] != res[1][2]                    # different synthetic queries
    assert all(r[3] == 1.5 + (world - 1) for r in res)  # max over ranks on every rank


def test_bench_byte_model_matches_hand_count():
    import bench
    from long_context_decode_02_b200 import synth
    sh = synth.CONFIGS[2]
    # landmarks dominate kernel (a): 8 x 8 x 16384 chunks x 128 dims x 2 bytes
    assert bench.select_bytes(sh) == 8 * 8 * 16384 * 128 * 2 + 8 * 32 * 128 * 2 + 8 * 8 * 256 * 4
    coef = 8 * 8 * 256 * 8 * 160 * 2
    assert bench.attend_bytes(sh, 0) > coef
    assert bench.attend_tensor_flops(sh) == 8 * 8 * 2048 * (2 * 128 * 160 + 2 * 128 * 256)


def test_binding_refuses_strided_tensors():
    import torch
    from long_context_decode_02_b200 import build
    build.build()
    from long_context_decode_02_b200 import lowram as L
    t = torch.zeros(4, 8).t()
    with pytest.raises(ValueError):
        L._ptr(t)
