"""Host logic of the multi-GPU bench on CPU: two gloo ranks, each with its own
step time, agree on the max over ranks and on the whole-job throughput."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    my_ms = 1.0 + rank            # rank 1 is the slow one
    t = bench.reduce_max(my_ms)
    gbps, tmax = bench.aggregate([t] * world, bench.step_bytes(bench.HEADLINE, 1))
    bench.barrier()
    dist.destroy_process_group()
    q.put((rank, t, gbps, tmax))


def test_two_gloo_ranks_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    import bench
    b = bench.step_bytes(bench.HEADLINE, 1)
    for rank, t, gbps, tmax in res:
        assert t == 2.0 and tmax == 2.0
        assert gbps == pytest.approx(2 * b / 2e-3 / 1e9)


def test_step_bytes_headline():
    sys.path.insert(0, ROOT)
    import bench
    # 32 layers of q, k, v, o 4096->4096, gate, up 4096->11008, down 11008->4096:
    # 4-bit codes + fp16 scale/zero per 128 inputs + x + y
    exp = 0
    for N, K in [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]:
        exp += N * K * 4 // 8 + N * (K // 128) * 4 + K * 2 + N * 2
    assert bench.step_bytes(bench.HEADLINE, 1) == 32 * exp
    assert abs(32 * exp / 1e9 - 3.44) < 0.01
