"""N-split (column-parallel) quantised linear: the host logic of the row
shards and of the y all-gather, on CPU ranks over gloo, against the oracle's
single-rank product.  Each rank computes its shard with the oracle (the
local-product hook of NSplitLinear), so the gathered y must equal the
single-rank oracle result bit for bit."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case(N, K, bits, group, M, sym, seed=50):
    import oracle
    import wq_inputs
    Wb = wq_inputs.f16_bits(wq_inputs.weight_f16(seed, bits, N, K, dist="t4"))
    if sym:
        q, s = oracle.quantize_rtn_sym(Wb, bits, group)
        z = None
    else:
        q, s, z = oracle.quantize_rtn(Wb, bits, group)
    words = oracle.pack(q, bits)
    x = wq_inputs.activations_bf16(seed, 1, M, K)
    return words, s, z, x


def _oracle_y(x, words, s, z, N, K, bits, group):
    import oracle
    import wq_inputs
    zz = z if z is not None else oracle.sym_zeros(s, bits)
    y, _ = oracle.gemm(wq_inputs.bf16_bits(x), words, s, zz, N, K, bits, group)
    return torch.from_numpy(y).to(torch.bfloat16)


def _oracle_local(K, bits, group):
    def run(x, codes, scales, zeros, n_rows, out):
        w = codes.numpy().view(np.uint32)
        s = scales.numpy().view(np.uint16)
        z = None if zeros is None else zeros.numpy().view(np.uint16)
        out.copy_(_oracle_y(x, w, s, z, n_rows, K, bits, group))
        return out
    return run


def _rank(rank, world, port, cases, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    from quantized_gemm_wq_b200.nsplit import NSplitLinear
    dist.init_process_group("gloo", rank=rank, world_size=world)
    out = []
    for (N, K, bits, group, M, sym) in cases:
        words, s, z, x = _case(N, K, bits, group, M, sym)
        lin = NSplitLinear(torch.from_numpy(words.view(np.int32)), torch.from_numpy(s.view(np.int16)),
                           None if z is None else torch.from_numpy(z.view(np.int16)), N, K, bits, group,
                           local=_oracle_local(K, bits, group))
        y = lin(x)
        ref = _oracle_y(x, words, s, z, N, K, bits, group)
        out.append((lin.n0, lin.n1, bool(torch.equal(y, ref)), tuple(y.shape)))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, out))


CASES = [(70, 256, 4, 128, 1, False), (70, 256, 3, 64, 3, False), (130, 128, 2, 0, 2, True),
         (33, 512, 8, 128, 1, True), (256, 384, 4, 128, 5, False)]


@pytest.mark.parametrize("world", [2, 3])
def test_nsplit_gloo_ranks_match_single_rank_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, world, port, CASES, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=300) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for ci, (N, K, bits, group, M, sym) in enumerate(CASES):
        covered = []
        for r in range(world):
            n0, n1, equal, shape = res[r][ci]
            assert equal, (world, r, CASES[ci])
            assert shape == (M, N)
            covered.append((n0, n1))
        # the shards tile [0, N) in order, 32-row aligned
        assert covered[0][0] == 0 and covered[-1][1] == N
        for (a0, a1), (b0, b1) in zip(covered, covered[1:]):
            assert a1 == b0 and a0 % 32 == 0


def test_shard_bounds():
    sys.path.insert(0, ROOT)
    from quantized_gemm_wq_b200.nsplit import shard_bounds
    assert shard_bounds(4096, 2, 0) == (0, 2048, 2048)
    assert shard_bounds(4096, 2, 1) == (2048, 4096, 2048)
    assert shard_bounds(70, 2, 1) == (64, 70, 64)
    assert shard_bounds(33, 4, 3) == (33, 33, 32)        # a rank with no rows
    for N in (1, 31, 32, 100, 49152):
        for world in (1, 2, 3, 8):
            b = [shard_bounds(N, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == N
            assert all(x[1] == y[0] for x, y in zip(b, b[1:]))
    with pytest.raises(ValueError):
        shard_bounds(10, 2, 2)
