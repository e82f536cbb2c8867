"""Host logic of the row-sharded layer (bit_gemv_rabit_b200/shard.py) on CPU with gloo.

The ranks' kernels are replaced by the float64 oracle on the same rows (these tests check
the plumbing: row blocks, the contiguous slice of the packed layout, the scales' columns,
ranks without rows, and the all-gather back into [batch][N]); the kernels themselves are
checked against the oracle by the GPU parity tests.  The sharded result must equal the
oracle on the whole matrix bit for bit, since every output row is computed by the same
arithmetic either way.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_gemv_rabit_b200 import shard  # noqa: E402


@pytest.mark.parametrize("N,world", [(1, 1), (7, 2), (8, 3), (4096, 3), (2, 5), (11008, 8)])
def test_row_blocks_partition_the_rows(N, world):
    blocks = [shard.row_block(N, world, r) for r in range(world)]
    assert blocks[0][0] == 0 and blocks[-1][1] == N
    for (b0, e0), (b1, e1) in zip(blocks, blocks[1:]):
        assert e0 == b1
    sizes = [e - b for b, e in blocks]
    assert max(sizes) - min(sizes) <= 1 and max(sizes) == -(-N // world)
    with pytest.raises(ValueError):
        shard.row_block(N, world, world)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, N, K, B, use_derive, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import oracle
    from bit_gemv_rabit_b200 import inputs, rabit, shard as sh

    def fake_gemv(packed, a, b, N_, K_, x, y, P=2, stream=None):
        S = oracle.unpack(packed.numpy(), N_, K_, P=P)
        y.copy_(torch.from_numpy(oracle.layer(S, a.numpy(), b.numpy(), x.numpy()).astype(np.float32)))
        return y

    def fake_derive(W, a, b, packed, P=2, stream=None):
        S = oracle.derive_signs(W.numpy(), a.numpy(), b.numpy(), P=P)
        packed.copy_(torch.from_numpy(oracle.pack(S)))
        return packed

    rabit.rabit_gemv = fake_gemv
    rabit.rabit_read_fault = lambda clear=True, stream=None: 0   # no device here
    rabit.rabit_derive_pack = fake_derive
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        W = inputs.weight(5, N, K)
        a, b = inputs.scales(5, W)
        x = inputs.activations(5, B, K, dtype="f32")
        cpu = torch.device("cpu")
        s = sh.RowShard(N, K, 2, rank, world, device=cpu)
        if use_derive:
            s.derive(torch.from_numpy(W[s.begin:s.end]), torch.from_numpy(a), torch.from_numpy(b))
        else:
            S = oracle.derive_signs(W, a, b)
            s.attach(torch.from_numpy(oracle.pack(S)), torch.from_numpy(a), torch.from_numpy(b))
        y = torch.full((B, N), float("nan"))
        s.gemv(torch.from_numpy(x), y)
        ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x).astype(np.float32)
        out[rank] = bool(np.array_equal(y.numpy(), ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N,K,B,world,use_derive", [(70, 300, 3, 2, False), (70, 300, 1, 2, True),
                                                    (2, 129, 2, 3, True)])
def test_sharded_gemv_equals_whole_layer(N, K, B, world, use_derive):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as manager:
        out = manager.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, N, K, B, use_derive, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0] * world, codes
        assert dict(out) == {r: True for r in range(world)}
