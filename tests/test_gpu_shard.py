"""Row sharding (bit_gemv_rabit_b200.shard) with the library's real kernels on the GPU.

One GPU cannot hold two NCCL ranks, so the ranks' row blocks run one after another in this
process (derive and GEMV of each block with the CUDA kernels, the blocks assembled as the
all-gather would), and a one-rank NCCL group runs the whole path, collective included.
Every output row is checked against the float64 oracle.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit
from bit_gemv_rabit_b200 import shard

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from bit_gemv_rabit_b200 import build
    build.build()
    oracle.build()
    rabit.load()
    rabit.rabit_read_fault(clear=True)
    yield
    assert rabit.rabit_read_fault(clear=True) == 0


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("N,K,B,world,use_derive", [(4096, 4096, 1, 2, True), (1000, 2048, 5, 3, True),
                                                    (4099, 1024, 3, 4, False)])
def test_row_blocks_with_real_kernels(N, K, B, world, use_derive):
    W = inputs.weight(31 + N, N, K)
    a, b = inputs.scales(31 + N, W)
    x = inputs.activations(32 + K, B, K)
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    Wt = torch.from_numpy(W).cuda()
    full = None
    if not use_derive:
        full = rabit.alloc_packed(N, K)
        rabit.rabit_derive_pack(Wt, at, bt, full)
    y = np.full((B, N), np.nan, np.float32)
    for r in range(world):
        s = shard.RowShard(N, K, 2, r, world)
        if use_derive:
            s.derive(Wt[s.begin:s.end], at, bt)
        else:
            s.attach(full, at, bt)
        y[:, s.begin:s.end] = s.local(bf16_dev(x)).cpu().numpy()[:, :s.rows]
    torch.cuda.synchronize()
    ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x)
    assert not np.isnan(y).any()
    assert normwise(y.astype(np.float64), ref) <= 2e-3


def test_one_rank_nccl_group_runs_the_whole_path():
    import torch.distributed as dist
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        N, K, B = 3000, 1536, 4
        W = inputs.weight(41, N, K)
        a, b = inputs.scales(41, W)
        x = inputs.activations(42, B, K)
        s = shard.RowShard(N, K, 2, 0, 1)
        s.derive(torch.from_numpy(W).cuda(), torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
        y = torch.full((B, N), float("nan"), device="cuda")
        s.gemv(bf16_dev(x), y)
        torch.cuda.synchronize()
        ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x)
        assert normwise(y.cpu().numpy().astype(np.float64), ref) <= 2e-3
    finally:
        dist.destroy_process_group()
