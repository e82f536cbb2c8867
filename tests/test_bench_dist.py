"""Host logic of bench.py's multi-rank path, on CPU with the gloo backend (world size 2):
every rank reports its own elapsed time and processed units; the job time is the maximum
over ranks and the units are summed (weak scaling, no data-path collective)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, local, dist = bench.dist_init()
    assert (r, w) == (rank, world)
    ms, units = bench.aggregate(10.0 + 5.0 * rank, 100.0 * (rank + 1), dist, None)
    bench.barrier(dist, None)
    out[rank] = (ms, units)
    dist.destroy_process_group()


def test_aggregate_max_time_sum_units_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as manager:
        out = manager.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        for r in range(world):
            assert out[r] == (15.0, 300.0)


def test_single_rank_aggregate_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(3.5, 7.0) == (3.5, 7.0)


def test_reference_arm_line_shape():
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse_args(["--impl", "reference", "--steps", "2", "--warmup", "1"])
    line = bench.run_reference(args, 0, 1)
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert bench.run_reference(args, 1, 2) is None


def test_secondary_failure_is_recorded_not_raised():
    sys.path.insert(0, ROOT)
    import bench
    line = {"value": 1.0}
    bench.secondary(line, "ok", lambda: {"x": 1})
    bench.secondary(line, "merged", lambda: {"derive_pack": {"y": 2}}, merge=True)

    def boom():
        raise RuntimeError("out of memory")
    bench.secondary(line, "bad", boom)
    assert line["ok"] == {"x": 1} and line["derive_pack"] == {"y": 2} and "merged" not in line
    assert line["bad"] == {"error": "RuntimeError: out of memory"}
