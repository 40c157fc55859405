"""The bench's multi-rank plumbing on CPU: two ranks on the gloo backend
(one process each, as torchrun launches them).  Each rank reads its rank from
the environment, draws its own batch, and the timed duration every rank
reports is the maximum over ranks."""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from selective_state_space_14_b200 import workloads as W
    w, r, local = bench.dist_init(world, backend="gloo")
    p = W.make("m1_f32_b1_d64_n16_l256", shard=r)
    bench.barrier(w)
    ms = bench.max_over_ranks(w, 10.0 + r, device="cpu")
    # the first u value identifies the rank's batch
    out.put((r, w, local, ms, float(p.u.data.ravel()[0])))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == world and r[2] == r[0] for r in res)
    assert all(r[3] == 11.0 for r in res)  # max over ranks, seen by every rank
    assert res[0][4] != res[1][4]  # each rank draws its own batch


def test_world_size_must_match_gpus(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.dist_init(2)


def test_shards_share_shape_and_distribution():
    from selective_state_space_14_b200 import workloads as W
    a, b = W.make("m1_f32_b1_d64_n16_l256"), W.make("m1_f32_b1_d64_n16_l256", shard=1)
    assert a.u.data.shape == b.u.data.shape
    assert not np.array_equal(a.u.data, b.u.data)
    np.testing.assert_array_equal(a.A, b.A)  # A = -(n+1) is not drawn
