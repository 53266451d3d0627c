"""Host-side multi-rank logic of the bench, run as world-size-2 gloo ranks on CPU."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_time = 1.0 + 0.5 * rank                  # rank 1 is the slow one
        slowest = bench.max_over_ranks(local_time, world, torch.device("cpu"))
        # each rank works on its own data
        g = torch.Generator().manual_seed(bench.rank_seed(rank))
        first = float(torch.randn(1, generator=g))
        gathered = [None] * world
        dist.all_gather_object(gathered, first)
        out_q.put((rank, slowest, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_data():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, gathered in res:
        assert slowest == 1.5                          # max over ranks, on every rank
        assert gathered[0] != gathered[1]              # distinct pools per rank


def test_reference_arm_other_ranks_exit_silently(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert rc == 0 and buf.getvalue() == ""


def test_reference_arm_rank0_prints_one_json_line(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert rc == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def _dp_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_circulant_layers_b200.dp import GradCBucket, shard_tokens
        import numpy as np
        import oracle
        from synthetic import normal
        # a layer's grad_c over 10 tokens equals the sum of the ranks' grad_c over their shards
        q, p, B = 2, 8, 10
        x = normal(70, (B, q * p))
        g = normal(71, (B, q * p))
        c = normal(72, (q, q, p))
        sl = shard_tokens(B, rank, world)
        _, gc_local = oracle.circ_backward(g[sl], x[sl], c)
        shapes = [torch.Size([q, q, p]), torch.Size([3, 5])]
        bucket = GradCBucket(shapes, device="cpu", dtype=torch.float64)
        bucket.views[0].copy_(torch.from_numpy(gc_local))
        bucket.views[1].fill_(rank + 1.0)
        views = bucket.allreduce()
        _, gc_full = oracle.circ_backward(g, x, c)
        out_q.put((rank, float(np.abs(views[0].numpy() - gc_full).max()), float(views[1][0, 0]),
                   (sl.start, sl.stop)))
    finally:
        dist.destroy_process_group()


def test_data_parallel_grad_c_allreduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, err0, s0, sl0), (r1, err1, s1, sl1) = res
    assert err0 < 1e-12 and err1 < 1e-12         # summed shards equal the full-batch grad_c
    assert s0 == s1 == 3.0                        # 1 + 2
    assert sl0 == (0, 5) and sl1 == (5, 10)


def test_shard_tokens_covers_everything():
    from block_circulant_layers_b200.dp import shard_tokens
    for total in (0, 1, 7, 4096):
        for world in (1, 2, 3, 8):
            covered = []
            for r in range(world):
                s = shard_tokens(total, r, world)
                covered.extend(range(s.start, s.stop))
            assert covered == list(range(total))
