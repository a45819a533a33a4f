"""The multi-rank path of bench.py on CPU: two gloo ranks.

With N GPUs every rank decodes its own independent batch of the same shape
(sequences are independent: no collective on the data path), and the only
collectives are the barrier around the timed region and the max over ranks
of the measured times.  These tests run those pieces as two processes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        args = bench.parse_args(["--gpus", str(world)])
        w, r, local = bench.dist_setup(args)
        assert (w, r, local) == (world, rank, rank)
        # each rank times something different; everyone must see the maximum
        bench.barrier(w)
        t_max = bench.max_over_ranks(10.0 + rank, w, "cpu")
        # each rank builds its own batch: same shape, different contents
        sc = bench.make_scenario("mha7b", seed=1 + rank, num_seqs=4, num_blocks=2048)
        st = sc.steps[0]
        # the extension workloads shard the same way: per-rank batches of one shape
        ext = []
        for name, kw in (("spec8b", dict(num_seqs=4, num_blocks=2048)), ("prefix8b", dict(num_seqs=16, num_blocks=1024)),
                         ("window70b", dict(num_seqs=1, num_blocks=4096))):
            e = bench.make_scenario(name, seed=1 + rank, **kw).steps[0]
            ext.append((name, e.q.shape, e.block_tables.shape, int(e.q.reshape(-1)[0])))
        fp8 = bench.make_scenario("gqa8b", seed=1 + rank, num_seqs=4, num_blocks=4096, kv="fp8")
        q.put((rank, t_max, st.q.shape, st.block_tables.shape, int(st.q[0, 0, 0]), st.context_lens.tolist(), ext,
               fp8.kv_dtype))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[1] for o in out] == [11.0, 11.0], "max over ranks"
    assert out[0][2] == out[1][2] and out[0][3] == out[1][3], "same batch shape on every rank"
    assert out[0][5] != out[1][5] or out[0][4] != out[1][4], "ranks must decode different batches"
    for (n0, qs0, bs0, v0), (n1, qs1, bs1, v1) in zip(out[0][6], out[1][6]):
        assert n0 == n1 and qs0 == qs1 and bs0 == bs1, f"{n0}: ranks differ in shape"
        assert v0 != v1, f"{n0}: ranks must decode different batches"
    assert out[0][7] == out[1][7] == "fp8"


def test_rank_count_mismatch_is_refused(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.dist_setup(bench.parse_args(["--gpus", "4"]))
