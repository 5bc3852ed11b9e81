"""Multi-rank host logic on CPU (gloo, world size 2): the max-over-ranks time
reduction, per-rank seeds, batch partitioning, and that splitting the batch
across ranks leaves every (batch, head) problem's result unchanged (the
sharding has no data-path collective because the problems are independent)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_delta_rule_128_b200 import dist as gd

NAMES = ("q", "k", "v", "g", "b", "w", "S0")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle
    from gated_delta_rule_128_b200 import workloads
    info = gd.rank_info()
    gd.init("gloo", info, timeout_s=60)
    try:
        # max over ranks
        m = gd.max_over_ranks([float(rank + 1), float(10 - rank)])
        # each rank computes its share of one batch with the oracle
        x = workloads.draw(4, 40, 2, 8, 8, 123, s0_std=0.1, with_dO=False)
        rows = gd.batch_rows(4, info.world, info.rank)
        sl = slice(rows.start, rows.stop)
        r = {n: x[n][sl].double().numpy() for n in NAMES}
        o, ST = oracle.forward(*(r[n] for n in NAMES), nthreads=1)
        gd.barrier()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), o=o, ST=ST, m=np.array(m),
                 seed=gd.rank_seed(1002, rank), start=rows.start, stop=rows.stop)
    finally:
        gd.shutdown()


def test_two_rank_gloo(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    for r in res:
        np.testing.assert_array_equal(r["m"], [2.0, 10.0])
    assert res[0]["seed"] == 1002 and res[1]["seed"] != res[0]["seed"]
    assert (res[0]["start"], res[0]["stop"], res[1]["start"], res[1]["stop"]) == (0, 2, 2, 4)
    # sharded results equal the unsharded batch
    import oracle
    from gated_delta_rule_128_b200 import workloads
    x = workloads.draw(4, 40, 2, 8, 8, 123, s0_std=0.1, with_dO=False)
    o, ST = oracle.forward(*(x[n].double().numpy() for n in NAMES))
    np.testing.assert_array_equal(np.concatenate([r["o"] for r in res]), o)
    np.testing.assert_array_equal(np.concatenate([r["ST"] for r in res]), ST)


@pytest.mark.parametrize("total,world", [(4, 2), (5, 2), (3, 4), (16, 8)])
def test_batch_rows_partition(total, world):
    parts = [gd.batch_rows(total, world, r) for r in range(world)]
    covered = [i for p in parts for i in p]
    assert covered == list(range(total))
    sizes = [len(p) for p in parts]
    assert max(sizes) - min(sizes) <= 1


def test_single_rank_is_identity():
    assert gd.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    gd.barrier()
