"""The multi-GPU host path on CPU: two gloo ranks (127.0.0.1) run the process-group plumbing of
gated_delta_rule_looped_b200.dist (barrier, max over ranks, the split of units, the whole-job
rate) and show that splitting a workload's (loop, batch, head) units between ranks gives the
same result as the whole workload on one process: the units are independent recurrences, so
the data path needs no collective.  The per-unit arithmetic here is the fp64 oracle."""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_delta_rule_looped_b200 import dist as gdist
from gated_delta_rule_looped_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _tiny_case():
    w = inputs.workload("tiny_fp32", T=2, B=2, H=3, L=20, d=8, s0="normal")
    x = inputs.make_inputs(w, seed=13, device="cpu")
    units = w.T * w.B * w.H
    flat = {n: x[n].reshape((units,) + tuple(x[n].shape[3:])).double().numpy()
            for n in ("q", "k", "v", "alpha", "beta", "S0")}
    return flat, units


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    got_world, got_rank, _ = gdist.init("gloo", timeout_s=60)
    res = {"world": got_world, "rank": got_rank}
    res["max"] = gdist.max_over_ranks(rank + 0.25, world)
    gdist.barrier(world)
    res["shares"] = {n: list(gdist.split_units(n, world, rank)) for n in (0, 1, 2, 5, 12, 13)}
    # this rank's share of the tiny workload, through the oracle
    import oracle
    flat, units = _tiny_case()
    a, b = gdist.split_units(units, world, rank)
    o, S = oracle.prefill_sequential(*(flat[n][a:b] for n in ("q", "k", "v", "alpha", "beta")),
                                     S0=flat["S0"][a:b], per_key=False)
    np.save(os.path.join(outdir, f"o{rank}.npy"), o)
    np.save(os.path.join(outdir, f"S{rank}.npy"), S)
    with open(os.path.join(outdir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    torch.distributed.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    outdir = str(tmp_path_factory.mktemp("gloo"))
    mp.start_processes(_worker, args=(2, _free_port(), outdir), nprocs=2, start_method="spawn", join=True)
    res = []
    for r in range(2):
        with open(os.path.join(outdir, f"r{r}.json")) as f:
            res.append(json.load(f))
    return outdir, res


def test_ranks_join_and_agree_on_the_slowest(two_ranks):
    _, res = two_ranks
    assert [r["rank"] for r in res] == [0, 1]
    assert all(r["world"] == 2 for r in res)
    assert all(r["max"] == 1.25 for r in res)


def test_unit_shares_cover_every_unit_once(two_ranks):
    _, res = two_ranks
    for n in ("0", "1", "2", "5", "12", "13"):
        covered = []
        for r in res:
            a, b = r["shares"][n]
            covered.extend(range(a, b))
        assert covered == list(range(int(n)))


def test_split_units_local():
    for n in range(0, 40):
        for world in (1, 2, 3, 8):
            shares = [gdist.split_units(n, world, r) for r in range(world)]
            assert [u for a, b in shares for u in range(a, b)] == list(range(n))
            sizes = [b - a for a, b in shares]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        gdist.split_units(4, 2, 2)


def test_sharded_units_equal_the_whole_workload(two_ranks):
    import oracle
    outdir, _ = two_ranks
    flat, units = _tiny_case()
    o_all, S_all = oracle.prefill_sequential(*(flat[n] for n in ("q", "k", "v", "alpha", "beta")),
                                             S0=flat["S0"], per_key=False)
    o = np.concatenate([np.load(os.path.join(outdir, f"o{r}.npy")) for r in range(2)])
    S = np.concatenate([np.load(os.path.join(outdir, f"S{r}.npy")) for r in range(2)])
    assert np.array_equal(o, o_all) and np.array_equal(S, S_all)


def test_whole_job_rate():
    assert gdist.whole_job_rate(1000, 4, 2.0) == pytest.approx(2e6)
    assert gdist.whole_job_rate(1000, 1, 1.0) == pytest.approx(1e6)
    with pytest.raises(ValueError):
        gdist.whole_job_rate(1, 1, 0.0)
    assert gdist.env_ranks() == (1, 0, 0) or "WORLD_SIZE" in os.environ
