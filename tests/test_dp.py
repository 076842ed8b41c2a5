"""Data-parallel plumbing on CPU: two gloo ranks, as the benchmark runs one rank per GPU.

The path shards by (sequence, kv head) unit with no exchange step, so what two ranks compute on their own batches
must equal what one process computes on both batches; ranks meet only in the barrier and the max-reduction of the
elapsed time.  A rank that never joins turns into an error on the other rank within the group's timeout.
"""
import json
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))


def _shard_records(seed: int) -> list:
    """A rank's work on its own batch: one block of one (sequence, kv head) unit, quantised by the oracle."""
    import oracle
    from bit_kv_cache_token_b200 import synth
    k, _ = synth.layer_kv(seed, 0, 1, 1, 128, 64, n_outliers=2)
    rec = oracle.pack_record(oracle.quantize_block(k[0, 0].double().numpy(), 64, 4), oracle.K_ORDER)
    return rec.tolist()


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import sys
    sys.path.insert(0, ROOT)
    _env(rank, world, port)
    from bit_kv_cache_token_b200 import dp
    import torch.distributed as dist
    w, r, local = dp.world_from_env()
    dp.init(w, "gloo", timeout_s=30)
    seed = dp.rank_seed(2, r)
    rec = _shard_records(seed)
    dp.barrier(w)
    slowest = dp.max_over_ranks(1.5 + r, w)
    gathered = [None] * w
    dist.all_gather_object(gathered, seed)  # test-side check only: every rank drew a batch of its own
    rate = dp.aggregate_rate(1024, slowest, w)
    dp.finish(w)
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(dict(world=w, rank=r, local=local, seed=seed, rec=rec, slowest=slowest, seeds=gathered,
                       rate=rate), f)


def _lonely_rank(port: int, out_dir: str) -> None:
    import sys
    sys.path.insert(0, ROOT)
    _env(0, 2, port)
    from bit_kv_cache_token_b200 import dp
    try:
        dp.init(2, "gloo", timeout_s=3)
        msg = "joined"
    except Exception as e:  # the peer never arrives
        msg = "error: " + type(e).__name__
    with open(os.path.join(out_dir, "lonely.json"), "w") as f:
        json.dump(dict(result=msg), f)


def _run(procs, timeout):
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "rank did not finish"
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]


def test_two_gloo_ranks_shard_without_exchange(tmp_path):
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    port = _free_port()
    _run([ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)], 240)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, x in enumerate(res):
        assert (x["world"], x["rank"], x["local"]) == (2, r, r)
        assert x["slowest"] == 2.5  # max over ranks of 1.5 + rank
        assert x["seeds"] == [2, 1002]
        assert x["rate"] == pytest.approx(1024 * 2 / 2.5)
    assert res[0]["rec"] != res[1]["rec"]  # independent batches
    # one process doing both batches computes exactly what the two ranks computed
    from bit_kv_cache_token_b200 import dp
    for r in range(2):
        assert res[r]["rec"] == _shard_records(dp.rank_seed(2, r))


def test_single_process_world_needs_no_group(monkeypatch):
    from bit_kv_cache_token_b200 import dp
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert dp.world_from_env() == (1, 0, 0)
    dp.init(1)
    dp.barrier(1)
    assert dp.max_over_ranks(3.25, 1) == 3.25
    assert dp.aggregate_rate(100, 2.0, 1) == 50.0
    dp.finish(1)


def test_rank_that_never_joins_is_an_error(tmp_path):
    ctx = mp.get_context("spawn")
    port = _free_port()
    _run([ctx.Process(target=_lonely_rank, args=(port, str(tmp_path)))], 120)
    res = json.load(open(tmp_path / "lonely.json"))
    assert res["result"].startswith("error"), res


def test_rank_seeds_distinct():
    from bit_kv_cache_token_b200 import dp
    seeds = [dp.rank_seed(2, r) for r in range(8)]
    assert len(set(seeds)) == 8
    assert np.all(np.diff(seeds) > 0)
