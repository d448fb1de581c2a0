"""The N > 1 benchmark path on CPU: two gloo ranks, each with its own batch.

The data path shards by batch (every rank runs the whole layer stack on its
own packed batch; no collective touches activations), so what there is to
test across ranks is the host logic: the slowest rank's step time decides
the whole-job throughput, each rank draws a distinct batch of the same
shape, and the reference arm runs on rank 0 alone.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 1.0 + 0.5 * rank  # the last rank is the slowest
        ms_max = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.job_value(6823, 8, world, ms_max)
        case = bench.make_workload("layer", rank)
        res = {"rank": rank, "ms_max": ms_max, "value": value, "T": case.total_tokens,
               "x_sum": float(np.asarray(case.x, np.float64).sum()),
               "cu": [int(v) for v in case.cu_seqlens]}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    slowest = 1.0 + 0.5 * (world - 1)
    for r in res:
        assert r["ms_max"] == pytest.approx(slowest)
        # whole-job tokens x layers over the slowest rank's time
        assert r["value"] == pytest.approx(6823 * 8 * world / (slowest / 1e3))
        assert r["T"] == 6823
    # same packing (weak scaling: per-rank work fixed), different data
    assert res[0]["cu"] == res[1]["cu"]
    assert res[0]["x_sum"] != res[1]["x_sum"]


def test_single_rank_helpers_need_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_value(1000, 8, 1, 2.0) == pytest.approx(4e6)


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    class Args:
        workload, steps, warmup, gpus = "layer", 1, 0, 2
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "time_oracle_layers", lambda *a, **k: called.append(1) or (1.0, 1))
    assert bench.run_reference(Args) == 0
    assert called == [] and capsys.readouterr().out == ""


def test_masked_leg_pair_count_matches_the_oracle_mask():
    from oracle import ptl_oracle as O
    lengths = [0, 1, 7, 40, 129, 300]
    ctx, tgt = bench.masked_counts(lengths)
    want = sum(int(O.hstu_user_mask(L, bench.MASKED_LEG["causal"], C, N, bench.MASKED_LEG["group"],
                                    bench.MASKED_LEG["window"]).sum())
               for L, C, N in zip(lengths, ctx, tgt) if L > 0)
    assert bench.visible_pairs(lengths, ctx, tgt) == want
    assert (ctx + tgt <= np.asarray(lengths)).all()
    # with no contexts or candidates the count is the causal one
    zero = np.zeros(len(lengths), np.int32)
    assert bench.visible_pairs(lengths, zero, zero) == sum(L * (L + 1) // 2 for L in lengths)
