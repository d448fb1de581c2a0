"""The N > 1 benchmark path on CPU: two gloo ranks splitting one batch.

Users are independent, so the job's batch (N copies of the packing, one set
of weights) is split into contiguous user ranges balanced by cost
(ptl_partition_users); each rank runs the stack on its range with rebased
offsets and the head probabilities are all-gathered at the end.  Here the
oracle stands in for the GPU stack on a small batch, and the test checks that
the gathered result equals the whole batch run on one rank, that the slowest
rank's step time decides the whole-job throughput, and that the reference arm
runs on rank 0 alone.
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


def _small_job(world):
    from packed_sequence_transformer_b200 import synthetic as S
    base = S.make_case("split", lengths=[3, 40, 0, 7, 129, 12, 1, 20], seed=5, dtype="bf16",
                       num_layers=2, with_head=True)
    return S.replicate_batch(base, world, seed=50)


def _worker(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist
    from oracle import ptl_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 1.0 + 0.5 * rank  # the last rank is the slowest
        ms_max = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.job_value(6823, 8, world, ms_max)
        # one batch split by users: this rank's part through the oracle stack
        job = _small_job(world)
        t0, t1, cu = bench.rank_part(job, world, rank)
        h, probs = O.stack_forward(job.x[t0:t1], cu, job.layers, head=job.head,
                                   pred_mask=job.pred_mask[t0:t1])
        cap = int(bench.max_over_ranks(t1 - t0, world, "cpu"))
        loc = torch.zeros(cap, dtype=torch.float64)
        loc[:probs.size] = torch.from_numpy(probs)
        buf, cnt = bench.gather_parts(loc, torch.tensor([probs.size], dtype=torch.int64), world, cap)
        rows = torch.zeros(cap * 512, dtype=torch.float64)
        rows[:h.size] = torch.from_numpy(h.reshape(-1))
        rbuf, rcnt = bench.gather_parts(rows, torch.tensor([h.size], dtype=torch.int64), world, cap * 512)
        res = {"rank": rank, "ms_max": ms_max, "value": value, "tokens": [t0, t1],
               "probs": bench.concat_parts(buf, cnt, cap).tolist(),
               "rows_sum": float(bench.concat_parts(rbuf, rcnt, cap * 512).sum()),
               "rows_n": int(bench.concat_parts(rbuf, rcnt, cap * 512).size)}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_batch_and_gather(tmp_path):
    from oracle import ptl_oracle as O
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    slowest = 1.0 + 0.5 * (world - 1)
    job = _small_job(world)
    h_all, p_all = O.stack_forward(job.x, job.cu_seqlens, job.layers, head=job.head,
                                   pred_mask=job.pred_mask)
    for r in res:
        assert r["ms_max"] == pytest.approx(slowest)
        # whole-job tokens x layers over the slowest rank's time
        assert r["value"] == pytest.approx(6823 * 8 * world / (slowest / 1e3))
        # every rank gathers the whole batch's result, in token order
        np.testing.assert_allclose(r["probs"], p_all, rtol=0, atol=1e-12)
        assert r["rows_n"] == h_all.size
        assert r["rows_sum"] == pytest.approx(float(h_all.sum()), abs=1e-9)
    # the parts are contiguous, disjoint and cover the batch
    assert res[0]["tokens"][0] == 0 and res[0]["tokens"][1] == res[1]["tokens"][0]
    assert res[1]["tokens"][1] == job.total_tokens


def test_job_batch_copies_share_weights_not_data():
    one = bench.make_workload("layer", 1)
    two = bench.make_workload("layer", 2)
    T = one.total_tokens
    assert two.total_tokens == 2 * T and two.num_users == 2 * one.num_users
    np.testing.assert_array_equal(two.x[:T], one.x)
    assert not np.array_equal(two.x[T:], one.x)
    for a, b in zip(two.layers, one.layers):
        for k in a:
            np.testing.assert_array_equal(a[k], b[k])
    # the cost-balanced split gives each rank one copy of the packing
    for rank in range(2):
        t0, t1, cu = bench.rank_part(two, 2, rank)
        assert (t0, t1) == (rank * T, (rank + 1) * T)
        np.testing.assert_array_equal(cu, one.cu_seqlens)


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
