"""Row sharding over ranks and the path's one collective, on CPU: shards cover every query row
once, causal shards balance the work, and two gloo ranks that each compute the indexer loss
of their rows (with the oracle) sum to the single-process total."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle as ref
from sparse_attention_tcgen05_b200 import sharding


@pytest.mark.parametrize("n,world", [(0, 2), (1, 2), (7, 2), (32, 3), (1000, 8)])
def test_shard_rows_cover_each_row_once(n, world):
    spans = [sharding.shard_rows(n, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("Lq,Lk,k,world", [(8192, 8192, 2048, 2), (8192, 8192, 2048, 8), (300, 1000, 64, 3)])
def test_causal_shards_balance_the_work(Lq, Lk, k, world):
    cost = sharding.causal_row_cost(Lq, Lk, k)
    spans = [sharding.shard_causal_rows(Lq, Lk, k, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == Lq
    assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
    work = [cost[a:b].sum() for a, b in spans]
    # each cut lands within one row of its quantile
    assert max(work) <= cost.sum() / world + cost.max() + 1e-9
    # plain equal-row shards would give the last rank far more than its share
    plain = [cost[a:b].sum() for a, b in (sharding.shard_rows(Lq, r, world) for r in range(world))]
    if Lq == Lk:
        assert max(work) < max(plain)


def _loss_case(seed=11, rows=40, Lk=300, k=48):
    rng = np.random.default_rng(seed)
    scores = rng.normal(size=(rows, Lk)) * 2.0
    idx = np.stack([np.sort(rng.permutation(Lk)[:k]) for _ in range(rows)]).astype(np.int32)
    idx[3, 20:] = -1
    p = rng.dirichlet(np.ones(k), size=rows)
    p[3, 20:] = 0.0
    return scores, idx, p


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        scores, idx, p = _loss_case()
        a, b = sharding.shard_rows(scores.shape[0], rank, world)
        part = sum(ref.kl_row(scores[r], idx[r], p[r]) for r in range(a, b))
        loss = sharding.sum_over_ranks(torch.tensor([part], dtype=torch.float64))
        slowest = sharding.max_over_ranks(float(rank + 1))
        out[rank] = torch.tensor([loss.item(), slowest], dtype=torch.float64)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_sum_the_loss_and_agree_on_the_slowest_time():
    world = 2
    out = torch.zeros(world, 2, dtype=torch.float64).share_memory_()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    scores, idx, p = _loss_case()
    total = sum(ref.kl_row(scores[r], idx[r], p[r]) for r in range(scores.shape[0]))
    for r in range(world):
        assert abs(out[r, 0].item() - total) <= 1e-12 * abs(total)
        assert out[r, 1].item() == float(world)


def test_helpers_are_identity_on_one_process():
    x = torch.tensor([2.5])
    assert sharding.sum_over_ranks(x) is x and x.item() == 2.5
    assert sharding.max_over_ranks(3.0) == 3.0


@pytest.mark.parametrize("Lq,Lk,world", [(160, 160, 3), (120, 250, 2)])
def test_causal_shard_calls_reproduce_the_whole_sequence_rows(Lq, Lk, world):
    # a rank calls the path on its rows with Lq' = stop - start and Lk' = stop + (Lk - Lq) over the
    # key prefix [0, Lk'): each of its rows must get the whole sequence's scores, top-k set and
    # attention output (the oracle run both ways)
    import dsa_inputs
    H_I, d_I, k, H, d_qk, d_v = 2, 16, 24, 2, 40, 32
    seed = 0x5A4D + Lq
    qI = dsa_inputs.e4m3_small_int(seed, 1, Lq * H_I * d_I).reshape(Lq, H_I, d_I)
    kI = dsa_inputs.e4m3_small_int(seed, 2, Lk * d_I).reshape(Lk, d_I)
    w = (dsa_inputs.uniform_int(seed, 3, Lq * H_I, -8, 8) / 8.0).astype(np.float32).reshape(Lq, H_I)
    q = dsa_inputs.normal_bf16_bits(seed, 4, Lq * H * d_qk).reshape(Lq, H, d_qk)
    kv = dsa_inputs.normal_bf16_bits(seed, 5, Lk * d_qk).reshape(Lk, d_qk)
    scale = 1 / np.sqrt(d_qk)
    for rank in range(world):
        start, stop = sharding.shard_causal_rows(Lq, Lk, k, rank, world, mla_weight=sharding.MLA_WEIGHT)
        Lq_loc, Lk_loc = stop - start, stop + (Lk - Lq)
        for i in (0, Lq_loc // 2, Lq_loc - 1):
            g = start + i
            t_full, t_loc = g + Lk - Lq, i + Lk_loc - Lq_loc
            assert t_loc == t_full
            s_full = ref.indexer_row(qI[g], kI, w[g], t_full)
            s_loc = ref.indexer_row(qI[g], kI[:Lk_loc], w[g], t_loc)
            np.testing.assert_array_equal(s_loc[: t_loc + 1], s_full[: t_full + 1])
            idx_full, n_full = ref.topk_row(s_full, t_full, k)
            idx_loc, n_loc = ref.topk_row(s_loc, t_loc, k)
            np.testing.assert_array_equal(idx_loc, idx_full)
            assert n_loc == n_full
            o_full, lse_full, _ = ref.sparse_mla_row(q[g], kv, idx_full, d_v, scale)
            o_loc, lse_loc, _ = ref.sparse_mla_row(q[g], kv[:Lk_loc], idx_loc, d_v, scale)
            np.testing.assert_array_equal(o_loc, o_full)
            np.testing.assert_array_equal(lse_loc, lse_full)
