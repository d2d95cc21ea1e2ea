"""Pins of the oracle's HISA retrieval ("DeepSeek-V3.2" analysis page, sec. 5.3: block-level
coarse selection, then exact token scores inside the kept blocks; eq. (24) and (25)).

Anchors independent of the HISA code: numpy means of the decoded keys; the page's block-mean
example (a single key with dot product 10 among 63 keys near -0.2 gives the block a mean dot
product below zero, so the coarse stage can drop the block that holds the best token); the
reduction to plain DSA selection when the kept blocks cover every visible key; and eq. (24)'s
decomposition, in which exact second-stage scores make R_token|block = 1.
"""
import numpy as np
import pytest
import torch

import dsa_inputs
from oracle import oracle as ref


def _f64(b):
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _case(seed, Lk=700, H_I=8, d_I=32):
    q = dsa_inputs.e4m3_small_int(seed, 1, H_I * d_I).reshape(H_I, d_I)
    k = dsa_inputs.e4m3_small_int(seed, 2, Lk * d_I).reshape(Lk, d_I)
    w = (dsa_inputs.uniform_int(seed, 3, H_I, -16, 16) / 16.0).astype(np.float32)
    return q, k, w


def test_block_mean_is_the_mean_of_the_decoded_keys():
    _, k, _ = _case(1)
    for s0, n in ((0, 64), (64, 64), (640, 60), (5, 1)):
        np.testing.assert_allclose(ref.block_mean(k, s0, n), _f64(k[s0: s0 + n]).mean(0), rtol=0, atol=1e-15)


def test_block_mean_drowns_a_single_spike():
    # the page's example: one key with dot product 10, 63 keys near -0.2 (here -13/64, the nearest
    # e4m3 value), one head, w = 1: the spike's block has a negative mean dot product
    # (10 - 63 * 13/64) / 64 = -0.0437, so it scores ReLU(.) = 0 and loses to a block of plain
    # keys, although its spike is the best token of the sequence
    q = dsa_inputs.int_to_e4m3(np.array([[1]]))
    spike = np.full((64, 1), 0xA5, np.uint8)  # e4m3 0xA5 = -13/64
    spike[17, 0] = 0x52  # e4m3 0x52 = 10
    plain = np.full((64, 1), 0x18, np.uint8)  # e4m3 0x18 = 1/16
    keys = np.concatenate([spike, plain])
    assert _f64(keys[17, 0]) == 10.0 and _f64(keys[0, 0]) == -13 / 64 and _f64(keys[64, 0]) == 1 / 16
    w = np.ones(1, np.float32)
    m = ref.block_mean(keys, 0, 64)
    assert abs(m[0] - (10 - 63 * 13 / 64) / 64) < 1e-15
    assert ref.block_score(q, m, w) == 0.0
    assert ref.block_score(q, ref.block_mean(keys, 64, 64), w) == 1 / 16
    t = 127
    idx1, blocks1, n1 = ref.hisa_row(q, keys, w, t, 64, 1, 1)   # one block kept: the plain one
    assert list(blocks1) == [1] and n1 == 1 and idx1[0] == 64
    dsa, _ = ref.topk_row(ref.indexer_row(q, keys, w, t), t, 1)
    assert dsa[0] == 17                                         # DSA picks the spike
    idx2, blocks2, _ = ref.hisa_row(q, keys, w, t, 64, 2, 1)    # both blocks kept: the spike
    assert list(blocks2) == [0, 1] and idx2[0] == 17


@pytest.mark.parametrize("t,bsize,r,k", [(699, 64, 11, 64), (450, 64, 8, 100), (300, 32, 10, 16), (63, 64, 1, 8)])
def test_hisa_equals_dsa_when_the_kept_blocks_cover_every_visible_key(t, bsize, r, k):
    q, keys, w = _case(3 + t)
    assert r * bsize >= t + 1
    idx, blocks, n = ref.hisa_row(q, keys, w, t, bsize, r, k)
    dsa, n_dsa = ref.topk_row(ref.indexer_row(q, keys, w, t), t, k)
    np.testing.assert_array_equal(idx, dsa)
    assert n == n_dsa
    assert list(blocks[blocks >= 0]) == list(range(t // bsize + 1))


@pytest.mark.parametrize("seed", [5, 6, 7, 8])
def test_recall_decomposes_with_exact_second_stage_scores(seed):
    # eq. (24): R_final = R_block * R_token|block, and with the second stage on the exact scores
    # every DSA-selected token that falls in a kept block is kept (R_token|block = 1)
    q, keys, w = _case(seed, Lk=1500)
    t, bsize, r, k = 1499, 64, 6, 128
    idx, blocks, n = ref.hisa_row(q, keys, w, t, bsize, r, k)
    dsa, _ = ref.topk_row(ref.indexer_row(q, keys, w, t), t, k)
    T = set(int(s) for s in dsa if s >= 0)
    S = set(int(s) for s in idx if s >= 0)
    U = set(s for b in blocks if b >= 0 for s in range(b * bsize, min((b + 1) * bsize, t + 1)))
    assert T & U <= S                      # R_token|block = 1
    r_block = len(T & U) / len(T)
    r_final = len(T & S) / len(T)
    assert r_final == r_block
    assert len(S) == min(k, len(U))


def test_kept_blocks_are_the_best_block_scores_with_causal_means():
    q, keys, w = _case(9)
    t, bsize, r = 450, 64, 3  # block 7 holds the query: its mean covers keys 448..450 only
    scores = []
    for b in range(t // bsize + 1):
        s0 = b * bsize
        n = min(bsize, t + 1 - s0)
        mean = _f64(keys[s0: s0 + n]).mean(0)
        qf = _f64(q)
        scores.append(float((w.astype(np.float64) * np.maximum(qf @ mean, 0)).sum()))
    scores = np.array(scores)
    # rank counting with the tie rule (larger score, then smaller block)
    rank = [sum(1 for c in range(len(scores)) if scores[c] > scores[b] or (scores[c] == scores[b] and c < b))
            for b in range(len(scores))]
    expected = sorted(b for b in range(len(scores)) if rank[b] < r)
    _, blocks, _ = ref.hisa_row(q, keys, w, t, bsize, r, 32)
    assert list(blocks) == expected
