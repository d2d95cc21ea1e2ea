"""Pins of the CPU oracle's indexer (eq. (1)) and top-k selection (eq. (2)/(4)).

Each check ties the oracle to something fixed outside it: a hand-worked example,
a library decoder, an invariant the pages state, or an independent definition
(rank counting) on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

import dsa_inputs
from oracle import oracle as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _two_token_fixture():
    g = _parse(os.path.join(GOLDEN, "indexer_two_token.txt"))
    H_I = int(next(r for r in g if r[0] == "H_I")[1])
    d_I = int(next(r for r in g if r[0] == "d_I")[1])
    k_I = np.zeros((2, d_I), dtype=np.int64)
    q_I = np.zeros((2, H_I, d_I), dtype=np.int64)
    w = np.zeros((2, H_I), dtype=np.float32)
    I_exp = np.zeros((2, 2))
    topk, tie = [], {}
    for r in g:
        if r[0] == "k_I":
            k_I[int(r[1])] = [int(x) for x in r[2:]]
        elif r[0] == "q_I":
            q_I[int(r[1]), int(r[2])] = [int(x) for x in r[3:]]
        elif r[0] == "w":
            w[int(r[1])] = [float(x) for x in r[2:]]
        elif r[0] == "I":
            I_exp[int(r[1])] = [float(x) for x in r[2:]]
        elif r[0] == "topk":
            topk.append((int(r[1]), int(r[2]), [int(x) for x in r[3:]]))
        elif r[0] in ("tie_w", "tie_I", "tie_topk"):
            tie[r[0]] = r[1:]
    return H_I, d_I, k_I, q_I, w, I_exp, topk, tie


def test_e4m3_decoder_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in codes:
        mine = ref.e4m3_to_double(int(c))
        if math.isnan(lib[c]):
            assert math.isnan(mine)
        else:
            assert mine == lib[c], hex(c)


def test_bf16_decoder_matches_torch():
    bits = dsa_inputs.normal_bf16_bits(7, 1, 4096)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for b, v in zip(bits[:512], lib[:512]):
        assert ref.bf16_to_double(int(b)) == v


def test_generator_integers_encode_exactly_in_e4m3():
    v = np.arange(-3, 4)
    enc = dsa_inputs.int_to_e4m3(v)
    back = torch.from_numpy(enc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(back, v.astype(np.float64))


def test_indexer_hand_worked_two_token_example():
    H_I, d_I, k_I, q_I, w, I_exp, topk, tie = _two_token_fixture()
    kI = dsa_inputs.int_to_e4m3(k_I)
    for t in range(2):
        got = ref.indexer_row(dsa_inputs.int_to_e4m3(q_I[t]), kI, w[t], t)
        assert np.array_equal(got, I_exp[t]), (t, got)
    # top-k sets of the example
    scores = [ref.indexer_row(dsa_inputs.int_to_e4m3(q_I[t]), kI, w[t], t) for t in range(2)]
    for t, k, exp in topk:
        idx, n = ref.topk_row(scores[t], t, k)
        assert n == len(exp)
        assert list(idx[:n]) == exp
        assert all(x == -1 for x in idx[n:])
    # tie variant: equal scores, the smaller position wins
    w_tie = w.copy()
    w_tie[int(tie["tie_w"][0])] = [float(x) for x in tie["tie_w"][1:]]
    s1 = ref.indexer_row(dsa_inputs.int_to_e4m3(q_I[1]), kI, w_tie[1], 1)
    assert list(s1) == [float(x) for x in tie["tie_I"][1:]]
    idx, n = ref.topk_row(s1, 1, 1)
    assert n == 1 and idx[0] == int(tie["tie_topk"][2])


def _rand_indexer_case(seed, H_I=4, d_I=32, Lk=40, w_lo=-8, w_hi=8):
    q = dsa_inputs.uniform_int(seed, 1, H_I * d_I, -3, 3).reshape(H_I, d_I)
    k = dsa_inputs.uniform_int(seed, 2, Lk * d_I, -3, 3).reshape(Lk, d_I)
    w = dsa_inputs.uniform_int(seed, 3, H_I, w_lo, w_hi).astype(np.float32) / 8
    return q, k, w


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_indexer_relu_terms_are_nonnegative(seed):
    # Every head term ReLU(q.k) >= 0 (analysis page sec. 5.2 on eq. (17)): with w >= 0 the score
    # is >= 0, with w <= 0 it is <= 0, and a single head with w = 1 equals max(0, q.k).
    q, k, w = _rand_indexer_case(seed)
    t = k.shape[0] - 1
    pos = ref.indexer_row(dsa_inputs.int_to_e4m3(q), dsa_inputs.int_to_e4m3(k), np.abs(w), t)
    neg = ref.indexer_row(dsa_inputs.int_to_e4m3(q), dsa_inputs.int_to_e4m3(k), -np.abs(w), t)
    assert (pos >= 0).all() and (neg <= 0).all()
    one = ref.indexer_row(dsa_inputs.int_to_e4m3(q[:1]), dsa_inputs.int_to_e4m3(k),
                          np.ones(1, np.float32), t)
    assert (one >= 0).all()
    assert (one == 0).any() and (one > 0).any()


def test_indexer_causal_mask_and_head_additivity():
    q, k, w = _rand_indexer_case(11)
    kI = dsa_inputs.int_to_e4m3(k)
    t = 17
    full = ref.indexer_row(dsa_inputs.int_to_e4m3(q), kI, w, t)
    assert np.isneginf(full[t + 1:]).all() and np.isfinite(full[: t + 1]).all()
    # heads enter additively: I over heads {0,1} + I over heads {2,3} = I over all four
    a = ref.indexer_row(dsa_inputs.int_to_e4m3(q[:2]), kI, w[:2], t)
    b = ref.indexer_row(dsa_inputs.int_to_e4m3(q[2:]), kI, w[2:], t)
    assert np.array_equal(a[: t + 1] + b[: t + 1], full[: t + 1])
    # scaling w scales the score (w enters linearly, outside the ReLU)
    d = ref.indexer_row(dsa_inputs.int_to_e4m3(q), kI, 2 * w, t)
    assert np.array_equal(d[: t + 1], 2 * full[: t + 1])


def test_indexer_scores_are_exact_in_fp32_at_full_dims():
    # H_I=64, d_I=128, integer q/k in [-3,3], w in (1/16)Z: |I| <= 64*128*9 on a 1/16 grid,
    # below 2^24/16, so the fp64 value is an fp32 value (the GPU must match it bit for bit).
    wl = dsa_inputs.WORKLOADS["decode_32k"]
    q = dsa_inputs.q_index(wl, 0, 1)[0]
    w = dsa_inputs.w_index(wl, 0, 1)[0]
    k = dsa_inputs.k_index(wl, 0)[:300]
    s = ref.indexer_row(q, k, w, 299)
    assert np.array_equal(s.astype(np.float32).astype(np.float64), s)
    assert np.array_equal(np.round(s * 16), s * 16)


def _rank_count_select(scores, t, k):
    """Independent definition of S_t: s is selected iff fewer than k candidates beat it,
    where s' beats s when its score is larger, or equal with a smaller position."""
    sel = []
    for s in range(t + 1):
        beaten_by = sum(1 for u in range(t + 1)
                        if scores[u] > scores[s] or (scores[u] == scores[s] and u < s))
        if beaten_by < k:
            sel.append(s)
    return sel


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_rank_counting_with_heavy_ties(seed):
    rng = np.random.default_rng(seed)
    L = 37
    scores = rng.integers(-3, 4, size=L).astype(np.float64)  # many ties
    scores[rng.integers(0, L, 3)] = rng.normal(size=3)
    for t in (0, 1, 5, 20, L - 1):
        row = scores.copy()
        row[t + 1:] = -np.inf
        for k in (1, 2, 7, 16, 36, 40):
            idx, n = ref.topk_row(row, t, k)
            exp = _rank_count_select(row, t, k)
            assert n == min(k, t + 1) == len(exp)
            assert list(idx[:n]) == exp
            assert (idx[n:] == -1).all()


def test_topk_partial_order_on_generated_scores():
    wl = dsa_inputs.WORKLOADS["tiny_prefill"]
    q = dsa_inputs.q_index(wl, 200, 1)[0]
    w = dsa_inputs.w_index(wl, 200, 1)[0]
    k = dsa_inputs.k_index(wl, 0)
    s = ref.indexer_row(q, k, w, 200)
    idx, n = ref.topk_row(s, 200, wl.k)
    sel = set(idx[:n].tolist())
    assert n == wl.k
    unsel = [u for u in range(201) if u not in sel]
    lo = min(s[list(sel)])
    for u in unsel:
        assert s[u] <= lo
        if s[u] == lo:  # at the cutoff value, every selected tie has a smaller position
            assert all(v < u for v in sel if s[v] == lo)


def test_topk_selects_everything_when_k_covers_the_prefix():
    row = np.array([5.0, 5.0, 1.0, 7.0, -np.inf, -np.inf])
    idx, n = ref.topk_row(row, 3, 8)
    assert n == 4 and list(idx) == [0, 1, 2, 3, -1, -1, -1, -1]
