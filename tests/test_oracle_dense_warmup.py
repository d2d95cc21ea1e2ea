"""Pins of the oracle's dense warm-up target and loss ("DSA Continued Pre-Training" page, Stage 1;
analysis page eq. (3)).

Anchors independent of the oracle's code: torch's fp64 softmax of the MQA logits (a library
routine) summed over heads for the target p; scipy's relative entropy for the KL; the closed form
KL = 0 when I = ln p; and the pages' statement that eq. (4) differs from eq. (3) only in the range
of the sum, so that a selection covering every s <= t gives the same target and loss.
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import dsa_inputs
from oracle import oracle as ref


def _case(seed, H=4, d_qk=80, L=40):
    q = dsa_inputs.normal_bf16_bits(seed, 4, H * d_qk).reshape(H, d_qk)
    kv = dsa_inputs.normal_bf16_bits(seed, 5, L * d_qk).reshape(L, d_qk)
    return q, kv


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(torch.float64)


@pytest.mark.parametrize("t", [0, 1, 17, 39])
def test_dense_target_is_the_head_summed_softmax_normalised(t):
    q, kv = _case(41)
    scale = 1 / math.sqrt(80)
    p = ref.dense_p_row(q, kv, t, scale)
    logits = torch.einsum("hd,sd->hs", _bf16(q), _bf16(kv[: t + 1])) * scale
    lib = torch.softmax(logits, dim=-1).sum(0)
    lib = (lib / lib.sum()).numpy()
    np.testing.assert_allclose(p, lib, rtol=1e-12, atol=1e-15)
    assert abs(p.sum() - 1.0) < 1e-12


def test_one_head_target_is_that_heads_attention():
    q, kv = _case(43, H=1)
    t = 25
    scale = 0.1
    p = ref.dense_p_row(q, kv, t, scale)
    _, _, A = ref.dense_mla_row(q, kv, t, 64, scale, want_A=True)
    np.testing.assert_allclose(p, A[0], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("t", [3, 30])
def test_dense_target_equals_sparse_target_when_the_selection_covers_the_prefix(t):
    q, kv = _case(47)
    scale = 1 / math.sqrt(80)
    k = 40
    idx = np.full(k, -1, np.int32)
    idx[: t + 1] = np.arange(t + 1)
    _, _, P = ref.sparse_mla_row(q, kv, idx, 64, scale, want_P=True)
    p_sel = ref.p_sel_row(P, idx)
    p_dense = ref.dense_p_row(q, kv, t, scale)
    np.testing.assert_allclose(p_sel[: t + 1], p_dense, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_dense_kl_matches_scipy_relative_entropy(seed):
    rng = np.random.default_rng(seed)
    t = 50
    scores = np.full(64, -np.inf)
    scores[: t + 1] = rng.normal(size=t + 1) * 3
    p = rng.dirichlet(np.ones(t + 1))
    p[7] = 0.0
    p /= p.sum()
    got = ref.dense_kl_row(scores, t, p)
    q = scipy.special.softmax(scores[: t + 1])
    assert abs(got - scipy.stats.entropy(p, q)) <= 1e-12 * max(1.0, abs(got))


def test_dense_kl_is_zero_when_the_scores_are_the_log_target():
    rng = np.random.default_rng(5)
    t = 30
    p = rng.dirichlet(np.ones(t + 1))
    scores = np.log(p) + 4.25  # any per-row shift: Softmax removes it
    assert abs(ref.dense_kl_row(scores, t, p)) < 1e-13


def test_eq3_and_eq4_agree_when_the_selection_covers_the_prefix():
    rng = np.random.default_rng(9)
    t, k = 20, 32
    scores = rng.normal(size=40) * 2
    p = rng.dirichlet(np.ones(t + 1))
    idx = np.full(k, -1, np.int32)
    idx[: t + 1] = np.arange(t + 1)
    p_slots = np.zeros(k)
    p_slots[: t + 1] = p
    assert abs(ref.kl_row(scores, idx, p_slots) - ref.dense_kl_row(scores, t, p)) < 1e-13
