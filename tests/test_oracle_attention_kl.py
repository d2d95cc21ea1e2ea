"""Pins of the CPU oracle's sparse MQA attention, head-summed target p and KL loss.

Anchors: torch's fp64 scaled-dot-product attention (a library routine) for dense
causal MQA; the pages' statements that sparse attention over a set covering every
s <= t equals dense attention, eq. (19) (renormalised restriction) and eq. (20)
(error bound) of the analysis page sec. 5.2; the three-head example of sec. 5.1;
scipy's relative entropy for KL; and a closed form on a 2-element set.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import dsa_inputs
from oracle import oracle as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_to_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(
        torch.float64)


def _case(seed, H=4, d_qk=80, d_v=64, L=48):
    q = dsa_inputs.normal_bf16_bits(seed, 4, H * d_qk).reshape(H, d_qk)
    kv = dsa_inputs.normal_bf16_bits(seed, 5, L * d_qk).reshape(L, d_qk)
    return q, kv


@pytest.mark.parametrize("t", [0, 1, 13, 47])
def test_dense_mqa_matches_torch_sdpa_fp64(t):
    H, d_qk, d_v = 4, 80, 64
    q, kv = _case(3, H, d_qk, d_v)
    scale = 1 / math.sqrt(80)
    out, lse, _ = ref.dense_mla_row(q, kv, t, d_v, scale)
    Q = _bf16_to_f64(q).reshape(1, H, 1, d_qk)
    K = _bf16_to_f64(kv[: t + 1]).reshape(1, 1, t + 1, d_qk).expand(1, H, t + 1, d_qk)
    V = _bf16_to_f64(kv[: t + 1, :d_v]).reshape(1, 1, t + 1, d_v).expand(1, H, t + 1, d_v)
    o_lib = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)[0, :, 0].numpy()
    logits = torch.einsum("hd,sd->hs", _bf16_to_f64(q), _bf16_to_f64(kv[: t + 1])) * scale
    lse_lib = torch.logsumexp(logits, dim=-1).numpy()
    np.testing.assert_allclose(out, o_lib, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_lib, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("t", [0, 5, 30])
def test_sparse_equals_dense_when_selection_covers_prefix(t):
    q, kv = _case(5)
    scale = 1 / math.sqrt(80)
    k = 40
    idx = np.full(k, -1, np.int32)
    idx[: t + 1] = np.arange(t + 1)[::-1]  # any order, with -1 padding
    o_s, lse_s, _ = ref.sparse_mla_row(q, kv, idx, 64, scale)
    o_d, lse_d, _ = ref.dense_mla_row(q, kv, t, 64, scale)
    np.testing.assert_allclose(o_s, o_d, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse_s, lse_d, rtol=1e-12, atol=1e-13)


def test_sparse_is_renormalised_restriction_eq19_and_obeys_eq20_bound():
    q, kv = _case(9, L=48)
    scale = 1 / math.sqrt(80)
    t = 47
    _, _, A = ref.dense_mla_row(q, kv, t, 64, scale, want_A=True)
    o_d, _, _ = ref.dense_mla_row(q, kv, t, 64, scale)
    rng = np.random.default_rng(0)
    S = np.sort(rng.choice(t + 1, size=12, replace=False)).astype(np.int32)
    o_s, _, _ = ref.sparse_mla_row(q, kv, S, 64, scale)
    v = _bf16_to_f64(kv[:, :64]).numpy()
    Vmax = np.linalg.norm(v[: t + 1], axis=1).max()
    for h in range(q.shape[0]):
        M = A[h, S].sum()
        eq19 = (A[h, S][:, None] / M * v[S]).sum(0)
        np.testing.assert_allclose(o_s[h], eq19, rtol=1e-11, atol=1e-12)
        assert np.linalg.norm(o_d[h] - o_s[h]) <= 2 * (1 - M) * Vmax + 1e-12


def test_single_head_single_entry_returns_that_value_row():
    q, kv = _case(12, H=1)
    idx = np.array([-1, 29, -1], np.int32)
    out, lse, P = ref.sparse_mla_row(q, kv, idx, 64, 0.1, want_P=True)
    np.testing.assert_array_equal(out[0], _bf16_to_f64(kv[29, :64]).numpy())
    z = 0.1 * float(_bf16_to_f64(q[0]) @ _bf16_to_f64(kv[29]))
    assert abs(lse[0] - z) < 1e-12
    assert list(P[0]) == [0.0, 1.0, 0.0]


def test_probabilities_match_torch_softmax_and_p_is_their_normalised_head_sum():
    q, kv = _case(21, H=6, L=60)
    scale = 1 / math.sqrt(80)
    idx = np.array([3, 17, -1, 40, 41, 59, 0, -1], np.int32)
    _, _, P = ref.sparse_mla_row(q, kv, idx, 64, scale, want_P=True)
    valid = idx >= 0
    logits = torch.einsum("hd,sd->hs", _bf16_to_f64(q), _bf16_to_f64(kv[idx[valid]])) * scale
    P_lib = torch.softmax(logits, dim=-1).numpy()
    np.testing.assert_allclose(P[:, valid], P_lib, rtol=1e-12, atol=1e-15)
    assert (P[:, ~valid] == 0).all()
    p = ref.p_sel_row(P, idx)
    assert abs(p.sum() - 1) < 1e-12
    np.testing.assert_allclose(p[valid], P_lib.sum(0) / P_lib.sum(), rtol=1e-12)
    # single head: p equals that head's probabilities
    p1 = ref.p_sel_row(P[:1], idx)
    np.testing.assert_allclose(p1, P[0], rtol=1e-12, atol=1e-15)


def test_three_head_example_of_shared_budget():
    # Analysis page sec. 5.1 (after eq. (16)): three heads put 0.9 of their mass on
    # positions 10, 20 and 30; with k = 2 every shared set drops at least one head's peak.
    L = 40
    P = np.full((3, L), 0.1 / (L - 1))
    for h, pos in enumerate((10, 20, 30)):
        P[h, pos] = 0.9
    idx = np.arange(L, dtype=np.int32)
    p = ref.p_sel_row(P, idx)
    assert abs(p[10] - (0.9 + 2 * 0.1 / 39) / 3) < 1e-15
    assert p[10] == p[20] == p[30]
    for pair in ((10, 20), (10, 30), (20, 30)):
        per_head = [P[h, list(pair)].sum() for h in range(3)]
        assert min(per_head) < 0.01  # the head whose peak is outside the pair keeps < 1% mass
        assert abs(p[list(pair)].sum() - 2 * p[10]) < 1e-15


def test_kl_two_element_closed_form():
    g = {}
    with open(os.path.join(GOLDEN, "kl_two_element.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                a = line.split()
                g[a[0]] = a[1:]
    p = np.array([float(x) for x in g["p"]])
    scores = np.array([math.log(3.0), 0.0])
    kl = ref.kl_row(scores, np.array([0, 1], np.int32), p)
    assert abs(kl - float(g["kl"][0])) < 1e-15


def test_kl_zero_when_scores_are_log_p_and_shift_invariant():
    rng = np.random.default_rng(4)
    p = rng.dirichlet(np.ones(9))
    idx = np.array([4, 0, 8, 2, 6, 1, 7, 3, 5], np.int32)
    scores = np.full(9, -np.inf)
    scores[idx] = np.log(p)
    assert abs(ref.kl_row(scores, idx, p)) < 1e-14
    s2 = rng.normal(size=9) * 3
    a = ref.kl_row(s2, idx, p)
    b = ref.kl_row(s2 + 123.25, idx, p)
    assert a >= 0 and abs(a - b) < 1e-12


@pytest.mark.parametrize("seed", range(4))
def test_kl_matches_scipy_relative_entropy(seed):
    rng = np.random.default_rng(seed)
    k = 16
    idx = rng.permutation(40)[:k].astype(np.int32)
    idx[rng.integers(0, k, 3)] = -1  # empty slots are skipped
    scores = rng.normal(size=40) * 4
    p = rng.dirichlet(np.ones(k))
    p[idx < 0] = 0
    p[rng.integers(0, k)] = 0.0  # a zero-probability term contributes 0
    p /= p.sum()
    v = idx >= 0
    q = scipy.special.softmax(scores[idx[v]])
    exp = scipy.stats.entropy(p[v], q)
    assert abs(ref.kl_row(scores, idx, p) - exp) < 1e-12


def test_path_rows_composes_the_row_functions():
    wl = dsa_inputs.WORKLOADS["tiny_prefill"]
    wl = dsa_inputs.custom("tiny_kl", wl.seed, 1, 64, 64, 4, 32, 8, 16, 8, 80, 64, emit_p=True)
    qI, kI, w = dsa_inputs.q_index(wl), dsa_inputs.k_index(wl), dsa_inputs.w_index(wl)
    q, kv = dsa_inputs.q_attn(wl), dsa_inputs.kv_latent(wl)
    rows = [0, 1, 15, 16, 63]
    res = ref.path_rows(wl, rows, qI, kI, w, q, kv, rows_packed=False, nthreads=2)
    for j, r in enumerate(rows):
        t = wl.t_of(r)
        s = ref.indexer_row(qI[r], kI[0], w[r], t)
        np.testing.assert_array_equal(res["scores"][j], s)
        idx, n = ref.topk_row(s, t, wl.k)
        np.testing.assert_array_equal(res["idx"][j], idx)
        out, lse, P = ref.sparse_mla_row(q[r], kv[0], idx, wl.d_v, wl.scale, want_P=True)
        np.testing.assert_array_equal(res["out"][j], out)
        p = ref.p_sel_row(P, idx)
        np.testing.assert_array_equal(res["p"][j], p)
        assert res["kl"][j] == ref.kl_row(s, idx, p)
