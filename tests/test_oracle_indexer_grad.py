"""Pins of the oracle's indexer-loss gradient (the indexer is trained from L^I alone: "DSA
Continued Pre-Training" page, Stage 2; analysis page eq. (4) and the detached-input paragraph).

Anchors independent of the gradient code: central finite differences of the oracle's own loss
(a different function: it never forms a derivative) at random real inputs, where no ReLU argument
sits at its kink; torch autograd in fp64 of the loss written with library ops; and the softmax
identity that the logit gradient sums to zero when p sums to one.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as ref


def _case(seed, H_I=4, d_I=8, Lk=30, k=12, holes=True):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(H_I, d_I))
    kk = rng.normal(size=(Lk, d_I))
    w = rng.normal(size=H_I)
    idx = np.sort(rng.permutation(Lk)[:k]).astype(np.int32)
    p = rng.dirichlet(np.ones(k))
    if holes:
        idx[3] = -1
        p[3] = 0.0
        p[5] = 0.0
        p /= p.sum()
    return q, kk, w, idx, p


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_gradient_matches_central_finite_differences(seed):
    q, kk, w, idx, p = _case(seed)
    dq, dw, dk, g = ref.indexer_grad_row(q, kk, w, idx, p)
    f = lambda q_, k_, w_: ref.indexer_loss_row_f64(q_, k_, w_, idx, p)
    h = 1e-6
    for j in range(q.shape[0]):
        for d in range(q.shape[1]):
            a, b = q.copy(), q.copy()
            a[j, d] += h
            b[j, d] -= h
            fd = (f(a, kk, w) - f(b, kk, w)) / (2 * h)
            assert abs(fd - dq[j, d]) <= 1e-6 * max(1.0, abs(fd)), ("dq", j, d, fd, dq[j, d])
    for j in range(w.shape[0]):
        a, b = w.copy(), w.copy()
        a[j] += h
        b[j] -= h
        fd = (f(q, kk, a) - f(q, kk, b)) / (2 * h)
        assert abs(fd - dw[j]) <= 1e-6 * max(1.0, abs(fd)), ("dw", j, fd, dw[j])
    for s in range(kk.shape[0]):
        for d in range(kk.shape[1]):
            a, b = kk.copy(), kk.copy()
            a[s, d] += h
            b[s, d] -= h
            fd = (f(q, a, w) - f(q, b, w)) / (2 * h)
            assert abs(fd - dk[s, d]) <= 1e-6 * max(1.0, abs(fd)), ("dk", s, d, fd, dk[s, d])


def test_gradient_matches_torch_autograd():
    q, kk, w, idx, p = _case(7, H_I=6, d_I=16, Lk=50, k=20)
    dq, dw, dk, g = ref.indexer_grad_row(q, kk, w, idx, p)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(kk, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    valid = torch.tensor(idx >= 0)
    sel = torch.tensor(np.where(idx >= 0, idx, 0), dtype=torch.long)
    scores = (wt[None, :] * torch.relu(kt[sel] @ qt.T)).sum(1)            # I over the slots
    logq = torch.log_softmax(scores.masked_fill(~valid, float("-inf")), 0)
    pt = torch.tensor(p)
    terms = torch.where(pt > 0, pt * (torch.log(torch.where(pt > 0, pt, torch.ones_like(pt))) - logq),
                        torch.zeros_like(pt))
    terms.sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_logit_gradient_sums_to_zero_and_vanishes_off_the_selection():
    q, kk, w, idx, p = _case(11)
    dq, dw, dk, g = ref.indexer_grad_row(q, kk, w, idx, p)
    assert abs(g.sum()) < 1e-14
    assert np.all(g[idx < 0] == 0)
    unselected = np.setdiff1d(np.arange(kk.shape[0]), idx[idx >= 0])
    assert np.all(dk[unselected] == 0)


def test_gradient_is_zero_when_the_indexer_already_matches_the_target():
    # with one head, w = 1 and every dot product positive, I = q . k; choose p = Softmax(I)
    rng = np.random.default_rng(13)
    q = np.abs(rng.normal(size=(1, 4))) + 0.1
    kk = np.abs(rng.normal(size=(10, 4))) + 0.1
    w = np.ones(1)
    idx = np.arange(10, dtype=np.int32)
    I = kk @ q[0]
    p = np.exp(I - I.max())
    p /= p.sum()
    dq, dw, dk, g = ref.indexer_grad_row(q, kk, w, idx, p)
    assert np.abs(g).max() < 1e-15 and np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    assert abs(ref.indexer_loss_row_f64(q, kk, w, idx, p)) < 1e-14
