"""Pins of the oracle's masked MHA ("DeepSeek-V3.2-Exp" page, sec. 3, inference costs: short
prefills run MLA's MHA mode with a mask that keeps each query's top-k set, which simulates DSA).

Anchors: torch's fp64 scaled-dot-product attention with a boolean mask (a library routine); and
the two MLA modes of the analysis page (sec. 1.1 and Fig. 7: MHA mode decompresses the latent into
per-head keys and values, MQA mode absorbs the decompression into the query and the output), so
masked MHA over S_t equals DSA's MQA-mode attention over S_t, up-projected."""
import numpy as np
import pytest
import torch

from oracle import oracle as ref


def _case(seed, L=60, H=4, dqk=24, dv=16):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(H, dqk)), rng.normal(size=(L, H, dqk)), rng.normal(size=(L, H, dv))


@pytest.mark.parametrize("t,k", [(59, 16), (30, 40), (0, 4), (45, 45)])
def test_masked_mha_matches_torch_sdpa_with_a_mask(t, k):
    q, kk, v = _case(t + k)
    rng = np.random.default_rng(k)
    n = min(k, t + 1)
    idx = np.full(k, -1, np.int32)
    idx[:n] = np.sort(rng.permutation(t + 1)[:n])
    out, lse = ref.masked_mha_row(q, kk, v, idx, 0.2)
    mask = torch.zeros(1, 1, 1, kk.shape[0], dtype=torch.bool)
    mask[..., idx[idx >= 0]] = True
    Q = torch.tensor(q)[None, :, None, :]
    K = torch.tensor(kk).permute(1, 0, 2)[None]
    V = torch.tensor(v).permute(1, 0, 2)[None]
    o_lib = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=0.2)[0, :, 0].numpy()
    logits = torch.einsum("hd,hsd->hs", torch.tensor(q), K[0]) * 0.2
    lse_lib = torch.logsumexp(logits.masked_fill(~mask[0, 0], float("-inf")), -1).numpy()
    np.testing.assert_allclose(out, o_lib, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse_lib, rtol=1e-12, atol=1e-12)


def test_an_empty_selection_gives_zeros_and_minus_infinity():
    q, kk, v = _case(3)
    out, lse = ref.masked_mha_row(q, kk, v, np.full(8, -1, np.int32), 0.3)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_masked_mha_equals_mqa_mode_attention_through_the_absorbed_projections():
    # latent c = [c_nope (dc) | rope (dr)]; MHA mode: k_h = [W_uk_h c_nope ; rope], v_h = W_uv_h c_nope;
    # MQA mode: q~_h = [W_uk_h^T q_nope ; q_rope], o_h = W_uv_h sum_s P_s c_nope,s
    rng = np.random.default_rng(11)
    L, H, dc, dr, dn, dv, t, k = 50, 3, 20, 6, 8, 7, 49, 12
    c = rng.normal(size=(L, dc + dr))
    Wuk = rng.normal(size=(H, dn, dc)) / np.sqrt(dc)
    Wuv = rng.normal(size=(H, dv, dc)) / np.sqrt(dc)
    q = rng.normal(size=(H, dn + dr))
    idx = np.sort(rng.permutation(t + 1)[:k]).astype(np.int32)
    k_mha = np.concatenate([np.einsum("hnc,sc->shn", Wuk, c[:, :dc]), np.repeat(c[:, None, dc:], H, 1)], -1)
    v_mha = np.einsum("hvc,sc->shv", Wuv, c[:, :dc])
    out, lse = ref.masked_mha_row(q, k_mha, v_mha, idx, 0.5)
    q_abs = np.concatenate([np.einsum("hnc,hn->hc", Wuk, q[:, :dn]), q[:, dn:]], -1)  # [H, dc + dr]
    z = 0.5 * q_abs @ c[idx].T
    P = np.exp(z - z.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    o_lat = P @ c[idx, :dc]
    np.testing.assert_allclose(out, np.einsum("hvc,hc->hv", Wuv, o_lat), rtol=1e-10, atol=1e-12)
