"""GPU parity of the masked-MHA short-prefill path (dsa_masked_mha_fwd; "DeepSeek-V3.2-Exp" page,
sec. 3, inference costs) against the fp64 oracle: ragged causal tiles, rows whose whole prefix is
selected (t + 1 <= k), sparse rows, holes in idx, and several heads and sequences."""
import numpy as np
import pytest
import torch

import dsa_inputs
from oracle import oracle as ref
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as m
    m.load()
    return m


def _bf16(seed, tid, shape):
    bits = dsa_inputs.normal_bf16_bits(seed, tid, int(np.prod(shape))).reshape(shape)
    return bits, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("B,L,H,k", [(2, 300, 4, 64), (1, 1000, 3, 256), (1, 520, 2, 600)])
def test_masked_mha_matches_the_oracle(dsa, B, L, H, k):
    seed = 4000 + L + k
    qb, q = _bf16(seed, 4, (B, L, H, 192))
    kb, kk = _bf16(seed, 5, (B, L, H, 192))
    vb, v = _bf16(seed, 6, (B, L, H, 128))
    rng = np.random.default_rng(seed)
    idx = np.full((B, L, k), -1, np.int32)
    for b in range(B):
        for t in range(L):
            n = min(k, t + 1)
            idx[b, t, :n] = rng.permutation(t + 1)[:n]  # any order
            if t % 7 == 3 and n > 2:
                idx[b, t, 1] = -1                         # a hole
    dev = lambda a, dt: torch.from_numpy(a.view(np.int16)).view(dt).cuda()
    out = torch.empty(B, L, H, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, L, H, device="cuda")
    ws = torch.empty(dsa.dsa_workspace_bytes(dsa.DSA_OP_MASKED_MHA, B, L, L, k, H), dtype=torch.uint8, device="cuda")
    scale = 1 / np.sqrt(192.0)
    dsa.dsa_masked_mha_fwd(dev(qb, torch.bfloat16), dev(kb, torch.bfloat16), dev(vb, torch.bfloat16),
                           torch.from_numpy(idx).cuda(), scale, out, lse, ws)
    assert dsa.dsa_last_device_status() == 0
    g_out = out.float().cpu().numpy()
    g_lse = lse.cpu().numpy()
    rows = [(b, t) for b in range(B) for t in range(L) if t < 140 or t % 13 == 0 or t == L - 1]
    for b, t in rows:
        e_out, e_lse = ref.masked_mha_row(q[b, t], kk[b], v[b], idx[b, t], scale)
        parity.check_attention_row(g_out[b, t], e_out, f"row ({b},{t})")
        assert np.abs(g_lse[b, t] - e_lse).max() <= parity.LSE_ATOL, f"lse row ({b},{t})"
