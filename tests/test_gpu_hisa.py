"""GPU parity of HISA's decode selection ("DeepSeek-V3.2" analysis page, sec. 5.3) against the fp64
oracle: the block sums, the kept blocks and the selected tokens, exact for integer-valued FP8
inputs (whole blocks of 64 keys: every block mean is a multiple of 1/64 and every block score an
exact fp32 value); and the reduction to the DSA selection when the kept blocks cover the cache."""
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


def _run(dsa, wl, dw, block, r):
    B, Lk, k = wl.B, wl.Lk, wl.k
    sums = torch.empty(B, -(-Lk // block), 128, device="cuda")
    dsa.dsa_hisa_block_sums(dw.kI, block, sums)
    idx = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    blocks = torch.full((B, 1, r), -7, dtype=torch.int32, device="cuda")
    ws = torch.zeros(dsa.dsa_hisa_workspace_bytes(B, Lk, block, r, k), dtype=torch.uint8, device="cuda")
    dsa.dsa_hisa_topk(dw.qI, dw.kI, dw.w, sums, block, r, idx, blocks, ws)
    assert dsa.dsa_last_device_status() == 0
    return sums.cpu().numpy(), idx.cpu().numpy(), blocks.cpu().numpy()


@pytest.mark.parametrize("B,Lk,block,r,k,w_den", [
    (4, 8192, 64, 16, 512, 16),     # 128 blocks, keep 16 (1024 candidates)
    (3, 32768, 64, 64, 2048, 16),   # 512 blocks, keep 64 (4096 candidates)
    (5, 4096, 64, 8, 1024, 1),      # w in {-1, 0, 1}: tied block and token scores; k = r * block
    (2, 6400, 128, 50, 2048, 16),   # blocks of 128, every block kept: the DSA selection
])
def test_hisa_selection_matches_the_oracle(dsa, B, Lk, block, r, k, w_den):
    wl = dsa_inputs.custom(f"hisa_{Lk}_{r}", 8080 + Lk + r, B, 1, Lk, 64, 128, w_den, k, 1, 16, 16)
    dw = parity.DeviceWorkload(wl, with_attention=False)
    sums, idx, blocks = _run(dsa, wl, dw, block, r)
    kf = torch.from_numpy(dw.kI_np).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(sums, kf.reshape(B, Lk // block, block, 128).sum(2).astype(np.float32))
    qI = dw.qI_np.reshape(B, 64, 128)
    w = dw.w_np.reshape(B, 64)
    for b in range(B):
        e_idx, e_blocks, n = ref.hisa_row(qI[b], dw.kI_np[b], w[b], Lk - 1, block, r, k)
        np.testing.assert_array_equal(blocks[b, 0], e_blocks, err_msg=f"blocks row {b}")
        np.testing.assert_array_equal(idx[b, 0], e_idx, err_msg=f"idx row {b}")
        if r * block >= Lk:  # every block kept: the plain DSA selection
            dsa_idx, _ = ref.topk_row(ref.indexer_row(qI[b], dw.kI_np[b], w[b], Lk - 1), Lk - 1, k)
            np.testing.assert_array_equal(idx[b, 0], dsa_idx)
