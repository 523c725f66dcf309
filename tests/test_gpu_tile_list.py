"""Compacted tile list of a block mask on the GPU: bit-exact against the oracle's CSR."""
import numpy as np
import pytest
import torch

import oracle
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,S,seed", [(40, 32768, 0), (40, 32768, 1), (3, 1000, 2), (1, 128, 3), (5, 57344, 4)])
def test_tile_list_bit_exact(H, S, seed):
    mask = synth.block_mask(H, S, seed=seed)
    T = mask.shape[-1]
    row_ptr = torch.full((H * T + 1,), -7, dtype=torch.int32, device="cuda")
    col_idx = torch.full((H * T * T,), -7, dtype=torch.int32, device="cuda")
    counts = torch.empty((H * T,), dtype=torch.int32, device="cuda")
    spattn.sp_build_tile_list(mask.cuda(), S, row_ptr, col_idx, counts)
    ref_ptr, ref_idx = oracle.tile_list(mask.numpy())
    assert np.array_equal(row_ptr.cpu().numpy(), ref_ptr)
    nnz = int(ref_ptr[-1])
    got = col_idx.cpu().numpy()
    assert np.array_equal(got[:nnz], ref_idx)
    assert np.all(got[nnz:] == -7)  # nothing written past the list


def test_tile_list_empty_and_full_rows():
    H, S = 2, 640
    T = 5
    mask = torch.zeros((H, T, T), dtype=torch.uint8)
    mask[1] = 1
    row_ptr = torch.empty((H * T + 1,), dtype=torch.int32, device="cuda")
    col_idx = torch.empty((H * T * T,), dtype=torch.int32, device="cuda")
    counts = torch.empty((H * T,), dtype=torch.int32, device="cuda")
    spattn.sp_build_tile_list(mask.cuda(), S, row_ptr, col_idx, counts)
    ref_ptr, ref_idx = oracle.tile_list(mask.numpy())
    assert np.array_equal(row_ptr.cpu().numpy(), ref_ptr)
    assert np.array_equal(col_idx.cpu().numpy()[: len(ref_idx)], ref_idx)
