"""The allocation-free top-k entry point (csa_topk_from_scores_noalloc).

Some callers cannot allocate device memory when they select entries (a
plug-in whose host framework owns all device allocations and gives it no
workspace; a serving loop that forbids allocation after start-up). The
selection keeps its scratch in on-chip shared memory. This checks, through
the C ABI, that calls in a row return exactly what the workspace-taking
csa_topk_from_scores returns (top-k is integer work: the comparison is
bit-exact), at row lengths up to 2^20 and k up to the maximum. (Its host-side
argument checks are in test_abi.py.) This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call_noalloc(csa, scores, valid, valid_div, k, idx, top):
    nq, ncols = scores.shape
    return csa._lib.csa_topk_from_scores_noalloc(scores.data_ptr(), ncols, valid.data_ptr(), valid_div, nq, ncols, k,
                                                 idx.data_ptr(), top.data_ptr(),
                                                 torch.cuda.current_stream().cuda_stream)


def test_noalloc_topk_equals_workspace_topk_two_calls_in_a_row():
    import compressed_sparse_attention_14_b200 as csa
    g = torch.Generator().manual_seed(2024)
    cases = [
        # (rows, columns, k, valid divisor): sampled-threshold rows, short rows
        (32, 262144, 1024, 4),
        (64, 40000, 512, 1),
        (8, 1 << 20, 2048, 1),
    ]
    for nq, ncols, k, div in cases:
        S = torch.randn(nq, ncols, generator=g)
        S[0] = torch.randint(-2, 3, (ncols,), generator=g).float()   # ties
        valid = torch.randint(0, ncols * div + 5, (nq,), generator=g, dtype=torch.int32)
        valid[1] = (k - 1) * div                                      # fewer candidates than k
        S_d, v_d = S.to(DEV), valid.to(DEV)
        ref_idx, ref_top = csa.csa_topk_from_scores(S_d, k, valid=v_d, valid_div=div)
        idx = torch.empty((nq, k), dtype=torch.int32, device=DEV)
        top = torch.empty((nq, k), dtype=torch.float32, device=DEV)
        assert _call_noalloc(csa, S_d, v_d, div, k, idx, top) == csa.CSA_OK, csa._lib.csa_last_error()
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(top, ref_top)
