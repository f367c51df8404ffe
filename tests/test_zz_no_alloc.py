"""The allocation-free indexer + top-k entry point (csa_index_topk_noalloc).

Some callers cannot allocate device memory when they select entries: a
plug-in whose host framework owns every device allocation and gives it no
scratch, a serving loop whose memory footprint is fixed after start-up, or a
latency-critical path that cannot afford cudaMalloc. For them the score
block between the indexer and the selection lives in a fixed array inside
the library instead of a caller workspace.

This checks, through the C ABI, that two calls in a row each return exactly
what the workspace-taking csa_index_topk returns on the same inputs. The
indices are integer results and both paths run the same kernels, so the
comparison is bit-exact (indices and their fp32 scores). The second call is
smaller than the first, so it runs over an array still holding the first
call's scores, and one of its queries reads a sequence outside the cache
(it must get no entry, not a stale one). Host-side argument checks, such as
the size limit, are in test_abi.py. This file is collected last on purpose.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(g, nq, n_seq, Nmax, HI, cI, lo, hi):
    qI = torch.randn(nq, HI, cI, generator=g, device=DEV).to(torch.bfloat16)
    w = torch.softmax(torch.randn(nq, HI, generator=g, device=DEV), dim=1)
    K = torch.randn(n_seq, Nmax, cI, generator=g, device=DEV).to(torch.bfloat16)
    pos = torch.randint(lo, hi + 1, (nq,), generator=g, device=DEV, dtype=torch.int32)
    return qI, w, K, pos


def _call_noalloc(csa, qI, w, K, pos, seq, m, k, idx, top):
    nq, HI, cI = qI.shape
    n_seq, Nmax = K.shape[0], K.shape[1]
    return csa._lib.csa_index_topk_noalloc(qI.data_ptr(), w.data_ptr(), K.data_ptr(), pos.data_ptr(),
                                           None if seq is None else seq.data_ptr(), nq, n_seq, HI, cI, Nmax, m, k,
                                           idx.data_ptr(), top.data_ptr(), csa.CSA_BF16,
                                           torch.cuda.current_stream().cuda_stream)


def test_noalloc_index_topk_equals_workspace_index_topk_two_calls_in_a_row():
    import compressed_sparse_attention_14_b200 as csa
    g = torch.Generator(device=DEV).manual_seed(2024)
    m = 4
    # call 1: decode-shaped (one query per sequence, 32768 entries, k = 512:
    # 8 MiB of scores); call 2: 24 queries over 3 sequences of 20000 entries,
    # k = 2048, one query on a sequence outside the cache
    calls = [
        dict(nq=64, n_seq=64, Nmax=32768, k=512, lo=65536, hi=131072, seq=None),
        dict(nq=24, n_seq=3, Nmax=20000, k=2048, lo=0, hi=80000, seq="mapped"),
    ]
    for c in calls:
        qI, w, K, pos = _inputs(g, c["nq"], c["n_seq"], c["Nmax"], 64, 128, c["lo"], c["hi"])
        seq = None
        if c["seq"]:
            seq = torch.randint(0, c["n_seq"], (c["nq"],), generator=g, device=DEV, dtype=torch.int32)
            seq[5] = c["n_seq"]          # no such sequence: no entry
            pos[1] = 4 * 2048 + 3        # exactly k visible entries
        ref_idx, ref_top = csa.csa_index_topk(qI, w, K, pos, m, c["k"], seq_of_q=seq)
        idx = torch.full((c["nq"], c["k"]), 7, dtype=torch.int32, device=DEV)
        top = torch.zeros((c["nq"], c["k"]), dtype=torch.float32, device=DEV)
        launches = csa.launch_count()
        rc = _call_noalloc(csa, qI, w, K, pos, seq, m, c["k"], idx, top)
        assert rc == csa.CSA_OK, csa._lib.csa_last_error()
        assert csa.launch_count() - launches == 2      # the indexer and the selection, nothing else
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(top, ref_top)
        if seq is not None:
            assert bool((idx[5] == -1).all())
    csa.poll_status()
