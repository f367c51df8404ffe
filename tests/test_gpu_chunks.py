"""Prefill chunks at any start and length, then decode steps, through the
per-sequence state ring [Walk §5 item 2: the tail tokens that have not yet
formed a block stay in a fixed per-request state; Notes §2.6 Fig. 6].

A sequence is prefilled in chunks that start and end mid-block and then
compressed token by token; its caches must equal the oracle's compression of
the whole sequence in one chunk, and every prefill output row must equal the
oracle's attention for that token over those caches."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import assert_close, assert_topk_sets, host

pytestmark = pytest.mark.gpu
DEV = "cuda"
MODES = [torch.bfloat16, torch.float32]


@pytest.fixture(scope="module")
def csa():
    import compressed_sparse_attention_14_b200 as m
    return m


def _conv(t, dtype):
    return t.to(dtype) if t.dtype == torch.bfloat16 else t


@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("chunks", [(1021, 3, 517), (2, 1, 6, 1021, 510)])
def test_prefill_unaligned_chunks_then_decode_equal_one_chunk(csa, dtype, chunks):
    s = synth.TINY
    m, k = s.m, s.k
    n_pre = sum(chunks)
    n_dec = 7
    T = n_pre + n_dec
    Nmax = T // m + 2
    inp = synth.prefill_inputs(s, n=T)
    inp = {kk: (_conv(v, dtype) if isinstance(v, torch.Tensor) else v) for kk, v in inp.items()}
    dev = {kk: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for kk, v in inp.items()}
    c, cI = s.c, s.idx_dim
    kv = torch.zeros((Nmax, c), dtype=dtype, device=DEV)
    ik = torch.zeros((Nmax, cI), dtype=dtype, device=DEV)
    st_kv = torch.full((2 * m, 4 * c), float("nan"), dtype=torch.float32, device=DEV)
    st_idx = torch.full((2 * m, 4 * cI), float("nan"), dtype=torch.float32, device=DEV)
    outs, sels = [], []
    p0 = 0
    for n in chunks:
        sl = slice(p0, p0 + n)
        o, _, sel = csa.csa_prefill(dev["x"][sl], None, dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"], p0, kv,
                                    ik, dev["qI"][sl].contiguous(), dev["w"][sl].contiguous(), dev["q"][sl].contiguous(),
                                    k, m=m, return_topk=True, state_kv=st_kv, state_idx=st_idx)
        outs.append(o)
        sels.append(sel)
        p0 += n
    # then token by token (the decode-time step), continuing the same rings
    for p in range(n_pre, T):
        csa.csa_decode_compress(dev["x"][p:p + 1].contiguous(), dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"],
                                torch.tensor([p], dtype=torch.int32, device=DEV), st_kv[None], st_idx[None],
                                kv[None], ik[None], m)
    torch.cuda.synchronize()
    rnd = oracle.bf16_round if dtype == torch.bfloat16 else (lambda a: a)
    nb = T // m
    ref_kv = rnd(oracle.csa_compress_from_hidden(inp["x"][: nb * m], inp["W_kv"], inp["B_kv"], m))
    ref_ik = rnd(oracle.csa_compress_from_hidden(inp["x"][: nb * m], inp["W_idx"], inp["B_idx"], m))
    assert_close(kv[:nb], ref_kv, dtype, "KV entries")
    assert_close(ik[:nb], ref_ik, dtype, "index keys")
    assert bool((kv[nb:] == 0).all()) and bool((ik[nb:] == 0).all())
    # the prefill rows: indexer + top-k + MQA over the whole sequence's caches
    out = torch.cat(outs)
    sel = torch.cat(sels)
    pos = np.arange(0, n_pre, dtype=np.int32)
    ref_idx, S = oracle.index_topk(inp["qI"][:n_pre], inp["w"][:n_pre], ref_ik, pos, m, k)
    assert_topk_sets(sel, ref_idx, S, k)
    ref_o, _ = oracle.sparse_mqa(inp["q"][:n_pre], ref_kv, host(sel).astype(np.int32), 1 / math.sqrt(c))
    assert_close(out, ref_o, dtype, "prefill out")


@pytest.mark.parametrize("dtype", MODES)
def test_chunk_compression_any_split_equals_chunk_definition(csa, dtype):
    # csa_compress_chunk and hca_compress_chunk from projected rows, the
    # sequence split at arbitrary points (and empty chunks), against the
    # chunk compressors of the oracle over the whole sequence
    m, mp, c = 4, 16, 64
    T = 203
    P4 = synth.normal((T, 4 * c), 21, "ck_p4", dtype=torch.float32)
    P2 = synth.normal((T, 2 * c), 21, "ck_p2", dtype=torch.float32)
    Bc = synth.normal((2 * m, c), 21, "ck_b", std=math.sqrt(0.1), dtype=torch.float32)
    Bh = synth.normal((mp, c), 21, "ck_bh", std=math.sqrt(0.1), dtype=torch.float32)
    cuts = [0, 1, 1, 3, 10, 47, 48, 49, 130, 131, 200, T]
    kv = torch.zeros((T // m, c), dtype=dtype, device=DEV)
    hv = torch.zeros((T // mp, c), dtype=dtype, device=DEV)
    st4 = torch.zeros((2 * m, 4 * c), dtype=torch.float32, device=DEV)
    st2 = torch.zeros((mp, 2 * c), dtype=torch.float32, device=DEV)
    P4d, P2d, Bcd, Bhd = P4.to(DEV), P2.to(DEV), Bc.to(DEV), Bh.to(DEV)
    for a, b in zip(cuts[:-1], cuts[1:]):
        csa.csa_compress_chunk(P4d[a:b].contiguous(), st4, Bcd, a, kv, m)
        csa.hca_compress_chunk(P2d[a:b].contiguous(), st2, Bhd, a, hv, mp)
    torch.cuda.synchronize()
    rnd = oracle.bf16_round if dtype == torch.bfloat16 else (lambda a: a)
    ref = rnd(oracle.csa_compress(P4[: (T // m) * m], Bc, m))
    refh = rnd(oracle.hca_compress(P2[: (T // mp) * mp], Bh, mp))
    assert_close(kv, ref, dtype, "CSA entries")
    assert_close(hv, refh, dtype, "HCA entries")
