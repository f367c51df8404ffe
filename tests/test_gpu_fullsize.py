"""Parity at the full workload sizes, in the launch configuration the
benchmark times: the GPU runs the whole batch, the oracle checks a sample of
queries (or compressed blocks) that it can compute one by one."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import assert_close, assert_topk_sets, host

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def csa():
    import compressed_sparse_attention_14_b200 as m
    return m


def _decode_check(csa, s, sample):
    inp = synth.decode_inputs(s, device=DEV)
    out, lse, sel = csa.csa_decode(inp["qI"], inp["w"], inp["idx_cache"], inp["q"], inp["kv_cache"],
                                   inp["ctx_len"], s.m, s.k, return_topk=True)
    torch.cuda.synchronize()
    for b in sample:
        h = {k: v[b:b + 1].cpu() for k, v in inp.items()}
        v = int(h["ctx_len"][0]) // s.m
        K = h["idx_cache"][:, :v]
        ref_idx, S = oracle.index_topk(h["qI"], h["w"], K, h["ctx_len"], s.m, s.k)
        assert_topk_sets(sel[b:b + 1], ref_idx, S, s.k)
        ref_o, ref_l = oracle.sparse_mqa(h["q"], h["kv_cache"][:, :v], host(sel[b:b + 1]).astype(np.int32),
                                         1 / math.sqrt(s.c))
        assert_close(out[b:b + 1], ref_o, torch.bfloat16, f"decode out (query {b})")
        assert_close(lse[b:b + 1], ref_l, torch.bfloat16, f"decode lse (query {b})")
    # properties at every query: selections are visible, distinct and full
    sel_h = host(sel)
    vis = inp["ctx_len"].cpu().numpy() // s.m
    assert np.all(sel_h < vis[:, None])
    assert np.all(sel_h >= 0)
    for b in range(sel_h.shape[0]):
        assert len(set(sel_h[b].tolist())) == s.k
    assert torch.isfinite(out.float()).all()


def test_flash_decode_full_size(csa):
    _decode_check(csa, synth.FLASH_DECODE, sample=(0, 31, 63))


def test_pro_decode_full_size(csa):
    _decode_check(csa, synth.PRO_DECODE, sample=(0, 31))


def test_hca_decode_full_size(csa):
    s = synth.HCA
    inp = synth.hca_decode_inputs(s, device=DEV)
    out, lse = csa.hca_decode(inp["q"], inp["kv_cache"], inp["ctx_len"], s.mp)
    torch.cuda.synchronize()
    for b in (0, 15):
        ref_o, ref_l = oracle.dense_mqa(inp["q"][b:b + 1].cpu(), inp["kv_cache"][b:b + 1].cpu(),
                                        inp["ctx_len"][b:b + 1].cpu(), s.mp, 1 / math.sqrt(s.c))
        assert_close(out[b:b + 1], ref_o, torch.bfloat16, f"hca out (query {b})")
        assert_close(lse[b:b + 1], ref_l, torch.bfloat16, f"hca lse (query {b})")


def test_hca_compress_chunk_full_size(csa):
    s = synth.HCA
    inp = synth.hca_compress_inputs(s, device=DEV)
    out = csa.hca_compress_from_hidden(inp["x"], inp["W"], inp["bias"], s.mp)
    torch.cuda.synchronize()
    W = inp["W"].cpu()
    bias = inp["bias"].cpu()
    for blk in (0, 511, 1023):
        rows = inp["x"][blk * s.mp:(blk + 1) * s.mp].cpu()
        ref = oracle.hca_compress_from_hidden(rows, W, bias, s.mp)
        assert_close(out[blk:blk + 1], ref, torch.bfloat16, f"hca compress block {blk}")


def test_csa_prefill_full_size(csa):
    s = synth.PREFILL
    inp = synth.prefill_inputs(s, device=DEV)
    out, lse, sel = csa.csa_prefill(inp["x"], inp["x_left"], inp["W_kv"], inp["B_kv"], inp["W_idx"],
                                    inp["B_idx"], inp["start"], inp["kv_cache"], inp["idx_cache"], inp["qI"],
                                    inp["w"], inp["q"], s.k, m=s.m, return_topk=True)
    torch.cuda.synchronize()
    m, start, n = s.m, inp["start"], inp["n"]
    e0 = start // m
    # oracle caches: the prefix as generated, the new entries compressed from the hidden states
    kv = oracle._f64(inp["kv_cache"][:e0].cpu())
    ik = oracle._f64(inp["idx_cache"][:e0].cpu())
    xh, xl = inp["x"].cpu(), inp["x_left"].cpu()
    new_kv = oracle.bf16_round(oracle.csa_compress_from_hidden(xh, inp["W_kv"].cpu(), inp["B_kv"].cpu(), m, X_left=xl))
    new_ik = oracle.bf16_round(oracle.csa_compress_from_hidden(xh, inp["W_idx"].cpu(), inp["B_idx"].cpu(), m,
                                                               X_left=xl))
    assert_close(inp["kv_cache"][e0:], new_kv, torch.bfloat16, "prefill kv entries")
    assert_close(inp["idx_cache"][e0:], new_ik, torch.bfloat16, "prefill idx entries")
    kv = np.concatenate([kv, new_kv])
    ik = np.concatenate([ik, new_ik])
    for t in (0, 1, 2, 3, 4095, 32768, n - 1):
        p = np.array([start + t], dtype=np.int32)
        ref_idx, S = oracle.index_topk(inp["qI"][t:t + 1].cpu(), inp["w"][t:t + 1].cpu(), ik, p, m, s.k)
        assert_topk_sets(sel[t:t + 1], ref_idx, S, s.k)
        ref_o, _ = oracle.sparse_mqa(inp["q"][t:t + 1].cpu(), kv, host(sel[t:t + 1]).astype(np.int32),
                                     1 / math.sqrt(s.c))
        assert_close(out[t:t + 1], ref_o, torch.bfloat16, f"prefill out (token {t})")
    sel_h = host(sel)
    vis = (start + np.arange(n)) // m
    assert np.all(sel_h < vis[:, None]) and np.all(sel_h >= 0)
