"""The indexer's top-k filter (candidate lists written by the indexer
epilogue, then an exact selection over them) against the score-block path
(every score stored, then the top-k kernel), and against the oracle.

The two paths compute the same fp32 scores in the same kernel arithmetic, so
their selections must agree bit for bit: same indices in the same order, and
the same attention output. The oracle checks the selected sets by the gap
rule. Rows are ragged (visible counts off the tile size, below k, zero), and
two adversarial patterns defeat the running bound: scores that rise along the
row (every score beats the bound so far, so every visible column becomes a
candidate and a list outgrows the shared-memory selection) and rows of equal
scores (ties decided by the lower column)."""
import dataclasses
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
    yield m
    m.debug_set(0, 0)


def _both_paths(csa, run):
    """run() under the top-k filter (opt-in) and under the score block (the
    default)."""
    csa.debug_set(0, csa.CSA_DEBUG_TOPK_FILTER)
    try:
        a = run()
    finally:
        csa.debug_set(0, 0)
    csa.debug_set(0, csa.CSA_DEBUG_SCORE_BLOCK)
    try:
        b = run()
    finally:
        csa.debug_set(0, 0)
    torch.cuda.synchronize()
    return a, b


def _decode_inputs(B, Nmax, HI, cI, H, c, ctx, seed):
    g = lambda shape, tag: synth.normal(shape, seed, tag)
    return dict(idx_cache=g((B, Nmax, cI), "f_idx"), kv_cache=g((B, Nmax, c), "f_kv"), q=g((B, H, c), "f_q"),
                qI=g((B, HI, cI), "f_qI"), w=synth.head_weights(B, HI, seed),
                ctx_len=torch.tensor(ctx, dtype=torch.int32))


def _decode(csa, inp, m, k):
    dev = {kk: v.to(DEV) for kk, v in inp.items()}
    return lambda: csa.csa_decode(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], dev["kv_cache"], dev["ctx_len"],
                                  m, k, return_topk=True)


# (B, Nmax, HI, cI, H, c, k, context lengths): the decode instantiation (64
# index heads of 128), the general one (32 heads of 64), a k of 1024
DECODE_CASES = [
    (6, 3000, 64, 128, 8, 128, 512, [12000, 11999, 4 * 1000 + 3, 4 * 511, 0, 4 * 2999 + 1]),
    (5, 2200, 32, 64, 8, 128, 96, [8800, 5000, 4 * 97 + 2, 3, 6001]),
    (3, 5000, 64, 128, 8, 128, 1024, [20000, 4 * 3333, 4 * 1500]),
]


@pytest.mark.parametrize("B,Nmax,HI,cI,H,c,k,ctx", DECODE_CASES)
def test_decode_filter_equals_score_block_and_the_oracle(csa, B, Nmax, HI, cI, H, c, k, ctx):
    inp = _decode_inputs(B, Nmax, HI, cI, H, c, ctx, seed=31)
    (o1, l1, s1), (o2, l2, s2) = _both_paths(csa, _decode(csa, inp, 4, k))
    assert torch.equal(s1, s2), "selection differs between the filter and the score block"
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ref_idx, S = oracle.index_topk(inp["qI"], inp["w"], inp["idx_cache"], inp["ctx_len"], 4, k, seq=torch.arange(B))
    assert_topk_sets(s1, ref_idx, S, k)
    # rows with fewer visible entries than k list all of them, then -1
    for b, L in enumerate(ctx):
        v = min(L // 4, Nmax)
        if v < k:
            row = host(s1)[b]
            assert sorted(row[:v].tolist()) == list(range(v)) and (row[v:] == -1).all()


def test_decode_filter_rising_scores(csa):
    # K_s = a_s * u with a_s increasing and q^I . u > 0 for every head: the
    # score rises along the row, so each new score beats the bound so far and
    # every visible column is a candidate (lists of 12,000 > the 8,192 that
    # the selection holds in shared memory)
    B, Nmax, HI, cI, H, c, k = 2, 12288, 64, 128, 8, 128, 512
    u = torch.ones(cI)
    a = torch.linspace(0.05, 1.0, Nmax)
    inp = _decode_inputs(B, Nmax, HI, cI, H, c, [4 * 12000, 4 * 9000], seed=32)
    inp["idx_cache"] = (a[None, :, None] * u[None, None, :]).expand(B, Nmax, cI).to(torch.bfloat16).contiguous()
    inp["qI"] = inp["qI"].abs()
    (o1, l1, s1), (o2, l2, s2) = _both_paths(csa, _decode(csa, inp, 4, k))
    assert torch.equal(s1, s2)
    ref_idx, S = oracle.index_topk(inp["qI"], inp["w"], inp["idx_cache"], inp["ctx_len"], 4, k, seq=torch.arange(B))
    assert_topk_sets(s1, ref_idx, S, k)


def test_decode_filter_equal_scores(csa):
    # every key the same: all scores tie, the k lowest columns win, in order
    B, Nmax, HI, cI, H, c, k = 2, 4000, 64, 128, 8, 128, 512
    inp = _decode_inputs(B, Nmax, HI, cI, H, c, [4 * 4000, 4 * 2500 + 1], seed=33)
    inp["idx_cache"] = inp["idx_cache"][:, :1].expand(B, Nmax, cI).contiguous()
    (o1, l1, s1), (o2, l2, s2) = _both_paths(csa, _decode(csa, inp, 4, k))
    assert torch.equal(s1, s2)
    assert (host(s1) == np.arange(k)[None, :]).all()


def _prefill(csa, s, inp):
    def run():
        dev = {kk: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for kk, v in inp.items()}
        return csa.csa_prefill(dev["x"], dev["x_left"], dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"],
                               inp["start"], dev["kv_cache"], dev["idx_cache"], dev["qI"], dev["w"], dev["q"], s.k,
                               m=s.m, return_topk=True)
    return run


# the grouped prefill instantiation (4 tokens x 64 index heads of 128 per
# MMA), k = 512 and 1024; and the general one (the tiny shape's 4 heads of 64)
PREFILL_CASES = [
    dataclasses.replace(synth.PREFILL, n=2048, start=8192, d=256, c=128, heads=8),
    dataclasses.replace(synth.PREFILL, n=1024, start=4096 + 512, d=256, c=128, heads=8, k=1024),
    dataclasses.replace(synth.TINY, n=1024, start=512, k=40),
]


@pytest.mark.parametrize("s", PREFILL_CASES, ids=lambda s: f"n{s.n}_at{s.start}_HI{s.idx_heads}_k{s.k}")
def test_prefill_filter_equals_score_block_and_the_oracle(csa, s):
    inp = synth.prefill_inputs(s)
    (o1, l1, s1), (o2, l2, s2) = _both_paths(csa, _prefill(csa, s, inp))
    assert torch.equal(s1, s2), "selection differs between the filter and the score block"
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # the oracle on a sample of rows (every 37th token and the last one)
    m = s.m
    ik = oracle._f64(inp["idx_cache"]).copy()
    ik[s.start // m:(s.start + s.n) // m] = oracle.bf16_round(
        oracle.csa_compress_from_hidden(inp["x"], inp["W_idx"], inp["B_idx"], m, X_left=inp["x_left"]))
    rows = np.unique(np.r_[np.arange(0, s.n, 37), s.n - 1])
    pos = (s.start + rows).astype(np.int32)
    ref_idx, S = oracle.index_topk(inp["qI"][rows], inp["w"][rows], ik, pos, m, s.k)
    assert_topk_sets(s1[torch.as_tensor(rows)], ref_idx, S, s.k)
    ref_o, _ = oracle.sparse_mqa(inp["q"][rows], _kv_after(inp, s), host(s1)[rows].astype(np.int32),
                                 1 / math.sqrt(s.c))
    assert_close(o1[torch.as_tensor(rows)], ref_o, torch.bfloat16, "prefill out (sampled rows)")


def _kv_after(inp, s):
    kv = oracle._f64(inp["kv_cache"]).copy()
    kv[s.start // s.m:(s.start + s.n) // s.m] = oracle.bf16_round(
        oracle.csa_compress_from_hidden(inp["x"], inp["W_kv"], inp["B_kv"], s.m, X_left=inp["x_left"]))
    return kv


def test_attend_and_fp8kv_decode_filter_equals_score_block(csa):
    # the complete-output decode and the FP8-KV decode select through the same
    # step: the filter gives them the same entries and the same bits
    B, Nmax, HI, cI, H, c, k, n_win = 5, 3000, 64, 128, 8, 128, 512, 128
    inp = _decode_inputs(B, Nmax, HI, cI, H, c, [12000, 4 * 2200 + 1, 4 * 700, 4 * 1999, 11000], seed=34)
    ring = synth.normal((B, n_win, c), 34, "f_ring")
    dev = {kk: v.to(DEV) for kk, v in inp.items()}
    kv_ext = torch.cat([inp["kv_cache"], ring], dim=1).contiguous().to(DEV)
    gamma = (1.0 + synth.normal((c,), 34, "f_gamma", std=0.1, dtype=torch.float32)).to(DEV)
    sink = synth.normal((H,), 34, "f_sink", dtype=torch.float32).to(DEV)

    def attend():
        return csa.csa_attend_decode(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], kv_ext, dev["ctx_len"], 4, k,
                                     n_win=n_win, ring_len=n_win, q_gamma=gamma, rope_dims=64, sink=sink,
                                     return_topk=True)

    (o1, l1, s1), (o2, l2, s2) = _both_paths(csa, attend)
    assert torch.equal(s1, s2) and torch.equal(o1, o2) and torch.equal(l1, l2)

    codes, scales, rope = csa.csa_quantize_kv_fp8(dev["kv_cache"], rope_dims=64)

    def fp8kv():
        return csa.csa_decode_fp8kv(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], codes, scales, rope,
                                    dev["ctx_len"], 4, k, return_topk=True)

    (o1, l1, s1), (o2, l2, s2) = _both_paths(csa, fp8kv)
    assert torch.equal(s1, s2) and torch.equal(o1, o2) and torch.equal(l1, l2)
