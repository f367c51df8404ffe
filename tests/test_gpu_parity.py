"""GPU parity: each entry point of the C ABI against the CPU oracle on the same
seeded inputs, element by element, at sizes that span several kernel tiles
and a ragged tail, in both storage modes (bf16 and fp32)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import (TOL, assert_close, assert_scores_close, assert_topk_order, assert_topk_sets, host,
                          score_bound)

pytestmark = pytest.mark.gpu

DEV = "cuda"
MODES = [torch.bfloat16, torch.float32]


@pytest.fixture(scope="module")
def csa():
    import compressed_sparse_attention_14_b200 as m
    return m


def _g(shape, tag, dtype=torch.bfloat16, std=1.0, seed=100):
    """seeded host tensor (the oracle reads this copy) and its device copy"""
    h = synth.normal(shape, seed, tag, std=std, dtype=dtype)
    return h, h.to(DEV)


# ---------------------------------------------------------------- a2 / a3
@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("with_left", [False, True])
def test_csa_compress(csa, dtype, with_left):
    m, c, n = 4, 136, 4 * 333          # 333 blocks: ragged against 256-thread CTAs
    proj_h, proj = _g((n, 4 * c), "proj", dtype)
    bias_h, bias = _g((2 * m, c), "bias", torch.float32, std=0.3)
    left_h, left = _g((m, 4 * c), "left", dtype) if with_left else (None, None)
    got = csa.csa_compress(proj, bias, m, left=left)
    ref = oracle.csa_compress(proj_h, bias_h, m, left=left_h)
    assert_close(got, ref, dtype, "csa_compress")


@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("mp", [128, 4, 1])
def test_hca_compress(csa, dtype, mp):
    c, n = 64, mp * 37
    proj_h, proj = _g((n, 2 * c), "hproj", dtype)
    bias_h, bias = _g((mp, c), "hbias", torch.float32, std=0.3)
    got = csa.hca_compress(proj, bias, mp)
    assert_close(got, oracle.hca_compress(proj_h, bias_h, mp), dtype, "hca_compress")


# ---------------------------------------------------------------- a1
@pytest.mark.parametrize("dtype", MODES)
def test_project(csa, dtype):
    n, d, M = 333, 264, 200
    x_h, x = _g((n, d), "x", dtype)
    W_h, W = _g((M, d), "W", dtype, std=1 / math.sqrt(d))
    got = csa.csa_project(x, W)
    ref = oracle.project(x_h, W_h)
    # fp32 accumulation over d terms of unit-scale products
    err = np.abs(host(got) - ref).max()
    assert err <= 1e-5 * math.sqrt(d) * 4, err


@pytest.mark.parametrize("dtype", MODES)
def test_csa_compress_from_hidden(csa, dtype):
    m, c, d, n = 4, 64, 256, 4 * 70
    x_h, x = _g((n, d), "xh", dtype)
    xl_h, xl = _g((m, d), "xl", dtype)
    W_h, W = _g((4 * c, d), "Wc", dtype, std=1 / math.sqrt(d))
    b_h, b = _g((2 * m, c), "bc", torch.float32, std=math.sqrt(0.1))
    for left_h, left in ((None, None), (xl_h, xl)):
        got = csa.csa_compress_from_hidden(x, W, b, m, x_left=left)
        ref = oracle.csa_compress_from_hidden(x_h, W_h, b_h, m, X_left=left_h)
        assert_close(got, ref, dtype, "csa_compress_from_hidden")


@pytest.mark.parametrize("dtype", MODES)
def test_hca_compress_from_hidden(csa, dtype):
    mp, c, d, n = 128, 64, 256, 128 * 5
    x_h, x = _g((n, d), "xhh", dtype)
    W_h, W = _g((2 * c, d), "Wh", dtype, std=1 / math.sqrt(d))
    b_h, b = _g((mp, c), "bh", torch.float32, std=math.sqrt(0.1))
    got = csa.hca_compress_from_hidden(x, W, b, mp)
    assert_close(got, oracle.hca_compress_from_hidden(x_h, W_h, b_h, mp), dtype, "hca_compress_from_hidden")


# ---------------------------------------------------------------- a4
def _index_inputs(dtype, nq, HI, cI, B, Nmax, m, seed=7):
    qI_h, qI = _g((nq, HI, cI), "qI", dtype, seed=seed)
    K_h, K = _g((B, Nmax, cI), "K", dtype, seed=seed)
    w_h = synth.head_weights(nq, HI, seed)
    pos_h = synth.uniform_int(nq, 0, Nmax * m + 2 * m, seed, "pos")
    pos_h[0] = 0
    pos_h[-1] = Nmax * m + m - 1
    return qI_h, qI, K_h, K, w_h, w_h.to(DEV), pos_h, pos_h.to(DEV)


@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("shape", [(16, 64, 128, 16, 1000, 4), (40, 4, 64, 1, 531, 4)])
def test_index_scores(csa, dtype, shape):
    nq, HI, cI, B, Nmax, m = shape
    qI_h, qI, K_h, K, w_h, w, pos_h, pos = _index_inputs(dtype, nq, HI, cI, B, Nmax, m)
    seq_h = torch.arange(nq, dtype=torch.int32) % B
    got = csa.csa_index_scores(qI, w, K, pos, m, seq_of_q=seq_h.to(DEV))
    ref = oracle.index_scores(qI_h, w_h, K_h, pos_h, m, seq=seq_h)
    assert_scores_close(got, ref, score_bound(qI_h, w_h, K_h, pos_h, m, seq=seq_h))


# ---------------------------------------------------------------- a5
def _tie_scores(nq, ncols, seed):
    g = torch.Generator().manual_seed(seed)
    S = torch.randn(nq, ncols, generator=g)
    # force ties and signed zeros in some rows
    S[0] = torch.randint(-3, 4, (ncols,), generator=g).float()
    S[1, ::2] = 0.0
    S[1, 1::2] = -0.0
    S[2] = 1.5
    return S


# odd column counts: rows start off the 16-byte boundary (the row pass reads
# an unaligned head and tail one score at a time)
@pytest.mark.parametrize("ncols,k", [(100, 16), (5000, 512), (40000, 1024), (70000, 2048), (300000, 512),
                                     (10001, 512), (20003, 64)])
def test_topk_bitexact(csa, ncols, k):
    nq = 6
    S = _tie_scores(nq, ncols, ncols + k)
    valid = torch.tensor([ncols, ncols - 1, k - 1, 0, min(ncols, 3 * k + 7), ncols // 2], dtype=torch.int32)
    idx, top = csa.csa_topk_from_scores(S.to(DEV), k, valid=valid.to(DEV))
    ref = oracle.topk(S.double().numpy(), valid.numpy(), k)
    np.testing.assert_array_equal(host(idx), ref)
    want = np.where(ref >= 0, np.take_along_axis(S.numpy(), np.maximum(ref, 0), 1), -np.inf)
    np.testing.assert_array_equal(top.cpu().numpy(), want.astype(np.float32))


def test_topk_valid_div(csa):
    nq, ncols, k, m = 9, 3000, 64, 4
    S = torch.randn(nq, ncols)
    pos = torch.randint(0, ncols * m + 9, (nq,), dtype=torch.int32)
    idx, _ = csa.csa_topk_from_scores(S.to(DEV), k, valid=pos.to(DEV), valid_div=m)
    ref = oracle.topk(S.double().numpy(), np.minimum(pos.numpy() // m, ncols), k)
    np.testing.assert_array_equal(host(idx), ref)


def test_topk_rows_against_a_strided_sample(csa):
    """Rows built so that a strided sample misleads the estimate: the sampled
    positions hold the largest scores (too few candidates reach the estimate)
    or the smallest (too many). The selection must stay exact."""
    nq, ncols, k = 4, 50000, 512
    g = torch.Generator().manual_seed(5)
    S = torch.rand(nq, ncols, generator=g)
    for S_pos in (4096, 1024):
        pos = (torch.arange(S_pos, dtype=torch.int64) * ncols) // S_pos
        S[0, pos] += 10.0
        S[1, pos] -= 10.0
    S[2, ::97] += 10.0            # a regular stride unrelated to the sample's
    S[3] = torch.round(S[3] * 4) / 4   # heavy ties
    idx, top = csa.csa_topk_from_scores(S.to(DEV), k)
    ref = oracle.topk(S.double().numpy(), np.full(nq, ncols, dtype=np.int32), k)
    np.testing.assert_array_equal(host(idx), ref)


@pytest.mark.parametrize("score_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("ncols,k", [(20003, 512), (9000, 128)])
def test_topk_many_long_rows(csa, score_dtype, ncols, k):
    """More rows than SMs (one CTA per row), every row past the in-shared-
    memory limit, so every row goes through the sampled estimate and the
    filter pass; rows that mislead the estimate (too many or too few
    candidates) and heavy ties fall back to the exact selection on the whole
    row."""
    nq = 200
    g = torch.Generator().manual_seed(77)
    S = torch.randn(nq, ncols, generator=g)
    S[0] = torch.round(S[0] * 2) / 2              # heavy ties
    S[1, 1::2] = 0.0                              # signed zeros
    S[1, ::2] = -0.0
    pos = (torch.arange(4096, dtype=torch.int64) * ncols) // 4096
    S[2, pos] += 10.0                             # the sample sees only the largest
    S[3, pos] -= 10.0                             # the sample sees only the smallest
    S[4, 7::3] = 2.0                              # many equal scores above the k-th
    S = S.to(score_dtype)
    if score_dtype == torch.bfloat16:
        idx, top = csa.csa_topk_from_scores_bf16(S.to(DEV), k)
    else:
        idx, top = csa.csa_topk_from_scores(S.to(DEV), k)
    ref = oracle.topk(S.float().double().numpy(), np.full(nq, ncols, dtype=np.int32), k)
    np.testing.assert_array_equal(host(idx), ref)
    want = np.take_along_axis(S.float().numpy(), np.maximum(ref, 0), 1)
    np.testing.assert_array_equal(top.cpu().numpy(), want.astype(np.float32))


# ---------------------------------------------------------------- a4 + a5
@pytest.mark.parametrize("dtype", MODES)
def test_index_topk(csa, dtype):
    nq, HI, cI, B, Nmax, m, k = 24, 64, 128, 24, 3000, 4, 512
    qI_h, qI, K_h, K, w_h, w, pos_h, pos = _index_inputs(dtype, nq, HI, cI, B, Nmax, m, seed=11)
    idx, top = csa.csa_index_topk(qI, w, K, pos, m, k)
    ref_idx, S = oracle.index_topk(qI_h, w_h, K_h, pos_h, m, k, seq=torch.arange(nq))
    assert_topk_sets(idx, ref_idx, S, k)
    assert_topk_order(idx, S)
    sel = host(idx)
    for t in range(nq):
        s = sel[t][sel[t] >= 0]
        assert np.all(s < pos_h[t].item() // m)


@pytest.mark.parametrize("dtype", MODES)
def test_index_topk_query_on_a_missing_sequence_selects_nothing(csa, dtype):
    # a query whose sequence is outside [0, n_seq) sees no entry (csa.h): its
    # indexer row is never written, so the selection must not read it
    nq, HI, cI, B, Nmax, m, k = 6, 64, 128, 3, 2000, 4, 64
    qI_h, qI, K_h, K, w_h, w, _, _ = _index_inputs(dtype, nq, HI, cI, B, Nmax, m, seed=12)
    pos_h = torch.tensor([8000, 5000, 7999, 300, 8000, 64], dtype=torch.int32)
    seq_h = torch.tensor([0, 2, 3, 1, -1, 2], dtype=torch.int32)
    idx, _ = csa.csa_index_topk(qI, w, K, pos_h.to(DEV), m, k, seq_of_q=seq_h.to(DEV))
    sel = host(idx)
    assert np.all(sel[2] == -1) and np.all(sel[4] == -1)
    ok = [0, 1, 3, 5]
    ref_idx, S = oracle.index_topk(qI_h[ok], w_h[ok], K_h, pos_h[ok], m, k, seq=seq_h[ok])
    assert_topk_sets(idx[ok], ref_idx, S, k)


# ---------------------------------------------------------------- a6 / a7
@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("H,c,k", [(64, 512, 512), (8, 128, 16), (128, 512, 96)])
@pytest.mark.parametrize("with_sink", [False, True])
def test_sparse_mqa(csa, dtype, H, c, k, with_sink):
    nq, B, Nmax = 5, 3, 1500
    q_h, q = _g((nq, H, c), "q", dtype)
    KV_h, KV = _g((B, Nmax, c), "KV", dtype)
    g = torch.Generator().manual_seed(5)
    idx_h = torch.stack([torch.randperm(Nmax, generator=g)[:k] for _ in range(nq)]).to(torch.int32)
    idx_h[1, k // 3:] = -1          # a partly filled selection
    idx_h[2, :] = -1                # an empty selection
    seq_h = torch.tensor([0, 1, 2, 1, 0], dtype=torch.int32)
    sink_h = synth.normal((H,), 3, "sink", dtype=torch.float32) if with_sink else None
    out, lse = csa.csa_sparse_mqa(q, KV, idx_h.to(DEV), 0.0, sink=None if sink_h is None else sink_h.to(DEV),
                                  seq_of_q=seq_h.to(DEV))
    ref_o, ref_l = oracle.sparse_mqa(q_h, KV_h, idx_h, 1 / math.sqrt(c), sink=sink_h, seq=seq_h)
    assert_close(out, ref_o, dtype, "sparse_mqa out")
    assert_close(lse, ref_l, torch.float32 if dtype == torch.float32 else dtype, "sparse_mqa lse")


# (kind, queries, head dim, heads, k or visible entries): query counts chosen
# so that the KV of one query is split 2 ways (the two splits form a cluster
# and merge on chip) or 3, 4, 5, 6, 8 or 10 ways (every split writes fp32
# partials, merged in split order by the combine launch), some splits seeing
# no entry at all, with one and two head groups and head
# dims of 128 to 512. The split count of a launch is the SM count over the
# (query, head group) blocks, capped by the 128-entry tiles and then reduced
# to the count the tiles per split need.
SPLIT_CASES = [
    ("sparse", 40, 512, 64, 512),
    ("sparse", 40, 128, 64, 384),
    ("sparse", 24, 512, 128, 512),
    ("sparse", 20, 256, 64, 1024),     # 4 ways
    ("dense", 40, 512, 64, 700),
    ("dense", 20, 128, 64, 1100),      # 5 ways
    ("dense", 24, 512, 128, 700),      # two head groups, 3 ways
    ("dense", 40, 384, 64, 900),       # three 128-dim M tiles through the two rings
    ("sparse", 40, 384, 64, 512),
    ("sparse", 12, 512, 64, 1024),     # 8 ways
    ("sparse", 24, 512, 64, 768),      # 6 ways
    ("dense", 16, 256, 64, 1100),      # 5 ways, one head group
    ("dense", 8, 512, 64, 1100),       # 10 ways
    ("dense", 64, 512, 64, 700),       # 2 ways
    ("dense", 32, 256, 128, 1100),     # two head groups, 2 ways
]


@pytest.mark.parametrize("kind,nq,c,H,kv", SPLIT_CASES)
def test_mqa_split_merges(csa, kind, nq, c, H, kv):
    B, Nmax = 4, 1200
    q_h, q = _g((nq, H, c), "qs", torch.bfloat16)
    KV_h, KV = _g((B, Nmax, c), "KVs", torch.bfloat16)
    seq_h = (torch.arange(nq, dtype=torch.int32) % B)
    sink_h = synth.normal((H,), 4, "sink_s", dtype=torch.float32)
    if kind == "sparse":
        g = torch.Generator().manual_seed(9)
        idx_h = torch.stack([torch.randperm(Nmax, generator=g)[:kv] for _ in range(nq)]).to(torch.int32)
        idx_h[3, kv // 2:] = -1         # one split of this query sees nothing
        out, lse = csa.csa_sparse_mqa(q, KV, idx_h.to(DEV), 0.0, sink=sink_h.to(DEV), seq_of_q=seq_h.to(DEV))
        ref_o, ref_l = oracle.sparse_mqa(q_h, KV_h, idx_h, 1 / math.sqrt(c), sink=sink_h, seq=seq_h)
    else:
        mp = 4
        pos_h = torch.full((nq,), kv * mp + 1, dtype=torch.int32)
        pos_h[1] = 5 * mp               # few visible entries: most splits empty
        out, lse = csa.hca_dense_mqa(q, KV, pos_h.to(DEV), mp, 0.0, sink=sink_h.to(DEV), seq_of_q=seq_h.to(DEV))
        ref_o, ref_l = oracle.dense_mqa(q_h, KV_h, pos_h, mp, 1 / math.sqrt(c), sink=sink_h, seq=seq_h)
    assert_close(out, ref_o, torch.bfloat16, f"{kind} split out")
    assert_close(lse, ref_l, torch.bfloat16, f"{kind} split lse")


@pytest.mark.parametrize("dtype", MODES)
def test_dense_mqa(csa, dtype):
    nq, H, c, Nmax, mp = 4, 64, 512, 700, 128
    q_h, q = _g((nq, H, c), "qd", dtype)
    KV_h, KV = _g((nq, Nmax, c), "KVd", dtype)
    pos_h = torch.tensor([0, 127, 128 * 333 + 5, 128 * Nmax + 1000], dtype=torch.int32)
    out, lse = csa.hca_dense_mqa(q, KV, pos_h.to(DEV), mp, 0.0, seq_of_q=torch.arange(nq, dtype=torch.int32,
                                                                                         device=DEV))
    ref_o, ref_l = oracle.dense_mqa(q_h, KV_h, pos_h, mp, 1 / math.sqrt(c), seq=torch.arange(nq))
    assert_close(out, ref_o, dtype, "dense_mqa out")
    assert_close(lse, ref_l, dtype, "dense_mqa lse")


def test_sparse_with_all_visible_equals_dense(csa):
    # spec invariant on the GPU: top-k >= visible count -> CSA == dense MQA
    nq, H, c, Nmax, m = 3, 64, 512, 300, 4
    q_h, q = _g((nq, H, c), "qa", torch.bfloat16)
    KV_h, KV = _g((nq, Nmax, c), "KVa", torch.bfloat16)
    pos = torch.tensor([Nmax * m, 4 * 101 + 3, 4 * 17], dtype=torch.int32)
    idx = torch.full((nq, 512), -1, dtype=torch.int32)
    for t in range(nq):
        v = pos[t].item() // m
        idx[t, :v] = torch.arange(v - 1, -1, -1, dtype=torch.int32)
    seq = torch.arange(nq, dtype=torch.int32, device=DEV)
    o1, l1 = csa.csa_sparse_mqa(q, KV, idx.to(DEV), seq_of_q=seq)
    o2, l2 = csa.hca_dense_mqa(q, KV, pos.to(DEV), m, seq_of_q=seq)
    assert_close(o1, host(o2), torch.bfloat16, "sparse vs dense")
    assert_close(l1, host(l2), torch.bfloat16, "sparse vs dense lse")


# ---------------------------------------------------------------- fused
@pytest.mark.parametrize("dtype", MODES)
def test_csa_decode_scaled_flash(csa, dtype):
    s = synth.FLASH_DECODE.scale_ctx(16)           # ctx 4K..8K -> <= 2048 entries, same heads/dims
    inp = synth.decode_inputs(s, device="cpu", batch=12)
    cast = (lambda t: t.to(dtype)) if dtype == torch.float32 else (lambda t: t)
    dev = {k: (cast(v).to(DEV) if v.dtype == torch.bfloat16 else v.to(DEV)) for k, v in inp.items()}
    k = 512
    out, lse, sel = csa.csa_decode(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], dev["kv_cache"], dev["ctx_len"],
                                   s.m, k, return_topk=True)
    B = inp["q"].shape[0]
    seq = torch.arange(B)
    ref_idx, S = oracle.index_topk(inp["qI"], inp["w"], inp["idx_cache"], inp["ctx_len"], s.m, k, seq=seq)
    assert_topk_sets(sel, ref_idx, S, k)
    ref_o, ref_l = oracle.sparse_mqa(inp["q"], inp["kv_cache"], host(sel).astype(np.int32), 1 / math.sqrt(s.c),
                                     seq=seq)
    assert_close(out, ref_o, dtype, "csa_decode out")
    assert_close(lse, ref_l, dtype, "csa_decode lse")


@pytest.mark.parametrize("dtype", MODES)
def test_hca_decode_scaled(csa, dtype):
    s = synth.HCA
    inp = synth.hca_decode_inputs(s, batch=4, n_max=900)
    inp["ctx_len"][1] = 128 * 450 + 77
    inp["ctx_len"][2] = 100
    cast = (lambda t: t.to(dtype)) if dtype == torch.float32 else (lambda t: t)
    out, lse = csa.hca_decode(cast(inp["q"]).to(DEV), cast(inp["kv_cache"]).to(DEV), inp["ctx_len"].to(DEV), s.mp)
    ref_o, ref_l = oracle.dense_mqa(inp["q"], inp["kv_cache"], inp["ctx_len"], s.mp, 1 / math.sqrt(s.c),
                                    seq=torch.arange(4))
    assert_close(out, ref_o, dtype, "hca_decode out")
    assert_close(lse, ref_l, dtype, "hca_decode lse")


def _prefill_oracle(inp, s, k):
    """Oracle chain for one prefill chunk: compress both streams into copies of
    the caches (bf16 storage rounding when the caches are bf16), then indexer,
    top-k and MQA for every new token."""
    m, start, n = s.m, inp["start"], inp["n"]
    bf = inp["kv_cache"].dtype == torch.bfloat16
    rnd = oracle.bf16_round if bf else (lambda a: a)
    kv = oracle._f64(inp["kv_cache"]).copy()
    ik = oracle._f64(inp["idx_cache"]).copy()
    kv[start // m:(start + n) // m] = rnd(oracle.csa_compress_from_hidden(inp["x"], inp["W_kv"], inp["B_kv"], m,
                                                                          X_left=inp["x_left"]))
    ik[start // m:(start + n) // m] = rnd(oracle.csa_compress_from_hidden(inp["x"], inp["W_idx"], inp["B_idx"], m,
                                                                          X_left=inp["x_left"]))
    pos = np.arange(start, start + n, dtype=np.int32)
    ref_idx, S = oracle.index_topk(inp["qI"], inp["w"], ik, pos, m, k)
    return kv, ik, ref_idx, S


@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("start", [0, 256])
def test_csa_prefill_tiny(csa, dtype, start):
    s = synth.TINY
    inp = synth.prefill_inputs(s, start=start, n=512 if start else None)
    if dtype == torch.float32:
        inp = {k: (v.float() if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else v)
               for k, v in inp.items()}
    dev = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse, sel = csa.csa_prefill(dev["x"], dev["x_left"], dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"],
                                    inp["start"], dev["kv_cache"], dev["idx_cache"], dev["qI"], dev["w"], dev["q"],
                                    s.k, m=s.m, return_topk=True)
    kv, ik, ref_idx, S = _prefill_oracle(inp, s, s.k)
    e0, e1 = inp["start"] // s.m, (inp["start"] + inp["n"]) // s.m
    assert_close(dev["kv_cache"][e0:e1], kv[e0:e1], dtype, "prefill kv cache")
    assert_close(dev["idx_cache"][e0:e1], ik[e0:e1], dtype, "prefill idx cache")
    assert_topk_sets(sel, ref_idx, S, s.k)
    ref_o, ref_l = oracle.sparse_mqa(inp["q"], kv, host(sel).astype(np.int32), 1 / math.sqrt(s.c))
    assert_close(out, ref_o, dtype, "prefill out")
    # queries at positions < m see nothing: zero output, lse = -inf
    if inp["start"] == 0:
        assert torch.all(out[: s.m] == 0) and torch.all(torch.isneginf(lse[: s.m]))


def test_prefill_chunked_equals_whole(csa):
    # composition: two chunks (the second with the m hidden rows before it as
    # left context) give the same caches and outputs as one chunk
    s = synth.TINY
    inp = synth.prefill_inputs(s)
    dev = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    kv1, ik1 = dev["kv_cache"].clone(), dev["idx_cache"].clone()
    o1, _ = csa.csa_prefill(dev["x"], None, dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"], 0, kv1, ik1,
                            dev["qI"], dev["w"], dev["q"], s.k, m=s.m)
    kv2, ik2 = dev["kv_cache"].clone(), dev["idx_cache"].clone()
    a = 384
    o2a, _ = csa.csa_prefill(dev["x"][:a], None, dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"], 0, kv2, ik2,
                             dev["qI"][:a], dev["w"][:a], dev["q"][:a], s.k, m=s.m)
    o2b, _ = csa.csa_prefill(dev["x"][a:], dev["x"][a - s.m:a].contiguous(), dev["W_kv"], dev["B_kv"], dev["W_idx"],
                             dev["B_idx"], a, kv2, ik2, dev["qI"][a:], dev["w"][a:], dev["q"][a:], s.k, m=s.m)
    torch.testing.assert_close(kv1, kv2, rtol=0, atol=0)
    torch.testing.assert_close(ik1, ik2, rtol=0, atol=0)
    torch.testing.assert_close(o1, torch.cat([o2a, o2b]), rtol=0, atol=0)


def test_decode_equals_last_prefill_row(csa):
    # a decode query at position p over the caches equals the prefill output
    # of the token at position p (same qI, w, q)
    s = synth.TINY
    inp = synth.prefill_inputs(s)
    dev = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, _, sel = csa.csa_prefill(dev["x"], None, dev["W_kv"], dev["B_kv"], dev["W_idx"], dev["B_idx"], 0,
                                  dev["kv_cache"], dev["idx_cache"], dev["qI"], dev["w"], dev["q"], s.k, m=s.m,
                                  return_topk=True)
    for p in (1023, 700, 4):
        o, _, dsel = csa.csa_decode(dev["qI"][p:p + 1].contiguous(), dev["w"][p:p + 1].contiguous(),
                                    dev["idx_cache"][None], dev["q"][p:p + 1].contiguous(), dev["kv_cache"][None],
                                    torch.tensor([p], dtype=torch.int32, device=DEV), s.m, s.k, return_topk=True)
        torch.testing.assert_close(dsel[0], sel[p], rtol=0, atol=0)
        torch.testing.assert_close(o[0], out[p], rtol=0, atol=0)


def test_errors_surface_as_exceptions(csa):
    x = torch.zeros(6, 32, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(csa.CsaError) as e:
        csa.csa_compress(x, torch.zeros(8, 8, device=DEV), 4)
    assert e.value.code == csa.CSA_ERR_INVALID_ARG
    csa.poll_status()


def test_indexer_wait_timeout_is_reported_and_the_next_call_is_correct(csa):
    # the failure path of the bounded device waits [failure detection without
    # a fault]: the indexer is made to wait for a key tile that is never
    # loaded, with a short wait bound; the kernel must return, the status word
    # must say CSA_ERR_TIMEOUT, and the context must stay usable
    nq, HI, cI, B, Nmax, m = 8, 64, 128, 8, 4000, 4
    qI_h, qI, K_h, K, w_h, w, pos_h, pos = _index_inputs(torch.bfloat16, nq, HI, cI, B, Nmax, m, seed=13)
    csa.poll_status()                                   # start from a clean word
    csa.debug_set(4096, csa.CSA_DEBUG_SKIP_FIRST_TILE)
    try:
        csa.csa_index_scores(qI, w, K, pos, m)
        torch.cuda.synchronize()                        # the kernel returned
    finally:
        csa.debug_set(0, 0)
    with pytest.raises(csa.CsaError) as e:
        csa.poll_status()
    assert e.value.code == csa.CSA_ERR_TIMEOUT
    csa.poll_status()                                   # the word was reset
    got = csa.csa_index_scores(qI, w, K, pos, m)
    ref = oracle.index_scores(qI_h, w_h, K_h, pos_h, m, seq=torch.arange(nq))
    assert_scores_close(got, ref, score_bound(qI_h, w_h, K_h, pos_h, m, seq=torch.arange(nq)))
