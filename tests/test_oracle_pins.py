"""Pins for the CPU oracle: checks against facts fixed by the pages and by
mathematics, never against the oracle itself or the CUDA path.

Kinds of pin used here:
  * hand-worked examples in tests/golden/ (values chosen so every softmax
    weight is a simple fraction, derivation written in the fixture);
  * closed forms (uniform weights give the window mean, m'=1 gives identity);
  * invariants (weights sum to 1, causality, chunked composition);
  * reductions to a library routine (numpy matmul, torch's attention);
  * brute force over every k-subset for top-k.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _num(v):
    """Parse the fixture notation: numbers, 'ln3', 'ln3+0.5', '6/7', '-inf'."""
    if v is None:
        return None
    if isinstance(v, (int, float)):
        return float(v)
    s = v.strip()
    if s == "-inf":
        return -math.inf
    if "/" in s:
        a, b = s.split("/")
        return float(a) / float(b)
    total = 0.0
    for sign, term in _terms(s):
        total += sign * (math.log(float(term[2:])) if term.startswith("ln") else float(term))
    return total


def _terms(s):
    out, sign, cur = [], 1.0, ""
    for ch in s:
        if ch in "+-" and cur:
            out.append((sign, cur))
            sign, cur = (1.0 if ch == "+" else -1.0), ""
        elif ch == "-" and not cur:
            sign = -sign
        else:
            cur += ch
    out.append((sign, cur))
    return out


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


rng = np.random.default_rng(12345)


# --------------------------------------------------------------------------
# bf16 storage rounding
# --------------------------------------------------------------------------

def test_bf16_round_matches_torch_on_fp32_values():
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # fp32 subnormals
        (rng.standard_normal(2000) * 1e38).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 3.4e38], dtype=np.float32),
    ])
    # exact ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> even (1.0)
    ties = np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 2**-130 + 2**-134], dtype=np.float32)
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = oracle.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_bf16_round_ties_to_even_by_hand():
    assert oracle.bf16_round(np.array([1 + 2**-8]))[0] == 1.0
    assert oracle.bf16_round(np.array([1 + 3 * 2**-8]))[0] == 1 + 2**-6
    assert oracle.bf16_round(np.array([1 + 2**-8 + 2**-20]))[0] == 1 + 2**-7


# --------------------------------------------------------------------------
# a1 projections
# --------------------------------------------------------------------------

def test_project_loops_match_library_matmul():
    X = rng.standard_normal((37, 53))
    W = rng.standard_normal((19, 53))
    np.testing.assert_allclose(oracle.project_loops(X, W), X @ W.T, rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(oracle.project(X, W), oracle.project_loops(X, W), rtol=1e-13, atol=1e-12)
    # by hand: [1, 2] . [3, 4] = 11, [1, 2] . [-1, 0.5] = 0
    np.testing.assert_array_equal(oracle.project_loops([[1.0, 2.0]], [[3.0, 4.0], [-1.0, 0.5]]), [[11.0, 0.0]])


# --------------------------------------------------------------------------
# a2 CSA compressor
# --------------------------------------------------------------------------

def _csa_fixture():
    g = _load("csa_compress_m2.json")
    cols = [[_num(v) for v in g[k]] for k in ("Ca", "Cb", "Za", "Zb")]
    proj = np.array(cols).T  # [n, 4] with c = 1
    bias = np.array([[_num(v) for v in r] for r in g["bias"]])
    return g, proj, bias


def test_csa_compress_handworked():
    g, proj, bias = _csa_fixture()
    out = oracle.csa_compress(proj, bias, g["m"])
    np.testing.assert_allclose(out[:, 0], g["expected"], rtol=0, atol=1e-12)


def test_csa_compress_handworked_with_left_context():
    g, proj, bias = _csa_fixture()
    m = g["m"]
    out = oracle.csa_compress(proj[m:], bias, m, left=proj[:m])
    np.testing.assert_allclose(out[:, 0], g["expected_second_block_alone_with_left_context"],
                               rtol=0, atol=1e-12)


def test_csa_uniform_weights_give_window_mean():
    # Z = const and B = 0 make every softmax weight equal; with Ca = Cb = C the
    # compressed entry is the plain mean of C over the window: 2m tokens, or
    # m tokens for block 0 (no b-window at the start of a sequence).
    m, c, n = 4, 6, 40
    C = rng.standard_normal((n, c))
    Z = np.full((n, c), 0.37)
    proj = np.concatenate([C, C, Z, Z], axis=1)
    out = oracle.csa_compress(proj, np.zeros((2 * m, c)), m)
    want = np.stack([C[0:m].mean(0)] + [C[m * (i - 1): m * (i + 1)].mean(0) for i in range(1, n // m)])
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-13)


def test_csa_weights_sum_to_one_and_block0_has_no_b_window():
    m, c, n = 4, 16, 64
    proj = rng.standard_normal((n, 4 * c)) * 3
    bias = rng.standard_normal((2 * m, c))
    out, w = oracle.csa_compress(proj, bias, m, return_weights=True)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(w[0, m:, :] == 0.0)
    assert np.all(w[1:, m:, :] > 0.0)
    # with a left context the first block does have a b-window
    _, w2 = oracle.csa_compress(proj[m:], bias, m, left=proj[:m], return_weights=True)
    assert np.all(w2[0, m:, :] > 0.0)


def test_csa_with_b_logits_at_minus_inf_is_non_overlapping():
    # Z^b -> -inf removes the b-window: each entry is then the softmax(Za + Ba)
    # average of its own m tokens, which is the HCA form with m' = m.
    m, c, n = 4, 8, 32
    Ca, Cb, Za = (rng.standard_normal((n, c)) for _ in range(3))
    Zb = np.full((n, c), -1e300)
    bias = rng.standard_normal((2 * m, c))
    out = oracle.csa_compress(np.concatenate([Ca, Cb, Za, Zb], 1), bias, m)
    want = np.empty((n // m, c))
    for i in range(n // m):
        lg = Za[m * i: m * i + m] + bias[:m]
        e = np.exp(lg - lg.max(0))
        want[i] = (e / e.sum(0) * Ca[m * i: m * i + m]).sum(0)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)
    hca = oracle.hca_compress(np.concatenate([Ca, Za], 1), bias[:m], m)
    np.testing.assert_allclose(out, hca, rtol=1e-12, atol=1e-13)


def test_csa_chunked_composition():
    # compress(0..n) == compress(0..a) ++ compress(a..n with the m rows before a)
    m, c, n = 4, 8, 96
    proj = rng.standard_normal((n, 4 * c))
    bias = rng.standard_normal((2 * m, c))
    full = oracle.csa_compress(proj, bias, m)
    for a in (4, 28, 60, 92):
        head = oracle.csa_compress(proj[:a], bias, m)
        tail = oracle.csa_compress(proj[a:], bias, m, left=proj[a - m: a])
        np.testing.assert_array_equal(np.concatenate([head, tail]), full)


def test_csa_from_hidden_is_projection_then_compression():
    m, c, d, n = 4, 4, 24, 16
    X = rng.standard_normal((n, d))
    W = rng.standard_normal((4 * c, d))
    bias = rng.standard_normal((2 * m, c))
    got = oracle.csa_compress_from_hidden(X, W, bias, m)
    np.testing.assert_allclose(got, oracle.csa_compress(X @ W.T, bias, m), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# a3 HCA compressor
# --------------------------------------------------------------------------

def test_hca_compress_handworked():
    g = _load("hca_compress_mp2.json")
    C = np.array([[_num(v) for v in r] for r in g["C"]])
    Z = np.array([[_num(v) for v in r] for r in g["Z"]])
    bias = np.array(g["bias"], dtype=float)
    out = oracle.hca_compress(np.concatenate([C, Z], 1), bias, g["mp"])
    np.testing.assert_allclose(out, np.array(g["expected"]), rtol=0, atol=1e-12)


def test_hca_mp1_is_identity():
    n, c = 20, 7
    C = rng.standard_normal((n, c))
    Z = rng.standard_normal((n, c))
    out = oracle.hca_compress(np.concatenate([C, Z], 1), np.zeros((1, c)), 1)
    np.testing.assert_array_equal(out, C)


def test_hca_uniform_weights_give_block_mean_and_weights_sum_to_one():
    mp, c, n = 128, 4, 512
    C = rng.standard_normal((n, c))
    out = oracle.hca_compress(np.concatenate([C, np.zeros((n, c))], 1), np.zeros((mp, c)), mp)
    np.testing.assert_allclose(out, C.reshape(n // mp, mp, c).mean(1), rtol=1e-12, atol=1e-13)
    proj = rng.standard_normal((n, 2 * c)) * 4
    _, w = oracle.hca_compress(proj, rng.standard_normal((mp, c)), mp, return_weights=True)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)


def test_entry_counts_match_the_pages():
    g = _load("entry_counts.json")
    n = g["tokens"]
    # the oracle emits n/m entries per sequence; use a proportionally small run
    # to confirm the count rule, then apply it at the pages' size
    assert oracle.csa_compress(np.zeros((64, 4)), np.zeros((8, 1)), 4).shape[0] == 64 // 4
    assert oracle.hca_compress(np.zeros((256, 2)), np.zeros((128, 1)), 128).shape[0] == 256 // 128
    assert n // g["m"] == g["expected_csa_entries"]
    assert abs(n / g["mp"] - g["expected_hca_entries_approx"]) <= g["hca_tolerance_fraction"] * n / g["mp"]


# --------------------------------------------------------------------------
# a4 indexer + a5 top-k
# --------------------------------------------------------------------------

def _indexer_fixture():
    g = _load("indexer_topk.json")
    K = np.array(g["K"], dtype=float)
    npos = len(g["pos"])
    q = np.broadcast_to(np.array(g["q"], dtype=float), (npos, 2, 2)).copy()
    w = np.broadcast_to(np.array(g["w"], dtype=float), (npos, 2)).copy()
    return g, K, q, w


def test_indexer_handworked():
    g, K, q, w = _indexer_fixture()
    S = oracle.index_scores(q, w, K, g["pos"], g["m"])
    want = np.array([[_num(v) for v in r] for r in g["expected_scores"]])
    np.testing.assert_array_equal(S, want)


def test_topk_handworked():
    g, K, q, w = _indexer_fixture()
    idx, _ = oracle.index_topk(q, w, K, g["pos"], g["m"], g["k"])
    np.testing.assert_array_equal(idx, np.array(g["expected_topk"]))


def test_indexer_single_head_unit_weight_is_relu_dot():
    nq, cI, N, m = 9, 32, 50, 4
    q = rng.standard_normal((nq, 1, cI))
    K = rng.standard_normal((N, cI))
    pos = np.full(nq, N * m)
    S = oracle.index_scores(q, np.ones((nq, 1)), K, pos, m)
    np.testing.assert_allclose(S, np.maximum(q[:, 0, :] @ K.T, 0.0), rtol=1e-13, atol=1e-13)


def test_indexer_is_linear_in_head_weights():
    nq, H, cI, N, m = 5, 4, 16, 40, 4
    q = rng.standard_normal((nq, H, cI))
    K = rng.standard_normal((N, cI))
    pos = np.full(nq, N * m)
    w = rng.random((nq, H))
    total = oracle.index_scores(q, w, K, pos, m)
    parts = sum(oracle.index_scores(q, np.eye(H)[h][None].repeat(nq, 0), K, pos, m) * w[:, h:h + 1]
                for h in range(H))
    np.testing.assert_allclose(total, parts, rtol=1e-12, atol=1e-12)


def test_indexer_causality():
    # a query at position p must not depend on any entry s >= floor(p/m)
    nq, H, cI, N, m = 12, 3, 8, 32, 4
    q = rng.standard_normal((nq, H, cI))
    w = rng.random((nq, H))
    K = rng.standard_normal((N, cI))
    pos = rng.integers(0, N * m, nq)
    S1 = oracle.index_scores(q, w, K, pos, m)
    for t in range(nq):
        v = pos[t] // m
        assert np.all(np.isinf(S1[t, v:])) and np.all(np.isfinite(S1[t, :v]))
        K2 = K.copy()
        K2[v:] = rng.standard_normal((N - v, cI)) * 100
        S2 = oracle.index_scores(q[t:t + 1], w[t:t + 1], K2, pos[t:t + 1], m)
        np.testing.assert_array_equal(S2[0], S1[t])
    idx, _ = oracle.index_topk(q, w, K, pos, m, k=40)
    for t in range(nq):
        sel = idx[t][idx[t] >= 0]
        assert np.all(sel < pos[t] // m)
        assert len(sel) == min(40, pos[t] // m)


def _brute_topk(row, v, k):
    kk = min(k, v)
    best, best_key = (), None
    for sub in itertools.combinations(range(v), kk):
        key = (sum(row[list(sub)]) if sub else 0.0, tuple(-s for s in sub))
        if best_key is None or key > best_key:
            best, best_key = sub, key
    ordered = sorted(best, key=lambda s: (-row[s], s))
    return ordered + [-1] * (k - kk)


def test_topk_brute_force_with_ties():
    # integer scores from a small range force many ties; the brute force takes
    # the max-sum k-subset and, among equal sums, the lexicographically smallest
    # index set, then orders it (score desc, index asc)
    for trial in range(300):
        V = int(rng.integers(0, 11))
        ncols = V + int(rng.integers(0, 3))
        k = int(rng.integers(1, 5))
        row = rng.integers(-3, 4, ncols).astype(float)
        got = oracle.topk(row[None], [V], k)[0]
        assert list(got) == _brute_topk(row, V, k), (row, V, k)


def test_topk_matches_library_sort():
    S = rng.standard_normal((20, 3000))
    valid = rng.integers(0, 3001, 20)
    k = 512
    idx = oracle.topk(S, valid, k)
    for t in range(20):
        v = valid[t]
        order = np.lexsort((np.arange(v), -S[t, :v]))[:k]
        want = np.full(k, -1)
        want[: len(order)] = order
        np.testing.assert_array_equal(idx[t], want)


# --------------------------------------------------------------------------
# a6 / a7 shared-KV MQA
# --------------------------------------------------------------------------

def test_mqa_handworked_with_sink():
    g = _load("mqa_sink.json")
    KV = np.array(g["KV"], dtype=float)
    q = np.array([[[_num(v) for v in g["q"]]]])
    for case in g["cases"]:
        sink = None if case["sink"] is None else np.array([_num(case["sink"])])
        out, lse = oracle.sparse_mqa(q, KV, np.array([case["idx"]]), 1.0, sink=sink)
        np.testing.assert_allclose(out[0, 0], [_num(v) for v in case["out"]], rtol=0, atol=1e-14)
        want_lse = _num(case["lse"])
        if math.isinf(want_lse):
            assert lse[0, 0] == want_lse
        else:
            assert abs(lse[0, 0] - want_lse) < 1e-14


def test_mqa_single_entry_returns_that_entry():
    H, c, N = 4, 32, 10
    q = rng.standard_normal((3, H, c))
    KV = rng.standard_normal((N, c))
    idx = np.array([[7, -1, -1], [-1, 2, -1], [-1, -1, 0]])
    out, _ = oracle.sparse_mqa(q, KV, idx, 0.125)
    for t, s in enumerate((7, 2, 0)):
        np.testing.assert_array_equal(out[t], np.broadcast_to(KV[s], (H, c)))


def test_mqa_matches_torch_attention():
    # shared-KV MQA over a set of entries is standard attention with one KV
    # head and a boolean mask; torch's scaled_dot_product_attention in fp64
    nq, H, c, N = 6, 4, 16, 30
    q = rng.standard_normal((nq, H, c))
    KV = rng.standard_normal((N, c))
    idx = np.stack([rng.permutation(N)[:8] for _ in range(nq)]).astype(np.int32)
    idx[0, 3:] = -1
    scale = 1.0 / math.sqrt(c)
    out, lse = oracle.sparse_mqa(q, KV, idx, scale)
    mask = np.zeros((nq, N), dtype=bool)
    for t in range(nq):
        mask[t, idx[t][idx[t] >= 0]] = True
    qt = torch.from_numpy(q).transpose(0, 1)[:, :, None, :]          # [H, nq, 1, c]
    kt = torch.from_numpy(KV)[None, None].expand(H, nq, N, c)         # [H, nq, N, c]
    mt = torch.from_numpy(mask)[None, :, None, :].expand(H, nq, 1, N)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=mt, scale=scale)
    np.testing.assert_allclose(out, ref[:, :, 0, :].transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)
    logits = torch.einsum("thc,nc->thn", torch.from_numpy(q), torch.from_numpy(KV)) * scale
    logits = logits.masked_fill(~torch.from_numpy(mask)[:, None, :], -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_sparse_with_k_at_least_visible_equals_dense():
    # with top-k >= the visible count CSA's selection keeps every visible entry,
    # and sparse MQA equals dense MQA over all of them
    nq, HI, cI, H, c, N, m = 8, 4, 16, 4, 32, 40, 4
    qI = rng.standard_normal((nq, HI, cI))
    w = rng.random((nq, HI))
    K = rng.standard_normal((N, cI))
    KV = rng.standard_normal((N, c))
    q = rng.standard_normal((nq, H, c))
    pos = rng.integers(0, N * m, nq)
    idx, _ = oracle.index_topk(qI, w, K, pos, m, k=N)
    sp, lse_s = oracle.sparse_mqa(q, KV, idx, 0.2)
    de, lse_d = oracle.dense_mqa(q, KV, pos, m, 0.2)
    np.testing.assert_allclose(sp, de, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_s, lse_d, rtol=1e-12, atol=1e-12)


def test_sink_scales_output_below_one():
    # with a sink the attention weights sum to D / (D + e^{z'}) < 1:
    # out_sink = out * e^{lse} / (e^{lse} + e^{z'}),  lse_sink = log(e^{lse} + e^{z'})
    nq, H, c, N = 4, 3, 16, 12
    q = rng.standard_normal((nq, H, c))
    KV = rng.standard_normal((N, c))
    idx = np.tile(np.arange(N, dtype=np.int32), (nq, 1))
    sink = rng.standard_normal(H)
    o0, l0 = oracle.sparse_mqa(q, KV, idx, 0.3)
    o1, l1 = oracle.sparse_mqa(q, KV, idx, 0.3, sink=sink)
    frac = np.exp(l0) / (np.exp(l0) + np.exp(sink)[None])
    assert np.all(frac < 1.0)
    np.testing.assert_allclose(o1, o0 * frac[..., None], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, np.logaddexp(l0, sink[None]), rtol=1e-12, atol=1e-12)


def test_dense_mqa_causality_and_empty():
    H, c, N, mp = 2, 8, 6, 128
    q = rng.standard_normal((3, H, c))
    KV = rng.standard_normal((N, c))
    pos = np.array([0, 127, 128 * 3 + 5])
    out, lse = oracle.dense_mqa(q, KV, pos, mp, 0.5)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    want, _ = oracle.sparse_mqa(q[2:], KV, np.array([[0, 1, 2]]), 0.5)
    np.testing.assert_allclose(out[2], want[0], rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# Attention output completion: q/KV RMSNorm, partial rotary encoding with the
# output's back-rotation, the sliding-window branch in the same softmax
# (DeepSeek-V4 walk-through §2.3.3 items 1-3; study notes §1.3)
# --------------------------------------------------------------------------

def test_rmsnorm_closed_form():
    # x = (3, 4, 0, 0): mean of squares 25/4, root 5/2 -> (6/5, 8/5, 0, 0)
    x = np.array([[3.0, 4.0, 0.0, 0.0]])
    y = oracle.norm_rope(x, [0], gamma=np.ones(4), eps=0.0, rope_dims=0)
    np.testing.assert_allclose(y, [[1.2, 1.6, 0.0, 0.0]], rtol=0, atol=1e-15)
    y = oracle.norm_rope(x, [0], gamma=np.array([1.0, 2.0, 3.0, 4.0]), eps=0.0, rope_dims=0)
    np.testing.assert_allclose(y, [[1.2, 3.2, 0.0, 0.0]], rtol=0, atol=1e-15)
    # eps = 7/4 moves the denominator to sqrt(25/4 + 7/4) = sqrt(8)
    y = oracle.norm_rope(x, [0], gamma=np.ones(4), eps=1.75, rope_dims=0)
    np.testing.assert_allclose(y, x / math.sqrt(8.0), rtol=0, atol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = rng.standard_normal((5, 3, 64))
    y = oracle.norm_rope(x, np.arange(5), gamma=np.ones(64), eps=0.0, rope_dims=0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(-1)), 1.0, rtol=1e-14)
    y2 = oracle.norm_rope(7.5 * x, np.arange(5), gamma=np.ones(64), eps=0.0, rope_dims=0)
    np.testing.assert_allclose(y2, y, rtol=1e-13, atol=1e-14)


def test_rope_closed_form_pairs_and_frequencies():
    # c = 8, R = 4: the pairs are channels (4,5) and (6,7) with frequencies
    # 10000^0 = 1 and 10000^(-2/4) = 0.01; at position 50 they turn by 50 and
    # 0.5 radians. A unit vector on channel 4 goes to (cos 50, sin 50); one on
    # channel 7 to (-sin 0.5, cos 0.5); channels 0-3 do not move.
    x = np.zeros((1, 8))
    x[0, 4] = 1.0
    x[0, 7] = 1.0
    x[0, 1] = 2.0
    y = oracle.norm_rope(x, [50], rope_dims=4)
    want = [0, 2.0, 0, 0, math.cos(50.0), math.sin(50.0), -math.sin(0.5), math.cos(0.5)]
    np.testing.assert_allclose(y[0], want, rtol=0, atol=1e-13)


def test_rope_is_complex_multiplication():
    # the rotation of each pair is multiplication of a + ib by exp(i p theta)
    c, R, base = 32, 16, 10000.0
    x = rng.standard_normal((6, c))
    pos = rng.integers(0, 1 << 20, 6)
    y = oracle.norm_rope(x, pos, rope_dims=R, base=base)
    z = x[:, c - R::2] + 1j * x[:, c - R + 1::2]
    theta = base ** (-np.arange(R // 2) * 2.0 / R)
    z = z * np.exp(1j * pos[:, None] * theta[None])
    np.testing.assert_allclose(y[:, c - R::2], z.real, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(y[:, c - R + 1::2], z.imag, rtol=1e-9, atol=1e-9)
    np.testing.assert_array_equal(y[:, :c - R], x[:, :c - R])


def test_rope_relative_position_and_inverse():
    c, R = 64, 64
    q = rng.standard_normal((1, c))
    k = rng.standard_normal((1, c))
    for p, s in ((1000, 10), (131072, 131000), (7, 7)):
        lhs = (oracle.norm_rope(q, [p], rope_dims=R) @ oracle.norm_rope(k, [s], rope_dims=R).T).item()
        rhs = (oracle.norm_rope(q, [p - s], rope_dims=R) @ k.T).item()
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(rhs))
    x = rng.standard_normal((4, 2, c))
    pos = np.array([0, 5, 1 << 19, 1 << 20])
    back = oracle.norm_rope(oracle.norm_rope(x, pos, rope_dims=R), pos, rope_dims=R, inverse=True)
    np.testing.assert_allclose(back, x, rtol=1e-9, atol=1e-9)


def test_rope_heads_of_a_query_share_its_position():
    # rows of one query are its heads: each is normalised on its own and
    # turned by the query's position, as a one-row call on that head gives
    x = rng.standard_normal((3, 4, 16))
    pos = np.array([3, 99, 12345])
    g = rng.random(16) + 0.5
    y = oracle.norm_rope(x, pos, gamma=g, rope_dims=8)
    for t in range(3):
        for h in range(4):
            one = oracle.norm_rope(x[t, h][None], [pos[t]], gamma=g, rope_dims=8)[0]
            np.testing.assert_array_equal(y[t, h], one)


def _ring_after(tokens_kv, n_tokens, ring_len):
    """Window ring of one sequence after tokens 0..n_tokens-1 were written in
    order, token tau overwriting row tau mod ring_len."""
    ring = np.zeros((ring_len, tokens_kv.shape[1]))
    for tau in range(n_tokens):
        ring[tau % ring_len] = tokens_kv[tau]
    return ring


@pytest.mark.parametrize("n_win,ring_len", [(8, 8), (8, 13), (1, 4)])
def test_window_branch_is_banded_causal_attention(n_win, ring_len):
    # With no compressed entry selected, the branch is plain causal attention
    # restricted to the last n_win tokens (itself included), computed here by
    # torch over the token-ordered rows with a band mask.
    T, H, c = 30, 3, 16
    tok = rng.standard_normal((T, c))
    qs = rng.standard_normal((T, H, c))
    scale = 0.25
    band = np.tril(np.ones((T, T), dtype=bool)) & ~np.tril(np.ones((T, T), dtype=bool), -n_win)
    qt = torch.from_numpy(qs).transpose(0, 1)[:, :, None, :]
    kt = torch.from_numpy(tok)[None, None].expand(H, T, T, c)
    mt = torch.from_numpy(band)[None, :, None, :].expand(H, T, 1, T)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=mt, scale=scale)
    ref = ref[:, :, 0, :].transpose(0, 1).numpy()
    Nmax = 5                                     # compressed rows before the ring
    for p in range(T):
        cache = np.concatenate([rng.standard_normal((Nmax, c)), _ring_after(tok, p + 1, ring_len)])
        ent = oracle.window_entries([p], n_win, Nmax, ring_len)
        out, _ = oracle.sparse_mqa(qs[p][None], cache, ent, scale)
        np.testing.assert_allclose(out[0], ref[p], rtol=1e-12, atol=1e-12)


def test_window_joins_the_selection_in_one_softmax():
    # one softmax over selected entries + window rows equals the merge of the
    # two partial softmaxes by their log-sum-exp (sink counted once); two
    # separately normalised branches would not
    H, c, N = 4, 16, 40
    q = rng.standard_normal((3, H, c))
    KV = rng.standard_normal((N, c))
    sel = np.array([[1, 5, 9, -1], [0, 2, -1, -1], [3, 4, 6, 7]], dtype=np.int32)
    win = oracle.window_entries([2, 40, 70], 6, 30, 10)
    sink = rng.standard_normal(H)
    o, l = oracle.sparse_mqa(q, KV, np.concatenate([sel, win], 1), 0.3, sink=sink)
    o1, l1 = oracle.sparse_mqa(q, KV, sel, 0.3)
    o2, l2 = oracle.sparse_mqa(q, KV, win, 0.3)
    den = np.exp(l1) + np.exp(l2) + np.exp(sink)[None]
    want = (np.exp(l1)[..., None] * o1 + np.exp(l2)[..., None] * o2) / den[..., None]
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, np.log(den), rtol=1e-12, atol=1e-12)
    assert not np.allclose(o, 0.5 * (o1 + o2))


def test_back_rotated_output_depends_only_on_relative_positions():
    # KV rows rotated at their positions, the query rotated at p, the output
    # turned back by p: shifting every position by the same amount changes
    # nothing (the reason the pages give for the output's back-rotation)
    H, c, R, N = 2, 32, 16, 12
    v = rng.standard_normal((N, c))
    q = rng.standard_normal((1, H, c))
    epos = np.sort(rng.integers(0, 5000, N))
    p = 6000
    outs = []
    for shift in (0, 777, 1 << 19):
        kv = oracle.norm_rope(v, epos + shift, rope_dims=R)
        qq = oracle.norm_rope(q, [p + shift], rope_dims=R)
        o, _ = oracle.sparse_mqa(qq, kv, np.arange(N, dtype=np.int32)[None], 0.2)
        outs.append(oracle.norm_rope(o, [p + shift], rope_dims=R, inverse=True))
    np.testing.assert_allclose(outs[1], outs[0], rtol=1e-8, atol=1e-8)
    np.testing.assert_allclose(outs[2], outs[0], rtol=1e-8, atol=1e-8)


def test_attend_decode_reduces_to_plain_decode():
    # no norm, no rotation, no window: the complete step is indexer -> top-k ->
    # sparse MQA over the selection
    B, HI, cI, H, c, m, k, N = 3, 4, 16, 2, 32, 4, 5, 20
    qI = rng.standard_normal((B, HI, cI))
    w = rng.random((B, HI))
    K = rng.standard_normal((B, N, cI))
    q = rng.standard_normal((B, H, c))
    KVc = rng.standard_normal((B, N + 4, c))
    ctx = np.array([9, 50, 79])
    out, lse, idx, _ = oracle.attend_decode(qI, w, K, q, KVc, ctx, m, k, n_win=0, ring_len=4, scale=0.3,
                                            rope_dims=0)
    seq = np.arange(B)
    ref_idx, _ = oracle.index_topk(qI, w, K, ctx, m, k, seq=seq)
    ref, ref_l = oracle.sparse_mqa(q, KVc, ref_idx, 0.3, seq=seq)
    np.testing.assert_array_equal(idx, ref_idx)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, ref_l, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# FP8 (e4m3) storage for the low-precision indexer and KV (walk-through
# §2.3.4 and study notes §1.3, mixed-precision storage)
# --------------------------------------------------------------------------

def test_e4m3_round_matches_torch_on_every_bf16_value_in_range():
    # torch's float8_e4m3fn conversion (nearest, ties to even) agrees with the
    # oracle wherever torch does not overflow to NaN (|x| <= 464)
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    x = bits.float()
    x = x[torch.isfinite(x) & (x.abs() <= 464)]
    want = x.to(torch.float8_e4m3fn).float().double().numpy()
    got = oracle.e4m3_round(x.double().numpy())
    np.testing.assert_array_equal(got, want)
    r = torch.from_numpy(rng.standard_normal(20000) * np.exp(rng.uniform(-12, 6, 20000))).float()
    r = r[r.abs() <= 464]
    np.testing.assert_array_equal(oracle.e4m3_round(r.double().numpy()), r.to(torch.float8_e4m3fn).double().numpy())


def test_fp8_kv_storage_pins():
    # rotary dims untouched; each entry's largest quantised magnitude exact;
    # every other value within half an e4m3 step (2^-4 relative for normal
    # codes, 2^-10 * s for subnormal ones); an all-zero part gets s = 1
    R, c = 16, 64
    KV = rng.standard_normal((5, 7, c)) * np.exp(rng.uniform(-6, 6, (5, 7, 1)))
    KV[0, 0, :c - R] = 0.0
    codes, s, rope = oracle.quantize_kv_fp8(KV, R)
    np.testing.assert_array_equal(rope, KV[..., c - R:])
    assert s[0, 0] == 1.0 and not codes[0, 0].any()
    x = KV[..., :c - R]
    deq = oracle.dequantize_kv_fp8(codes, s, rope)
    np.testing.assert_array_equal(deq[..., c - R:], KV[..., c - R:])
    amax = np.abs(x).max(-1)
    got_max = np.abs(deq[..., :c - R]).max(-1)
    np.testing.assert_allclose(got_max, amax, rtol=1e-15, atol=0)
    err = np.abs(deq[..., :c - R] - x)
    normal = np.abs(codes) >= 2.0 ** -6
    bound = np.where(normal, 2.0 ** -4 * np.abs(x) * (1 + 1e-12), 2.0 ** -10 * s[..., None] * (1 + 1e-12))
    assert (err <= bound).all()
    # the codes are e4m3 values (what torch's conversion gives on x / s)
    want = torch.from_numpy((x / s[..., None]).astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(codes, want)


def test_e4m3_round_by_hand():
    cases = {1.0625: 1.0,           # tie between 1 and 1.125: even mantissa
             1.1875: 1.25,          # tie between 1.125 and 1.25
             448.0: 448.0, 464.0: 448.0, 500.0: 448.0, -1e9: -448.0,   # saturation, no infinity
             2.0 ** -9: 2.0 ** -9,  # smallest subnormal
             2.0 ** -10: 0.0,       # tie between 0 and 2^-9
             3 * 2.0 ** -11: 2.0 ** -9,
             0.0: 0.0}
    for x, want in cases.items():
        assert oracle.e4m3_round(np.array([x]))[0] == want, x


def test_row_quantisation_bounds():
    x = rng.standard_normal((50, 128)) * np.exp(rng.uniform(-3, 3, (50, 1)))
    x[3] = 0.0
    y, s = oracle.quantize_rows_e4m3(x)
    amax = np.abs(x).max(1)
    np.testing.assert_allclose(s[amax > 0], amax[amax > 0] / 448.0, rtol=1e-15)
    assert s[3] == 1.0 and np.all(y[3] == 0.0)
    # the largest element of a row is exact; every element is within half a
    # quantum of 3 mantissa bits (normal range) or 2^-10 * s (subnormal range)
    for r in range(50):
        j = np.argmax(np.abs(x[r]))
        assert abs(y[r, j] - x[r, j]) <= 1e-12 * abs(x[r, j])
        u = np.abs(x[r]) / s[r]
        bound = np.where(u >= 2.0 ** -6, u * 2.0 ** -4, 2.0 ** -10) * s[r]
        assert np.all(np.abs(y[r] - x[r]) <= bound * (1 + 1e-12))


def test_fp8_indexer_equals_exact_indexer_on_representable_inputs():
    # rows whose values lie on the e4m3 grid with a largest magnitude of 448
    # quantise exactly (scale 1), so the FP8 indexer is the exact one
    grid = np.unique(oracle.e4m3_round(np.linspace(-448, 448, 4001)))
    nq, HI, cI, N, m = 5, 3, 16, 40, 4
    qI = rng.choice(grid, (nq, HI, cI))
    K = rng.choice(grid, (N, cI))
    qI[..., 0] = 448.0
    K[:, 0] = -448.0
    w = rng.random((nq, HI))
    pos = rng.integers(0, N * m, nq)
    np.testing.assert_array_equal(oracle.index_scores_fp8(qI, w, K, pos, m), oracle.index_scores(qI, w, K, pos, m))
    # and a common factor on every row changes only the scale
    a = oracle.index_scores_fp8(qI * 0.01, w, K * 3.0, pos, m)
    b = oracle.index_scores(qI, w, K, pos, m) * 0.03
    np.testing.assert_allclose(a, b, rtol=1e-12)


def test_topk_recall_by_hand():
    assert oracle.topk_recall([[1, 2, 3, -1]], [[3, 2, 9, -1]]) == pytest.approx(2 / 3)
    assert oracle.topk_recall([[0, 1], [5, 4]], [[1, 0], [4, 6]]) == pytest.approx(0.75)


def test_fp8_scales_factor_out_of_the_relu():
    # positive row scales commute with the ReLU, so the FP8 indexer can run on
    # raw e4m3 codes: I = s_k * sum_h (w_h s_q,h) ReLU(codes_q,h . codes_k)
    nq, HI, cI, N, m = 4, 3, 32, 30, 4
    qI = rng.standard_normal((nq, HI, cI)) * 3.0
    K = rng.standard_normal((N, cI)) * 0.2
    w = rng.random((nq, HI))
    pos = rng.integers(m, N * m, nq)
    q8, sq = oracle.quantize_rows_e4m3(qI)
    k8, sk = oracle.quantize_rows_e4m3(K)
    # the codes: dequantised values over their scales, on the e4m3 grid up to
    # the rounding of that division
    codes_q = oracle.e4m3_round(q8 / sq[..., None])
    codes_k = oracle.e4m3_round(k8 / sk[:, None])
    np.testing.assert_allclose(codes_q, q8 / sq[..., None], rtol=1e-14)
    np.testing.assert_allclose(codes_k, k8 / sk[:, None], rtol=1e-14)
    assert np.abs(codes_q).max() == 448.0 and np.abs(codes_k).max() == 448.0
    direct = oracle.index_scores_fp8(qI, w, K, pos, m)
    factored = oracle.index_scores(codes_q, w * sq, codes_k, pos, m) * sk[None, :]
    vis = np.isfinite(direct)
    assert np.array_equal(vis, np.isfinite(factored))
    np.testing.assert_allclose(factored[vis], direct[vis], rtol=1e-12, atol=1e-12)
