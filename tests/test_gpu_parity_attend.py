"""GPU parity of the steps around the hot path against the CPU oracle:
query / KV RMSNorm with partial rotary encoding and the output's
back-rotation, the sliding-window entry lists, the complete decode step (the
window joined to the top-k selection in one softmax with a sink), and
decode-time compression through the per-sequence state cache (token by token
it must give the chunk compressor's entries)."""
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


def _gamma(c, seed):
    return 1.0 + synth.normal((c,), seed, "gamma", std=0.1, dtype=torch.float32)


# ---------------------------------------------------------------- norm + rotary
@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("c,R,with_gamma", [(512, 64, True), (136, 8, True), (128, 0, True), (64, 64, False),
                                            (512, 64, False)])
def test_norm_rope(csa, dtype, c, R, with_gamma):
    nq, H = 37, 6                       # 222 rows: ragged against 32 rows per CTA
    x = synth.normal((nq, H, c), 11, f"nr_x{c}", dtype=dtype)
    pos = synth.uniform_int(nq, 0, 1 << 21, 11, "nr_pos")
    pos[0], pos[1], pos[2] = 0, 1, (1 << 30) + 12345
    g = _gamma(c, 11) if with_gamma else None
    gd = None if g is None else g.to(DEV)
    y = csa.csa_norm_rope(x.to(DEV), pos.to(DEV), gamma=gd, eps=1e-6, rope_dims=R)
    assert_close(y, oracle.norm_rope(x, pos, gamma=g, eps=1e-6, rope_dims=R), dtype, "norm_rope")
    # the back-rotation, and the same call in place
    yi = csa.csa_norm_rope(x.to(DEV), pos.to(DEV), rope_dims=R, inverse=True)
    assert_close(yi, oracle.norm_rope(x, pos, rope_dims=R, inverse=True), dtype, "inverse rotation")
    xd = x.to(DEV)
    csa.csa_norm_rope(xd, pos.to(DEV), gamma=gd, eps=1e-6, rope_dims=R, out=xd)
    assert torch.equal(xd, y), "in-place result differs from the out-of-place one"


@pytest.mark.parametrize("dtype", MODES)
def test_norm_rope_affine_positions(csa, dtype):
    # prefill queries: rows of token t (all heads) at start + t; compressed KV
    # entries: one row each at m * (e0 + i)
    n, H, c, m, start, e0 = 45, 4, 512, 4, 196608, 4100
    q = synth.normal((n, H, c), 12, "aq", dtype=dtype)
    kv = synth.normal((n, c), 12, "akv", dtype=dtype)
    g = _gamma(c, 12)
    yq = csa.csa_norm_rope(q.to(DEV), None, gamma=g.to(DEV), rope_dims=64, pos0=start, pos_step=1, group=H)
    assert_close(yq, oracle.norm_rope(q, np.arange(start, start + n), gamma=g, rope_dims=64), dtype, "queries")
    yk = csa.csa_norm_rope(kv.to(DEV), None, gamma=g.to(DEV), rope_dims=64, pos0=m * e0, pos_step=m)
    assert_close(yk, oracle.norm_rope(kv, m * np.arange(e0, e0 + n), gamma=g, rope_dims=64), dtype, "KV entries")


# ---------------------------------------------------------------- window entry lists
def test_window_entries_bitexact(csa):
    nq, k, n_win, ring_off, ring_len = 50, 37, 128, 5000, 160
    sel = synth.uniform_int(nq * k, -1, 4999, 13, "we_sel").reshape(nq, k)
    pos = synth.uniform_int(nq, 0, 400, 13, "we_pos")
    pos[0], pos[1], pos[2], pos[3] = 0, 126, 127, 128
    ent = csa.csa_window_entries(sel.to(DEV), pos.to(DEV), n_win, ring_off, ring_len)
    want = np.concatenate([sel.numpy(), oracle.window_entries(pos, n_win, ring_off, ring_len)], axis=1)
    np.testing.assert_array_equal(host(ent), want)
    # positions pos0 + t and no selection
    ent = csa.csa_window_entries(None, None, 8, 100, 8, pos0=3, nq=20)
    np.testing.assert_array_equal(host(ent), oracle.window_entries(np.arange(3, 23), 8, 100, 8))


# ---------------------------------------------------------------- complete decode step
def _attend_inputs(dtype, ring_len=160):
    s = synth.FLASH_DECODE.scale_ctx(16)            # ctx 4K..8K -> <= 2048 entries, same heads/dims
    inp = synth.attend_decode_inputs(s, device="cpu", batch=12, n_win=128, ring_len=ring_len)
    inp["ctx_len"][0] = 3                            # no compressed entry; 4 window tokens
    inp["ctx_len"][1] = 100                          # window partly before the sequence start
    inp["ctx_len"][2] = 4 * s.n_max                  # every entry visible
    cast = (lambda t: t.to(dtype)) if dtype == torch.float32 else (lambda t: t)
    dev = {k: (cast(v).to(DEV) if v.dtype == torch.bfloat16 else v.to(DEV))
           for k, v in inp.items() if isinstance(v, torch.Tensor)}
    return s, inp, dev


@pytest.mark.parametrize("dtype", MODES)
def test_attend_decode(csa, dtype):
    s, inp, dev = _attend_inputs(dtype)
    k, n_win, L = 512, 128, inp["ring_len"]
    out, lse, sel = csa.csa_attend_decode(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], dev["kv_cache"],
                                          dev["ctx_len"], s.m, k, n_win=n_win, ring_len=L, q_gamma=dev["q_gamma"],
                                          rope_dims=64, sink=dev["sink"], return_topk=True)
    ref_o, ref_l, ref_idx, S = oracle.attend_decode(inp["qI"], inp["w"], inp["idx_cache"], inp["q"], inp["kv_cache"],
                                                    inp["ctx_len"], s.m, k, n_win, L, 1 / math.sqrt(s.c),
                                                    q_gamma=inp["q_gamma"], rope_dims=64, sink=inp["sink"],
                                                    sel=host(sel).astype(np.int32))
    assert_topk_sets(sel, ref_idx, S, k)
    assert_close(out, ref_o, dtype, "attend_decode out")
    assert_close(lse, ref_l, dtype, "attend_decode lse")


def test_attend_decode_without_extras_is_csa_decode(csa):
    # no norm, no rotation, no window, no sink: the same kernels on the same
    # entries as csa_decode, so the same bits
    s, inp, dev = _attend_inputs(torch.bfloat16, ring_len=0)
    kv = dev["kv_cache"][:, :s.n_max].contiguous()
    o1, l1, s1 = csa.csa_attend_decode(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], kv, dev["ctx_len"], s.m, 512,
                                       n_win=0, ring_len=0, rope_dims=0, return_topk=True)
    o2, l2, s2 = csa.csa_decode(dev["qI"], dev["w"], dev["idx_cache"], dev["q"], kv, dev["ctx_len"], s.m, 512,
                                return_topk=True)
    assert torch.equal(s1, s2) and torch.equal(o1, o2) and torch.equal(l1, l2)


def test_attend_prefill_composed_from_the_entry_points(csa):
    # a prefill chunk with the complete attention output, composed from the C
    # entry points: KV entries normalised and rotated at m * entry, queries at
    # their token positions, indexer + top-k, window rows of the chunk's ring,
    # one softmax with the sink, output turned back
    n, start, m, H, c, HI, cI, k, n_win = 256, 1024, 4, 8, 128, 4, 64, 64, 128
    N = (start + n) // m
    L = n + n_win                                   # >= n + n_win - 1 distinct rows
    seed = 14
    kv_raw = synth.normal((N, c), seed, "p_kv")
    ik = synth.normal((N, cI), seed, "p_ik")
    ring_tok = synth.normal((L, c), seed, "p_ring")     # token tau's row at tau mod L
    q = synth.normal((n, H, c), seed, "p_q")
    qI = synth.normal((n, HI, cI), seed, "p_qI")
    w = synth.head_weights(n, HI, seed)
    gq, gk = _gamma(c, seed), _gamma(c, seed + 1)
    sink = synth.normal((H,), seed, "p_sink", dtype=torch.float32)
    pos = np.arange(start, start + n, dtype=np.int32)
    scale = 1 / math.sqrt(c)

    # GPU
    kv_d = torch.cat([kv_raw, ring_tok]).to(DEV)
    csa.csa_norm_rope(kv_d[:N], None, gamma=gk.to(DEV), rope_dims=64, pos0=0, pos_step=m, out=kv_d[:N])
    qn = csa.csa_norm_rope(q.to(DEV), None, gamma=gq.to(DEV), rope_dims=64, pos0=start, group=H)
    pos_d = torch.from_numpy(pos).to(DEV)
    seq0 = torch.zeros(n, dtype=torch.int32, device=DEV)
    sel, _ = csa.csa_index_topk(qI.to(DEV), w.to(DEV), ik.to(DEV), pos_d, m, k, seq_of_q=seq0)
    ent = csa.csa_window_entries(sel, None, n_win, N, L, pos0=start)
    out, lse = csa.csa_sparse_mqa(qn, kv_d, ent, scale, sink=sink.to(DEV), seq_of_q=seq0)
    csa.csa_norm_rope(out, None, rope_dims=64, inverse=True, pos0=start, group=H, out=out)

    # oracle, the same steps (KV entries rounded to bf16 at the cache store)
    kv_o = np.concatenate([oracle.bf16_round(oracle.norm_rope(kv_raw, m * np.arange(N), gamma=gk, rope_dims=64)),
                           oracle._f64(ring_tok)])
    ref_idx, S = oracle.index_topk(qI, w, ik, pos, m, k)
    assert_topk_sets(sel, ref_idx, S, k)
    ent_o = np.concatenate([host(sel).astype(np.int32), oracle.window_entries(pos, n_win, N, L)], axis=1)
    qn_o = oracle.norm_rope(q, pos, gamma=gq, rope_dims=64)
    ref_o, ref_l = oracle.sparse_mqa(qn_o, kv_o, ent_o, scale, sink=sink)
    ref_o = oracle.norm_rope(ref_o, pos, rope_dims=64, inverse=True)
    assert_close(out, ref_o, torch.bfloat16, "composed prefill out")
    assert_close(lse, ref_l, torch.bfloat16, "composed prefill lse")


# ---------------------------------------------------------------- decode-time compression
def _step_schedule(T_b):
    """pos per step: sequence b takes token s at step s while s < T_b[b], then sits out (-1)."""
    T = max(T_b)
    return [torch.tensor([s if s < t else -1 for t in T_b], dtype=torch.int32) for s in range(T)]


@pytest.mark.parametrize("dtype", MODES)
def test_csa_compress_step_equals_chunk_compression(csa, dtype):
    m, c, Nmax = 4, 136, 10                  # 17 channel groups; entry 10 of the longest sequence is out of range
    T_b = [37, 4, 5, 44, 1, 0]
    B = len(T_b)
    rows = synth.normal((B, max(T_b), 4 * c), 15, "step_rows", dtype=torch.float32)
    bias = synth.normal((2 * m, c), 15, "step_bias", std=math.sqrt(0.1), dtype=torch.float32)
    state = torch.zeros((B, 2 * m, 4 * c), dtype=torch.float32, device=DEV)
    sentinel = 7.0
    cache = torch.full((B, Nmax, c), sentinel, dtype=dtype, device=DEV)
    rows_d, bias_d = rows.to(DEV), bias.to(DEV)
    for s, pos in enumerate(_step_schedule(T_b)):
        csa.csa_compress_step(rows_d[:, s].contiguous(), state, bias_d, pos.to(DEV), cache, m)
    got = host(cache)
    for b, T in enumerate(T_b):
        n = min((T // m), Nmax)
        if n:
            ref = oracle.csa_compress(rows[b, :n * m], bias, m)
            assert_close(got[b, :n], ref, dtype, f"sequence {b}")
        assert np.all(got[b, n:] == sentinel), f"sequence {b}: rows past its closed blocks were written"
    if dtype == torch.float32:
        # the chunk kernel on the same rows: the same operations in the same order
        for b, T in enumerate(T_b):
            n = min((T // m), Nmax)
            if n:
                chunk = csa.csa_compress(rows_d[b, :n * m].contiguous(), bias_d, m)
                assert float((chunk - cache[b, :n]).abs().max()) <= 1e-6


@pytest.mark.parametrize("dtype", MODES)
@pytest.mark.parametrize("mp", [8, 128])
def test_hca_compress_step_equals_chunk_compression(csa, dtype, mp):
    c, Nmax = 64, 3
    T_b = [3 * mp + 5, mp, mp - 1, 2 * mp + 1]
    B = len(T_b)
    rows = synth.normal((B, max(T_b), 2 * c), 16, f"hstep_rows{mp}", dtype=torch.float32)
    bias = synth.normal((mp, c), 16, f"hstep_bias{mp}", std=math.sqrt(0.1), dtype=torch.float32)
    state = torch.zeros((B, mp, 2 * c), dtype=torch.float32, device=DEV)
    cache = torch.full((B, Nmax, c), 7.0, dtype=dtype, device=DEV)
    rows_d, bias_d = rows.to(DEV), bias.to(DEV)
    for s, pos in enumerate(_step_schedule(T_b)):
        csa.hca_compress_step(rows_d[:, s].contiguous(), state, bias_d, pos.to(DEV), cache, mp)
    got = host(cache)
    for b, T in enumerate(T_b):
        n = min(T // mp, Nmax)
        if n:
            assert_close(got[b, :n], oracle.hca_compress(rows[b, :n * mp], bias, mp), dtype, f"sequence {b}")
        assert np.all(got[b, n:] == 7.0)


@pytest.mark.parametrize("dtype", MODES)
def test_decode_compress_from_hidden(csa, dtype):
    # both CSA streams of a decode loop, projected from each step's hidden
    # states, against the chunk definition over each sequence's history
    m, d, c, cI, Nmax = 4, 256, 64, 64, 8
    T_b = [13, 8, 3, 11]
    B = len(T_b)
    X = synth.normal((B, max(T_b), d), 17, "dc_x", dtype=dtype)
    W_kv = synth.normal((4 * c, d), 17, "dc_Wkv", std=1 / math.sqrt(d), dtype=dtype)
    W_idx = synth.normal((4 * cI, d), 17, "dc_Widx", std=1 / math.sqrt(d), dtype=dtype)
    B_kv = synth.normal((2 * m, c), 17, "dc_Bkv", std=math.sqrt(0.1), dtype=torch.float32)
    B_idx = synth.normal((2 * m, cI), 17, "dc_Bidx", std=math.sqrt(0.1), dtype=torch.float32)
    st_kv = torch.zeros((B, 2 * m, 4 * c), dtype=torch.float32, device=DEV)
    st_idx = torch.zeros((B, 2 * m, 4 * cI), dtype=torch.float32, device=DEV)
    kv = torch.zeros((B, Nmax, c), dtype=dtype, device=DEV)
    ik = torch.zeros((B, Nmax, cI), dtype=dtype, device=DEV)
    dev = [t.to(DEV) for t in (X, W_kv, B_kv, W_idx, B_idx)]
    for s, pos in enumerate(_step_schedule(T_b)):
        csa.csa_decode_compress(dev[0][:, s].contiguous(), dev[1], dev[2], dev[3], dev[4], pos.to(DEV), st_kv, st_idx,
                                kv, ik, m)
    for b, T in enumerate(T_b):
        n = T // m
        if n:
            ref_kv = oracle.csa_compress_from_hidden(X[b, :n * m], W_kv, B_kv, m)
            ref_ik = oracle.csa_compress_from_hidden(X[b, :n * m], W_idx, B_idx, m)
            assert_close(kv[b, :n], ref_kv, dtype, f"KV entries of sequence {b}")
            assert_close(ik[b, :n], ref_ik, dtype, f"index keys of sequence {b}")
