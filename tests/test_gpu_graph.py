"""The decode entry points captured in a CUDA graph: a serving loop captures
a step once and replays it, so the calls must make no allocation and no host
synchronisation inside the capture, and a replay must give the same bits as
the eager call on the same inputs (also after the inputs change in place)."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def csa():
    import compressed_sparse_attention_14_b200 as m
    return m


def _graph_of(fn):
    fn()                                   # one-time set-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_csa_decode_replays_bit_exactly(csa):
    s = synth.FLASH_DECODE.scale_ctx(16)
    inp = {k: v.to(DEV) for k, v in synth.decode_inputs(s, device="cpu", batch=10).items()}
    B, k = inp["q"].shape[0], 512
    out = torch.empty_like(inp["q"])
    lse = torch.empty((B, s.heads), dtype=torch.float32, device=DEV)
    sel = torch.empty((B, k), dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.csa_decode_workspace_size(B, s.n_max, s.heads, s.c, s.idx_heads, s.idx_dim, k, csa.CSA_BF16),
                     dtype=torch.uint8, device=DEV)

    def step():
        csa.csa_decode(inp["qI"], inp["w"], inp["idx_cache"], inp["q"], inp["kv_cache"], inp["ctx_len"], s.m, k,
                       out=out, lse=lse, topk_idx=sel, ws=ws)

    g = _graph_of(step)
    for trial in range(2):
        if trial == 1:                     # new queries in the same buffers
            inp["q"].copy_(synth.normal(tuple(inp["q"].shape), 77, "graph_q").to(DEV))
            inp["qI"].copy_(synth.normal(tuple(inp["qI"].shape), 77, "graph_qI").to(DEV))
        out.zero_(); lse.zero_(); sel.zero_()
        g.replay()
        torch.cuda.synchronize()
        o1, l1, s1 = out.clone(), lse.clone(), sel.clone()
        step()
        torch.cuda.synchronize()
        assert torch.equal(s1, sel) and torch.equal(o1, out) and torch.equal(l1, lse)


def test_hca_decode_replays_bit_exactly(csa):
    s = synth.HCA
    inp = synth.hca_decode_inputs(s, batch=4, n_max=900)
    q, kv, ctx = inp["q"].to(DEV), inp["kv_cache"].to(DEV), inp["ctx_len"].to(DEV)
    B = q.shape[0]
    out = torch.empty_like(q)
    lse = torch.empty((B, s.heads), dtype=torch.float32, device=DEV)
    ws = torch.empty(max(1, csa.workspace_size("hca_decode", B, 900, s.heads, s.c, csa.CSA_BF16)), dtype=torch.uint8,
                     device=DEV)

    def hstep():
        csa.hca_decode(q, kv, ctx, s.mp, out=out, lse=lse, ws=ws)

    g = _graph_of(hstep)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    o1, l1 = out.clone(), lse.clone()
    hstep()
    torch.cuda.synchronize()
    assert torch.equal(o1, out) and torch.equal(l1, lse)
