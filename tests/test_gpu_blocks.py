"""Caches in the lcm(m, m')-token block layout [Notes §2.6: one block covers
lcm(m, m') raw tokens and holds their CSA and HCA entries; Walk §5 item 2].

The blocked calls must compute exactly what the contiguous calls compute on
the same entries (the same kernels and arithmetic; only where a row is read
or written differs): decode attention from block caches equals decode
attention from contiguous caches bit for bit, and compression into block
caches writes the same bytes the contiguous compression writes, leaving the
other parts of each block untouched."""
import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def csa():
    import compressed_sparse_attention_14_b200 as m
    return m


def _rand(shape, seed, std=1.0, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(dtype).to(DEV)


def _to_blocks(lay, kv, ik, hca):
    """Contiguous caches kv [B, nblk*r1, c], ik [B, nblk*r1, cI], hca
    [B, nblk*r2, c] (bf16) into blocks [B, nblk, block_bytes]."""
    B, n1, c = kv.shape
    r1, r2 = lay["csa_rows"], lay["hca_rows"]
    nblk = n1 // r1
    blocks = torch.full((B, nblk, lay["block_bytes"]), 0xA5, dtype=torch.uint8, device=DEV)
    parts = [(lay["kv_offset"], kv, r1), (lay["idx_offset"], ik, r1), (lay["hca_offset"], hca, r2)]
    for off, t, r in parts:
        raw = t.reshape(B, nblk, r * t.shape[2]).view(torch.uint8)
        blocks[:, :, off:off + raw.shape[2]] = raw
    return blocks


def _from_blocks(lay, blocks, c, cI):
    B, nblk, _ = blocks.shape
    r1, r2 = lay["csa_rows"], lay["hca_rows"]
    out = []
    for off, w, r in [(lay["kv_offset"], c, r1), (lay["idx_offset"], cI, r1), (lay["hca_offset"], c, r2)]:
        raw = blocks[:, :, off:off + r * w * 2].contiguous()
        out.append(raw.view(torch.bfloat16).reshape(B, nblk * r, w))
    return out


def test_blocks_round_trip(csa):
    lay = csa.csa_cache_block_layout(4, 128, 512, 128)
    B, nblk = 2, 3
    kv, ik, hca = _rand((B, nblk * 32, 512), 1), _rand((B, nblk * 32, 128), 2), _rand((B, nblk, 512), 3)
    back = _from_blocks(lay, _to_blocks(lay, kv, ik, hca), 512, 128)
    for a, b in zip((kv, ik, hca), back):
        assert torch.equal(a, b)


@pytest.mark.parametrize("shape", [(3, 2048, 64, 512, 64, 128, 512), (5, 1024, 128, 256, 64, 64, 256)])
def test_csa_decode_blocked_equals_contiguous(csa, shape):
    B, Nmax, H, c, HI, cI, k = shape
    m, mp = 4, 128
    lay = csa.csa_cache_block_layout(m, mp, c, cI)
    kv = _rand((B, Nmax, c), 11)
    ik = _rand((B, Nmax, cI), 12)
    hca = _rand((B, Nmax // lay["csa_rows"], c), 13)
    blocks = _to_blocks(lay, kv, ik, hca)
    qI = _rand((B, HI, cI), 14)
    w = _rand((B, HI), 15, std=1 / math.sqrt(HI), dtype=torch.float32)
    q = _rand((B, H, c), 16)
    sink = _rand((H,), 17, dtype=torch.float32)
    g = torch.Generator().manual_seed(18)
    ctx = torch.randint(m, Nmax * m + 1, (B,), generator=g, dtype=torch.int32)
    ctx[0] = Nmax * m           # every entry visible
    ctx[-1] = 3 * m + 2         # fewer entries than k
    ctx = ctx.to(DEV)
    ref = csa.csa_decode(qI, w, ik, q, kv, ctx, m, k, sink=sink, return_topk=True)
    got = csa.csa_decode_blocked(qI, w, q, blocks, lay, ctx, k, sink=sink, return_topk=True)
    for name, a, b in zip(("out", "lse", "topk"), ref, got):
        assert torch.equal(a, b), f"{name} differs between the block and the contiguous caches"


@pytest.mark.parametrize("B,nblk,H,c", [(16, 256, 64, 512), (3, 40, 128, 256)])
def test_hca_decode_blocked_equals_contiguous(csa, B, nblk, H, c):
    m, mp, cI = 4, 128, 64
    lay = csa.csa_cache_block_layout(m, mp, c, cI)
    kv = _rand((B, nblk * lay["csa_rows"], c), 21)
    ik = _rand((B, nblk * lay["csa_rows"], cI), 22)
    hca = _rand((B, nblk, c), 23)
    blocks = _to_blocks(lay, kv, ik, hca)
    q = _rand((B, H, c), 24)
    sink = _rand((H,), 25, dtype=torch.float32)
    g = torch.Generator().manual_seed(26)
    ctx = torch.randint(1, nblk * mp + 1, (B,), generator=g, dtype=torch.int32)
    ctx[0] = nblk * mp
    ctx[1] = mp - 1             # no entry visible yet: the sink alone
    ctx = ctx.to(DEV)
    ref = csa.hca_decode(q, hca, ctx, mp, sink=sink)
    got = csa.hca_decode_blocked(q, blocks, lay, ctx, sink=sink)
    for name, a, b in zip(("out", "lse"), ref, got):
        assert torch.equal(a, b), f"{name} differs between the block and the contiguous caches"


def _step_schedule(T_b, B):
    # one new token per sequence per step; a sequence past its length sits out
    for s in range(max(T_b)):
        yield torch.tensor([s if s < T else -1 for T in T_b], dtype=torch.int32)


def test_decode_compress_blocked_equals_contiguous(csa):
    m, mp, d, c, cI = 4, 128, 256, 64, 64
    lay = csa.csa_cache_block_layout(m, mp, c, cI)
    nblk = 3
    Nmax = nblk * lay["csa_rows"]
    T_b = [150, 97, 3, 64]
    B = len(T_b)
    X = synth.normal((B, max(T_b), d), 31, "blk_x", dtype=torch.bfloat16).to(DEV)
    W_kv = synth.normal((4 * c, d), 31, "blk_Wkv", std=1 / math.sqrt(d), dtype=torch.bfloat16).to(DEV)
    W_idx = synth.normal((4 * cI, d), 31, "blk_Widx", std=1 / math.sqrt(d), dtype=torch.bfloat16).to(DEV)
    B_kv = synth.normal((2 * m, c), 31, "blk_Bkv", std=math.sqrt(0.1), dtype=torch.float32).to(DEV)
    B_idx = synth.normal((2 * m, cI), 31, "blk_Bidx", std=math.sqrt(0.1), dtype=torch.float32).to(DEV)
    st = [torch.zeros((B, 2 * m, 4 * w), dtype=torch.float32, device=DEV) for w in (c, cI)]
    st_b = [t.clone() for t in st]
    kv = torch.zeros((B, Nmax, c), dtype=torch.bfloat16, device=DEV)
    ik = torch.zeros((B, Nmax, cI), dtype=torch.bfloat16, device=DEV)
    hca = _rand((B, nblk, c), 32)
    blocks = _to_blocks(lay, kv, ik, hca)
    for s, pos in enumerate(_step_schedule(T_b, B)):
        x = X[:, s].contiguous()
        p = pos.to(DEV)
        csa.csa_decode_compress(x, W_kv, B_kv, W_idx, B_idx, p, st[0], st[1], kv, ik, m)
        csa.csa_decode_compress_blocked(x, W_kv, B_kv, W_idx, B_idx, p, st_b[0], st_b[1], blocks, lay)
    kv_b, ik_b, hca_b = _from_blocks(lay, blocks, c, cI)
    assert torch.equal(kv, kv_b)
    assert torch.equal(ik, ik_b)
    assert torch.equal(hca, hca_b), "the HCA part of the blocks was written"
    assert torch.equal(st[0], st_b[0]) and torch.equal(st[1], st_b[1])
    assert kv[0, 36].abs().sum() > 0   # entries were written (sequence 0 closed 37 blocks of m)


def test_hca_compress_step_blocked_equals_contiguous(csa):
    m, mp, c, cI = 4, 8, 64, 32
    lay = csa.csa_cache_block_layout(m, mp, c, cI)   # 8 tokens: 2 CSA rows, 1 HCA row
    nblk, B, T = 6, 3, 45
    proj = synth.normal((T, B, 2 * c), 41, "blk_hproj", dtype=torch.float32).to(DEV)
    bias = synth.normal((mp, c), 41, "blk_hbias", std=math.sqrt(0.1), dtype=torch.float32).to(DEV)
    st = torch.zeros((B, mp, 2 * c), dtype=torch.float32, device=DEV)
    st_b = st.clone()
    kv = _rand((B, nblk * 2, c), 42)
    ik = _rand((B, nblk * 2, cI), 43)
    hca = torch.zeros((B, nblk, c), dtype=torch.bfloat16, device=DEV)
    blocks = _to_blocks(lay, kv, ik, hca)
    for s in range(T):
        pos = torch.tensor([s, s if s < 30 else -1, s if s < 7 else -1], dtype=torch.int32, device=DEV)
        csa.hca_compress_step(proj[s].contiguous(), st, bias, pos, hca, mp)
        csa.hca_compress_step_blocked(proj[s].contiguous(), st_b, bias, pos, blocks, lay)
    kv_b, ik_b, hca_b = _from_blocks(lay, blocks, c, cI)
    assert torch.equal(hca, hca_b)
    assert torch.equal(kv, kv_b) and torch.equal(ik, ik_b), "the CSA parts of the blocks were written"
    assert hca[0, 4].abs().sum() > 0
