"""Comparison rules shared by the GPU parity tests.

Tolerances (stated by the method's acceptance criteria for compressed KV and
attention outputs): bf16 mode max-abs <= 2e-2 and rel-L2 <= 5e-3; fp32 mode
both <= 1e-5. Indexer scores are fp32 sums of exact bf16 products in both
modes, so they are held to a relative bound of 1e-5 of the absolute-value sum
sum_h w_h |q_h . K_s| (a rounding-error bound for fp32 accumulation of a few
hundred terms, with margin).

Top-k: given identical fp32 score tensors the GPU result must be bit-exact.
End to end, the GPU's selected set may differ from the oracle's only in
entries whose oracle score lies within 1e-3 (relative) of the oracle's k-th
score; the attention output is then compared against the oracle run on the
GPU's own selection.
"""
import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-5, 1e-5)}


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.int32 else t.cpu().numpy()


def assert_close(gpu, ref, dtype, what=""):
    """max-abs and rel-L2 bounds of the mode."""
    g = host(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: finite pattern differs"
    assert np.array_equal(g[~fin], r[~fin]), f"{what}: non-finite values differ"
    if not fin.any():
        return
    d = g[fin] - r[fin]
    max_abs = float(np.abs(d).max())
    rel_l2 = float(np.linalg.norm(d) / max(np.linalg.norm(r[fin]), 1e-30))
    ma, rl = TOL[dtype]
    assert max_abs <= ma and rel_l2 <= rl, f"{what}: max_abs={max_abs:.3e} (<= {ma}) rel_l2={rel_l2:.3e} (<= {rl})"


def assert_scores_close(gpu_scores, ref_scores, bound):
    """|gpu - ref| <= 1e-5 * bound elementwise on visible entries; -inf elsewhere."""
    g, r = host(gpu_scores), np.asarray(ref_scores)
    vis = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), vis), "visible pattern differs"
    err = np.abs(g[vis] - r[vis])
    lim = 1e-5 * np.asarray(bound)[vis] + 1e-30
    worst = float((err / lim).max()) if err.size else 0.0
    assert worst <= 1.0, f"score error {worst:.2f}x the bound"


def score_bound(qI, w, K, pos, m, seq=None):
    """sum_h w_h |q_h . K_s| (the scale against which score rounding is measured)."""
    qa = np.abs(oracle._f64(qI))
    # |q . K| <= |q| . |K|: a valid upper bound that avoids a second dot product pass
    return oracle.index_scores(qa, np.abs(oracle._f64(w)), np.abs(oracle._f64(K)), pos, m, seq=seq)


def assert_topk_sets(gpu_idx, ref_idx, ref_scores, k, rel_gap=1e-3):
    """Sets may differ only in entries scored within rel_gap of the oracle's k-th score."""
    g, r = host(gpu_idx), np.asarray(ref_idx)
    S = np.asarray(ref_scores)
    n_diff_rows = 0
    for t in range(g.shape[0]):
        gs, rs = set(g[t][g[t] >= 0].tolist()), set(r[t][r[t] >= 0].tolist())
        assert len(gs) == len(rs), f"row {t}: {len(gs)} selected, oracle {len(rs)}"
        assert len(gs) == int((g[t] >= 0).sum()), f"row {t}: duplicate indices"
        if gs == rs:
            continue
        n_diff_rows += 1
        kth = S[t, r[t][len(rs) - 1]]
        for s in gs ^ rs:
            assert abs(S[t, s] - kth) <= rel_gap * abs(kth), (
                f"row {t}: entry {s} score {S[t, s]} vs k-th {kth} beyond the {rel_gap} gap rule")
    return n_diff_rows


def assert_topk_order(gpu_idx, ref_scores):
    """GPU order must be (oracle score desc, index asc) up to score ties within rounding."""
    g = host(gpu_idx)
    S = np.asarray(ref_scores)
    for t in range(g.shape[0]):
        sel = g[t][g[t] >= 0]
        assert np.all(g[t][len(sel):] == -1), f"row {t}: padding not at the end"
        sc = S[t, sel]
        assert np.all(sc[:-1] >= sc[1:] - 1e-5 * np.abs(sc[1:]) - 1e-30), f"row {t}: not in descending order"
