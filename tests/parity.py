"""Shared checks for GPU-vs-oracle parity tests.

Acceptance rules (selection ties are legitimate, so sets are compared where
they are unique and checked for validity elsewhere):
  * strict: where the K-th and (K+1)-th oracle group scores differ by more
    than ``eps``, the chosen set is identical;
  * tie-tolerant (every row): every chosen chunk scores, in the oracle, at
    least as high as every unchosen candidate minus ``eps``, and the set size
    equals min(K, #candidates);
  * outputs: compared with the oracle run on the CUDA path's own selection
    (forced selection), using the oracle's s^ for those chunks.
"""
from __future__ import annotations

import numpy as np

EPS_SEL = 1e-2
TOL_F32 = 1e-5
TOL_BF16 = 1.5e-2
# k' (bf16 runs): one bf16 rounding of the stored value (|k'| 2^-8 relative), plus
# an absolute term.  The summary kernel splits each softmax weight p into a bf16
# high part ph = bf16(p) and a low part p - ph, which the bf16 MMA rounds again:
# |p - ph| <= 2^-8 p, so each weight enters with error <= 2^-16 p, and the
# weighted key sum with error <= 2^-16 * max|k| (the weights sum to 1).  The
# fp32 accumulation of the 64 products adds at most 63 * 2^-24 * max|k|.  The
# largest |k| of the biggest workload (8.6e9 N(0,1) draws) is about 6.5, so the
# two give 9.9e-5 + 2.4e-5 < 1.25e-4.  Its effect on s^ is ~1e-4, far below the
# 1e-2 selection gap.
KSUM_ATOL = 1.25e-4


def to_np(t):
    return t.detach().float().cpu().numpy() if hasattr(t, "detach") else np.asarray(t)


def check_selection(idx_gpu, g_or, K, eps=EPS_SEL):
    """idx_gpu [R, Hkv, K] int; g_or [R, Hkv, C] oracle group scores (-inf off-candidate).

    Returns (n_strict_rows, n_rows).  Raises AssertionError on any violation.
    """
    idx_gpu = np.asarray(idx_gpu)
    R, Hkv, _ = idx_gpu.shape
    n_strict = 0
    for r in range(R):
        for g in range(Hkv):
            gs = g_or[r, g]
            cand = np.flatnonzero(np.isfinite(gs))
            sel = idx_gpu[r, g]
            chosen = sel[sel >= 0]
            assert len(chosen) == min(K, len(cand)), (r, g, len(chosen), len(cand))
            assert np.all(np.diff(chosen) > 0), (r, g, chosen)  # ascending, distinct
            assert np.all(sel[len(chosen):] == -1), (r, g, sel)
            if len(chosen) == 0:
                continue
            assert np.isin(chosen, cand).all(), (r, g, chosen)
            if len(cand) > K:
                order = np.sort(gs[cand])[::-1]
                gap = order[K - 1] - order[K]
                rest = np.setdiff1d(cand, chosen)
                assert gs[chosen].min() >= gs[rest].max() - eps, (r, g, gs[chosen].min(), gs[rest].max())
                if gap > eps:
                    n_strict += 1
                    want = np.sort(cand[np.lexsort((cand, -gs[cand]))][:K])
                    assert np.array_equal(chosen, want), (r, g, chosen, want)
    return n_strict, R * Hkv


def forced_s_sel(idx_gpu, s_all_or, G):
    """Oracle s^ of the CUDA-chosen chunks: [R, Hq, K] (-inf where idx == -1)."""
    R, Hkv, K = idx_gpu.shape
    Hq = Hkv * G
    out = np.full((R, Hq, K), -np.inf)
    for h in range(Hq):
        sel = idx_gpu[:, h // G, :]
        ok = sel >= 0
        rr, kk = np.nonzero(ok)
        out[rr, h, kk] = s_all_or[rr, h, sel[rr, kk]]
    return out
