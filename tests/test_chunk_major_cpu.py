"""CPU checks of the numerics the chunk-major bf16 attention relies on (no GPU).

The chunk-major pass computes, for every (position, selected chunk) pair
independently, O_c = softmax over the chunk's keys of q.k * scale, times V_c
(hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
(Method): each selected chunk is attended with its own softmax).  It stores
O_c rounded to bf16 (the 1 KB partial record) and fuses the records with the
window's exact terms and the weights exp(s^_c).

1. The per-pair decomposition, evaluated in fp64 with records kept exact,
   reproduces the oracle's output.  This is the structural claim of the pass:
   O_c depends only on the position's query and the chunk, so computing the
   pairs in any grouping and fusing them afterwards changes nothing.
2. Rounding every record to bf16 moves each output by at most
   2^-9 * max |O_c| <= 2^-9 * max |v|: the fused output is a convex
   combination of the records and the window values, and round-to-nearest bf16
   has relative error <= 2^-9.  The bf16 tolerance (1.5e-2) is far above this.
"""
import numpy as np
import torch

import oracle
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, prefill_inputs
from tests.parity import TOL_BF16


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def _fused(w, q, k, v, rows, idx, s_sel, round_records):
    """Chunk-major evaluation: per-pair O_c records, then the fusion."""
    S, nw, scale = w.S, w.W // w.S, 1.0 / np.sqrt(w.d)
    G = w.Hq // w.Hkv
    out = np.zeros((len(rows), w.Hq, w.d))
    for r, (b, i) in enumerate(rows):
        cur = i // S
        lo = max(0, (cur - nw + 1) * S)
        for h in range(w.Hq):
            g = h // G
            qv = q[b, h, i].astype(np.float64)
            # window terms, exact
            kw, vw = k[b, g, lo:i + 1].astype(np.float64), v[b, g, lo:i + 1].astype(np.float64)
            sw = kw @ qv * scale
            # selected chunks: one record per (position, chunk)
            recs, wts = [], []
            for x in range(w.K):
                c = idx[r, g, x]
                if c < 0:
                    continue
                kc = k[b, g, c * S:(c + 1) * S].astype(np.float64)
                vc = v[b, g, c * S:(c + 1) * S].astype(np.float64)
                sc = kc @ qv * scale
                p = np.exp(sc - sc.max())
                o = (p / p.sum()) @ vc
                recs.append(_bf16(o) if round_records else o)
                wts.append(s_sel[r, h, x])
            m = max([sw.max()] + wts)
            ew = np.exp(sw - m)
            num = ew @ vw
            den = ew.sum()
            for o, s_hat in zip(recs, wts):
                e = np.exp(s_hat - m)
                num = num + e * o
                den += e
            out[r, h] = num / den
    return out


def _case():
    w = WORKLOADS["prefill_8k"].scaled(name="cm_cpu", N=1024, Hq=4, Hkv=1, W=128, K=4, needles_per_head=2,
                                       needle_gap=None)
    x = prefill_inputs(w)
    q, k, v, ql = (x[n].float().numpy() for n in ("q", "k", "v", "q_lmk"))
    dm = oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K)
    rng = np.random.default_rng(7)
    pos = sorted(set([0, 63, 64, 191, 192, 255, 256, 511, 1023] + rng.integers(0, w.N, 40).tolist()))
    rows = [(0, p) for p in pos]
    ks, bs = oracle.summaries(dm, k, ql)
    idx, s_sel = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs)
    ref = oracle.attend(dm, rows, q, k, v, idx, s_sel)
    return w, q, k, v, rows, idx, s_sel, ref


def test_per_pair_records_fused_equal_the_method():
    w, q, k, v, rows, idx, s_sel, ref = _case()
    assert (idx >= 0).sum() > 0
    got = _fused(w, q, k, v, rows, idx, s_sel, round_records=False)
    assert np.abs(got - ref).max() < 1e-10


def test_bf16_records_stay_within_the_rounding_bound():
    w, q, k, v, rows, idx, s_sel, ref = _case()
    got = _fused(w, q, k, v, rows, idx, s_sel, round_records=True)
    bound = 2.0 ** -9 * np.abs(v).max() * (1 + 1e-9)
    err = np.abs(got - ref).max()
    assert 0 < err <= bound, (err, bound)
    assert bound < TOL_BF16
