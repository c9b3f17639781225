"""GPU parity at the workloads' full sizes, in the launch configuration that
bench.py times (the whole problem through the same entry points), checked on
sampled outputs the oracle computes one by one:

* 128K prefill (B=1, N=131072, K=32, W=512);
* 512K prefill with Q-Cal (N=524288, K=64, W=1024, rank 64, d_model 4096);
* decode over 16 caches of 512K (two of the sequences checked).

Rows: edge positions (first and last rows, chunk and block borders, the first
rows with candidates), a subset of the planted-needle queries and a seeded
random sample.  Selection uses the tie-tolerant rule (strict where the oracle's
K-th and (K+1)-th group scores differ by more than 1e-2); outputs are compared
with the oracle run on the GPU's own selection, within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, decode_inputs, prefill_inputs
from tests.parity import KSUM_ATOL, TOL_BF16, check_selection, forced_s_sel, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rows(w, needles, n_needles=64, n_random=128, seed=1):
    N, S, W = w.N, w.S, w.W
    pos = {0, 1, N - 1, N - 2, W - 1, W, W + S - 1, W + S, W + S + 1}
    for c in (8, 9, N // S // 2, N // S - 1):
        for off in (-1, 0, 13, 14, 63):
            pos.add(c * S + off)
    rng = np.random.default_rng(seed)
    if needles:
        for t in rng.choice(len(needles), size=min(n_needles, len(needles)), replace=False):
            pos.add(needles[int(t)][2])
    pos.update(rng.integers(0, N, n_random).tolist())
    return [(0, p) for p in sorted(p for p in pos if 0 <= p < N)]


def _prefill_full(w):
    x = prefill_inputs(w, device=DEV)
    cfg = H.config_of(w)
    qc = (x["h"], x["w_down"], x["w_up"]) if w.d_model else None
    pre = H.Prefill(cfg, DEV, qcal_rank=w.qcal_rank)
    pre.run(x["q"], x["k"], x["v"], x["q_lmk"], qcal=qc)
    H.hils_sync_status()
    dm = oracle.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K)
    q, k, v, ql = (to_np(x[n]) for n in ("q", "k", "v", "q_lmk"))
    ks, bs = oracle.summaries(dm, k, ql)
    excess = np.abs(to_np(pre.k_sum) - ks) - np.abs(ks) * 2.0 ** -8
    assert excess.max() <= KSUM_ATOL, excess.max()
    np.testing.assert_allclose(to_np(pre.b_sum), bs, rtol=0, atol=2e-5)
    rows = _rows(w, x["needles"])
    ridx = np.array([p for _, p in rows])
    qs = None
    if w.d_model:
        # Q-Cal rows one by one: a compact problem holding only the sampled positions
        n = len(rows)
        dq = oracle.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, N=n, d=w.d, S=w.S, W=w.W, K=w.K)
        q_r = np.ascontiguousarray(q[:, :, ridx])
        h_r = to_np(x["h"][:, torch.from_numpy(ridx).to(DEV)])
        qs = oracle.qcal(dq, [(0, j) for j in range(n)], q_r, h_r, to_np(x["w_down"]), to_np(x["w_up"]))
    idx_or, ssel_or, s_all, g_all = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs, qs=qs, want_all=True)
    rdev = torch.from_numpy(ridx).to(DEV)
    idx_g = to_np(pre.idx[0][:, rdev]).astype(np.int64).transpose(1, 0, 2)    # [rows, Hkv, K]
    n_strict, n = check_selection(idx_g, g_all, w.K)
    ssel_g = to_np(pre.s_sel[0][:, rdev]).transpose(1, 0, 2)                  # [rows, Hq, K]
    ssel_f = forced_s_sel(idx_g, s_all, w.G)
    fin = np.isfinite(ssel_f)
    assert np.array_equal(fin, np.isfinite(ssel_g))
    assert np.abs(ssel_g[fin] - ssel_f[fin]).max() < 5e-3
    out_f = oracle.attend(dm, rows, q, k, v, idx_g, ssel_f)
    got = to_np(pre.out[0][:, rdev]).transpose(1, 0, 2)
    err = np.abs(got - out_f).max()
    assert err <= TOL_BF16, err
    assert n_strict > 0
    return err


def test_full_prefill_128k_sampled_rows():
    _prefill_full(WORKLOADS["prefill_128k"])


def test_full_prefill_512k_qcal_sampled_rows():
    _prefill_full(WORKLOADS["prefill_512k_qcal"])


def test_full_decode_16x512k_sampled_sequences():
    w = WORKLOADS["decode_512k"]
    x = decode_inputs(w, device=DEV)
    cfg = H.config_of(w)
    dec = H.Decode(cfg, DEV)
    dec.summarize(x["k"], x["q_lmk"])
    dec.step(x["q"], x["k"], x["v"])
    H.hils_sync_status()
    for b in (0, w.B - 1):
        dm = oracle.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K, nq=1, q_pos0=w.N - 1)
        q = to_np(x["q"][b:b + 1])[:, :, None, :]
        k, v, ql = (to_np(x[n][b:b + 1]) for n in ("k", "v", "q_lmk"))
        ks, bs = oracle.summaries(dm, k, ql)
        assert (np.abs(to_np(dec.k_sum[b:b + 1]) - ks) <= np.abs(ks) * 2.0 ** -8 + KSUM_ATOL).all()
        np.testing.assert_allclose(to_np(dec.b_sum[b:b + 1]), bs, rtol=0, atol=2e-5)
        rows = [(0, w.N - 1)]
        _, _, s_all, g_all = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
        idx_g = to_np(dec.idx[b:b + 1]).astype(np.int64)
        check_selection(idx_g, g_all, w.K)
        out_f = oracle.attend(dm, rows, q, k, v, idx_g, forced_s_sel(idx_g, s_all, w.G))
        err = np.abs(to_np(dec.out[b:b + 1]) - out_f).max()
        assert err <= TOL_BF16, err
        del k, v
