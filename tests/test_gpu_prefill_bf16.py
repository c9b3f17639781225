"""GPU parity of the bf16 prefill path against the oracle, through the C ABI.

Attention is first checked on its own (forced selection: the oracle's chunk
sets and scores are fed to hils_attn_prefill), so that selection ties cannot
mask an attention error; the end-to-end tests then check scoring, selection
and attention together with the tie-tolerant rule."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, prefill_inputs
from tests.parity import TOL_BF16, check_selection, forced_s_sel, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dims(w):
    return oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K)


def sample_rows(w, needles=(), n_random=256, seed=0):
    """Edge rows (first/last positions, chunk and 32-position block borders,
    the first rows with candidates, the ragged tail) plus needle rows and a
    seeded random sample."""
    N, S, W = w.N, w.S, w.W
    pos = {0, 1, N - 1, N - 2, W - 1, W, W + S - 1, W + S, W + S + 1}
    for c in (1, 2, 7, 8, 9, N // S // 2, N // S - 1):
        for off in (-1, 0, 31, 32, 63):
            pos.add(c * S + off)
    pos.update(i for (_, _, i, _) in needles)
    rng = np.random.default_rng(seed)
    pos.update(rng.integers(0, N, n_random).tolist())
    pos = sorted(p for p in pos if 0 <= p < N)
    return [(b, p) for b in range(w.B) for p in pos]


def _run_forced(w, x):
    dm = _dims(w)
    q, k, v, ql = (to_np(x[n]) for n in ("q", "k", "v", "q_lmk"))
    ks, bs = oracle.summaries(dm, k, ql)
    rows_all = oracle.all_rows(w.B, w.N)
    idx, ssel = oracle.select(dm, rows_all, q, k_sum=ks, b_sum=bs)
    idx_t = torch.from_numpy(idx.reshape(w.B, w.N, w.Hkv, w.K).transpose(0, 2, 1, 3).copy()).to(DEV)
    ssel32 = ssel.astype(np.float32)
    ssel_t = torch.from_numpy(ssel32.reshape(w.B, w.N, w.Hq, w.K).transpose(0, 2, 1, 3).copy()).to(DEV)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v")}
    out = torch.empty((w.B, w.Hq, w.N, w.d), dtype=torch.bfloat16, device=DEV)
    H.hils_attn_prefill(H.config_of(w), d["q"], d["k"], d["v"], idx_t.int().contiguous(), ssel_t.contiguous(), out)
    H.hils_sync_status()
    rows = sample_rows(w, x["needles"])
    ridx = np.array([b * w.N + p for b, p in rows])
    ref = oracle.attend(dm, rows, q, k, v, idx[ridx], ssel32[ridx].astype(np.float64))
    got = to_np(out).transpose(0, 2, 1, 3).reshape(w.B * w.N, w.Hq, w.d)[ridx]
    return np.abs(got - ref).max(), got, ref


def test_attn_forced_selection_8k():
    w = WORKLOADS["prefill_8k"]
    err, _, _ = _run_forced(w, prefill_inputs(w))
    assert err <= TOL_BF16, err


def test_attn_forced_selection_ragged_tail_and_batch():
    w = WORKLOADS["prefill_8k"].scaled(name="ragged", B=2, N=4096 + 45, Hq=8, Hkv=2, K=8, needles_per_head=2)
    err, _, _ = _run_forced(w, prefill_inputs(w))
    assert err <= TOL_BF16, err


def test_attn_forced_selection_long_context_reduced():
    # the 128K workload's K and window on a shorter sequence and fewer heads
    w = WORKLOADS["prefill_128k"].scaled(name="p128r", N=32768, Hq=8, Hkv=2, needles_per_head=8)
    err, _, _ = _run_forced(w, prefill_inputs(w))
    assert err <= TOL_BF16, err


def test_attn_forced_selection_wide_window_k64():
    # the 512K workload's K = 64 and W = 1024 on a short sequence
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="k64r", N=16384, Hq=4, Hkv=1, d_model=0, qcal_rank=0,
                                              needles_per_head=4)
    err, _, _ = _run_forced(w, prefill_inputs(w))
    assert err <= TOL_BF16, err


def test_attn_constant_values_pass_through():
    """v_j = u for all j gives out = u (the fusion weights sum to one)."""
    w = WORKLOADS["prefill_8k"].scaled(name="const", N=4096, Hq=8, Hkv=2, needles_per_head=0)
    x = prefill_inputs(w)
    u = torch.randn(w.d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    x["v"] = u.expand_as(x["v"]).contiguous()
    err, got, _ = _run_forced(w, x)
    assert np.abs(got - to_np(u)).max() <= 1e-2
