"""GPU parity of the prefill backward (hils_prefill_bwd) against the oracle's
backward, through the C ABI.

The oracle runs on the GPU forward's own intermediate values (its selection,
its chunk scores s_sel and its summaries k'), so that the comparison isolates
the backward arithmetic: attention backward with the GPU's s_sel, score
backward with the GPU's k', summary backward on the inputs.  The GPU kernels
compute in fp32 from exactly widened inputs, the oracle in fp64; the bound is
relative to each gradient's largest entry (sums over at most W + K S keys)."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, prefill_inputs
from tests.parity import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
RTOL_MAX = 1e-4  # |err| <= 1e-4 * max|gradient| (fp32 sums of <= W + K S terms)


def _backward_case(w, seed=5):
    x = prefill_inputs(w)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v", "q_lmk")}
    cfg = H.config_of(w)
    pre = H.Prefill(cfg, DEV)
    pre.run(d["q"], d["k"], d["v"], d["q_lmk"])
    H.hils_sync_status()
    gen = torch.Generator().manual_seed(seed)
    dout = torch.randn((w.B, w.Hq, w.N, w.d), generator=gen).to(w.torch_dtype)
    f32 = dict(dtype=torch.float32, device=DEV)
    dq = torch.full((w.B, w.Hq, w.N, w.d), float("nan"), **f32)
    dk = torch.full((w.B, w.Hkv, w.N, w.d), float("nan"), **f32)
    dv = torch.full_like(dk, float("nan"))
    dql = torch.full((w.B, w.Hq, w.C, w.d), float("nan"), **f32)
    dss = torch.full((w.B, w.Hq, w.N, w.K), float("nan"), **f32)
    ws = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_PREFILL_BWD), DEV)
    H.hils_prefill_bwd(cfg, d["q"], d["k"], d["v"], d["q_lmk"], pre.idx, pre.s_sel, pre.k_sum, dout.to(DEV), dq, dk,
                       dv, dql, ws, ds_sel=dss)
    H.hils_sync_status()
    # the oracle on the GPU forward's selection, scores and summaries
    dm = oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K)
    q, k, v, ql = (to_np(x[n]) for n in ("q", "k", "v", "q_lmk"))
    rows = oracle.all_rows(w.B, w.N)
    idx = to_np(pre.idx).astype(np.int64).transpose(0, 2, 1, 3).reshape(-1, w.Hkv, w.K)
    ssel = to_np(pre.s_sel).astype(np.float64).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.K)
    go = to_np(dout).astype(np.float64).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.d)
    dq_a, dk_a, dv_a, ds = oracle.attend_bwd(dm, rows, q, k, v, idx, ssel, go)
    dqs, dks, dbs = oracle.score_bwd(dm, rows, q, to_np(pre.k_sum), idx, ds)
    dk_s, dql_o = oracle.summaries_bwd(dm, k, ql, dks, dbs)
    ref = {"dq": dq_a + dqs.reshape(w.B, w.N, w.Hq, w.d).transpose(0, 2, 1, 3), "dk": dk_a + dk_s, "dv": dv_a,
           "dq_lmk": dql_o, "ds_sel": ds.reshape(w.B, w.N, w.Hq, w.K).transpose(0, 2, 1, 3)}
    got = {"dq": to_np(dq), "dk": to_np(dk), "dv": to_np(dv), "dq_lmk": to_np(dql), "ds_sel": to_np(dss)}
    errs = {}
    for n in ref:
        assert np.isfinite(got[n]).all(), n
        scale = np.abs(ref[n]).max()
        err = np.abs(got[n] - ref[n]).max()
        errs[n] = (err, scale)
        assert err <= RTOL_MAX * scale + 1e-7, (n, err, scale)
    return errs


def test_backward_fp32_tiny():
    errs = _backward_case(WORKLOADS["tiny_f32"])
    assert errs["dq_lmk"][1] > 0 and errs["ds_sel"][1] > 0  # every path carries gradient


def test_backward_fp32_groups_and_ragged_tail():
    w = WORKLOADS["tiny_f32"].scaled(name="bwd_g2", B=2, N=700 + 13, Hq=4, Hkv=2, d=32, S=16, W=64, K=5)
    _backward_case(w)


def test_backward_bf16_reduced():
    # the 8K workload's d, S, W and K on a shorter sequence with one KV group
    w = WORKLOADS["prefill_8k"].scaled(name="bwd_bf16", N=2048 + 40, Hq=4, Hkv=1, needles_per_head=2)
    _backward_case(w)


def test_backward_repeats():
    """dq and ds_sel come from one warp per row and repeat bit for bit.  dk, dv
    and dq_lmk sum the rows of a chunk in the order of its bucket list, which
    the scatter fills by atomic arrival, so repeats agree to fp32 rounding."""
    w = WORKLOADS["prefill_8k"].scaled(name="bwd_det", N=1024, Hq=4, Hkv=1, needles_per_head=0)
    x = {n: t.to(DEV) for n, t in prefill_inputs(w).items() if isinstance(t, torch.Tensor)}
    cfg = H.config_of(w)
    pre = H.Prefill(cfg, DEV)
    pre.run(x["q"], x["k"], x["v"], x["q_lmk"])
    dout = torch.randn_like(x["q"])
    ws = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_PREFILL_BWD), DEV)
    outs = []
    for _ in range(2):
        g = [torch.empty((w.B, w.Hq, w.N, w.d), dtype=torch.float32, device=DEV),
             torch.empty((w.B, w.Hkv, w.N, w.d), dtype=torch.float32, device=DEV),
             torch.empty((w.B, w.Hkv, w.N, w.d), dtype=torch.float32, device=DEV),
             torch.empty((w.B, w.Hq, w.C, w.d), dtype=torch.float32, device=DEV)]
        H.hils_prefill_bwd(cfg, x["q"], x["k"], x["v"], x["q_lmk"], pre.idx, pre.s_sel, pre.k_sum, dout, *g, ws)
        H.hils_sync_status()
        outs.append(g)
    (dq0, dk0, dv0, dl0), (dq1, dk1, dv1, dl1) = outs
    assert torch.equal(dq0, dq1)
    for a, b in ((dk0, dk1), (dv0, dv1), (dl0, dl1)):
        assert (a - b).abs().max().item() <= 1e-6 * a.abs().max().item()
