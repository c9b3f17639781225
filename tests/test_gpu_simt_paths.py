"""GPU parity of the fp32 prefill path, the decode path (fp32 and bf16) and
the summary kernel, through the C ABI, against the oracle on the same seeded
inputs; plus the bounded-wait and bad-index status paths."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, decode_inputs, prefill_inputs
from tests.parity import KSUM_ATOL, TOL_BF16, TOL_F32, check_selection, forced_s_sel, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dims(w, decode=False):
    if decode:
        return oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K, nq=1, q_pos0=w.N - 1)
    return oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K)


def _to_dev(x):
    return {k: (v.to(DEV).contiguous() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def test_tiny_fp32_prefill_end_to_end():
    w = WORKLOADS["tiny_f32"]
    x = prefill_inputs(w)
    d = _to_dev(x)
    cfg = H.config_of(w)
    pre = H.Prefill(cfg, DEV)
    pre.run(d["q"], d["k"], d["v"], d["q_lmk"])
    H.hils_sync_status()
    dm = _dims(w)
    q, k, v, ql = (to_np(x[n]) for n in ("q", "k", "v", "q_lmk"))
    ks, bs = oracle.summaries(dm, k, ql)
    np.testing.assert_allclose(to_np(pre.k_sum), ks, rtol=0, atol=TOL_F32)
    np.testing.assert_allclose(to_np(pre.b_sum), bs, rtol=0, atol=TOL_F32)
    rows = oracle.all_rows(w.B, w.N)
    idx_or, ssel_or, s_all, g_all = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    idx_g = to_np(pre.idx).astype(np.int64).transpose(0, 2, 1, 3).reshape(-1, w.Hkv, w.K)
    check_selection(idx_g, g_all, w.K)
    ssel_g = to_np(pre.s_sel).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.K)
    ssel_f = forced_s_sel(idx_g, s_all, w.G)
    fin = np.isfinite(ssel_f)
    assert np.array_equal(fin, np.isfinite(ssel_g))
    np.testing.assert_allclose(ssel_g[fin], ssel_f[fin], rtol=0, atol=TOL_F32)
    out_f = oracle.attend(dm, rows, q, k, v, idx_g, ssel_f)
    out_g = to_np(pre.out).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.d)
    err = np.abs(out_g - out_f).max()
    assert err <= TOL_F32, err
    # the oracle's own end-to-end result agrees on rows whose sets agree
    same = (idx_g == idx_or).all(axis=(1, 2))
    assert same.mean() > 0.99
    out_or = oracle.attend(dm, rows, q, k, v, idx_or, ssel_or)
    assert np.abs(out_g[same] - out_or[same]).max() <= TOL_F32


def test_tiny_fp32_exact_window_rows():
    """Rows before any candidate chunk reduce to sliding-window attention."""
    w = WORKLOADS["tiny_f32"]
    x = prefill_inputs(w)
    d = _to_dev(x)
    pre = H.Prefill(H.config_of(w), DEV)
    pre.run(d["q"], d["k"], d["v"], d["q_lmk"])
    early = w.W  # positions < W have no candidates
    assert (to_np(pre.idx)[:, :, :early] == -1).all()
    assert np.isneginf(to_np(pre.s_sel)[:, :, :early]).all()


def _decode_check(w, tol):
    x = decode_inputs(w, device="cpu")
    d = _to_dev(x)
    cfg = H.config_of(w)
    dec = H.Decode(cfg, DEV)
    dec.summarize(d["k"], d["q_lmk"])
    dec.step(d["q"], d["k"], d["v"])
    H.hils_sync_status()
    dm = _dims(w, decode=True)
    q = to_np(x["q"])[:, :, None, :]
    k, v, ql = to_np(x["k"]), to_np(x["v"]), to_np(x["q_lmk"])
    ks, bs = oracle.summaries(dm, k, ql)
    if w.dtype == "f32":
        np.testing.assert_allclose(to_np(dec.k_sum), ks, rtol=0, atol=1e-5)
    else:  # one bf16 rounding of k'
        assert (np.abs(to_np(dec.k_sum) - ks) <= np.abs(ks) * 2.0 ** -8 + KSUM_ATOL).all()
    np.testing.assert_allclose(to_np(dec.b_sum), bs, rtol=0, atol=2e-5 if w.dtype == "bf16" else 1e-5)
    rows = [(b, w.N - 1) for b in range(w.B)]
    idx_or, ssel_or, s_all, g_all = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    idx_g = to_np(dec.idx).astype(np.int64)
    check_selection(idx_g, g_all, w.K)
    ssel_f = forced_s_sel(idx_g, s_all, w.G)
    out_f = oracle.attend(dm, rows, q, k, v, idx_g, ssel_f)
    err = np.abs(to_np(dec.out) - out_f).max()
    assert err <= tol, err
    return err


def test_decode_fp32_small():
    w = WORKLOADS["tiny_f32"].scaled(name="dec_f32", B=3, N=4096 + 17, Hq=8, Hkv=2, decode=True)
    _decode_check(w, TOL_F32)


def test_decode_bf16_reduced():
    w = WORKLOADS["decode_512k"].scaled(name="dec_bf16", B=2, N=16384)
    _decode_check(w, TOL_BF16)


def test_decode_bf16_partial_last_chunk():
    w = WORKLOADS["decode_512k"].scaled(name="dec_bf16_tail", B=2, N=16384 + 37, K=8)
    _decode_check(w, TOL_BF16)


def test_summaries_bf16_prefill_8k():
    w = WORKLOADS["prefill_8k"]
    x = prefill_inputs(w)
    d = _to_dev(x)
    cfg = H.config_of(w)
    ks_g = torch.empty((w.B, w.Hq, w.C, w.d), dtype=torch.bfloat16, device=DEV)
    bs_g = torch.empty((w.B, w.Hq, w.C), dtype=torch.float32, device=DEV)
    H.hils_build_summaries(cfg, d["k"], d["q_lmk"], ks_g, bs_g)
    H.hils_sync_status()
    ks, bs = oracle.summaries(_dims(w), to_np(x["k"]), to_np(x["q_lmk"]))
    # k' is stored in bf16: error bounded by one bf16 rounding of |k'| (< 2^-8 relative)
    err_k = np.abs(to_np(ks_g) - ks)
    assert (err_k <= np.abs(ks) * 2.0 ** -8 + KSUM_ATOL).all(), err_k.max()
    np.testing.assert_allclose(to_np(bs_g), bs, rtol=0, atol=2e-5)


def test_decode_wait_timeout_reports_status():
    # the fp32 decode kernel stages tiles with bounded waits (the bf16 one loads
    # straight into registers and has none)
    w = WORKLOADS["tiny_f32"].scaled(name="dec_to", B=1, N=4096, Hq=8, Hkv=2, decode=True)
    x = _to_dev(decode_inputs(w))
    dec = H.Decode(H.config_of(w), DEV)
    dec.summarize(x["k"], x["q_lmk"])
    H.hils_score_topk(dec.cfg, x["q"], dec.k_sum, dec.b_sum, dec.idx, dec.s_sel, dec.ws_score, True)
    H.hils_sync_status()
    try:
        H.hils_set_wait_budget(2_000_000)  # ~1 ms
        H.hils_set_fault_injection(1)
        H.hils_attn_decode(dec.cfg, x["q"], x["k"], x["v"], dec.idx, dec.s_sel, dec.out, dec.ws_attn)
        with pytest.raises(H.HilsError) as ei:
            H.hils_sync_status()
        assert ei.value.status == H.HILS_ERR_TIMEOUT
    finally:
        H.hils_set_fault_injection(0)
        H.hils_set_wait_budget(0)
    # the context is still usable and the status word was cleared
    H.hils_attn_decode(dec.cfg, x["q"], x["k"], x["v"], dec.idx, dec.s_sel, dec.out, dec.ws_attn)
    H.hils_sync_status()
    assert torch.isfinite(dec.out.float()).all()


def test_bad_index_is_skipped_and_reported():
    w = WORKLOADS["tiny_f32"]
    x = _to_dev(prefill_inputs(w))
    pre = H.Prefill(H.config_of(w), DEV)
    pre.run(x["q"], x["k"], x["v"], x["q_lmk"])
    H.hils_sync_status()
    idx = pre.idx.clone()
    idx[0, 0, w.N - 1, 0] = 10_000  # not a candidate of that position
    H.hils_attn_prefill(pre.cfg, x["q"], x["k"], x["v"], idx, pre.s_sel, pre.out)
    with pytest.raises(H.HilsError) as ei:
        H.hils_sync_status()
    assert ei.value.status == H.HILS_ERR_INVALID_ARG
    H.hils_sync_status()  # cleared


def test_landmark_free_summaries_fp32():
    """fp32 landmark-free summaries (one shared query per head) against the oracle."""
    w = WORKLOADS["tiny_f32"]
    x = prefill_inputs(w)
    qs = torch.randn((w.Hq, w.d), generator=torch.Generator().manual_seed(3))
    cfg = H.config_of(w)
    ks_g = torch.empty((w.B, w.Hq, w.C, w.d), dtype=torch.float32, device=DEV)
    bs_g = torch.empty((w.B, w.Hq, w.C), dtype=torch.float32, device=DEV)
    H.hils_build_summaries_shared(cfg, x["k"].to(DEV), qs.to(DEV), ks_g, bs_g)
    H.hils_sync_status()
    ks, bs = oracle.summaries_shared(_dims(w), to_np(x["k"]), to_np(qs))
    np.testing.assert_allclose(to_np(ks_g), ks, rtol=0, atol=TOL_F32)
    np.testing.assert_allclose(to_np(bs_g), bs, rtol=0, atol=TOL_F32)
