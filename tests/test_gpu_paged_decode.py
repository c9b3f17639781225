"""GPU parity of decode across steps on a paged, chunk-aligned cache, through
the C ABI: sequences of different lengths share one pool of one-chunk pages
(in shuffled order); summaries are built for the cache, one token per
sequence is appended (completing a chunk for some of them, whose summary is
then built from its landmark query), and the step scores, selects and attends
at each sequence's own length.  Each sequence is checked against the oracle
run on its own contiguous cache of that length."""
import numpy as np
import pytest
import torch

import oracle
from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, decode_inputs
from tests.parity import KSUM_ATOL, TOL_BF16, TOL_F32, check_selection, forced_s_sel, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _paged_case(w, lens, seed=3, spare_pages=5):
    """Pool of the logical caches' chunks in a shuffled page order."""
    x = decode_inputs(w)  # k, v [B, Hkv, L_max, d], q_lmk [B, Hq, C, d], q [B, Hq, d]
    B, S = w.B, w.S
    max_pages = -(-w.N // S)
    num_pages = B * max_pages + spare_pages
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages)
    kp = torch.zeros((num_pages, w.Hkv, S, w.d), dtype=x["k"].dtype)
    vp = torch.zeros_like(kp)
    kl = torch.nn.functional.pad(x["k"], (0, 0, 0, max_pages * S - w.N))
    vl = torch.nn.functional.pad(x["v"], (0, 0, 0, max_pages * S - w.N))
    for b in range(B):
        for c in range(max_pages):
            kp[perm[b, c]] = kl[b, :, c * S:(c + 1) * S]
            vp[perm[b, c]] = vl[b, :, c * S:(c + 1) * S]
    return x, kp, vp, torch.from_numpy(perm.astype(np.int32)), num_pages


def _run(w, lens):
    x, kp, vp, table, num_pages = _paged_case(w, lens)
    cfg = H.config_of(w)
    B, S = w.B, w.S
    d = {n: x[n].to(DEV) for n in ("q", "q_lmk")}
    kp, vp, table = kp.to(DEV), vp.to(DEV), table.to(DEV)
    # the pool holds each sequence's keys up to its full length; position
    # L_b - 1 is overwritten by the append below, so blank it first
    for b, L in enumerate(lens):
        c, j = (L - 1) // S, (L - 1) % S
        kp[table[b, c], :, j] = 0
        vp[table[b, c], :, j] = 0
    k_sum = torch.full((B, w.Hq, w.C, w.d), float("nan"), dtype=x["k"].dtype, device=DEV)
    b_sum = torch.full((B, w.Hq, w.C), float("nan"), dtype=torch.float32, device=DEV)
    before = torch.tensor([L - 1 for L in lens], dtype=torch.int32, device=DEV)
    after = torch.tensor(lens, dtype=torch.int32, device=DEV)
    H.hils_build_summaries_paged(cfg, H.paged(before, table, num_pages), kp, d["q_lmk"], k_sum, b_sum)
    # the new token: its key and value, and the landmark query of the chunk it completes
    k_new = torch.stack([x["k"][b, :, L - 1] for b, L in enumerate(lens)]).to(DEV).contiguous()
    v_new = torch.stack([x["v"][b, :, L - 1] for b, L in enumerate(lens)]).to(DEV).contiguous()
    q_lmk_new = torch.stack([x["q_lmk"][b, :, max(0, L // S - 1)] for b, L in enumerate(lens)]).to(DEV).contiguous()
    pg = H.paged(after, table, num_pages)
    H.hils_decode_append(cfg, pg, k_new, v_new, q_lmk_new, kp, vp, k_sum, b_sum)
    idx = torch.empty((B, w.Hkv, w.K), dtype=torch.int32, device=DEV)
    s_sel = torch.empty((B, w.Hq, w.K), dtype=torch.float32, device=DEV)
    out = torch.empty((B, w.Hq, w.d), dtype=x["k"].dtype, device=DEV)
    ws_s = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_SCORE_DECODE), DEV)
    ws_a = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_ATTN_DECODE), DEV)
    H.hils_score_topk_paged(cfg, d["q"], pg, k_sum, b_sum, idx, s_sel, ws_s)
    H.hils_attn_decode_paged(cfg, d["q"], kp, vp, pg, idx, s_sel, out, ws_a)
    H.hils_sync_status()
    tol_out = TOL_F32 if w.dtype == "f32" else TOL_BF16
    for b, L in enumerate(lens):
        dm = oracle.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, N=L, d=w.d, S=S, W=w.W, K=w.K, nq=1, q_pos0=L - 1)
        k, v = to_np(x["k"][b:b + 1, :, :L]), to_np(x["v"][b:b + 1, :, :L])
        C = L // S
        ql = to_np(x["q_lmk"][b:b + 1, :, :C])
        ks, bs = oracle.summaries(dm, k, ql)
        kg, bg = to_np(k_sum[b:b + 1, :, :C]), to_np(b_sum[b:b + 1, :, :C])
        if w.dtype == "f32":
            np.testing.assert_allclose(kg, ks, rtol=0, atol=1e-5)
        else:
            assert (np.abs(kg - ks) <= np.abs(ks) * 2.0 ** -8 + KSUM_ATOL).all()
        np.testing.assert_allclose(bg, bs, rtol=0, atol=2e-5)
        q = to_np(x["q"][b:b + 1])[:, :, None, :]
        _, _, s_all, g_all = oracle.select(dm, [(0, L - 1)], q, k_sum=ks, b_sum=bs, want_all=True)
        idx_g = to_np(idx[b:b + 1]).astype(np.int64)
        check_selection(idx_g, g_all, w.K)
        ref = oracle.attend(dm, [(0, L - 1)], q, k, v, idx_g, forced_s_sel(idx_g, s_all, w.G))
        err = np.abs(to_np(out[b:b + 1]) - ref).max()
        assert err <= tol_out, (b, L, err)


def test_paged_decode_bf16_variable_lengths():
    # lengths: mid-chunk, completing a chunk on this step, and short of one window
    w = WORKLOADS["decode_512k"].scaled(name="paged", B=4, N=8192 + 64, K=8)
    _run(w, [4096 + 37, 8192, 6000, 300])


def test_paged_decode_fp32_variable_lengths():
    w = WORKLOADS["tiny_f32"].scaled(name="paged_f32", B=3, N=2048, Hq=8, Hkv=2, decode=True)
    _run(w, [2048, 1000, 33])


def test_paged_bad_page_is_reported_not_read():
    w = WORKLOADS["decode_512k"].scaled(name="paged_bad", B=2, N=4096, K=8)
    x, kp, vp, table, num_pages = _paged_case(w, [4096, 4096])
    cfg = H.config_of(w)
    table[1, 5] = num_pages + 100  # outside the pool
    pg_lens = torch.tensor([4096, 4096], dtype=torch.int32, device=DEV)
    table = table.to(DEV)
    kp, vp = kp.to(DEV), vp.to(DEV)
    pg = H.paged(pg_lens, table, num_pages)
    k_sum = torch.zeros((w.B, w.Hq, w.C, w.d), dtype=torch.bfloat16, device=DEV)
    b_sum = torch.zeros((w.B, w.Hq, w.C), dtype=torch.float32, device=DEV)
    H.hils_build_summaries_paged(cfg, pg, kp, x["q_lmk"].to(DEV), k_sum, b_sum)
    with pytest.raises(H.HilsError) as ei:
        H.hils_sync_status()
    assert ei.value.status == H.HILS_ERR_INVALID_ARG
    H.hils_sync_status()  # cleared
