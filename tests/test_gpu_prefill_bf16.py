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
from tests.parity import KSUM_ATOL, TOL_BF16, check_selection, forced_s_sel, to_np

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


def _run_forced(w, x, chunked=True):
    """chunked: the chunk-major pass with its workspace; otherwise the pass
    without scratch (each block streams its chunk union)."""
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
    cfg = H.config_of(w)
    ws = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_ATTN_PREFILL), DEV) if chunked else None
    H.hils_attn_prefill(cfg, d["q"], d["k"], d["v"], idx_t.int().contiguous(), ssel_t.contiguous(), out, ws)
    H.hils_sync_status()
    del ws
    rows = sample_rows(w, x["needles"])
    ridx = np.array([b * w.N + p for b, p in rows])
    ref = oracle.attend(dm, rows, q, k, v, idx[ridx], ssel32[ridx].astype(np.float64))
    got = to_np(out).transpose(0, 2, 1, 3).reshape(w.B * w.N, w.Hq, w.d)[ridx]
    return np.abs(got - ref).max(), got, ref


PASSES = pytest.mark.parametrize("chunked", [True, False], ids=["chunk_major", "union_stream"])


@PASSES
def test_attn_forced_selection_8k(chunked):
    w = WORKLOADS["prefill_8k"]
    err, _, _ = _run_forced(w, prefill_inputs(w), chunked)
    assert err <= TOL_BF16, err


@PASSES
def test_attn_forced_selection_ragged_tail_and_batch(chunked):
    w = WORKLOADS["prefill_8k"].scaled(name="ragged", B=2, N=4096 + 45, Hq=8, Hkv=2, K=8, needles_per_head=2)
    err, _, _ = _run_forced(w, prefill_inputs(w), chunked)
    assert err <= TOL_BF16, err


@PASSES
def test_attn_forced_selection_long_context_reduced(chunked):
    # the 128K workload's K and window on a shorter sequence and fewer heads
    w = WORKLOADS["prefill_128k"].scaled(name="p128r", N=32768, Hq=8, Hkv=2, needles_per_head=8)
    err, _, _ = _run_forced(w, prefill_inputs(w), chunked)
    assert err <= TOL_BF16, err


@PASSES
def test_attn_forced_selection_wide_window_k64(chunked):
    # the 512K workload's K = 64 and W = 1024 on a short sequence
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="k64r", N=16384, Hq=4, Hkv=1, d_model=0, qcal_rank=0,
                                              needles_per_head=4)
    err, _, _ = _run_forced(w, prefill_inputs(w), chunked)
    assert err <= TOL_BF16, err


@PASSES
@pytest.mark.parametrize("window", [64, 192], ids=["one_chunk", "three_chunks"])
def test_attn_forced_selection_odd_window_chunk_counts(chunked, window):
    """Windows of 1 and 3 chunks: the window kernel takes chunks two at a time,
    so every item of these windows pads its last tile with a chunk whose keys
    all lie after the position (masked), not only the first items of a
    sequence."""
    w = WORKLOADS["prefill_8k"].scaled(name=f"w{window}", B=2, N=3000 + 19, Hq=8, Hkv=2, W=window, K=8,
                                       needles_per_head=2)
    err, _, _ = _run_forced(w, prefill_inputs(w), chunked)
    assert err <= TOL_BF16, err


def test_attn_forced_selection_several_position_tiles():
    """B Hkv K = 1024 partial records per position: 8 GiB hold 8192 positions,
    so this sequence runs as two position tiles (4544 + 4456, multiples of a
    chunk)."""
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="tiles", B=4, N=9000, Hq=16, Hkv=4, d_model=0, qcal_rank=0,
                                              needles_per_head=2)
    assert w.B * w.Hkv * w.K == 1024
    err, _, _ = _run_forced(w, prefill_inputs(w))
    assert err <= TOL_BF16, err


def test_attn_chunk_major_graph_capture_matches_eager():
    """The chunk-major pass runs the next position tile's window kernel on an
    internal stream and joins it back with events.  Captured into a CUDA graph
    (two position tiles) and replayed, the call gives the eager output bit for
    bit; a side-stream launch left unjoined would make the capture fail."""
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="tiles", B=4, N=9000, Hq=16, Hkv=4, d_model=0, qcal_rank=0,
                                              needles_per_head=2)
    x = prefill_inputs(w)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v", "q_lmk")}
    pre = H.Prefill(H.config_of(w), DEV)
    pre.run(d["q"], d["k"], d["v"], d["q_lmk"])
    H.hils_sync_status()
    ref = pre.out.clone()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):  # one eager call on the capture stream first
        H.hils_attn_prefill(pre.cfg, d["q"], d["k"], d["v"], pre.idx, pre.s_sel, pre.out, pre.ws_attn, st)
    torch.cuda.synchronize()
    H.hils_sync_status()
    assert torch.equal(pre.out, ref)
    pre.out.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        H.hils_attn_prefill(pre.cfg, d["q"], d["k"], d["v"], pre.idx, pre.s_sel, pre.out, pre.ws_attn, st)
    g.replay()
    torch.cuda.synchronize()
    H.hils_sync_status()
    assert torch.equal(pre.out, ref)
    del g


def test_attn_chunk_major_is_deterministic_and_matches_union_stream():
    """Bucket order inside the chunk-major pass follows atomic arrival order;
    the output must not: two runs agree bit for bit.  The two passes compute
    the same quantity (within the bf16 tolerance)."""
    w = WORKLOADS["prefill_8k"].scaled(name="det", N=6000, Hq=8, Hkv=2, needles_per_head=2)
    x = prefill_inputs(w)
    _, a, _ = _run_forced(w, x, True)
    _, b, _ = _run_forced(w, x, True)
    _, c, _ = _run_forced(w, x, False)
    assert np.array_equal(a, b)
    assert np.abs(a - c).max() <= TOL_BF16


def test_attn_constant_values_pass_through():
    """v_j = u for all j gives out = u (the fusion weights sum to one)."""
    w = WORKLOADS["prefill_8k"].scaled(name="const", N=4096, Hq=8, Hkv=2, needles_per_head=0)
    x = prefill_inputs(w)
    u = torch.randn(w.d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    x["v"] = u.expand_as(x["v"]).contiguous()
    err, got, _ = _run_forced(w, x)
    assert np.abs(got - to_np(u)).max() <= 1e-2


def _e2e(w, x, all_rows_select=True):
    """Run the whole bf16 prefill through the C ABI and check every stage."""
    dm = _dims(w)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v", "q_lmk")}
    qc = (x["h"].to(DEV), x["w_down"].to(DEV), x["w_up"].to(DEV)) if w.d_model else None
    pre = H.Prefill(H.config_of(w), DEV, qcal_rank=w.qcal_rank)
    pre.run(d["q"], d["k"], d["v"], d["q_lmk"], qcal=qc)
    H.hils_sync_status()
    q, k, v, ql = (to_np(x[n]) for n in ("q", "k", "v", "q_lmk"))
    ks, bs = oracle.summaries(dm, k, ql)
    excess = np.abs(to_np(pre.k_sum) - ks) - np.abs(ks) * 2.0 ** -8
    assert excess.max() <= KSUM_ATOL, excess.max()
    np.testing.assert_allclose(to_np(pre.b_sum), bs, rtol=0, atol=2e-5)
    rows = oracle.all_rows(w.B, w.N) if all_rows_select else sample_rows(w, x["needles"], n_random=2048)
    ridx = np.array([b * w.N + p for b, p in rows])
    qs = None
    if w.d_model:
        qs = oracle.qcal(dm, rows, q, to_np(x["h"]), to_np(x["w_down"]), to_np(x["w_up"]))
        # the scoring query sits at the start of the workspace, in the layout of q (bf16)
        qt = pre.ws[: w.B * w.Hq * w.N * w.d * 2].view(torch.bfloat16).view(w.B, w.Hq, w.N, w.d)
        qt = to_np(qt).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.d)[ridx]
        assert (np.abs(qt - qs) <= np.abs(qs) * 2.0 ** -8 + 2e-3).all(), np.abs(qt - qs).max()
    idx_or, ssel_or, s_all, g_all = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs, qs=qs, want_all=True)
    idx_g = to_np(pre.idx).astype(np.int64).transpose(0, 2, 1, 3).reshape(-1, w.Hkv, w.K)[ridx]
    n_strict, n = check_selection(idx_g, g_all, w.K)
    ssel_g = to_np(pre.s_sel).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.K)[ridx]
    ssel_f = forced_s_sel(idx_g, s_all, w.G)
    fin = np.isfinite(ssel_f)
    assert np.array_equal(fin, np.isfinite(ssel_g))
    score_err = np.abs(ssel_g[fin] - ssel_f[fin]).max() if fin.any() else 0.0
    assert score_err < 5e-3, score_err  # k' is stored in bf16; << the 1e-2 selection gap
    orows = sample_rows(w, x["needles"])
    oidx = np.array([b * w.N + p for b, p in orows])
    pos_in = {r: j for j, r in enumerate(ridx.tolist())}
    sel_rows = [pos_in[r] for r in oidx.tolist()]
    out_f = oracle.attend(dm, orows, q, k, v, idx_g[sel_rows], ssel_f[sel_rows])
    got = to_np(pre.out).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.d)[oidx]
    err = np.abs(got - out_f).max()
    assert err <= TOL_BF16, err
    # needle recall of the selection (information): needle chunk chosen for its query
    hit = 0
    for (b, hq, i, j) in x["needles"]:
        hit += int(j // w.S in to_np(pre.idx)[b, hq // w.G, i].tolist() or i // w.S - j // w.S < w.W // w.S)
    return dict(n_strict=n_strict, n=n, score_err=float(score_err), out_err=float(err),
                needle_recall=hit / max(1, len(x["needles"])))


def test_end_to_end_8k():
    w = WORKLOADS["prefill_8k"]
    r = _e2e(w, prefill_inputs(w))
    assert r["n_strict"] > 0


def test_end_to_end_long_context_reduced():
    w = WORKLOADS["prefill_128k"].scaled(name="p128r", N=32768, Hq=8, Hkv=2, needles_per_head=16)
    _e2e(w, prefill_inputs(w), all_rows_select=False)


def test_end_to_end_ragged_batch_k64():
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="k64b", B=2, N=12288 + 77, Hq=8, Hkv=2, d_model=0, qcal_rank=0,
                                              needles_per_head=4)
    _e2e(w, prefill_inputs(w))


def test_end_to_end_tiny_sequences():
    # fewer positions than one window, one 128-row tile, a partial tile
    for n in (100, 576, 700):
        w = WORKLOADS["prefill_8k"].scaled(name=f"n{n}", N=n, Hq=4, Hkv=1, needles_per_head=0)
        _e2e(w, prefill_inputs(w))


@pytest.mark.parametrize("K", [8, 32, 48])
def test_score_exact_ties_take_smaller_chunks(K):
    """k' = 0 and whole-number b' make every surrogate score exact (s^ = b')
    and make most group scores tie.  The chosen chunks must then be the
    oracle's bit for bit: among equal group scores the smaller chunk wins,
    across the two 32-chunk halves of a tile and across tiles, and each s^ is
    the chunk's own b'.  K = 8, 32 and 48 cover the three list lengths of the
    kernel (16, 32, 64) and both ways of writing the result."""
    w = WORKLOADS["prefill_8k"].scaled(name=f"tie{K}", B=2, N=64 * 300 + 17, Hq=8, Hkv=2, K=K, W=128,
                                       needles_per_head=0)
    dm = _dims(w)
    C = w.N // w.S
    gen = torch.Generator().manual_seed(101 + K)
    q = torch.randn((w.B, w.Hq, w.N, w.d), generator=gen).to(torch.bfloat16)
    b_sum = torch.randint(0, 4, (w.B, w.Hq, C), generator=gen).float()
    k_sum = torch.zeros((w.B, w.Hq, C, w.d), dtype=torch.bfloat16)
    idx = torch.empty((w.B, w.Hkv, w.N, K), dtype=torch.int32, device=DEV)
    s_sel = torch.empty((w.B, w.Hq, w.N, K), dtype=torch.float32, device=DEV)
    H.hils_score_topk(H.config_of(w), q.to(DEV), k_sum.to(DEV), b_sum.to(DEV), idx, s_sel)
    H.hils_sync_status()
    rows = oracle.all_rows(w.B, w.N)
    idx_o, ssel_o = oracle.select(dm, rows, to_np(q), k_sum=np.zeros((w.B, w.Hq, C, w.d)),
                                  b_sum=b_sum.numpy().astype(np.float64))
    got_idx = idx.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, w.Hkv, K)
    assert np.array_equal(got_idx, idx_o)
    got_s = s_sel.cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, w.Hq, K)
    assert np.array_equal(got_s, ssel_o.astype(np.float32))


@pytest.mark.parametrize("stage", ["score", "qcal", "attn"])
def test_prefill_wait_timeout_reports_status(stage):
    """The kernels that wait on tile copies (scoring, Q-Cal, attention) report a
    wait that runs out, return, and leave the context usable."""
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="to", N=2048, Hq=4, Hkv=1, needles_per_head=0)
    x = {n: t.to(DEV) for n, t in prefill_inputs(w).items() if isinstance(t, torch.Tensor)}
    qc = (x["h"], x["w_down"], x["w_up"])
    pre = H.Prefill(H.config_of(w), DEV, qcal_rank=w.qcal_rank)
    pre.run(x["q"], x["k"], x["v"], x["q_lmk"])
    H.hils_sync_status()
    try:
        H.hils_set_wait_budget(2_000_000)
        H.hils_set_fault_injection(1)
        if stage == "attn":
            H.hils_attn_prefill(pre.cfg, x["q"], x["k"], x["v"], pre.idx, pre.s_sel, pre.out, pre.ws_attn)
        else:
            H.hils_score_topk(pre.cfg, x["q"], pre.k_sum, pre.b_sum, pre.idx, pre.s_sel, pre.ws,
                              qcal=qc if stage == "qcal" else None)
        with pytest.raises(H.HilsError) as ei:
            H.hils_sync_status()
        assert ei.value.status == H.HILS_ERR_TIMEOUT
    finally:
        H.hils_set_fault_injection(0)
        H.hils_set_wait_budget(0)
    pre.run(x["q"], x["k"], x["v"], x["q_lmk"])
    H.hils_sync_status()
    assert torch.isfinite(pre.out.float()).all()


def test_end_to_end_qcal_reduced():
    # the 512K Q-Cal workload's K, window, rank and d_model on a shorter sequence
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="qcal_r", N=8192, Hq=8, Hkv=2, needles_per_head=8)
    _e2e(w, prefill_inputs(w))


def test_qcal_zero_up_projection_changes_nothing():
    w = WORKLOADS["prefill_512k_qcal"].scaled(name="qcal0", N=4096, Hq=8, Hkv=2, needles_per_head=0)
    x = {n: t.to(DEV) for n, t in prefill_inputs(w).items() if isinstance(t, torch.Tensor)}
    base = H.Prefill(H.config_of(w), DEV)
    base.run(x["q"], x["k"], x["v"], x["q_lmk"])
    qc = H.Prefill(H.config_of(w), DEV, qcal_rank=w.qcal_rank)
    qc.run(x["q"], x["k"], x["v"], x["q_lmk"], qcal=(x["h"], x["w_down"], torch.zeros_like(x["w_up"])))
    H.hils_sync_status()
    assert torch.equal(base.idx, qc.idx)
    assert torch.equal(base.s_sel, qc.s_sel)
    # the same selection through deterministic kernels: the same bits
    assert torch.equal(base.out, qc.out)


def _list_form(lst, ncand):
    """The list form every attention pass accepts (include/hils.h): strictly
    ascending candidates, then -1.  Entries that break it become -1."""
    out, prev = [], -1
    for c in lst:
        out.append(int(c) if 0 <= c < ncand and c > prev else -1)
        prev = 1 << 30 if c < 0 else max(prev, int(c))
    return out


@PASSES
def test_bad_list_entries_are_dropped_and_reported(chunked):
    """A duplicate, a -7 and a non-ascending pair in the bf16 path: those
    entries (and, after the -7, the rest of its list) are dropped by both
    passes, hils_sync_status reports HILS_ERR_INVALID_ARG, and every row
    equals the oracle run on the cleaned lists."""
    w = WORKLOADS["prefill_8k"].scaled(name="badidx", N=4096, Hq=8, Hkv=2, needles_per_head=0)
    x = prefill_inputs(w)
    dm = _dims(w)
    q, k, v, ql = (to_np(x[n]) for n in ("q", "k", "v", "q_lmk"))
    ks, bs = oracle.summaries(dm, k, ql)
    rows_all = oracle.all_rows(w.B, w.N)
    idx, ssel = oracle.select(dm, rows_all, q, k_sum=ks, b_sum=bs)  # [N, Hkv, K]
    bad = idx.copy()
    p_dup, p_neg, p_swap = 3000, 3500, 4095
    assert (bad[[p_dup, p_neg, p_swap]] >= 0).all()  # full lists
    bad[p_dup, 0, 5] = bad[p_dup, 0, 4]
    bad[p_neg, 1, 2] = -7
    bad[p_swap, 0, 7], bad[p_swap, 0, 8] = idx[p_swap, 0, 8], idx[p_swap, 0, 7]
    clean = bad.copy()
    for p in (p_dup, p_neg, p_swap):
        for g in range(w.Hkv):
            clean[p, g] = _list_form(bad[p, g], max(0, p // w.S - w.W // w.S + 1))
    assert (clean != idx).sum() >= 1 + 13 + 1
    idx_t = torch.from_numpy(bad.reshape(w.B, w.N, w.Hkv, w.K).transpose(0, 2, 1, 3).copy()).int().to(DEV)
    ssel32 = ssel.astype(np.float32)
    ssel_t = torch.from_numpy(ssel32.reshape(w.B, w.N, w.Hq, w.K).transpose(0, 2, 1, 3).copy()).to(DEV)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v")}
    out = torch.empty((w.B, w.Hq, w.N, w.d), dtype=torch.bfloat16, device=DEV)
    cfg = H.config_of(w)
    ws = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_ATTN_PREFILL), DEV) if chunked else None
    H.hils_attn_prefill(cfg, d["q"], d["k"], d["v"], idx_t.contiguous(), ssel_t.contiguous(), out, ws)
    with pytest.raises(H.HilsError) as ei:
        H.hils_sync_status()
    assert ei.value.status == H.HILS_ERR_INVALID_ARG
    H.hils_sync_status()  # cleared
    rows = [(0, p) for p in (0, 700, 2999, p_dup, p_neg, p_swap)]
    ridx = np.array([p for _, p in rows])
    ref = oracle.attend(dm, rows, q, k, v, clean[ridx], ssel32[ridx].astype(np.float64))
    got = to_np(out).transpose(0, 2, 1, 3).reshape(w.N, w.Hq, w.d)[ridx]
    assert np.abs(got - ref).max() <= TOL_BF16


def test_landmark_free_summaries_and_prefill():
    """The landmark-free variant (one shared query per head): its summaries
    equal the per-chunk call given that query tiled over the chunks (bit for
    bit), match the oracle, and drive an end-to-end prefill that passes the
    selection and output checks."""
    w = WORKLOADS["prefill_8k"].scaled(name="lmkfree", N=6144 + 40, Hq=8, Hkv=2, needles_per_head=4)
    x = prefill_inputs(w)
    qs = torch.randn((w.Hq, w.d), generator=torch.Generator().manual_seed(11)).to(torch.bfloat16)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v")}
    qs_d = qs.to(DEV)
    cfg = H.config_of(w)
    ks_a = torch.empty((w.B, w.Hq, w.C, w.d), dtype=torch.bfloat16, device=DEV)
    bs_a = torch.empty((w.B, w.Hq, w.C), dtype=torch.float32, device=DEV)
    H.hils_build_summaries_shared(cfg, d["k"], qs_d, ks_a, bs_a)
    tiled = qs_d[None, :, None, :].expand(w.B, w.Hq, w.C, w.d).contiguous()
    ks_b, bs_b = torch.empty_like(ks_a), torch.empty_like(bs_a)
    H.hils_build_summaries(cfg, d["k"], tiled, ks_b, bs_b)
    H.hils_sync_status()
    assert torch.equal(ks_a, ks_b) and torch.equal(bs_a, bs_b)
    dm = _dims(w)
    q, k, v = (to_np(x[n]) for n in ("q", "k", "v"))
    ks, bs = oracle.summaries_shared(dm, k, to_np(qs))
    assert (np.abs(to_np(ks_a) - ks) - np.abs(ks) * 2.0 ** -8).max() <= KSUM_ATOL
    np.testing.assert_allclose(to_np(bs_a), bs, rtol=0, atol=2e-5)
    pre = H.Prefill(cfg, DEV)
    pre.run(d["q"], d["k"], d["v"], qs_d, shared_lmk=True)
    H.hils_sync_status()
    rows = sample_rows(w, x["needles"])
    ridx = np.array([p for _, p in rows])
    _, _, s_all, g_all = oracle.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    idx_g = to_np(pre.idx).astype(np.int64).transpose(0, 2, 1, 3).reshape(-1, w.Hkv, w.K)[ridx]
    check_selection(idx_g, g_all, w.K)
    out_f = oracle.attend(dm, rows, q, k, v, idx_g, forced_s_sel(idx_g, s_all, w.G))
    got = to_np(pre.out).transpose(0, 2, 1, 3).reshape(-1, w.Hq, w.d)[ridx]
    assert np.abs(got - out_f).max() <= TOL_BF16
