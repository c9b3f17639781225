"""Pins for the oracle: closed forms, invariants, special cases that reduce to
textbook attention, and brute force on tiny inputs.

None of these compares the oracle with itself: each expected value is either
hand-derived (``tests/golden/closed_forms.json``), a mathematical identity of
the method (the Taylor expansion of the chunk log-sum-exp is exact at its
expansion point; the Gibbs bound), or an independent brute-force computation
written here with numpy (dense causal softmax attention, softmax over an
explicit token set, a plain sort).
"""
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")
RNG = np.random.default_rng(1234)


def _ev(expr):
    return eval(expr, {"__builtins__": {}}, {"exp": math.exp, "log": math.log})


def _rand(*shape, scale=1.0):
    return (RNG.standard_normal(shape) * scale).astype(np.float32)


def _lse(x):
    m = np.max(x)
    return m + np.log(np.sum(np.exp(x - m)))


def _dense_causal(q, k, v, scale):
    """Textbook causal softmax attention, brute force. q [Hq,N,d], k/v [Hkv,N,d]."""
    Hq, N, d = q.shape
    G = Hq // k.shape[0]
    out = np.zeros((Hq, N, d))
    for h in range(Hq):
        kk = k[h // G].astype(np.float64)
        vv = v[h // G].astype(np.float64)
        for i in range(N):
            s = kk[: i + 1] @ q[h, i].astype(np.float64) * scale
            p = np.exp(s - s.max())
            out[h, i] = p @ vv[: i + 1] / p.sum()
    return out


def _softmax_over(q_i, kk, vv, tokens, scale):
    s = kk[tokens] @ q_i.astype(np.float64) * scale
    p = np.exp(s - s.max())
    return p @ vv[tokens] / p.sum()


def _window(i, S, W):
    nw = W // S
    first = i // S - nw + 1
    return list(range(max(0, first * S), i + 1))


def _small(B=1, Hq=4, Hkv=2, N=96, d=8, S=8, W=16, K=3):
    from oracle import Dims

    dm = Dims(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, S=S, W=W, K=K)
    q = _rand(B, Hq, N, d)
    k = _rand(B, Hkv, N, d)
    v = _rand(B, Hkv, N, d)
    ql = _rand(B, Hq, N // S, d)
    return dm, q, k, v, ql


# ---------------------------------------------------------------- golden ---

def test_golden_landmark_two_keys(oracle_mod):
    g = json.load(open(GOLDEN))["landmark_two_keys"]
    dm = oracle_mod.Dims(B=1, Hq=1, Hkv=1, N=2, d=2, S=2, W=2, K=1, scale=g["scale"])
    k = np.array(g["keys"], np.float32).reshape(1, 1, 2, 2)
    ql = np.array(g["q_lmk"], np.float32).reshape(1, 1, 1, 2)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    want_k = [_ev(e) for e in g["expected"]["k_sum"]]
    np.testing.assert_allclose(ks[0, 0, 0], want_k, rtol=0, atol=1e-14)
    assert abs(bs[0, 0, 0] - _ev(g["expected"]["b_sum"])) < 1e-14
    # s^ at q = q' (needs a query row after the window: use a longer toy sequence)
    dm2 = oracle_mod.Dims(B=1, Hq=1, Hkv=1, N=4, d=2, S=2, W=2, K=1, scale=g["scale"])
    k2 = np.zeros((1, 1, 4, 2), np.float32)
    k2[0, 0, :2] = g["keys"]
    ql2 = np.zeros((1, 1, 2, 2), np.float32)
    ql2[0, 0, 0] = g["q_lmk"]
    q2 = np.zeros((1, 1, 4, 2), np.float32)
    q2[0, 0, 3] = g["q_lmk"]
    ks2, bs2 = oracle_mod.summaries(dm2, k2, ql2)
    _, _, s_all, _ = oracle_mod.select(dm2, [(0, 3)], q2, k_sum=ks2, b_sum=bs2, want_all=True)
    assert abs(s_all[0, 0, 0] - _ev(g["expected"]["s_hat_at_q_equals_q_lmk"])) < 1e-14


@pytest.mark.parametrize("case", ["hierarchical_row", "hierarchical_row_tie"])
def test_golden_hierarchical_row(oracle_mod, case):
    allg = json.load(open(GOLDEN))
    base = allg["hierarchical_row"]
    g = allg[case]
    N = base["N"]
    dm = oracle_mod.Dims(B=1, Hq=1, Hkv=1, N=N, d=1, S=1, W=1, K=1, scale=base["scale"])
    q = np.zeros((1, 1, N, 1), np.float32)
    q[0, 0, 3, 0] = base["q_row3"]
    k = np.array(g["keys"], np.float32).reshape(1, 1, N, 1)
    v = np.array(g["values"], np.float32).reshape(1, 1, N, 1)
    ql = np.zeros((1, 1, N, 1), np.float32)  # S=1: the landmark query cannot matter
    res = oracle_mod.prefill(dm, q, k, v, ql, rows=[(0, 3)])
    assert res["idx"][0, 0, 0] == g["expected"]["idx_row3"]
    assert abs(res["out"][0, 0, 0] - _ev(g["expected"]["out_row3"])) < 1e-14


# ------------------------------------------------------------------ pins ---

def test_P1_taylor_identity_at_landmark_query(oracle_mod):
    """q = q'_{h,c}  =>  s^_{h,i,c} = LSE_{j in c} s_ij exactly (expansion point)."""
    dm, q, k, v, ql = _small()
    ks, bs = oracle_mod.summaries(dm, k, ql)
    i = dm.N - 1
    checks = []
    for h in range(dm.Hq):
        for c in range(0, i // dm.S - dm.W // dm.S + 1):
            qq = q.copy()
            qq[0, h, i] = ql[0, h, c]
            _, _, s_all, _ = oracle_mod.select(dm, [(0, i)], qq, k_sum=ks, b_sum=bs, want_all=True)
            kc = k[0, h // (dm.Hq // dm.Hkv), c * dm.S:(c + 1) * dm.S].astype(np.float64)
            lse = _lse(kc @ ql[0, h, c].astype(np.float64) / math.sqrt(dm.d))
            checks.append(abs(s_all[0, h, c] - lse))
    assert max(checks) < 1e-12


def test_P2_gibbs_bound(oracle_mod):
    """For any q, s^_{i,c} <= LSE_{j in c} s_ij (convexity of log-sum-exp)."""
    dm, q, k, v, ql = _small(N=128)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    rows = [(0, i) for i in range(dm.N)]
    _, _, s_all, _ = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    _, _, e_all, _ = oracle_mod.select(dm, rows, q, k=k, exact_mass=True, want_all=True)
    fin = np.isfinite(e_all)
    assert np.array_equal(fin, np.isfinite(s_all))
    assert fin.sum() > 100
    gap = e_all[fin] - s_all[fin]
    assert gap.min() > -1e-12
    assert gap.max() > 1e-3  # the bound is not trivially tight


def test_P3_entropy_range_and_limits(oracle_mod):
    dm, q, k, v, ql = _small()
    ks, bs = oracle_mod.summaries(dm, k, ql)
    assert bs.min() >= -1e-12 and bs.max() <= math.log(dm.S) + 1e-12
    # q' = 0: uniform p -> b' = log S and k' = mean key (the mean-pool case)
    ks0, bs0 = oracle_mod.summaries(dm, k, np.zeros_like(ql))
    np.testing.assert_allclose(bs0, math.log(dm.S), rtol=0, atol=1e-12)
    kk = k.astype(np.float64).reshape(dm.B, dm.Hkv, dm.C, dm.S, dm.d).mean(3)
    G = dm.Hq // dm.Hkv
    for h in range(dm.Hq):
        np.testing.assert_allclose(ks0[:, h], kk[:, h // G], rtol=0, atol=1e-12)
    # q' scaled onto one key: p -> one-hot, b' -> 0, k' -> that key
    c, j, h = 3, 5, 1
    big = ql.copy()
    big[0, h, c] = k[0, h // G, c * dm.S + j] * 1e3
    ks1, bs1 = oracle_mod.summaries(dm, k, big)
    assert bs1[0, h, c] < 1e-6
    np.testing.assert_allclose(ks1[0, h, c], k[0, h // G, c * dm.S + j], rtol=0, atol=1e-6)


def test_P4_chunk_size_one_is_token_topk(oracle_mod):
    """S = 1: b' = 0 and s^ = s_ij; with K >= |Cand| the output is dense causal attention."""
    from oracle import Dims

    N, d = 24, 4
    dm = Dims(B=1, Hq=2, Hkv=1, N=N, d=d, S=1, W=2, K=N)
    q, k, v = _rand(1, 2, N, d), _rand(1, 1, N, d), _rand(1, 1, N, d)
    ql = _rand(1, 2, N, d)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    assert np.abs(bs).max() < 1e-12
    rows = [(0, i) for i in range(N)]
    res = oracle_mod.prefill(dm, q, k, v, ql, rows=rows)
    # s^ equals the token logit
    _, _, s_all, _ = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    for i in range(N):
        for c in range(max(0, i - 1)):
            for h in range(2):
                assert abs(s_all[i, h, c] - float(q[0, h, i].astype(np.float64) @ k[0, 0, c].astype(np.float64)) / 2.0) < 1e-12
    dense = _dense_causal(q[0], k[0], v[0], 1.0 / math.sqrt(d))
    np.testing.assert_allclose(res["out"].transpose(1, 0, 2), dense, rtol=0, atol=1e-12)


def test_P5_exact_mass_full_selection_is_dense_attention(oracle_mod):
    dm, q, k, v, ql = _small(K=64)
    res = oracle_mod.prefill(dm, q, k, v, ql, exact_mass=True)
    dense = _dense_causal(q[0], k[0], v[0], 1.0 / math.sqrt(dm.d))
    np.testing.assert_allclose(res["out"].reshape(dm.N, dm.Hq, dm.d).transpose(1, 0, 2), dense, rtol=0, atol=1e-12)


def test_P6_exact_mass_sparse_is_softmax_over_kept_tokens(oracle_mod):
    dm, q, k, v, ql = _small(K=2)
    res = oracle_mod.prefill(dm, q, k, v, ql, exact_mass=True)
    G = dm.Hq // dm.Hkv
    out = res["out"].reshape(dm.N, dm.Hq, dm.d)
    idx = res["idx"].reshape(dm.N, dm.Hkv, dm.K)
    # the selection must be the K largest exact group masses (ties: smaller c)
    _, _, e_all, g_all = oracle_mod.select(dm, res["rows"], q, k=k, exact_mass=True, want_all=True)
    worst = 0.0
    for i in range(dm.N):
        for g in range(dm.Hkv):
            gs = g_all[i, g]
            cand = np.flatnonzero(np.isfinite(gs))
            order = sorted(cand, key=lambda c: (-gs[c], c))
            want = sorted(order[: dm.K])
            got = [c for c in idx[i, g] if c >= 0]
            assert got == want
        for h in range(dm.Hq):
            kk = k[0, h // G].astype(np.float64)
            vv = v[0, h // G].astype(np.float64)
            toks = set(_window(i, dm.S, dm.W))
            for c in idx[i, h // G]:
                if c >= 0:
                    toks.update(range(c * dm.S, (c + 1) * dm.S))
            ref = _softmax_over(q[0, h, i], kk, vv, sorted(toks), 1.0 / math.sqrt(dm.d))
            worst = max(worst, np.abs(out[i, h] - ref).max())
    assert worst < 1e-12


def test_P7_constant_values_pass_through(oracle_mod):
    dm, q, k, v, ql = _small()
    u = _rand(dm.d)
    v = np.broadcast_to(u, v.shape).copy()
    res = oracle_mod.prefill(dm, q, k, v, ql)
    np.testing.assert_allclose(res["out"], np.broadcast_to(u.astype(np.float64), res["out"].shape), rtol=0, atol=1e-12)


def test_P8_early_rows_are_sliding_window_attention(oracle_mod):
    dm, q, k, v, ql = _small()
    nw = dm.W // dm.S
    rows = [(0, i) for i in range(nw * dm.S)]  # cur(i) < n_w: no candidate chunk
    res = oracle_mod.prefill(dm, q, k, v, ql, rows=rows)
    assert (res["idx"] == -1).all()
    G = dm.Hq // dm.Hkv
    for n, (_, i) in enumerate(rows):
        for h in range(dm.Hq):
            ref = _softmax_over(q[0, h, i], k[0, h // G].astype(np.float64), v[0, h // G].astype(np.float64),
                                _window(i, dm.S, dm.W), 1.0 / math.sqrt(dm.d))
            assert np.abs(res["out"][n, h] - ref).max() < 1e-12


def test_P9_permutation_inside_chunks(oracle_mod):
    dm, q, k, v, ql = _small()
    a = oracle_mod.prefill(dm, q, k, v, ql)
    perm = np.concatenate([c * dm.S + RNG.permutation(dm.S) for c in range(dm.C)])
    kp, vp = k.copy(), v.copy()
    kp[:, :, : dm.C * dm.S] = k[:, :, perm]
    vp[:, :, : dm.C * dm.S] = v[:, :, perm]
    b = oracle_mod.prefill(dm, q, kp, vp, ql)
    np.testing.assert_allclose(a["k_sum"], b["k_sum"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(a["b_sum"], b["b_sum"], rtol=0, atol=1e-12)
    # rows whose window holds only whole chunks are invariant: the last query of each chunk
    last_rows = [n for n, (_, i) in enumerate(a["rows"]) if (i + 1) % dm.S == 0]
    np.testing.assert_array_equal(a["idx"][last_rows], b["idx"][last_rows])
    np.testing.assert_allclose(a["out"][last_rows], b["out"][last_rows], rtol=0, atol=1e-12)


def test_P10_qcal_zero_correction(oracle_mod):
    dm, q, k, v, ql = _small()
    Dm, r = 16, 3
    h = _rand(dm.B, dm.N, Dm)
    wd = _rand(r, Dm)
    wu = np.zeros((dm.Hq * dm.d, r), np.float32)
    base = oracle_mod.prefill(dm, q, k, v, ql)
    for args in ((h, wd, wu), (np.zeros_like(h), wd, _rand(dm.Hq * dm.d, r))):
        res = oracle_mod.prefill(dm, q, k, v, ql, qcal_args=args)
        np.testing.assert_array_equal(res["idx"], base["idx"])
        np.testing.assert_array_equal(res["s_sel"], base["s_sel"])
        np.testing.assert_array_equal(res["out"], base["out"])


def test_qcal_identity_projection(oracle_mod):
    """W_down = I, W_up = I (r = d_model = Hq*d): the scoring query is q + h."""
    from oracle import Dims

    dm = Dims(B=1, Hq=2, Hkv=1, N=8, d=4, S=2, W=2, K=1)
    q = _rand(1, 2, 8, 4)
    Dm = 8
    h = _rand(1, 8, Dm)
    eye = np.eye(Dm, dtype=np.float32)
    rows = [(0, i) for i in range(8)]
    qs = oracle_mod.qcal(dm, rows, q, h, eye, eye)
    want = q[0].transpose(1, 0, 2).astype(np.float64) + h[0].reshape(8, 2, 4).astype(np.float64)
    np.testing.assert_allclose(qs, want, rtol=0, atol=1e-12)


def test_golden_qcal_layout(oracle_mod):
    """Hand-derived Q-Cal rows with non-square, non-symmetric W_down / W_up
    (tests/golden): a transposed read of either matrix, a swapped head/dim
    reshape or a wrong hidden-state row gives another answer."""
    from oracle import Dims

    g = json.load(open(GOLDEN))["qcal_layout"]
    Hq, d = g["Hq"], g["d"]
    dm = Dims(B=1, Hq=Hq, Hkv=1, N=2, d=d, S=1, W=1, K=1)
    q = np.full((1, Hq, 2, d), g["q_value"], np.float32)
    h = np.array(g["h"], np.float32).reshape(1, 2, g["d_model"])
    wd = np.array(g["w_down"], np.float32)
    wu = np.array(g["w_up"], np.float32)
    assert wd.shape == (g["r"], g["d_model"]) and wu.shape == (Hq * d, g["r"])
    qs = oracle_mod.qcal(dm, [(0, 0), (0, 1)], q, h, wd, wu)
    for n, key in enumerate(("q_tilde_pos0", "q_tilde_pos1")):
        want = np.array([[_ev(e) for e in row] for row in g["expected"][key]])
        np.testing.assert_array_equal(qs[n], want)


def test_P11_single_head_groups_select_by_sort(oracle_mod):
    from oracle import Dims

    dm = Dims(B=1, Hq=2, Hkv=2, N=160, d=8, S=8, W=16, K=5)
    q, k, ql = _rand(1, 2, 160, 8), _rand(1, 2, 160, 8), _rand(1, 2, 20, 8)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    rows = [(0, i) for i in range(160)]
    idx, s_sel, s_all, g_all = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    np.testing.assert_array_equal(g_all, s_all)  # G=1: the group max is the identity
    for n in range(160):
        for h in range(2):
            row = s_all[n, h]
            cand = np.flatnonzero(np.isfinite(row))
            order = cand[np.lexsort((cand, -row[cand]))]
            want = np.sort(order[: dm.K])
            got = idx[n, h][idx[n, h] >= 0]
            np.testing.assert_array_equal(got, want)
            np.testing.assert_array_equal(s_sel[n, h][: len(want)], row[want])


def test_group_max_and_own_head_weights(oracle_mod):
    """Selection ranks by the max over the group's heads; each head keeps its own s^."""
    dm, q, k, v, ql = _small(Hq=4, Hkv=1, K=2, N=128)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    rows = [(0, i) for i in range(dm.N)]
    idx, s_sel, s_all, g_all = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs, want_all=True)
    np.testing.assert_array_equal(g_all[:, 0], s_all.max(1))
    for n in range(dm.N):
        sel = idx[n, 0][idx[n, 0] >= 0]
        for h in range(dm.Hq):
            np.testing.assert_array_equal(s_sel[n, h][: len(sel)], s_all[n, h, sel])


def test_tie_break_prefers_smaller_chunk(oracle_mod):
    from oracle import Dims

    dm = Dims(B=1, Hq=1, Hkv=1, N=64, d=4, S=8, W=8, K=2)
    q, v = _rand(1, 1, 64, 4), _rand(1, 1, 64, 4)
    k = np.tile(_rand(1, 1, 8, 4), (1, 1, 8, 1))  # all chunks identical
    ql = np.tile(_rand(1, 1, 1, 4), (1, 1, 8, 1))
    res = oracle_mod.prefill(dm, q, k, v, ql, rows=[(0, 63)])
    assert list(res["idx"][0, 0]) == [0, 1]


def test_decode_row_equals_prefill_last_row(oracle_mod):
    from oracle import Dims

    dm, q, k, v, ql = _small(N=128)
    L = dm.N
    full = oracle_mod.prefill(dm, q, k, v, ql, rows=[(0, L - 1)])
    ddm = Dims(B=1, Hq=dm.Hq, Hkv=dm.Hkv, N=L, d=dm.d, S=dm.S, W=dm.W, K=dm.K, nq=1, q_pos0=L - 1)
    qd = q[:, :, L - 1:L]
    dec = oracle_mod.prefill(ddm, qd, k, v, ql, rows=[(0, L - 1)])
    np.testing.assert_array_equal(dec["idx"], full["idx"])
    np.testing.assert_allclose(dec["out"], full["out"], rtol=0, atol=1e-14)


def test_union_stats_bounds(oracle_mod):
    idx = np.array([[0, 1], [0, 1], [2, 3], [4, 5]])
    st = oracle_mod.union_stats(idx, (1, 2, 4))
    assert st[1] == 1.0 and st[2] == 1.5 and st[4] == 3.0


def test_landmark_free_zero_query_is_mean_pool(oracle_mod):
    """Landmark-free variant with the shared query 0: every chunk's p is uniform,
    so b' = log S and k' = the chunk's mean key (the mean-pool case)."""
    dm, q, k, v, ql = _small()
    ks, bs = oracle_mod.summaries_shared(dm, k, np.zeros((dm.Hq, dm.d), np.float32))
    np.testing.assert_allclose(bs, math.log(dm.S), rtol=0, atol=1e-12)
    kk = k.astype(np.float64).reshape(dm.B, dm.Hkv, dm.C, dm.S, dm.d).mean(3)
    G = dm.Hq // dm.Hkv
    for h in range(dm.Hq):
        np.testing.assert_allclose(ks[:, h], kk[:, h // G], rtol=0, atol=1e-12)


def test_landmark_free_same_keys_same_summary(oracle_mod):
    """One query shared by all chunks: two chunks holding the same keys (in any
    order) get the same k' and b'; with per-chunk queries they would not."""
    dm, q, k, v, ql = _small()
    G = dm.Hq // dm.Hkv
    k = k.copy()
    perm = RNG.permutation(dm.S)
    k[:, :, dm.S:2 * dm.S] = k[:, :, :dm.S][:, :, perm]
    qs = _rand(dm.Hq, dm.d)
    ks, bs = oracle_mod.summaries_shared(dm, k, qs)
    np.testing.assert_allclose(ks[:, :, 1], ks[:, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(bs[:, :, 1], bs[:, :, 0], rtol=0, atol=1e-12)
    # the shared query is the landmark query of head h for every chunk: check one
    # chunk of one head against its definition, the softmax-weighted key sum
    h, c = 1, 3
    kc = k[0, h // G, c * dm.S:(c + 1) * dm.S].astype(np.float64)
    l = kc @ qs[h].astype(np.float64) / math.sqrt(dm.d)
    p = np.exp(l - l.max())
    p /= p.sum()
    np.testing.assert_allclose(ks[0, h, c], p @ kc, rtol=0, atol=1e-12)
    assert abs(bs[0, h, c] + (p * np.log(p)).sum()) < 1e-12
