"""Pins for the oracle's backward pass (CPU, fp64).

The gradients are those of the forward pass with the chunk selection held
fixed (top-K is a discrete choice; hyper.ai summary of arXiv 2607.02980,
Method section: the loss reaches the chunk scores through the fusion weights
exp(s^)/Z^, and from them the landmark summaries and their queries).

Two independent checks pin them:

* central finite differences of the oracle's FORWARD functions (summaries,
  Q-Cal, scores at the fixed selection, attention) on tiny inputs, for every
  input tensor, Richardson-extrapolated;
* S = 1, no Q-Cal, K >= |Cand|: HiLS is dense causal softmax attention (every
  chunk is one key, b' = 0, s^ = s_ij), so its gradients are the textbook
  softmax-attention gradients, written here with numpy loops.
"""
import math

import numpy as np
import pytest

RNG = np.random.default_rng(77)


def _rand(*shape):
    return RNG.standard_normal(shape).astype(np.float32)


def _loss(oracle_mod, dm, q, k, v, ql, idx, gout, qcal_args=None):
    """sum(out * gout) of the forward pass at the fixed selection idx."""
    rows = oracle_mod.all_rows(dm.B, dm.N)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    qs = oracle_mod.qcal(dm, rows, q, *qcal_args) if qcal_args is not None else None
    _, _, s_all, _ = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs, qs=qs, want_all=True)
    G = dm.Hq // dm.Hkv
    sel = np.repeat(idx, G, axis=1)
    s_sel = np.where(sel >= 0, np.take_along_axis(s_all, np.maximum(sel, 0), axis=2), -np.inf)
    out = oracle_mod.attend(dm, rows, q, k, v, idx, s_sel)
    return float((out * gout).sum())


def _fd(f, x, coord, h=2.0 ** -11):
    """Central difference at one float32 coordinate, Richardson-extrapolated
    over steps h and h/2 (the perturbed values are re-read from the float32
    array, so the true step is used)."""
    def cd(step):
        xp, xm = x.copy(), x.copy()
        xp[coord] = x[coord] + np.float32(step)
        xm[coord] = x[coord] - np.float32(step)
        return (f(xp) - f(xm)) / (float(xp[coord]) - float(xm[coord]))
    d1, d2 = cd(h), cd(h / 2)
    return (4 * d2 - d1) / 3


def _case(oracle_mod, qcal=False, S=4):
    from oracle import Dims

    N, d = 48, 8
    dm = Dims(B=1, Hq=4, Hkv=2, N=N, d=d, S=S, W=2 * S, K=3)
    q, k, v = _rand(1, 4, N, d), _rand(1, 2, N, d), _rand(1, 2, N, d)
    ql = _rand(1, 4, N // S, d)
    qcal_args = None
    if qcal:
        Dm, r = 6, 2
        qcal_args = (_rand(1, N, Dm), 0.5 * _rand(r, Dm), 0.5 * _rand(4 * d, r))
    rows = oracle_mod.all_rows(1, N)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    qs = oracle_mod.qcal(dm, rows, q, *qcal_args) if qcal else None
    idx, _ = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs, qs=qs)
    assert (idx >= 0).sum() > 20
    gout = RNG.standard_normal((len(rows), 4, d))
    return dm, q, k, v, ql, qcal_args, idx, gout


@pytest.mark.parametrize("qcal", [False, True], ids=["plain", "qcal"])
def test_backward_matches_finite_differences(oracle_mod, qcal):
    dm, q, k, v, ql, qa, idx, gout = _case(oracle_mod, qcal)
    g = oracle_mod.prefill_bwd(dm, q, k, v, ql, idx, gout, qcal_args=qa)
    ins = {"q": q, "k": k, "v": v, "q_lmk": ql}
    if qa is not None:
        ins.update(h=qa[0], w_down=qa[1], w_up=qa[2])
    names = {"q": "dq", "k": "dk", "v": "dv", "q_lmk": "dq_lmk", "h": "dh", "w_down": "dw_down", "w_up": "dw_up"}

    def f_of(name):
        def f(x):
            a = dict(ins)
            a[name] = x
            qa2 = (a["h"], a["w_down"], a["w_up"]) if qa is not None else None
            return _loss(oracle_mod, dm, a["q"], a["k"], a["v"], a["q_lmk"], idx, gout, qa2)
        return f

    worst = 0.0
    for name, x in ins.items():
        grad = g[names[name]]
        assert grad.shape == x.shape, (name, grad.shape, x.shape)
        flat = RNG.choice(x.size, size=10, replace=False)
        # include the coordinates with the largest analytic gradient
        flat = np.concatenate([flat, np.argsort(-np.abs(grad).ravel())[:3]])
        f = f_of(name)
        for fl in flat:
            coord = np.unravel_index(fl, x.shape)
            num = _fd(f, x, coord)
            err = abs(num - grad[coord])
            worst = max(worst, err / (1e-6 + abs(num)))
            assert err <= 1e-6 + 1e-5 * abs(num), (name, coord, num, grad[coord])
    assert worst < 1e-5


def test_backward_chunk_size_one_is_dense_attention_gradient(oracle_mod):
    """S = 1, K >= |Cand|: the HiLS output is dense causal softmax attention, so
    dq, dk, dv must be its textbook gradients; the landmark queries get none
    (a one-key softmax is constant)."""
    from oracle import Dims

    N, d, Hq, Hkv = 20, 4, 2, 1
    dm = Dims(B=1, Hq=Hq, Hkv=Hkv, N=N, d=d, S=1, W=2, K=N)
    q, k, v, ql = _rand(1, Hq, N, d), _rand(1, Hkv, N, d), _rand(1, Hkv, N, d), _rand(1, Hq, N, d)
    rows = oracle_mod.all_rows(1, N)
    ks, bs = oracle_mod.summaries(dm, k, ql)
    idx, _ = oracle_mod.select(dm, rows, q, k_sum=ks, b_sum=bs)
    gout = RNG.standard_normal((N, Hq, d))
    g = oracle_mod.prefill_bwd(dm, q, k, v, ql, idx, gout)
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros((Hq, N, d))
    dk = np.zeros((N, d))
    dv = np.zeros((N, d))
    kk, vv = k[0, 0].astype(np.float64), v[0, 0].astype(np.float64)
    for h in range(Hq):
        for i in range(N):
            qi = q[0, h, i].astype(np.float64)
            s = kk[: i + 1] @ qi * scale
            p = np.exp(s - s.max())
            p /= p.sum()
            o = p @ vv[: i + 1]
            go = gout[i, h]
            ds = p * (vv[: i + 1] @ go - go @ o)
            dv[: i + 1] += np.outer(p, go)
            dq[h, i] = scale * ds @ kk[: i + 1]
            dk[: i + 1] += scale * np.outer(ds, qi)
    np.testing.assert_allclose(g["dq"][0], dq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dk"][0, 0], dk, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dv"][0, 0], dv, rtol=0, atol=1e-12)
    assert np.abs(g["dq_lmk"]).max() < 1e-12
