"""HiLS oracle: plain fp64 CPU restatement of Hierarchical Landmark Sparse attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it.

The arithmetic lives in ``hils_oracle.c`` (plain C, double precision); this
module compiles it with gcc on first use and exposes numpy wrappers.  Every
function follows the hyper.ai summary of arXiv 2607.02980 (HiLS-Attention),
section "方法" (Method):

* :func:`summaries`  -- landmark summaries k'_c (p-weighted key sum) and
  b'_c (entropy of p), the paragraph after the surrogate-score equation;
  :func:`summaries_shared` -- the landmark-free variant (one shared query
  per head, the last practical design choice);
* :func:`qcal`       -- the Q-Cal scoring query q + W_up W_down h (second
  practical design choice);
* :func:`select`     -- surrogate score s^ = q.k'/sqrt(d) + b', GQA group max,
  top-K over complete chunks before the chunk-aligned window (mode 0), or the
  exact chunk log-mass log Z_{i,c} of naive BSA (mode 1, "exact mass");
* :func:`attend`     -- hierarchical-softmax fusion: per-chunk softmax outputs
  weighted by exp(s^)/Z^ plus the window weighted by Z_swa/Z^.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, brute force and the hand-derived fixture in
``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hils_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libhils_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("B", "Hq", "Hkv", "N", "d", "S", "W", "K", "nq", "q_pos0")] + [
        ("scale", ctypes.c_double)
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            dims_p = ctypes.POINTER(_Dims)
            lib.hils_oracle_summaries.argtypes = [dims_p, P, P, P, P]
            lib.hils_oracle_qcal.argtypes = [dims_p, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int64, P, P, P, P, P]
            lib.hils_oracle_select.argtypes = [dims_p, ctypes.c_int, P, ctypes.c_int64, P, P, P, P, P, P, P, P, P]
            lib.hils_oracle_attend.argtypes = [dims_p, P, ctypes.c_int64, P, P, P, P, P, P, P]
            for f in (lib.hils_oracle_summaries, lib.hils_oracle_qcal, lib.hils_oracle_select, lib.hils_oracle_attend):
                f.restype = None
            _lib = lib
    return _lib


@dataclass(frozen=True)
class Dims:
    """Problem sizes, in the pages' notation (B, H_q, H_kv, N, d, S, W, K).

    ``nq``/``q_pos0`` describe where the stored query rows sit: prefill stores
    all N positions (nq=N, q_pos0=0); decode stores one query at L-1
    (nq=1, q_pos0=N-1).
    """

    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    S: int
    W: int
    K: int
    nq: int | None = None
    q_pos0: int = 0
    scale: float | None = None

    def c(self) -> _Dims:
        nq = self.N if self.nq is None else self.nq
        sc = 1.0 / math.sqrt(self.d) if self.scale is None else self.scale
        return _Dims(self.B, self.Hq, self.Hkv, self.N, self.d, self.S, self.W, self.K, nq, self.q_pos0, sc)

    @property
    def C(self) -> int:
        return self.N // self.S


def _f32(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.float32:
        a = a.astype(np.float32)
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows) -> np.ndarray:
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    return r


def summaries(dm: Dims, k, q_lmk):
    """k'_c [B,Hq,C,d] and b'_c [B,Hq,C] (float64) for every complete chunk."""
    lib = _load()
    k = _f32(k)
    q_lmk = _f32(q_lmk)
    assert k.shape == (dm.B, dm.Hkv, dm.N, dm.d), k.shape
    assert q_lmk.shape == (dm.B, dm.Hq, dm.C, dm.d), q_lmk.shape
    ks = np.empty((dm.B, dm.Hq, dm.C, dm.d), np.float64)
    bs = np.empty((dm.B, dm.Hq, dm.C), np.float64)
    cd = dm.c()
    lib.hils_oracle_summaries(ctypes.byref(cd), _ptr(k), _ptr(q_lmk), _ptr(ks), _ptr(bs))
    return ks, bs


def summaries_shared(dm: Dims, k, q_shared):
    """The landmark-free variant (Method section, last practical design
    choice: one shared learnable query per layer instead of per-chunk landmark
    queries), read as one query per query head [Hq, d] used by every chunk of
    every sequence: exactly :func:`summaries` with q'_{h,c} = q_shared[h]."""
    q_shared = _f32(q_shared)
    assert q_shared.shape == (dm.Hq, dm.d), q_shared.shape
    q_lmk = np.ascontiguousarray(np.broadcast_to(q_shared[None, :, None, :], (dm.B, dm.Hq, dm.C, dm.d)))
    return summaries(dm, k, q_lmk)


def qcal(dm: Dims, rows, q, h, w_down, w_up):
    """Q-Cal scoring queries [nrows, Hq, d] (float64) for the listed (b, position) rows."""
    lib = _load()
    rows = _rows(rows)
    q, h, w_down, w_up = _f32(q), _f32(h), _f32(w_down), _f32(w_up)
    r, dmod = w_down.shape
    assert w_up.shape == (dm.Hq * dm.d, r)
    out = np.empty((rows.shape[0], dm.Hq, dm.d), np.float64)
    cd = dm.c()
    lib.hils_oracle_qcal(ctypes.byref(cd), dmod, r, _ptr(rows), rows.shape[0], _ptr(q), _ptr(h), _ptr(w_down),
                         _ptr(w_up), _ptr(out))
    return out


def select(dm: Dims, rows, q, *, k=None, k_sum=None, b_sum=None, qs=None, exact_mass=False, want_all=False):
    """Chunk selection for the listed rows.

    Returns ``idx [nrows,Hkv,K]`` (int32, ascending, -1 padded), ``s_sel
    [nrows,Hq,K]`` (float64, -inf padded) and, with ``want_all``, the per-head
    scores ``s_all [nrows,Hq,C]`` and group scores ``g_all [nrows,Hkv,C]``.
    """
    lib = _load()
    rows = _rows(rows)
    n = rows.shape[0]
    q = _f32(q)
    k = None if k is None else _f32(k)
    if exact_mass:
        assert k is not None
    else:
        k_sum = np.ascontiguousarray(k_sum, np.float64)
        b_sum = np.ascontiguousarray(b_sum, np.float64)
    if qs is not None:
        qs = np.ascontiguousarray(qs, np.float64)
    idx = np.empty((n, dm.Hkv, dm.K), np.int32)
    s_sel = np.empty((n, dm.Hq, dm.K), np.float64)
    s_all = np.empty((n, dm.Hq, dm.C), np.float64) if want_all else None
    g_all = np.empty((n, dm.Hkv, dm.C), np.float64) if want_all else None
    cd = dm.c()
    lib.hils_oracle_select(ctypes.byref(cd), 1 if exact_mass else 0, _ptr(rows), n, _ptr(qs), _ptr(q), _ptr(k),
                           _ptr(None if exact_mass else k_sum), _ptr(None if exact_mass else b_sum), _ptr(idx),
                           _ptr(s_sel), _ptr(s_all), _ptr(g_all))
    if want_all:
        return idx, s_sel, s_all, g_all
    return idx, s_sel


def attend(dm: Dims, rows, q, k, v, idx, s_sel, want_lse=False):
    """Hierarchical-softmax attention output [nrows, Hq, d] (float64) for the listed rows."""
    lib = _load()
    rows = _rows(rows)
    n = rows.shape[0]
    q, k, v = _f32(q), _f32(k), _f32(v)
    idx = np.ascontiguousarray(idx, np.int32).reshape(n, dm.Hkv, dm.K)
    s_sel = np.ascontiguousarray(s_sel, np.float64).reshape(n, dm.Hq, dm.K)
    out = np.empty((n, dm.Hq, dm.d), np.float64)
    lse = np.empty((n, dm.Hq), np.float64) if want_lse else None
    cd = dm.c()
    lib.hils_oracle_attend(ctypes.byref(cd), _ptr(rows), n, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(s_sel),
                           _ptr(out), _ptr(lse))
    return (out, lse) if want_lse else out


def all_rows(B: int, N: int):
    """(b, i) for every position of every sequence."""
    b, i = np.meshgrid(np.arange(B), np.arange(N), indexing="ij")
    return np.stack([b.ravel(), i.ravel()], 1)


def prefill(dm: Dims, q, k, v, q_lmk, rows=None, *, qcal_args=None, exact_mass=False):
    """The whole forward path for the listed rows (default: all).

    Returns a dict with k_sum, b_sum, idx, s_sel, out (float64 where real).
    ``qcal_args`` = (h, w_down, w_up) enables the Q-Cal scoring query.
    """
    rows = all_rows(dm.B, dm.N) if rows is None else _rows(rows)
    res = {}
    if exact_mass:
        idx, s_sel = select(dm, rows, q, k=k, exact_mass=True)
    else:
        ks, bs = summaries(dm, k, q_lmk)
        qs = qcal(dm, rows, q, *qcal_args) if qcal_args is not None else None
        idx, s_sel = select(dm, rows, q, k_sum=ks, b_sum=bs, qs=qs)
        res.update(k_sum=ks, b_sum=bs, qs=qs)
    res.update(idx=idx, s_sel=s_sel, out=attend(dm, rows, q, k, v, idx, s_sel), rows=rows)
    return res


def union_stats(idx, M_list=(1, 2, 4, 8, 16)):
    """Mean size of the union of the chunk sets of M adjacent queries, divided by K.

    ``idx`` is [N, K] (one KV group of one sequence, -1 padded).  Rows with no
    candidate are skipped.  This is the reuse measure of the M-adjacent-query
    grouping in the Method section's hardware paragraph.
    """
    idx = np.asarray(idx)
    N, K = idx.shape
    out = {}
    for M in M_list:
        ratios = []
        for s in range(0, N - M + 1, M):
            blk = idx[s:s + M]
            sel = blk[blk >= 0]
            if sel.size == 0:
                continue
            ratios.append(len(np.unique(sel)) / K)
        out[M] = float(np.mean(ratios)) if ratios else float("nan")
    return out


# ------------------------------------------------------------- backward ---
# Gradients of the forward pass with the chunk selection held fixed (top-K is
# a discrete choice).  The fusion weights exp(s^)/Z^ carry the loss into the
# chunk scores, and from there into k', b' (the landmark summaries), q'_c and
# the keys, and into the Q-Cal weights (Method section: the factorised w_ij and
# Z^; the wmrh.cn article's point that the hierarchical softmax lets gradients
# reach the summaries).  Each function is a plain restatement in the C file.

def _bwd_lib():
    lib = _load()
    if not getattr(lib, "_bwd_ready", False):
        P, dims_p = ctypes.c_void_p, ctypes.POINTER(_Dims)
        lib.hils_oracle_attend_bwd.argtypes = [dims_p, P, ctypes.c_int64, P, P, P, P, P, P, P, P, P, P]
        lib.hils_oracle_score_bwd.argtypes = [dims_p, P, ctypes.c_int64, P, P, P, P, P, P, P, P]
        lib.hils_oracle_summaries_bwd.argtypes = [dims_p, P, P, P, P, P, P]
        lib.hils_oracle_qcal_bwd.argtypes = [dims_p, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int64, P, P, P, P,
                                             P, P, P]
        for f in (lib.hils_oracle_attend_bwd, lib.hils_oracle_score_bwd, lib.hils_oracle_summaries_bwd,
                  lib.hils_oracle_qcal_bwd):
            f.restype = None
        lib._bwd_ready = True
    return lib


def attend_bwd(dm: Dims, rows, q, k, v, idx, s_sel, dout):
    """Attention backward for the listed rows: dq [B,Hq,nq,d] (through the
    attention logits), dk, dv [B,Hkv,N,d] and ds_sel [nrows,Hq,K], the gradient
    of each chosen chunk's score s^ (float64)."""
    lib = _bwd_lib()
    rows = _rows(rows)
    n = rows.shape[0]
    q, k, v = _f32(q), _f32(k), _f32(v)
    idx = np.ascontiguousarray(idx, np.int32).reshape(n, dm.Hkv, dm.K)
    s_sel = np.ascontiguousarray(s_sel, np.float64).reshape(n, dm.Hq, dm.K)
    dout = np.ascontiguousarray(dout, np.float64).reshape(n, dm.Hq, dm.d)
    nq = dm.N if dm.nq is None else dm.nq
    dq = np.zeros((dm.B, dm.Hq, nq, dm.d))
    dk = np.zeros((dm.B, dm.Hkv, dm.N, dm.d))
    dv = np.zeros((dm.B, dm.Hkv, dm.N, dm.d))
    ds = np.zeros((n, dm.Hq, dm.K))
    cd = dm.c()
    lib.hils_oracle_attend_bwd(ctypes.byref(cd), _ptr(rows), n, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(s_sel),
                               _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds))
    return dq, dk, dv, ds


def score_bwd(dm: Dims, rows, q, k_sum, idx, ds_sel, qs=None):
    """Chunk-score backward: dqs [nrows,Hq,d] (gradient of the scoring query),
    dk_sum [B,Hq,C,d] and db_sum [B,Hq,C] (float64)."""
    lib = _bwd_lib()
    rows = _rows(rows)
    n = rows.shape[0]
    q = _f32(q)
    k_sum = np.ascontiguousarray(k_sum, np.float64)
    idx = np.ascontiguousarray(idx, np.int32).reshape(n, dm.Hkv, dm.K)
    ds_sel = np.ascontiguousarray(ds_sel, np.float64).reshape(n, dm.Hq, dm.K)
    qs = None if qs is None else np.ascontiguousarray(qs, np.float64)
    dqs = np.zeros((n, dm.Hq, dm.d))
    dks = np.zeros((dm.B, dm.Hq, dm.C, dm.d))
    dbs = np.zeros((dm.B, dm.Hq, dm.C))
    cd = dm.c()
    lib.hils_oracle_score_bwd(ctypes.byref(cd), _ptr(rows), n, _ptr(qs), _ptr(q), _ptr(k_sum), _ptr(idx),
                              _ptr(ds_sel), _ptr(dqs), _ptr(dks), _ptr(dbs))
    return dqs, dks, dbs


def summaries_bwd(dm: Dims, k, q_lmk, dk_sum, db_sum):
    """Summary backward: dk [B,Hkv,N,d] (through the summaries only) and
    dq_lmk [B,Hq,C,d] (float64)."""
    lib = _bwd_lib()
    k, q_lmk = _f32(k), _f32(q_lmk)
    dk_sum = np.ascontiguousarray(dk_sum, np.float64)
    db_sum = np.ascontiguousarray(db_sum, np.float64)
    dk = np.zeros((dm.B, dm.Hkv, dm.N, dm.d))
    dql = np.zeros((dm.B, dm.Hq, dm.C, dm.d))
    cd = dm.c()
    lib.hils_oracle_summaries_bwd(ctypes.byref(cd), _ptr(k), _ptr(q_lmk), _ptr(dk_sum), _ptr(db_sum), _ptr(dk),
                                  _ptr(dql))
    return dk, dql


def qcal_bwd(dm: Dims, rows, h, w_down, w_up, dqs):
    """Q-Cal backward: dh [B,nq,Dm], dw_down [r,Dm], dw_up [Hq d, r] (float64)."""
    lib = _bwd_lib()
    rows = _rows(rows)
    h, w_down, w_up = _f32(h), _f32(w_down), _f32(w_up)
    r, Dm = w_down.shape
    dqs = np.ascontiguousarray(dqs, np.float64)
    dh = np.zeros(h.shape)
    dwd = np.zeros((r, Dm))
    dwu = np.zeros((dm.Hq * dm.d, r))
    cd = dm.c()
    lib.hils_oracle_qcal_bwd(ctypes.byref(cd), Dm, r, _ptr(rows), rows.shape[0], _ptr(h), _ptr(w_down), _ptr(w_up),
                             _ptr(dqs), _ptr(dh), _ptr(dwd), _ptr(dwu))
    return dh, dwd, dwu


def prefill_bwd(dm: Dims, q, k, v, q_lmk, idx, dout, *, qcal_args=None):
    """Gradients of sum(out * dout) over every position, for the selection idx
    [B*N, Hkv, K] (rows in all_rows order) held fixed: a dict with dq, dk, dv,
    dq_lmk (and dh, dw_down, dw_up with Q-Cal), all float64."""
    rows = all_rows(dm.B, dm.N)
    ks, bs = summaries(dm, k, q_lmk)
    qs = qcal(dm, rows, q, *qcal_args) if qcal_args is not None else None
    _, _, s_all, _ = select(dm, rows, q, k_sum=ks, b_sum=bs, qs=qs, want_all=True)
    idx = np.ascontiguousarray(idx, np.int32).reshape(len(rows), dm.Hkv, dm.K)
    G = dm.Hq // dm.Hkv
    sel = np.repeat(idx, G, axis=1)
    s_sel = np.where(sel >= 0, np.take_along_axis(s_all, np.maximum(sel, 0), axis=2), -np.inf)
    dq, dk, dv, ds = attend_bwd(dm, rows, q, k, v, idx, s_sel, dout)
    dqs, dks, dbs = score_bwd(dm, rows, q, ks, idx, ds, qs=qs)
    dk2, dql = summaries_bwd(dm, k, q_lmk, dks, dbs)
    # the scoring query is q (+ the Q-Cal term): its gradient reaches q either way
    dq = dq + dqs.reshape(dm.B, dm.N, dm.Hq, dm.d).transpose(0, 2, 1, 3)
    res = dict(dq=dq, dk=dk + dk2, dv=dv, dq_lmk=dql, ds_sel=ds, dk_sum=dks, db_sum=dbs, s_sel=s_sel)
    if qcal_args is not None:
        dh, dwd, dwu = qcal_bwd(dm, rows, *qcal_args, dqs)
        res.update(dh=dh, dw_down=dwd, dw_up=dwu)
    return res
