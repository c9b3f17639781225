"""Thin Python binding of libhils.so (C ABI in include/hils.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch tensors supply device memory and the current CUDA stream.
The library is loaded from this package's directory; if it is missing the
first call raises (there is no fallback of any kind).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhils.so")

HILS_OK, HILS_ERR_INVALID_ARG, HILS_ERR_UNSUPPORTED, HILS_ERR_CUDA, HILS_ERR_TIMEOUT = range(5)
HILS_F32, HILS_BF16 = 0, 1
(HILS_WS_SCORE_PREFILL, HILS_WS_SCORE_DECODE, HILS_WS_ATTN_DECODE, HILS_WS_PREFILL_HOST, HILS_WS_ATTN_PREFILL,
 HILS_WS_PREFILL_BWD) = range(6)

EXPORTS = (
    "hils_build_summaries",
    "hils_build_summaries_shared",
    "hils_score_topk",
    "hils_attn_prefill",
    "hils_attn_decode",
    "hils_attn_decode_noalloc",
    "hils_prefill_host",
    "hils_prefill_bwd",
    "hils_decode_append",
    "hils_build_summaries_paged",
    "hils_score_topk_paged",
    "hils_attn_decode_paged",
    "hils_host_device_pointer",
    "hils_workspace_bytes",
    "hils_sync_status",
    "hils_last_error",
    "hils_set_wait_budget",
    "hils_set_fault_injection",
    "hils_version",
)


class HilsError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"hils status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("seq_len", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("chunk", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("query_block", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("dtype", ctypes.c_int32),
    ]


class QCal(ctypes.Structure):
    _fields_ = [
        ("h", ctypes.c_void_p),
        ("w_down", ctypes.c_void_p),
        ("w_up", ctypes.c_void_p),
        ("rank", ctypes.c_int32),
        ("d_model", ctypes.c_int32),
    ]


class Paged(ctypes.Structure):
    """A paged, chunk-aligned decode cache (include/hils.h, hils_paged_t)."""
    _fields_ = [
        ("seq_lens", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load libhils.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m chunk_wise_sparse_landmark_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, C = ctypes.c_void_p, ctypes.POINTER(Config)
        lib.hils_build_summaries.argtypes = [C, P, P, P, P, P]
        lib.hils_build_summaries_shared.argtypes = [C, P, P, P, P, P]
        lib.hils_score_topk.argtypes = [C, P, ctypes.POINTER(QCal), P, P, P, P, P, ctypes.c_size_t, ctypes.c_int32, P]
        lib.hils_attn_prefill.argtypes = [C, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.hils_attn_decode.argtypes = [C, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.hils_attn_decode_noalloc.argtypes = [C, P, P, P, P, P, P, P]
        lib.hils_prefill_host.argtypes = [C, P, P, P, P, ctypes.POINTER(QCal), P, P, ctypes.c_size_t, P]
        lib.hils_prefill_bwd.argtypes = [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.hils_host_device_pointer.argtypes = [P, ctypes.POINTER(ctypes.c_void_p)]
        lib.hils_host_device_pointer.restype = ctypes.c_int
        PG = ctypes.POINTER(Paged)
        lib.hils_decode_append.argtypes = [C, PG, P, P, P, P, P, P, P, P]
        lib.hils_build_summaries_paged.argtypes = [C, PG, P, P, P, P, P]
        lib.hils_score_topk_paged.argtypes = [C, P, PG, P, P, P, P, P, ctypes.c_size_t, P]
        lib.hils_attn_decode_paged.argtypes = [C, P, P, P, PG, P, P, P, P, ctypes.c_size_t, P]
        lib.hils_workspace_bytes.argtypes = [C, ctypes.c_int32, ctypes.c_int32]
        lib.hils_workspace_bytes.restype = ctypes.c_size_t
        lib.hils_sync_status.argtypes = [P]
        lib.hils_last_error.restype = ctypes.c_char_p
        lib.hils_set_wait_budget.argtypes = [ctypes.c_int64]
        lib.hils_set_wait_budget.restype = None
        lib.hils_set_fault_injection.argtypes = [ctypes.c_int32]
        lib.hils_set_fault_injection.restype = None
        lib.hils_version.restype = ctypes.c_char_p
        for n in ("hils_build_summaries", "hils_build_summaries_shared", "hils_score_topk", "hils_attn_prefill",
                  "hils_attn_decode", "hils_attn_decode_noalloc", "hils_prefill_host", "hils_prefill_bwd",
                  "hils_decode_append", "hils_build_summaries_paged", "hils_score_topk_paged",
                  "hils_attn_decode_paged", "hils_sync_status"):
            getattr(lib, n).restype = ctypes.c_int
        _lib = lib
    return _lib


def make_config(B, N, Hq, Hkv, d, S, W, K, dtype, M=0, scale=0.0) -> Config:
    dt = HILS_F32 if dtype in ("f32", torch.float32, HILS_F32) else HILS_BF16
    return Config(B, N, Hq, Hkv, d, S, W, K, M, scale, dt)


def config_of(w) -> Config:
    """Config for an :class:`inputs.Workload`."""
    return make_config(w.B, w.N, w.Hq, w.Hkv, w.d, w.S, w.W, w.K, w.dtype, M=w.M)


def _p(t: torch.Tensor | None):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int):
    if st != HILS_OK:
        raise HilsError(st, load().hils_last_error().decode())


def workspace_bytes(cfg: Config, which: int, qcal_rank: int = 0) -> int:
    n = load().hils_workspace_bytes(ctypes.byref(cfg), which, qcal_rank)
    if n == ctypes.c_size_t(-1).value:
        raise HilsError(HILS_ERR_INVALID_ARG, load().hils_last_error().decode())
    return n


def hils_build_summaries(cfg: Config, k, q_lmk, k_sum, b_sum, stream=None):
    _check(load().hils_build_summaries(ctypes.byref(cfg), _p(k), _p(q_lmk), _p(k_sum), _p(b_sum), _stream(stream)))


def hils_build_summaries_shared(cfg: Config, k, q_shared, k_sum, b_sum, stream=None):
    """Landmark-free summaries: q_shared [Hq, d] is every chunk's landmark query."""
    _check(load().hils_build_summaries_shared(ctypes.byref(cfg), _p(k), _p(q_shared), _p(k_sum), _p(b_sum),
                                              _stream(stream)))


def hils_score_topk(cfg: Config, q, k_sum, b_sum, idx, s_sel, workspace=None, decode=False, qcal=None, stream=None):
    """qcal: None or (h, w_down, w_up) tensors."""
    qc = None
    if qcal is not None:
        h, wd, wu = qcal
        qc = ctypes.byref(QCal(_p(h), _p(wd), _p(wu), wd.shape[0], wd.shape[1]))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hils_score_topk(ctypes.byref(cfg), _p(q), qc, _p(k_sum), _p(b_sum), _p(idx), _p(s_sel),
                                  _p(workspace), ws_bytes, 1 if decode else 0, _stream(stream)))


def hils_attn_prefill(cfg: Config, q, k, v, idx, s_sel, out, workspace=None, stream=None):
    """workspace: None (bf16: the pass without scratch) or a device buffer of
    workspace_bytes(cfg, HILS_WS_ATTN_PREFILL) bytes."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hils_attn_prefill(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(idx), _p(s_sel), _p(out),
                                    _p(workspace), ws_bytes, _stream(stream)))


def hils_prefill_bwd(cfg: Config, q, k, v, q_lmk, idx, s_sel, k_sum, dout, dq, dk, dv, dq_lmk, workspace,
                     ds_sel=None, stream=None):
    """Gradients of the prefill (float32 outputs dq, dk, dv, dq_lmk and
    optionally ds_sel), selection held fixed; see include/hils.h."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().hils_prefill_bwd(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(q_lmk), _p(idx), _p(s_sel), _p(k_sum),
                                   _p(dout), _p(dq), _p(dk), _p(dv), _p(dq_lmk), _p(ds_sel), _p(workspace), ws_bytes,
                                   _stream(stream)))


def paged(seq_lens, block_table, num_pages: int) -> Paged:
    """seq_lens [B] and block_table [B, max_pages] are int32 CUDA tensors."""
    assert seq_lens.dtype == torch.int32 and block_table.dtype == torch.int32
    return Paged(_p(seq_lens).value, _p(block_table).value, block_table.shape[1], num_pages)


def hils_decode_append(cfg: Config, pg: Paged, k_new, v_new, q_lmk_new, k_pool, v_pool, k_sum, b_sum, stream=None):
    _check(load().hils_decode_append(ctypes.byref(cfg), ctypes.byref(pg), _p(k_new), _p(v_new), _p(q_lmk_new),
                                     _p(k_pool), _p(v_pool), _p(k_sum), _p(b_sum), _stream(stream)))


def hils_build_summaries_paged(cfg: Config, pg: Paged, k_pool, q_lmk, k_sum, b_sum, stream=None):
    _check(load().hils_build_summaries_paged(ctypes.byref(cfg), ctypes.byref(pg), _p(k_pool), _p(q_lmk), _p(k_sum),
                                             _p(b_sum), _stream(stream)))


def hils_score_topk_paged(cfg: Config, q, pg: Paged, k_sum, b_sum, idx, s_sel, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().hils_score_topk_paged(ctypes.byref(cfg), _p(q), ctypes.byref(pg), _p(k_sum), _p(b_sum), _p(idx),
                                        _p(s_sel), _p(workspace), ws_bytes, _stream(stream)))


def hils_attn_decode_paged(cfg: Config, q, k_pool, v_pool, pg: Paged, idx, s_sel, out, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().hils_attn_decode_paged(ctypes.byref(cfg), _p(q), _p(k_pool), _p(v_pool), ctypes.byref(pg), _p(idx),
                                         _p(s_sel), _p(out), _p(workspace), ws_bytes, _stream(stream)))


def _ph(t: torch.Tensor):
    """Host tensor argument (contiguous CPU memory; pinned for overlapping copies)."""
    assert not t.is_cuda and t.is_contiguous(), "host tensors must be contiguous CPU tensors"
    return ctypes.c_void_p(t.data_ptr())


def hils_prefill_host(cfg: Config, q, k, v, q_lmk, out, workspace, qcal=None, stream=None):
    """The prefill path from host memory (q, k, v, q_lmk, qcal tensors and out on the host)."""
    qc = None
    if qcal is not None:
        h, w_down, w_up = qcal
        qc = ctypes.byref(QCal(_ph(h).value, _ph(w_down).value, _ph(w_up).value, w_down.shape[0], w_down.shape[1]))
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().hils_prefill_host(ctypes.byref(cfg), _ph(q), _ph(k), _ph(v), _ph(q_lmk), qc, _ph(out),
                                    _p(workspace), ws_bytes, _stream(stream)))


def _pc(t):
    """A CUDA tensor, or a device address (int) such as hils_host_device_pointer's."""
    return ctypes.c_void_p(t) if isinstance(t, int) else _p(t)


def hils_attn_decode(cfg: Config, q, k_cache, v_cache, idx, s_sel, out, workspace, stream=None):
    """k_cache / v_cache: CUDA tensors, or device addresses of pinned host memory."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().hils_attn_decode(ctypes.byref(cfg), _p(q), _pc(k_cache), _pc(v_cache), _p(idx), _p(s_sel), _p(out),
                                   _p(workspace), ws_bytes, _stream(stream)))


def hils_host_device_pointer(t: torch.Tensor) -> int:
    """Device address of a pinned host tensor (for a host-resident decode cache)."""
    assert not t.is_cuda and t.is_pinned() and t.is_contiguous()
    out = ctypes.c_void_p()
    _check(load().hils_host_device_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(out)))
    return out.value


def hils_attn_decode_noalloc(cfg: Config, q, k_cache, v_cache, idx, s_sel, out, stream=None):
    """hils_attn_decode for callers that cannot allocate device memory: the
    partial records go to the library's fixed device scratch (see hils.h)."""
    _check(load().hils_attn_decode_noalloc(ctypes.byref(cfg), _p(q), _p(k_cache), _p(v_cache), _p(idx), _p(s_sel),
                                           _p(out), _stream(stream)))


def hils_sync_status(stream=None):
    _check(load().hils_sync_status(_stream(stream)))


def hils_set_wait_budget(cycles: int):
    load().hils_set_wait_budget(int(cycles))


def hils_set_fault_injection(mode: int):
    load().hils_set_fault_injection(int(mode))


# ------------------------------------------------------------- pipelines ---

def alloc_workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device)


class Prefill:
    """Buffers and calls for one prefill configuration (all device-resident)."""

    def __init__(self, cfg: Config, device, qcal_rank: int = 0):
        self.cfg = cfg
        B, N, Hq, Hkv, d, S, K = cfg.batch, cfg.seq_len, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.chunk, cfg.top_k
        dt = torch.float32 if cfg.dtype == HILS_F32 else torch.bfloat16
        C = N // S
        self.k_sum = torch.empty((B, Hq, C, d), dtype=dt, device=device)
        self.b_sum = torch.empty((B, Hq, C), dtype=torch.float32, device=device)
        self.idx = torch.empty((B, Hkv, N, K), dtype=torch.int32, device=device)
        self.s_sel = torch.empty((B, Hq, N, K), dtype=torch.float32, device=device)
        self.out = torch.empty((B, Hq, N, d), dtype=dt, device=device)
        self.ws = alloc_workspace(workspace_bytes(cfg, HILS_WS_SCORE_PREFILL, qcal_rank), device)
        self.ws_attn = alloc_workspace(workspace_bytes(cfg, HILS_WS_ATTN_PREFILL), device)

    def run(self, q, k, v, q_lmk, qcal=None, stream=None, shared_lmk=False):
        """shared_lmk: q_lmk is the landmark-free variant's [Hq, d] shared query."""
        if shared_lmk:
            hils_build_summaries_shared(self.cfg, k, q_lmk, self.k_sum, self.b_sum, stream)
        else:
            hils_build_summaries(self.cfg, k, q_lmk, self.k_sum, self.b_sum, stream)
        hils_score_topk(self.cfg, q, self.k_sum, self.b_sum, self.idx, self.s_sel, self.ws, False, qcal, stream)
        hils_attn_prefill(self.cfg, q, k, v, self.idx, self.s_sel, self.out, self.ws_attn, stream)
        return self.out


class Decode:
    """Buffers and calls for one decode configuration; summaries are built by
    :meth:`summarize` (once per cache state) and reused by :meth:`step`."""

    def __init__(self, cfg: Config, device):
        self.cfg = cfg
        B, L, Hq, Hkv, d, S, K = cfg.batch, cfg.seq_len, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.chunk, cfg.top_k
        dt = torch.float32 if cfg.dtype == HILS_F32 else torch.bfloat16
        C = L // S
        self.k_sum = torch.empty((B, Hq, C, d), dtype=dt, device=device)
        self.b_sum = torch.empty((B, Hq, C), dtype=torch.float32, device=device)
        self.idx = torch.empty((B, Hkv, K), dtype=torch.int32, device=device)
        self.s_sel = torch.empty((B, Hq, K), dtype=torch.float32, device=device)
        self.out = torch.empty((B, Hq, d), dtype=dt, device=device)
        self.ws_score = alloc_workspace(workspace_bytes(cfg, HILS_WS_SCORE_DECODE), device)
        self.ws_attn = alloc_workspace(workspace_bytes(cfg, HILS_WS_ATTN_DECODE), device)

    def summarize(self, k_cache, q_lmk, stream=None):
        hils_build_summaries(self.cfg, k_cache, q_lmk, self.k_sum, self.b_sum, stream)

    def step(self, q, k_cache, v_cache, stream=None):
        hils_score_topk(self.cfg, q, self.k_sum, self.b_sum, self.idx, self.s_sel, self.ws_score, True, None, stream)
        hils_attn_decode(self.cfg, q, k_cache, v_cache, self.idx, self.s_sel, self.out, self.ws_attn, stream)
        return self.out
