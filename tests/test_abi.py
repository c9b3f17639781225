"""The C ABI without a GPU: the library loads, exports every entry point that
include/hils.h declares, and rejects bad arguments on the host before any
device work."""
import ctypes
import os
import re

import pytest

from chunk_wise_sparse_landmark_b200 import hils as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hils.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = H.load()
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(H.EXPORTS)


def test_version():
    assert H.load().hils_version().startswith(b"hils-b200")


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(Hkv=3), H.HILS_ERR_INVALID_ARG),        # Hq % Hkv
        (dict(W=48), H.HILS_ERR_INVALID_ARG),         # W % S
        (dict(W=16), H.HILS_ERR_INVALID_ARG),         # W < S
        (dict(K=0), H.HILS_ERR_INVALID_ARG),
        (dict(K=65), H.HILS_ERR_UNSUPPORTED),
        (dict(d=48), H.HILS_ERR_UNSUPPORTED),
        (dict(dtype="bf16"), H.HILS_ERR_UNSUPPORTED),  # bf16 needs d=128, S=64
    ],
)
def test_bad_config_rejected_on_host(kw, status):
    base = dict(B=1, N=512, Hq=4, Hkv=1, d=64, S=32, W=64, K=4, dtype="f32")
    base.update(kw)
    cfg = H.make_config(**base)
    lib = H.load()
    st = lib.hils_build_summaries(ctypes.byref(cfg), None, None, None, None, None)
    assert st == status, lib.hils_last_error()
    assert lib.hils_workspace_bytes(ctypes.byref(cfg), 0, 0) == ctypes.c_size_t(-1).value


def test_null_and_unaligned_pointers_rejected():
    lib = H.load()
    cfg = H.make_config(1, 512, 4, 1, 64, 32, 64, 4, "f32")
    assert lib.hils_build_summaries(ctypes.byref(cfg), None, None, None, None, None) == H.HILS_ERR_INVALID_ARG
    p = ctypes.c_void_p(0x1000)
    bad = ctypes.c_void_p(0x1004)
    assert lib.hils_attn_prefill(ctypes.byref(cfg), p, p, p, p, p, bad, None, 0, None) == H.HILS_ERR_INVALID_ARG
    assert b"unaligned" in lib.hils_last_error()
    # workspace too small for decode attention
    assert lib.hils_attn_decode(ctypes.byref(cfg), p, p, p, p, p, p, p, 0, None) == H.HILS_ERR_INVALID_ARG
    assert b"workspace" in lib.hils_last_error()


def test_workspace_sizes():
    cfg = H.make_config(16, 524288, 32, 8, 128, 64, 512, 32, "bf16")
    ws = H.workspace_bytes(cfg, H.HILS_WS_SCORE_DECODE)
    assert ws == (16 * 32 * 8192 + 16 * 8 * 8192) * 4
    assert H.workspace_bytes(cfg, H.HILS_WS_ATTN_DECODE) > 0


def test_attn_prefill_workspace_size():
    """Chunk-major attention scratch: bucket counts / offsets / item offsets
    (U + 1 ints each, U = B Hkv C buckets), the pairs of one position tile
    (ints), the item table (int4: bucket, first pair, count; at most
    pairs / 32 + U + 1 items), the tile's query rows regrouped per KV group
    (1 KB per position and group), the window pass's fp32 state for two
    tiles (4 heads x (128 accumulators + reference exponent + sum) per
    position and group) and one 1 KB bf16 partial record per pair; the fewest equal tiles whose
    records fit about 8 GiB, rounded up to a multiple of 64 positions."""
    up = lambda n: (n + 255) // 256 * 256
    B, N, Hq, Hkv, K = 1, 131072, 32, 8, 32
    cfg = H.make_config(B, N, Hq, Hkv, 128, 64, 512, K, "bf16")
    per_pos = B * Hkv * K * 4 * 128 * 2
    cap = (8 << 30) // per_pos
    ntiles = -(-N // cap)
    PT = -(-(-(-N // ntiles)) // 64) * 64
    assert (ntiles, PT) == (4, 32768)
    U, pairs = B * Hkv * (N // 64), B * Hkv * PT * K
    want = (3 * up((U + 1) * 4) + up(pairs * 4) + up((pairs // 32 + U + 1) * 16) + up(pairs // K * 1024)
            + up(2 * (pairs // K) * 2080) + up(pairs * 1024))
    assert H.workspace_bytes(cfg, H.HILS_WS_ATTN_PREFILL) == want
    # short sequences: one tile of N rounded up to 64 positions
    small = H.make_config(2, 1000, 8, 2, 128, 64, 128, 8, "bf16")
    PT, U = 1024, 2 * 2 * (1000 // 64)
    pairs = 2 * 2 * PT * 8
    want = (3 * up((U + 1) * 4) + up(pairs * 4) + up((pairs // 32 + U + 1) * 16) + up(pairs // 8 * 1024)
            + up(2 * (pairs // 8) * 2080) + up(pairs * 1024))
    assert H.workspace_bytes(small, H.HILS_WS_ATTN_PREFILL) == want
    assert H.workspace_bytes(H.make_config(1, 512, 4, 1, 64, 32, 64, 4, "f32"), H.HILS_WS_ATTN_PREFILL) == 0
    lib = H.load()
    p = ctypes.c_void_p(0x1000)
    st = lib.hils_attn_prefill(ctypes.byref(small), p, p, p, p, p, p, p, want - 1, None)
    assert st == H.HILS_ERR_INVALID_ARG and b"workspace" in lib.hils_last_error()


def test_prefill_host_workspace_and_host_checks():
    """Workspace size of the host-memory prefill and its argument checks (no GPU needed)."""
    lib = H.load()
    B, N, Hq, Hkv, d, S, K = 1, 512, 4, 1, 64, 32, 4
    cfg = H.make_config(B, N, Hq, Hkv, d, S, 64, K, "f32")
    up = lambda n: (n + 255) // 256 * 256
    C = N // S
    want = (up(B * Hq * N * d * 4) + 2 * up(B * Hkv * N * d * 4) + 2 * up(B * Hq * C * d * 4) + up(B * Hq * C * 4)
            + up(B * Hkv * N * K * 4) + up(B * Hq * N * K * 4) + up(B * Hq * N * d * 4))
    assert lib.hils_workspace_bytes(ctypes.byref(cfg), H.HILS_WS_PREFILL_HOST, 0) == want
    p = ctypes.c_void_p(0x1000)
    st = lib.hils_prefill_host(ctypes.byref(cfg), None, p, p, p, None, p, p, want, None)
    assert st == H.HILS_ERR_INVALID_ARG
    st = lib.hils_prefill_host(ctypes.byref(cfg), p, p, p, p, None, p, p, want - 1, None)
    assert st == H.HILS_ERR_INVALID_ARG and b"workspace" in lib.hils_last_error()


@pytest.mark.parametrize(
    "call,kw",
    [
        ("summaries", dict(d=32, S=64)),                      # f32 summaries: no (d=32, S=64) kernel
        ("score_prefill", dict(d=128, S=64, Hq=8, Hkv=1)),    # f32 prefill scoring: no G=8 kernel at d=128
        ("attn_decode", dict(d=32, S=32)),                    # f32 decode attention: d=32
        ("attn_decode", dict(d=64, S=16)),                    # f32 decode attention: S=16
        ("score_prefill", dict(dtype="bf16", d=128, S=64, Hq=8, Hkv=1)),  # bf16 prefill: G=4 only
        ("attn_prefill", dict(dtype="bf16", d=128, S=64, Hq=8, Hkv=4)),   # bf16 prefill: G=4 only
    ],
)
def test_shapes_without_a_kernel_are_unsupported_on_host(call, kw):
    """Shapes that no kernel serves return HILS_ERR_UNSUPPORTED from the host
    checks, before any device work (so this runs without a GPU)."""
    base = dict(B=1, N=512, Hq=4, Hkv=1, d=64, S=32, W=64, K=4, dtype="f32")
    base.update(kw)
    if base["W"] < base["S"]:
        base["W"] = base["S"]
    base["W"] = max(base["W"], 2 * base["S"])
    cfg = H.make_config(**base)
    lib = H.load()
    p = ctypes.c_void_p(0x1000)
    if call == "summaries":
        st = lib.hils_build_summaries(ctypes.byref(cfg), p, p, p, p, None)
    elif call == "score_prefill":
        st = lib.hils_score_topk(ctypes.byref(cfg), p, None, p, p, p, p, p, 1 << 30, 0, None)
    elif call == "attn_prefill":
        st = lib.hils_attn_prefill(ctypes.byref(cfg), p, p, p, p, p, p, None, 0, None)
    else:
        st = lib.hils_attn_decode(ctypes.byref(cfg), p, p, p, p, p, p, p, 1 << 30, None)
    assert st == H.HILS_ERR_UNSUPPORTED, (st, lib.hils_last_error())
    which = {"summaries": None, "score_prefill": H.HILS_WS_SCORE_PREFILL, "attn_prefill": H.HILS_WS_ATTN_PREFILL,
             "attn_decode": H.HILS_WS_ATTN_DECODE}[call]
    if which is not None:
        assert lib.hils_workspace_bytes(ctypes.byref(cfg), which, 0) == ctypes.c_size_t(-1).value


def test_qcal_rank_other_than_64_is_unsupported_on_host():
    lib = H.load()
    cfg = H.make_config(1, 1024, 4, 1, 128, 64, 128, 4, "bf16")
    p = ctypes.c_void_p(0x1000)
    qc = H.QCal(0x1000, 0x1000, 0x1000, 32, 4096)
    st = lib.hils_score_topk(ctypes.byref(cfg), p, ctypes.byref(qc), p, p, p, p, p, 1 << 40, 0, None)
    assert st == H.HILS_ERR_UNSUPPORTED, lib.hils_last_error()
