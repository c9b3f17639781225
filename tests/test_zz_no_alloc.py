"""hils_attn_decode_noalloc — decode attention for callers that cannot
allocate device memory for the call (for example a serving engine that has
given all free HBM to its own KV-cache pool, or a plug-in interface that
hands over only input and output buffers).  Its split-KV partial records go
to a fixed device array inside the library instead of a caller workspace.

It must give the same result as hils_attn_decode with a workspace, call after
call (the array is shared and keeps the previous call's contents), and must
refuse a configuration whose records do not fit the array."""
import ctypes

import pytest
import torch

from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("shape", [dict(B=4, N=32768 + 21), dict(B=2, N=16384 + 5, Hq=32, Hkv=4),
                                   dict(B=3, N=8192, Hq=8, Hkv=8)], ids=["G4", "G8", "G1"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(shape):
    """Same kernels and split count as hils_attn_decode, only the scratch lives
    elsewhere: the outputs agree bit for bit, on two calls in a row (the second
    call reads records the first one overwrote).  Three group sizes give three
    split counts against the one fixed array."""
    w = WORKLOADS["decode_512k"].scaled(name="noalloc", **shape)
    x = decode_inputs(w, device=DEV)
    cfg = H.config_of(w)
    dec = H.Decode(cfg, DEV)
    dec.summarize(x["k"], x["q_lmk"])
    queries = [x["q"], (-x["q"]).contiguous()]  # the second call sees another token
    for q in queries:
        H.hils_score_topk(cfg, q, dec.k_sum, dec.b_sum, dec.idx, dec.s_sel, dec.ws_score, True)
        ref = torch.empty_like(dec.out)
        H.hils_attn_decode(cfg, q, x["k"], x["v"], dec.idx, dec.s_sel, ref, dec.ws_attn)
        got = torch.full_like(dec.out, float("nan"))
        H.hils_attn_decode_noalloc(cfg, q, x["k"], x["v"], dec.idx, dec.s_sel, got)
        H.hils_sync_status()
        assert torch.isfinite(got.float()).all()
        assert torch.equal(got, ref)


def test_noalloc_rejects_configuration_larger_than_its_scratch():
    cfg = H.make_config(256, 524288, 32, 8, 128, 64, 512, 32, "bf16")
    need = H.workspace_bytes(cfg, H.HILS_WS_ATTN_DECODE)
    assert need > 4 * 1024 * 1024
    dummy = torch.empty(16, dtype=torch.int32, device=DEV)
    p = ctypes.c_void_p(dummy.data_ptr())
    lib = H.load()
    st = lib.hils_attn_decode_noalloc(ctypes.byref(cfg), p, p, p, p, p, p, None)
    assert st == H.HILS_ERR_UNSUPPORTED
    assert b"scratch" in lib.hils_last_error()
