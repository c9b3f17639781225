"""Decode with the KV cache in page-locked host memory: the decode attention
reads only the token's selected chunks and its window over the host link
(hils_host_device_pointer), and gives the same bits as with the cache in
device memory (same kernels, same data)."""
import ctypes

import pytest
import torch

from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_host_resident_cache_matches_device_cache():
    w = WORKLOADS["decode_512k"].scaled(name="offload", B=3, N=16384 + 29, K=16)
    x = decode_inputs(w)
    cfg = H.config_of(w)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v", "q_lmk")}
    dec = H.Decode(cfg, DEV)
    dec.summarize(d["k"], d["q_lmk"])
    dec.step(d["q"], d["k"], d["v"])
    H.hils_sync_status()
    ref = dec.out.clone()
    kh, vh = x["k"].contiguous().pin_memory(), x["v"].contiguous().pin_memory()
    kp, vp = H.hils_host_device_pointer(kh), H.hils_host_device_pointer(vh)
    out = torch.full_like(ref, float("nan"))
    H.hils_attn_decode(cfg, d["q"], kp, vp, dec.idx, dec.s_sel, out, dec.ws_attn)
    H.hils_sync_status()
    assert torch.equal(out, ref)


def test_host_device_pointer_rejects_pageable_memory():
    t = torch.zeros(1024)  # pageable host memory
    lib = H.load()
    p = ctypes.c_void_p()
    st = lib.hils_host_device_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(p))
    assert st == H.HILS_ERR_INVALID_ARG
