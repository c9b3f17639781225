"""hils_prefill_host: the prefill path from host memory (pipelined uploads,
per-(sequence, KV group) kernels, downloads) gives exactly the results of the
three device calls, which the other GPU tests check against the oracle."""
import pytest
import torch

from chunk_wise_sparse_landmark_b200 import hils as H
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, prefill_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _host_vs_device(w):
    x = prefill_inputs(w)
    names = ["q", "k", "v", "q_lmk"]
    cfg = H.config_of(w)
    d = {n: x[n].to(DEV) for n in names}
    qc_d = (x["h"].to(DEV), x["w_down"].to(DEV), x["w_up"].to(DEV)) if w.d_model else None
    pre = H.Prefill(cfg, DEV, qcal_rank=w.qcal_rank)
    pre.run(d["q"], d["k"], d["v"], d["q_lmk"], qcal=qc_d)
    H.hils_sync_status()
    host = {n: x[n].contiguous().pin_memory() for n in names}
    qc_h = tuple(x[n].contiguous().pin_memory() for n in ("h", "w_down", "w_up")) if w.d_model else None
    out_h = torch.empty(pre.out.shape, dtype=pre.out.dtype).pin_memory()
    ws = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_PREFILL_HOST, w.qcal_rank), DEV)
    for _ in range(2):  # the second call reuses the library's copy streams and events
        out_h.zero_()
        H.hils_prefill_host(cfg, host["q"], host["k"], host["v"], host["q_lmk"], out_h, ws, qcal=qc_h)
        H.hils_sync_status()
        assert torch.equal(out_h, pre.out.cpu())


def test_prefill_host_bf16_8k():
    _host_vs_device(WORKLOADS["prefill_8k"])


def test_prefill_host_bf16_two_sequences_ragged():
    # B = 2 sequences x 2 KV groups = 4 pieces; N not a multiple of the chunk
    _host_vs_device(WORKLOADS["prefill_8k"].scaled(name="host_r", B=2, N=3000, Hq=8, Hkv=2, K=32, needles_per_head=0))


def test_prefill_host_f32():
    _host_vs_device(WORKLOADS["tiny_f32"])


def test_prefill_host_qcal():
    # Q-Cal through the host call needs d_model = Hq * d (4096 = 32 x 128)
    _host_vs_device(WORKLOADS["prefill_512k_qcal"].scaled(name="host_q", N=4096, needles_per_head=0))
