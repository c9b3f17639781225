"""Benchmark of the HiLS forward hot path on B200 (one JSON line on rank 0).

Step (prefill workloads): landmark summaries -> [Q-Cal ->] scoring + GQA
group max + top-K -> hierarchical-softmax attention, all through the C ABI on
device-resident synthetic inputs.  Metric: prefill tokens/s.  The decode
workload (one token per sequence, score + top-K + split-KV attention over a
pre-summarised cache) is measured in the same run and reported in "decode".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl reference] [--no-decode] [--no-e2e] [--no-cpu]

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of
the workload (independent sequences: the path has no exchange step), the time
is the max over ranks, and the value is all ranks' tokens / that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunk_wise_sparse_landmark_b200 import hils as H  # noqa: E402
from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS, decode_inputs, prefill_inputs  # noqa: E402

METRIC = "HiLS prefill tokens/s & decode seqs/s at 128K-512K ctx; % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------- utilities ---

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Clocks:
    """nvidia-smi sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.gpu = gpu_index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        try:
            lines = [ln.split(",") for ln in open(self.f.name).read().strip().splitlines() if ln.strip()]
        except Exception:
            lines = []
        os.unlink(self.f.name)
        if not lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(x[1]) for x in lines if x[1].strip().replace(".", "").isdigit()]
        mx = [float(x[2]) for x in lines if x[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for x in lines for k in range(4) if len(x) > 5 + k and x[5 + k].strip() == "Active"})
        loaded = [v for v in sm if mx and v > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(lines)}


def prefill_flops(w):
    """Algorithmic FLOP of one prefill pass (per token and query head:
    2d|Cand(i)| scoring + 4d(|I_i| S + |Win(i)|) attention), and of the
    attention kernel alone."""
    nw = w.W // w.S
    score = attn = 0
    for i in range(w.N):
        cur = i // w.S
        cand = max(0, cur - nw + 1)
        win = i - max(0, (cur - nw + 1) * w.S) + 1
        score += 2 * w.d * cand
        attn += 4 * w.d * (min(w.K, cand) * w.S + win)
    return score * w.B * w.Hq, attn * w.B * w.Hq


def decode_bytes(w):
    """Algorithmic bytes of one decode step: k'/b' of every candidate for every
    head, plus the K chunks and the window of K and V per KV head."""
    cur = (w.N - 1) // w.S
    nw = w.W // w.S
    cand = max(0, cur - nw + 1)
    win = w.N - max(0, (cur - nw + 1) * w.S)
    esz = 2 if w.dtype == "bf16" else 4
    score = w.B * w.Hq * cand * (w.d * esz + 4)
    gather = w.B * w.Hkv * (min(w.K, cand) * w.S + win) * w.d * esz * 2
    q_out = w.B * w.Hq * w.d * esz * 2
    return score, gather, q_out


def attention_stats(w, idx):
    """Executed work of the chunk-major attention, and the reuse measure of
    grouping adjacent queries, from the selection the step produced.

    * pairs: (position, KV group, selected chunk) triples; each is 4 heads x
      (2 d S + 2 S d) FLOP of algorithmic selected-chunk work.
    * items: per position tile and bucket (sequence, group, chunk), ceil(n/32)
      items of 128 query rows; each executes 128 rows x 4 d S FLOP on tcgen05.
    * window: an item of the window kernel is 32 aligned positions x 4 heads
      (128 rows) of one group against its block's window chunks, taken two at
      a time (an odd count padded with one chunk whose keys are all masked);
      two passes, S then S and P V: 128 x 6 d S FLOP per chunk taken.
    * union_over_k_m4: mean size of the union of the chunk sets of M = 4
      adjacent positions divided by K (rows with full lists), the reuse measure
      of grouping adjacent queries.
    Counting runs on the GPU with torch after the timed region (measurement
    only, not part of the path)."""
    B, Hkv, N, K = idx.shape
    S, nw, d = w.S, w.W // w.S, w.d
    C = N // S
    PT = attn_tile_positions(w)
    valid = idx >= 0
    pairs = int(valid.sum().item())
    items = 0
    for t0 in range(0, N, PT):
        sl = idx[:, :, t0:t0 + PT]
        bg = torch.arange(B * Hkv, device=idx.device).view(B, Hkv, 1, 1).expand_as(sl)
        u = (bg * C + sl.clamp(min=0))[sl >= 0]
        cnt = torch.bincount(u.long(), minlength=B * Hkv * C)
        items += int(((cnt + 31) // 32).sum().item())
    win_chunks = 0
    for p0 in range(0, N, 32):
        cur = p0 // S
        win_chunks += 2 * ((cur - max(0, cur - nw + 1) + 2) // 2)
    exec_chunk = items * 128 * 4 * d * S
    exec_win = B * Hkv * win_chunks * 128 * 6 * d * S
    M = 4
    nb = N // M
    blk = idx[:, :, : nb * M].reshape(B, Hkv, nb, M * K)
    full = (idx[:, :, : nb * M] >= 0).sum(-1).reshape(B, Hkv, nb, M).min(-1).values == K
    srt, _ = torch.sort(blk, dim=-1)
    distinct = ((srt[..., 1:] != srt[..., :-1]) & (srt[..., 1:] >= 0)).sum(-1) + (srt[..., 0] >= 0).long()
    union_k = float((distinct[full].float() / K).mean().item()) if bool(full.any()) else None
    return {"pairs": pairs, "items": items, "item_fill": round(pairs / max(1, 32 * items), 4),
            "executed_flop_per_launch": exec_chunk + exec_win, "union_over_k_m4": union_k}


def source_sha(kernel_files) -> str:
    """Hash of the kernel sources a traffic figure was measured with."""
    if isinstance(kernel_files, str):
        kernel_files = [kernel_files]
    h = hashlib.sha256()
    for f in kernel_files:
        h.update(open(os.path.join(ROOT, "chunk_wise_sparse_landmark_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel_files, kernel: str, workload: str):
    """DRAM bytes per launch (or per call) from a committed ncu capture
    (profiles/traffic.json), or None if absent or if a source changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d[kernel][workload]
        return e["bytes_per_launch"] if e.get("source_sha") == source_sha(kernel_files) else None
    except Exception:
        return None


def timed(fn, stream):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    fn()
    b.record(stream)
    return a, b


# ----------------------------------------------------------------- arms -----

def run_prefill(w, dev, steps, warmup, stream):
    x = prefill_inputs(w, device=dev)
    cfg = H.config_of(w)
    qc = (x["h"], x["w_down"], x["w_up"]) if w.d_model else None
    pre = H.Prefill(cfg, dev, qcal_rank=w.qcal_rank)
    ev = {"summaries": [], "score_topk": [], "attn_prefill": []}

    def step(record):
        if record:
            ev["summaries"].append(timed(lambda: H.hils_build_summaries(cfg, x["k"], x["q_lmk"], pre.k_sum,
                                                                        pre.b_sum, stream), stream))
            ev["score_topk"].append(timed(lambda: H.hils_score_topk(cfg, x["q"], pre.k_sum, pre.b_sum, pre.idx,
                                                                    pre.s_sel, pre.ws, False, qc, stream), stream))
            ev["attn_prefill"].append(timed(lambda: H.hils_attn_prefill(cfg, x["q"], x["k"], x["v"], pre.idx,
                                                                        pre.s_sel, pre.out, pre.ws_attn, stream),
                                            stream))
        else:
            pre.run(x["q"], x["k"], x["v"], x["q_lmk"], qcal=qc, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step(False)
        H.hils_sync_status(stream)
    return x, pre, step, ev


def run_decode(w, dev, steps, warmup, stream):
    x = decode_inputs(w, device=dev)
    cfg = H.config_of(w)
    dec = H.Decode(cfg, dev)
    with torch.cuda.stream(stream):
        a, b = timed(lambda: dec.summarize(x["k"], x["q_lmk"], stream), stream)
        for _ in range(warmup):
            dec.step(x["q"], x["k"], x["v"], stream)
        H.hils_sync_status(stream)
    summ_ms = a.elapsed_time(b)
    # The decode step is a few microsecond-scale launches: capture each call in a
    # CUDA graph (after the warm-up above has done every once-per-device set-up)
    # so that host-side argument handling cannot show up as device time.
    g_score, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_score, stream=stream):
        H.hils_score_topk(cfg, x["q"], dec.k_sum, dec.b_sum, dec.idx, dec.s_sel, dec.ws_score, True, None,
                          torch.cuda.current_stream())
    with torch.cuda.graph(g_attn, stream=stream):
        H.hils_attn_decode(cfg, x["q"], x["k"], x["v"], dec.idx, dec.s_sel, dec.out, dec.ws_attn,
                           torch.cuda.current_stream())
    ev = {"score_topk": [], "attn_decode": []}

    def step():
        ev["score_topk"].append(timed(g_score.replay, stream))
        ev["attn_decode"].append(timed(g_attn.replay, stream))

    dec._graphs = (g_score, g_attn)
    return x, dec, step, ev, summ_ms


def mean_ms(pairs):
    return sum(a.elapsed_time(b) for a, b in pairs) / max(1, len(pairs))


def max_over_ranks(ms, dist_on, device="cuda"):
    """The slowest rank's time: every rank contributes its own and gets the max."""
    if not dist_on:
        return ms
    t = torch.tensor([float(ms)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world_size, ms):
    """Units all ranks processed per second, over the max-over-ranks time (weak scaling)."""
    return units_per_rank * world_size / (ms / 1e3)


def device_time(stream, fn, steps, dist_on):
    """Barrier + sync, K steps between CUDA events, sync; max over ranks (ms)."""
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            fn()
    b.record(stream)
    torch.cuda.synchronize()
    return max_over_ranks(a.elapsed_time(b), dist_on)


def e2e_prefill(w, x, pre, stream, steps, dist_on):
    """Through the C ABI with host buffers (hils_prefill_host): every step copies
    the inputs from pinned host memory to the device, runs the prefill and copies
    the output back; the library pipelines the transfers with the kernels by
    (sequence, KV group)."""
    names = ["q", "k", "v", "q_lmk"]
    host = {n: x[n].to("cpu").contiguous().pin_memory() for n in names}
    qc = tuple(x[n].to("cpu").contiguous().pin_memory() for n in ("h", "w_down", "w_up")) if w.d_model else None
    out_h = torch.empty(pre.out.shape, dtype=pre.out.dtype).pin_memory()
    ws = H.alloc_workspace(H.workspace_bytes(pre.cfg, H.HILS_WS_PREFILL_HOST, w.qcal_rank), pre.out.device)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    h2d += sum(t.numel() * t.element_size() for t in qc) if qc else 0
    d2h = out_h.numel() * out_h.element_size()

    def step():
        H.hils_prefill_host(pre.cfg, host["q"], host["k"], host["v"], host["q_lmk"], out_h, ws, qcal=qc,
                            stream=stream)

    with torch.cuda.stream(stream):
        step()
    H.hils_sync_status(stream)
    ms = device_time(stream, step, steps, dist_on)
    H.hils_sync_status(stream)
    del ws
    return ms / steps, h2d, d2h


def cpu_baseline_prefill(w, x, budget_s=15.0, rows=None, seed=0):
    """The oracle, as it stands, on the host cores, on a sample of positions:
    summaries of the whole sequence amortised per position, plus scoring,
    selection and attention of the sampled positions for every head."""
    import numpy as np

    import oracle

    dm = oracle.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, S=w.S, W=w.W, K=w.K)
    q = x["q"][:1].float().cpu().numpy()
    k = x["k"][:1].float().cpu().numpy()
    v = x["v"][:1].float().cpu().numpy()
    ql = x["q_lmk"][:1].float().cpu().numpy()
    t0 = time.perf_counter()
    ks, bs = oracle.summaries(dm, k, ql)
    t_summ = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    n = rows or 32
    done = 0
    t_rows = 0.0
    while True:
        sel = [(0, int(i)) for i in rng.integers(0, w.N, n)]
        t0 = time.perf_counter()
        qs = None
        if w.d_model:
            qs = oracle.qcal(dm, sel, q, x["h"][:1].float().cpu().numpy(), x["w_down"].float().cpu().numpy(),
                             x["w_up"].float().cpu().numpy())
        idx, ssel = oracle.select(dm, sel, q, k_sum=ks, b_sum=bs, qs=qs)
        oracle.attend(dm, sel, q, k, v, idx, ssel)
        t_rows += time.perf_counter() - t0
        done += n
        if rows is not None or t_rows > budget_s:
            break
    per_token = t_rows / done + t_summ / w.N
    return 1.0 / per_token, done, t_summ, t_rows


def prefill_launches(w) -> int:
    """Kernels one prefill step launches: summaries, [Q-Cal,] scoring, and per
    attention position tile bucket count, scan, scatter, the query regroup,
    the chunk-major pass, the window pass and the fusion."""
    return 2 + (1 if w.d_model else 0) + 7 * attn_tiles(w)


def prefill_roofline(w, pre, ev, pk, pk_kind):
    """Roofline of the dominant call (hils_attn_prefill) and per-kernel times of
    a timed prefill run; the executed-work statistics come from its selection."""
    score_f, attn_f = prefill_flops(w)
    t_attn = mean_ms(ev["attn_prefill"])
    t_score = mean_ms(ev["score_topk"])
    t_summ = mean_ms(ev["summaries"])
    peak_tf = pk["bf16_tflops_sustained"]
    ach = attn_f / (t_attn / 1e3) / 1e12
    st = attention_stats(w, pre.idx)
    roofline = {"kernel": f"hils_attn_prefill (attn_chunk_kernel + attn_window_kernel + attn_fuse_kernel + "
                          f"bucketing, {attn_tiles(w)} position tiles)",
                "bound": "tensor", "achieved": round(ach, 2),
                "peak": peak_tf, "unit": "TFLOP/s", "frac": round(ach / peak_tf, 4),
                "traffic": traffic_for(["attn_chunk.cu", "attn_window.cu", "common.cuh"], "hils_attn_prefill", w.name),
                "peak_source": f"{pk_kind} bf16_tflops_sustained",
                "algorithmic_flop_per_launch": attn_f,
                "executed_flop_per_launch": st["executed_flop_per_launch"],
                "executed_tflops": round(st["executed_flop_per_launch"] / (t_attn / 1e3) / 1e12, 2),
                "union_over_k_m4": st["union_over_k_m4"], "pairs": st["pairs"], "items": st["items"],
                "item_fill": st["item_fill"]}
    per_kernel = {"summaries_ms": round(t_summ, 4), "score_topk_ms": round(t_score, 4),
                  "attn_prefill_ms": round(t_attn, 4),
                  "score_tflops_alg": round(score_f / (t_score / 1e3) / 1e12, 2),
                  "score_frac": round(score_f / (t_score / 1e3) / 1e12 / peak_tf, 4)}
    return roofline, per_kernel


FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x fp32 lanes x FMA x max clock (74.4)


def backward_flops(w):
    """Algorithmic FLOP of the prefill backward (selection held fixed), per
    (position, query head): 10 d per attended key (recompute s and dout.v, then
    dq, dk, dv: five d-long products) + 4 d per chosen chunk (score path), and
    8 S d per (query head, chunk) for the summary backward."""
    nw = w.W // w.S
    tot = 0
    for i in range(w.N):
        cur = i // w.S
        cand = max(0, cur - nw + 1)
        win = i - max(0, (cur - nw + 1) * w.S) + 1
        sel = min(w.K, cand)
        tot += 10 * w.d * (sel * w.S + win) + 4 * w.d * sel
    return tot * w.B * w.Hq + 8 * w.S * w.d * w.B * w.Hq * w.C


def bench_backward(w, dev, stream, args, ws, dist_on):
    """hils_prefill_bwd after a forward of the same workload: W >= 3 untimed
    calls, then K calls between CUDA events (max over ranks)."""
    x = prefill_inputs(w, device=dev)
    cfg = H.config_of(w)
    pre = H.Prefill(cfg, dev)
    with torch.cuda.stream(stream):
        pre.run(x["q"], x["k"], x["v"], x["q_lmk"], stream=stream)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    dout = torch.randn(x["q"].shape, generator=gen, device=dev).to(x["q"].dtype)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = [torch.empty((w.B, w.Hq, w.N, w.d), **f32), torch.empty((w.B, w.Hkv, w.N, w.d), **f32),
             torch.empty((w.B, w.Hkv, w.N, w.d), **f32), torch.empty((w.B, w.Hq, w.C, w.d), **f32)]
    wsb = H.alloc_workspace(H.workspace_bytes(cfg, H.HILS_WS_PREFILL_BWD), dev)

    def step():
        H.hils_prefill_bwd(cfg, x["q"], x["k"], x["v"], x["q_lmk"], pre.idx, pre.s_sel, pre.k_sum, dout, *grads,
                           wsb, stream=stream)

    steps = max(2, args.steps // 3)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    H.hils_sync_status(stream)
    ms = device_time(stream, step, steps, dist_on) / steps
    H.hils_sync_status(stream)
    fl = backward_flops(w)
    ach = fl / (ms / 1e3) / 1e12
    out = {"workload": w.name, "value": round(whole_job_rate(w.B * w.N, ws, ms), 1), "unit": "tokens/s",
           "ms_per_call": round(ms, 3), "steps": steps, "warmup": args.warmup,
           "roofline": {"kernel": "hils_prefill_bwd (bwd_rows_kernel + bwd_keys_kernel + bucketing)", "bound": "alu",
                        "achieved": round(ach, 2), "peak": round(FP32_ALU_TFLOPS, 1), "unit": "TFLOP/s",
                        "frac": round(ach / FP32_ALU_TFLOPS, 4), "traffic": None,
                        "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz",
                        "algorithmic_flop_per_launch": fl},
           "gpu_launches": 5 * steps}
    del x, pre, grads, wsb
    torch.cuda.empty_cache()
    return out


def bench_decode_offload(dev, stream, args, ws, dist_on):
    """Decode attention with the KV cache in page-locked host memory (the
    summaries stay on the device): the kernel reads the token's K chunks and
    window over the host link.  Workload: the decode workload's shapes at 4
    sequences of 128K (2 x 1 GiB of pinned host cache)."""
    w = WORKLOADS["decode_512k"].scaled(name="decode_offload_4x128k", B=4, N=131072)
    x = decode_inputs(w, device=dev)
    cfg = H.config_of(w)
    dec = H.Decode(cfg, dev)
    with torch.cuda.stream(stream):
        dec.summarize(x["k"], x["q_lmk"], stream)
        dec.step(x["q"], x["k"], x["v"], stream)
    H.hils_sync_status(stream)
    kh, vh = x["k"].cpu().pin_memory(), x["v"].cpu().pin_memory()
    del x["k"], x["v"]
    kp, vp = H.hils_host_device_pointer(kh), H.hils_host_device_pointer(vh)

    def step():
        H.hils_attn_decode(cfg, x["q"], kp, vp, dec.idx, dec.s_sel, dec.out, dec.ws_attn, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    H.hils_sync_status(stream)
    n = args.steps * 5
    ms = device_time(stream, step, n, dist_on) / n
    H.hils_sync_status(stream)
    _, gb, _ = decode_bytes(w)
    out = {"workload": w.name, "attn_decode_ms": round(ms, 4), "link_gbs": round(gb / (ms / 1e3) / 1e9, 1),
           "bytes_per_step": gb, "cache_bytes_on_host": 2 * kh.numel() * kh.element_size(),
           "note": "KV cache in pinned host memory; only the selected chunks and the window cross the link",
           "gpu_launches": 2 * n}
    del kh, vh, dec, x
    torch.cuda.empty_cache()
    return out


def dense_comparator(dev, stream, reps=2):
    """Dense causal attention of the same shapes on this GPU, for context only:
    the pages quote HiLS against full attention (13.5x prefill and 15.7x decode
    at 512K, hardware not stated).  This is a library kernel (torch's scaled
    dot-product attention, GQA, bf16), not part of the path; it times one
    attention call per shape, L2 not flushed (inputs far larger than L2)."""
    import torch.nn.functional as F

    res = {}
    shapes = {"prefill_128k": (1, 32, 8, 131072), "prefill_512k": (1, 32, 8, 524288)}
    for name, (B, Hq, Hkv, N) in shapes.items():
        g = torch.Generator(device=dev)
        g.manual_seed(9)
        q = torch.randn((B, Hq, N, 128), generator=g, device=dev, dtype=torch.bfloat16)
        k = torch.randn((B, Hkv, N, 128), generator=g, device=dev, dtype=torch.bfloat16)
        v = torch.randn((B, Hkv, N, 128), generator=g, device=dev, dtype=torch.bfloat16)
        with torch.cuda.stream(stream):
            F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        ms = device_time(stream, lambda: F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True),
                         reps, False) / reps
        flop = 4 * 128 * B * Hq * N * (N + 1) / 2
        res[name] = {"ms": round(ms, 3), "tflops": round(flop / (ms / 1e3) / 1e12, 1)}
        del q, k, v
    # decode: one query per sequence over a 512K cache, 16 sequences
    B, Hq, Hkv, L = 16, 32, 8, 524288
    g = torch.Generator(device=dev)
    g.manual_seed(10)
    q = torch.randn((B, Hq, 1, 128), generator=g, device=dev, dtype=torch.bfloat16)
    k = torch.randn((B, Hkv, L, 128), generator=g, device=dev, dtype=torch.bfloat16)
    v = torch.randn((B, Hkv, L, 128), generator=g, device=dev, dtype=torch.bfloat16)
    with torch.cuda.stream(stream):
        F.scaled_dot_product_attention(q, k, v, enable_gqa=True)
    ms = device_time(stream, lambda: F.scaled_dot_product_attention(q, k, v, enable_gqa=True), reps * 5, False) / (
        reps * 5)
    res["decode_512k"] = {"ms": round(ms, 3), "gbs": round(2 * k.numel() * 2 / (ms / 1e3) / 1e9, 1)}
    del q, k, v
    torch.cuda.empty_cache()
    res["kernel"] = "torch scaled_dot_product_attention (library, bf16, GQA), context only"
    return res


def extra_prefill(w, dev, stream, args, ws, dist_on, pk, pk_kind):
    """Another prefill workload timed the same way (device-resident inputs,
    W >= 3 warm-up steps, K timed steps between CUDA events, max over ranks),
    reported beside the main line."""
    steps = max(3, args.steps // 2)
    x, pre, step, ev = run_prefill(w, dev, steps, args.warmup, stream)
    with Clocks(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        ms_total = device_time(stream, lambda: step(True), steps, dist_on)
    H.hils_sync_status(stream)
    ms_step = ms_total / steps
    roofline, per_kernel = prefill_roofline(w, pre, ev, pk, pk_kind)
    out = {"workload": w.name, "value": round(whole_job_rate(w.B * w.N, ws, ms_step), 1), "unit": "tokens/s",
           "ms_per_step": round(ms_step, 3), "steps": steps, "warmup": args.warmup, "config": run_config(w, ws),
           "roofline": roofline, "kernels": per_kernel, "clocks": clk.summary(),
           "gpu_launches": prefill_launches(w) * steps}
    del x, pre
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ main -----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_128k", choices=[k for k, v in WORKLOADS.items() if not v.decode])
    ap.add_argument("--decode-workload", default="decode_512k")
    ap.add_argument("--impl", default="hils", choices=["hils", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-qcal", action="store_true", help="skip the 512K Q-Cal prefill reported beside the line")
    ap.add_argument("--no-bwd", action="store_true", help="skip the prefill backward reported beside the line")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip timing dense attention of the same shapes (library kernel, context only)")
    ap.add_argument("--bwd-workload", default="prefill_8k", choices=[k for k, v in WORKLOADS.items() if not v.decode])
    ap.add_argument("--seq-len", type=int, default=0, help="override N of the prefill workload (profiling)")
    ap.add_argument("--decode-seq-len", type=int, default=0, help="override L of the decode workload (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    ws, rank, local = dist_env()
    dist_on = ws > 1
    if args.impl == "reference":
        return reference_arm(args, ws, rank)
    if dist_on:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    H.load()
    stream = torch.cuda.Stream()
    pk, pk_kind = peaks()

    w = WORKLOADS[args.workload]
    if args.seq_len:
        w = w.scaled(N=args.seq_len, needles_per_head=min(w.needles_per_head, max(1, args.seq_len // 2048)))
    x, pre, step, ev = run_prefill(w, dev, args.steps, args.warmup, stream)
    with Clocks(local) as clk:
        ms_total = device_time(stream, lambda: step(True), args.steps, dist_on)
    H.hils_sync_status(stream)
    clocks = clk.summary()
    ms_step = ms_total / args.steps
    tokens = w.B * w.N * ws
    value = whole_job_rate(w.B * w.N, ws, ms_step)
    roofline, per_kernel = prefill_roofline(w, pre, ev, pk, pk_kind)
    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": run_config(w, ws),
            "roofline": roofline, "kernels": per_kernel, "clocks": clocks,
            "gpu_launches": prefill_launches(w) * args.steps}
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_prefill(w, x, pre, stream, max(2, args.steps // 3), dist_on)
        line["e2e"] = {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3)}
    del pre
    if not args.no_decode:
        wd = WORKLOADS[args.decode_workload]
        if args.decode_seq_len:
            wd = wd.scaled(N=args.decode_seq_len)
        xd, dec, dstep, dev_ev, summ_ms = run_decode(wd, dev, args.steps, args.warmup, stream)
        d_ms = device_time(stream, dstep, args.steps * 5, dist_on) / (args.steps * 5)
        H.hils_sync_status(stream)
        sb, gb, qb = decode_bytes(wd)
        t_att = mean_ms(dev_ev["attn_decode"])
        t_sc = mean_ms(dev_ev["score_topk"])
        hbm = pk["hbm_gbs"]
        line["decode"] = {
            "workload": wd.name, "value": round(whole_job_rate(wd.B, ws, d_ms), 1), "unit": "seqs/s",
            "ms_per_step": round(d_ms, 4), "score_topk_ms": round(t_sc, 4), "attn_decode_ms": round(t_att, 4),
            "roofline": {"kernel": "attn_decode_partial (hils_attn_decode, KV gather)", "bound": "hbm",
                         "achieved": round(gb / (t_att / 1e3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gb / (t_att / 1e3) / 1e9 / hbm, 4), "traffic": None,
                         "peak_source": f"{pk_kind} hbm_gbs", "algorithmic_bytes_per_launch": gb},
            "score_roofline": {"bound": "hbm", "achieved": round(sb / (t_sc / 1e3) / 1e9, 1), "peak": hbm,
                               "unit": "GB/s", "frac": round(sb / (t_sc / 1e3) / 1e9 / hbm, 4),
                               "algorithmic_bytes_per_launch": sb},
            "step_roofline_frac": round((sb + gb + qb) / (d_ms / 1e3) / 1e9 / hbm, 4),
            "summaries_ms": round(summ_ms, 3),
            "summaries_gbs": round((wd.B * wd.Hkv * wd.N * wd.d * 2 + 2 * wd.B * wd.Hq * wd.C * wd.d * 2)
                                   / (summ_ms / 1e3) / 1e9, 1),
            "gpu_launches": 4 * args.steps * 5}
        del xd, dec
        try:
            line["decode"]["offload"] = bench_decode_offload(dev, stream, args, ws, dist_on)
        except Exception as ex:  # host memory can run short on a box; report rather than stop
            line["decode"]["offload"] = {"unavailable": f"{type(ex).__name__}: {str(ex)[:200]}"}
    if not args.no_qcal and args.workload != "prefill_512k_qcal" and not args.seq_len:
        line["prefill_512k_qcal"] = extra_prefill(WORKLOADS["prefill_512k_qcal"], dev, stream, args, ws, dist_on, pk,
                                                  pk_kind)
    if not args.no_bwd:
        line["backward"] = bench_backward(WORKLOADS[args.bwd_workload], dev, stream, args, ws, dist_on)
    if not args.no_dense:
        try:
            dc = dense_comparator(dev, stream)
        except Exception as ex:  # the library comparator is context: its failure must not stop the bench
            dc = {"unavailable": f"{type(ex).__name__}: {str(ex)[:200]}"}
        if "prefill_512k_qcal" in line and "prefill_512k" in dc:
            dc["prefill_512k_ratio"] = round(dc["prefill_512k"]["ms"] / line["prefill_512k_qcal"]["ms_per_step"], 2)
        if not args.seq_len and args.workload == "prefill_128k" and "prefill_128k" in dc:
            dc["prefill_128k_ratio"] = round(dc["prefill_128k"]["ms"] / line["ms_per_step"], 2)
        if "decode" in line and "decode_512k" in dc:
            dc["decode_512k_ratio"] = round(dc["decode_512k"]["ms"] / line["decode"]["ms_per_step"], 2)
        line["dense_context"] = dc
    if rank == 0 and not args.no_cpu:
        v, done, t_s, t_r = cpu_baseline_prefill(w, x)
        line["cpu_baseline"] = {"value": round(v, 2), "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                                "sample": f"{done} random positions of {w.name} (all {w.Hq} heads; summaries of "
                                          f"the whole sequence amortised per position; {t_s:.1f}s summaries + "
                                          f"{t_r:.1f}s rows)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def attn_tiles(w) -> int:
    """Position tiles of the chunk-major attention (hils.h, hils_attn_prefill):
    the fewest tiles whose 1 KB partial records (one per position, KV group and
    selected chunk) fit about 8 GiB each.  Each tile launches seven kernels:
    bucket count, scan and scatter, the query regroup, the chunk-major pass,
    the window pass and the fusion."""
    per_pos = w.B * w.Hkv * w.K * w.G * w.d * 2
    cap = max(1, (8 << 30) // per_pos)
    return (w.N + cap - 1) // cap


def attn_tile_positions(w) -> int:
    """Positions per tile: N split evenly over the tiles, rounded up to 64."""
    nt = attn_tiles(w)
    pt = -(-w.N // nt)
    return -(-pt // 64) * 64


def run_config(w, ws):
    """The `config` object of both arms' JSON lines."""
    return {"workload": w.name, "batch": w.B, "seq_len": w.N, "n_q_heads": w.Hq, "n_kv_heads": w.Hkv,
            "head_dim": w.d, "chunk": w.S, "window": w.W, "top_k": w.K, "qcal_rank": w.qcal_rank,
            "parallelism": f"replica x{ws}",
            "l2": "inputs larger than L2 (q %.2f GB, k/v %.0f MB each)" % (
                w.B * w.Hq * w.N * w.d * 2 / 1e9, w.B * w.Hkv * w.N * w.d * 2 / 1e6)}


def reference_arm(args, ws, rank):
    """The oracle as the reference implementation, on the host cores."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    x = prefill_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    # every host core gets rows: the oracle spreads positions over its threads
    nrows = max(16, 2 * (os.cpu_count() or 8))
    vals = []
    for it in range(args.warmup + args.steps):
        v, done, _, _ = cpu_baseline_prefill(w, x, rows=nrows, seed=it)
        if it >= args.warmup:
            vals.append(v)
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * nrows / v, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run_config(w, ws),
            "cpu_baseline": {"value": round(v, 2), "unit": "tokens/s", "kind": "oracle", "cores": os.cpu_count(),
                             "sample": f"{nrows} random positions of {w.name} per step, all heads"},
            "e2e": {"value": round(v, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
