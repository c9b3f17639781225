"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2): every
rank reports the slowest rank's time, the whole-job rate counts every rank's
units over that time, and the reference arm runs on rank 0 only."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(ms, True, device="cpu")
        rate = bench.whole_job_rate(131072, world, got)
        dist.barrier()
        out[rank] = torch.tensor([got, rate], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_rate_gloo():
    world = 2
    out = torch.zeros(world, 2, dtype=torch.float64).share_memory_()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        assert out[r, 0].item() == 15.0                          # the max, on every rank
        assert abs(out[r, 1].item() - 2 * 131072 / 0.015) < 1e-6  # all ranks' tokens / max time


def test_single_rank_is_local():
    assert bench.max_over_ranks(3.5, False) == 3.5
    assert bench.whole_job_rate(100, 1, 1000.0) == 100.0


def test_reference_arm_other_ranks_do_no_work():
    class A:
        workload, warmup, steps = "prefill_128k", 3, 1
    assert bench.reference_arm(A(), 2, 1) is None  # returns before touching inputs


def test_both_arms_share_the_config_object():
    w = bench.WORKLOADS["prefill_128k"]
    c = bench.run_config(w, 2)
    assert c["workload"] == "prefill_128k" and c["seq_len"] == 131072 and c["parallelism"] == "replica x2"


def test_attention_tiles_and_traffic_lookup():
    """Tile counts of the chunk-major attention (fewest tiles of <= 8 GiB of
    1 KB records) and the traffic record, which is used only while the
    measured kernel sources are unchanged."""
    from chunk_wise_sparse_landmark_b200.inputs import WORKLOADS
    assert bench.attn_tiles(WORKLOADS["prefill_128k"]) == 4
    assert bench.attn_tiles(WORKLOADS["prefill_512k_qcal"]) == 32
    assert bench.attn_tiles(WORKLOADS["prefill_8k"]) == 1
    files = ["attn_chunk.cu", "attn_window.cu", "common.cuh"]
    t = bench.traffic_for(files, "hils_attn_prefill", "prefill_128k")
    assert t is None or t > 0
    assert bench.traffic_for(["attn_chunk.cu"], "hils_attn_prefill", "prefill_128k") is None  # other sources
    assert bench.traffic_for(files, "hils_attn_prefill", "no_such_workload") is None
