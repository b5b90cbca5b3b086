"""bench.py's multi-process plumbing on CPU (gloo, world size 2) and its work model.

The timed GPU legs need a B200; what runs per rank around them -- process-group set-up,
barriers, the max-over-ranks reduction of the timed region, per-rank seeds (every rank
runs its own independent sequence: weak scaling, no collective on the data path) and the
reference arm's rank-0-only rule -- is exercised here with real processes."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from selective_state_space_10_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    assert bench.dist_env() == (rank, world, rank)
    dist = bench.init_dist(world, "gloo")
    bench.barrier(world)
    t_max = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
    seed = bench.rank_seed(inputs.BY_NAME["mamba2_2.7b_prefill"].seed, rank)
    seeds = [None] * world
    dist.all_gather_object(seeds, seed)
    # the reference arm: ranks other than 0 leave at once, without work
    rc = bench.run_reference(type("A", (), {"workload": "mamba2_2.7b_prefill", "steps": 1, "warmup": 3})()) \
        if rank != 0 else 0
    bench.barrier(world)
    dist.destroy_process_group()
    out.put((rank, t_max, seeds, rc))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, t_max, seeds, rc in res:
        assert t_max == 11.0            # the slowest rank's time is the job's time
        assert len(set(seeds)) == 2     # independent sequences per rank
        assert rc == 0
    assert res[0][2] == res[1][2]


def test_work_model_matches_the_hand_computed_budgets():
    """Dense-tile FLOPs and minimum bytes of the 2.7B- and 130M-shaped prefills."""
    w2 = inputs.BY_NAME["mamba2_2.7b_prefill"]
    dense, causal, min_bytes = bench.prefill_work(w2)
    assert dense == pytest.approx(21.74e9, rel=2e-3)
    assert causal == pytest.approx(16.26e9, rel=2e-3)
    # x, B, C bf16 + dt + A, D in; y fp32 + final state out
    assert min_bytes == 4096 * 80 * 64 * 2 + 2 * 4096 * 128 * 2 + 4096 * 80 * 4 + 2 * 80 * 4 \
        + 4096 * 80 * 64 * 4 + 80 * 64 * 128 * 4
    w1 = inputs.BY_NAME["mamba2_130m_prefill"]
    assert bench.prefill_work(w1)[0] == pytest.approx(6.71e9, rel=3e-3)


def test_kernel_work_is_below_the_ridge_for_the_tensor_core_kernels():
    """The tensor-core kernels report tensor work first; their intensity over the bytes
    that must cross DRAM is still below the measured ridge (1657.6 TFLOP/s / 6539.2 GB/s),
    and the pipeline bytes (with L2 intermediates) exceed the DRAM minimum."""
    w = inputs.BY_NAME["mamba2_2.7b_prefill"]
    for name in ("chunk_state_tc", "chunk_scan_tc"):
        kind, pipe, dram_min, flops = bench.kernel_work(name, w, w.chunk)
        assert kind == "tensor" and pipe > dram_min > 0
        assert flops / dram_min < 1657.6e12 / 6539.2e9


def test_roofline_entry_of_a_tensor_core_kernel():
    w = inputs.BY_NAME["mamba2_2.7b_prefill"]
    peaks = {"hbm_gbs": 6539.2, "bf16_tflops": 1657.6, "source": "measured"}
    e = bench.roofline_entry("chunk_scan_tc", w, w.chunk, 0.025, peaks, None)
    flops = bench.kernel_work("chunk_scan_tc", w, w.chunk)[3]
    assert e["bound"] == "tensor" and e["unit"] == "TFLOP/s"
    assert e["achieved"] == pytest.approx(flops / 25e-6 / 1e12)
    assert e["frac"] == pytest.approx(e["achieved"] / 1657.6)
    assert e["hbm_min"]["frac"] == pytest.approx(e["hbm_min"]["bytes"] / 25e-6 / 1e9 / 6539.2)
    assert "not an HBM figure" in e["pipeline"]["what"]


def test_committed_traffic_counters_follow_the_kernel_sources(tmp_path, monkeypatch):
    """The roofline's `traffic` comes from a committed ncu summary only while the code of the
    kernel's sources is the code that was profiled: a summary in profiles/ gives its counters
    for the sources it names or nothing (the bench then reports null), a changed statement
    voids it, a changed comment does not."""
    for kernel in ("chunk_scan_tc", "chunk_state_tc", "state_passing_bf16", "decode_step"):
        wl = "mamba2_2.7b_decode_b256" if kernel == "decode_step" else "mamba2_2.7b_prefill"
        t = bench.profile_traffic(kernel, wl)
        assert t is None or t > 0, kernel
    assert bench.profile_traffic("chunk_scan_tc", "no_such_workload") is None

    src = tmp_path / "k.cu"
    src.write_text("__global__ void k(float *p) { p[0] = 1.f; }  // one\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cu"])
    (tmp_path / "profiles" / "k.w.txt").write_text(
        f"# summary\ntraffic_bytes_per_launch = 1234\nsources = k.cu\nsources_sha256 = {digest}\n")
    assert bench.profile_traffic("k", "w") == 1234.0
    src.write_text("__global__ void k(float *p) {\n  p[0] = 1.f;  /* two */\n}\n")
    assert bench.profile_traffic("k", "w") == 1234.0      # comments and layout only
    src.write_text("__global__ void k(float *p) { p[0] = 2.f; }\n")
    assert bench.profile_traffic("k", "w") is None        # the code changed
