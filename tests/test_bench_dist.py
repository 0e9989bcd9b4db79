"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

With N GPUs every rank times its own independent batch; the job's time is
the slowest rank's (max over ranks) and its throughput counts every rank's
work. The reference arm runs on rank 0 only; the other ranks do no work.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slowest
        total = bench.max_over_ranks(local_ms, world)
        value = bench.job_tflops(world, 1e12, 4, total)
        dist.barrier()
        results[rank] = (total, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    assert res[0] == res[1]
    total, value = res[0]
    assert total == 15.0
    # 2 ranks x 4 steps x 1e12 FLOP in 15 ms
    assert value == pytest.approx(2 * 4 * 1e12 / 15e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tflops(1, 2e12, 10, 20.0) == pytest.approx(1000.0)


def test_flop_counts():
    # causal pairs T(T+1)/2; key padding sum of L(L+1)/2 + (T-L)L
    assert bench.allowed_pairs(1, 4096) == 4096 * 4097 // 2
    assert bench.allowed_pairs(2, 8, valid_len=[8, 3]) == 36 + (6 + 5 * 3)
    assert bench.attn_flops(1, 4096) == 64 * (4096 * 4097 // 2) * 2 * (192 + 128)
    assert bench.oproj_flops(4096) == 2 * 4096 * 8192 * 7168


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        steps, warmup = 1, 3
    bench.run_reference(A(), None, rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_fp8_oproj_flag_host_logic():
    """--oproj fp8 names the FP8 o_proj in the config, and is refused for
    the compact-mask workload (no fused FP8 varlen call) and the reference
    arm."""
    import subprocess
    import sys
    from mla_causal_attention_attn_b200 import inputs
    w = inputs.WORKLOADS["b1_t4096_causal"]
    assert "e4m3" in bench.workload_config(w, oproj="fp8")["o_proj"]
    assert bench.workload_config(w)["o_proj"] == "8192 -> 7168"
    for extra in (["--workload", "b8_t4096_keypad_varlen"], ["--impl", "reference"]):
        r = subprocess.run([sys.executable, bench.__file__, "--oproj", "fp8"] + extra,
                           capture_output=True, text=True, timeout=120)
        assert r.returncode == 2 and "--oproj fp8" in r.stderr, r.stderr
