"""The N > 1 path of bench.py on the CPU: two gloo ranks exercise the barrier and the
max-over-ranks timing reduction (the layer itself needs no collective: each rank is
an independent replica), and the reference arm exits on non-zero ranks."""

import os
import socket
import sys
import types

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        mx = bench.max_over_ranks(1.5 + rank, world)   # rank r reports 1.5 + r
        results[rank] = mx
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    mgr = mp.Manager()
    results = mgr.dict()
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, results), nprocs=2, join=True)
    assert dict(results) == {0: 2.5, 1: 2.5}


def test_single_rank_helpers_are_no_ops():
    sys.path.insert(0, ROOT)
    import bench
    bench.barrier(1)
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench
    args = types.SimpleNamespace(workload="tiny", steps=1, warmup=0, seed=0, gpus=2)
    assert bench.reference_arm(args, ws=2, rank=1) == 0     # no work, no output


def test_reference_arm_prints_one_line(capsys):
    sys.path.insert(0, ROOT)
    import json
    import bench
    args = types.SimpleNamespace(workload="tiny", steps=1, warmup=0, seed=0, gpus=1)
    assert bench.reference_arm(args, ws=1, rank=0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    # the same workload description as the main arm, so both lines name one config
    from mixture_experts_layer_sort_b200 import synth
    wl = synth.WORKLOADS["tiny"]
    assert line["config"] == bench.bench_config(wl, list(wl.Ms), 1, bench.l2_plan(wl, "bf16", "rotate")[2])


def test_l2_plan_weight_sets():
    """The rotation keeps at least 2 x L2 of other weights between two forwards on one
    set: the decode layer needs 5 bf16 sets (M = 1 streams 8 experts, 75.5 MB) and 8 e4m3
    sets; the E=256 layer 2; the tiny layer would need hundreds and is flushed instead."""
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_sort_b200 import synth
    W = synth.WORKLOADS
    assert bench.l2_plan(W["decode"], "bf16", "rotate")[:2] == ("rotate", 5)
    assert bench.l2_plan(W["decode_fp8"], "fp8", "rotate")[:2] == ("rotate", 8)
    assert bench.l2_plan(W["large_decode"], "bf16", "rotate")[:2] == ("rotate", 2)
    assert bench.l2_plan(W["prefill"], "fp8", "rotate")[:2] == ("rotate", 2)
    assert bench.l2_plan(W["tiny"], "bf16", "rotate")[:2] == ("flush", 1)
    assert bench.l2_plan(W["decode"], "bf16", "flush")[:2] == ("flush", 1)
    assert bench.l2_plan(W["decode"], "bf16", "warm")[:2] == ("warm", 1)
    for name, dt in (("decode", "bf16"), ("decode_fp8", "fp8"), ("large_decode", "bf16"), ("prefill", "fp8")):
        wl = W[name]
        mode, R, _ = bench.l2_plan(wl, dt, "rotate")
        fewest = wl.k * 3 * wl.H * wl.I * bench.weight_bytes(dt)
        assert (R - 1) * fewest >= 2 * bench.L2_BYTES and (R - 2) * fewest < 2 * bench.L2_BYTES


def test_roofline_numerators_by_hand():
    """The bytes and FLOPs the roofline fractions divide by, worked out by hand for the
    decode layer (E=128, k=8, H=2048, I=768) and the prefill layer (E=256, H=7168,
    I=2048): each active expert streams W_gate, W_up and W_down once (3*H*I weights),
    plus x in, out back, the logits and (FP8) the scale table; 2*M*k*3*H*I FLOPs."""
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_sort_b200 import synth
    dec, pre = synth.WORKLOADS["decode"], synth.WORKLOADS["prefill"]
    # M = 1 activates k = 8 experts: 8 * 3 * 2048 * 768 * 2 B + 2048*2*2 (x, out) + 128*4 (logits)
    assert bench.alg_bytes_layer(dec, "bf16", 1, 8) == 75497472 + 8192 + 512
    # e4m3: one byte per weight, plus 128 experts x 3 fp32 scales
    assert bench.alg_bytes_layer(dec, "fp8", 1, 8) == 37748736 + 8192 + 512 + 1536
    # prefill, every expert active: 256 * 3 * 7168 * 2048 * 2 B = 22.5 GB of weights
    assert bench.alg_bytes_layer(pre, "bf16", 4096, 256) == 22548578304 + 4096 * 7168 * 4 + 4096 * 256 * 4
    assert bench.alg_flops_layer(dec, 1) == 2 * 8 * 3 * 2048 * 768
    assert bench.alg_flops_layer(pre, 4096) == 2 * 4096 * 8 * 3 * 7168 * 2048
