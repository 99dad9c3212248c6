"""The N>1 host logic of bench.py on CPU: two gloo ranks, max-over-ranks
timing, and the launcher checks.  No GPU is touched."""
import json

import numpy as np
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


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.aggregate_max(values[rank], world)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    values = [3.25, 7.5]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert out[0] == 7.5 and out[1] == 7.5


def test_single_rank_needs_no_process_group():
    assert bench.aggregate_max(1.5, 1) == 1.5


def test_gpus_must_match_world_size(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2"])
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "1"])


def test_reference_arm_is_silent_on_other_ranks(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--gpus", "2", "--impl", "reference", "--steps", "1"]) == 0
    assert capsys.readouterr().out == ""


def test_algorithmic_counts_of_the_qkv_workload():
    import workloads
    wl = workloads.make_workload("qkv_prefill_4096", M=4, N=8, with_weights=False)
    ops, rq, gm = bench.algorithmic_counts(wl, 2048, 4096)
    assert ops == 2.0 * 2048 * 12288 * 4096
    assert rq == 2048 * 4096 * 2 + 2048 * 4096 / 2 + 2048 * 4


def test_fused_decode_step_bytes():
    # the fused step moves X in, the codes, scales and outlier copy out, the
    # weight side in and Y out, counted by hand for the QUIK decode layer
    import workloads
    wl = workloads.make_workload("quik_decode_8192", M=4, N=8, with_weights=False)
    M, K, N, n_out = 64, 8192, 8192, 256
    kp = 8192
    x_in = M * K * 2
    a_out = M * (K - n_out) // 2 + M * 4 + M * n_out * 2
    w_in = N * (K - n_out) // 2 + N * 4 + N * n_out * 2
    y_out = M * N * 2
    assert bench.fused_step_bytes(wl, M, kp) == x_in + a_out + w_in + y_out
    # asymmetric activations add a zero point per token and a code sum per weight row
    assert bench.fused_step_bytes(wl, M, kp, asym=True) == x_in + a_out + w_in + y_out + M * 4 + N * 4


def test_reference_arm_with_random_signs(capsys):
    # the oracle arm takes the same randomized rotation as the GPU arm
    assert bench.main(["--impl", "reference", "--workload", "tiny_256", "--random-signs",
                       "--steps", "2", "--warmup", "3", "--reference-tokens", "8"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["workload"] == "tiny_256"
    import workloads
    wl = workloads.make_workload("tiny_256")
    d = bench.oracle_signs(wl, True)
    assert d is not None and d.shape == (256,) and bench.oracle_rotation(wl, d).signs is d
    # the GPU arm sizes the same signs from its own packed width
    assert np.array_equal(bench.workload_signs(wl, True, 256), d)


def test_gpu_arm_never_reaches_the_oracle():
    # the GPU arm, and every helper it calls to shape its inputs, imports and
    # calls nothing from the oracle; only the CPU-baseline and reference legs do
    import inspect
    for fn in (bench.run_ours, bench.workload_signs, bench.rotation_for, bench.run_kv,
               bench.rotate_quant_roofline, bench.algorithmic_counts, bench.kron_split_flops,
               bench.fused_step_bytes):
        src = inspect.getsource(fn)
        assert "import oracle" not in src and "O." not in src, fn.__name__
        assert "oracle_signs" not in src and "oracle_rotation" not in src, fn.__name__


def test_kv_cache_reference_arm(capsys):
    # the KV-cache workload's reference arm: the oracle's R3 + g128 step
    assert bench.main(["--impl", "reference", "--workload", "kv_cache_llama2_7b", "--steps", "1",
                       "--warmup", "3", "--reference-tokens", "4"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.KV_METRIC
    assert line["config"]["tokens"] == 4 and line["config"]["group"] == 128
    import workloads
    s = workloads.KV_SPECS["kv_cache_llama2_7b"]
    # q, k, v read, q written (fp16); k and v codes (half a byte) + scale and zero per group
    w = s.heads * s.head_dim
    assert bench.kv_bytes(s, 4) == 4 * w * 8 + 2 * (4 * w // 2 + 4 * (w // 128) * 8)
