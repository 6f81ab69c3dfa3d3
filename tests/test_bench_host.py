"""Host logic of bench.py that runs without a GPU: the cross-rank reduction of
timings (two gloo ranks on CPU), the whole-job throughput and the reference
arm's behaviour on ranks other than 0."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q.put((rank, bench.max_over_ranks(values[rank], "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    # Each rank reports its own time; both must see the slowest one.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    values = [3.25, 7.5]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 7.5, 1: 7.5}


def test_max_over_ranks_without_process_group():
    assert bench.max_over_ranks(2.5, "cpu") == 2.5


def test_job_tflops_counts_every_rank():
    # 2 ranks x 10 steps x 90.19 GFLOP in 5.2 ms (slowest rank).
    v = bench.job_tflops(2, 10, 90.194313216e9, 5.2)
    assert v == pytest.approx(2 * 10 * 90.194313216e9 / 5.2e-3 / 1e12)
    assert bench.job_tflops(1, 10, 90.194313216e9, 5.2) == pytest.approx(v / 2)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    # Under torchrun only rank 0 times the oracle and prints; the others exit
    # 0 at once, without output.
    monkeypatch.setenv("RANK", "1")
    from causal_self_attention_flashattention_b200.workload import WORKLOADS

    class Args:
        steps, warmup, gpus = 3, 3, 2

    assert bench.run_reference(Args, WORKLOADS["gpt2-124m-b16-t1024"]) == 0
    assert capsys.readouterr().out == ""


def test_traffic_figures_follow_their_kernel_sources(tmp_path, monkeypatch):
    # A committed DRAM figure counts only while its kernel's sources are the
    # ones it was measured on.
    import json

    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.kernel_digest("bwd_dkdv")
    (prof / "traffic.json").write_text(json.dumps({"kernels": {
        "bwd_dkdv": {"dram_bytes_per_launch": 1.0, "src_digest": good},
        "fwd": {"dram_bytes_per_launch": 2.0, "src_digest": "0" * 16},
        "unknown_kernel": {"dram_bytes_per_launch": 3.0, "src_digest": good}}}))
    csrc = os.path.join(ROOT, "causal_self_attention_flashattention_b200", "csrc")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_digest",
                        lambda k, c=None, _orig=bench.kernel_digest: _orig(k, c or csrc))
    assert bench.load_traffic() == {"bwd_dkdv": {"dram_bytes_per_launch": 1.0, "src_digest": good}}
