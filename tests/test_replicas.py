"""Multi-GPU runs of bench.py are independent replicas (the path has no exchange
step). What is shared between ranks is host logic: the whole job's step time is
the slowest rank's, the value counts the units of every rank, and the reference
arm runs on rank 0 only. These tests run that logic as two gloo ranks on the CPU."""
import json
import os
import socket
import sys
import types

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 2.0 + 3.0 * rank                      # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        e2e = bench.max_over_ranks(10.0 - rank, dist, torch.device("cpu"))   # rank 0 is slow here
        value = bench.job_value(1000, world, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "e2e": e2e, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_rank(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["slowest"] == 5.0          # max over ranks, seen identically by every rank
        assert r["e2e"] == 10.0
        assert r["value"] == pytest.approx(1000 * 2 / 5e-3)   # all ranks' units over the slowest time


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.job_value(10, 1, 2.0) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    args = types.SimpleNamespace(workload="decode_32k", steps=1, warmup=0, gpus=2)
    bench.run_reference(args, rank=1)      # returns before building anything
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line(capsys):
    """Rank 0 times the oracle on a bounded sample and prints one JSON line with the
    arm's keys and the same workload config as the CUDA arm."""
    import json

    args = types.SimpleNamespace(workload="single_layer_2k", steps=1, warmup=0, gpus=1)
    bench.run_reference(args, rank=0)
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["higher_is_better"] is True and line["n_gpus"] == 1
    cfg = dict(line["config"])
    cfg.pop("sample")
    assert cfg == bench.workload_config("single_layer_2k", 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def _fake_measure(name, args, dist_, world, steps, headline):
    """Stands in for the GPU measurement: rank r's step takes 2 + r ms."""
    ms = bench.max_over_ranks(2.0 + dist_.get_rank(), dist_, torch.device("cpu"))
    return {"value": bench.job_value(100, world, ms), "unit": bench.UNIT, "ms_per_step": ms, "steps": steps,
            "gpu_launches": 2 * steps, "clocks": {"sm_mhz": None}, "roofline": None, "e2e": None,
            "tokens_per_s": world / (ms * 1e-3), "graph": True}


def _main_rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import contextlib
    with open(os.path.join(out_dir, f"main{rank}.txt"), "w") as f, contextlib.redirect_stdout(f):
        bench.main(["--gpus", str(world), "--steps", "3", "--warmup", "3", "--extra", "verify_2req_229k"],
                   measure=_fake_measure)


def test_bench_main_runs_two_ranks_end_to_end(tmp_path):
    """bench.main()'s rank logic on two gloo ranks: process-group set-up, the same
    measurements in the same order on every rank, max over ranks, one JSON line
    from rank 0 (headline + extra workload), one clean teardown, exit 0."""
    world = 2
    mp.spawn(_main_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    out0 = (tmp_path / "main0.txt").read_text().splitlines()
    out1 = (tmp_path / "main1.txt").read_text().splitlines()
    assert out1 == []
    assert len(out0) == 1
    line = json.loads(out0[0])
    assert line["n_gpus"] == 2 and line["ms_per_step"] == 3.0
    assert line["value"] == pytest.approx(100 * 2 / 3e-3)
    assert line["scaling"] == "weak" and line["config"]["parallelism"] == "replicas x2"
    assert list(line["workloads"]) == ["verify_2req_229k"]
    assert line["workloads"]["verify_2req_229k"]["ms_per_step"] == 3.0


def test_bench_refuses_gpus_that_do_not_match_the_ranks(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "8"], measure=_fake_measure)
