"""`bench.py --gpus N` on one node: N ranks under torch.distributed.run, the
world-size checks, the max over ranks and the line that rank 0 alone prints.
Run on the CPU with two gloo ranks; each rank's GPU measurement is replaced
by a stub that reports a different step time per rank."""
import json
import os
import sys
import textwrap

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STUB = textwrap.dedent('''
    import os, sys
    sys.path.insert(0, {root!r})
    import bench

    def measure(args, world, local):
        import torch
        rank = int(os.environ["RANK"])
        with open(os.path.join({out!r}, "rank%d" % rank), "w") as fh:
            fh.write("%d %d" % (world, local))
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world,
                                  torch.device("cpu"))
        per_kind = {{"gemm_block_scaled": {{"ms": ms, "units": 2e12,
                                           "launches": 4}}}}
        return {{"ms": ms, "flops": 2e12, "per_kind": per_kind,
                "next_rows": None, "clocks": None, "e2e": None,
                "launches_per_step": 4}}

    sys.exit(bench.main(sys.argv[1:], measure=measure))
''')


def test_two_ranks_are_started_and_rank_zero_reports_the_job(tmp_path, capfd):
    script = tmp_path / "stub_bench.py"
    script.write_text(STUB.format(root=ROOT, out=str(tmp_path)))
    rc = bench.launch_ranks(
        2, ["--gpus", "2", "--steps", "3", "--warmup", "1",
            "--no-cpu-baseline"], script=str(script), timeout_s=600)
    out = capfd.readouterr().out
    assert rc == 0, out
    # both ranks ran, each saw a world of 2 and its own local rank
    assert (tmp_path / "rank0").read_text() == "2 0"
    assert (tmp_path / "rank1").read_text() == "2 1"
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["ms_per_step"] == 15.0      # the slower rank's time
    # whole-job throughput: both ranks' work over the max time
    assert abs(line["value"] - 2 * 2e12 / 0.015 / 1e12) < 1e-6
    assert line["config"]["parallelism"] == "replicas"
    assert line["gpu_launches"] == 4 * 3


def test_world_size_must_match_gpus(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.check_launch(4) == 2
    assert "WORLD_SIZE=2" in capsys.readouterr().err
    assert bench.check_launch(2) is None


def test_gpus_above_one_outside_torchrun_starts_ranks(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    seen = []
    monkeypatch.setattr(bench, "launch_ranks",
                        lambda n, argv, **kw: seen.append((n, argv)) or 7)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4"])
    assert bench.check_launch(4) == 7
    assert seen == [(4, ["--gpus", "4"])]
    assert bench.check_launch(1) is None    # one GPU: this process runs it
