"""The benchmark's host side, without a GPU: the JSON line of the reference
arm (the oracle timed on the host cores), the rank and argument rules, and
the algorithmic byte accounting of every workload shape."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env=None, timeout=300):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          timeout=timeout, env=e, cwd=ROOT)


def test_reference_arm_line():
    res = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, "one JSON line"
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "rows/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["data"] == "synthetic" and d["dtype"] == "bf16"
    assert d["config"]["workload"] == "greedy_llama3"
    assert (d["config"]["B"], d["config"]["k"], d["config"]["V"]) == (64, 5, 128256)
    # the same config dict as our arm's line for the same workload
    assert d["config"] == bench.line_config("greedy_llama3", bench.make_workload("greedy_llama3"), 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_nothing():
    res = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"], env={"RANK": "1", "WORLD_SIZE": "2"})
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_argument_rules():
    a = bench.parse_args([])
    assert a.workload == "greedy_llama3" and a.intervals >= 30 and a.gpus is None
    assert set(a.also) == set(bench.SUITE) - {"greedy_llama3"}
    assert bench.parse_args(["--also", ""]).also == []
    with pytest.raises(SystemExit):
        bench.parse_args(["--also", "greedy_tiny,nonsense"])


def test_gpus_must_match_the_launcher():
    """Under a launcher, --gpus N must equal the ranks it started."""
    res = _run(["--gpus", "1", "--steps", "1", "--warmup", "3"], env={"WORLD_SIZE": "2", "RANK": "0"})
    assert res.returncode != 0 and "WORLD_SIZE" in res.stderr


def test_gpus_without_a_launcher_starts_the_ranks(monkeypatch):
    """`--gpus N` (N > 1) with no launcher starts N ranks under
    torch.distributed.run on 127.0.0.1 instead of timing one GPU."""
    seen = {}

    class FakeProc:
        pid = 0

        def wait(self, timeout=None):
            return 0

    def fake_popen(cmd, start_new_session=False):
        seen["cmd"], seen["session"] = cmd, start_new_session
        return FakeProc()

    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "Popen", fake_popen)
    monkeypatch.setattr(bench, "run_ours", lambda a: pytest.fail("timed one GPU instead of starting the ranks"))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "3", "--warmup", "3"])
    assert bench.main() == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1" and seen["session"]
    assert cmd[-6:] == ["--gpus", "4", "--steps", "3", "--warmup", "3"]


def test_warmup_floor():
    res = _run(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert res.returncode != 0 and "warmup" in res.stderr


def _greedy(B, k, V, dtype, topk=0):
    return gen.GreedyInputs("shape", dtype, None, None, B, k, V, topk)


def test_algorithmic_bytes_of_the_workload_shapes():
    # greedy: one read of every row, the drafts, accept_len and out_tokens
    assert gen.algorithmic_bytes(_greedy(64, 5, 128256, gen.BF16)) == 64 * 6 * 128256 * 2 + 64 * 5 * 4 + 64 * 4 + 64 * 6 * 4
    assert gen.algorithmic_bytes(_greedy(64, 5, 128256, gen.BF16)) == 98503680
    # top-8 adds an id and a value (4 + 4 bytes) per row and slot
    c4 = gen.algorithmic_bytes(_greedy(256, 8, 128256, gen.BF16, topk=8))
    assert c4 == 256 * 9 * 128256 * 2 + 256 * 8 * 4 + 256 * 4 + 256 * 9 * 4 + 256 * 9 * 8 * 8
    # tree: the rows, parents and node tokens, and the three outputs
    t = gen.TreeInputs("shape", gen.BF16, None, None, None, 16, 64, 128256, 6)
    assert gen.algorithmic_bytes(t) == 16 * 65 * 128256 * 2 + 2 * 16 * 65 * 4 + 16 * 4 + 16 * 6 * 4 + 16 * 7 * 4
    # rejection: the target rows, the drafts, the two gathers per draft, the outputs
    r = gen.RejectionInputs("shape", gen.F32, None, None, None, 32, 4, 151936)
    assert gen.algorithmic_bytes(r) == 32 * 5 * 151936 * 4 + 32 * 4 * 4 + 2 * 32 * 4 * 4 + 32 * 4 + 32 * 5 * 4


@pytest.mark.parametrize("stats", [False, True])
def test_resample_bytes_follow_the_accepted_lengths(stats):
    import torch
    r = gen.RejectionInputs("shape", gen.F32, None, None, None, 4, 3, 1000)
    r.stats = stats
    al = torch.tensor([0, 3, -1, 2], dtype=torch.int32)
    got = bench.resample_bytes(r, (al,))
    # row h of the target for every valid request, q_h where h < k
    want = 1000 * (4 * 3 + 4 * 2)
    if stats:  # the statistics re-read rows 0..k-1 of target and q of every valid request
        want += 3 * 3 * (1000 * 8 + 16)
    assert got == want
    assert bench.resample_bytes(_greedy(4, 3, 1000, gen.F32), (al,)) == 0


def test_greedy_launch_count():
    """One launch for requests of at most 32 KB of logits without top-k (the
    tiny batch), two otherwise."""
    assert bench.greedy_launches(gen.GreedyInputs("s", gen.F32, None, None, 4, 4, 1000)) == 1
    assert bench.greedy_launches(gen.GreedyInputs("s", gen.F32, None, None, 4, 3, 2048)) == 1
    assert bench.greedy_launches(gen.GreedyInputs("s", gen.F32, None, None, 4, 3, 2049)) == 2
    assert bench.greedy_launches(gen.GreedyInputs("s", gen.F32, None, None, 4, 4, 1000, topk=8)) == 2
    assert bench.greedy_launches(gen.GreedyInputs("s", gen.BF16, None, None, 64, 5, 128256)) == 2


def test_rows_of_each_layout():
    g = _greedy(7, 3, 50, gen.F32)
    assert bench.rows_of(g) == 28 and bench.rows_of(g, 2) == 8
    t = gen.TreeInputs("shape", gen.BF16, None, None, None, 5, 64, 100, 6)
    assert bench.rows_of(t) == 5 * 65
    off = np.array([0, 1, 4, 4, 11], np.int32)
    rg = gen.RaggedInputs("shape", gen.BF16, None, None, off, 4, 7, 100)
    assert bench.rows_of(rg) == 15 and bench.rows_of(rg, 2) == 4 + 2
