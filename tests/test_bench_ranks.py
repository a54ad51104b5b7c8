"""Host logic of the multi-GPU benchmark on the CPU: two gloo ranks.

The benchmark runs one independent replica per GPU (weak scaling, no
collective on the data path); torch.distributed only takes the barrier and
the maximum over ranks of the step time.  Checked here with world size 2: the
reduction returns the slowest rank's time on every rank, the replicas draw
different prompt blocks, and the reference arm prints its one line from rank
0 only (the other ranks exit 0 without work)."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_max_over_ranks_and_distinct_prompts():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.join(ROOT, "tests", "rank_worker.py")],
                                      env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for pr in procs:
        out, err = pr.communicate(timeout=180)
        assert pr.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert [o["max"] for o in outs] == [107.0, 107.0]
    assert [o["max2"] for o in outs] == [5.0, 5.0]
    assert outs[0]["prompt_tid"] != outs[1]["prompt_tid"]


def _reference(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "3"],
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_on_rank0_only():
    r1 = _reference(1)
    assert r1.returncode == 0 and r1.stdout.strip() == "", (r1.stdout, r1.stderr[-2000:])
    r0 = _reference(0)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
