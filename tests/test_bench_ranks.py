"""bench.py's multi-rank plumbing on the CPU with world size 2 (gloo over
127.0.0.1, launched by torchrun): the ranks rendezvous, the timing is the
maximum over ranks, and the reference arm runs and prints on rank 0 alone
while rank 1 exits cleanly without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun(args, timeout=240):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}"] + args
    env = dict(os.environ, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def json_lines(text):
    """Every JSON object printed by the ranks (their lines may arrive joined)."""
    dec, out, i = json.JSONDecoder(), [], 0
    while True:
        i = text.find("{", i)
        if i < 0:
            return out
        obj, i = dec.raw_decode(text, i)
        out.append(obj)


def test_ranks_meet_and_time_is_the_max_over_ranks():
    p = torchrun([os.path.join("tests", "rank_worker.py")])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = json_lines(p.stdout)
    assert sorted(l["rank"] for l in lines) == [0, 1]
    for l in lines:
        assert l["world"] == 2 and l["local"] == l["rank"]
        assert l["max"] == 3.0  # max(1.5 * 1, 1.5 * 2) on both ranks


def test_reference_arm_runs_on_rank_zero_only():
    p = torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "2",
                  "--warmup", "1", "--workload", "tiny-f32", "--ref-seconds", "3"])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = json_lines(p.stdout)
    assert len(lines) == 1  # one line, from rank 0
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
