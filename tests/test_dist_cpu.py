"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1 (the data
path has no collective; only the timing reductions and barriers cross ranks)."""
import json
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def run_ranks(code: str, world: int = 2, timeout: int = 120):
    port = free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code], cwd=ROOT, env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=timeout)
        outs.append((p.returncode, out, err))
    return outs


def test_timing_reductions_over_two_gloo_ranks():
    code = textwrap.dedent("""
        import json, types
        import bench
        world, rank, local = bench.dist_setup(types.SimpleNamespace())
        bench.barrier(world)
        r = {"world": world, "rank": rank,
             "max": bench.max_over_ranks(rank + 1.5, world),
             "sum": bench.sum_over_ranks(1.0 + rank, world)}
        bench.barrier(world)
        import torch.distributed as dist
        dist.destroy_process_group()
        print(json.dumps(r))
    """)
    for rc, out, err in run_ranks(code):
        assert rc == 0, err[-2000:]
        r = json.loads(out.strip().splitlines()[-1])
        assert r["world"] == 2 and r["max"] == 2.5 and r["sum"] == 3.0


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
