"""The benchmark's multi-rank bookkeeping (barrier, max and sum over ranks,
one JSON line from rank 0) with two gloo ranks on the CPU. The data path has
no collective: each rank runs an independent layer (replicas)."""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_max_and_sum(tmp_path):
    script = tmp_path / "ranks.py"
    script.write_text(textwrap.dedent(f"""
        import os, sys
        sys.path.insert(0, {ROOT!r})
        import torch.distributed as dist
        import bench
        rank, world, local = bench.dist_setup(2)
        assert world == 2 and dist.get_backend() == "gloo"
        bench.barrier(world)
        mx = bench.max_over_ranks(10.0 + rank, world)
        sm = bench.sum_over_ranks(1.5 * (rank + 1), world)
        print(f"rank {{rank}} max {{mx}} sum {{sm}}", flush=True)
        dist.destroy_process_group()
    """))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), WORLD_SIZE="2",
               CUDA_VISIBLE_DEVICES="")
    procs = []
    for r in range(2):
        e = dict(env, RANK=str(r), LOCAL_RANK=str(r))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=e, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    for r, (p, out) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, out
        assert f"rank {r} max 11.0 sum 4.5" in out, out
