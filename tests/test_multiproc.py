"""The N > 1 host path of bench.py on world-size-2 gloo ranks (CPU only):
max/sum over ranks, the barrier, and the reference arm that only rank 0 runs.
Each rank of a multi-GPU run processes its own batch (weak scaling, no
data-path collective), so these reductions are the only cross-rank steps."""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_CODE = r"""
import os, sys
sys.path.insert(0, {root!r})
import bench
rank, ws, _ = bench.dist_setup("gloo", timeout_s=60)
assert ws == 2
assert bench.max_over_ranks(rank + 1.5, ws) == 2.5
assert bench.sum_over_ranks(rank + 1.0, ws) == 3.0
bench.barrier(ws, cuda=False)
if rank == 1:
    # the reference arm: rank 0 alone runs the oracle, the others exit 0
    assert bench.run_reference(bench.parse(["--impl", "reference", "--steps", "1",
                                            "--warmup", "0"])) == 0
bench.barrier(ws, cuda=False)
import torch.distributed as dist
dist.destroy_process_group()
print("rank", rank, "ok")
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_CODE.format(root=ROOT)],
                                      env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        outs.append((p.returncode, out, err))
    for rank, (rc, out, err) in enumerate(outs):
        assert rc == 0, f"rank {rank}: {err[-2000:]}"
        assert f"rank {rank} ok" in out
