"""The multi-replica host logic of bench.py on CPU: two gloo ranks on
127.0.0.1 check the max-over-ranks reduction of the timed region, the
barrier, the whole-job rate (units of all ranks over the slowest rank's
time), and that the reference arm runs on rank 0 only (other ranks return at
once, without work)."""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import datetime, sys
sys.path.insert(0, ROOT_DIR)
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
bench._DIST["on"] = True
r, w = dist.get_rank(), dist.get_world_size()
m = bench._max_over_ranks(1.5 + r)
assert m == 1.5 + (w - 1), m
bench._barrier()
assert bench.whole_job_rate(1, w, 100, 2000.0) == w * 100 / 2.0
if r != 0:
    sys.argv = ["bench.py", "--impl", "reference"]
    assert bench.main() == 0
dist.barrier()
dist.destroy_process_group()
print("rank", r, "ok", flush=True)
"""


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_bench_host_logic():
    port = _free_port()
    code = WORKER.replace("ROOT_DIR", repr(ROOT))
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT))
    outs = []
    for p in procs:
        try:
            outs.append(p.communicate(timeout=180)[0].decode())
        except subprocess.TimeoutExpired:
            p.kill()
            outs.append(p.communicate()[0].decode())
    for r, (p, o) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, o
        assert f"rank {r} ok" in o, o
