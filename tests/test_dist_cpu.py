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


EP_WORKER = r"""
import datetime, sys
sys.path.insert(0, ROOT_DIR)
import numpy as np
import torch
import torch.distributed as dist
import oracle
from nvfp4_weight_only_flint_b200 import ep
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
r, R = dist.get_rank(), dist.get_world_size()
ex = ep.AllToAll()

# 1. uneven splits, zero splits included: rank r sends (r + 1) * (dst + 1) % 3 rows to dst
sc = [((r + 1) * (dst + 1)) % 3 for dst in range(R)]
send = torch.cat([torch.full((n, 2), float(100 * r + dst)) for dst, n in enumerate(sc)])
rc = ex.counts(torch.tensor(sc, dtype=torch.int32)).tolist()
assert rc == [((src + 1) * (r + 1)) % 3 for src in range(R)], rc
recv = ex.rows(send, sc, rc, torch.empty((sum(rc), 2)))
want = torch.cat([torch.full((n, 2), float(100 * src + r)) for src, n in enumerate(rc)])
assert torch.equal(recv, want)


# 2. the layer step's orchestration (counts, three row exchanges, the reverse
# exchange, the combine) with host stand-ins for the kernels: dispatch by the
# oracle's plan, experts y = gate * x, combine = sum of a token's rows.
class HostLayer(ep.ExpertParallelLayer):
    def __init__(self, rank, n_ranks, T, k, E, d):
        self.rank, self.R, self.T, self.k, self.E, self.d = rank, n_ranks, T, k, E, d
        self.slots = k + 1
        P = T * self.slots
        self.max_recv = n_ranks * T * k + T
        self.send_x = torch.zeros((P, d)); self.send_ids = torch.zeros(P, dtype=torch.int32)
        self.send_gates = torch.zeros(P); self.recv_x = torch.zeros((self.max_recv, d))
        self.recv_ids = torch.zeros(self.max_recv, dtype=torch.int32); self.recv_gates = torch.zeros(self.max_recv)
        self.y = torch.zeros((self.max_recv, d)); self.y_back = torch.zeros((P, d))

    def send(self, x, T):
        rng = np.random.default_rng(self.rank)
        self.ids = np.array([rng.choice(self.E, self.k, replace=False) for _ in range(T)], np.int32)
        self.gates = rng.random((T, self.k)).astype(np.float32)
        p = oracle.ep_plan(self.ids, self.gates, S=1, E=self.E, R=self.R, rank=self.rank)
        n = int(p["counts"].sum())
        self.send_x[:n] = x[torch.from_numpy(p["send_token"]).long()]
        self.send_ids[:n] = torch.from_numpy(p["send_ids"])
        self.send_gates[:n] = torch.from_numpy(p["send_gates"])
        self.pair_pos = p["pair_pos"]
        return torch.from_numpy(p["counts"])

    def experts(self, n_recv):
        self.y[:n_recv] = self.recv_x[:n_recv] * self.recv_gates[:n_recv, None]
        # ids arrived with their rows: local ids of this rank's experts or the shared one
        assert n_recv == 0 or int(self.recv_ids[:n_recv].max()) <= self.E // self.R
        return self.y[:n_recv]

    def finish(self, T, out, residual=None):
        for t in range(T):
            out[t] = sum(self.y_back[int(q)] for q in self.pair_pos[t] if q >= 0)
        return out


T, k, E, d = 5, 3, 8, 4
layer = HostLayer(r, R, T, k, E, d)
x = torch.arange(T * d, dtype=torch.float32).reshape(T, d) + 1000 * r
out = layer.forward(x, T, torch.zeros((T, d)), exchange=ex)
want = x * (torch.from_numpy(layer.gates).sum(dim=1, keepdim=True) + 1.0)
assert torch.allclose(out, want, rtol=1e-6, atol=1e-4), (out, want)
dist.barrier()
dist.destroy_process_group()
print("rank", r, "ok", flush=True)
"""


def test_two_gloo_ranks_expert_parallel_exchange():
    """The expert-parallel layer's exchange on two gloo ranks: uneven and
    empty all-to-all splits, and a whole layer step's orchestration with the
    kernels replaced by host stand-ins -- every row comes back to the pair it
    left from."""
    port = _free_port()
    code = EP_WORKER.replace("ROOT_DIR", repr(ROOT))
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
