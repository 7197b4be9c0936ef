"""The one-rank-per-GPU driver (shard.DistributedRank) on a real GPU at world
size 1: the IPC-shared workspace and its rendezvous (handle export and the
object all-gather), the peer pointer tables, the NCCL all-gather of the counts and the
stream-ordered NCCL barriers all run for real, one rank holding every expert.
Each case runs in a child process of its own (one NCCL job each) and checks
every layout array, receive row and output token against the CPU oracle.

The bench's per-GPU path (bench.py --one-rank-per-gpu) runs the same driver
at world size 1 and prints its line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch

from conftest import ROOT

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env():
    env = dict(os.environ)
    env["NCCL_NVLS_ENABLE"] = "0"  # plain peer memory; no NVLink multicast objects
    env.pop("WORLD_SIZE", None)
    env.pop("RANK", None)
    env.pop("LOCAL_RANK", None)
    return env


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("name", ["prefill_r1", "skewed_r1"])
def test_distributed_rank_world1_against_oracle(cuda, name):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "dist_rank_child.py"), name,
                        str(_free_port())], capture_output=True, text=True, timeout=600, env=_env())
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert f"OK {name}" in r.stdout


def test_bench_one_rank_per_gpu_world1(cuda):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--one-rank-per-gpu", "--tokens", "1024",
                        "--steps", "3", "--warmup", "3", "--no-cpu-baseline"],
                       capture_output=True, text=True, timeout=600, env=_env())
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["n_gpus"] == 1 and line["config"]["ep_ranks"] == 1 and line["value"] > 0
    assert line["output_check"]["passed"] is True
    assert line["nccl_alltoallv"]["bytes_moved"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["gpu_launches"] == 4 * 3
    assert line["rows_to_other_gpus_per_rank"] == 0  # one rank: every row stays on this GPU


def test_ipc_peer_memory_two_processes_one_gpu(cuda):
    """The IPC mapping DistributedRank uses between GPUs, exercised between two
    processes that share this GPU: each exports its workspace (an interior
    view of an allocation), imports the other's, and reads its bytes."""
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, os.path.join(ROOT, "tests", "dist_rank_child.py"), "ipc", str(r), "2",
                               str(port)], stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, env=_env())
             for r in range(2)]
    outs = [p.communicate(timeout=300) for p in procs]
    for r, (p, (out, err)) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, out[-2000:] + err[-3000:]
        assert f"IPC_OK {r}" in out
