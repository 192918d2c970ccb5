"""Multi-rank host logic on CPU: two gloo ranks launched by torchrun, the way
the benchmark is launched on GPUs (127.0.0.1 rendezvous).  Channels are
sharded across ranks with no data-path exchange; these tests check the shard
recipe, the output gather, the max-over-ranks timing and that a rank which
leaves makes its peer fail instead of wait."""
import json
import os
import socket
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(mode, tmp_path, nproc=2, timeout=180):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(HERE, "multirank_worker.py"), mode, str(tmp_path)]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=timeout)
    out = {}
    for r in range(nproc):
        f = tmp_path / f"rank{r}.json"
        if f.exists():
            out[r] = json.loads(f.read_text())
    return p, out


def test_two_rank_channel_shards_match_whole_problem(tmp_path):
    p, out = _torchrun("shard", tmp_path)
    assert p.returncode == 0, p.stderr[-3000:]
    r0, r1 = out[0], out[1]
    assert r0["world"] == r1["world"] == 2
    assert r0["tmax"] == r1["tmax"] == 2.5                 # max of 1.5 and 2.5
    assert r0["channels"] == [0, 3] and r1["channels"] == [3, 6]
    assert r0["throughput"] == 2 * (2 * 3 * 256) / 2e-3    # all ranks' elements / slowest time
    assert r0["shards_differ"] and r0["shard0_is_workload"]
    assert r0["max_err"] <= 1e-12 * max(1.0, r0["scale"])


def test_peer_that_leaves_fails_the_barrier(tmp_path):
    p, out = _torchrun("peer_exit", tmp_path, timeout=240)
    assert 0 in out and 1 in out, p.stderr[-3000:]
    assert out[0]["error"] is not None
