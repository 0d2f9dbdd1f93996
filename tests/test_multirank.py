"""Host logic of the multi-process bench on CPU: two gloo ranks, no GPU.

The decode path has no exchange between GPUs: each rank decodes its own batch (weak
scaling), and the ranks only meet to time the job, taking the slowest rank's time and
summing the bytes moved.  These tests run that logic in two processes over gloo, and the
reference arm under torchrun, where rank 0 alone prints the line.
"""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from top_sparse_decode_topk_b200 import workload as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], "cpu")
        sm = bench.sum_over_ranks([100.0 * (rank + 1), 1.0], "cpu")
        w = W.make_workload(W.CONFIGS["tiny"], seed=bench.rank_seed(rank))
        digest = int(np.bitwise_xor.reduce(w.q_bits.reshape(-1).astype(np.uint64)))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "sum": sm, "q_digest": digest}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_and_own_their_batches(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    for r in (r0, r1):
        assert r["max"] == [2.0, 10.0, 5.0]          # slowest rank per leg
        assert r["sum"] == [300.0, 2.0]              # bytes of the whole job
    assert r0["q_digest"] != r1["q_digest"]          # each rank decodes a different batch


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--config", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _cp_rank_main(rank: int, world: int, port: int, out_dir: str):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from top_sparse_decode_topk_b200 import context_parallel as CP
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # what a rank contributes to the candidate exchange: [T, Hq, k] indices and scores
        idx = torch.arange(12, dtype=torch.int32).reshape(2, 2, 3) + 100 * rank
        sc = torch.full((2, 2, 3), float(rank), dtype=torch.float32)
        gi, gs = CP.gather_rank_major(idx), CP.gather_rank_major(sc)
        with open(os.path.join(out_dir, f"cp{rank}.json"), "w") as f:
            json.dump({"shape": list(gi.shape), "idx": gi.tolist(), "sc": gs[:, 0, 0, 0].tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_context_parallel_exchange_is_rank_major(tmp_path):
    """The candidate and partial exchanges stack every rank's tensor in rank order, which the
    merge kernels rely on (rank r's token range precedes rank r + 1's)."""
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_cp_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "cp0.json"))
    r1 = json.load(open(tmp_path / "cp1.json"))
    assert r0 == r1
    assert r0["shape"] == [2, 2, 2, 3]
    assert r0["sc"] == [0.0, 1.0]
    assert r0["idx"][1][0][0] == [100, 101, 102]


def test_shard_lengths_cover_the_context():
    from top_sparse_decode_topk_b200 import context_parallel as CP
    for n, world in ((32768, 4), (20001, 3), (131072, 8), (100, 7)):
        S = CP.shard_length(n, world, 16)
        assert S % 16 == 0 and S * world >= n and S * (world - 1) < n + 16 * world
