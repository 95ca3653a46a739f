"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Multi-GPU runs shard independent batches over ranks (weak scaling, no
data-path collective).  What the ranks share is host logic: each rank's own
seeds and inputs, and the max-over-ranks reduction of the device time.  The
reference arm under torchrun runs on rank 0 alone and prints one line."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    from moe_expert_layer_renorm_b200 import inputs

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(1.5 + rank)
        w = inputs.WORKLOADS["tiny"]
        li = inputs.make_layer_inputs(inputs.custom_workload(w, seed=bench.rank_layer_seed(w, rank, 0)), 0)
        digest = torch.tensor([int(np.bitwise_xor.reduce(li.x_bits.view(np.uint16).astype(np.int64).ravel()))],
                              dtype=torch.int64)
        allx = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(allx, digest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "digests": [int(t.item()) for t in allx]}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_independent_inputs(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == 1.5 + (world - 1)          # every rank sees the slowest rank's time
    assert res[0]["digests"] == res[1]["digests"]
    assert len(set(res[0]["digests"])) == world        # each rank draws its own batch


def test_max_over_ranks_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25) == 3.25


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "1",
           "--cpu-sample-tokens", "2"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_kernel_source_hash_ignores_comments_only():
    """The traffic records are keyed by the kernels' code: a comment edit keeps
    the key, a code edit changes it."""
    sys.path.insert(0, ROOT)
    import bench
    src = "// header\nint f(int x) {  // trailing\n  /* block\n comment */ return x + 1;\n}\n\n"
    assert bench._code_only(src) == bench._code_only(src.replace("trailing", "other words"))
    assert bench._code_only(src) != bench._code_only(src.replace("x + 1", "x + 2"))
    assert "header" not in bench._code_only(src) and "block" not in bench._code_only(src)
    assert len(bench.kernel_source_hash()) == 16
