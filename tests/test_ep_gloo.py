"""The expert-parallel exchange on CPU: gloo ranks (2 and 3) move rows with the
library's plan (ft_ep_plan) and transport (DistExchange), and the oracle does
the arithmetic on each side.  Each rank's output must equal the oracle's
single-process layer over that rank's tokens: every row reached the owner of
its expert and came back to the row it left from.

The same exchange runs between GPUs over NCCL; this covers its host logic
(split sizes, maps, collective order) where no GPU is needed."""
import datetime
import os
import socket
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


def _experts(E, H, I, seed):
    from oracle import moe_layer as M
    from oracle import nvfp4
    from moe_expert_layer_renorm_b200 import inputs
    out = {}
    for e in range(E):
        mats = []
        for which, (N, K) in enumerate(((I, H), (I, H), (H, I))):
            c, s, g = nvfp4.pack(inputs.make_weight_fp32_host(N, K, seed, e, which))
            mats.append(M.Nvfp4Tensor(c, s, float(np.float32(g)), N, K))
        out[e] = M.Expert(*mats)
    return out


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _rank_main(rank, world, port, cfg):
    sys.path.insert(0, ROOT)
    from oracle import moe_layer as M
    from moe_expert_layer_renorm_b200 import inputs
    from moe_expert_layer_renorm_b200.ep import DistExchange, ExchangePlan, owned_experts

    E, k, H, I, Ts, seed = cfg
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        T = Ts[rank]
        experts = _experts(E, H, I, seed)
        x_bits = inputs.make_x_bits(T, H, seed + 17 * rank)
        logits = inputs.make_logits(T, E, k, 1.0, seed + 17 * rank)
        ids, w = M.route(logits, k)
        offsets, perm_src, pair_to_row = M.permute(ids, E)

        ex = DistExchange()
        assert (ex.world_size, ex.rank) == (world, rank)
        plan = ExchangePlan(ex.gather_offsets(torch.from_numpy(offsets)), world, E, rank)
        n = plan.n_recv
        x_send = _bf16(x_bits[perm_src // k].reshape(T * k, H))
        x_recv = torch.empty((n, H), dtype=torch.bfloat16)
        ex.rows(x_recv, x_send, plan.recv_rows, plan.send_rows)

        xr = M.bf16_bits_to_f64(x_recv.view(torch.int16).numpy().view(np.uint16))
        out_local = np.zeros((n, H))
        mine = owned_experts(E, world, rank)
        for j, e in enumerate(mine):
            rows = np.arange(plan.local_offsets[j], plan.local_offsets[j + 1])
            if rows.size:
                out_local[rows] = M.expert_ffn(xr[plan.perm_src_local[rows]], experts[e])
        out_send = torch.from_numpy(out_local[plan.ret_idx[:n]])
        out_perm = torch.empty((T * k, H), dtype=torch.float64)
        ex.rows(out_perm, out_send, plan.send_rows, plan.recv_rows)

        op = out_perm.numpy()
        y = np.zeros((T, H))
        for t in range(T):
            for j in range(k):
                y[t] += w[t, j] * op[pair_to_row[t * k + j]]
        ref = M.moe_layer(x_bits, logits, k, experts).y
        err = float(np.max(np.abs(y - ref))) if T else 0.0
        assert err <= 1e-12 * (1.0 + float(np.max(np.abs(ref), initial=0.0))), err
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cfg", [
    (2, (8, 2, 256, 256, (12, 7), 4242)),
    (3, (12, 3, 256, 256, (9, 0, 5), 4343)),     # one rank without tokens still serves its experts
])
def test_gloo_ranks_exchange_rows_to_owners_and_back(world, cfg):
    mp.start_processes(_rank_main, args=(world, _free_port(), cfg), nprocs=world, join=True,
                       start_method="spawn")


def _leaver_main(rank, world, port, out_dir):
    """Rank 1 leaves between steps; rank 0's next collective fails within the
    process group's timeout instead of waiting for good."""
    sys.path.insert(0, ROOT)
    from moe_expert_layer_renorm_b200.ep import DistExchange
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    ex = DistExchange()
    ex.gather_offsets(torch.zeros(5, dtype=torch.int32))     # one step's first collective, together
    if rank == 1:
        os._exit(0)                                           # leaves without a word
    try:
        ex.rows(torch.empty((0, 4)), torch.empty((0, 4)), [0, 0], [0, 0])
        ex.gather_offsets(torch.zeros(5, dtype=torch.int32))
        outcome = "no error"
    except RuntimeError as e:
        outcome = "error: " + str(e).splitlines()[0][:200]
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(outcome)
    os._exit(0)


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error(tmp_path):
    ctx = mp.start_processes(_leaver_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=False,
                             start_method="spawn")
    while not ctx.join(timeout=120):
        pass
    out = (tmp_path / "rank0.txt").read_text()
    assert out.startswith("error"), out
