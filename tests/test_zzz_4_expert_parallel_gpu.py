"""Expert parallelism on one GPU, against the oracle.

* ft_gather_rows bit for bit against indexing, and its bad-index status.
* G ranks emulated as G host threads sharing the GPU: each thread runs
  ExpertParallelMoE.forward (the product path: route, permute, gather, plan,
  FFN over its own experts, gather, combine) with a transport that hands the
  rows over in device memory between the threads.  No kernel waits on another
  thread's kernels: the hand-over is a host barrier after a device
  synchronisation, so the threads' launches never depend on one another on
  the device.  Each rank's y must match the oracle's layer over its tokens.
* One rank over NCCL (a process group of size 1): the same path through
  torch.distributed.

Named to be collected last: it starts host threads and a process group in
the test process."""
import datetime
import socket
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist

from moe_expert_layer_renorm_b200 import _lib, inputs
from moe_expert_layer_renorm_b200.ep import DistExchange, ExpertParallelMoE, owned_experts
from moe_expert_layer_renorm_b200.layer import ExpertPool
from oracle import cpp
from oracle import moe_layer as M

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("row_bytes,div", [(2 * 2048, 8), (4 * 2880, 1), (16, 3)])
def test_gather_rows_bit_exact(cuda_device, row_bytes, div):
    g = np.random.default_rng(row_bytes + div)
    n_src, n = 97, 613
    src = torch.from_numpy(g.integers(0, 256, size=(n_src, row_bytes), dtype=np.uint8)).cuda()
    idx_np = g.integers(0, n_src * div, size=n).astype(np.int32)
    idx = torch.from_numpy(idx_np).cuda()
    dst = torch.full((n, row_bytes), 0xAB, dtype=torch.uint8, device="cuda")
    _lib.device_status(clear=True)
    _lib.gather_rows(src.data_ptr(), n_src, row_bytes, idx.data_ptr(), div, n, dst.data_ptr(), _stream())
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), src.cpu()[torch.from_numpy(idx_np // div).long()])
    assert _lib.device_status(clear=True) == 0


def test_gather_rows_bad_index_gives_zero_row_and_status(cuda_device):
    src = torch.ones((4, 64), dtype=torch.uint8, device="cuda")
    idx = torch.tensor([0, 4, -1, 3], dtype=torch.int32, device="cuda")
    dst = torch.full((4, 64), 7, dtype=torch.uint8, device="cuda")
    _lib.device_status(clear=True)
    _lib.gather_rows(src.data_ptr(), 4, 64, idx.data_ptr(), 1, 4, dst.data_ptr(), _stream())
    torch.cuda.synchronize()
    assert _lib.device_status(clear=True) == _lib.FT_DEV_BAD_INDEX
    d = dst.cpu()
    assert d[0].eq(1).all() and d[3].eq(1).all() and d[1].eq(0).all() and d[2].eq(0).all()


class _Shared:
    def __init__(self, G):
        self.G = G
        self.barrier = threading.Barrier(G, timeout=120)
        self.slot = [None] * G


class ThreadExchange:
    """Transport between threads of one process on one GPU (test only)."""

    def __init__(self, shared: _Shared, rank: int):
        self.sh, self.rank, self.world_size = shared, rank, shared.G

    def gather_offsets(self, offsets):
        self.sh.slot[self.rank] = offsets.cpu().numpy().astype(np.int32)
        self.sh.barrier.wait()
        out = np.stack(self.sh.slot)
        self.sh.barrier.wait()
        return out

    def rows(self, out, inp, out_rows, in_rows):
        torch.cuda.synchronize()
        self.sh.slot[self.rank] = (inp, [int(v) for v in in_rows])
        self.sh.barrier.wait()
        at = 0
        for s in range(self.world_size):
            src, splits = self.sh.slot[s]
            start = sum(splits[:self.rank])
            n = splits[self.rank]
            assert n == int(out_rows[s])
            if n:
                out[at:at + n].copy_(src[start:start + n])
            at += n
        assert at == out.shape[0]
        torch.cuda.synchronize()
        self.sh.barrier.wait()


def _rank_pool(w, G, rank):
    """This rank's experts packed on the device into slots 0 .. E/G - 1."""
    mine = owned_experts(w.E, G, rank)
    pool = ExpertPool(w.H, w.I, len(mine))
    for j, e in enumerate(mine):
        for mat in range(3):
            N, K = pool.shape(mat)
            pool.pack_into(j, mat, inputs.make_weight_fp32_torch(N, K, w.seed, e, mat, "cuda"))
    torch.cuda.synchronize()
    return pool


def _oracle_y(w, pools, G, x_bits, logits, tok):
    """The C++ oracle's layer for tokens `tok`, experts read from the ranks'
    pools (the packed bytes the GPU used)."""
    ids, _ = M.route(logits, w.k)
    need = sorted(set(int(e) for e in ids[tok].reshape(-1)))
    L = pools[0].rows_layout        # slots read back row-major
    nb = int(L.slot_bytes)
    buf = np.zeros(max(1, len(need)) * nb, np.uint8)
    table = np.full(w.E, -1, np.int32)
    El = w.E // G
    for i, e in enumerate(need):
        buf[i * nb:(i + 1) * nb] = pools[e // El].export_slot(e % El)
        table[e] = i
    return cpp.moe_layer(x_bits, logits, w.k, table, buf, nb, list(L.codes_off), list(L.scales_off),
                         list(L.global_off), list(L.ld_scale), w.H, w.I, tokens=tok)


CASES = {
    # decode-sized: 8 tokens per rank, 128 experts over 4 ranks (weight-streaming kernel on each)
    "decode_4ranks": (inputs.WORKLOADS["decode_T8"], 4, (8, 8, 3, 8), 1),
    # prefill-sized: 512 and 300 tokens per rank, 32 wide experts over 2 ranks (tcgen05 kernel)
    "wide_2ranks": (inputs.WORKLOADS["wide_T8192"], 2, (512, 300), 29),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_emulated_ranks_match_oracle(cuda_device, case):
    w, G, Ts, stride = CASES[case]
    pools = [_rank_pool(w, G, r) for r in range(G)]
    ins = [inputs.make_layer_inputs(inputs.custom_workload(w, seed=w.seed + 101 * r), T=Ts[r]) for r in range(G)]
    sh = _Shared(G)
    ys, errs = [None] * G, [None] * G
    _lib.device_status(clear=True)

    def run(r):
        try:
            ep = ExpertParallelMoE(Ts[r], w.E, w.k, w.H, w.I, exchange=ThreadExchange(sh, r), mode=w.route_mode)
            x = torch.from_numpy(ins[r].x_bits.view(np.int16)).view(torch.bfloat16).cuda()
            logits = torch.from_numpy(ins[r].logits).cuda()
            table = torch.arange(w.E // G, dtype=torch.int32, device="cuda")
            ep.layer.out_perm.fill_(float("nan"))
            y = ep.forward(x, logits, table, pools[r])
            torch.cuda.synchronize()
            ys[r] = y.cpu().numpy().astype(np.float64)
        except BaseException as e:          # surfaces in the main thread; the barrier breaks for the others
            errs[r] = e
            sh.barrier.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=600)
    assert not any(t.is_alive() for t in threads)
    for e in errs:
        if e is not None and not isinstance(e, threading.BrokenBarrierError):
            raise e
    assert all(e is None for e in errs), errs
    assert _lib.device_status(clear=True) == 0
    for r in range(G):
        tok = np.arange(0, Ts[r], stride)
        ref = _oracle_y(w, pools, G, ins[r].x_bits, ins[r].logits, tok)
        err = np.abs(ys[r][tok] - ref)
        tol = M.tolerance(ref)
        assert np.all(err <= tol), (r, float(err.max()), tol)


def test_one_rank_over_nccl(cuda_device):
    w = inputs.WORKLOADS["tiny"]
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        pool = _rank_pool(w, 1, 0)
        li = inputs.make_layer_inputs(w)
        ep = ExpertParallelMoE(w.T, w.E, w.k, w.H, w.I, exchange=DistExchange(), mode=w.route_mode)
        x = torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
        logits = torch.from_numpy(li.logits).cuda()
        table = torch.arange(w.E, dtype=torch.int32, device="cuda")
        _lib.device_status(clear=True)
        y = ep.forward(x, logits, table, pool)
        torch.cuda.synchronize()
        assert _lib.device_status(clear=True) == 0
        ref = _oracle_y(w, [pool], 1, li.x_bits, li.logits, np.arange(w.T))
        err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
        assert np.all(err <= M.tolerance(ref)), float(err.max())
        assert ep.plan.n_recv == w.T * w.k
    finally:
        dist.destroy_process_group()
