"""MXFP4 experts on the GPU, against the oracle: the pack kernel bit for bit,
and the whole layer (decode and prefill kernels) within the layer tolerance."""
import math

import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from oracle import cpp
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _pack_gpu(w: np.ndarray, ld: int):
    N, K = w.shape
    d = torch.from_numpy(w).cuda()
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.full((N, ld), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    _lib.mxfp4_pack(d.data_ptr(), N, K, codes.data_ptr(), scales.data_ptr(), ld, g.data_ptr(), ws.data_ptr(),
                    _stream())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), float(g.cpu().numpy()[0])


@pytest.mark.parametrize("N,K,ld", [(64, 256, 16), (17, 2880, 192), (512, 2048, 128), (3, 32, 16)])
def test_mxfp4_pack_bit_exact(cuda_device, N, K, ld):
    g = np.random.default_rng(N * K + 1)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :32] = 0.0                       # an all-zero block
    w[(2 % N), 5] = 3.0                   # outlier sets the tensor's largest exponent
    w[(1 % N), 32 % K] = -0.0
    c_ref, s_ref = cpp.pack_mxfp4(w)
    c, s, gg = _pack_gpu(w, ld)
    assert np.array_equal(c, c_ref)
    assert np.array_equal(s[:, 0:K // 16:2], s_ref) and np.array_equal(s[:, 1:K // 16:2], s_ref)
    assert not s[:, K // 16:].any()       # row padding
    amax = float(np.abs(w).max())
    x_max = max(-127, min(127, math.frexp(amax)[1] - 1 - 2))
    assert gg == math.ldexp(1.0, x_max - 13)
    assert _lib.device_status(clear=True) == 0


@pytest.mark.parametrize("name", ["tiny", "decode_T8", "decode_T64"])
def test_mxfp4_layer_parity(cuda_device, name):
    w = W[name]
    pool, st = G.build_pool(w, fmt=_lib.FT_SCALE_MXFP4)
    run = G.run_gpu(w, pool=pool, slot_table=st)
    G.check_routing(run, w.k)
    G.check_output(run, w.k)


def test_mxfp4_prefill_layer_parity_sampled(cuda_device):
    # 1024 tokens x top-4 of 32 experts: ~128 rows per expert, the tcgen05 prefill kernel
    w = inputs.custom_workload(W["wide_T8192"], T=1024)
    pool, st = G.build_pool(w, fmt=_lib.FT_SCALE_MXFP4)
    run = G.run_gpu(w, pool=pool, slot_table=st)
    G.check_output(run, w.k, tokens=np.arange(0, 1024, 37))


def test_mxfp4_large_groups_layer_parity(cuda_device):
    # 600 tokens over 4 experts at top-2 (~300 rows per expert): the gate/up GEMM's large-group shape
    # (A operand in shared memory), with the MXFP4 scale decode, K = 320 (not a multiple of 256)
    w = inputs.custom_workload(W["tiny"], H=320, I=448, E=4, k=2, T=600, seed=6161)
    pool, st = G.build_pool(w, fmt=_lib.FT_SCALE_MXFP4)
    run = G.run_gpu(w, pool=pool, slot_table=st)
    G.check_routing(run, w.k)
    G.check_output(run, w.k)

