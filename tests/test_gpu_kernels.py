"""Kernel-level parity with the oracle, through the C ABI: route, permute and
pack bit-exact; combine to fp32 rounding."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from moe_expert_layer_renorm_b200.layer import ExpertPool, MoELayer
from oracle import moe_layer as M
from oracle import nvfp4

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("T,E,k,mode,sigma", [
    (16, 8, 2, 0, 1.0), (64, 128, 8, 0, 1.0), (300, 512, 10, 0, 1.0), (333, 32, 4, 1, 1.5),
    (50, 1024, 32, 0, 1.0), (40, 6, 6, 1, 1.0), (7, 1, 1, 0, 1.0), (129, 33, 3, 1, 1.0),
])
def test_route_bit_exact(cuda_device, T, E, k, mode, sigma):
    lg = inputs.make_logits(T, E, k, sigma, seed=T * 7 + E)
    ids_ref, w_ref = M.route(lg, k)
    d_lg = torch.from_numpy(lg).cuda()
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    _lib.route(d_lg.data_ptr(), T, E, k, mode, ids.data_ptr(), w.data_ptr(), _stream())
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.allclose(w.cpu().numpy(), w_ref, rtol=2e-6, atol=1e-7)
    assert np.allclose(w.cpu().numpy().sum(axis=1), 1.0, atol=2e-6)


def test_route_ties_go_to_lower_id(cuda_device):
    lg = np.zeros((3, 40), np.float32)
    lg[0, [5, 9, 33]] = 2.0                  # three equal maxima
    lg[1, :] = 1.0                           # everything equal
    lg[2, [39, 0]] = -0.0                    # -0 == +0
    lg[2, 1:39] = -1.0
    ids_ref, _ = M.route(lg, 3)
    d = torch.from_numpy(lg).cuda()
    ids = torch.empty((3, 3), dtype=torch.int32, device="cuda")
    w = torch.empty((3, 3), dtype=torch.float32, device="cuda")
    _lib.route(d.data_ptr(), 3, 40, 3, 0, ids.data_ptr(), w.data_ptr(), _stream())
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert ids.cpu().numpy()[0].tolist() == [5, 9, 33]
    assert ids.cpu().numpy()[1].tolist() == [0, 1, 2]


@pytest.mark.parametrize("T,E,k", [(1, 128, 8), (16, 8, 2), (128, 128, 8), (129, 8, 8), (4096, 128, 8),
                                   (8192, 512, 10), (1000, 1024, 1), (3000, 3, 2)])
def test_permute_bit_exact(cuda_device, T, E, k):
    g = np.random.default_rng(T + E + k)
    if T == 4096:   # skewed: a few experts take most pairs
        ids = np.stack([g.choice(E, size=k, replace=False, p=np.r_[[0.3] * 2, [0.4 / (E - 2)] * (E - 2)])
                        for _ in range(T)]).astype(np.int32)
    else:
        ids = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off, ps, p2r = M.permute(ids, E)
    d_ids = torch.from_numpy(ids).cuda()
    P = T * k
    o = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    a = torch.empty(P, dtype=torch.int32, device="cuda")
    b = torch.empty(P, dtype=torch.int32, device="cuda")
    wsb = _lib.permute_workspace_size(T, k, E)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    for _ in range(2):   # deterministic: same bytes on a rerun
        _lib.permute(d_ids.data_ptr(), T, k, E, o.data_ptr(), a.data_ptr(), b.data_ptr(), ws.data_ptr(), wsb,
                     _stream())
        torch.cuda.synchronize()
        assert np.array_equal(o.cpu().numpy(), off)
        assert np.array_equal(a.cpu().numpy(), ps)
        assert np.array_equal(b.cpu().numpy(), p2r)


def test_permute_bad_id_in_a_large_batch_sets_status(cuda_device):
    # several chunks: the out-of-range id sits in the second chunk, in a warp's run
    # that is not the first; the bad pair gets no row and the call records the status
    g = np.random.default_rng(77)
    T, k, E = 2000, 2, 16
    ids = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    ids[700, 1] = 99
    d_ids = torch.from_numpy(ids).cuda()
    P = T * k
    o = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    a = torch.full((P,), -7, dtype=torch.int32, device="cuda")
    b = torch.full((P,), -7, dtype=torch.int32, device="cuda")
    wsb = _lib.permute_workspace_size(T, k, E)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    _lib.device_status(clear=True)
    _lib.permute(d_ids.data_ptr(), T, k, E, o.data_ptr(), a.data_ptr(), b.data_ptr(), ws.data_ptr(), wsb,
                 _stream())
    torch.cuda.synchronize()
    assert _lib.device_status(clear=True) == _lib.FT_DEV_BAD_INDEX
    assert int(b.cpu().numpy()[700 * k + 1]) == -7
    assert int(o.cpu().numpy()[E]) == P - 1


def test_permute_bad_id_sets_status(cuda_device):
    _lib.device_status(clear=True)
    ids = torch.tensor([[0, 9]], dtype=torch.int32, device="cuda")
    o = torch.empty(5, dtype=torch.int32, device="cuda")
    a = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    b = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    _lib.permute(ids.data_ptr(), 1, 2, 4, o.data_ptr(), a.data_ptr(), b.data_ptr(), 0, 0, _stream())
    assert _lib.device_status(clear=True) == _lib.FT_DEV_BAD_INDEX


def _pack_gpu(w: np.ndarray, ld: int):
    N, K = w.shape
    d = torch.from_numpy(w).cuda()
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.full((N, ld), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    _lib.nvfp4_pack(d.data_ptr(), N, K, codes.data_ptr(), scales.data_ptr(), ld, g.data_ptr(), ws.data_ptr(),
                    _stream())
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), np.float32(g.cpu().numpy()[0])


@pytest.mark.parametrize("N,K,ld", [(64, 256, 16), (17, 2880, 192), (512, 2048, 128), (3, 16, 16)])
def test_pack_bit_exact(cuda_device, N, K, ld):
    g = np.random.default_rng(N * K)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :16] = 0.0                                   # zero block
    w[1 % N, 16 % K:32 % K or 16] *= 1e-7             # scale underflows to 0
    w[2 % N, 5] = 3.0                                 # outlier sets the tensor amax
    c_ref, s_ref, g_ref = nvfp4.pack(w, ld_scale=ld)
    c, s, gg = _pack_gpu(w, ld)
    assert gg == g_ref
    assert np.array_equal(s, s_ref)
    assert np.array_equal(c, c_ref)


def test_pack_hand_worked_example(cuda_device):
    from tests.conftest import golden_lines
    w = np.zeros((2, 32), np.float32)
    for row in golden_lines("pack_worked.txt"):
        if row[0] == "w":
            w[int(row[1])] = [float(x) for x in row[2:]]
    c_ref, s_ref, g_ref = nvfp4.pack(w, ld_scale=16)
    c, s, gg = _pack_gpu(w, 16)
    assert gg == g_ref and np.array_equal(s, s_ref) and np.array_equal(c, c_ref)


def test_pack_ties_and_saturation(cuda_device):
    # every E2M1 midpoint, exactly representable: amax = 6 * 448 * 2^-12 gives step 448 * 2^-12
    step = np.float32(448 * 2.0 ** -12)
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -6.0],
                 np.float32)
    w = (v * step).astype(np.float32)[None, :]
    c_ref, s_ref, g_ref = nvfp4.pack(w, ld_scale=16)
    c, s, gg = _pack_gpu(w, 16)
    assert np.array_equal(c, c_ref) and np.array_equal(s, s_ref) and gg == g_ref


def test_combine_matches_definition(cuda_device):
    T, k, H = 37, 4, 512
    g = np.random.default_rng(1)
    P = T * k
    out_perm = torch.randn((P, H), dtype=torch.float32)
    p2r = torch.from_numpy(g.permutation(P).astype(np.int32))
    w = torch.from_numpy(g.random((T, k)).astype(np.float32))
    y = torch.empty((T, H), dtype=torch.float32, device="cuda")
    d_op, d_p2r, d_w = out_perm.cuda(), p2r.cuda(), w.cuda()   # keep the device copies alive
    _lib.combine(d_op.data_ptr(), d_p2r.data_ptr(), d_w.data_ptr(), T, k, H, y.data_ptr(), _stream())
    torch.cuda.synchronize()
    o = out_perm.double().numpy()[p2r.numpy()].reshape(T, k, H)
    ref = (o * w.double().numpy()[:, :, None]).sum(axis=1)
    got = y.double().cpu().numpy()
    # fp32 fused multiply-adds in the order j = 0..k-1
    assert np.all(np.abs(got - ref) <= np.abs(o * w.double().numpy()[:, :, None]).sum(axis=1) * 2.0 ** -22 + 1e-30)
