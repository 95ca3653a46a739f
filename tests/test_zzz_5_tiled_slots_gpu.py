"""Stage-tiled expert slots (ft_tiled_slot_layout_init): the same bytes as the
row-major slots, arranged so that each weight box the GEMMs load is one
contiguous block.  The packed tensors read back identical to row-major
packing, and the layer gives bit-identical outputs on both layouts (the
kernels only load from other addresses), and matches the oracle.

Collected last: the layout is new and has not yet run on a B200."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from moe_expert_layer_renorm_b200.layer import ExpertPool
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS


@pytest.mark.parametrize("H,I", [(256, 512), (2880, 2880), (2048, 768)])
@pytest.mark.parametrize("fmt", [_lib.FT_SCALE_NVFP4, _lib.FT_SCALE_MXFP4])
def test_tiled_slots_hold_the_row_major_bytes(cuda_device, H, I, fmt):
    rows = ExpertPool(H, I, 2, fmt=fmt)
    tiled = ExpertPool(H, I, 2, fmt=fmt, tiled=True)
    tiled.buf.fill_(0xAB)          # the pack writes every byte of the tensors' regions, padding included
    for mat in range(3):
        N, K = rows.shape(mat)
        wt = inputs.make_weight_fp32_torch(N, K, 77, 5, mat, "cuda")
        rows.pack_into(1, mat, wt)
        tiled.pack_into(1, mat, wt)
    torch.cuda.synchronize()
    assert _lib.device_status(clear=True) == 0
    assert np.array_equal(tiled.export_slot(1), rows.export_slot(1))
    # the padding of the last stage (K not a multiple of 256) holds zero codes
    L = tiled.layout
    s = tiled.slot_view(1).cpu().numpy()
    for mat in range(3):
        N, K = tiled.shape(mat)
        S = (K + 255) // 256
        codes = s[L.codes_off[mat]:L.codes_off[mat] + S * N * 128].reshape(S, N, 128)
        assert not codes[S - 1, :, (K // 2) - 128 * (S - 1):].any()


@pytest.mark.parametrize("name", ["tiny", "decode_T8", "decode_T64", "slots512_T1"])
def test_layer_on_tiled_slots_is_bit_identical(cuda_device, name):
    w = W[name]
    li = inputs.make_layer_inputs(w)
    pool_r, st = G.build_pool(w)
    pool_t, st_t = G.build_pool(w, tiled=True)
    assert np.array_equal(st, st_t)
    a = G.run_gpu(w, pool=pool_r, slot_table=st, li=li)
    b = G.run_gpu(w, pool=pool_t, slot_table=st_t, li=li)
    assert np.array_equal(a.y, b.y)
    G.check_output(b, w.k)


def test_prefill_on_tiled_slots(cuda_device):
    # 1024 tokens x top-4 of 32 wide experts (K = 2880: a partial last stage): the tcgen05 kernel
    w = inputs.custom_workload(W["wide_T8192"], T=1024)
    li = inputs.make_layer_inputs(w)
    pool_r, st = G.build_pool(w)
    pool_t, _ = G.build_pool(w, tiled=True)
    a = G.run_gpu(w, pool=pool_r, slot_table=st, li=li)
    b = G.run_gpu(w, pool=pool_t, slot_table=st, li=li)
    assert np.array_equal(a.y, b.y)
    G.check_output(b, w.k, tokens=np.arange(0, 1024, 37))


def test_mxfp4_layer_on_tiled_slots(cuda_device):
    w = W["decode_T64"]
    li = inputs.make_layer_inputs(w)
    pool_r, st = G.build_pool(w, fmt=_lib.FT_SCALE_MXFP4)
    pool_t, _ = G.build_pool(w, fmt=_lib.FT_SCALE_MXFP4, tiled=True)
    a = G.run_gpu(w, pool=pool_r, slot_table=st, li=li)
    b = G.run_gpu(w, pool=pool_t, slot_table=st, li=li)
    assert np.array_equal(a.y, b.y)


def test_pack_slot_row_major_equals_the_plain_pack(cuda_device):
    # ft_pack_slot on a row-major layout places the bytes as ft_nvfp4_pack does
    H, I = 2880, 2880
    a = ExpertPool(H, I, 1)
    b = ExpertPool(H, I, 1)
    for mat in range(3):
        N, K = a.shape(mat)
        wt = inputs.make_weight_fp32_torch(N, K, 78, 2, mat, "cuda")
        a.pack_into(0, mat, wt)
        _lib.pack_slot(wt.data_ptr(), mat, b.layout, b.ptr, b._pack_ws.data_ptr(),
                       torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(a.buf, b.buf)
