"""ft_moe_permute_noalloc against ft_moe_permute (with its workspace): the
same rows, bit for bit, on two calls in a row, on inputs that fit the
library's fixed scratch, and a clear rejection of inputs that do not.

Named to be collected last, so that it also runs after every other test
has used the library in the same process."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _ids(T, E, k, seed):
    g = np.random.default_rng(seed)
    return np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def _outputs(P, E):
    return (torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
            torch.full((max(P, 1),), -1, dtype=torch.int32, device="cuda"),
            torch.full((max(P, 1),), -1, dtype=torch.int32, device="cuda"))


# (T, E, k): one chunk (no scratch used), several chunks with a ragged tail,
# many experts, and the largest input the scratch takes (64 chunks x 1024).
@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (4096, 128, 8), (1000, 100, 3), (2048, 512, 10),
                                   (65536, 1024, 1)])
def test_noalloc_matches_permute(cuda_device, T, E, k):
    P = T * k
    d_ids = torch.from_numpy(_ids(T, E, k, seed=T * 31 + E)).cuda()
    o_ref, a_ref, b_ref = _outputs(P, E)
    wsb = _lib.permute_workspace_size(T, k, E)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    _lib.permute(d_ids.data_ptr(), T, k, E, o_ref.data_ptr(), a_ref.data_ptr(), b_ref.data_ptr(),
                 ws.data_ptr(), wsb, _stream())
    for _ in range(2):   # two calls in a row: the scratch holds nothing over
        o, a, b = _outputs(P, E)
        _lib.permute_noalloc(d_ids.data_ptr(), T, k, E, o.data_ptr(), a.data_ptr(), b.data_ptr(), _stream())
        torch.cuda.synchronize()
        assert _lib.device_status(clear=True) == 0
        assert torch.equal(o, o_ref)
        assert torch.equal(a, a_ref)
        assert torch.equal(b, b_ref)


def test_noalloc_empty_batch(cuda_device):
    o = torch.full((9,), -1, dtype=torch.int32, device="cuda")
    _lib.permute_noalloc(0, 0, 2, 8, o.data_ptr(), 0, 0, _stream())
    torch.cuda.synchronize()
    assert torch.equal(o.cpu(), torch.zeros(9, dtype=torch.int32))


def test_noalloc_rejects_input_beyond_scratch(cuda_device):
    T, E, k = 65537, 1024, 1           # 65 chunks x 1024 experts > 65536 counts
    d_ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    o, a, b = _outputs(T * k, E)
    with pytest.raises(_lib.FtError, match="scratch"):
        _lib.permute_noalloc(d_ids.data_ptr(), T, k, E, o.data_ptr(), a.data_ptr(), b.data_ptr(), _stream())
    torch.cuda.synchronize()
    assert int(o[0]) == -1             # nothing was launched
