"""rr_search_static: the pattern search for callers that cannot allocate.

Some callers have no way to give the library device memory: an operator
interface that passes only its input and output tensors, or a process whose
device memory is all owned by another allocator.  rr_search_static keeps the
search's scratch in a 32 MiB array inside the library instead of a caller
workspace.  Its masks must equal those of rr_search (which takes a workspace)
on the same inputs, on consecutive calls that reuse the shared array with
different shapes, and shapes that need more scratch must be rejected before
anything runs.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rr():
    from dynamic_block_sparse_rr_b200 import _build
    _build.build()
    import dynamic_block_sparse_rr_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def _dev(a):
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def _static_search(rr, qd, kd, B, S, tau):
    L, H, d = qd.shape
    Hkv = kd.shape[1]
    Nb = L // B
    count = torch.full((H, Nb), -7, dtype=torch.int32, device="cuda")
    idx = torch.full((H, Nb, Nb), -7, dtype=torch.int32, device="cuda")
    code = rr.lib().rr_search_static(qd.data_ptr(), kd.data_ptr(), L, H, Hkv, d, B, S, ctypes.c_float(tau),
                                     count.data_ptr(), idx.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    assert code == rr.RR_OK, rr.status_string(code)
    torch.cuda.synchronize()
    return count.cpu().numpy(), idx.cpu().numpy()


def _same_mask(a, b):
    ca, ia = a
    cb, ib = b
    assert np.array_equal(ca, cb)
    H, Nb = ca.shape
    for h in range(H):
        for I in range(Nb):
            assert np.array_equal(ia[h, I, :ca[h, I]], ib[h, I, :cb[h, I]])


def test_static_scratch_matches_workspace_entry_on_consecutive_calls(rr):
    cases = [
        (8192, 8, 2, 128, 128, 16, 0.95, gen.PLANTED, 3),
        (1024, 4, 4, 64, 64, 4, 0.9, gen.IID, 0),          # smaller shape reuses the same array
        (8192, 8, 2, 128, 128, 16, 0.95, gen.PLANTED, 4),  # and back, with new inputs
    ]
    for L, H, Hkv, d, B, S, tau, structure, seed in cases:
        q, k, _ = gen.make_qkv(L, H, Hkv, d, structure, seed)
        qd, kd = _dev(q), _dev(k)
        got = _static_search(rr, qd, kd, B, S, tau)
        ws = rr.workspace(L, H, Hkv, d, B, S)
        c, i = rr.search(qd, kd, B, S, tau, ws=ws)
        assert rr.check_status(ws) == rr.RR_OK
        _same_mask(got, (c.cpu().numpy(), i.cpu().numpy()))


def test_static_scratch_rejects_large_shapes(rr):
    g = 1 << 20   # aligned placeholder addresses: the call must return before using them
    code = rr.lib().rr_search_static(g, g, 65536, 32, 8, 128, 128, 16, ctypes.c_float(0.95), g, g, None)
    assert code == rr.RR_ESCRATCH
    assert "32 MiB" in rr.status_string(code)
    code = rr.lib().rr_search_static(g, g, 1000, 4, 4, 64, 64, 4, ctypes.c_float(0.9), g, g, None)
    assert code == rr.RR_EINVAL
