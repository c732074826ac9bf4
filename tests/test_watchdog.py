"""Bounded device-side waits: a wait that runs out ends the kernel with a status
the host reads (RR_ETIMEOUT), and the context stays usable.

The failure is made on the host, without faulting anything: RR_DEBUG_STALL_WAIT=1
makes the attention kernel's MMA issuer wait on an mbarrier that nothing ever
arrives on, with the wait bound lowered to 20 ms.  The wait gives up, the CTA
takes its abort path (other waits give up too, in-flight copies are drained,
TMEM is released) and the status word reads RR_ETIMEOUT.  Afterwards the
injection is removed and the bound restored; the same call must succeed with
correct results."""
import os

import numpy as np
import pytest
import torch

import gen
import oracle
from tests.mask_compare import output_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rr():
    from dynamic_block_sparse_rr_b200 import _build
    _build.build()
    import dynamic_block_sparse_rr_b200 as m
    m.lib()
    return m


def _dev(a):
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def test_wait_timeout_is_reported_and_context_survives(rr):
    L, H, Hkv, d, B, S = 4096, 8, 2, 128, 128, 16
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 9)
    qd, kd, vd = _dev(q), _dev(k), _dev(v)
    ws = rr.workspace(L, H, Hkv, d, B, S)
    prev = rr.set_wait_limit_ns(20_000_000)
    os.environ["RR_DEBUG_STALL_WAIT"] = "1"
    try:
        rr.attention(qd, kd, vd, B, S, 0.95, ws=ws)
        status = rr.check_status(ws)
    finally:
        del os.environ["RR_DEBUG_STALL_WAIT"]
        rr.set_wait_limit_ns(prev)
    assert status == rr.RR_ETIMEOUT
    # the context is still usable and the operator still correct
    o, count, idx = rr.attention(qd, kd, vd, B, S, 0.95, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    Q, K, V = (gen.bf16_bits_to_f32(x) for x in (q, k, v))
    c, i = count.cpu().numpy(), idx.cpu().numpy()
    O_ref = oracle.sparse_attention(Q, K, V, c, i, B, rows=[(0, 0), (3, 17), (H - 1, L // B - 1)])
    mx, mean = output_errors(o.float().cpu().numpy(), O_ref)
    assert mx <= 2e-2 and mean <= 2e-3
