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


def test_decode_wait_timeout_is_reported_and_context_survives(rr):
    """The same injection in the decode step: every attention CTA's first wait
    runs out, its rows get empty partials (zero outputs), the status reads
    RR_ETIMEOUT, and the next call is correct again."""
    N, Lmax, H, Hkv, d, B, S, tau = 2, 1024, 8, 2, 128, 128, 16, 0.9
    lens = [1024, 700]
    qs, ks, vs = [], [], []
    for n in range(N):
        q, k, v = gen.make_qkv(Lmax, H, Hkv, d, gen.PLANTED, 21 + n)
        qs.append(gen.bf16_bits_to_f32(q)[lens[n] - 1])
        ks.append(gen.bf16_bits_to_f32(k))
        vs.append(gen.bf16_bits_to_f32(v))
    Q, K, V = np.stack(qs), np.stack(ks), np.stack(vs)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()
    qd, kd, vd = to(Q), to(K), to(V)
    ld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(rr.decode_workspace_size(N, Lmax, H, Hkv, d, B, S), dtype=torch.uint8, device="cuda")
    prev = rr.set_wait_limit_ns(20_000_000)
    os.environ["RR_DEBUG_STALL_WAIT"] = "1"
    try:
        o, _, _ = rr.decode(qd, kd, vd, ld, B, S, tau, ws=ws)
        status = rr.check_status(ws)
    finally:
        del os.environ["RR_DEBUG_STALL_WAIT"]
        rr.set_wait_limit_ns(prev)
    assert status == rr.RR_ETIMEOUT
    assert not torch.any(o.float() != 0)
    o, count, idx = rr.decode(qd, kd, vd, ld, B, S, tau, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    og, c, i = o.float().cpu().numpy(), count.cpu().numpy(), idx.cpu().numpy()
    for n in range(N):
        ref = oracle.decode_attention(Q[n], K[n], V[n], lens[n] - 1, [i[n, h, :c[n, h]] for h in range(H)], B)
        assert np.abs(og[n] - ref).max() <= 2e-2
