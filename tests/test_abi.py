"""The C ABI: the library loads, exports every symbol rr.h declares, and rejects
bad arguments on the host (no GPU needed; no compute call is made)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rr.h")


@pytest.fixture(scope="module")
def rr():
    from dynamic_block_sparse_rr_b200 import _build
    _build.build()
    import dynamic_block_sparse_rr_b200 as m
    m.lib()
    return m


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rr_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(rr):
    names = _declared()
    assert names == sorted(rr.EXPORTS)
    for n in names:
        assert hasattr(rr.lib(), n), n


def test_status_strings(rr):
    for code in range(8):
        s = rr.status_string(code)
        assert isinstance(s, str) and s
    assert rr.status_string(0) == "ok"


def test_wait_limit_roundtrip(rr):
    prev = rr.set_wait_limit_ns(12345)
    assert rr.set_wait_limit_ns(prev) == 12345


def _ws(L, H, Hkv, d, B, S):
    n = ctypes.c_size_t()
    code = rr_lib().rr_workspace_size(L, H, Hkv, d, B, S, ctypes.byref(n))
    return code, n.value


def rr_lib():
    import dynamic_block_sparse_rr_b200 as m
    return m.lib()


@pytest.mark.parametrize("args,code", [
    ((1024, 4, 4, 64, 64, 4), 0),
    ((131072, 32, 8, 128, 128, 16), 0),
    ((1024, 4, 3, 64, 64, 4), 1),      # H % Hkv
    ((1000, 4, 4, 64, 64, 4), 1),      # L % B
    ((1024, 4, 4, 64, 64, 3), 1),      # B % S
    ((1024, 4, 4, 64, 64, 0), 1),
    ((1024, 4, 4, 96, 64, 4), 2),      # d
    ((1024, 4, 4, 64, 32, 4), 2),      # B
    ((64 * 8192, 1, 1, 64, 64, 4), 2),  # Nb > 4096
    ((0, 4, 4, 64, 64, 4), 1),
])
def test_workspace_size_validation(rr, args, code):
    c, n = _ws(*args)
    assert c == code
    if code == 0:
        L, H, Hkv, d, B, S = args
        assert n >= H * (L // B) ** 2 * 4


def test_search_rejects_before_any_launch(rr):
    lib = rr.lib()
    good = 1 << 20            # fake, 16-byte aligned "device" addresses: never dereferenced
    L, H, Hkv, d, B, S = 1024, 4, 4, 64, 64, 4
    _, n = _ws(L, H, Hkv, d, B, S)
    args = dict(q=good, k=good, tau=0.9, count=good, idx=good, mass=None, ws=good, nws=n)

    def call(**kw):
        a = dict(args, **kw)
        return lib.rr_search(a["q"], a["k"], L, H, Hkv, d, B, S, a["tau"], a["count"], a["idx"], a["mass"],
                             a["ws"], a["nws"], None)

    assert call(q=None) == rr.RR_EINVAL
    assert call(idx=None) == rr.RR_EINVAL
    assert call(tau=0.0) == rr.RR_EINVAL
    assert call(tau=-1.0) == rr.RR_EINVAL
    assert call(tau=float("nan")) == rr.RR_EINVAL
    assert call(q=good + 8) == rr.RR_EALIGN
    assert call(mass=good + 4) == rr.RR_EALIGN
    assert call(ws=good + 16) == rr.RR_EALIGN
    assert call(nws=n - 1) == rr.RR_EINVAL
    assert call(ws=None) == rr.RR_EINVAL
    assert lib.rr_search(good, good, L, H, Hkv, d, 32, S, 0.9, good, good, None, good, n, None) == rr.RR_EUNSUPPORTED


def test_sparse_attn_and_attention_reject(rr):
    lib = rr.lib()
    g = 1 << 20
    L, H, Hkv, d, B = 1024, 4, 2, 128, 128
    assert lib.rr_sparse_attn(g, g, g, L, H, Hkv, d, B, g, g, None, g, 256, None) == rr.RR_EINVAL
    assert lib.rr_sparse_attn(g, g, g + 2, L, H, Hkv, d, B, g, g, g, g, 256, None) == rr.RR_EALIGN
    assert lib.rr_sparse_attn(g, g, g, L, H, Hkv, d, B, g, g, g, g + 64, 256, None) == rr.RR_EALIGN
    assert lib.rr_sparse_attn(g, g, g, L, H, 3, d, B, g, g, g, g, 256, None) == rr.RR_EINVAL
    assert lib.rr_sparse_attn(g, g, g, L, H, Hkv, 80, B, g, g, g, g, 256, None) == rr.RR_EUNSUPPORTED
    assert lib.rr_attention(g, g, None, L, H, Hkv, d, B, 16, 0.95, g, g, g, g, 1 << 30, None) == rr.RR_EINVAL
    assert lib.rr_attention(g, g, g, L, H, Hkv, d, B, 16, 0.0, g, g, g, g, 1 << 30, None) == rr.RR_EINVAL


def test_binding_fails_loudly_without_library(monkeypatch):
    import dynamic_block_sparse_rr_b200 as m
    monkeypatch.setattr(m, "LIB_PATH", os.path.join(ROOT, "no", "such", "librr.so"))
    monkeypatch.setattr(m, "_lib", None)
    with pytest.raises(ImportError):
        m.lib()


def _ws_var(L, H, Hkv, d, B, S, flags):
    n = ctypes.c_size_t()
    code = rr_lib().rr_workspace_size_variant(L, H, Hkv, d, B, S, flags, ctypes.byref(n))
    return code, n.value


def test_variant_workspace_sizes(rr):
    L, H, Hkv, d, B, S = 4096, 8, 2, 128, 128, 16
    Ns, Nb = L // S, L // B
    assert _ws_var(L, H, Hkv, d, B, S, 0) == _ws(L, H, Hkv, d, B, S)
    base = _ws_var(L, H, Hkv, d, B, S, 0)[1]
    # stride-mean keys add the pooled (hi, lo) pair
    assert _ws_var(L, H, Hkv, d, B, S, rr.VAR_MEAN_KEYS)[1] == base + 2 * Ns * Hkv * d * 2
    # rotation adds the gathered queries and the gathered keys (sampled keys)
    assert _ws_var(L, H, Hkv, d, B, S, rr.VAR_ROTATE)[1] == base + 2 * Ns * H * d * 2
    assert (_ws_var(L, H, Hkv, d, B, S, rr.VAR_ROTATE | rr.VAR_MEAN_KEYS)[1]
            == base + 2 * Ns * Hkv * d * 2 + Ns * H * d * 2)
    # the GQA mask adds the group masses
    assert _ws_var(L, H, Hkv, d, B, S, rr.VAR_GQA_MASK)[1] == base + Hkv * Nb * Nb * 4
    assert _ws_var(L, H, Hkv, d, B, S, 8)[0] == rr.RR_EINVAL
    assert _ws_var(L, H, Hkv, d, B, 3, 1)[0] == rr.RR_EINVAL


def test_search_variant_rejects_before_any_launch(rr):
    lib = rr.lib()
    g = 1 << 20
    L, H, Hkv, d, B, S = 1024, 4, 2, 64, 64, 4
    flags = rr.VAR_ROTATE | rr.VAR_MEAN_KEYS | rr.VAR_GQA_MASK
    _, n = _ws_var(L, H, Hkv, d, B, S, flags)

    def call(flags=flags, q=g, nws=n, tau=0.9):
        return lib.rr_search_variant(q, g, L, H, Hkv, d, B, S, tau, flags, g, g, None, g, nws, None)

    assert call(flags=16) == rr.RR_EINVAL
    assert call(q=None) == rr.RR_EINVAL
    assert call(q=g + 2) == rr.RR_EALIGN
    assert call(tau=0.0) == rr.RR_EINVAL
    assert call(nws=n - 1) == rr.RR_EINVAL           # the variant workspace is larger than the plain one
    assert n > _ws(L, H, Hkv, d, B, S)[1]


def test_host_workspace_and_rejections(rr):
    lib = rr.lib()
    g = 1 << 20
    L, H, Hkv, d, B, S = 4096, 8, 2, 128, 128, 16
    n = ctypes.c_size_t()
    assert lib.rr_workspace_size_host(L, H, Hkv, d, B, S, ctypes.byref(n)) == rr.RR_OK
    gq = H // Hkv
    # two slots of one kv head's q, k, v, o plus one kv head's search scratch
    assert n.value >= 2 * (2 * L * gq * d * 2 + 2 * L * d * 2) + gq * (L // B) ** 2 * 4
    assert lib.rr_workspace_size_host(L, H, 3, d, B, S, ctypes.byref(n)) == rr.RR_EINVAL
    nws = rr.workspace_size_host(L, H, Hkv, d, B, S)

    def call(qh=g, oh=g, count=g, ws=g, nb=nws, tau=0.9):
        return lib.rr_attention_host(qh, g, g, L, H, Hkv, d, B, S, tau, count, g, oh, ws, nb, None, None)

    assert call(qh=None) == rr.RR_EINVAL
    assert call(oh=None) == rr.RR_EINVAL
    assert call(count=g + 4) == rr.RR_EALIGN
    assert call(ws=g + 64) == rr.RR_EALIGN
    assert call(nb=nws - 1) == rr.RR_EINVAL
    assert call(tau=0.0) == rr.RR_EINVAL


def test_decode_workspace_and_rejections(rr):
    lib = rr.lib()
    g = 1 << 20
    n = ctypes.c_size_t()
    N, Lmax, H, Hkv, d, B, S = 2, 4096, 8, 2, 128, 128, 16
    assert lib.rr_decode_workspace_size(N, Lmax, H, Hkv, d, B, S, ctypes.byref(n)) == rr.RR_OK
    W, NC = (Lmax // B + 31) // 32, (Lmax // B + 15) // 16
    # status word, sampled scores, bitmaps and per-chunk partials
    assert n.value >= N * H * (Lmax // S) * 4 + N * H * W * 4 + N * H * NC * (d + 2) * 4
    nws = n.value
    for args, code in [((N, Lmax, H, 3, d, B, S), rr.RR_EINVAL),        # H % Hkv
                       ((N, 4000, H, Hkv, d, B, S), rr.RR_EINVAL),      # Lmax % B
                       ((N, Lmax, H, Hkv, d, B, 3), rr.RR_EINVAL),      # B % S
                       ((N, Lmax, 18, 2, d, B, S), rr.RR_EUNSUPPORTED),  # more than 8 heads per kv head
                       ((N, Lmax, H, Hkv, 96, B, S), rr.RR_EUNSUPPORTED),
                       ((0, Lmax, H, Hkv, d, B, S), rr.RR_EINVAL)]:
        assert lib.rr_decode_workspace_size(*args, ctypes.byref(n)) == code, args

    def call(q=g, lens=g, tau=0.9, ws=g, nws=nws):
        return lib.rr_decode(q, g, g, lens, N, Lmax, H, Hkv, d, B, S, tau, g, g, g, ws, nws, None)

    assert call(q=None) == rr.RR_EINVAL
    assert call(tau=0.0) == rr.RR_EINVAL
    assert call(q=g + 8) == rr.RR_EALIGN
    assert call(lens=g + 2) == rr.RR_EALIGN
    assert call(ws=g + 16) == rr.RR_EALIGN
    assert call(nws=nws - 1) == rr.RR_EINVAL
    # the decode variants take only the GQA-mask flag
    assert lib.rr_decode_variant(g, g, g, g, N, Lmax, H, Hkv, d, B, S, 0.9, rr.VAR_ROTATE, g, g, g, g, nws,
                                 None) == rr.RR_EINVAL
    assert lib.rr_decode_variant(g, g, g, g, N, Lmax, H, Hkv, d, B, S, 0.0, rr.VAR_GQA_MASK, g, g, g, g, nws,
                                 None) == rr.RR_EINVAL

