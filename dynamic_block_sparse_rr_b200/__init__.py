"""Python binding of the B200 RRAttention prefill operator (``librr.so``).

Argument marshalling only: every step of the operator runs in the CUDA kernels
behind the C ABI of ``include/rr.h``.  PyTorch supplies device memory and the
current stream.  There is no fallback: if ``librr.so`` is missing or cannot be
loaded, importing the operator functions raises.

Tensors: q ``[L, H, d]``, k and v ``[L, Hkv, d]``, bf16, contiguous, on one CUDA
device.  Masks: ``count [H, Nb]`` and ``idx [H, Nb, Nb]`` int32 (see rr.h).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librr.so")

RR_OK, RR_EINVAL, RR_EUNSUPPORTED, RR_EALIGN, RR_ECUDA, RR_ETIMEOUT, RR_ESCRATCH, RR_EMASK = range(8)

# every symbol that include/rr.h declares
EXPORTS = ("rr_workspace_size", "rr_search", "rr_sparse_attn", "rr_attention", "rr_check_status",
           "rr_set_wait_limit_ns", "rr_status_string", "rr_search_static", "rr_mask_recall",
           "rr_workspace_size_variant", "rr_search_variant", "rr_mask_to_dense",
           "rr_workspace_size_host", "rr_attention_host", "rr_decode_workspace_size", "rr_decode",
           "rr_decode_variant")

# sampling-variant flags of rr_search_variant (rr.h)
VAR_ROTATE, VAR_MEAN_KEYS, VAR_GQA_MASK = 1, 2, 4


class RRError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"librr.so not built at {LIB_PATH}; run python -m dynamic_block_sparse_rr_b200._build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.rr_workspace_size.argtypes = [i, i, i, i, i, i, ctypes.POINTER(sz)]
        L.rr_search.argtypes = [vp, vp, i, i, i, i, i, i, f, vp, vp, vp, vp, sz, vp]
        L.rr_sparse_attn.argtypes = [vp, vp, vp, i, i, i, i, i, vp, vp, vp, vp, sz, vp]
        L.rr_attention.argtypes = [vp, vp, vp, i, i, i, i, i, i, f, vp, vp, vp, vp, sz, vp]
        L.rr_check_status.argtypes = [vp, vp]
        L.rr_search_static.argtypes = [vp, vp, i, i, i, i, i, i, f, vp, vp, vp]
        L.rr_search_static.restype = ctypes.c_int
        L.rr_mask_recall.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.rr_mask_recall.restype = ctypes.c_int
        u = ctypes.c_uint
        L.rr_workspace_size_variant.argtypes = [i, i, i, i, i, i, u, ctypes.POINTER(sz)]
        L.rr_workspace_size_variant.restype = ctypes.c_int
        L.rr_search_variant.argtypes = [vp, vp, i, i, i, i, i, i, f, u, vp, vp, vp, vp, sz, vp]
        L.rr_search_variant.restype = ctypes.c_int
        L.rr_mask_to_dense.argtypes = [vp, vp, i, i, vp, vp]
        L.rr_workspace_size_host.argtypes = [i, i, i, i, i, i, ctypes.POINTER(sz)]
        L.rr_workspace_size_host.restype = ctypes.c_int
        L.rr_attention_host.argtypes = [vp, vp, vp, i, i, i, i, i, i, f, vp, vp, vp, vp, sz, vp, vp]
        L.rr_attention_host.restype = ctypes.c_int
        L.rr_mask_to_dense.restype = ctypes.c_int
        L.rr_decode_workspace_size.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(sz)]
        L.rr_decode_workspace_size.restype = ctypes.c_int
        L.rr_decode.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp, vp, sz, vp]
        L.rr_decode.restype = ctypes.c_int
        L.rr_decode_variant.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, ctypes.c_uint, vp, vp, vp, vp, sz, vp]
        L.rr_decode_variant.restype = ctypes.c_int
        L.rr_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.rr_set_wait_limit_ns.restype = ctypes.c_uint64
        L.rr_status_string.argtypes = [i]
        L.rr_status_string.restype = ctypes.c_char_p
        for name in ("rr_workspace_size", "rr_search", "rr_sparse_attn", "rr_attention", "rr_check_status"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().rr_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != RR_OK:
        raise RRError(code, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _shape(q, k):
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q must be [L, H, d] and k [L, Hkv, d]")
    L, H, d = q.shape
    if k.shape[0] != L or k.shape[2] != d:
        raise ValueError("q and k disagree on L or d")
    for t in (q, k):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    return L, H, k.shape[1], d


def workspace_size(L: int, H: int, Hkv: int, d: int, B: int, S: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().rr_workspace_size(L, H, Hkv, d, B, S, ctypes.byref(n)), "rr_workspace_size")
    return n.value


def workspace(L: int, H: int, Hkv: int, d: int, B: int, S: int, device=None, flags: int = 0) -> torch.Tensor:
    """A device workspace (uint8) of the size the operator needs (for the sampling
    variant ``flags`` when given)."""
    n = workspace_size(L, H, Hkv, d, B, S) if flags == 0 else workspace_size_variant(L, H, Hkv, d, B, S, flags)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def workspace_size_variant(L: int, H: int, Hkv: int, d: int, B: int, S: int, flags: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().rr_workspace_size_variant(L, H, Hkv, d, B, S, int(flags), ctypes.byref(n)),
           "rr_workspace_size_variant")
    return n.value


def empty_mask(H: int, Nb: int, device=None):
    dev = device or "cuda"
    return (torch.empty((H, Nb), dtype=torch.int32, device=dev),
            torch.empty((H, Nb, Nb), dtype=torch.int32, device=dev))


def search(q, k, B: int, S: int, tau: float, count=None, idx=None, mass=None, ws=None, stream=None):
    """Pattern search -> (count [H, Nb], idx [H, Nb, Nb]).  ``mass`` (optional, fp32
    [H, Nb, Nb]) receives the unnormalised block masses."""
    L, H, Hkv, d = _shape(q, k)
    Nb = L // B
    if count is None or idx is None:
        count, idx = empty_mask(H, Nb, q.device)
    if ws is None:
        ws = workspace(L, H, Hkv, d, B, S, q.device)
    _check(lib().rr_search(q.data_ptr(), k.data_ptr(), L, H, Hkv, d, B, S, float(tau), count.data_ptr(),
                           idx.data_ptr(), _ptr(mass), ws.data_ptr(), ws.numel(), _stream(stream)), "rr_search")
    return count, idx


def search_variant(q, k, B: int, S: int, tau: float, flags: int, count=None, idx=None, mass=None, ws=None,
                   stream=None):
    """Pattern search with the sampling variants ``flags`` (VAR_ROTATE,
    VAR_MEAN_KEYS, VAR_GQA_MASK, or-ed) -> (count, idx).  ``mass`` receives the
    per-head block masses."""
    L, H, Hkv, d = _shape(q, k)
    Nb = L // B
    if count is None or idx is None:
        count, idx = empty_mask(H, Nb, q.device)
    if ws is None:
        ws = workspace(L, H, Hkv, d, B, S, q.device, flags=flags)
    _check(lib().rr_search_variant(q.data_ptr(), k.data_ptr(), L, H, Hkv, d, B, S, float(tau), int(flags),
                                   count.data_ptr(), idx.data_ptr(), _ptr(mass), ws.data_ptr(), ws.numel(),
                                   _stream(stream)), "rr_search_variant")
    return count, idx


def sparse_attn(q, k, v, count, idx, B: int, out=None, ws=None, stream=None):
    """Causal block-sparse attention over (count, idx) -> o [L, H, d] bf16."""
    L, H, Hkv, d = _shape(q, k)
    _shape(v, k)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = torch.empty(256, dtype=torch.uint8, device=q.device)
    _check(lib().rr_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), L, H, Hkv, d, B, count.data_ptr(),
                                idx.data_ptr(), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
           "rr_sparse_attn")
    return out


def attention(q, k, v, B: int, S: int, tau: float, out=None, count=None, idx=None, ws=None, stream=None):
    """Search then sparse attention on one stream -> (o, count, idx)."""
    L, H, Hkv, d = _shape(q, k)
    _shape(v, k)
    Nb = L // B
    if out is None:
        out = torch.empty_like(q)
    if count is None or idx is None:
        count, idx = empty_mask(H, Nb, q.device)
    if ws is None:
        ws = workspace(L, H, Hkv, d, B, S, q.device)
    _check(lib().rr_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), L, H, Hkv, d, B, S, float(tau),
                              count.data_ptr(), idx.data_ptr(), out.data_ptr(), ws.data_ptr(), ws.numel(),
                              _stream(stream)), "rr_attention")
    return out, count, idx


def exact_block_mass(q, k, B: int, mass=None, stream=None):
    """Exact full-attention block mass [H, Nb, Nb] fp32 (unnormalised, J <= I):
    the search at stride S = 1, where every query is sampled and every key is its
    own stride."""
    L, H, Hkv, d = _shape(q, k)
    Nb = L // B
    if mass is None:
        mass = torch.zeros((H, Nb, Nb), dtype=torch.float32, device=q.device)
    search(q, k, B, 1, 1.0, mass=mass, stream=stream)
    return mass


def mask_recall(mass, count, idx, out=None, stream=None):
    """Share of each row's mass kept by the mask -> recall [H, Nb] fp32."""
    H, Nb = count.shape
    if out is None:
        out = torch.empty((H, Nb), dtype=torch.float32, device=count.device)
    _check(lib().rr_mask_recall(mass.data_ptr(), count.data_ptr(), idx.data_ptr(), H, Nb, out.data_ptr(),
                                _stream(stream)), "rr_mask_recall")
    return out


def check_status(ws, stream=None) -> int:
    """Synchronise and return the device-side status of the last call on ``ws``."""
    return lib().rr_check_status(ws.data_ptr(), _stream(stream))


def set_wait_limit_ns(ns: int) -> int:
    return lib().rr_set_wait_limit_ns(int(ns))


def mask_to_dense(count, idx, out=None, stream=None):
    """Dense uint8 view [H, Nb, Nb] of a block mask (1 where a block is listed)."""
    H, Nb = count.shape
    if out is None:
        out = torch.empty((H, Nb, Nb), dtype=torch.uint8, device=count.device)
    _check(lib().rr_mask_to_dense(count.data_ptr(), idx.data_ptr(), H, Nb, out.data_ptr(), _stream(stream)),
           "rr_mask_to_dense")
    return out


def workspace_size_host(L: int, H: int, Hkv: int, d: int, B: int, S: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().rr_workspace_size_host(L, H, Hkv, d, B, S, ctypes.byref(n)), "rr_workspace_size_host")
    return n.value


_copy_streams = {}


def attention_host(qh, kh, vh, B: int, S: int, tau: float, out=None, count=None, idx=None, ws=None,
                   stream=None, copy_stream=None, device=None):
    """rr_attention on host tensors (CPU, bf16, contiguous; page-locked for
    asynchronous copies), copies pipelined against the kernels kv head by kv
    head -> (o_host, count, idx); the mask stays on the device."""
    if qh.dim() != 3 or kh.dim() != 3 or vh.shape != kh.shape:
        raise ValueError("q must be [L, H, d], k and v [L, Hkv, d]")
    for t in (qh, kh, vh):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 host tensors")
    L, H, d = qh.shape
    Hkv = kh.shape[1]
    Nb = L // B
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if out is None:
        out = torch.empty(qh.shape, dtype=torch.bfloat16, pin_memory=True)
    if count is None or idx is None:
        count, idx = empty_mask(H, Nb, dev)
    if ws is None:
        ws = torch.empty(workspace_size_host(L, H, Hkv, d, B, S), dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    if copy_stream is None:
        if dev not in _copy_streams:
            _copy_streams[dev] = torch.cuda.Stream(device=dev)
        copy_stream = _copy_streams[dev]
    _check(lib().rr_attention_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), L, H, Hkv, d, B, S, float(tau),
                                   count.data_ptr(), idx.data_ptr(), out.data_ptr(), ws.data_ptr(), ws.numel(),
                                   s.cuda_stream, copy_stream.cuda_stream), "rr_attention_host")
    return out, count, idx


def decode_workspace_size(N: int, Lmax: int, H: int, Hkv: int, d: int, B: int, S: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().rr_decode_workspace_size(N, Lmax, H, Hkv, d, B, S, ctypes.byref(n)), "rr_decode_workspace_size")
    return n.value


def decode(q, k_cache, v_cache, lens, B: int, S: int, tau: float, out=None, count=None, idx=None, ws=None,
           stream=None, flags: int = 0):
    """One decode step: q [N, H, d], caches [N, Lmax, Hkv, d] bf16, lens [N] int32
    (device) -> (o [N, H, d], count [N, H], idx [N, H, Lmax/B]).  flags:
    VAR_GQA_MASK for one list per GQA group (rr_decode_variant)."""
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be [N, H, d], k_cache and v_cache [N, Lmax, Hkv, d]")
    N, H, d = q.shape
    _, Lmax, Hkv, dk = k_cache.shape
    if k_cache.shape[0] != N or dk != d or lens.shape != (N,) or lens.dtype != torch.int32:
        raise ValueError("shapes disagree (q, caches, lens)")
    for t in (q, k_cache, v_cache):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q and the caches must be contiguous bf16 CUDA tensors")
    Nb = Lmax // B
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if count is None or idx is None:
        count = torch.empty((N, H), dtype=torch.int32, device=dev)
        idx = torch.empty((N, H, Nb), dtype=torch.int32, device=dev)
    if ws is None:
        ws = torch.empty(decode_workspace_size(N, Lmax, H, Hkv, d, B, S), dtype=torch.uint8, device=dev)
    _check(lib().rr_decode_variant(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), lens.data_ptr(), N, Lmax,
                                   H, Hkv, d, B, S, float(tau), int(flags), count.data_ptr(), idx.data_ptr(),
                                   out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)), "rr_decode_variant")
    return out, count, idx

