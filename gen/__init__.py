"""Seeded synthetic inputs shared by the CUDA path and the fp64 oracle.

The generator itself is plain C (``gen.c``, counter-based, OpenMP, thread-count
independent); this module builds it on first use and exposes:

* ``CONFIGS``: the workloads, named by what they are, with their sizes.
* ``make_qkv(cfg, seed=0)``: bf16 bit patterns (numpy ``uint16``) for Q, K, V in
  the ``[L, heads, d]`` layout.
* ``bf16_bits_to_f64`` / ``bf16_bits_to_f32``: widening helpers.

Nothing here computes any step of the method.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libgen.so")

IID, PLANTED, PLANTED_BAND, VIDEO = 0, 1, 2, 3
ROLE_Q, ROLE_K, ROLE_V = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    L: int
    H: int
    Hkv: int
    d: int
    B: int
    S: int
    taus: tuple
    structure: int
    seed: int = 0

    @property
    def tau(self) -> float:
        return self.taus[0] if len(self.taus) == 1 else self.taus[1]


CONFIGS = {
    # correctness workload: i.i.d. N(0,1), softmax scale 1/sqrt(d)
    "tiny": Config("tiny", L=1024, H=4, Hkv=4, d=64, B=64, S=4, taus=(0.9,), structure=IID),
    # LLaMA-3.1-8B-shaped GQA layer with planted sinks / periodic keys
    "llama16k": Config("llama16k", L=16384, H=32, Hkv=8, d=128, B=128, S=16, taus=(0.95,),
                       structure=PLANTED),
    "llama32k": Config("llama32k", L=32768, H=32, Hkv=8, d=128, B=128, S=16,
                       taus=(0.9, 0.95, 0.99), structure=PLANTED),
    # headline: 128K context with an additional local band
    "llama128k": Config("llama128k", L=131072, H=32, Hkv=8, d=128, B=128, S=16, taus=(0.95,),
                        structure=PLANTED_BAND),
    # video-like multimodal prefill: 256 frames x 256 tokens
    "video64k": Config("video64k", L=65536, H=28, Hkv=4, d=128, B=128, S=16, taus=(0.95,),
                       structure=VIDEO),
}


def build(force: bool = False) -> str:
    """Compile ``libgen.so`` next to this file (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.rr_gen_fill.restype = ctypes.c_int
        lib.rr_gen_fill.argtypes = [ctypes.c_int, ctypes.c_uint64, ctypes.c_int, ctypes.c_int64,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        lib.rr_gen_normal.restype = ctypes.c_double
        lib.rr_gen_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        _lib = lib
    return _lib


def normal(seed: int, tid: int, n: int) -> float:
    """Element ``n`` of stream ``tid`` (one N(0,1) draw)."""
    return _load().rr_gen_normal(seed, tid, n)


def fill(structure: int, seed: int, role: int, L: int, H: int, Hkv: int, d: int) -> np.ndarray:
    """One tensor as bf16 bits, shape ``[L, heads, d]``."""
    heads = H if role == ROLE_Q else Hkv
    out = np.empty((L, heads, d), dtype=np.uint16)
    rc = _load().rr_gen_fill(structure, seed, role, L, H, Hkv, d, out.ctypes.data)
    if rc != 0:
        raise ValueError("rr_gen_fill rejected its arguments")
    return out


def make_qkv(L: int, H: int, Hkv: int, d: int, structure: int = IID, seed: int = 0):
    """Q ``[L,H,d]``, K and V ``[L,Hkv,d]`` as bf16 bit patterns (numpy uint16)."""
    return (fill(structure, seed, ROLE_Q, L, H, Hkv, d),
            fill(structure, seed, ROLE_K, L, H, Hkv, d),
            fill(structure, seed, ROLE_V, L, H, Hkv, d))


def make_config(cfg: Config, seed: int | None = None):
    return make_qkv(cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.structure, cfg.seed if seed is None else seed)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)
