"""Parity of the search's sampling variants (rr_search_variant) against the oracle.

V1 rotates the sampled offset across strides, V2 replaces the key at the head's
own sampled position by the mean of the stride's keys, V3 selects one mask per GQA
group from the group's summed block mass; any combination.  The per-head block
mass must agree with the oracle's within the same bound as the plain search, the
mask within the near-threshold band, and every head of a GQA group must carry
the same mask.
"""
import numpy as np
import pytest
import torch

import gen
import oracle
from tests.mask_compare import check_mask_format, compare_masks

pytestmark = pytest.mark.gpu

MASS_ERR = 2e-5

ROT, MK, GQA = 1, 2, 4
ALL_FLAGS = [0, ROT, MK, ROT | MK, GQA, ROT | GQA, MK | GQA, ROT | MK | GQA]


@pytest.fixture(scope="module")
def rr():
    from dynamic_block_sparse_rr_b200 import _build
    _build.build()
    import dynamic_block_sparse_rr_b200 as m
    assert torch.cuda.is_available(), "the variant parity tests need a CUDA device"
    m.lib()
    return m


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def run_case(rr, L, H, Hkv, d, B, S, tau, flags, structure, seed):
    q, k, _ = gen.make_qkv(L, H, Hkv, d, structure, seed)
    Q, K = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k)
    qd, kd = to_dev(q), to_dev(k)
    Nb = L // B
    mass = torch.zeros((H, Nb, Nb), dtype=torch.float32, device="cuda")
    ws = rr.workspace(L, H, Hkv, d, B, S, flags=flags)
    count, idx = rr.search_variant(qd, kd, B, S, tau, flags, mass=mass, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    torch.cuda.synchronize()
    count, idx = count.cpu().numpy(), idx.cpu().numpy()
    M_g = mass.cpu().numpy().astype(np.float64)
    rot, mk, gqa = bool(flags & ROT), bool(flags & MK), bool(flags & GQA)

    check_mask_format(count, idx)
    M_o = oracle.block_mass(Q, K, B, S, rotate=rot, mean_keys=mk)
    tri = np.tri(Nb, dtype=bool)[None]
    err = float(np.max(np.abs(np.where(tri, oracle.normalise_mass(M_g) - oracle.normalise_mass(M_o), 0.0))))
    assert err <= MASS_ERR, f"per-head block mass error {err} (flags {flags})"
    count_o, idx_o, m_o = oracle.rr_search(Q, K, B, S, tau, rotate=rot, mean_keys=mk, gqa_mask=gqa)
    st = compare_masks(count, idx, count_o, idx_o, m_o, tau)
    assert st["blocks_fail"] == 0, (flags, st)
    if gqa:
        g = H // Hkv
        for kv in range(Hkv):
            for t in range(1, g):
                assert np.array_equal(count[kv * g + t], count[kv * g]), (flags, kv, t)
                for I in range(Nb):
                    c = count[kv * g, I]
                    assert np.array_equal(idx[kv * g + t, I, :c], idx[kv * g, I, :c])
    return count, idx, st


@pytest.mark.parametrize("flags", ALL_FLAGS)
def test_variant_flags(rr, flags):
    run_case(rr, 2048, 8, 2, 128, 128, 16, 0.9, flags, gen.PLANTED, seed=21)


@pytest.mark.parametrize("L,H,Hkv,d,B,S,tau,structure", [
    (1600, 4, 2, 64, 64, 4, 0.9, gen.PLANTED),        # ragged sampled-row tile (Ns = 400)
    (4096, 7, 1, 128, 128, 16, 0.95, gen.VIDEO),     # GQA 7:1, video-like frames
    (2240, 4, 4, 128, 64, 8, 0.9, gen.PLANTED_BAND),  # Nb = 35 (no float4 group sums needed)
    (512, 3, 3, 64, 64, 64, 0.5, gen.IID),           # r = 1
])
def test_variants_shapes(rr, L, H, Hkv, d, B, S, tau, structure):
    for flags in (ROT, ROT | GQA, MK, ROT | MK | GQA):
        run_case(rr, L, H, Hkv, d, B, S, tau, flags, structure, seed=22)


def test_variants_reduce_to_plain_search_at_stride_one(rr):
    """At S = 1 every query and key is sampled and each stride is one key:
    rotation and stride-mean keys change nothing, so the masks equal the plain
    search's."""
    L, H, Hkv, d, B = 1024, 4, 2, 64, 64
    q, k, _ = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 23)
    qd, kd = to_dev(q), to_dev(k)
    c0, i0 = rr.search(qd, kd, B, 1, 0.9)
    c1, i1 = rr.search_variant(qd, kd, B, 1, 0.9, ROT | MK)
    torch.cuda.synchronize()
    assert torch.equal(c0, c1)
    Nb = L // B
    cols = torch.arange(Nb, device="cuda")[None, None, :] < c0[:, :, None]
    assert torch.equal(torch.where(cols, i0, 0), torch.where(cols, i1, 0))


def test_flags_zero_is_rr_search(rr):
    """rr_search_variant with flags 0 returns rr_search's mask bit for bit."""
    L, H, Hkv, d, B, S = 2048, 4, 2, 128, 128, 16
    q, k, _ = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 24)
    qd, kd = to_dev(q), to_dev(k)
    c0, i0 = rr.search(qd, kd, B, S, 0.9)
    c1, i1 = rr.search_variant(qd, kd, B, S, 0.9, 0)
    torch.cuda.synchronize()
    assert torch.equal(c0, c1)
    Nb = L // B
    cols = torch.arange(Nb, device="cuda")[None, None, :] < c0[:, :, None]
    assert torch.equal(torch.where(cols, i0, 0), torch.where(cols, i1, 0))


def test_gqa_mask_long_rows_radix_path(rr):
    """Rows longer than 1024 blocks (Nb = 2048) with one mask per GQA group: the
    CTA-per-row Top-tau path writing each selection to both heads of a group.
    Checked on sampled rows against the group mass the GPU selected on (the
    heads' fp32 block masses summed in head order): every head of a group has
    the same list, the list reaches tau of the row, dropping its lightest block
    falls below tau, and no dropped block outweighs a kept one (equal masses
    keep the lower J)."""
    L, H, Hkv, d, B, S, tau = 131072, 4, 2, 64, 64, 16, 0.9
    Nb = L // B
    q, k, _ = gen.make_qkv(L, H, Hkv, d, gen.PLANTED_BAND, 61)
    mass = torch.zeros((H, Nb, Nb), dtype=torch.float32, device="cuda")
    ws = rr.workspace(L, H, Hkv, d, B, S, flags=GQA)
    count, idx = rr.search_variant(to_dev(q), to_dev(k), B, S, tau, GQA, mass=mass, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    count, idx = count.cpu().numpy(), idx.cpu().numpy()
    check_mask_format(count, idx)
    g = H // Hkv
    rng = np.random.default_rng(62)
    rows = sorted(set(rng.integers(1024, Nb - 1, 48).tolist()) | {1024, Nb - 2})
    for kv in range(Hkv):
        for I in rows:
            per_head = mass[kv * g:(kv + 1) * g, I, :I + 1].cpu().numpy()
            gm = per_head[0].copy()
            for t in range(1, g):
                gm = gm + per_head[t]                     # fp32, head order
            c = count[kv * g, I]
            kept = idx[kv * g, I, :c]
            for t in range(1, g):
                assert count[kv * g + t, I] == c and np.array_equal(idx[kv * g + t, I, :c], kept)
            gm = gm.astype(np.float64)
            total = gm.sum()
            drop = np.setdiff1d(np.arange(I + 1), kept)
            share = gm[kept].sum() / total
            assert share >= tau - 1e-6, (kv, I, share)
            assert share - gm[kept].min() / total < tau + 1e-6, (kv, I)
            if drop.size:
                assert gm[kept].min() >= gm[drop].max(), (kv, I)
                tied = drop[gm[drop] == gm[kept].min()]
                if tied.size:
                    assert tied.min() > kept[gm[kept] == gm[kept].min()].max(), (kv, I)


@pytest.mark.slow
def test_variants_video64k_full_size(rr):
    """Stride-mean keys and the GQA mask on the full video workload (H=28/Hkv=4,
    L=65536): masks against the oracle's in full."""
    cfg = gen.CONFIGS["video64k"]
    for flags in (MK, GQA):
        count, idx, st = run_case(rr, cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S, cfg.tau, flags,
                                  cfg.structure, seed=cfg.seed)
        Nb = cfg.L // cfg.B
        print(flags, st, "visited", count.sum() / (cfg.H * Nb * (Nb + 1) / 2))
