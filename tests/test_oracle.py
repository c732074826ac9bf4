"""Pins of the fp64 oracle against what the method and the mathematics fix.

Every check here compares the oracle with something other than itself: a
library routine (torch scaled_dot_product_attention in fp64), a closed form, a
hand-derived fixture, or brute force.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fig2_uniform_keys.txt")


def _fixture():
    m, sel, pos = {}, {}, {}
    with open(GOLDEN) as f:
        for line in f:
            t = line.split()
            if not t or t[0].startswith("#"):
                continue
            if t[0] == "m":
                m[(int(t[1]), int(t[2]))] = Fraction(int(t[3]), int(t[4]))
            elif t[0] == "sel":
                sel[(float(t[1]), int(t[2]))] = [int(x) for x in t[3:]]
            elif t[0] == "pos":
                pos[int(t[1])] = [int(x) for x in t[2:]]
    return m, sel, pos


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa_probs(Q, K):
    """Causal attention probabilities A[h, q, k] from torch's SDPA with V = identity."""
    L, H, d = Q.shape
    g = H // K.shape[1]
    q = torch.from_numpy(Q).permute(1, 0, 2)                       # [H, L, d]
    k = torch.from_numpy(np.repeat(K, g, axis=1)).permute(1, 0, 2)
    eye = torch.eye(L, dtype=torch.float64).expand(H, L, L)
    return F.scaled_dot_product_attention(q, k, eye, is_causal=True).numpy()


def _sdpa(Q, K, V, mask=None, causal=False):
    H = Q.shape[1]
    g = H // K.shape[1]
    q = torch.from_numpy(Q).permute(1, 0, 2)
    k = torch.from_numpy(np.repeat(K, g, axis=1)).permute(1, 0, 2)
    v = torch.from_numpy(np.repeat(V, g, axis=1)).permute(1, 0, 2)
    am = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(q, k, v, attn_mask=am, is_causal=causal).permute(1, 0, 2).numpy()


# ------------------------------------------------------------------ sampling
def test_sampling_fig2_fixture():
    _, _, pos = _fixture()
    p = oracle.sampled_positions(32, 4, 4)
    for h, want in pos.items():
        assert p[h].tolist() == want


@pytest.mark.parametrize("L,H,S", [(1024, 4, 4), (16384, 32, 16), (4096, 28, 16), (512, 3, 8)])
def test_sampling_round_robin_properties(L, H, S):
    p = oracle.sampled_positions(L, H, S)
    Ns = L // S
    i = np.arange(Ns)
    assert p.shape == (H, Ns)
    for h in range(H):
        assert np.all(p[h] >= i * S) and np.all(p[h] < (i + 1) * S)
        assert np.all(p[h] - i * S == h % S)
    if H >= S:  # heads 0..S-1 cover every position exactly once
        cover = np.sort(p[:S].reshape(-1))
        assert np.array_equal(cover, np.arange(L))


# --------------------------------------------------------------- key pooling
def test_pool_keys_closed_forms():
    K = _rand((64, 2, 8), 1)
    assert np.array_equal(oracle.pool_keys(K, 1), K)                       # S = 1: identity
    ramp = np.arange(64, dtype=np.float64)[:, None, None] * np.ones((1, 2, 8))
    pooled = oracle.pool_keys(ramp, 4)                                     # mean of j*4..j*4+3
    assert np.allclose(pooled[:, 0, 0], np.arange(16) * 4 + 1.5, atol=0, rtol=0)
    const = np.repeat(_rand((16, 2, 8), 2), 4, axis=0)                     # constant per stride
    assert np.allclose(oracle.pool_keys(const, 4), const[::4], atol=1e-15)


# --------------------------------------------------------------- block mass
def test_uniform_keys_fig2_fixture():
    m_want, sel_want, _ = _fixture()
    Q = _rand((32, 4, 8), 3)
    K = np.zeros((32, 2, 8))
    m = oracle.normalise_mass(oracle.block_mass(Q, K, B=8, S=4))
    for h in range(4):
        for (I, J), fr in m_want.items():
            assert abs(m[h, I, J] - float(fr)) < 1e-15
    for (tau, I), want in sel_want.items():
        count, idx = oracle.select(m, tau)
        for h in range(4):
            assert idx[h, I, :count[h, I]].tolist() == want


@pytest.mark.parametrize("L,B,S", [(64, 8, 4), (128, 16, 2), (256, 32, 8), (96, 32, 32)])
def test_uniform_keys_closed_form(L, B, S):
    """All-zero keys: P[i,j] = 1/(i+1); M[I,J] = sum of 1/(i+1) over the block (exact fractions)."""
    r, Nb = B // S, L // B
    Q = _rand((L, 2, 4), 4)
    M = oracle.block_mass(Q, np.zeros((L, 1, 4)), B, S)
    for I in range(Nb):
        for J in range(Nb):
            want = sum((Fraction(1, i + 1) for i in range(I * r, I * r + r)
                        for j in range(J * r, J * r + r) if j <= i), Fraction(0))
            assert abs(M[0, I, J] - float(want)) < 1e-13
            assert abs(M[1, I, J] - float(want)) < 1e-13


@pytest.mark.parametrize("H,Hkv,B", [(2, 1, 32), (4, 2, 16), (3, 3, 64)])
def test_stride1_equals_exact_block_mass(H, Hkv, B):
    """S = 1: the block scores are the exact full-attention block mass (1/B) sum A[q,k]."""
    L, d = 256, 16
    Q, K = _rand((L, H, d), 5), _rand((L, Hkv, d), 6) * 1.5
    m = oracle.normalise_mass(oracle.block_mass(Q, K, B, 1))
    A = _sdpa_probs(Q, K)                                   # [H, L, L]
    Nb = L // B
    exact = A.reshape(H, Nb, B, Nb, B).sum(axis=(2, 4)) / B
    tri = np.tri(Nb, dtype=bool)
    assert np.max(np.abs(np.where(tri, m - exact, 0.0))) < 1e-12


def test_mass_rows_sum_to_one_and_nonnegative():
    cfg = gen.CONFIGS["tiny"]
    q, k, _ = gen.make_config(cfg)
    Q, K = gen.bf16_bits_to_f64(q), gen.bf16_bits_to_f64(k)
    M = oracle.block_mass(Q, K, cfg.B, cfg.S)
    r = cfg.B // cfg.S
    assert np.all(M >= 0)
    assert np.allclose(M.sum(axis=2), r, atol=1e-12)       # each sampled row carries mass 1
    assert np.all(np.triu(M[0], 1) == 0)


# ------------------------------------------------------------- Top-tau rules
def _dirichlet_rows(n_rows, Nb, seed, conc=0.3):
    rng = np.random.default_rng(seed)
    m = np.zeros((1, Nb, Nb))
    for I in range(Nb):
        m[0, I, :I + 1] = rng.dirichlet(np.full(I + 1, conc))
    return m


@pytest.mark.parametrize("tau", [0.3, 0.9, 0.95, 0.99])
def test_top_tau_mass_minimality_protection(tau):
    Nb = 40
    m = _dirichlet_rows(1, Nb, 7)
    count, idx = oracle.select(m, tau)
    for I in range(Nb):
        sel = idx[0, I, :count[0, I]]
        assert 1 <= count[0, I] <= I + 1
        assert np.all(np.diff(sel) > 0) and sel[-1] <= I
        if I == Nb - 1:
            assert sel.tolist() == list(range(Nb))           # last query block always dense
            continue
        tot = m[0, I, sel].sum()
        assert tot >= tau - 1e-12                              # selected mass reaches tau
        smallest = sel[np.argmin(m[0, I, sel])]
        assert tot - m[0, I, smallest] < tau                   # dropping one block falls short


@pytest.mark.parametrize("tau", [0.5, 0.8, 0.95])
def test_top_tau_brute_force(tau):
    """Enumerate every subset of each row (n <= 12): no smaller set reaches tau, and the
    selected set has the largest mass among sets of its size."""
    Nb = 13
    m = _dirichlet_rows(1, Nb, 11, conc=0.5)
    count, idx = oracle.select(m, tau)
    for I in range(Nb - 1):
        n = I + 1
        vals = m[0, I, :n]
        bits = np.array(list(itertools.product([0, 1], repeat=n)), dtype=np.float64)
        sums = bits @ vals
        sizes = bits.sum(axis=1)
        ok = sums >= tau
        kmin = int(sizes[ok].min())
        assert count[0, I] == kmin
        sel_mass = vals[idx[0, I, :kmin]].sum()
        assert abs(sel_mass - sums[sizes == kmin].max()) < 1e-12


def test_top_tau_ties_prefer_lower_block():
    m = np.zeros((1, 5, 5))
    m[0, 3, :4] = [0.2, 0.3, 0.3, 0.2]
    count, idx = oracle.select(m, 0.5)
    assert idx[0, 3, :count[0, 3]].tolist() == [1, 2]
    count, idx = oracle.select(m, 0.3)
    assert idx[0, 3, :count[0, 3]].tolist() == [1]
    m[0, 2, :3] = [0.25, 0.5, 0.25]
    count, idx = oracle.select(m, 0.7)
    assert idx[0, 2, :count[0, 2]].tolist() == [0, 1]


def test_top_tau_reaching_tau_exactly_stops():
    """"Reaches tau" is >=: a prefix whose mass equals tau is complete."""
    m = np.zeros((1, 4, 4))
    m[0, 2, :3] = [0.25, 0.25, 0.5]
    count, idx = oracle.select(m, 0.5)
    assert idx[0, 2, :count[0, 2]].tolist() == [2]


def test_tau_one_selects_all_causal_blocks():
    m = _dirichlet_rows(1, 17, 3)
    count, idx = oracle.select(m, 1.0)
    c2, i2 = oracle.full_causal_mask(1, 17)
    assert np.array_equal(count, c2) and np.array_equal(idx, i2)


# ------------------------------------------------------------ sparse attention
@pytest.mark.parametrize("H,Hkv,d,B", [(2, 1, 16, 32), (4, 4, 64, 64), (4, 2, 32, 16)])
def test_tau_one_equals_dense_causal_attention(H, Hkv, d, B):
    L = 256
    Q, K, V = _rand((L, H, d), 20), _rand((L, Hkv, d), 21), _rand((L, Hkv, d), 22)
    count, idx = oracle.full_causal_mask(H, L // B)
    O = oracle.sparse_attention(Q, K, V, count, idx, B)
    ref = _sdpa(Q, K, V, causal=True)
    assert np.max(np.abs(O - ref)) < 1e-12


def test_sparse_attention_equals_masked_sdpa():
    L, H, Hkv, d, B = 256, 4, 2, 16, 32
    Nb = L // B
    rng = np.random.default_rng(30)
    Q, K, V = _rand((L, H, d), 31), _rand((L, Hkv, d), 32), _rand((L, Hkv, d), 33)
    count = np.zeros((H, Nb), np.int32)
    idx = np.full((H, Nb, Nb), -1, np.int32)
    allowed = np.zeros((H, L, L), dtype=bool)
    for h in range(H):
        for I in range(Nb):
            sel = np.nonzero(rng.random(I + 1) < 0.5)[0]
            if sel.size == 0:
                sel = np.array([rng.integers(0, I + 1)])
            count[h, I] = sel.size
            idx[h, I, :sel.size] = sel
            for J in sel:
                allowed[h, I * B:(I + 1) * B, J * B:(J + 1) * B] = True
    allowed &= np.tri(L, dtype=bool)[None]
    O = oracle.sparse_attention(Q, K, V, count, idx, B)
    ref = _sdpa(Q, K, V, mask=allowed)
    assert np.max(np.abs(O - ref)) < 1e-12


def test_sparse_attention_row_subset_matches_full():
    L, H, d, B = 128, 2, 8, 32
    Q, K, V = _rand((L, H, d), 40), _rand((L, H, d), 41), _rand((L, H, d), 42)
    count, idx = oracle.full_causal_mask(H, L // B)
    full = oracle.sparse_attention(Q, K, V, count, idx, B)
    part = oracle.sparse_attention(Q, K, V, count, idx, B, rows=[(1, 2)])
    assert np.array_equal(part[64:96, 1], full[64:96, 1])
    assert np.isnan(part[0, 0, 0])


# ------------------------------------------------------------ whole search
def test_rr_search_tiny_invariants():
    cfg = gen.CONFIGS["tiny"]
    q, k, _ = gen.make_config(cfg)
    Q, K = gen.bf16_bits_to_f64(q), gen.bf16_bits_to_f64(k)
    count, idx, m = oracle.rr_search(Q, K, cfg.B, cfg.S, cfg.tau)
    Nb = cfg.L // cfg.B
    assert np.all(count[:, -1] == Nb)
    for h in range(cfg.H):
        for I in range(Nb - 1):
            sel = idx[h, I, :count[h, I]]
            assert m[h, I, sel].sum() >= cfg.tau - 1e-12
    # a mass-ordered selection is a subset of the mask for any larger tau
    c2, i2 = oracle.select(m, 0.99)
    for h in range(cfg.H):
        for I in range(Nb):
            assert set(idx[h, I, :count[h, I]]) <= set(i2[h, I, :c2[h, I]])


def test_band_blocks_flags_the_cut():
    m = np.array([0.5, 0.44995, 0.05005])
    near, ties = oracle.band_blocks(m, 2, 0.95)
    assert 1 in near                                     # running sum 0.94995 sits at tau
    near, ties = oracle.band_blocks(np.array([0.6, 0.2, 0.2]), 2, 0.7)
    assert ties == {1, 2}


# ------------------------------------------------------------ mask diagnostics
def test_recall_of_full_mask_is_one_and_top_tau_reaches_tau():
    L, H, Hkv, d, B = 256, 2, 1, 16, 32
    Q, K = _rand((L, H, d), 50), _rand((L, Hkv, d), 51) * 2.0
    M = oracle.exact_block_mass(Q, K, B)
    Nb = L // B
    c_full, i_full = oracle.full_causal_mask(H, Nb)
    assert np.allclose(oracle.mask_recall(M, c_full, i_full), 1.0, atol=1e-12)
    for tau in (0.3, 0.8, 0.95):
        c, i = oracle.select(oracle.normalise_mass(M), tau)
        rec = oracle.mask_recall(M, c, i)
        assert np.all(rec[:, :-1] >= tau - 1e-12)          # Top-tau of the exact mass reaches tau
        assert np.allclose(rec[:, -1], 1.0)                  # protected last row


def test_recall_of_single_block_equals_its_exact_share():
    L, H, d, B = 128, 1, 8, 32
    Q, K = _rand((L, H, d), 52), _rand((L, H, d), 53)
    A = _sdpa_probs(Q, K)[0]                                # exact attention probabilities
    M = oracle.exact_block_mass(Q, K, B)
    count = np.ones((1, 4), np.int32)
    idx = np.zeros((1, 4, 4), np.int32)                      # keep only J = 0 in every row
    rec = oracle.mask_recall(M, count, idx)
    for I in range(4):
        want = A[I * B:(I + 1) * B, 0:B].sum() / B
        assert abs(rec[0, I] - want) < 1e-12


# ------------------------------------------------------------ sampling variants
@pytest.mark.parametrize("L,H,S", [(1024, 4, 4), (4096, 32, 16), (512, 3, 8)])
def test_rotated_positions_rotate_across_strides(L, H, S):
    p = oracle.rotated_positions(L, H, S)
    Ns = L // S
    i = np.arange(Ns)
    for h in range(H):
        off = p[h] - i * S
        assert np.all((off >= 0) & (off < S))
        assert np.array_equal(off, (h + i) % S)
        # over S consecutive strides every head visits every offset once
        for a in range(0, Ns - S + 1, S):
            assert sorted(off[a:a + S].tolist()) == list(range(S))
    if H >= S:
        for i0 in range(min(Ns, 8)):
            assert sorted((p[:S, i0] - i0 * S).tolist()) == list(range(S))


def test_sampled_keys_equal_mean_keys_when_strides_are_constant():
    L, H, Hkv, d, B, S = 256, 4, 2, 16, 32, 4
    Q = _rand((L, H, d), 60)
    K = np.repeat(_rand((L // S, Hkv, d), 61), S, axis=0)       # keys constant inside each stride
    for rotate in (False, True):
        a = oracle.block_mass(Q, K, B, S, rotate=rotate)
        b = oracle.block_mass(Q, K, B, S, rotate=rotate, mean_keys=True)
        assert np.max(np.abs(a - b)) < 1e-12


@pytest.mark.parametrize("rotate", [False, True])
def test_sampled_keys_take_the_heads_own_offset(rotate):
    """Sampled keys (R2): head h scores its sampled queries against the single key
    at its own sampled position of every stride, on its own kv head h // g.

    Every key is zero except one per query head: head h's key at its own offset
    in stride j_h (a distinct stride per head) on kv head h // g, of size
    30*sqrt(d) along e_0, and every query is e_0.  Head h then sees one logit of
    30 (at stride j_h) and zeros elsewhere, so each of its sampled rows i >= j_h
    puts all but i*e^-30 of its probability on stride j_h: the normalised mass of
    key block j_h // r is 1 to within 1e-9 in every row whose first sampled row
    is at or past j_h.  A key read at another offset (the next head's), from
    another kv head, or averaged over the stride spreads that mass."""
    L, H, Hkv, d, B, S = 512, 4, 2, 16, 32, 8
    r, Nb, Ns = B // S, L // B, L // S
    g = H // Hkv
    Q = np.zeros((L, H, d))
    Q[:, :, 0] = 1.0
    K = np.zeros((L, Hkv, d))
    j_of = {h: 9 + 11 * h for h in range(H)}                 # 9, 20, 31, 42: distinct blocks 2, 5, 7, 10
    for h in range(H):
        j = j_of[h]
        off = (h + j) % S if rotate else h % S
        K[j * S + off, h // g, 0] = 30.0 * math.sqrt(d)
    m = oracle.normalise_mass(oracle.block_mass(Q, K, B, S, rotate=rotate))
    for h in range(H):
        Jh = j_of[h] // r
        rows = [I for I in range(Nb) if I * r >= j_of[h]]
        assert rows and len(rows) >= 4
        for I in rows:
            assert m[h, I, Jh] > 1.0 - 1e-9, (h, I, m[h, I, Jh])
        # rows wholly before the planted stride see only zero keys: uniform 1/(i+1)
        for I in range(Nb):
            if (I + 1) * r - 1 < j_of[h]:
                want = np.zeros(Nb)
                for i in range(I * r, (I + 1) * r):
                    for j in range(i + 1):
                        want[j // r] += 1.0 / (i + 1)
                assert np.allclose(m[h, I], want / r, atol=1e-12)


def test_variants_at_stride_one_are_exact():
    L, H, Hkv, d, B = 256, 2, 1, 16, 32
    Q, K = _rand((L, H, d), 62), _rand((L, Hkv, d), 63)
    ref = oracle.block_mass(Q, K, B, 1)
    for rotate in (False, True):
        for mk in (False, True):
            assert np.max(np.abs(oracle.block_mass(Q, K, B, 1, rotate=rotate, mean_keys=mk) - ref)) < 1e-12


def test_gqa_group_mask_shares_lists_and_reaches_tau():
    L, H, Hkv, d, B, S, tau = 512, 4, 2, 16, 32, 4, 0.9
    Q, K = _rand((L, H, d), 64), _rand((L, Hkv, d), 65)
    count, idx, m = oracle.rr_search(Q, K, B, S, tau, gqa_mask=True)
    M = oracle.block_mass(Q, K, B, S)
    Mg = M[0] + M[1]
    assert np.allclose(oracle.normalise_mass(Mg[None])[0], m[0], atol=1e-14)
    Nb = L // B
    for kv in range(Hkv):
        for h in (2 * kv, 2 * kv + 1):
            assert np.array_equal(count[h], count[2 * kv])
            for I in range(Nb):
                assert np.array_equal(idx[h, I, :count[h, I]], idx[2 * kv, I, :count[2 * kv, I]])
        for I in range(Nb - 1):
            assert m[2 * kv, I, idx[2 * kv, I, :count[2 * kv, I]]].sum() >= tau - 1e-12
    c1, i1, _ = oracle.rr_search(Q, K.repeat(2, axis=1), B, S, tau, gqa_mask=True)   # g = 1: per-head masks
    c2, i2, _ = oracle.rr_search(Q, K.repeat(2, axis=1), B, S, tau)
    assert np.array_equal(c1, c2)
