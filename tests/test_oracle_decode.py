"""Pins of the oracle's decode stage (D1-D5) against a library routine, closed
forms and brute force, and planted mistakes that each must fail a pin.

The decode readings carry the prefill rules over to one new token per step; the
pages only name decoding-stage sparsification (sciencestack page, TL;DR).
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa_one(q, K, V, t):
    """Attention of the single query at position t over keys 0..t, from torch's
    scaled_dot_product_attention (fp64): [H, d]."""
    H, d = q.shape
    g = H // K.shape[1]
    qq = torch.from_numpy(q).reshape(H, 1, d)
    kk = torch.from_numpy(np.repeat(K[:t + 1], g, axis=1)).permute(1, 0, 2)
    vv = torch.from_numpy(np.repeat(V[:t + 1], g, axis=1)).permute(1, 0, 2)
    return F.scaled_dot_product_attention(qq, kk, vv).reshape(H, d).numpy()


def _sdpa_probs_one(q, K, t):
    """Attention probabilities of the query over keys 0..t (SDPA with V = identity)."""
    H, d = q.shape
    g = H // K.shape[1]
    qq = torch.from_numpy(q).reshape(H, 1, d)
    kk = torch.from_numpy(np.repeat(K[:t + 1], g, axis=1)).permute(1, 0, 2)
    eye = torch.eye(t + 1, dtype=torch.float64).expand(H, t + 1, t + 1)
    return F.scaled_dot_product_attention(qq, kk, eye).reshape(H, t + 1).numpy()


@pytest.mark.parametrize("t", [0, 37, 63, 64, 200, 255])
def test_tau_one_equals_dense_decode_attention(t):
    L, H, Hkv, d, B, S = 256, 4, 2, 16, 32, 4
    q, K, V = _rand((H, d), 1), _rand((L, Hkv, d), 2), _rand((L, Hkv, d), 3)
    count, sel, _, out = oracle.rr_decode(q, K, V, t, B, S, 1.0)
    assert np.array_equal(count, np.full(H, t // B + 1))
    assert np.allclose(out, _sdpa_one(q, K, V, t), atol=1e-12)


@pytest.mark.parametrize("t", [5, 100, 255])
def test_stride_one_mass_equals_exact_attention_mass(t):
    """S = 1: every key is sampled, so the block mass is the query's exact
    attention mass per key block."""
    L, H, Hkv, d, B = 256, 4, 2, 16, 32
    q, K = _rand((H, d), 4), _rand((L, Hkv, d), 5)
    M = oracle.decode_block_mass(q, K, t, B, 1)
    A = _sdpa_probs_one(q, K, t)
    want = np.zeros_like(M)
    for J in range(t // B + 1):
        want[:, J] = A[:, J * B:min((J + 1) * B, t + 1)].sum(axis=1)
    assert np.allclose(M, want, atol=1e-12)


def test_planted_key_at_the_heads_own_offset():
    """One key per head at that head's own offset in a stride of its own, on its
    own kv head, of logit 30; every other key zero.  The head's mass sits on the
    planted block to within 1e-9; a key at another offset, on another kv head, or
    averaged over the stride would spread it."""
    L, H, Hkv, d, B, S = 512, 4, 2, 16, 32, 8
    t = L - 1
    g, r = H // Hkv, B // S
    q = np.zeros((H, d))
    q[:, 0] = 1.0
    K = np.zeros((L, Hkv, d))
    j_of = {h: 9 + 11 * h for h in range(H)}
    for h in range(H):
        K[j_of[h] * S + h % S, h // g, 0] = 30.0 * math.sqrt(d)
    M = oracle.decode_block_mass(q, K, t, B, S)
    for h in range(H):
        assert M[h, j_of[h] // r] > 1.0 - 1e-9, (h, M[h])


def test_keys_sampled_past_the_query_do_not_count():
    """The current stride's sampled position may lie after t: that key must not
    enter the scores (a huge key there would otherwise take all the mass)."""
    L, H, Hkv, d, B, S = 128, 4, 1, 8, 32, 8
    t = 50                                   # stride 6 covers 48..55; heads sample 48 + (h mod 8)
    q = np.zeros((H, d))
    q[:, 0] = 1.0
    K = np.zeros((L, Hkv, d))
    K[51, 0, 0] = 1e3                        # head 3 would sample 51 > t
    K[53, 0, 0] = 1e3                        # (no head samples 53 here: offsets 0..3)
    M = oracle.decode_block_mass(q, K, t, B, S)
    # every sampled key at or before t is zero: the mass is uniform over the sampled strides
    for h in range(H):
        pos = oracle.decode_positions(t, h, S)
        assert pos.max() <= t
        want = np.zeros(t // B + 1)
        np.add.at(want, pos // B, 1.0 / pos.size)
        assert np.allclose(M[h], want, atol=1e-12), h
    assert oracle.decode_positions(50, 3, S).max() == 43
    assert oracle.decode_positions(51, 3, S).max() == 51


def test_query_before_its_heads_first_sample():
    """t < (h mod S): the head samples no key; its mass row is zero and only the
    current block is kept."""
    L, H, Hkv, d, B, S = 64, 4, 1, 8, 32, 4
    q, K, V = _rand((H, d), 6), _rand((L, Hkv, d), 7), _rand((L, Hkv, d), 8)
    t = 1
    count, sel, M, out = oracle.rr_decode(q, K, V, t, B, S, 0.9)
    for h in (2, 3):
        assert M[h].sum() == 0.0 and list(sel[h]) == [0]
    assert np.allclose(out, _sdpa_one(q, K, V, t), atol=1e-12)   # block 0 holds every key <= t


@pytest.mark.parametrize("tau", [0.3, 0.7, 0.9])
def test_selection_brute_force_and_current_block(tau):
    """Per head: the kept set is the shortest (mass desc, J asc) prefix reaching
    tau plus the current block; no smaller set of blocks reaches tau."""
    L, H, Hkv, d, B, S = 384, 4, 2, 16, 32, 4
    rng = np.random.default_rng(9)
    q, K = 2.0 * rng.standard_normal((H, d)), rng.standard_normal((L, Hkv, d))
    t = 370
    Jt = t // B
    M = oracle.decode_block_mass(q, K, t, B, S)
    for h in range(H):
        sel = oracle.decode_select(M[h], Jt, tau)
        assert Jt in sel and np.all(np.diff(sel) > 0)
        m = M[h] / M[h].sum()
        order = oracle.sorted_order(m)
        k = int(np.nonzero(np.cumsum(m[order]) >= tau)[0][0]) + 1
        assert set(sel) == set(order[:k].tolist()) | {Jt}
        best = min(len(c) for n in range(1, Jt + 2) for c in itertools.combinations(range(Jt + 1), n)
                   if m[list(c)].sum() >= tau)
        assert best == k
        assert m[sel].sum() >= tau


def test_decode_row_matches_prefill_row_when_the_query_is_sampled():
    """With B = S a query block holds one sampled row.  When t is head h's sampled
    position in stride i (t = i*S + h mod S), the decode scores are that row's
    prefill scores, so the decode mass equals the prefill block mass of row i."""
    L, H, Hkv, d, S = 256, 4, 2, 16, 8
    B = S
    Q, K = _rand((L, H, d), 10), _rand((L, Hkv, d), 11)
    Mp = oracle.block_mass(Q, K, B, S)
    for h in range(H):
        for i in (3, 17, 31):
            t = i * S + h % S
            Md = oracle.decode_block_mass(Q[t][None, h].copy().reshape(1, d).repeat(H, axis=0), K, t, B, S)
            assert np.allclose(Md[h], Mp[h, i, :i + 1], atol=1e-12), (h, i)


def test_group_mask_shares_lists_and_reaches_tau():
    """V3 for decode: every head of a GQA group gets the list selected on the
    group's summed mass; it reaches tau of that mass, keeps the current block,
    and with one head per group it is the per-head list."""
    L, H, Hkv, d, B, S, tau = 512, 8, 2, 16, 32, 4, 0.8
    rng = np.random.default_rng(12)
    q, K, V = 2.0 * rng.standard_normal((H, d)), rng.standard_normal((L, Hkv, d)), rng.standard_normal((L, Hkv, d))
    t = 450
    Jt = t // B
    count, sel, Mg, _ = oracle.rr_decode(q, K, V, t, B, S, tau, gqa_mask=True)
    M = oracle.decode_block_mass(q, K, t, B, S)
    g = H // Hkv
    for c in range(Hkv):
        grp = M[c * g:(c + 1) * g].sum(axis=0)
        for h in range(c * g, (c + 1) * g):
            assert np.array_equal(sel[h], sel[c * g])
            assert np.allclose(Mg[h], grp, atol=1e-14)
        m = grp / grp.sum()
        assert Jt in sel[c * g] and m[sel[c * g]].sum() >= tau
    # one head per group: the group mask is the per-head mask
    K8 = np.repeat(K, 4, axis=1)
    c1, s1, _, o1 = oracle.rr_decode(q, K8, np.repeat(V, 4, axis=1), t, B, S, tau, gqa_mask=True)
    c2, s2, _, o2 = oracle.rr_decode(q, K8, np.repeat(V, 4, axis=1), t, B, S, tau)
    assert all(np.array_equal(a, b) for a, b in zip(s1, s2)) and np.allclose(o1, o2)


def test_group_mask_groups_the_heads_of_each_kv_head():
    """Planted keys: each head's mass sits on a block of its own (one key per
    head at that head's own offset, on its own kv head, logit 30).  With one
    list per GQA group and tau = 0.9, a group's list must hold exactly the
    planted blocks of the heads that share its kv head (each carries 1/g of the
    group mass) and the current block; grouping other heads together, or
    selecting on one head's mass, gives other sets."""
    L, H, Hkv, d, B, S = 1024, 6, 3, 16, 32, 8
    t = L - 1
    g, r = H // Hkv, B // S
    q = np.zeros((H, d))
    q[:, 0] = 1.0
    K = np.zeros((L, Hkv, d))
    j_of = {h: 3 + 11 * h for h in range(H)}
    for h in range(H):
        K[j_of[h] * S + h % S, h // g, 0] = 30.0 * math.sqrt(d)
    V = np.zeros((L, Hkv, d))
    _, sel, _, _ = oracle.rr_decode(q, K, V, t, B, S, 0.9, gqa_mask=True)
    for h in range(H):
        c = h // g
        want = {j_of[u] // r for u in range(c * g, (c + 1) * g)} | {t // B}
        assert set(sel[h].tolist()) == want, (h, sel[h], want)


# ------------------------------------------------------------ planted mistakes
_orig = {n: getattr(oracle, n) for n in ("decode_positions", "decode_select", "decode_attention",
                                         "decode_group_mass")}


def _positions_past_t(t, h, S):
    off = h % S
    return np.arange((t - off) // S + 2, dtype=np.int64) * S + off if t >= off else np.zeros(0, np.int64)


def _select_unprotected(m_row, Jt, tau):
    sel = [j for j in _orig["decode_select"](m_row, Jt, tau).tolist()]
    m = m_row[:Jt + 1]
    if Jt in sel and len(sel) > 1:
        # drop the protection when the prefix alone did not need it
        order = oracle.sorted_order(m)
        run = np.cumsum(m[order] / m.sum())
        k = int(np.nonzero(run >= tau)[0][0]) + 1
        if Jt not in order[:k].tolist():
            sel.remove(Jt)
    return np.array(sel, dtype=np.int32)


def _attention_whole_block(q, K, V, t, blocks, B):
    H, d = q.shape
    g = H // K.shape[1]
    out = np.zeros((H, d))
    for h in range(H):
        b = np.asarray(blocks[h], dtype=np.int64)
        keys = (b[:, None] * B + np.arange(B)[None, :]).reshape(-1)
        keys = keys[keys < K.shape[0]]
        s = (K[keys, h // g, :] @ q[h]) / math.sqrt(d)
        p = np.exp(s - s.max())
        out[h] = (p / p.sum()) @ V[keys, h // g, :]
    return out


def _group_mass_by_modulo(M, Hkv):
    H, n = M.shape
    g = H // Hkv
    out = np.zeros_like(M)
    for h in range(H):
        out[h] = M[[u for u in range(H) if u % Hkv == h % Hkv]].sum(axis=0)
    return out


def _group_mass_first_head(M, Hkv):
    H, n = M.shape
    g = H // Hkv
    return np.repeat(M[::g], g, axis=0)


DECODE_PINS = [
    lambda: test_tau_one_equals_dense_decode_attention(37),
    lambda: test_stride_one_mass_equals_exact_attention_mass(100),
    test_planted_key_at_the_heads_own_offset,
    test_keys_sampled_past_the_query_do_not_count,
    test_query_before_its_heads_first_sample,
    lambda: test_selection_brute_force_and_current_block(0.7),
    test_group_mask_groups_the_heads_of_each_kv_head,
]

DECODE_MUTANTS = {
    "sampled key past the query counted": ("decode_positions", _positions_past_t),
    "offset h instead of h mod S": ("decode_positions", lambda t, h, S: np.arange(max(t - h, -1) // S + 1,
                                                                                  dtype=np.int64) * S + h
                                    if t >= h else np.zeros(0, np.int64)),
    "current block not protected": ("decode_select", _select_unprotected),
    "attention reads keys past the query": ("decode_attention", _attention_whole_block),
    "group mask groups heads by h mod Hkv": ("decode_group_mass", _group_mass_by_modulo),
    "group mask selects on the group's first head only": ("decode_group_mass", _group_mass_first_head),
}


@pytest.mark.parametrize("name", list(DECODE_MUTANTS))
def test_decode_mutant_is_caught(name, monkeypatch):
    attr, fn = DECODE_MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    failed = 0
    for pin in DECODE_PINS:
        try:
            pin()
        except Exception:
            failed += 1
    assert failed > 0, f"no pin catches: {name}"


def test_unmutated_decode_oracle_passes_every_pin():
    for pin in DECODE_PINS:
        pin()
