"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Each case patches one oracle function with a plausible slip (a dropped term, a
wrong index or sign, a transposed reduction) and runs the pins of
test_oracle.py against the patched module.
"""
import math

import numpy as np
import pytest

import oracle
import tests.test_oracle as pins

_orig = {name: getattr(oracle, name) for name in
         ("sampled_positions", "pool_keys", "block_mass", "top_tau_row", "sparse_attention_block",
          "sorted_order")}


def _no_shift(L, H, S):
    Ns = L // S
    return np.stack([np.arange(Ns) * S for _ in range(H)])


def _head_not_mod(L, H, S):
    Ns = L // S
    return np.stack([np.arange(Ns) * S + h for h in range(H)])


def _pool_sum(K, S):
    L, Hkv, d = K.shape
    return K.reshape(L // S, S, Hkv, d).sum(axis=1)


def _mass_variant(strict_causal=False, no_scale=False, swap=False):
    def block_mass(Q, K, B, S, row_chunk=2048, rotate=False, mean_keys=False):
        L, H, d = Q.shape
        g = H // K.shape[1]
        Ns, Nb, r = L // S, L // B, B // S
        pos = oracle.sampled_positions(L, H, S)
        scale = 1.0 if no_scale else 1.0 / math.sqrt(d)
        M = np.zeros((H, Nb, Nb))
        for h in range(H):
            s = (Q[pos[h], h, :] @ K[pos[h], h // g, :].T) * scale
            i, j = np.arange(Ns)[:, None], np.arange(Ns)[None, :]
            s = np.where((j < i) | ((j == i) & (i == 0)) if strict_causal else (j <= i), s, -np.inf)
            P = np.exp(s - s.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            blk = P.reshape(Nb, r, Nb, r).sum(axis=(1, 3))
            M[h] = blk.T if swap else blk
        return M
    return block_mass


def _sampled_keys_variant(offset_shift=0, kv_by_q_head=False, mean=False):
    """block_mass whose sampled-key side (R2) takes the key at the head's offset
    + offset_shift, or on kv head h instead of h // g, or averages the stride."""
    orig = _orig["block_mass"]

    def block_mass(Q, K, B, S, row_chunk=2048, rotate=False, mean_keys=False):
        if mean_keys:
            return orig(Q, K, B, S, row_chunk=row_chunk, rotate=rotate, mean_keys=True)
        L, H, d = Q.shape
        g = H // K.shape[1]
        Ns, Nb, r = L // S, L // B, B // S
        pos = oracle.rotated_positions(L, H, S) if rotate else oracle.sampled_positions(L, H, S)
        Kbar = oracle.pool_keys(K, S)
        M = np.zeros((H, Nb, Nb))
        for h in range(H):
            kv = h if kv_by_q_head else h // g
            kpos = np.arange(Ns) * S + (pos[h] - np.arange(Ns) * S + offset_shift) % S
            Kb = Kbar[:, kv, :] if mean else K[kpos, kv, :]
            s = (Q[pos[h], h, :] @ Kb.T) / math.sqrt(d)
            i, j = np.arange(Ns)[:, None], np.arange(Ns)[None, :]
            s = np.where(j <= i, s, -np.inf)
            P = np.exp(s - s.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            M[h] = P.reshape(Nb, r, Nb, r).sum(axis=(1, 3))
        return M
    return block_mass


def _top_tau_strict(m_row, I, Nb, tau):
    n = I + 1
    if tau >= 1.0 or I == Nb - 1:
        return np.arange(n, dtype=np.int32)
    order = oracle.sorted_order(m_row[:n])
    run = np.cumsum(m_row[:n][order])
    hit = np.nonzero(run > tau)[0]
    k = int(hit[0]) + 1 if hit.size else n
    return np.sort(order[:k]).astype(np.int32)


def _top_tau_unprotected(m_row, I, Nb, tau):
    return _orig["top_tau_row"](m_row, I, Nb + 1, tau)


def _order_ties_high(m_row):
    n = m_row.shape[0]
    return np.lexsort((-np.arange(n), -m_row))


def _attn_variant(no_causal=False, kv_mod=False):
    def sparse_attention_block(Q, K, V, h, I, blocks, B):
        L, H, d = Q.shape
        Hkv = K.shape[1]
        kv = h % Hkv if kv_mod else h // (H // Hkv)
        blocks = np.asarray(blocks, dtype=np.int64)
        keys = (blocks[:, None] * B + np.arange(B)[None, :]).reshape(-1)
        q_pos = I * B + np.arange(B)
        s = (Q[q_pos, h, :] @ K[keys, kv, :].T) / math.sqrt(d)
        if not no_causal:
            s = np.where(keys[None, :] <= q_pos[:, None], s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        return (p / p.sum(axis=1, keepdims=True)) @ V[keys, kv, :]
    return sparse_attention_block


ALL_PINS = [
    pins.test_sampling_fig2_fixture,
    lambda: pins.test_sampling_round_robin_properties(1024, 32, 16),
    pins.test_pool_keys_closed_forms,
    pins.test_uniform_keys_fig2_fixture,
    lambda: pins.test_uniform_keys_closed_form(128, 16, 2),
    lambda: pins.test_stride1_equals_exact_block_mass(4, 2, 16),
    lambda: pins.test_top_tau_mass_minimality_protection(0.9),
    lambda: pins.test_top_tau_brute_force(0.8),
    pins.test_top_tau_ties_prefer_lower_block,
    pins.test_top_tau_reaching_tau_exactly_stops,
    lambda: pins.test_tau_one_equals_dense_causal_attention(4, 2, 32, 16),
    pins.test_sparse_attention_equals_masked_sdpa,
    lambda: pins.test_sampled_keys_take_the_heads_own_offset(False),
    lambda: pins.test_sampled_keys_take_the_heads_own_offset(True),
]

MUTANTS = {
    "sampling without head shift": ("sampled_positions", _no_shift),
    "sampling shift h instead of h mod S": ("sampled_positions", _head_not_mod),
    "pooling sums instead of averaging": ("pool_keys", _pool_sum),
    "diagonal stride dropped": ("block_mass", _mass_variant(strict_causal=True)),
    "softmax scale dropped": ("block_mass", _mass_variant(no_scale=True)),
    "block reduction transposed": ("block_mass", _mass_variant(swap=True)),
    "top-tau compares with >": ("top_tau_row", _top_tau_strict),
    "last block not protected": ("top_tau_row", _top_tau_unprotected),
    "ties go to the higher block": ("sorted_order", _order_ties_high),
    "causal mask dropped in attention": ("sparse_attention_block", _attn_variant(no_causal=True)),
    "GQA head mapped with mod": ("sparse_attention_block", _attn_variant(kv_mod=True)),
    "sampled key one offset late": ("block_mass", _sampled_keys_variant(offset_shift=1)),
    "sampled key one offset early": ("block_mass", _sampled_keys_variant(offset_shift=-1)),
    "sampled key from the q head's index": ("block_mass", _sampled_keys_variant(kv_by_q_head=True)),
    "sampled key replaced by the stride mean": ("block_mass", _sampled_keys_variant(mean=True)),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    failed = 0
    for pin in ALL_PINS:
        try:
            pin()
        except Exception:  # an assertion, or a crash on the slipped index
            failed += 1
    assert failed > 0, f"no pin catches: {name}"


def test_unmutated_oracle_passes_every_pin():
    for pin in ALL_PINS:
        pin()
