"""fp64 CPU oracle for the RRAttention prefill operator.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path (``dynamic_block_sparse_rr_b200``) and the CUDA path never calls it.

It restates, plainly and slowly, what the method computes.  The source is the
RRAttention pages (sciencestack.ai page of "RRAttention: Dynamic Block Sparse
Attention via Per-Head Round-Robin Shifts for Long-Context Inference": Abstract,
TL;DR, Figure 2 and Figure 3 captions; the taxoreview, paperdot and fugumt pages
repeat the same abstract).  The pages carry no equations and no algorithm box,
so every definition below is the plainest reading of that text, stated in our
own words.  The readings:

R1  Sampling (Abstract: the sampled query position rotates from head to head
    inside every stride; title: per-head round-robin shifts).  Head h samples,
    in stride i, the position p(h, i) = i*S + (h mod S).  The shift is fixed per
    head; it does not rotate across strides.
R2  Stride-level keys (Abstract: the method is a sampling strategy, and that
    sampling is what lowers the search cost to O(L^2/S^2)).  Head h reads the
    key side of stride j at its own sampled position too: the key at
    p(h, j) = j*S + (h mod S) of its kv head.  Every score is then the logit of a
    real (query, key) token pair, and each head's search is causal attention
    over its own strided subsequence.  Across S heads every offset of every
    stride is seen.                                           [parity unpinned
    for S > 1 beyond the pins listed below]
R3  Scores.  s[h,i,j] = Q[p(h,i), h] . K[p(h,j), h/g] / sqrt(d) for stride-causal
    j <= i (the diagonal stride is included, so a row is never empty).
R4  Each sampled row is a softmax over its j <= i.
R5  Block mass (Abstract: stride-level scores aggregated to B x B blocks;
    Figure 2, stages 1-2).  A query block I holds the r = B/S sampled rows i
    with i*S in I, a key block J the r strides j with j*S in J.
    M[h,I,J] = sum_{i in I} sum_{j in J} P[h,i,j], normalised per row:
    m[h,I,J] = M[h,I,J] / sum_{J' <= I} M[h,I,J'].
R6  Adaptive Top-tau (Abstract; TL;DR).  For each row I < Nb-1: order J in
    [0, I] by (m descending, J ascending), keep the shortest prefix whose
    running sum is >= tau (the selected share reaches tau).  tau >= 1 keeps
    every J <= I.
R7  The last query block is protected (TL;DR): row I = Nb-1 keeps every
    J <= Nb-1, for every tau.  No other block is forced.
R8  Block-sparse causal attention (Abstract: only the selected blocks, about
    half of them on the pages' workloads, are computed).  Query q in block I
    attends, with softmax scale 1/sqrt(d), to every key k <= q that lies in a
    selected block of row I.
V1-V3 Alternatives the pages leave open (off by default): V1 rotates the
    sampled offset across strides too, p(h, i) = i*S + ((h + i) mod S), on both
    sides; V2 (mean_keys) replaces the sampled key of stride j by the mean of
    the stride's S keys, Kbar[j] = (1/S) sum_{t<S} K[j*S+t], which costs the
    same O(L^2/S^2) but blurs per-token structure; V3 keeps one mask per GQA
    group, selecting on the summed block mass of the group's heads.
                                                              [parity unpinned
    beyond the invariants in tests/test_oracle.py]
D1-D5 Decode stage.  The TL;DR names decoding-stage sparsification only as a
    future extension, so every definition here is a reading that carries the
    prefill rules over to one new token per step.  The query at position t
    (cache keys 0..t, its own key included):
    D1  head h scores the keys at its own sampled positions p(h, j) =
        j*S + (h mod S) that lie at or before t (R1-R2 on the key side);
    D2  s_j = q . K[p(h,j), h/g] / sqrt(d), softmax over those j;
    D3  block mass M[J] = sum of P_j over the strides j of block J, J <= J_t =
        floor(t/B) (a block with no sampled key at or before t has mass 0);
    D4  Top-tau over J <= J_t as R6, and the current block J_t is always kept
        (the prefill rule R7 keeps the whole last query block dense; carried
        over literally it would make every decode step dense, so the decode
        reading keeps only the block that holds the query and the newest keys);
    D5  the query attends, with scale 1/sqrt(d), to every key k <= t in the
        selected blocks.                                       [parity unpinned
    against the paper: the pages do not describe decoding]
R9  Mask comparison band (tolerance of the operator's specification): a block
    is near-threshold when the running sum just before or just after it, in
    the R6 order, lies within `band` of tau; a near-tie is a pair of blocks at
    the cut whose masses differ by less than `tie`.

Pins (tests/test_oracle.py): R8 against torch's scaled_dot_product_attention in
fp64 (tau = 1 and arbitrary block masks); R1-R5 at S = 1 against the exact
full-attention block mass from the attention matrix that scaled_dot_product_
attention returns; R3-R5 with all-zero keys against the closed form
P[i,j] = 1/(i+1) (a hand-derived fixture in the Figure 2 configuration S=4,
B=8); R2 by planted keys that only the head's own offset on its own kv head
sees; R6 against brute-force subset enumeration; R7 by inspection of every row.
That the paper samples the key side this way, rather than pooling it, is a
reading: "parity unpinned" for S > 1 against the paper itself.

All arithmetic is float64.  Inputs are the bf16 values both paths receive,
widened exactly (callers may pass them as float32 or float64 arrays; every
function widens to float64 before any arithmetic).
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------- R1 sampling
def sampled_positions(L: int, H: int, S: int) -> np.ndarray:
    """p[h, i] = i*S + (h mod S), shape [H, L/S] (R1)."""
    Ns = L // S
    i = np.arange(Ns, dtype=np.int64)
    return np.stack([i * S + (h % S) for h in range(H)])


def rotated_positions(L: int, H: int, S: int) -> np.ndarray:
    """Variant V1 (rotation across strides as well as heads): head h samples, in
    stride i, the query at i*S + ((h + i) mod S).  Shape [H, L/S]."""
    Ns = L // S
    i = np.arange(Ns, dtype=np.int64)
    return np.stack([i * S + (h + i) % S for h in range(H)])


# ------------------------------------------------------- V2 stride-mean keys
def pool_keys(K: np.ndarray, S: int) -> np.ndarray:
    """Kbar[j, kv, :] = mean over the S keys of stride j (V2).  K: [L, Hkv, d]."""
    L, Hkv, d = K.shape
    return K.astype(np.float64).reshape(L // S, S, Hkv, d).mean(axis=1)


# ------------------------------------------------------- R3-R5 block masses
def block_mass(Q: np.ndarray, K: np.ndarray, B: int, S: int, row_chunk: int = 2048,
               rotate: bool = False, mean_keys: bool = False) -> np.ndarray:
    """Unnormalised block mass M[h, I, J] (R2-R5), zero above the diagonal.

    Q: [L, H, d], K: [L, Hkv, d].  Returns [H, Nb, Nb] float64.
    Head h scores its sampled queries against the key at its own sampled
    position of every stride (R2).  Alternatives (off by default): rotate -> V1
    positions on both sides; mean_keys -> V2, the key side of stride j is the
    mean of the stride's S keys.
    """
    L, H, d = Q.shape
    Hkv = K.shape[1]
    g = H // Hkv
    Ns, Nb, r = L // S, L // B, B // S
    Kbar = pool_keys(K, S) if mean_keys else None
    pos = rotated_positions(L, H, S) if rotate else sampled_positions(L, H, S)
    scale = 1.0 / math.sqrt(d)
    M = np.zeros((H, Nb, Nb), dtype=np.float64)
    step = max(r, (row_chunk // r) * r)
    for h in range(H):
        Qs = Q[pos[h], h, :].astype(np.float64)  # [Ns, d] real sampled queries
        if mean_keys:
            Kb = Kbar[:, h // g, :]                  # [Ns, d] stride means (V2)
        else:
            Kb = K[pos[h], h // g, :].astype(np.float64)   # [Ns, d] one real key per stride (R2)
        for a in range(0, Ns, step):
            b = min(Ns, a + step)
            s = (Qs[a:b] @ Kb[:b].T) * scale     # rows i in [a,b), strides j < b
            i_idx = np.arange(a, b)[:, None]
            j_idx = np.arange(b)[None, :]
            s = np.where(j_idx <= i_idx, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            P = np.exp(s)
            P = P / P.sum(axis=1, keepdims=True)   # R4
            nI, nJ = (b - a) // r, b // r
            M[h, a // r:a // r + nI, :nJ] += P.reshape(nI, r, nJ, r).sum(axis=(1, 3))
    return M


def group_mass(M: np.ndarray, Hkv: int) -> np.ndarray:
    """Variant V3 (one mask per GQA group): the block masses of the g query heads
    of each kv head summed, repeated for every head of the group.  [H, Nb, Nb]."""
    H, Nb, _ = M.shape
    g = H // Hkv
    Mg = M.reshape(Hkv, g, Nb, Nb).sum(axis=1)
    return np.repeat(Mg, g, axis=0)


def normalise_mass(M: np.ndarray) -> np.ndarray:
    """m[h, I, J] = M[h, I, J] / sum_{J' <= I} M[h, I, J'] (R5); zero above the diagonal."""
    H, Nb, _ = M.shape
    tri = np.tril(np.ones((Nb, Nb), dtype=bool))
    Mt = np.where(tri[None], M, 0.0)
    return Mt / Mt.sum(axis=2, keepdims=True)


# ---------------------------------------------------------- R6/R7 selection
def sorted_order(m_row: np.ndarray) -> np.ndarray:
    """J order by mass descending, then J ascending (R6)."""
    n = m_row.shape[0]
    return np.lexsort((np.arange(n), -m_row))


def top_tau_row(m_row: np.ndarray, I: int, Nb: int, tau: float) -> np.ndarray:
    """Selected key blocks of row I, ascending (R6, R7).  m_row: masses of J = 0..I."""
    n = I + 1
    if tau >= 1.0 or I == Nb - 1:
        return np.arange(n, dtype=np.int32)
    order = sorted_order(m_row[:n])
    run = np.cumsum(m_row[:n][order])
    hit = np.nonzero(run >= tau)[0]
    k = int(hit[0]) + 1 if hit.size else n
    return np.sort(order[:k]).astype(np.int32)


def select(m: np.ndarray, tau: float):
    """count [H, Nb] int32 and idx [H, Nb, Nb] int32 (ascending, -1 past count)."""
    H, Nb, _ = m.shape
    count = np.zeros((H, Nb), dtype=np.int32)
    idx = np.full((H, Nb, Nb), -1, dtype=np.int32)
    for h in range(H):
        for I in range(Nb):
            sel = top_tau_row(m[h, I], I, Nb, tau)
            count[h, I] = sel.size
            idx[h, I, :sel.size] = sel
    return count, idx


def rr_search(Q: np.ndarray, K: np.ndarray, B: int, S: int, tau: float, rotate: bool = False,
              mean_keys: bool = False, gqa_mask: bool = False):
    """The pattern search: returns (count, idx, m) with m the normalised block mass
    (of the GQA group when gqa_mask)."""
    M = block_mass(Q, K, B, S, rotate=rotate, mean_keys=mean_keys)
    if gqa_mask:
        M = group_mass(M, K.shape[1])
    m = normalise_mass(M)
    count, idx = select(m, tau)
    return count, idx, m


def full_causal_mask(H: int, Nb: int):
    """Every causal block selected (the tau >= 1 mask)."""
    count = np.tile(np.arange(1, Nb + 1, dtype=np.int32), (H, 1))
    idx = np.tile(np.where(np.tri(Nb, dtype=bool), np.arange(Nb)[None, :], -1).astype(np.int32),
                  (H, 1, 1))
    return count, idx


# ------------------------------------------------------ R8 sparse attention
def sparse_attention_block(Q, K, V, h: int, I: int, blocks, B: int) -> np.ndarray:
    """Output rows of query block I, head h, over the listed key blocks (R8).

    Returns [B, d] float64.
    """
    L, H, d = Q.shape
    g = H // K.shape[1]
    kv = h // g
    blocks = np.asarray(blocks, dtype=np.int64)
    keys = (blocks[:, None] * B + np.arange(B)[None, :]).reshape(-1)
    q_pos = I * B + np.arange(B)
    s = (Q[q_pos, h, :].astype(np.float64) @ K[keys, kv, :].astype(np.float64).T) / math.sqrt(d)
    s = np.where(keys[None, :] <= q_pos[:, None], s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V[keys, kv, :].astype(np.float64)


def sparse_attention(Q, K, V, count, idx, B: int, rows=None) -> np.ndarray:
    """Block-sparse causal attention (R8).

    rows: None for every (h, I), else an iterable of (h, I); rows not computed
    stay NaN.  Returns [L, H, d] float64.
    """
    L, H, d = Q.shape
    Nb = L // B
    O = np.full((L, H, d), np.nan, dtype=np.float64)
    if rows is None:
        rows = [(h, I) for h in range(H) for I in range(Nb)]
    for h, I in rows:
        c = int(count[h, I])
        O[I * B:(I + 1) * B, h, :] = sparse_attention_block(Q, K, V, h, I, idx[h, I, :c], B)
    return O


# ------------------------------------------------ mask diagnostics (recall)
def exact_block_mass(Q, K, B: int) -> np.ndarray:
    """Exact full-attention block mass: the R2-R5 definitions at S = 1, where every
    query and every key is sampled (pinned against the attention matrix of
    torch's scaled_dot_product_attention)."""
    return block_mass(Q, K, B, 1)


def mask_recall(M: np.ndarray, count: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """recall[h, I] = sum of M[h, I, J] over the selected J / sum over J <= I."""
    H, Nb, _ = M.shape
    m = normalise_mass(M)
    out = np.zeros((H, Nb), dtype=np.float64)
    for h in range(H):
        for I in range(Nb):
            sel = idx[h, I, :count[h, I]]
            out[h, I] = m[h, I, sel].sum()
    return out


# -------------------------------------------------------- R9 comparison band
def band_blocks(m_row: np.ndarray, I: int, tau: float, band: float = 1e-4, tie: float = 1e-6):
    """Blocks of row I whose selection may legitimately differ (R9).

    Returns (near_threshold, near_tie): two sets of J.  near_threshold: the
    running sum (R6 order) just before or just after the block lies within
    `band` of tau.  near_tie: blocks at the cut whose mass is within `tie` of
    the mass of the block on the other side of the cut.
    """
    n = I + 1
    order = sorted_order(m_row[:n])
    vals = m_row[:n][order]
    run = np.cumsum(vals)
    before = np.concatenate([[0.0], run[:-1]])
    near = set(int(order[t]) for t in range(n)
               if abs(before[t] - tau) <= band or abs(run[t] - tau) <= band)
    hit = np.nonzero(run >= tau)[0]
    k = int(hit[0]) + 1 if hit.size else n
    ties = set()
    if 0 < k < n:
        cut_in, cut_out = vals[k - 1], vals[k]
        for t in range(n):
            if t < k and abs(vals[t] - cut_out) < tie:
                ties.add(int(order[t]))
            if t >= k and abs(vals[t] - cut_in) < tie:
                ties.add(int(order[t]))
    return near, ties


# ------------------------------------------------------ D1-D5 decode stage
def decode_positions(t: int, h: int, S: int) -> np.ndarray:
    """Sampled key positions of head h for a query at position t (D1):
    j*S + (h mod S) for every stride j whose sampled position is <= t."""
    off = h % S
    if t < off:
        return np.zeros(0, dtype=np.int64)
    return np.arange((t - off) // S + 1, dtype=np.int64) * S + off


def decode_block_mass(q: np.ndarray, K: np.ndarray, t: int, B: int, S: int) -> np.ndarray:
    """Block mass of one decode query (D1-D3).  q: [H, d] (the query at position
    t), K: [L, Hkv, d] with L > t.  Returns [H, J_t + 1] float64, each row
    summing to 1 (or all zero when the head samples no key at or before t)."""
    H, d = q.shape
    g = H // K.shape[1]
    Jt = t // B
    M = np.zeros((H, Jt + 1), dtype=np.float64)
    for h in range(H):
        pos = decode_positions(t, h, S)
        if pos.size == 0:
            continue
        s = (K[pos, h // g, :].astype(np.float64) @ q[h].astype(np.float64)) / math.sqrt(d)   # D2
        P = np.exp(s - s.max())
        P = P / P.sum()
        np.add.at(M[h], pos // B, P)                                                         # D3
    return M


def decode_select(m_row: np.ndarray, Jt: int, tau: float) -> np.ndarray:
    """Selected key blocks of one decode query, ascending (D4): the R6 prefix over
    J <= Jt by (mass desc, J asc), plus the current block Jt."""
    n = Jt + 1
    if tau >= 1.0:
        return np.arange(n, dtype=np.int32)
    m = m_row[:n]
    if m.sum() > 0:
        order = sorted_order(m)
        run = np.cumsum(m[order] / m.sum())
        hit = np.nonzero(run >= tau)[0]
        k = int(hit[0]) + 1 if hit.size else n
        sel = set(int(j) for j in order[:k])
    else:
        sel = set()
    sel.add(Jt)
    return np.array(sorted(sel), dtype=np.int32)


def decode_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, t: int, blocks, B: int) -> np.ndarray:
    """Output of one decode query over the listed key blocks (D5).  Returns [H, d]
    float64; `blocks` is a list (one array of block indices per head)."""
    H, d = q.shape
    g = H // K.shape[1]
    out = np.zeros((H, d), dtype=np.float64)
    for h in range(H):
        b = np.asarray(blocks[h], dtype=np.int64)
        keys = (b[:, None] * B + np.arange(B)[None, :]).reshape(-1)
        keys = keys[keys <= t]
        s = (K[keys, h // g, :].astype(np.float64) @ q[h].astype(np.float64)) / math.sqrt(d)
        p = np.exp(s - s.max())
        p = p / p.sum()
        out[h] = p @ V[keys, h // g, :].astype(np.float64)
    return out


def decode_group_mass(M: np.ndarray, Hkv: int) -> np.ndarray:
    """V3 for the decode step: the block masses of the g query heads of each kv
    head summed, repeated for every head of the group.  [H, J_t + 1]."""
    H, n = M.shape
    g = H // Hkv
    return np.repeat(M.reshape(Hkv, g, n).sum(axis=1), g, axis=0)


def rr_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray, t: int, B: int, S: int, tau: float,
              gqa_mask: bool = False):
    """One decode step of one sequence (D1-D5): returns (count [H], idx list per
    head, the mass the selection ran on [H, J_t + 1], output [H, d]).  gqa_mask
    (V3): one list per GQA group, selected on the group's summed mass."""
    M = decode_block_mass(q, K, t, B, S)
    if gqa_mask:
        M = decode_group_mass(M, K.shape[1])
    Jt = t // B
    sel = [decode_select(M[h], Jt, tau) for h in range(q.shape[0])]
    count = np.array([x.size for x in sel], dtype=np.int32)
    return count, sel, M, decode_attention(q, K, V, t, sel, B)


def decode_band_blocks(m_row: np.ndarray, Jt: int, tau: float, band: float = 1e-4, tie: float = 1e-6):
    """R9 for a decode row: the blocks whose selection may legitimately differ."""
    m = np.asarray(m_row[:Jt + 1], dtype=np.float64)
    tot = m.sum()
    return band_blocks(m / tot if tot > 0 else m, Jt, tau, band, tie)

