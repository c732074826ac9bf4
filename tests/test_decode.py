"""Decode stage on the GPU (rr_decode, through the C ABI) against the oracle's
decode readings D1-D5.

Masks: each (sequence, head) list must equal the oracle's, except for blocks the
oracle marks as near-threshold or near-tie (R9); the current block is always
listed.  Outputs (bf16) against the oracle fed the GPU's own lists: max |err| <=
2e-2, mean |err| <= 2e-3.
"""
import numpy as np
import pytest
import torch

import gen
import oracle

pytestmark = pytest.mark.gpu

MAX_ERR, MEAN_ERR = 2e-2, 2e-3


@pytest.fixture(scope="module")
def rr():
    from dynamic_block_sparse_rr_b200 import _build
    _build.build()
    import dynamic_block_sparse_rr_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _make(N, Lmax, H, Hkv, d, structure, seed):
    """Per sequence: caches from the generator (its keys and values), and the query
    of the token at the sequence's last position."""
    qs, ks, vs = [], [], []
    for n in range(N):
        q, k, v = gen.make_qkv(Lmax, H, Hkv, d, structure, seed + n)
        qs.append(gen.bf16_bits_to_f32(q))
        ks.append(gen.bf16_bits_to_f32(k))
        vs.append(gen.bf16_bits_to_f32(v))
    return qs, np.stack(ks), np.stack(vs)


def run_case(rr, N, Lmax, H, Hkv, d, B, S, tau, lens, structure=gen.PLANTED, seed=0, flags=0, check=None):
    Qs, K, V = _make(N, Lmax, H, Hkv, d, structure, seed)
    q = np.stack([Qs[n][lens[n] - 1] for n in range(N)])              # [N, H, d]
    qd, kd, vd = _bf16(q).cuda(), _bf16(K).cuda(), _bf16(V).cuda()
    ld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(rr.decode_workspace_size(N, Lmax, H, Hkv, d, B, S), dtype=torch.uint8, device="cuda")
    o, count, idx = rr.decode(qd, kd, vd, ld, B, S, tau, ws=ws, flags=flags)
    gqa = bool(flags & rr.VAR_GQA_MASK)
    assert rr.check_status(ws) == rr.RR_OK
    count, idx, og = count.cpu().numpy(), idx.cpu().numpy(), o.float().cpu().numpy()
    stats = {"rows_differing": 0, "band": 0, "tie": 0, "fail": 0}
    errs = []
    for n in (range(N) if check is None else check):
        t = lens[n] - 1
        Jt = t // B
        M = oracle.decode_block_mass(q[n], K[n], t, B, S)
        if gqa:
            M = oracle.decode_group_mass(M, Hkv)
            g = H // Hkv
            for h in range(H):
                c0 = (h // g) * g
                assert count[n, h] == count[n, c0] and np.array_equal(idx[n, h, :count[n, h]], idx[n, c0, :count[n, c0]])
        blocks = []
        for h in range(H):
            g_sel = idx[n, h, :count[n, h]]
            assert count[n, h] >= 1 and np.all(np.diff(g_sel) > 0) and g_sel[-1] == Jt
            assert g_sel.min() >= 0
            o_sel = oracle.decode_select(M[h], Jt, tau)
            diff = set(g_sel.tolist()) ^ set(o_sel.tolist())
            if diff:
                stats["rows_differing"] += 1
                near, ties = oracle.decode_band_blocks(M[h], Jt, tau)
                for J in diff:
                    if J in near:
                        stats["band"] += 1
                    elif J in ties:
                        stats["tie"] += 1
                    else:
                        stats["fail"] += 1
            blocks.append(g_sel)
        ref = oracle.decode_attention(q[n], K[n], V[n], t, blocks, B)
        errs.append(np.abs(og[n] - ref))
    assert stats["fail"] == 0, stats
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= MAX_ERR and err.mean() <= MEAN_ERR, (err.max(), err.mean())
    assert np.all(count >= 1) and np.all(np.isfinite(og))
    visited = float(count.sum()) / sum(H * ((l - 1) // B + 1) for l in lens)
    print({"stats": stats, "max_err": float(err.max()), "mean_err": float(err.mean()), "visited": visited})
    return count, idx


@pytest.mark.parametrize("tau", [0.9, 0.5])
def test_decode_llama_shaped(rr, tau):
    """Eight sequences of a 4096-key cache, GQA 4:1, d = 128, B = 128, S = 16:
    lengths on and next to block boundaries, a partial last block, and a query
    before the first sampled key of most heads (length 3)."""
    lens = [4096, 4095, 129, 128, 3000, 1, 3, 2049]
    run_case(rr, len(lens), 4096, 8, 2, 128, 128, 16, tau, lens)


@pytest.mark.parametrize("B,d,S", [(64, 64, 4), (64, 128, 8), (128, 64, 32), (128, 128, 1), (64, 64, 64)])
def test_decode_block_and_head_sizes(rr, B, d, S):
    """B, d in {64, 128} and strides per block r = B/S from 1 (one sampled key
    per block) to 128 (every key sampled)."""
    lens = [2048, 1000, 65]
    run_case(rr, len(lens), 2048, 4, 1, d, B, S, 0.9, lens, structure=gen.PLANTED_BAND, seed=3)


def test_decode_gqa_seven_to_one_video(rr):
    lens = [4096, 2500]
    run_case(rr, 2, 4096, 7, 1, 128, 128, 16, 0.95, lens, structure=gen.VIDEO, seed=5)


@pytest.mark.parametrize("structure,H,Hkv,tau", [(gen.PLANTED, 8, 2, 0.9), (gen.VIDEO, 7, 1, 0.95),
                                                  (gen.PLANTED_BAND, 4, 4, 0.8)])
def test_decode_gqa_group_mask(rr, structure, H, Hkv, tau):
    """One list per GQA group (rr_decode_variant, RR_VAR_GQA_MASK): selected on the
    group's summed mass, the same on every head of the group; with one head per
    group it is the per-head list."""
    lens = [4096, 3001, 200, 1]
    run_case(rr, len(lens), 4096, H, Hkv, 128, 128, 16, tau, lens, structure=structure, seed=17,
             flags=rr.VAR_GQA_MASK)


def test_decode_many_ragged_sequences(rr):
    """Thirty-seven sequences of very different lengths (one key, one block, a
    block and one key, full caches, the rest seeded): the attention CTAs' shares
    of the flattened (sequence, kv head, block) space cut rows at arbitrary
    blocks and span several short rows each."""
    rng = np.random.default_rng(23)
    lens = [1, 128, 129, 2048, 2047, 5] + [int(x) for x in rng.integers(1, 2049, 31)]
    run_case(rr, len(lens), 2048, 8, 2, 128, 128, 16, 0.9, lens, seed=29)


def test_decode_single_short_sequence(rr):
    """One sequence inside its first block: fewer flattened blocks than attention
    CTAs, so most CTAs have an empty share."""
    run_case(rr, 1, 1024, 4, 1, 128, 128, 16, 0.9, [100], seed=31)


def test_decode_more_rows_than_a_grid_dimension_holds(rr):
    """4100 sequences x 16 heads = 65 600 (sequence, head) rows, more than the
    65 535 of a grid's y or z dimension.  Caches of 256 keys (four 64-key
    blocks), seeded lengths; a seeded sample of 40 sequences, the first and the
    last among them, against the oracle, and every row checked for a non-empty
    list ending at its current block and a finite output."""
    N, Lmax, H, Hkv, d, B, S, tau = 4100, 256, 16, 2, 64, 64, 4, 0.9
    rng = np.random.default_rng(37)
    lens = [int(x) for x in rng.integers(1, Lmax + 1, N)]
    # one query row per sequence, and the caches, straight from the generator
    q = gen.bf16_bits_to_f32(gen.fill(gen.IID, 41, gen.ROLE_Q, N, H, Hkv, d))
    K = gen.bf16_bits_to_f32(gen.fill(gen.IID, 41, gen.ROLE_K, N * Lmax, H, Hkv, d)).reshape(N, Lmax, Hkv, d)
    V = gen.bf16_bits_to_f32(gen.fill(gen.IID, 41, gen.ROLE_V, N * Lmax, H, Hkv, d)).reshape(N, Lmax, Hkv, d)
    ws = torch.empty(rr.decode_workspace_size(N, Lmax, H, Hkv, d, B, S), dtype=torch.uint8, device="cuda")
    o, count, idx = rr.decode(_bf16(q).cuda(), _bf16(K).cuda(), _bf16(V).cuda(),
                              torch.tensor(lens, dtype=torch.int32, device="cuda"), B, S, tau, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    count, idx, og = count.cpu().numpy(), idx.cpu().numpy(), o.float().cpu().numpy()
    last = np.array([(l - 1) // B for l in lens])
    assert np.all(count >= 1) and np.all(np.isfinite(og))
    assert np.all(idx[np.arange(N)[:, None], np.arange(H)[None, :], count - 1] == last[:, None])
    check = sorted({0, N - 1} | {int(x) for x in rng.choice(N, 38, replace=False)})
    fails = 0
    for n in check:
        t = lens[n] - 1
        M = oracle.decode_block_mass(q[n], K[n], t, B, S)
        blocks = []
        for h in range(H):
            g_sel = idx[n, h, :count[n, h]]
            o_sel = oracle.decode_select(M[h], t // B, tau)
            diff = set(g_sel.tolist()) ^ set(o_sel.tolist())
            if diff:
                near, ties = oracle.decode_band_blocks(M[h], t // B, tau)
                fails += len(diff - near - ties)
            blocks.append(g_sel)
        ref = oracle.decode_attention(q[n], K[n], V[n], t, blocks, B)
        assert np.abs(og[n] - ref).max() <= MAX_ERR, n
    assert fails == 0


def test_decode_tau_one_is_dense(rr):
    lens = [3000, 4096, 17]
    count, idx = run_case(rr, 3, 4096, 4, 2, 128, 128, 16, 1.0, lens, seed=7)
    for n, l in enumerate(lens):
        assert np.all(count[n] == (l - 1) // 128 + 1)


def test_decode_length_out_of_range_is_reported(rr):
    """A cache length outside [1, Lmax] is found on the device: that sequence
    keeps nothing and its output is zero, the others are unaffected, and
    rr_check_status reports RR_EINVAL."""
    N, Lmax, H, Hkv, d, B, S = 3, 1024, 4, 2, 128, 128, 16
    Qs, K, V = _make(N, Lmax, H, Hkv, d, gen.IID, 11)
    lens = [1024, 0, 1025]
    q = np.stack([Qs[0][1023], Qs[1][0], Qs[2][0]])
    ws = torch.empty(rr.decode_workspace_size(N, Lmax, H, Hkv, d, B, S), dtype=torch.uint8, device="cuda")
    o, count, idx = rr.decode(_bf16(q).cuda(), _bf16(K).cuda(), _bf16(V).cuda(),
                              torch.tensor(lens, dtype=torch.int32, device="cuda"), B, S, 0.9, ws=ws)
    assert rr.check_status(ws) == rr.RR_EINVAL
    og, count = o.float().cpu().numpy(), count.cpu().numpy()
    assert np.all(count[1] == 0) and np.all(count[2] == 0)
    assert np.all(og[1] == 0) and np.all(og[2] == 0)
    ref = oracle.decode_attention(q[0], K[0], V[0], 1023, [idx[0, h, :count[0, h]].cpu().numpy()
                                                           for h in range(H)], B)
    assert np.abs(og[0] - ref).max() <= MAX_ERR


def test_decode_deterministic(rr):
    N, Lmax, H, Hkv, d, B, S = 2, 4096, 8, 2, 128, 128, 16
    Qs, K, V = _make(N, Lmax, H, Hkv, d, gen.PLANTED, 13)
    q = _bf16(np.stack([Qs[0][4095], Qs[1][2000]])).cuda()
    kd, vd = _bf16(K).cuda(), _bf16(V).cuda()
    ld = torch.tensor([4096, 2001], dtype=torch.int32, device="cuda")
    a = rr.decode(q, kd, vd, ld, B, S, 0.9)
    b = rr.decode(q, kd, vd, ld, B, S, 0.9)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.slow
def test_decode_llama128k_last_token(rr):
    """The headline layer's last token (H=32/Hkv=8, d=128, a 131072-key cache):
    every head's list against the oracle's, and every head's output."""
    cfg = gen.CONFIGS["llama128k"]
    q, k, v = gen.make_config(cfg)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    del q, k, v
    L, H, Hkv, d, B, S = cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S
    t = L - 1
    qd = _bf16(Q[t][None]).cuda()
    kd, vd = _bf16(K[None]).cuda(), _bf16(V[None]).cuda()
    o, count, idx = rr.decode(qd, kd, vd, torch.tensor([L], dtype=torch.int32, device="cuda"), B, S, cfg.tau)
    count, idx, og = count.cpu().numpy()[0], idx.cpu().numpy()[0], o.float().cpu().numpy()[0]
    M = oracle.decode_block_mass(Q[t], K, t, B, S)
    blocks, fails = [], 0
    for h in range(H):
        g_sel = idx[h, :count[h]]
        o_sel = oracle.decode_select(M[h], t // B, cfg.tau)
        diff = set(g_sel.tolist()) ^ set(o_sel.tolist())
        near, ties = oracle.decode_band_blocks(M[h], t // B, cfg.tau) if diff else (set(), set())
        fails += len(diff - near - ties)
        blocks.append(g_sel)
    assert fails == 0
    ref = oracle.decode_attention(Q[t], K, V, t, blocks, B)
    err = np.abs(og - ref)
    print({"visited": float(count.sum()) / (H * (t // B + 1)), "max_err": float(err.max()),
           "mean_err": float(err.mean())})
    assert err.max() <= MAX_ERR and err.mean() <= MEAN_ERR


def test_decode_replays_from_a_cuda_graph(rr):
    """A decode step captured in a CUDA graph (memset, search, attention and
    combine with their programmatic launch edges) and replayed gives the
    eager call's lists and outputs bit for bit."""
    N, Lmax, H, Hkv, d, B, S, tau = 3, 2048, 8, 2, 128, 128, 16, 0.9
    Qs, K, V = _make(N, Lmax, H, Hkv, d, gen.PLANTED, 43)
    lens = [2048, 1500, 130]
    q = _bf16(np.stack([Qs[n][lens[n] - 1] for n in range(N)])).cuda()
    kd, vd = _bf16(K).cuda(), _bf16(V).cuda()
    ld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(rr.decode_workspace_size(N, Lmax, H, Hkv, d, B, S), dtype=torch.uint8, device="cuda")
    o_e, c_e, i_e = rr.decode(q, kd, vd, ld, B, S, tau, ws=ws)
    o, c, i = torch.empty_like(o_e), torch.empty_like(c_e), torch.empty_like(i_e)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        rr.decode(q, kd, vd, ld, B, S, tau, out=o, count=c, idx=i, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    o.zero_()
    c.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        rr.decode(q, kd, vd, ld, B, S, tau, out=o, count=c, idx=i, ws=ws)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert rr.check_status(ws) == rr.RR_OK
    assert torch.equal(o, o_e) and torch.equal(c, c_e)
    for n in range(N):
        for h in range(H):
            assert torch.equal(i[n, h, :c[n, h]], i_e[n, h, :c_e[n, h]])
