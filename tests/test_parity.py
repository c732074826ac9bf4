"""CUDA path vs the fp64 oracle, through the C ABI.

Masks: bit-exact except blocks in the 1e-4 band around tau (or near-ties at the
cut), which are counted and reported.  Outputs (bf16) against the oracle fed
the GPU's own mask: max |err| <= 2e-2, mean |err| <= 2e-3.  Block masses are
also compared directly (normalised, |err| <= 2e-5): they are fp32 on the GPU.
"""
import numpy as np
import pytest
import torch

import gen
import oracle
from tests.mask_compare import check_mask_format, compare_masks, output_errors

pytestmark = pytest.mark.gpu

MAX_ERR, MEAN_ERR, MASS_ERR = 2e-2, 2e-3, 2e-5


@pytest.fixture(scope="module")
def rr():
    from dynamic_block_sparse_rr_b200 import _build
    _build.build()
    import dynamic_block_sparse_rr_b200 as m
    assert torch.cuda.is_available(), "the parity tests need a CUDA device"
    m.lib()
    return m


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(rr, qd, kd, vd, B, S, tau):
    L, H, d = qd.shape
    Hkv = kd.shape[1]
    Nb = L // B
    ws = rr.workspace(L, H, Hkv, d, B, S)
    mass = torch.zeros((H, Nb, Nb), dtype=torch.float32, device="cuda")
    count, idx = rr.search(qd, kd, B, S, tau, mass=mass, ws=ws)
    o = rr.sparse_attn(qd, kd, vd, count, idx, B, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    torch.cuda.synchronize()
    return count.cpu().numpy(), idx.cpu().numpy(), mass.cpu().numpy().astype(np.float64), o


def gpu_o_f32(o: torch.Tensor) -> np.ndarray:
    return o.float().cpu().numpy()


def normalised(M):
    return oracle.normalise_mass(M)


def check_case(rr, L, H, Hkv, d, B, S, tau, structure, seed=0, attn_rows=None, taus=None):
    q, k, v = gen.make_qkv(L, H, Hkv, d, structure, seed)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    Nb = L // B
    M_o = oracle.block_mass(Q, K, B, S)
    m_o = normalised(M_o)
    report = {}
    for t in (taus or [tau]):
        count, idx, M_g, o = run_gpu(rr, qd, kd, vd, B, S, t)
        check_mask_format(count, idx)
        tri = np.tri(Nb, dtype=bool)[None]
        mass_err = float(np.max(np.abs(np.where(tri, normalised(M_g) - m_o, 0.0))))
        assert mass_err <= MASS_ERR, f"block mass error {mass_err}"
        count_o, idx_o = oracle.select(m_o, t)
        st = compare_masks(count, idx, count_o, idx_o, m_o, t)
        assert st["blocks_fail"] == 0, st
        O_ref = oracle.sparse_attention(Q, K, V, count, idx, B, rows=attn_rows)
        mx, mean = output_errors(gpu_o_f32(o), O_ref)
        assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)
        report[t] = dict(mass_err=mass_err, max_err=mx, mean_err=mean,
                         visited=float(count.sum()) / (H * Nb * (Nb + 1) / 2), **st)
    print(report)
    return report


# ------------------------------------------------------------ small, full check
def test_tiny_config(rr):
    cfg = gen.CONFIGS["tiny"]
    check_case(rr, cfg.L, cfg.H, cfg.Hkv, cfg.d, cfg.B, cfg.S, cfg.tau, cfg.structure)


@pytest.mark.parametrize("L,H,Hkv,d,B,S,tau,structure", [
    (1600, 4, 2, 64, 64, 4, 0.9, gen.PLANTED),        # Ns = 400: ragged sampled-row tile
    (4096, 8, 2, 128, 128, 16, 0.95, gen.PLANTED),   # LLaMA-shaped head dim / block
    (2240, 4, 1, 128, 64, 8, 0.9, gen.PLANTED_BAND),  # B=64 with d=128, Nb = 35
    (2048, 2, 2, 64, 128, 2, 0.8, gen.IID),          # r = 64: cross-warp block reduction
    (1024, 2, 1, 128, 128, 1, 0.9, gen.PLANTED),     # S = 1: every query sampled, r = 128
    (4096, 7, 1, 128, 128, 16, 0.95, gen.VIDEO),     # video-like frames, GQA 7:1
    (512, 3, 3, 64, 64, 64, 0.5, gen.IID),           # r = 1
])
def test_small_shapes(rr, L, H, Hkv, d, B, S, tau, structure):
    check_case(rr, L, H, Hkv, d, B, S, tau, structure, seed=1)


@pytest.mark.parametrize("B,d", [(64, 64), (128, 128)])
def test_single_block_and_two_blocks(rr, B, d):
    for L in (B, 2 * B):
        check_case(rr, L, 2, 1, d, B, 4, 0.9, gen.IID, seed=2)


@pytest.mark.parametrize("B,d", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_tau_one_is_dense_causal(rr, B, d):
    L, H, Hkv = 8 * B, 4, 2
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.IID, 3)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    count, idx, _, o = run_gpu(rr, to_dev(q), to_dev(k), to_dev(v), B, 4, 1.0)
    c_ref, i_ref = oracle.full_causal_mask(H, L // B)
    assert np.array_equal(count, c_ref)
    for h in range(H):
        for I in range(L // B):
            assert np.array_equal(idx[h, I, :count[h, I]], i_ref[h, I, :count[h, I]])
    O_ref = oracle.sparse_attention(Q, K, V, c_ref, i_ref, B)
    mx, mean = output_errors(gpu_o_f32(o), O_ref)
    assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)


@pytest.mark.parametrize("B,d", [(64, 64), (128, 128), (64, 128)])
def test_arbitrary_masks(rr, B, d):
    """Attention over masks not produced by the search: single blocks, diagonal
    only, gaps, long lists."""
    L, H, Hkv = 12 * B, 4, 2
    Nb = L // B
    rng = np.random.default_rng(7)
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.IID, 4)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    count = np.zeros((H, Nb), np.int32)
    idx = np.zeros((H, Nb, Nb), np.int32)
    for h in range(H):
        for I in range(Nb):
            kind = (h + I) % 4
            if kind == 0:
                sel = np.array([I])
            elif kind == 1:
                sel = np.array([rng.integers(0, I + 1)])
            elif kind == 2:
                sel = np.arange(I + 1)
            else:
                sel = np.nonzero(rng.random(I + 1) < 0.4)[0]
                if sel.size == 0:
                    sel = np.array([0])
            count[h, I] = sel.size
            idx[h, I, :sel.size] = sel
    cd, idd = torch.from_numpy(count).cuda(), torch.from_numpy(idx).cuda()
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o = rr.sparse_attn(qd, kd, vd, cd, idd, B, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    O_ref = oracle.sparse_attention(Q, K, V, count, idx, B)
    mx, mean = output_errors(gpu_o_f32(o), O_ref)
    assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)


@pytest.mark.parametrize("B,d", [(128, 128), (64, 128)])
def test_mask_outside_format_is_reported_and_skipped(rr, B, d):
    """Rows whose block list breaks the mask format are not computed: a key block
    above the diagonal (J in (I, Nb), still inside the tensor, so nothing is read
    out of bounds), entries out of order, a repeated entry, a count of 0 and a
    count above I+1.  Their output rows are zero and rr_check_status reports
    RR_EMASK; every other row matches the oracle."""
    L, H, Hkv = 10 * B, 3, 1
    Nb = L // B
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.IID, 43)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    count, idx = oracle.full_causal_mask(H, Nb)
    count, idx = count.copy(), np.where(idx < 0, 0, idx).astype(np.int32)
    bad = {}
    idx[0, 3, 1] = 7;               bad[(0, 3)] = "future block"        # [0, 7, 2, 3]: J > I
    count[0, 5], idx[0, 5, :2] = 2, [4, 2];  bad[(0, 5)] = "descending"
    count[1, 4], idx[1, 4, :3] = 3, [1, 1, 4]; bad[(1, 4)] = "repeated"
    count[1, 6] = 0;                bad[(1, 6)] = "empty"
    count[2, 2] = 5;                bad[(2, 2)] = "count above I+1"
    count[2, 8], idx[2, 8, :2] = 2, [3, Nb - 1]; bad[(2, 8)] = "last entry above the diagonal"
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    o = rr.sparse_attn(to_dev(q), to_dev(k), to_dev(v), torch.from_numpy(count).cuda(),
                       torch.from_numpy(idx).cuda(), B, ws=ws)
    assert rr.check_status(ws) == rr.RR_EMASK
    og = gpu_o_f32(o)
    good = [(h, I) for h in range(H) for I in range(Nb) if (h, I) not in bad]
    O_ref = oracle.sparse_attention(Q, K, V, count, idx, B, rows=good)
    for (h, I), why in bad.items():
        assert np.all(og[I * B:(I + 1) * B, h, :] == 0.0), why
    mx, mean = output_errors(og, O_ref)
    assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)
    # the status word is reset by the next call, which then reports ok
    c2, i2 = oracle.full_causal_mask(H, Nb)
    rr.sparse_attn(to_dev(q), to_dev(k), to_dev(v), torch.from_numpy(c2).cuda(),
                   torch.from_numpy(np.where(i2 < 0, 0, i2).astype(np.int32)).cuda(), B, out=o, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK


@pytest.mark.parametrize("B,d", [(128, 128), (64, 64)])
@pytest.mark.parametrize("slope", [1.5, -1.5, 6.0])
def test_running_max_moves(rr, slope, B, d):
    """Scores that rise (or fall) steeply from key block to key block.  With a
    rising slope a row's running max, set by its first block, is far below the
    later blocks, so their exponentials pass the rescale bound again and again:
    the rows take the rescale path (exact block max, O and l rescaled, block
    redone) several times.  At slope 6 the last blocks score ~138 (log2 units)
    above the first block's max, past the fp32 range, so without that path the
    outputs would overflow.  A falling slope never moves it.  Outputs against
    the fp64 oracle over every causal block."""
    L, H, Hkv = 16 * B, 2, 1
    Nb = L // B
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.IID, 41)
    qn, kn = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k)
    c = -2.0 + slope * (np.arange(L) // B) if slope > 0 else 10.0 + slope * (np.arange(L) // B)
    qf = 0.5 * qn
    qf[:, :, 0] += 12.0 * np.sqrt(d / 128.0)             # every query along e_0 (same logits at any d)
    kf = 0.5 * kn
    kf[:, :, 0] += c[:, None].astype(np.float32)          # key block J scores ~ c(J)
    to_bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    qb, kb = to_bf16(qf), to_bf16(kf)
    Q, K = qb.float().numpy(), kb.float().numpy()
    V = gen.bf16_bits_to_f32(v)
    count, idx = oracle.full_causal_mask(H, Nb)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o = rr.sparse_attn(qb.cuda(), kb.cuda(), to_dev(v), torch.from_numpy(count).cuda(),
                       torch.from_numpy(idx).cuda(), B, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    O_ref = oracle.sparse_attention(Q, K, V, count, idx, B)
    mx, mean = output_errors(gpu_o_f32(o), O_ref)
    assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)


@pytest.mark.parametrize("L,tau", [(65536, 0.9), (131072, 0.5), (131072, 0.97)])
def test_tied_masses_keep_lowest_blocks(rr, L, tau):
    """Keys all zero: every score is 0, so sampled row i spreads 1/(i+1) over its
    strides and every full block of a row gets the same mass, bit for bit; the
    diagonal block gets less.  The selection must then be the lowest-J full
    blocks (ties go to the lower J), plus the diagonal only when the full blocks
    cannot reach tau.  Nb = 1024 and 2048 run every Top-tau path (one warp per
    row with 8, 16 and 32 masses per lane, and one CTA per row beyond 1024)."""
    H, Hkv, d, B, S = 2, 1, 64, 64, 4
    r, Nb = B // S, L // B
    q, _, _ = gen.make_qkv(L, H, Hkv, d, gen.IID, 51)
    kd = torch.zeros((L, Hkv, d), dtype=torch.bfloat16, device="cuda")
    ws = rr.workspace(L, H, Hkv, d, B, S)
    mass = torch.zeros((H, Nb, Nb), dtype=torch.float32, device="cuda")
    count, idx = rr.search(to_dev(q), kd, B, S, tau, mass=mass, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    count, idx, M = count.cpu().numpy(), idx.cpu().numpy(), mass.cpu().numpy()
    check_mask_format(count, idx)
    checked = 0
    for h in range(H):
        for I in range(Nb - 1):
            assert np.all(M[h, I, :I] == M[h, I, 0]), (h, I)   # the ties are exact
            # closed form: full block a = r * sum 1/(i+1), diagonal b = sum (i - I*r + 1)/(i+1)
            i = np.arange(I * r, I * r + r, dtype=np.float64)
            a, b = r * np.sum(1.0 / (i + 1)), np.sum((i - I * r + 1) / (i + 1))
            total = I * a + b
            k = next((k for k in range(1, I + 1) if k * a >= tau * total), None)
            want = list(range(k)) if k is not None else list(range(I + 1))
            share = (len(want) * a if k is not None else total) / total
            if abs(share - tau) < 1e-6 or (k is not None and abs((k - 1) * a / total - tau) < 1e-6):
                continue   # cut within rounding of tau: either side is right
            assert count[h, I] == len(want), (h, I, count[h, I], len(want))
            assert np.array_equal(idx[h, I, :count[h, I]], want), (h, I)
            checked += 1
    assert checked > 0.99 * H * (Nb - 1)


def test_deterministic(rr):
    L, H, Hkv, d, B, S = 4096, 8, 2, 128, 128, 16
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 5)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    a = run_gpu(rr, qd, kd, vd, B, S, 0.95)
    b = run_gpu(rr, qd, kd, vd, B, S, 0.95)
    assert np.array_equal(a[0], b[0])
    for h in range(H):
        for I in range(L // B):
            assert np.array_equal(a[1][h, I, :a[0][h, I]], b[1][h, I, :b[0][h, I]])
    assert np.array_equal(a[2], b[2])
    assert torch.equal(a[3], b[3])


def test_fused_attention_matches_two_calls(rr):
    L, H, Hkv, d, B, S = 2048, 4, 2, 128, 128, 16
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 6)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    c1, i1, _, o1 = run_gpu(rr, qd, kd, vd, B, S, 0.9)
    ws = rr.workspace(L, H, Hkv, d, B, S)
    o2, c2, i2 = rr.attention(qd, kd, vd, B, S, 0.9, ws=ws)
    assert rr.check_status(ws) == rr.RR_OK
    assert np.array_equal(c1, c2.cpu().numpy())
    assert torch.equal(o1, o2)


# ------------------------------------------------------------ full-size workloads
def _sampled_rows(count, H, Nb, seed, n_random=24):
    rng = np.random.default_rng(seed)
    rows = {(h, 0) for h in (0, H - 1)} | {(h, Nb - 1) for h in (0, H // 2, H - 1)}
    heavy = np.argsort(-count.reshape(-1))[:4]
    rows |= {(int(i // Nb), int(i % Nb)) for i in heavy}
    rows |= {(int(rng.integers(0, H)), int(rng.integers(0, Nb))) for _ in range(n_random)}
    return sorted(rows)


def check_full_config(rr, name, taus=None):
    cfg = gen.CONFIGS[name]
    q, k, v = gen.make_config(cfg)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    Nb = cfg.L // cfg.B
    m_o = oracle.normalise_mass(oracle.block_mass(Q, K, cfg.B, cfg.S))
    out = {}
    for t in (taus or [cfg.tau]):
        count, idx, M_g, o = run_gpu(rr, qd, kd, vd, cfg.B, cfg.S, t)
        check_mask_format(count, idx)
        tri = np.tri(Nb, dtype=bool)[None]
        mass_err = float(np.max(np.abs(np.where(tri, oracle.normalise_mass(M_g) - m_o, 0.0))))
        assert mass_err <= MASS_ERR, mass_err
        count_o, idx_o = oracle.select(m_o, t)
        st = compare_masks(count, idx, count_o, idx_o, m_o, t)
        assert st["blocks_fail"] == 0, st
        rows = _sampled_rows(count, cfg.H, Nb, 11)
        O_ref = oracle.sparse_attention(Q, K, V, count, idx, cfg.B, rows=rows)
        mx, mean = output_errors(gpu_o_f32(o), O_ref)
        assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)
        out[t] = dict(mass_err=mass_err, max_err=mx, mean_err=mean, rows_checked=len(rows),
                      visited=float(count.sum()) / (cfg.H * Nb * (Nb + 1) / 2), **st)
    print(name, out)
    return out


@pytest.mark.slow
def test_llama16k(rr):
    check_full_config(rr, "llama16k")


@pytest.mark.slow
def test_llama32k_tau_sweep(rr):
    check_full_config(rr, "llama32k", taus=[0.9, 0.95, 0.99])


@pytest.mark.slow
def test_video64k(rr):
    check_full_config(rr, "video64k")


@pytest.mark.slow
def test_llama128k(rr):
    check_full_config(rr, "llama128k")


# ------------------------------------------------------------ edge cases
def test_small_tau_single_block_rows(rr):
    """tau near 0: every row but the protected last one keeps exactly its heaviest block."""
    rep = check_case(rr, 2048, 4, 2, 128, 128, 16, 1e-4, gen.PLANTED, seed=8)
    assert rep[1e-4]["blocks_fail"] == 0


@pytest.mark.slow
def test_maximum_block_count(rr):
    """Nb = 4096, the largest the ABI accepts (L = 262144 with B = 64): the Top-tau sort runs on
    4096-entry rows and the attention kernel holds a 4096-entry block list."""
    L, H, Hkv, d, B, S, tau = 262144, 1, 1, 64, 64, 4, 0.9
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.PLANTED_BAND, 12)
    Q, K, V = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k), gen.bf16_bits_to_f32(v)
    count, idx, M_g, o = run_gpu(rr, to_dev(q), to_dev(k), to_dev(v), B, S, tau)
    Nb = L // B
    assert Nb == 4096
    check_mask_format(count, idx)
    m_o = oracle.normalise_mass(oracle.block_mass(Q, K, B, S))
    count_o, idx_o = oracle.select(m_o, tau)
    st = compare_masks(count, idx, count_o, idx_o, m_o, tau)
    assert st["blocks_fail"] == 0, st
    rows = [(0, 0), (0, Nb - 1), (0, Nb - 2), (0, 2048), (0, 17)]
    O_ref = oracle.sparse_attention(Q, K, V, count, idx, B, rows=rows)
    mx, mean = output_errors(gpu_o_f32(o), O_ref)
    assert mx <= MAX_ERR and mean <= MEAN_ERR, (mx, mean)
    print("Nb=4096", st, mx, mean)


# ------------------------------------------------------------ mask diagnostics
@pytest.mark.parametrize("L,H,Hkv,d,B,S,tau", [(2048, 4, 2, 128, 128, 16, 0.9), (1024, 4, 4, 64, 64, 4, 0.9)])
def test_mask_recall_matches_oracle(rr, L, H, Hkv, d, B, S, tau):
    q, k, _ = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 13)
    Q, K = gen.bf16_bits_to_f32(q), gen.bf16_bits_to_f32(k)
    qd, kd = to_dev(q), to_dev(k)
    count, idx = rr.search(qd, kd, B, S, tau)
    M_g = rr.exact_block_mass(qd, kd, B)
    rec = rr.mask_recall(M_g, count, idx).cpu().numpy()
    M_o = oracle.exact_block_mass(Q, K, B)
    tri = np.tri(L // B, dtype=bool)[None]
    assert np.max(np.abs(np.where(tri, oracle.normalise_mass(M_g.cpu().numpy().astype(np.float64))
                                  - oracle.normalise_mass(M_o), 0.0))) <= MASS_ERR
    rec_o = oracle.mask_recall(M_o, count.cpu().numpy(), idx.cpu().numpy())
    assert np.max(np.abs(rec - rec_o)) <= 1e-5
    assert np.all(rec[:, -1] > 1 - 1e-6)


def test_mask_to_dense_matches_lists(rr):
    """rr_mask_to_dense marks exactly the listed blocks, for a searched mask and
    for a hand-made one with gaps, duplicates of nothing and an empty row."""
    from tests.mask_compare import dense_from_lists
    L, H, Hkv, d, B, S = 2048, 4, 2, 128, 128, 16
    q, k, _ = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 14)
    count, idx = rr.search(to_dev(q), to_dev(k), B, S, 0.8)
    dense = rr.mask_to_dense(count, idx).cpu().numpy()
    c, i = count.cpu().numpy(), idx.cpu().numpy()
    assert np.array_equal(dense.astype(bool), dense_from_lists(c, i))
    Nb = L // B
    c2 = np.zeros((H, Nb), np.int32)
    i2 = np.zeros((H, Nb, Nb), np.int32)
    for h in range(H):
        for I in range(Nb):
            sel = list(range(0, I + 1, h + 1)) if I % 3 else []
            c2[h, I] = len(sel)
            i2[h, I, :len(sel)] = sel
    dense2 = rr.mask_to_dense(torch.from_numpy(c2).cuda(), torch.from_numpy(i2).cuda()).cpu().numpy()
    assert np.array_equal(dense2.astype(bool), dense_from_lists(c2, i2))


@pytest.mark.parametrize("L,H,Hkv,d,B,S,tau,structure", [
    (2048, 8, 2, 128, 128, 16, 0.9, gen.PLANTED),   # items 1+3 and 3+1 heads: both slots reused
    (1600, 6, 3, 64, 64, 4, 0.9, gen.PLANTED),      # five items of 1-2 heads, ragged tile
    (4096, 7, 1, 128, 128, 16, 0.95, gen.VIDEO),    # one kv head in three items (1, 5, 1 heads)
    (2048, 16, 8, 128, 64, 8, 0.8, gen.IID),        # ten items, B = 64
    (1024, 4, 4, 64, 64, 4, 0.9, gen.IID),          # g = 1: one item per kv head
])
def test_attention_host_matches_device_path(rr, L, H, Hkv, d, B, S, tau, structure):
    """rr_attention_host (host buffers, copies pipelined per kv head) returns the
    device path's output and mask bit for bit."""
    q, k, v = gen.make_qkv(L, H, Hkv, d, structure, 31)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o_d, c_d, i_d = rr.attention(qd, kd, vd, B, S, tau)
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    o_h, c_h, i_h = rr.attention_host(pin(q), pin(k), pin(v), B, S, tau)
    torch.cuda.synchronize()
    assert torch.equal(c_h, c_d)
    Nb = L // B
    cols = torch.arange(Nb, device="cuda")[None, None, :] < c_d[:, :, None]
    assert torch.equal(torch.where(cols, i_h, 0), torch.where(cols, i_d, 0))
    assert torch.equal(o_h.view(torch.int16), o_d.cpu().view(torch.int16))


def test_attention_host_pinned_and_pageable_outputs_agree(rr):
    """rr_attention_host fills a caller's page-locked or pageable output with the
    device path's O, bit for bit."""
    L, H, Hkv, d, B, S, tau = 3072, 8, 2, 128, 128, 16, 0.9
    q, k, v = gen.make_qkv(L, H, Hkv, d, gen.PLANTED, 33)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o_d, _, _ = rr.attention(qd, kd, vd, B, S, tau)
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    qh, kh, vh = pin(q), pin(k), pin(v)
    out_pinned = torch.full((L, H, d), float("nan"), dtype=torch.bfloat16).pin_memory()
    out_pageable = torch.full((L, H, d), float("nan"), dtype=torch.bfloat16)
    for out in (out_pinned, out_pageable):
        o_h, _, _ = rr.attention_host(qh, kh, vh, B, S, tau, out=out)
        torch.cuda.synchronize()
        assert o_h.data_ptr() == out.data_ptr()
        assert torch.equal(o_h.view(torch.int16), o_d.cpu().view(torch.int16))


@pytest.mark.slow
def test_attention_host_llama128k_matches_device_path(rr):
    """The end-to-end path at the benchmark size (128K, the launch configuration
    the bench times): rr_attention_host output and mask equal the device path's
    bit for bit."""
    cfg = gen.CONFIGS["llama128k"]
    q, k, v = gen.make_config(cfg)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o_d, c_d, i_d = rr.attention(qd, kd, vd, cfg.B, cfg.S, cfg.tau)
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    qh, kh, vh = pin(q), pin(k), pin(v)
    del q, k, v
    o_h, c_h, i_h = rr.attention_host(qh, kh, vh, cfg.B, cfg.S, cfg.tau)
    torch.cuda.synchronize()
    assert torch.equal(c_h, c_d)
    Nb = cfg.L // cfg.B
    cols = torch.arange(Nb, device="cuda")[None, None, :] < c_d[:, :, None]
    assert torch.equal(torch.where(cols, i_h, 0), torch.where(cols, i_d, 0))
    assert torch.equal(o_h.view(torch.int16), o_d.cpu().view(torch.int16))
