"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Tolerances: max-abs 1e-2 on bf16 outputs with bf16 KV and 2e-2 with e4m3 KV;
selections identical except for swaps whose oracle score lies within 1e-5
(relative) of the oracle's k-th score; windows identical.  The sparse kernels
are checked in isolation (fed the oracle's indices) and end to end (the
oracle re-run on the GPU's indices).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import check_selection, check_structure, max_abs
from token_level_top_hs2_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-2
TOL_E4M3 = 2e-2
TOL_LSE = 2e-3


def cuda(x):
    return x.cuda() if isinstance(x, torch.Tensor) else x


def sample_rows(B, L, n, seed, seg=256):
    """First 64, last 64, 64 at segment boundaries, the rest uniform; all b."""
    g = np.random.default_rng(seed)
    per = max(1, n // B)
    rows = []
    for b in range(B):
        t = set(range(min(64, L)))
        t |= set(range(max(0, L - 64), L))
        bnd = np.arange(seg, L, seg)
        if bnd.size:
            t |= set(g.choice(bnd, size=min(64, bnd.size), replace=False).tolist())
        rest = per - len(t)
        if rest > 0:
            t |= set(g.choice(L, size=min(rest, L), replace=False).tolist())
        rows += [b * L + x for x in sorted(t)]
    return np.array(sorted(rows), dtype=np.int64)


def run_full(hs2, x, rows=None):
    o, lse, idx = hs2.hs2_full_attn_select(cuda(x.q), cuda(x.k_), cuda(x.v), x.W, x.k)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == 0
    B, L, Hq, d = x.q.shape
    o = o.float().cpu().numpy().reshape(B * L, Hq, d)
    lse = lse.cpu().numpy().reshape(B * L, Hq)
    idx = idx.cpu().numpy().reshape(B * L, -1)
    return o, lse, idx


def check_full_layer(hs2, x, rows=None):
    B, L = x.q.shape[:2]
    o, lse, idx = run_full(hs2, x)
    t_all = np.tile(np.arange(L), B)
    check_structure(idx, t_all, x.W, x.k)
    if rows is None:
        rows = np.arange(B * L, dtype=np.int64)
    ora = oracle.full_select(x.q, x.k_, x.v, x.W, x.k, rows=rows, probe=idx[rows])
    assert max_abs(o[rows], ora["o"]) <= TOL_BF16
    assert max_abs(lse[rows], ora["lse"]) <= TOL_LSE
    n_swap, overlap = check_selection(idx[rows], ora, rows % L, x.W, x.k)
    return o, idx, ora, rows, n_swap, overlap


@pytest.mark.parametrize("shape", [
    dict(B=1, L=1024, Hq=4, d=64, W=32, k=128, n_topics=8, seg=128),   # the tiny prefill
    dict(B=2, L=777, Hq=16, d=128, W=128, k=256, n_topics=8, seg=256),  # ragged tail, B=2
    dict(B=1, L=300, Hq=8, d=128, W=16, k=0, n_topics=4, seg=64),       # window only
    dict(B=1, L=5, Hq=16, d=64, W=4, k=8, n_topics=2, seg=4),           # shorter than a tile
])
def test_full_attn_select_matches_oracle(cuda_lib, shape):
    s = dict(shape)
    x = inputs.make_prefill(seed=inputs.seed_for(0, 1), n_sparse=1, **s)
    _, idx, ora, rows, n_swap, overlap = check_full_layer(cuda_lib, x)
    assert overlap > 0.999


def _prefill_fail_flags(hs2, x, ws):
    """Per query block, whether the speculative stream thresholds failed the
    exact check (the workspace keeps them after the call: after the lse
    scratch, one word per 128-row query block)."""
    rows = x.B * x.L
    off = (rows * x.q.shape[2] * 4 + 255) // 256 * 256
    nqb = (x.L + 127) // 128
    return ws[off: off + 4 * x.B * nqb].view(torch.int32).cpu().numpy()


@pytest.mark.parametrize("decay", [0.0, 6.0])
def test_full_attn_select_speculative_thresholds(cuda_lib, decay):
    """Long rows (L = 8192, k = 256): the streams start from a speculative
    threshold.  With exchangeable keys (decay 0) it holds; with key relevance
    falling along the sequence (decay 6: early keys score higher) the first
    sample overestimates it, the per-row check fails and the exact re-run of
    those query blocks must give the same, exact selection."""
    B, L, Hq, d, W, k = 1, 8192, 16, 128, 128, 256
    x = inputs.make_prefill(B, L, Hq, d, W, k, n_topics=32, seg=256, seed=31, n_sparse=1)
    if decay:
        g = torch.Generator().manual_seed(32)
        u = torch.randn(d, generator=g)
        u /= u.norm()
        ramp = decay * (1.0 - torch.arange(L, dtype=torch.float32) / L)
        kf = x.k_.float() + ramp[None, :, None] * u
        qf = x.q.float() + 3.0 * u
        x = inputs.PrefillInputs(B, L, Hq, d, W, k, qf.bfloat16(), kf.bfloat16(), x.v, [],
                                 None, None, None)
    ws = torch.empty(cuda_lib.hs2_full_attn_select_workspace(
        cuda_lib.prefill_shape(B, L, Hq, d, W, k)), dtype=torch.uint8, device="cuda")
    o, lse, idx = cuda_lib.hs2_full_attn_select(cuda(x.q), cuda(x.k_), cuda(x.v), W, k,
                                                workspace=ws)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    fails = _prefill_fail_flags(cuda_lib, x, ws)
    if decay:
        assert fails.sum() > 0, "the decaying keys should defeat the speculative thresholds"
    idx = idx.cpu().numpy().reshape(B * L, -1)
    t_all = np.tile(np.arange(L), B)
    check_structure(idx, t_all, W, k)
    rows = sample_rows(B, L, 192, seed=5)
    ora = oracle.full_select(x.q, x.k_, x.v, W, k, rows=rows, probe=idx[rows])
    o = o.float().cpu().numpy().reshape(B * L, Hq, d)
    assert max_abs(o[rows], ora["o"]) <= TOL_BF16
    check_selection(idx[rows], ora, rows % L, W, k)


def test_full_attn_select_ties_take_lower_index(cuda_lib):
    """Keys drawn from 4 distinct rows: many exact score ties straddle the cut."""
    B, L, Hq, d, W, k = 1, 640, 16, 128, 16, 40
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    base = torch.randn(4, d, generator=g)
    k_ = base[torch.randint(0, 4, (L,), generator=g)].unsqueeze(0).bfloat16()
    v = torch.randn(B, L, d, generator=g).bfloat16()
    x = inputs.PrefillInputs(B, L, Hq, d, W, k, q, k_, v, [], None, None, None)
    o, lse, idx = run_full(cuda_lib, x)
    ora = oracle.full_select(q, k_, v, W, k, probe=idx)
    n_swap, _ = check_selection(idx, ora, np.arange(L), W, k, rel=1e-5)
    assert max_abs(o, ora["o"]) <= TOL_BF16


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_sparse_attn_isolated_and_end_to_end(cuda_lib, kv):
    B, L, Hq, d, W, k = 2, 900, 16, 128, 64, 192
    x = inputs.make_prefill(B, L, Hq, d, W, k, n_topics=8, seg=128, n_sparse=1,
                            seed=inputs.seed_for(0, 2))
    if kv == "e4m3":
        kc, ks = inputs.quantize_e4m3_per_token(x.k_)
        vc, vs = inputs.quantize_e4m3_per_token(x.v)
    else:
        kc, vc, ks, vs = x.k_, x.v, None, None
    ora_sel = oracle.full_select(x.q, x.k_, x.v, W, k)
    idx_ora = torch.from_numpy(ora_sel["idx"]).reshape(B, L, W + k)
    qs = x.q_sparse[0]
    # isolation: oracle indices
    o = cuda_lib.hs2_sparse_attn(cuda(qs), cuda(kc), cuda(vc), cuda(idx_ora), kv=kv,
                                 k_scale=cuda(ks), v_scale=cuda(vs), W=W, k_top=k)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    ref = oracle.sparse(qs, kc, vc, idx_ora, kv=kv, k_scale=ks, v_scale=vs)
    tol = TOL_E4M3 if kv == "e4m3" else TOL_BF16
    assert max_abs(o.float().cpu().numpy().reshape(B * L, Hq, d), ref) <= tol
    # end to end: GPU selection feeding the GPU sparse layer, oracle on the GPU's indices
    _, _, idx_gpu = cuda_lib.hs2_full_attn_select(cuda(x.q), cuda(x.k_), cuda(x.v), W, k)
    o2 = cuda_lib.hs2_sparse_attn(cuda(qs), cuda(kc), cuda(vc), idx_gpu, kv=kv,
                                  k_scale=cuda(ks), v_scale=cuda(vs), W=W, k_top=k)
    ref2 = oracle.sparse(qs, kc, vc, idx_gpu.cpu(), kv=kv, k_scale=ks, v_scale=vs)
    assert max_abs(o2.float().cpu().numpy().reshape(B * L, Hq, d), ref2) <= tol


def test_sparse_equals_full_when_budget_covers(cuda_lib):
    """W+k >= L selects everything: the sparse layer with the full layer's own
    queries must reproduce the full layer's output.  Both are bf16 roundings of
    the same exact attention, each checked against the oracle; between them
    the triangle bound 2 * TOL_BF16 applies (two roundings of one value can
    differ by an ulp, 2^-6 for |o| in [2, 4))."""
    B, L, Hq, d, W, k = 1, 200, 16, 128, 8, 200
    x = inputs.make_prefill(B, L, Hq, d, W, k, seed=5)
    o, _, idx = cuda_lib.hs2_full_attn_select(cuda(x.q), cuda(x.k_), cuda(x.v), W, k)
    o2 = cuda_lib.hs2_sparse_attn(cuda(x.q), cuda(x.k_), cuda(x.v), idx, W=W, k_top=k)
    torch.cuda.synchronize()
    ora = oracle.full_select(x.q, x.k_, x.v, W, k)
    assert max_abs(o.float().cpu().numpy().reshape(B * L, Hq, d), ora["o"]) <= TOL_BF16
    assert max_abs(o2.float().cpu().numpy().reshape(B * L, Hq, d), ora["o"]) <= TOL_BF16
    assert (o.float() - o2.float()).abs().max().item() <= 2 * TOL_BF16


def test_sparse_attn_flags_out_of_range_indices(cuda_lib):
    B, L, Hq, d = 1, 64, 16, 128
    x = inputs.make_prefill(B, L, Hq, d, 4, 4, seed=6)
    idx = torch.full((B, L, 8), -1, dtype=torch.int32)
    idx[0, :, 0] = torch.arange(L)
    idx[0, 10, 1] = 11  # beyond t = 10
    cuda_lib.hs2_sparse_attn(cuda(x.q), cuda(x.k_), cuda(x.v), cuda(idx), W=4, k_top=4)
    assert cuda_lib.hs2_get_last_device_error() == cuda_lib.HS2_ERR_DEVICE_DATA
    assert cuda_lib.hs2_get_last_device_error() == 0  # cleared


def _decode_case(kv, B, T, Hq, d, W, k, lengths=None, seed=0):
    return inputs.make_decode(B, T, Hq, d, W, k, kv=kv, seed=seed, lengths=lengths,
                              n_needles=16, n_sparse=1)


def run_decode(hs2, x):
    o, lse, idx = hs2.hs2_decode_select(cuda(x.q), cuda(x.k_cache), cuda(x.v_cache),
                                        cuda(x.lengths), x.W, x.k, kv=x.kv,
                                        k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale))
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()


@pytest.mark.parametrize("kv,B,T,Hq,d,W,k,lengths", [
    ("e4m3", 3, 20000, 16, 128, 128, 1024, [20000, 9000, 1100]),
    ("e4m3", 2, 70000, 16, 128, 128, 1024, None),     # several merge groups
    ("bf16", 2, 5000, 8, 64, 32, 128, [5000, 77]),
    ("e4m3", 4, 300, 4, 128, 16, 0, [300, 1, 17, 250]),  # window only, length 1
    ("e4m3", 3, 9000, 4, 128, 64, 512, [9000, 4000, 600]),  # 4 heads, 12 padded
    ("e4m3", 2, 5001, 16, 128, 128, 256, [5001, 3000]),  # Tmax % 4 != 0: register path
])
def test_decode_select_matches_oracle(cuda_lib, kv, B, T, Hq, d, W, k, lengths):
    x = _decode_case(kv, B, T, Hq, d, W, k, lengths, seed=inputs.seed_for(3, 7))
    o, lse, idx = run_decode(cuda_lib, x)
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv=kv,
                               k_scale=x.k_scale, v_scale=x.v_scale, probe=idx)
    tol = TOL_E4M3 if kv == "e4m3" else TOL_BF16
    assert max_abs(o, ora["o"]) <= tol
    assert max_abs(lse, ora["lse"]) <= TOL_LSE
    t = x.lengths.numpy().astype(np.int64) - 1
    check_structure(idx, t, W, k)
    check_selection(idx, ora, t, W, k)


@pytest.mark.parametrize("kv", ["e4m3", "bf16"])
def test_decode_sparse_isolated_and_end_to_end(cuda_lib, kv):
    B, T, Hq, d, W, k = 5, 12000, 16, 128, 128, 1024
    x = _decode_case(kv, B, T, Hq, d, W, k, [12000, 5000, 1152, 1000, 3], seed=11)
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv=kv,
                               k_scale=x.k_scale, v_scale=x.v_scale)
    idx_ora = torch.from_numpy(ora["idx"])
    qs = x.q_sparse[0]
    o = cuda_lib.hs2_decode_sparse(cuda(qs), cuda(x.k_cache), cuda(x.v_cache), cuda(x.lengths),
                                   cuda(idx_ora), kv=kv, k_scale=cuda(x.k_scale),
                                   v_scale=cuda(x.v_scale), W=W, k_top=k)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    ref = oracle.decode_sparse(qs, x.k_cache, x.v_cache, idx_ora, kv=kv, k_scale=x.k_scale,
                               v_scale=x.v_scale)
    tol = TOL_E4M3 if kv == "e4m3" else TOL_BF16
    assert max_abs(o.float().cpu().numpy(), ref) <= tol
    _, _, idx_gpu = run_decode(cuda_lib, x)
    o2 = cuda_lib.hs2_decode_sparse(cuda(qs), cuda(x.k_cache), cuda(x.v_cache), cuda(x.lengths),
                                    cuda(torch.from_numpy(idx_gpu)), kv=kv,
                                    k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale), W=W,
                                    k_top=k)
    ref2 = oracle.decode_sparse(qs, x.k_cache, x.v_cache, idx_gpu, kv=kv, k_scale=x.k_scale,
                                v_scale=x.v_scale)
    assert max_abs(o2.float().cpu().numpy(), ref2) <= tol


def test_decode_flags_bad_length(cuda_lib):
    x = _decode_case("e4m3", 2, 1000, 16, 128, 16, 32, seed=2)
    x.lengths[1] = 2000  # beyond Tmax
    o, lse, idx = cuda_lib.hs2_decode_select(cuda(x.q), cuda(x.k_cache), cuda(x.v_cache),
                                             cuda(x.lengths), 16, 32, kv="e4m3",
                                             k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale))
    assert cuda_lib.hs2_get_last_device_error() == cuda_lib.HS2_ERR_DEVICE_DATA
    assert (idx[1] == -1).all().item()


def test_e4m3_subnormal_codes_are_exact(cuda_lib):
    """Caches made only of subnormal and tiny normal e4m3 codes."""
    B, T, Hq, d, W, k = 1, 64, 16, 128, 8, 16
    g = torch.Generator().manual_seed(4)
    codes = torch.randint(0, 16, (B, T, d), generator=g).to(torch.uint8)  # exp field 0..1
    codes |= (torch.randint(0, 2, (B, T, d), generator=g).to(torch.uint8) << 7)
    kc = codes.clone()
    vc = torch.roll(codes, 1, dims=1).contiguous()
    ks = torch.full((B, T), 64.0)
    vs = torch.full((B, T), 32.0)
    q = torch.randn(B, Hq, d, generator=g).bfloat16()
    lengths = torch.tensor([T], dtype=torch.int32)
    o, lse, idx = cuda_lib.hs2_decode_select(cuda(q), cuda(kc), cuda(vc), cuda(lengths), W, k,
                                             kv="e4m3", k_scale=cuda(ks), v_scale=cuda(vs))
    ora = oracle.decode_select(q, kc, vc, lengths, W, k, kv="e4m3", k_scale=ks, v_scale=vs,
                               probe=idx.cpu())
    assert max_abs(o.float().cpu().numpy(), ora["o"]) <= TOL_E4M3
    assert max_abs(lse.cpu().numpy(), ora["lse"]) <= TOL_LSE
    check_selection(idx.cpu().numpy(), ora, np.array([T - 1]), W, k)


def test_decode_select_exact_ties_take_lower_index(cuda_lib):
    """Sequences whose older keys are all one row: every candidate score ties.

    Sequence 0 has far more tied candidates than the sketch selection's
    boundary buffer, so it goes through the exact fallback; sequence 2's tied
    candidates fit, so the sketch path rescoring cuts them; sequence 1 is
    ordinary.  Ties must go to the lower position in both paths."""
    B, T, Hq, d, W, k = 3, 20000, 16, 128, 128, 1024
    x = _decode_case("e4m3", B, T, Hq, d, W, k, [20000, 15000, 3000], seed=21)
    for b in (0, 2):
        x.k_cache[b, :] = x.k_cache[b, 5]
        x.k_scale[b, :] = x.k_scale[b, 5]
    o, lse, idx = run_decode(cuda_lib, x)
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv="e4m3",
                               k_scale=x.k_scale, v_scale=x.v_scale, probe=idx)
    assert max_abs(o, ora["o"]) <= TOL_E4M3
    assert max_abs(lse, ora["lse"]) <= TOL_LSE
    t = x.lengths.numpy().astype(np.int64) - 1
    check_structure(idx, t, W, k)
    check_selection(idx, ora, t, W, k)
    for b in (0, 2):
        assert sorted(idx[b, W:W + k].tolist()) == list(range(k))


def test_decode_select_every_sequence_overflows(cuda_lib):
    """Every sequence of the batch ties everywhere, so all of them take the
    exact fallback at once (each by all the CTAs of its chunks), with ragged
    lengths and one sequence short enough to take every candidate."""
    B, T, Hq, d, W, k = 5, 40000, 16, 128, 128, 1024
    x = _decode_case("e4m3", B, T, Hq, d, W, k, [40000, 33333, 26000, 9001, 1100], seed=23)
    for b in range(B):
        x.k_cache[b, :] = x.k_cache[b, 7]
        x.k_scale[b, :] = x.k_scale[b, 7]
    o, lse, idx = run_decode(cuda_lib, x)
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv="e4m3",
                               k_scale=x.k_scale, v_scale=x.v_scale, probe=idx)
    assert max_abs(o, ora["o"]) <= TOL_E4M3
    assert max_abs(lse, ora["lse"]) <= TOL_LSE
    t = x.lengths.numpy().astype(np.int64) - 1
    check_structure(idx, t, W, k)
    check_selection(idx, ora, t, W, k)
    for b in range(B):
        n_glob = min(k, int(x.lengths[b]) - W)
        assert sorted(idx[b, W:W + n_glob].tolist()) == list(range(n_glob))


def test_decode_needles_recovered(cuda_lib):
    x = _decode_case("e4m3", 4, 65536, 16, 128, 128, 1024, seed=inputs.seed_for(4, 3))
    _, _, idx = run_decode(cuda_lib, x)
    for b in range(4):
        assert set(x.needle_pos[b].tolist()) <= set(idx[b].tolist())


# ------------------------------------------------- cross-layer overlap
def _check_overlap(hs2, idx_a, idx_b, W, k, rows=None):
    """Counts bit-exact against the oracle; ratios equal to the one correctly
    rounded fp32 division of the exact count.  rows: flattened b*L+t sample."""
    inter, ratio = hs2.hs2_selection_overlap(cuda(idx_a), cuda(idx_b), W, k)
    torch.cuda.synchronize()
    err = hs2.hs2_get_last_device_error()
    B, L, S = idx_a.shape
    inter = inter.cpu().numpy().reshape(-1)
    ratio = ratio.cpu().numpy().reshape(-1)
    if rows is None:
        rows = np.arange(B * L)
    ra = idx_a.reshape(B * L, 1, S)[rows]
    rb = idx_b.reshape(B * L, 1, S)[rows]
    oi, orat = [], []
    for n, r in enumerate(rows):
        t = int(r % L)
        ga = oracle.global_picks(ra[n, 0].tolist(), t, W)
        gb = oracle.global_picks(rb[n, 0].tolist(), t, W)
        oi.append(len(ga & gb))
    oi = np.array(oi)
    assert np.array_equal(inter[rows], oi)
    t = rows % L
    denom = np.where((t >= W) & (k > 0), np.minimum(k, t - W + 1), 0)
    want = np.where(denom > 0, oi.astype(np.float32) / np.maximum(denom, 1).astype(np.float32),
                    np.float32(1.0)).astype(np.float32)
    assert np.array_equal(ratio[rows], want)
    return err, ratio[rows]


@pytest.mark.parametrize("B,L,W,k", [(2, 777, 128, 256), (1, 300, 16, 0), (1, 5, 4, 8),
                                     (3, 1500, 32, 1024), (1, 2999, 7, 30),
                                     (1, 140000, 8, 16)])  # L > 2^17: the hash-set kernel
def test_selection_overlap_matches_oracle(cuda_lib, B, L, W, k):
    a, b = inputs.make_selection_pair(B, L, W, k, seed=11)
    err, ratio = _check_overlap(cuda_lib, a, b, W, k)
    assert err == 0
    if k == 0:
        assert np.all(ratio == 1.0)
    # a selection against itself
    err, ratio = _check_overlap(cuda_lib, a, a, W, k)
    assert err == 0 and np.all(ratio == 1.0)


def test_selection_overlap_of_two_layers(cuda_lib):
    # the full layer's selection against the exact one of a sparse layer's
    # own queries: the oracle's selections, compared on the GPU
    x = inputs.make_workload("prefill_tiny_1k")
    L = x.q.shape[1]
    ia = torch.from_numpy(oracle.full_select(x.q, x.k_, x.v, x.W, x.k)["idx"]).view(1, L, -1)
    ib = torch.from_numpy(oracle.full_select(x.q_sparse[0], x.k_, x.v, x.W, x.k)["idx"])
    err, ratio = _check_overlap(cuda_lib, ia, ib.view(1, L, -1), x.W, x.k)
    assert err == 0 and 0.0 < ratio.mean() < 1.0


def test_selection_overlap_bench_size_sampled(cuda_lib):
    # 128k rows of W=128, k=1024: every count on the GPU, 2048 rows re-counted
    a, b = inputs.make_selection_pair(1, 131072, 128, 1024, seed=12)
    rows = np.unique(np.concatenate([np.arange(64), np.arange(131072 - 64, 131072),
                                     np.random.default_rng(1).choice(131072, 1920, False)]))
    err, _ = _check_overlap(cuda_lib, a, b, 128, 1024, rows=rows)
    assert err == 0


def test_selection_overlap_flags_out_of_range_entries(cuda_lib):
    a, b = inputs.make_selection_pair(1, 200, 8, 16, seed=13)
    a = a.clone()
    a[0, 50, 0] = 51          # beyond t = 50: skipped, flagged
    b = b.clone()
    b[0, 60, 3] = -7
    err, _ = _check_overlap(cuda_lib, a, b, 8, 16)
    assert err == cuda_lib.HS2_ERR_DEVICE_DATA
    assert cuda_lib.hs2_get_last_device_error() == 0


# ------------------------------------------------- block-level selector
def _check_block_rows(idx, ora, rows, L, W, k, blk):
    """Windows identical; chosen blocks equal to the oracle's except swaps whose
    oracle mass lies within 1e-5 (relative) of the smallest chosen mass; every
    chosen block contributes exactly its candidate positions."""
    n_swap = 0
    for r, row in enumerate(rows):
        t = int(row % L)
        g = idx[row]
        o = ora["idx"][r]
        wl = min(t + 1, W)
        assert g[:wl].tolist() == o[:wl].tolist(), t
        gg = g[wl:][g[wl:] >= 0]
        og = o[wl:][o[wl:] >= 0]
        gb, ob = set((gg // blk).tolist()), set((og // blk).tolist())
        assert len(gb) == len(ob) and len(gg) == len(set(gg.tolist()))
        for j in gb:
            want = list(range(blk * j, min(blk * j + blk, t - W + 1)))
            assert sorted(s for s in gg.tolist() if s // blk == j) == want, (t, j)
        diff = gb ^ ob
        if diff:
            sig = ora["sigma"][r]
            assert sig > 0
            for j in diff:
                assert abs(ora["mass"][r, j] - sig) <= 1e-5 * sig, (t, j)
            n_swap += len(diff) // 2
        assert np.all(g[wl + len(gg):] == -1)
    return n_swap


@pytest.mark.parametrize("shape", [
    dict(B=1, L=1024, Hq=4, d=64, W=32, k=128, n_topics=8, seg=128),
    dict(B=2, L=777, Hq=16, d=128, W=128, k=256, n_topics=8, seg=256),
    dict(B=1, L=5, Hq=16, d=64, W=4, k=64, n_topics=2, seg=4),
    dict(B=1, L=3000, Hq=8, d=128, W=64, k=1024, n_topics=8, seg=256),
])
def test_block_selector_matches_oracle(cuda_lib, shape):
    s = dict(shape)
    x = inputs.make_prefill(seed=inputs.seed_for(0, 2), n_sparse=1, **s)
    B, L, Hq, d = x.q.shape
    o, lse, idx = cuda_lib.hs2_full_attn_select_blocks(cuda(x.q), cuda(x.k_), cuda(x.v), x.W, x.k)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    o = o.float().cpu().numpy().reshape(B * L, Hq, d)
    lse = lse.cpu().numpy().reshape(B * L, Hq)
    idx = idx.cpu().numpy().reshape(B * L, -1)
    rows = np.arange(B * L) if B * L <= 1600 else sample_rows(B, L, 512, seed=3, seg=shape["seg"])
    ora = oracle.block_select(x.q, x.k_, x.v, x.W, x.k, block=64, rows=rows)
    full = oracle.full_select(x.q, x.k_, x.v, x.W, x.k, rows=rows)
    assert max_abs(o[rows], full["o"]) <= TOL_BF16
    assert max_abs(lse[rows], full["lse"]) <= TOL_LSE
    _check_block_rows(idx, ora, rows, L, x.W, x.k, 64)
    # the sparse layer consumes the block selection unchanged
    idx_t = torch.from_numpy(idx).view(B, L, -1)
    os_ = cuda_lib.hs2_sparse_attn(cuda(x.q_sparse[0]), cuda(x.k_), cuda(x.v), cuda(idx_t),
                                  W=x.W, k_top=x.k)
    ref = oracle.sparse(x.q_sparse[0], x.k_, x.v, idx_t, rows=rows)
    assert max_abs(os_.float().cpu().numpy().reshape(B * L, Hq, d)[rows], ref) <= TOL_BF16


# ------------------------------------------- the bench workloads
# Full sizes, in the launch configuration bench.py times.  Prefill: the
# oracle recomputes 512 sampled rows (first 64, last 64, 64 at segment
# boundaries, the rest uniform) one by one; the structure is checked on
# every row.  Decode: every sequence of the batch.  The sparse layers are
# checked end to end (the oracle on the GPU's selection) and in isolation
# (the GPU kernel fed the oracle's selection on the sampled rows).


def _splice_rows(idx_gpu, rows, idx_rows):
    """The GPU's [B*L, S] selection with the sampled rows replaced by
    another selection of those rows (the oracle's)."""
    out = idx_gpu.copy()
    out[rows] = idx_rows
    return out


def _check_prefill_workload(hs2, name, block_rows=0):
    x = inputs.make_workload(name)
    B, L, Hq, d = x.q.shape
    q, k, v = cuda(x.q), cuda(x.k_), cuda(x.v)
    o, lse, idx = hs2.hs2_full_attn_select(q, k, v, x.W, x.k)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == 0
    rows = sample_rows(B, L, 512, seed=5, seg=256)
    assert rows.size >= 500
    r_dev = torch.from_numpy(rows).cuda()
    o_r = o.view(B * L, Hq, d)[r_dev].float().cpu().numpy()
    lse_r = lse.view(B * L, Hq)[r_dev].cpu().numpy()
    idx_h = idx.view(B * L, -1).cpu().numpy()
    del o, lse
    check_structure(idx_h, np.tile(np.arange(L), B), x.W, x.k)
    ora = oracle.full_select(x.q, x.k_, x.v, x.W, x.k, rows=rows, probe=idx_h[rows])
    assert max_abs(o_r, ora["o"]) <= TOL_BF16
    assert max_abs(lse_r, ora["lse"]) <= TOL_LSE
    _, overlap = check_selection(idx_h[rows], ora, rows % L, x.W, x.k)
    assert overlap > 0.999
    # every sparse layer end to end, on the GPU's selection
    idx_t = torch.from_numpy(idx_h).view(B, L, -1)
    for j, qs in enumerate(x.q_sparse):
        os_ = hs2.hs2_sparse_attn(cuda(qs), k, v, idx, W=x.W, k_top=x.k)
        ref = oracle.sparse(qs, x.k_, x.v, idx_t, rows=rows)
        got = os_.view(B * L, Hq, d)[r_dev].float().cpu().numpy()
        assert max_abs(got, ref) <= TOL_BF16, f"sparse layer {j}"
    # every sparse layer in isolation: the oracle's selection on the sampled rows
    mix = torch.from_numpy(_splice_rows(idx_h, rows, ora["idx"])).view(B, L, -1)
    mix_d = cuda(mix)
    for j, qs in enumerate(x.q_sparse):
        os_ = hs2.hs2_sparse_attn(cuda(qs), k, v, mix_d, W=x.W, k_top=x.k)
        ref = oracle.sparse(qs, x.k_, x.v, mix, rows=rows)
        got = os_.view(B * L, Hq, d)[r_dev].float().cpu().numpy()
        assert max_abs(got, ref) <= TOL_BF16, f"sparse layer {j} on the oracle's selection"
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == 0
    if block_rows:
        # the block-level selector on a subset of the same rows
        brow = rows[np.linspace(0, rows.size - 1, block_rows).astype(np.int64)]
        _, _, bidx = hs2.hs2_full_attn_select_blocks(q, k, v, x.W, x.k, want_lse=False)
        bora = oracle.block_select(x.q, x.k_, x.v, x.W, x.k, block=64, rows=brow)
        _check_block_rows(bidx.view(B * L, -1).cpu().numpy(), bora, brow, L, x.W, x.k, 64)


@pytest.mark.parametrize("repeat", [0, 1, 2])
def test_tiny_prefill_three_seeds_every_row(cuda_lib, repeat):
    # the tiny workload (B=1, L=1024, Hq=4, d=64, W=32, k=128), three seeds:
    # the full layer and its sparse layer on every row, end to end and on the
    # oracle's selection
    x = inputs.make_workload("prefill_tiny_1k", repeat=repeat)
    B, L, Hq, d = x.q.shape
    _, idx, ora, rows, n_swap, overlap = check_full_layer(cuda_lib, x)
    assert overlap > 0.999
    for sel in (idx, ora["idx"]):
        idx_t = torch.from_numpy(np.ascontiguousarray(sel)).view(B, L, -1)
        os_ = cuda_lib.hs2_sparse_attn(cuda(x.q_sparse[0]), cuda(x.k_), cuda(x.v), cuda(idx_t),
                                       W=x.W, k_top=x.k)
        ref = oracle.sparse(x.q_sparse[0], x.k_, x.v, idx_t)
        assert max_abs(os_.float().cpu().numpy().reshape(B * L, Hq, d), ref) <= TOL_BF16
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0


def test_bench_prefill_32k_three_sparse_layers(cuda_lib):
    _check_prefill_workload(cuda_lib, "prefill_32k")


def test_bench_prefill_128k_sampled(cuda_lib):
    _check_prefill_workload(cuda_lib, "prefill_128k", block_rows=96)


@pytest.mark.parametrize("name", ["decode_256k_b16", "decode_1m_b4"])
def test_bench_decode_every_sequence(cuda_lib, name):
    x = inputs.make_workload(name)
    o, lse, idx = run_decode(cuda_lib, x)
    # every planted needle of every sequence is selected
    for b in range(x.B):
        assert set(x.needle_pos[b].tolist()) <= set(idx[b].tolist()), b
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, x.W, x.k, kv=x.kv,
                               k_scale=x.k_scale, v_scale=x.v_scale, probe=idx)
    assert max_abs(o, ora["o"]) <= TOL_E4M3
    assert max_abs(lse, ora["lse"]) <= TOL_LSE
    t = x.lengths.numpy().astype(np.int64) - 1
    check_structure(idx, t, x.W, x.k)
    check_selection(idx, ora, t, x.W, x.k)
    args = dict(kv=x.kv, k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale), W=x.W, k_top=x.k)
    kc, vc, lens = cuda(x.k_cache), cuda(x.v_cache), cuda(x.lengths)
    for sel, what in ((idx, "the GPU's"), (ora["idx"], "the oracle's")):
        sel_t = torch.from_numpy(np.ascontiguousarray(sel))
        for j, qs in enumerate(x.q_sparse):
            ods = cuda_lib.hs2_decode_sparse(cuda(qs), kc, vc, lens, cuda(sel_t), **args)
            refd = oracle.decode_sparse(qs, x.k_cache, x.v_cache, sel_t, kv=x.kv,
                                        k_scale=x.k_scale, v_scale=x.v_scale)
            assert max_abs(ods.float().cpu().numpy(), refd) <= TOL_E4M3, \
                f"decode sparse layer {j} on {what} selection"
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0


# ------------------------------------------- decode step with staged rows
@pytest.mark.parametrize("kv,B,T,Hq,d,W,k,lengths", [
    ("e4m3", 5, 12000, 16, 128, 128, 1024, [12000, 7000, 300, 1, 1152]),
    ("bf16", 3, 5000, 8, 64, 32, 128, [5000, 160, 77]),
    ("bf16", 2, 3000, 16, 128, 64, 256, None),
])
def test_decode_sparse_staged_equals_gathered(cuda_lib, kv, B, T, Hq, d, W, k, lengths):
    x = _decode_case(kv, B, T, Hq, d, W, k, lengths, seed=inputs.seed_for(3, 11))
    _, _, idx = run_decode(cuda_lib, x)
    idx_t = cuda(torch.from_numpy(idx))
    args = dict(kv=kv, k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale))
    o_g = cuda_lib.hs2_decode_sparse(cuda(x.q_sparse[0]), cuda(x.k_cache), cuda(x.v_cache),
                                     cuda(x.lengths), idx_t, W=W, k_top=k, **args)
    staged = cuda_lib.hs2_decode_stage(cuda(x.k_cache), cuda(x.v_cache), cuda(x.lengths), idx_t,
                                       Hq=Hq, W=W, k_top=k, **args)
    o_s = cuda_lib.hs2_decode_sparse_staged(cuda(x.q_sparse[0]), staged, T, W, k, kv=kv)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    # the same rows in the same order: bit-identical
    assert torch.equal(o_g, o_s)
    ref = oracle.decode_sparse(x.q_sparse[0], x.k_cache, x.v_cache, torch.from_numpy(idx), kv=kv,
                               k_scale=x.k_scale, v_scale=x.v_scale)
    assert max_abs(o_s.float().cpu().numpy(), ref) <= (TOL_E4M3 if kv == "e4m3" else TOL_BF16)


def test_decode_stage_flags_out_of_range_entries(cuda_lib):
    x = _decode_case("e4m3", 2, 4000, 16, 128, 16, 64, [4000, 900], seed=31)
    _, _, idx = run_decode(cuda_lib, x)
    bad = idx.copy()
    bad[1, 20] = 950          # beyond length 900: skipped (staged as -1), flagged
    staged = cuda_lib.hs2_decode_stage(cuda(x.k_cache), cuda(x.v_cache), cuda(x.lengths),
                                       cuda(torch.from_numpy(bad)), Hq=16, W=16, k_top=64,
                                       k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale))
    assert cuda_lib.hs2_get_last_device_error() == cuda_lib.HS2_ERR_DEVICE_DATA
    o_s = cuda_lib.hs2_decode_sparse_staged(cuda(x.q_sparse[0]), staged, 4000, 16, 64)
    bad[1, 20] = -1
    ref = oracle.decode_sparse(x.q_sparse[0], x.k_cache, x.v_cache, torch.from_numpy(bad),
                               kv="e4m3", k_scale=x.k_scale, v_scale=x.v_scale)
    assert max_abs(o_s.float().cpu().numpy(), ref) <= TOL_E4M3
    assert cuda_lib.hs2_get_last_device_error() == 0


def test_split_full_attn_and_select_equal_the_combined_call(cuda_lib):
    x = inputs.make_prefill(2, 777, 16, 128, 128, 256, n_topics=8, seg=256,
                            seed=inputs.seed_for(0, 5))
    q, k, v = cuda(x.q), cuda(x.k_), cuda(x.v)
    o, lse, idx = cuda_lib.hs2_full_attn_select(q, k, v, x.W, x.k)
    o2, lse2 = cuda_lib.hs2_full_attn(q, k, v)
    idx2 = cuda_lib.hs2_select(q, k, lse2, x.W, x.k)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(torch.sort(idx, dim=-1).values, torch.sort(idx2, dim=-1).values)


def test_row_range_calls_equal_the_full_layer(cuda_lib):
    """The full layer in query-row chunks (each chunk reads only the K/V rows
    it needs) gives the whole call's O and lse bit for bit and the same
    selections."""
    x = inputs.make_prefill(2, 1000, 16, 128, 64, 256, n_topics=8, seg=256,
                            seed=inputs.seed_for(0, 6))
    B, L, Hq, d = x.q.shape
    q, k, v = cuda(x.q), cuda(x.k_), cuda(x.v)
    o, lse, idx = cuda_lib.hs2_full_attn_select(q, k, v, x.W, x.k)
    o2, lse2 = torch.full_like(o, 7.0), torch.full_like(lse, 7.0)
    idx2 = torch.full_like(idx, -7)
    ws = torch.empty(cuda_lib.hs2_full_attn_select_workspace(
        cuda_lib.prefill_shape(B, L, Hq, d, x.W, x.k)), dtype=torch.uint8, device="cuda")
    cuts = [0, 128, 384, 512, 1000]
    for r0, r1 in zip(cuts[:-1], cuts[1:]):
        cuda_lib.hs2_full_attn_rows(q, k, v, r0, r1, o=o2, lse=lse2)
    for r0, r1 in zip(cuts[:-1], cuts[1:]):
        cuda_lib.hs2_select_rows(q, k, lse2, x.W, x.k, r0, r1, idx=idx2, workspace=ws)
    torch.cuda.synchronize()
    assert cuda_lib.hs2_get_last_device_error() == 0
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(torch.sort(idx, dim=-1).values, torch.sort(idx2, dim=-1).values)
    # a chunk writes only its own rows
    o3 = torch.full_like(o, 7.0)
    cuda_lib.hs2_full_attn_rows(q, k, v, 128, 384, o=o3, lse=lse2)
    torch.cuda.synchronize()
    assert torch.equal(o3[:, 128:384], o[:, 128:384])
    assert bool((o3[:, :128] == 7.0).all()) and bool((o3[:, 384:] == 7.0).all())


# ------------------------------------------------ the largest index rows
# W + k = 2048, the largest selection the library accepts.

def test_full_attn_select_largest_selection(cuda_lib):
    x = inputs.make_prefill(1, 3000, 8, 128, 128, 1920, n_topics=8, seg=256,
                            seed=inputs.seed_for(0, 21), n_sparse=1)
    B, L, Hq, d = x.q.shape
    rows = sample_rows(B, L, 256, seed=4, seg=256)
    _, idx, ora, rows, n_swap, overlap = check_full_layer(cuda_lib, x, rows=rows)
    assert overlap > 0.999
    idx_t = torch.from_numpy(idx).view(B, L, -1)
    os_ = cuda_lib.hs2_sparse_attn(cuda(x.q_sparse[0]), cuda(x.k_), cuda(x.v), cuda(idx_t),
                                  W=x.W, k_top=x.k)
    ref = oracle.sparse(x.q_sparse[0], x.k_, x.v, idx_t, rows=rows)
    assert max_abs(os_.float().cpu().numpy().reshape(B * L, Hq, d)[rows], ref) <= TOL_BF16


def test_decode_select_largest_selection(cuda_lib):
    x = _decode_case("e4m3", 3, 30000, 16, 128, 1024, 1024, [30000, 12000, 1500],
                     seed=inputs.seed_for(3, 21))
    o, lse, idx = run_decode(cuda_lib, x)
    ora = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, x.W, x.k, kv="e4m3",
                               k_scale=x.k_scale, v_scale=x.v_scale, probe=idx)
    assert max_abs(o, ora["o"]) <= TOL_E4M3
    assert max_abs(lse, ora["lse"]) <= TOL_LSE
    t = x.lengths.numpy().astype(np.int64) - 1
    check_structure(idx, t, x.W, x.k)
    check_selection(idx, ora, t, x.W, x.k)
    ods = cuda_lib.hs2_decode_sparse(cuda(x.q_sparse[0]), cuda(x.k_cache), cuda(x.v_cache),
                                     cuda(x.lengths), cuda(torch.from_numpy(idx)), kv="e4m3",
                                     k_scale=cuda(x.k_scale), v_scale=cuda(x.v_scale),
                                     W=x.W, k_top=x.k)
    refd = oracle.decode_sparse(x.q_sparse[0], x.k_cache, x.v_cache, torch.from_numpy(idx),
                                kv="e4m3", k_scale=x.k_scale, v_scale=x.v_scale)
    assert max_abs(ods.float().cpu().numpy(), refd) <= TOL_E4M3


def test_bounded_wait_gives_up_and_reports_timeout(cuda_lib):
    """The bounded wait every pipelined kernel uses: a wait on a barrier that
    nothing arrives at gives up after its limit (1 ms here), records the
    timeout, and leaves the device usable -- the next call works and reports
    no error."""
    assert cuda_lib.hs2_get_last_device_error() == 0
    cuda_lib.hs2_check_bounded_wait(1000)
    assert cuda_lib.hs2_get_last_device_error() == cuda_lib.HS2_ERR_TIMEOUT
    assert cuda_lib.hs2_get_last_device_error() == 0  # reported once, then cleared
    x = inputs.make_prefill(1, 300, 16, 128, 16, 32, seed=41)
    o, lse, idx = run_full(cuda_lib, x)
    ora = oracle.full_select(x.q, x.k_, x.v, 16, 32, probe=idx)
    assert max_abs(o, ora["o"]) <= TOL_BF16
    check_selection(idx, ora, np.arange(300), 16, 32)
