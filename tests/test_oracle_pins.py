"""Pins of the fp64 oracle against things other than itself.

Each test ties one oracle function to a closed form, an invariant, a library
routine (torch float64 attention / softmax / logsumexp, numpy sort, torch's
e4m3 and bf16 casts), exhaustive enumeration on tiny inputs, or the
hand-worked example in tests/golden.  Method: HySparse2 summary
(onedev.kr/papers/146), 'What differs' and 'How to use' sections.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.parity import check_structure
from token_level_top_hs2_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(x):
    return x.double() if isinstance(x, torch.Tensor) else torch.as_tensor(x, dtype=torch.float64)


def ref_full(q, k, v, scale):
    """Causal MQA attention in float64 with torch's own routines."""
    B, L, Hq, d = q.shape
    qh = f64(q).permute(0, 2, 1, 3)                      # [B,Hq,L,d]
    kh = f64(k).unsqueeze(1).expand(B, Hq, L, d)
    vh = f64(v).unsqueeze(1).expand(B, Hq, L, d)
    o = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, is_causal=True, scale=scale)
    logits = torch.einsum("bhtd,bhsd->bhts", qh, kh) * scale
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    logits = logits.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)                # [B,Hq,L]
    p = torch.softmax(logits, dim=-1)
    score = p.sum(dim=1)                                 # [B,L,L]
    return o.permute(0, 2, 1, 3), lse.permute(0, 2, 1), score


# ----------------------------------------------------------------- formats

def test_e4m3_codes_from_format_definition():
    v = oracle.e4m3_value
    assert v(0x7E) == 448.0
    assert v(0xFE) == -448.0
    assert v(0x38) == 1.0
    assert v(0x08) == 2.0 ** -6          # smallest normal
    assert v(0x01) == 2.0 ** -9          # smallest subnormal
    assert v(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert v(0x00) == 0.0 and math.copysign(1, v(0x80)) == -1
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))


def test_e4m3_all_codes_match_torch_cast():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_bf16_all_bit_patterns_match_torch_cast():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_value(b) for b in range(0, 65536, 1)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


# ---------------------------------------------------- full attention rows

@pytest.mark.parametrize("B,L,Hq,d", [(1, 37, 4, 16), (2, 50, 16, 8), (1, 1, 4, 64)])
def test_full_attention_matches_torch_float64(B, L, Hq, d):
    x = inputs.make_prefill(B, L, Hq, d, 4, 8, n_topics=3, seg=16, seed=11 + L)
    r = oracle.full_select(x.q, x.k_, x.v, 4, 8, want_score_row=True)
    o, lse, score = ref_full(x.q, x.k_, x.v, x.scale)
    np.testing.assert_allclose(r["o"], o.reshape(B * L, Hq, d).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse.reshape(B * L, Hq).numpy(), rtol=0, atol=1e-12)
    sr = r["score_row"].reshape(B, L, L)
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(sr[:, tri], score.numpy()[:, tri], rtol=0, atol=1e-12)


def test_closed_form_all_keys_equal():
    """All keys equal: P_h(s) = 1/(t+1), so O(t) = mean(v_0..v_t),
    lse_h = l_h + log(t+1), score = Hq/(t+1)."""
    B, L, Hq, d = 1, 40, 4, 8
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    krow = torch.randn(d, generator=g).bfloat16()
    k = krow.expand(B, L, d).contiguous()
    v = torch.randn(B, L, d, generator=g).bfloat16()
    scale = 0.3
    r = oracle.full_select(q, k, v, 4, 8, scale=scale, want_score_row=True)
    vd = v.double()[0].numpy()
    for t in range(L):
        np.testing.assert_allclose(r["o"][t], np.broadcast_to(vd[: t + 1].mean(0), (Hq, d)),
                                   atol=1e-13)
        l = scale * (q[0, t].double() @ krow.double()).numpy()
        np.testing.assert_allclose(r["lse"][t], l + math.log(t + 1), atol=1e-13)
        np.testing.assert_allclose(r["score_row"][t, : t + 1], Hq / (t + 1), rtol=1e-13)


def test_single_token_sequence():
    """L = 1: O = v_0, lse = l_00, selection = {0}."""
    q = torch.randn(1, 1, 4, 16).bfloat16()
    k = torch.randn(1, 1, 16).bfloat16()
    v = torch.randn(1, 1, 16).bfloat16()
    r = oracle.full_select(q, k, v, 2, 3)
    np.testing.assert_array_equal(r["o"][0], np.broadcast_to(v.double()[0, 0].numpy(), (4, 16)))
    np.testing.assert_allclose(r["lse"][0], 0.25 * (q[0, 0].double() @ k[0, 0].double()).numpy(),
                               atol=1e-14)
    assert r["idx"][0].tolist() == [0, -1, -1, -1, -1]


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_full_select.json")))
    qrow = torch.tensor(g["q_row"], dtype=torch.float32)
    q = qrow.expand(1, 3, 2, 2).contiguous().bfloat16()
    k = torch.tensor(g["k"]).unsqueeze(0).bfloat16()
    v = torch.tensor(g["v"]).unsqueeze(0).bfloat16()
    r = oracle.full_select(q, k, v, g["W"], g["k_top"], scale=g["scale"], rows=[2],
                           want_score_row=True)
    ev = lambda s: eval(s, {"e": math.e, "log": math.log})  # closed forms from the fixture
    ex = g["expected"]
    np.testing.assert_allclose(r["lse"][0], [ev(s) for s in ex["lse"]], rtol=1e-15)
    np.testing.assert_allclose(r["o"][0], [[ev(s) for s in row] for row in ex["o"]], rtol=1e-15)
    assert r["idx"][0].tolist() == ex["idx"]
    np.testing.assert_allclose(r["sel_score"][0], [ev(s) for s in ex["sel_score"]], rtol=1e-15)
    np.testing.assert_allclose(r["score_row"][0], [ev(s) for s in ex["score"]], rtol=1e-15)


def test_probability_mass_summed_over_heads_is_Hq():
    x = inputs.make_prefill(2, 96, 16, 32, 8, 16, n_topics=4, seg=32, seed=3)
    r = oracle.full_select(x.q, x.k_, x.v, 8, 16, want_score_row=True)
    L = 96
    for row in range(2 * L):
        t = row % L
        assert abs(r["score_row"][row, : t + 1].sum() - 16) < 1e-12


# ------------------------------------------------------------- selection

def _independent_selection(score_row, t, W, k):
    """Window ascending, then the k best of 0..t-W by (score desc, index asc)
    via numpy's lexsort."""
    w = list(range(max(0, t - W + 1), t + 1))
    nc = t - W + 1
    if nc <= 0:
        return w, []
    cand = np.arange(nc)
    if nc <= k:
        return w, cand.tolist()
    order = np.lexsort((cand, -score_row[:nc]))
    return w, cand[order[:k]].tolist()


def test_selection_matches_full_sort_on_torch_scores():
    B, L, Hq, d, W, k = 1, 300, 4, 16, 16, 40
    x = inputs.make_prefill(B, L, Hq, d, W, k, n_topics=4, seg=32, seed=9)
    r = oracle.full_select(x.q, x.k_, x.v, W, k)
    _, _, score = ref_full(x.q, x.k_, x.v, x.scale)
    score = score.numpy()[0]
    for t in range(L):
        w, gsel = _independent_selection(score[t], t, W, k)
        got = r["idx"][t]
        got = got[got >= 0].tolist()
        assert got[: len(w)] == w
        assert sorted(got[len(w):]) == sorted(gsel), t
        assert got[len(w):] == gsel or len(gsel) <= k


def _certified_topk(scores, k):
    """Exhaustive: the unique k-subset G with key(x) > key(y) for x in G,
    y not in G, where key = (score, -index)."""
    n = len(scores)
    key = lambda i: (scores[i], -i)
    hits = []
    for G in itertools.combinations(range(n), k):
        rest = [y for y in range(n) if y not in G]
        if all(key(x) > key(y) for x in G for y in rest):
            hits.append(set(G))
    assert len(hits) == 1
    return hits[0]


def test_topk_against_exhaustive_enumeration_with_ties():
    """Tiny rows where many keys are identical (equal scores): the lower
    index must win every tie at the cut."""
    B, L, Hq, d, W, k = 1, 14, 2, 4, 2, 4
    g = torch.Generator().manual_seed(7)
    q = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    base = torch.randn(3, d, generator=g)
    pick = torch.tensor([0, 1, 0, 2, 1, 0, 0, 2, 1, 1, 0, 2, 0, 1])  # many duplicates
    k_ = base[pick].unsqueeze(0).bfloat16()
    v = torch.randn(B, L, d, generator=g).bfloat16()
    r = oracle.full_select(q, k_, v, W, k, want_score_row=True)
    n_cut = 0
    for t in range(L):
        nc = t - W + 1
        got = r["idx"][t]
        got = got[got >= 0].tolist()
        if nc <= k:
            assert got[min(t + 1, W):] == list(range(max(nc, 0)))
            continue
        G = _certified_topk(r["score_row"][t, :nc].tolist(), k)
        assert set(got[W:]) == G, t
        n_cut += 1
    assert n_cut > 0


def test_ties_at_the_cut_take_lower_indices():
    """Every key identical: all candidates tie, so the first k candidates win."""
    B, L, Hq, d, W, k = 1, 64, 4, 8, 4, 10
    q = torch.randn(B, L, Hq, d).bfloat16()
    k_ = torch.randn(d).bfloat16().expand(B, L, d).contiguous()
    v = torch.randn(B, L, d).bfloat16()
    r = oracle.full_select(q, k_, v, W, k)
    for t in range(W + k, L):
        assert r["idx"][t, W:].tolist() == list(range(k))


def test_selection_structure_invariants():
    B, L, Hq, d, W, k = 2, 200, 4, 16, 8, 24
    x = inputs.make_prefill(B, L, Hq, d, W, k, n_topics=4, seg=32, seed=21)
    r = oracle.full_select(x.q, x.k_, x.v, W, k)
    t = np.tile(np.arange(L), B)
    check_structure(r["idx"], t, W, k)
    # sigma_k is the score of the last global pick when a cut is made
    for row in range(B * L):
        tt = row % L
        if tt - W + 1 > k:
            assert r["sigma_k"][row] == r["sel_score"][row, W + k - 1]
            assert np.all(r["sel_score"][row, W:] >= r["sigma_k"][row])
        else:
            assert r["sigma_k"][row] == -1


def test_probe_scores_are_row_scores():
    x = inputs.make_prefill(1, 80, 4, 16, 4, 8, seed=2)
    probe = np.tile(np.array([0, 5, 79, -1, 40], dtype=np.int32), (80, 1))
    r = oracle.full_select(x.q, x.k_, x.v, 4, 8, probe=probe, want_score_row=True)
    for t in range(80):
        for j, p in enumerate(probe[t]):
            if 0 <= p <= t:
                assert r["probe_score"][t, j] == r["score_row"][t, p]
            else:
                assert math.isnan(r["probe_score"][t, j])


# ----------------------------------------------------------- sparse layer

def test_sparse_equals_full_when_budget_covers_the_row():
    """W + k >= t + 1 selects every position, so the sparse layer with the
    same queries reproduces full attention."""
    B, L, Hq, d, W, k = 2, 48, 4, 16, 8, 40
    x = inputs.make_prefill(B, L, Hq, d, W, k, seed=4)
    r = oracle.full_select(x.q, x.k_, x.v, W, k)
    o_sp = oracle.sparse(x.q, x.k_, x.v, r["idx"])
    np.testing.assert_allclose(o_sp, r["o"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_sparse_over_arbitrary_sets_matches_torch_float64(kv):
    """Sparse layer over random index sets (with -1 padding) against float64
    softmax attention on the gathered, dequantised rows."""
    B, L, Hq, d, S = 2, 64, 16, 32, 20
    g = torch.Generator().manual_seed(8)
    q = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    kf = torch.randn(B, L, d, generator=g) * 2
    vf = torch.randn(B, L, d, generator=g)
    if kv == "e4m3":
        kc, ks = inputs.quantize_e4m3_per_token(kf)
        vc, vs = inputs.quantize_e4m3_per_token(vf)
        kd = kc.view(torch.float8_e4m3fn).double() * ks.double().unsqueeze(-1)
        vd = vc.view(torch.float8_e4m3fn).double() * vs.double().unsqueeze(-1)
    else:
        kc, vc, ks, vs = kf.bfloat16(), vf.bfloat16(), None, None
        kd, vd = kc.double(), vc.double()
    idx = torch.full((B * L, S), -1, dtype=torch.int32)
    for row in range(B * L):
        t = row % L
        n = min(S, t + 1) - (row % 3 == 0 and t > 2)
        idx[row, :n] = torch.randperm(t + 1, generator=g)[:n].int()
    o = oracle.sparse(q, kc, vc, idx, kv=kv, k_scale=ks, v_scale=vs)
    for row in range(B * L):
        b = row // L
        sel = idx[row][idx[row] >= 0].long()
        qq = q[b, row % L].double()                              # [Hq,d]
        logits = qq @ kd[b, sel].T / math.sqrt(d)
        ref = torch.softmax(logits, dim=-1) @ vd[b, sel]
        np.testing.assert_allclose(o[row], ref.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ decode

def test_decode_matches_prefill_last_row_bf16_cache():
    """Decode at length T equals row T-1 of the prefill oracle on the same
    cache and query (bf16 cache, ragged lengths)."""
    B, Tmax, Hq, d, W, k = 3, 120, 4, 16, 8, 16
    x = inputs.make_decode(B, Tmax, Hq, d, W, k, kv="bf16", seed=6, lengths=[120, 57, 9],
                           n_needles=4)
    probe = np.tile(np.arange(W + k, dtype=np.int32), (B, 1))
    r = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv="bf16", probe=probe)
    for b in range(B):
        T = int(x.lengths[b])
        qf = x.q[b].unsqueeze(0).unsqueeze(0).expand(1, T, Hq, d).contiguous()
        p = oracle.full_select(qf, x.k_cache[b:b + 1, :T], x.v_cache[b:b + 1, :T], W, k,
                               rows=[T - 1], probe=probe[b:b + 1])
        np.testing.assert_array_equal(r["o"][b], p["o"][0])
        np.testing.assert_array_equal(r["lse"][b], p["lse"][0])
        np.testing.assert_array_equal(r["idx"][b], p["idx"][0])
        np.testing.assert_array_equal(r["probe_score"][b], p["probe_score"][0])


def test_decode_e4m3_matches_torch_float64():
    B, Tmax, Hq, d, W, k = 2, 300, 16, 32, 8, 32
    x = inputs.make_decode(B, Tmax, Hq, d, W, k, kv="e4m3", seed=12, lengths=[300, 200],
                           n_needles=3)
    r = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv="e4m3",
                             k_scale=x.k_scale, v_scale=x.v_scale)
    kd = x.k_cache.view(torch.float8_e4m3fn).double() * x.k_scale.double().unsqueeze(-1)
    vd = x.v_cache.view(torch.float8_e4m3fn).double() * x.v_scale.double().unsqueeze(-1)
    for b in range(B):
        T = int(x.lengths[b])
        logits = x.q[b].double() @ kd[b, :T].T / math.sqrt(d)        # [Hq,T]
        lse = torch.logsumexp(logits, dim=-1)
        p = torch.softmax(logits, dim=-1)
        np.testing.assert_allclose(r["lse"][b], lse.numpy(), atol=1e-12)
        np.testing.assert_allclose(r["o"][b], (p @ vd[b, :T]).numpy(), atol=1e-12)
        score = p.sum(0).numpy()
        w, gsel = _independent_selection(score, T - 1, W, k)
        got = r["idx"][b]
        got = got[got >= 0].tolist()
        assert got[: len(w)] == w and sorted(got[len(w):]) == sorted(gsel)


def test_decode_sparse_matches_prefill_sparse():
    B, Tmax, Hq, d, W, k = 2, 90, 4, 16, 8, 16
    x = inputs.make_decode(B, Tmax, Hq, d, W, k, kv="e4m3", seed=13, n_needles=2)
    r = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv="e4m3",
                             k_scale=x.k_scale, v_scale=x.v_scale)
    o = oracle.decode_sparse(x.q_sparse[0], x.k_cache, x.v_cache, r["idx"], kv="e4m3",
                             k_scale=x.k_scale, v_scale=x.v_scale)
    for b in range(B):
        qf = x.q_sparse[0][b].expand(1, Tmax, Hq, d).contiguous()
        idx = np.full((Tmax, W + k), -1, dtype=np.int32)
        idx[Tmax - 1] = r["idx"][b]
        ref = oracle.sparse(qf, x.k_cache[b:b + 1], x.v_cache[b:b + 1], idx, rows=[Tmax - 1],
                            kv="e4m3", k_scale=x.k_scale[b:b + 1], v_scale=x.v_scale[b:b + 1])
        np.testing.assert_array_equal(o[b], ref[0])


def test_planted_needles_are_selected():
    B, T, Hq, d, W, k = 4, 4096, 16, 128, 128, 64
    x = inputs.make_decode(B, T, Hq, d, W, k, kv="e4m3", seed=14, n_needles=16)
    r = oracle.decode_select(x.q, x.k_cache, x.v_cache, x.lengths, W, k, kv="e4m3",
                             k_scale=x.k_scale, v_scale=x.v_scale)
    for b in range(B):
        assert set(x.needle_pos[b].tolist()) <= set(r["idx"][b].tolist())


# ---------------------------------------------------------------- overlap
# Cross-layer overlap |T(i) ∩ T(j)| / k of the IndexCache page (Appendix A),
# applied to the global picks of HySparse2 selections.

def test_overlap_hand_worked_rows():
    # W = 2, k = 3, L = 6.  Row t: window t-1..t, candidates 0..t-2.
    W, K, L = 2, 3, 6
    a = -np.ones((1, L, W + K), dtype=np.int32)
    b = -np.ones((1, L, W + K), dtype=np.int32)
    a[0, 1, :2] = [0, 1]                 # t=1: window only -> ratio 1
    b[0, 1, :2] = [1, 0]
    a[0, 2, :3] = [1, 2, 0]              # t=2: one candidate, both take it -> 1/1
    b[0, 2, :3] = [0, 1, 2]
    a[0, 3, :4] = [2, 3, 0, 1]           # t=3: a takes {0,1}, b takes {1} of 2 -> 1/2
    b[0, 3, :4] = [2, 3, 1, -1]
    a[0, 5, :] = [4, 5, 3, 1, 0]         # t=5: {0,1,3} vs {1,2,3} -> 2/3
    b[0, 5, :] = [2, 1, 4, 3, 5]
    inter, ratio = oracle.selection_overlap(a, b, W, K)
    assert inter[0].tolist() == [0, 0, 1, 1, 0, 2]
    # t=0: no candidates; t=4: both empty of 3 candidates -> 0/3
    assert ratio[0].tolist() == [1.0, 1.0, 1.0, 0.5, 0.0, 2.0 / 3.0]


def test_overlap_against_brute_force_pair_count():
    rng = np.random.default_rng(7)
    W, K, L, B = 4, 16, 200, 2
    a = -np.ones((B, L, W + K), dtype=np.int32)
    b = -np.ones((B, L, W + K), dtype=np.int32)
    for bb in range(B):
        for t in range(L):
            n = min(t + 1, W + K)
            for arr in (a, b):
                picks = rng.choice(t + 1, size=n, replace=False)
                arr[bb, t, :n] = picks
    inter, ratio = oracle.selection_overlap(a, b, W, K)
    for bb in range(B):
        for t in range(L):
            # every (i, j) pair of global entries, counted with plain loops
            cnt = 0
            for x in a[bb, t]:
                for y in b[bb, t]:
                    if x == y and 0 <= x <= t - W:
                        cnt += 1
            assert inter[bb, t] == cnt
            if t >= W:
                assert ratio[bb, t] == cnt / min(K, t - W + 1)


def test_overlap_of_real_selections_matches_numpy_intersect():
    x = inputs.make_workload("prefill_tiny_1k")
    q2 = x.q_sparse[0]
    L = x.q.shape[1]
    idx_a = oracle.full_select(x.q, x.k_, x.v, x.W, x.k)["idx"].reshape(1, L, -1)
    idx_b = oracle.full_select(q2, x.k_, x.v, x.W, x.k)["idx"].reshape(1, L, -1)
    inter, ratio = oracle.selection_overlap(idx_a, idx_b, x.W, x.k)
    a, b = np.asarray(idx_a), np.asarray(idx_b)
    for t in range(L):
        ga = a[0, t][(a[0, t] >= 0) & (a[0, t] <= t - x.W)]
        gb = b[0, t][(b[0, t] >= 0) & (b[0, t] <= t - x.W)]
        assert inter[0, t] == np.intersect1d(ga, gb).size
    # a selection against itself: every row overlaps fully
    same_i, same_r = oracle.selection_overlap(idx_a, idx_a, x.W, x.k)
    assert np.all(same_r == 1.0)
    # a query with itself agrees; a fresh query mostly does not repeat the picks
    assert 0.0 <= ratio.mean() < 1.0


def test_overlap_ignores_slot_order_window_and_padding():
    rng = np.random.default_rng(3)
    W, K, L = 3, 5, 40
    a = -np.ones((1, L, W + K), dtype=np.int32)
    b = -np.ones((1, L, W + K), dtype=np.int32)
    for t in range(L):
        n = min(t + 1, W + K)
        a[0, t, :n] = rng.choice(t + 1, size=n, replace=False)
        b[0, t, :n] = rng.choice(t + 1, size=n, replace=False)
    i0, r0 = oracle.selection_overlap(a, b, W, K)
    a2 = a.copy()
    for t in range(L):
        a2[0, t] = rng.permutation(a2[0, t])
    i1, r1 = oracle.selection_overlap(a2, b, W, K)
    assert np.array_equal(i0, i1) and np.array_equal(r0, r1)


# ------------------------------------------------- block-level selector
# HySparse (the predecessor in the HySparse2 summary, "Limits"): 64-token
# blocks ranked by attention mass (page 3's reading: the sum of the attention
# scores inside a block), the same forced window.

def _independent_block_selection(score_row, t, W, k, block):
    """Masses as plain sums of torch float64 scores; blocks ranked by
    (mass desc, index asc) with numpy's lexsort; positions <= t-W."""
    w = list(range(max(0, t - W + 1), t + 1))
    last = t - W
    if last < 0:
        return w, [], np.zeros(0)
    nb = last // block + 1
    mass = np.array([score_row[block * j: min(block * j + block, last + 1)].sum()
                     for j in range(nb)])
    nsel = k // block
    if nb <= nsel:
        chosen = list(range(nb))
    else:
        order = np.lexsort((np.arange(nb), -mass))
        chosen = sorted(order[:nsel].tolist())
    return w, [s for j in chosen for s in range(block * j, min(block * j + block, last + 1))], mass


def test_block_selection_matches_torch_masses_and_sort():
    B, L, Hq, d, W, k, blk = 1, 700, 4, 16, 16, 256, 64
    x = inputs.make_prefill(B, L, Hq, d, W, k, n_topics=4, seg=32, seed=21)
    r = oracle.block_select(x.q, x.k_, x.v, W, k, block=blk)
    _, _, score = ref_full(x.q, x.k_, x.v, x.scale)
    score = score.numpy()[0]
    for t in range(L):
        w, glob, mass = _independent_block_selection(score[t], t, W, k, blk)
        got = r["idx"][t]
        got = got[got >= 0].tolist()
        assert got == w + glob, t
        np.testing.assert_allclose(r["mass"][t, : mass.size], mass, rtol=1e-12, atol=1e-15)


def test_block_selection_all_keys_equal_takes_the_first_full_blocks():
    """Uniform scores Hq/(t+1): every full candidate block has the same mass,
    a partial last block less; ties go to the lower blocks."""
    B, L, Hq, d, W, k, blk = 1, 600, 4, 8, 16, 128, 64
    g = torch.Generator().manual_seed(8)
    q = torch.randn(B, L, Hq, d, generator=g).bfloat16()
    krow = torch.randn(d, generator=g).bfloat16()
    kk = krow.expand(B, L, d).contiguous()
    v = torch.randn(B, L, d, generator=g).bfloat16()
    r = oracle.block_select(q, kk, v, W, k, block=blk)
    for t in [16, 79, 80, 143, 144, 300, 599]:
        last = t - W
        nb = last // blk + 1
        got = r["idx"][t]
        glob = got[got >= 0].tolist()[min(t + 1, W):]
        if nb <= k // blk:
            assert glob == list(range(last + 1))
        else:
            assert glob == list(range(2 * blk))  # blocks 0 and 1
        np.testing.assert_allclose(r["mass"][t, 0], min(blk, last + 1) * Hq / (t + 1),
                                   rtol=1e-12)


def test_block_selection_structure():
    B, L, Hq, d, W, k, blk = 2, 333, 8, 32, 8, 192, 64
    x = inputs.make_prefill(B, L, Hq, d, W, k, n_topics=4, seg=32, seed=22)
    r = oracle.block_select(x.q, x.k_, x.v, W, k, block=blk)
    for row in range(B * L):
        t = row % L
        got = r["idx"][row]
        sel = got[got >= 0]
        wl = min(t + 1, W)
        assert sel[:wl].tolist() == list(range(t - wl + 1, t + 1))
        glob = sel[wl:]
        assert len(glob) == len(set(glob.tolist())) and np.all(glob <= t - W)
        blocks = sorted(set((glob // blk).tolist()))
        assert len(blocks) <= k // blk
        for j in blocks:  # whole blocks, clipped at t-W
            want = list(range(blk * j, min(blk * j + blk, t - W + 1)))
            assert [s for s in glob.tolist() if s // blk == j] == want
