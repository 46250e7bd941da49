"""The seeded input recipe (no method arithmetic): the structure it plants,
its formats and its determinism."""
import numpy as np
import torch

from token_level_top_hs2_b200 import inputs


def test_prefill_structure_and_determinism():
    a = inputs.make_prefill(2, 700, 4, 64, 16, 32, n_topics=5, seg=64, seed=17, n_sparse=2)
    b = inputs.make_prefill(2, 700, 4, 64, 16, 32, n_topics=5, seg=64, seed=17, n_sparse=2)
    assert torch.equal(a.q, b.q) and torch.equal(a.k_, b.k_) and torch.equal(a.v, b.v)
    assert a.q.dtype == torch.bfloat16 and a.k_.shape == (2, 700, 64)
    assert len(a.q_sparse) == 2 and a.q_sparse[0].shape == a.q.shape
    # 1% of the key positions, distinct, each with a topic; one topic per segment
    assert a.planted_pos.shape == (2, 7)
    for bb in range(2):
        assert len(set(a.planted_pos[bb].tolist())) == 7
    assert int(a.planted_pos.max()) < 700 and int(a.planted_topic.max()) < 5
    assert a.segment_topic.shape == (2, (700 + 63) // 64)
    # every head of a query in segment s leans towards that segment's topic:
    # the query rows of one segment share a mean direction
    q = a.q[0].float()
    seg0 = q[:64].mean(dim=(0, 1))
    seg_other = q[64 * 3: 64 * 4].mean(dim=(0, 1))
    same = int(a.segment_topic[0, 0]) == int(a.segment_topic[0, 3])
    cos = float(torch.nn.functional.cosine_similarity(seg0, seg_other, dim=0))
    assert (cos > 0.8) if same else True
    assert seg0.norm() > 2.0  # +3 u_c on top of N(0,1) noise averaged away


def test_decode_needles_scales_and_codes():
    x = inputs.make_decode(3, 5000, 16, 128, 128, 256, kv="e4m3", seed=5, n_sparse=1,
                           lengths=[5000, 2000, 100])
    assert x.k_cache.dtype == torch.uint8 and x.k_scale.shape == (3, 5000)
    for bb, length in enumerate([5000, 2000, 100]):
        pos = x.needle_pos[bb][x.needle_pos[bb] >= 0]
        span = max(1, length - 128)
        assert pos.numel() == min(16, span) and int(pos.max()) < span
        assert len(set(pos.tolist())) == pos.numel()
    # per-token e4m3: the largest |code value| of a row is 448 (its scale is max|x|/448)
    vals = x.k_cache[:, :50].view(torch.float8_e4m3fn).float()
    amax = vals.abs().amax(dim=-1)
    assert torch.all(amax == 448.0)
    assert torch.all(x.k_scale > 0)


def test_quantizer_roundtrip_within_e4m3_precision():
    g = torch.Generator().manual_seed(3)
    xr = torch.randn(64, 128, generator=g)
    xr[5] = 0.0
    codes, scale = inputs.quantize_e4m3_per_token(xr)
    back = codes.view(torch.float8_e4m3fn).float() * scale.unsqueeze(-1)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for values in the
    # normal range of each row (the largest ones), exact zeros stay zero
    big = xr.abs() > xr.abs().amax(dim=-1, keepdim=True) / 16
    rel = ((back - xr).abs() / xr.abs().clamp_min(1e-30))[big]
    assert float(rel.max()) <= 2.0 ** -4
    assert torch.all(back[5] == 0) and float(scale[5]) == 1.0


def test_selection_pair_rows_are_valid_selections():
    a, b = inputs.make_selection_pair(2, 400, 16, 48, seed=9)
    for arr in (a, b):
        for bb in range(2):
            for t in (0, 15, 16, 63, 64, 399):
                r = arr[bb, t]
                v = r[r >= 0]
                assert v.numel() == min(t + 1, 64)
                assert len(set(v.tolist())) == v.numel() and int(v.max()) <= t
                win = set(range(max(0, t - 15), t + 1))
                assert win <= set(v.tolist())
