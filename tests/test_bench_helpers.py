"""bench.py's host-side measurement arithmetic (no GPU): the algorithmic work
counts the roofline fractions divide by, the clock-sample summary, and the
gate that keeps a DRAM-traffic record to the kernel sources it was taken on.

The expected work counts are the per-unit figures of the hot-path scope
(HySparse2 summary (onedev.kr/papers/146), "How to use": W = 128, k = 1024, MQA,
d = 128, up to 1M tokens) worked out by hand, not re-derived from bench.py's
own formulas."""
import io
import json

import pytest

import bench


def test_prefill_flops_at_128k():
    # 6 * d * Hq flops per causal pair (QK^T and PV in the exact pass, QK^T
    # again in the selection pass) over L(L+1)/2 pairs
    L, Hq, d = 131072, 16, 128
    pairs = L * (L + 1) // 2
    assert bench.prefill_flops(L, Hq, d) == 6 * d * Hq * pairs
    assert bench.prefill_flops(L, Hq, d) == pytest.approx(1.056e14, rel=1e-3)
    assert bench.prefill_flops(1, 4, 64) == 6 * 64 * 4  # one pair


def test_sparse_bytes_counts_min_t_plus_1_S_rows():
    # tiny case by enumeration: L = 5, S = 3 -> rows 1, 2, 3, 3, 3
    assert bench.sparse_bytes(5, 3, 4) == (1 + 2 + 3 + 3 + 3) * 2 * 4 * 2
    assert bench.sparse_bytes(2, 3, 4) == (1 + 2) * 2 * 4 * 2  # L < S
    # 128k, S = 1152, bf16: L*S rows less the S(S-1)/2 the first S-1 queries
    # cannot name, 512 bytes of K+V each; L*S*512 = 77.3 GB is the bound
    L, S = 131072, 1152
    assert bench.sparse_bytes(L, S, 128) == (L * S - S * (S - 1) // 2) * 512
    assert bench.sparse_bytes(L, S, 128) == pytest.approx(77.3e9, rel=5e-3)
    assert bench.sparse_bytes(131072, 1152, 128, esz=1) * 2 == bench.sparse_bytes(
        131072, 1152, 128)


def test_decode_bytes_264_per_token():
    # 128 B of K + 128 B of V (e4m3) + two fp32 scales per cached token
    assert bench.decode_bytes(1, 1, 128) == 264
    assert bench.decode_bytes(16, 262144, 128) == pytest.approx(1.107e9, rel=1e-3)
    assert bench.decode_bytes(4, 1 << 20, 128) == bench.decode_bytes(16, 262144, 128)


def test_whole_job_rate_is_all_units_over_slowest_rank():
    assert bench.whole_job_rate(1, 131072, 0.5) == 262144
    assert bench.whole_job_rate(4, 100, 2.0) == 200


def _clocks_from(text):
    c = bench.Clocks(0, enabled=False)
    c.proc = object()  # stands for a sampler that ran
    c.f = io.StringIO(text)
    return c.summary()


def test_clock_summary_median_max_and_active_reasons():
    rows = [
        "1900, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active",
        "1920, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
        "1930, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "[N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",  # skipped
        "short line",
    ]
    s = _clocks_from("\n".join(rows) + "\n")
    assert s["sm_mhz"] == 1920 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    s = _clocks_from("1500, 1965, 700, 0x8, Active, Not Active, Active, Not Active\n")
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert _clocks_from("") is None
    assert bench.Clocks(0, enabled=False).summary() is None


def test_traffic_record_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    rec = {"csrc_hash": "0123456789abcdef", "kernels": {"decode_select": 1263116800}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_hash", lambda: "0123456789abcdef")
    assert bench.traffic_for("decode_select") == 1263116800
    assert bench.traffic_for("no_such_kernel") is None
    # counters taken on other kernel sources are not reported
    monkeypatch.setattr(bench, "csrc_hash", lambda: "fedcba9876543210")
    assert bench.traffic_for("decode_select") is None
    # nor is anything without a record
    (tmp_path / "profiles" / "traffic.json").unlink()
    assert bench.traffic_for("decode_select") is None


def test_source_hash_covers_every_kernel_source():
    h = bench.csrc_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    assert h == bench.csrc_hash()  # deterministic


def test_e2e_chunks_are_valid_row_ranges():
    # the row-range calls need chunk starts on 128-row query blocks and ends on
    # a block boundary or at L; the chunks tile [0, L)
    for L in (131072, 32768, 1024, 1000, 300):
        attn, sel = bench.e2e_chunks(L)
        for cuts in (attn, sel):
            assert cuts[0] == 0 and cuts[-1] == L
            assert all(a < b for a, b in zip(cuts[:-1], cuts[1:]))
            assert all(c % 128 == 0 for c in cuts[:-1])
    attn, sel = bench.e2e_chunks(131072)
    assert attn == [0, 32768, 65536, 131072]
    assert sel == [0, 131072 - 148 * 128, 131072]  # the last wave of query blocks
