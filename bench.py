"""Benchmark of the token-level KV Reuse hot path on B200.

One step = one pass of the whole hot path over synthetic inputs:
  prefill at 128k tokens (B=1, L=131072, Hq=16, d=128, W=128, k=1024):
      hs2_full_attn_select, then 3 sparse layers (hs2_sparse_attn) reusing its
      indices and the bf16 KV;
  decode at 256k tokens (B=16, T=262144, e4m3 KV with per-token scales):
      hs2_decode_select, then 3 decode sparse layers.
Reported `value` is the first figure of the metric, prefill tokens/s of the
full-attention + selection layer; the sparse-layer tokens/s and the decode
microseconds per step are in `components`.  Every kernel is timed with CUDA
events on the stream it runs on, with L2 flushed (256 MB write) before each
timed piece.  Multi-GPU runs (torchrun) are weak scaling: every rank runs its
own step on its own inputs, with no data-path collective.

--impl reference times the fp64 CPU oracle (tests' reference) on bounded
samples of the same workload on the host cores.
"""
import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s (full+select, sparse layer) at 128k; decode µs/step at 256k"
PREFILL = "prefill_128k"
DECODE = "decode_256k_b16"
# the other workloads, each measured after the timed step
OTHER_PREFILL = ["prefill_tiny_1k", "prefill_32k"]
OTHER_DECODE = ["decode_1m_b4"]
N_SPARSE = 3
FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--prefill", default=PREFILL)
    p.add_argument("--decode", default=DECODE)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads measured after the timed step")
    p.add_argument("--once", action="store_true",
                   help="call each bench kernel once on the workloads, untimed (for profilers)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sust=d.get("bf16_tflops_sustained", d["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


def csrc_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "token_level_top_hs2_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    if d.get("csrc_hash") != csrc_hash():
        return None
    return d.get("kernels", {}).get(kernel)


class Clocks:
    """nvidia-smi sampler running while the timed region runs."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, enabled=True):
        self.index, self.enabled, self.proc = index, enabled, None

    def __enter__(self):
        if self.enabled:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                     "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                    stderr=subprocess.DEVNULL)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        if not self.proc:
            return None
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus, backend=None):
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the
    environment); NCCL on GPUs, gloo for host-only checks."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
    if world > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def _dev():
    return "cuda" if torch.cuda.is_available() else "cpu"


def max_over_ranks(vals, world):
    """Element-wise maximum of a list of floats over all ranks."""
    t = torch.tensor(vals, dtype=torch.float64, device=_dev())
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def whole_job_rate(world, units_per_rank, t_max_s):
    """Weak scaling: every rank processes units_per_rank in its own timed
    region; the job's rate is all units over the slowest rank's time."""
    return world * units_per_rank / t_max_s


# ------------------------------------------------------------- workloads
def prefill_flops(L, Hq, d):
    """Tensor flops the two-pass method executes: QK^T + PV in pass 1 and QK^T
    again in pass 2 over the L(L+1)/2 causal pairs."""
    return 3.0 * d * Hq * L * (L + 1)


def sparse_bytes(L, S, d, esz=2):
    """Logical gathered K+V bytes of one sparse layer: each token reads
    min(t+1, S) rows of K and V (no reuse across tokens assumed)."""
    n = sum(min(t + 1, S) for t in range(0, min(L, S))) + max(0, L - S) * S
    return float(n) * 2 * d * esz


def decode_bytes(B, T, d):
    """HBM bytes of one decode select: every cached token read once,
    K and V e4m3 rows plus two fp32 scales."""
    return float(B) * T * (2 * d + 8)


class PrefillWork:
    """One prefill workload resident on the device: the full-attention select
    layer and its sparse layers reusing the selection and the bf16 KV."""

    def __init__(self, hs2, name, dev, repeat, n_sparse=N_SPARSE):
        from token_level_top_hs2_b200 import inputs
        x = inputs.make_workload(name, repeat=repeat)
        self.name, self.x = name, x
        self.B, self.L, self.Hq, self.d = B, L, Hq, d = x.q.shape
        self.W, self.K = W, K = x.W, x.k
        self.q, self.k, self.v = x.q.to(dev), x.k_.to(dev), x.v.to(dev)
        self.qs = [t.to(dev) for t in x.q_sparse[:n_sparse]]
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(B, L, Hq, dtype=torch.float32, device=dev)
        self.idx = torch.empty(B, L, W + K, dtype=torch.int32, device=dev)
        self.os_ = torch.empty_like(self.q)
        self.ws = torch.empty(hs2.hs2_full_attn_select_workspace(
            hs2.prefill_shape(B, L, Hq, d, W, K)), dtype=torch.uint8, device=dev)
        self.hs2 = hs2

    def full(self):
        self.hs2.hs2_full_attn_select(self.q, self.k, self.v, self.W, self.K, o=self.o,
                                      lse=self.lse, idx=self.idx, workspace=self.ws)

    def sparse(self, j):
        self.hs2.hs2_sparse_attn(self.qs[j], self.k, self.v, self.idx, W=self.W, k_top=self.K,
                                 o=self.os_)

    def pieces(self, prefix=""):
        return [(prefix + "full_select", self.full)] + [
            (prefix + f"sparse{j}", (lambda j=j: self.sparse(j))) for j in range(len(self.qs))]

    def flops(self):
        return prefill_flops(self.L, self.Hq, self.d) * self.B

    def sparse_bytes(self):
        return sparse_bytes(self.L, self.W + self.K, self.d) * self.B


class DecodeWork:
    """One decode workload resident on the device: the decode select and its
    sparse layers over an e4m3 cache with per-token scales."""

    def __init__(self, hs2, name, dev, repeat, n_sparse=N_SPARSE):
        from token_level_top_hs2_b200 import inputs
        x = inputs.make_workload(name, repeat=repeat)
        self.name, self.x = name, x
        self.B, self.Hq, self.d = B, Hq, d = x.q.shape
        self.T, self.W, self.K, self.kv = x.Tmax, x.W, x.k, x.kv
        self.q = x.q.to(dev)
        self.qs = [t.to(dev) for t in x.q_sparse[:n_sparse]]
        self.kc, self.vc = x.k_cache.to(dev), x.v_cache.to(dev)
        self.ks, self.vs = x.k_scale.to(dev), x.v_scale.to(dev)
        self.lens = x.lengths.to(dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
        self.idx = torch.empty(B, x.W + x.k, dtype=torch.int32, device=dev)
        self.os_ = torch.empty_like(self.q)
        self.ws = torch.empty(hs2.hs2_decode_select_workspace(
            hs2.decode_shape(B, self.T, Hq, d, x.W, x.k, x.kv)), dtype=torch.uint8, device=dev)
        self.staged = torch.empty(hs2.load().hs2_decode_stage_workspace(
            ctypes.byref(hs2.decode_shape(B, self.T, Hq, d, x.W, x.k, x.kv))),
            dtype=torch.uint8, device=dev)
        self.hs2 = hs2
        self.graph = self.graph_staged = None

    def select(self):
        self.hs2.hs2_decode_select(self.q, self.kc, self.vc, self.lens, self.W, self.K,
                                   kv=self.kv, k_scale=self.ks, v_scale=self.vs, o=self.o,
                                   lse=self.lse, idx=self.idx, workspace=self.ws)

    def sparse(self, j):
        self.hs2.hs2_decode_sparse(self.qs[j], self.kc, self.vc, self.lens, self.idx, kv=self.kv,
                                   k_scale=self.ks, v_scale=self.vs, W=self.W, k_top=self.K,
                                   o=self.os_)

    def step(self):
        self.select()
        for j in range(len(self.qs)):
            self.sparse(j)

    def step_staged(self):
        # the same step with the selected rows staged once for all sparse layers
        self.select()
        self.hs2.hs2_decode_stage(self.kc, self.vc, self.lens, self.idx, Hq=self.Hq, W=self.W,
                                  k_top=self.K, kv=self.kv, k_scale=self.ks, v_scale=self.vs,
                                  staged=self.staged)
        for j in range(len(self.qs)):
            self.hs2.hs2_decode_sparse_staged(self.qs[j], self.staged, self.T, self.W, self.K,
                                              kv=self.kv, o=self.os_)

    def capture(self):
        """The decode step as CUDA graphs (launch-bound inner loop)."""
        self.step()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        self.graph.replay()
        self.step_staged()
        self.graph_staged = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_staged):
            self.step_staged()
        self.graph_staged.replay()

    def pieces(self, prefix=""):
        return ([(prefix + "decode_select", self.select)] +
                [(prefix + f"decode_sparse{j}", (lambda j=j: self.sparse(j)))
                 for j in range(len(self.qs))] +
                [(prefix + "decode_step_graph", lambda: self.graph.replay()),
                 (prefix + "decode_step_graph_staged", lambda: self.graph_staged.replay())])

    def select_bytes(self):
        return decode_bytes(self.B, self.T, self.d)

    def sparse_bytes(self):
        return float(self.B) * (self.W + self.K) * (2 * self.d + 8)


def time_pieces(pieces, steps, flush, stream, times):
    """Time every piece `steps` times with CUDA events on the launching
    stream, L2 flushed (a 256 MB write) before each."""
    for _ in range(steps):
        evs = []
        for name, fn in pieces:
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((name, e0, e1))
        torch.cuda.synchronize()
        for name, a, b in evs:
            times.setdefault(name, []).append(a.elapsed_time(b))


def roof(kernel, bound, work, t, peak, unit, peak_src, traffic=None):
    """Roofline row: achieved = algorithmic work / time against the measured peak."""
    ach = work / t / (1e12 if unit == "TFLOP/s" else 1e9)
    return {"kernel": kernel, "bound": bound, "achieved": round(ach, 2), "peak": peak,
            "unit": unit, "frac": round(ach / peak, 4), "traffic": traffic,
            "peak_source": peak_src}


def gather_roof(kernel, logical_bytes, t, P):
    """Roofline row of a gather kernel.  achieved = the DRAM bytes ncu measured
    for this launch (profiles/traffic.json, while the kernel sources match) over
    the time, against the HBM peak; the logical gathered bytes (rows served from
    L2 count every time they are read) are reported beside it."""
    tr = traffic_for(kernel)
    logical = logical_bytes / t / 1e9
    if tr is not None:
        r = roof(kernel, "hbm", tr, t, P["hbm"], "GB/s", f"hbm_gbs ({P['src']})", traffic=tr)
        r["achieved_basis"] = "measured DRAM bytes per launch / time"
    else:
        r = {"kernel": kernel, "bound": "hbm", "achieved": None, "peak": P["hbm"],
             "unit": "GB/s", "frac": None, "traffic": None,
             "peak_source": f"hbm_gbs ({P['src']})",
             "achieved_basis": "no DRAM counters for the current kernel sources"}
    r["logical_gbs"] = round(logical, 2)
    r["logical_frac"] = round(logical / P["hbm"], 4)
    return r


def run_ours(args, world, rank, local):
    import token_level_top_hs2_b200 as hs2

    hs2.load()
    dev = torch.device("cuda", local)
    P = peaks()
    pf = PrefillWork(hs2, args.prefill, dev, rank)
    dc = DecodeWork(hs2, args.decode, dev, rank)
    B, L, Hq, d, W, K = pf.B, pf.L, pf.Hq, pf.d, pf.W, pf.K
    S = W + K
    nsp, ndsp = len(pf.qs), len(dc.qs)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    if args.once:
        # one call of each bench entry point on the workloads, untimed (for
        # profilers), in a fixed order: full+select (pass 1, selection, gated
        # re-run), a sparse layer, decode select (zeroing, pass 1, the sketch
        # selection with its exact fallback), a decode sparse layer, a
        # second full layer with the first sparse layer's queries and the
        # overlap of the two selections, the block-level selector
        pf.full()
        pf.sparse(0)
        dc.select()
        dc.sparse(0)
        own = torch.empty_like(pf.idx)
        hs2.hs2_full_attn_select(pf.qs[0], pf.k, pf.v, W, K, o=pf.os_, lse=pf.lse, idx=own,
                                 workspace=pf.ws)
        hs2.hs2_selection_overlap(pf.idx, own, W, K)
        hs2.hs2_full_attn_select_blocks(pf.q, pf.k, pf.v, W, K, o=pf.o, lse=pf.lse)
        torch.cuda.synchronize()
        assert hs2.hs2_get_last_device_error() == 0
        if rank == 0:
            print("once: ok", flush=True)
        return

    # cross-layer overlap (diagnostic): the inherited selection against the one
    # the first sparse layer's own queries give, made once outside the timing
    idx_own = torch.empty_like(pf.idx)
    inter = torch.empty(B, L, dtype=torch.int32, device=dev)
    ratio = torch.empty(B, L, dtype=torch.float32, device=dev)
    hs2.hs2_full_attn_select(pf.qs[0], pf.k, pf.v, W, K, o=pf.os_, lse=pf.lse, idx=idx_own,
                             workspace=pf.ws)

    def overlap():
        hs2.hs2_selection_overlap(pf.idx, idx_own, W, K, inter=inter, ratio=ratio)

    # HySparse's block-level selector on the same layer (64-token blocks)
    bws = torch.empty(hs2.hs2_full_attn_select_blocks_workspace(
        hs2.prefill_shape(B, L, Hq, d, W, K), 64), dtype=torch.uint8, device=dev)
    bidx = torch.empty_like(pf.idx)

    def full_blocks():
        hs2.hs2_full_attn_select_blocks(pf.q, pf.k, pf.v, W, K, o=pf.o, lse=pf.lse, idx=bidx,
                                        workspace=bws)

    # the other workloads, measured after the timed step: the tiny and 32k
    # prefills and the 1M-token decode (each rank its own inputs)
    others = []
    if not args.no_configs:
        for name in OTHER_PREFILL:
            if name != args.prefill:
                others.append(PrefillWork(hs2, name, dev, rank))
        for name in OTHER_DECODE:
            if name != args.decode:
                others.append(DecodeWork(hs2, name, dev, rank))

    # kernels per call: full select 3 (pass 1, pass 2 + selection, and pass 2
    # again gated: it returns at once unless a query block failed the check of
    # its speculative thresholds); sparse 1; decode select 3 (workspace zeroing,
    # pass 1, the sketch selection, which runs the exact fallback itself for a
    # sequence whose candidates overflow); decode sparse 1; stage 1; overlap 1;
    # block selector 3
    full_launches, dsel_launches = 3, 3

    def launches(work):
        if isinstance(work, PrefillWork):
            return full_launches + len(work.qs)
        n = len(work.qs)
        # the eager calls, then the two graphs (gathered rows; rows staged once)
        return (dsel_launches + n) * 2 + dsel_launches + 1 + n

    step_pieces = pf.pieces() + dc.pieces()[:1 + ndsp]
    graph_pieces = dc.pieces()[1 + ndsp:]
    extras = [("overlap", overlap), ("full_select_blocks", full_blocks)]
    for _ in range(args.warmup):
        for _, fn in step_pieces + extras:
            fn()
    dc.capture()
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == 0

    times = {}
    barrier(world)
    with Clocks(local, not args.no_clocks) as clk:
        barrier(world)
        t_wall = time.perf_counter()
        time_pieces(step_pieces + graph_pieces + extras, args.steps, flush, stream, times)
        barrier(world)
        wall = time.perf_counter() - t_wall
    assert hs2.hs2_get_last_device_error() == 0
    n_launch = (launches(pf) + launches(dc) + 1 + 3) * args.steps

    # worst case of the full layer: the same queries and keys with key
    # relevance falling along the sequence (early keys score higher), so the
    # selection's speculative stream thresholds fail on many query blocks and
    # their gated exact re-run does the work again
    worst = None
    if not args.no_configs:
        g = torch.Generator(device="cpu").manual_seed(32)
        u = torch.randn(d, generator=g)
        u = (u / u.norm()).to(dev)
        ramp = 6.0 * (1.0 - torch.arange(L, dtype=torch.float32, device=dev) / L)
        kw = (pf.k.float() + ramp[None, :, None] * u).bfloat16()
        qw = (pf.q.float() + 3.0 * u).bfloat16()
        del ramp

        def full_worst():
            hs2.hs2_full_attn_select(qw, kw, pf.v, W, K, o=pf.o, lse=pf.lse, idx=pf.idx,
                                     workspace=pf.ws)
        for _ in range(args.warmup):
            full_worst()
        torch.cuda.synchronize()
        time_pieces([("full_select_decaying_keys", full_worst)], args.steps, flush, stream, times)
        n_launch += full_launches * args.steps
        nqb = (L + 127) // 128
        fail_off = (B * L * Hq * 4 + 255) // 256 * 256
        worst = int(pf.ws[fail_off: fail_off + 4 * B * nqb].view(torch.int32).sum().item())
        del qw, kw

    # the other workloads: warm-up, then the same number of timed repetitions
    for w in others:
        if isinstance(w, DecodeWork):
            for _ in range(args.warmup):
                w.step()
            w.capture()
        else:
            for _ in range(args.warmup):
                for _, fn in w.pieces():
                    fn()
        torch.cuda.synchronize()
        time_pieces(w.pieces(w.name + "/"), args.steps, flush, stream, times)
        n_launch += launches(w) * args.steps
    assert hs2.hs2_get_last_device_error() == 0

    names = list(times)
    avg = max_over_ranks([sum(times[n]) / len(times[n]) for n in names], world)
    ms = dict(zip(names, avg))

    def prefill_summary(w, prefix=""):
        t_full = ms[prefix + "full_select"] / 1e3
        t_sp = sum(ms[prefix + f"sparse{j}"] for j in range(len(w.qs))) / len(w.qs) / 1e3
        r = roof("full_attn_select", "tensor", w.flops(), t_full, P["bf16"], "TFLOP/s",
                 f"bf16_tflops, burst ({P['src']})")
        return {"workload": w.name, "B": w.B, "L": w.L, "Hq": w.Hq, "d": w.d, "W": w.W,
                "k": w.K, "full_select_ms": round(t_full * 1e3, 4),
                "full_select_tok_s": round(world * w.B * w.L / t_full, 1),
                "full_select_tflops": r["achieved"], "full_select_frac_of_burst": r["frac"],
                "full_select_frac_of_sustained": round(r["achieved"] / P["bf16_sust"], 4),
                "sparse_layer_ms": round(t_sp * 1e3, 4),
                "sparse_layer_tok_s": round(world * w.B * w.L / t_sp, 1),
                "sparse_logical_gbs": round(w.sparse_bytes() / t_sp / 1e9, 1),
                "n_sparse_layers": len(w.qs)}

    def decode_summary(w, prefix=""):
        t_sel = ms[prefix + "decode_select"] / 1e3
        t_sp = sum(ms[prefix + f"decode_sparse{j}"] for j in range(len(w.qs))) / len(w.qs) / 1e3
        t_step = ms[prefix + "decode_step_graph"] / 1e3
        return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "d": w.d, "W": w.W,
                "k": w.K, "kv": w.kv, "us_per_step": round(t_step * 1e6, 1),
                "us_per_step_unfused_calls": round((t_sel + len(w.qs) * t_sp) * 1e6, 1),
                "us_per_step_staged_rows": round(ms[prefix + "decode_step_graph_staged"] * 1e3,
                                                 1),
                "select_us": round(t_sel * 1e6, 1),
                "select_gbs": round(w.select_bytes() / t_sel / 1e9, 1),
                "select_frac_of_hbm": round(w.select_bytes() / t_sel / 1e9 / P["hbm"], 4),
                "sparse_layer_us": round(t_sp * 1e6, 1),
                "sparse_gbs": round(w.sparse_bytes() / t_sp / 1e9, 1),
                "sparse_frac_of_hbm": round(w.sparse_bytes() / t_sp / 1e9 / P["hbm"], 4),
                "n_sparse_layers": len(w.qs)}

    cfg = {pf.name: prefill_summary(pf), dc.name: decode_summary(dc)}
    if worst is not None:
        t_w = ms["full_select_decaying_keys"] / 1e3
        cfg[pf.name]["full_select_decaying_keys_ms"] = round(t_w * 1e3, 4)
        cfg[pf.name]["full_select_decaying_keys_tok_s"] = round(world * B * L / t_w, 1)
        cfg[pf.name]["full_select_decaying_keys_failed_query_blocks"] = worst
        cfg[pf.name]["full_select_decaying_keys_note"] = (
            "worst case: key relevance falling along the sequence (+6u ramp on keys, +3u on "
            "queries) defeats the speculative stream thresholds; the failed query blocks are "
            "recomputed by the gated exact re-run")
    for w in others:
        cfg[w.name] = (prefill_summary(w, w.name + "/") if isinstance(w, PrefillWork)
                       else decode_summary(w, w.name + "/"))

    t_full = ms["full_select"] / 1e3
    t_sparse = sum(ms[f"sparse{j}"] for j in range(nsp)) / nsp / 1e3
    t_dsel = ms["decode_select"] / 1e3
    t_dsp = sum(ms[f"decode_sparse{j}"] for j in range(ndsp)) / ndsp / 1e3
    t_dstep = ms["decode_step_graph"] / 1e3
    t_ovl = ms["overlap"] / 1e3
    t_blk = ms["full_select_blocks"] / 1e3
    ms_per_step = sum(ms[n] for n, _ in step_pieces)

    value = whole_job_rate(world, B * L, t_full)
    ovl_bytes = float(B) * L * (2 * S * 4 + 8)
    burst = f"bf16_tflops, burst: the kernel is timed alone ({P['src']})"
    kernels = [
        roof("full_attn_select", "tensor", pf.flops(), t_full, P["bf16"], "TFLOP/s", burst,
             traffic_for("full_attn_select")),
        gather_roof("sparse_attn", pf.sparse_bytes(), t_sparse, P),
        roof("decode_select", "hbm", dc.select_bytes(), t_dsel, P["hbm"], "GB/s",
             f"hbm_gbs ({P['src']})", traffic_for("decode_select")),
        gather_roof("decode_sparse", dc.sparse_bytes(), t_dsp, P),
        gather_roof("selection_overlap", ovl_bytes, t_ovl, P),
        roof("full_attn_select_blocks", "tensor", pf.flops(), t_blk, P["bf16"], "TFLOP/s", burst,
             traffic_for("full_attn_select_blocks")),
    ]
    for kk in (kernels[0], kernels[5]):
        kk["frac_of_sustained_peak"] = round(kk["achieved"] / P["bf16_sust"], 4)
    kernels[0]["work"] = "3*d*Hq*L*(L+1) flops (pass 1 QK^T+PV, pass 2 QK^T)"
    kernels[1]["work"] = "sum_t min(t+1,S)*2*d*2 logical gathered bytes"
    kernels[2]["work"] = "B*T*(2d+8) bytes (e4m3 K,V rows + 2 fp32 scales)"
    kernels[3]["work"] = "B*S*(2d+8) bytes"
    kernels[4]["work"] = "B*L*(2*S*4 + 8) bytes (two idx rows in, count and ratio out)"
    kernels[5]["work"] = "3*d*Hq*L*(L+1) flops (as full_attn_select; 64-token block selection)"

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded planted-topic prefill, needle decode; no datasets)",
        "config": {"workload": f"{args.prefill} + {args.decode}", "prefill_B": B, "L": L,
                   "Hq": Hq, "d": d, "W": W, "k": K, "n_sparse_layers": nsp,
                   "decode_B": dc.B, "T": dc.T, "kv_decode": dc.kv, "l2": "flushed (256 MB "
                   "write) before every timed kernel", "parallelism": f"replicas x{world}"},
        "components": {
            "prefill_full_select_tok_s": round(world * B * L / t_full, 1),
            "prefill_sparse_layer_tok_s": round(world * B * L / t_sparse, 1),
            "decode_us_per_step": round(t_dstep * 1e6, 1),
            "decode_us_per_step_unfused_calls": round((t_dsel + ndsp * t_dsp) * 1e6, 1),
            "decode_us_per_step_staged_rows": round(ms["decode_step_graph_staged"] * 1e3, 1),
            "decode_select_us": round(t_dsel * 1e6, 1),
            "decode_sparse_us": round(t_dsp * 1e6, 1),
            "selection_overlap_us": round(t_ovl * 1e6, 1),
            "selection_overlap_mean": round(float(ratio.double().mean()), 4),
            "prefill_block_select_tok_s": round(world * B * L / t_blk, 1),
            "configs": cfg,
            "ms": {n: round(x, 4) for n, x in ms.items()},
        },
        "roofline": kernels[0],
        "kernels": kernels,
        "gpu_launches": n_launch,
        "gpu_launches_note": f"timed step: {full_launches} full-select (1 gated re-run) + {nsp} "
                             f"sparse + {dsel_launches} decode-select + {ndsp} decode sparse, "
                             "the decode step replayed as "
                             "two CUDA graphs (gathered rows; rows staged once), 1 overlap + 3 "
                             "block-selector kernels; then the other workloads' calls",
        "wall_s_timed_region": round(wall, 3),
    }

    if not args.no_e2e:
        line["e2e"] = e2e_prefill(hs2, pf.x, args, world, dev, W, K, pf.ws, flush)
    if rank == 0:
        clocks = clk.summary()
        if clocks:
            line["clocks"] = clocks
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(pf.x, dc.x, sample_s=15.0)
        print(json.dumps(line), flush=True)


def e2e_chunks(L, n_sms=148, bm=128):
    """Query-row chunks of the end-to-end pipeline.  Full layer: a first
    quarter (compute starts once it and its K/V rows are in), a second
    quarter, then the rest.  Selection: everything but the last wave of query
    blocks (n_sms blocks, the heaviest), then that wave, so that only its
    indices remain to be copied out after the last kernel."""
    def cut(x):
        return max(bm, min(L, (int(x) // bm) * bm))
    attn = sorted({0, cut(L / 4), cut(L / 2), L})
    last = L - n_sms * bm
    sel = [0, last, L] if last >= bm else [0, L]
    return attn, sel


def e2e_prefill(hs2, xp, args, world, dev, W, K, ws, flush):
    """Prefill full+select through the public calls with host buffers: Q, K, V
    copied in from pinned host memory, O and idx copied back, all timed.  The
    copies overlap the kernels: the full layer runs on query-row chunks
    (hs2_full_attn_rows) as their rows arrive, O chunks go back while later
    work runs, and the selection (hs2_select_rows) runs in two chunks with the
    first chunk's indices copied out during the second."""
    B, L, Hq, d = xp.q.shape
    hq, hk, hv = xp.q.pin_memory(), xp.k_.pin_memory(), xp.v.pin_memory()
    ho = torch.empty_like(hq).pin_memory()
    hidx = torch.empty(B, L, W + K, dtype=torch.int32).pin_memory()
    q = torch.empty_like(hq, device=dev)
    k = torch.empty_like(hk, device=dev)
    v = torch.empty_like(hv, device=dev)
    o = torch.empty_like(q)
    idx = torch.empty(B, L, W + K, dtype=torch.int32, device=dev)
    lse = torch.empty(B, L, Hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    attn, sel = e2e_chunks(L)
    ts = []
    for it in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cin.wait_stream(stream)
        cout.wait_stream(stream)
        arrived = []
        with torch.cuda.stream(cin):
            for a, b in zip(attn[:-1], attn[1:]):
                for dst, src in ((k, hk), (v, hv), (q, hq)):
                    dst[:, a:b].copy_(src[:, a:b], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(cin)
                arrived.append(ev)
        for (a, b), ev in zip(zip(attn[:-1], attn[1:]), arrived):
            stream.wait_event(ev)
            hs2.hs2_full_attn_rows(q, k, v, a, b, o=o, lse=lse, W=W, k_top=K)
            done = torch.cuda.Event()
            done.record(stream)
            cout.wait_event(done)
            with torch.cuda.stream(cout):
                ho[:, a:b].copy_(o[:, a:b], non_blocking=True)
        for a, b in zip(sel[:-1], sel[1:]):
            hs2.hs2_select_rows(q, k, lse, W, K, a, b, idx=idx, workspace=ws)
            done = torch.cuda.Event()
            done.record(stream)
            cout.wait_event(done)
            with torch.cuda.stream(cout):
                hidx[:, a:b].copy_(idx[:, a:b], non_blocking=True)
        stream.wait_stream(cout)
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            ts.append(e0.elapsed_time(e1) / 1e3)
    t = max_over_ranks([sum(ts) / len(ts)], world)[0]
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hidx.numel() * hidx.element_size()
    return {"value": round(world * B * L / t, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "what": f"prefill full+select at {L} tokens from pinned host buffers: q,k,v copied in "
                    f"by query-row chunks {attn} while hs2_full_attn_rows runs on the chunks "
                    f"already in, O copied back per chunk, hs2_select_rows on chunks {sel} with "
                    "the first chunk's idx copied back during the second"}


def cores_used():
    import oracle
    return oracle.num_threads()


def cpu_baseline_prefill(xp, sample_s=15.0, n_rows=None):
    """fp64 oracle on a bounded sample of query rows of the prefill full+select
    layer, extrapolated to all L rows by causal cost (sum of t+1)."""
    import oracle
    B, L, Hq, d = xp.q.shape
    if n_rows is None:
        # calibrate: cost ~ (t+1); a few rows first
        probe = np.array([L - 1], dtype=np.int64)
        t0 = time.perf_counter()
        oracle.full_select(xp.q, xp.k_, xp.v, xp.W, xp.k, rows=probe)
        per_full_row = time.perf_counter() - t0
        n_rows = int(max(4, min(512, 2 * sample_s / max(per_full_row, 1e-6))))
    rows = np.unique(np.linspace(0, L - 1, n_rows).astype(np.int64))
    t0 = time.perf_counter()
    oracle.full_select(xp.q, xp.k_, xp.v, xp.W, xp.k, rows=rows)
    dt = time.perf_counter() - t0
    frac = float((rows + 1).sum()) / (L * (L + 1) / 2.0)
    t_full = dt / frac
    return {"value": round(B * L / (t_full * B), 1), "unit": "tokens/s", "cores": cores_used(),
            "kind": "oracle",
            "sample": f"{rows.size} evenly spaced query rows of the {L}-token full+select "
                      f"layer ({dt:.1f} s fp64), extrapolated to all rows by causal cost"}


def cpu_baseline_sparse(xp, n_rows=4096):
    """fp64 oracle of one sparse layer on a sample of query rows past the first
    W+k (each of those attends to exactly W+k rows, so the per-row cost is the
    same for every such row), scaled to all L rows."""
    import oracle
    B, L, Hq, d = xp.q.shape
    S = xp.W + xp.k
    rows = np.unique(np.linspace(min(S, L - 1), L - 1, n_rows).astype(np.int64))
    # the selection the layer reuses: the window plus the k positions before it
    # (what it attends to does not change the cost per row)
    idx = np.full((B * L, S), -1, dtype=np.int32)
    for r in rows:
        t = int(r % L)
        n = min(t + 1, S)
        idx[r, :n] = np.arange(t - n + 1, t + 1)
    t0 = time.perf_counter()
    oracle.sparse(xp.q_sparse[0], xp.k_, xp.v, idx, rows=rows)
    dt = time.perf_counter() - t0
    return {"value": round(B * L / (dt * B * L / rows.size), 1), "unit": "tokens/s",
            "sample": f"{rows.size} query rows of one sparse layer ({dt:.2f} s fp64), "
                      f"scaled to all {L} rows"}


def cpu_baseline_decode(xd, n_sparse=N_SPARSE):
    """fp64 oracle of the whole decode step (select over every sequence, then
    the sparse layers on its selection)."""
    import oracle
    t0 = time.perf_counter()
    ora = oracle.decode_select(xd.q, xd.k_cache, xd.v_cache, xd.lengths, xd.W, xd.k, kv=xd.kv,
                               k_scale=xd.k_scale, v_scale=xd.v_scale)
    sel = torch.from_numpy(ora["idx"])
    for qs in xd.q_sparse[:n_sparse]:
        oracle.decode_sparse(qs, xd.k_cache, xd.v_cache, sel, kv=xd.kv, k_scale=xd.k_scale,
                             v_scale=xd.v_scale)
    dt = time.perf_counter() - t0
    return {"value": round(dt * 1e6, 1), "unit": "us/step",
            "sample": f"the whole step: {xd.B} sequences x {xd.Tmax} tokens, select + "
                      f"{len(xd.q_sparse[:n_sparse])} sparse layers ({dt:.1f} s fp64)"}


def cpu_baseline(xp, xd, sample_s=15.0):
    """The oracle as the CPU baseline: prefill full+select tokens/s (the
    headline), with the decode step and one sparse layer beside it."""
    r = cpu_baseline_prefill(xp, sample_s=sample_s)
    r["components"] = {"decode_us_per_step": cpu_baseline_decode(xd),
                       "prefill_sparse_layer_tok_s": cpu_baseline_sparse(xp)}
    return r


def run_reference(args):
    """The fp64 CPU oracle timed on bounded samples of our workload."""
    from token_level_top_hs2_b200 import inputs
    xp = inputs.make_workload(args.prefill)
    B, L, Hq, d = xp.q.shape
    rows_per_step = 24
    vals, secs = [], []
    t_all = time.perf_counter()
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r = cpu_baseline_prefill(xp, n_rows=rows_per_step)
        if it >= args.warmup:
            vals.append(r["value"])
            secs.append(time.perf_counter() - t0)
    value = statistics.mean(vals)
    sample = (f"per step {rows_per_step} evenly spaced query rows of the {L}-token full+select "
              "layer in fp64, extrapolated to all rows by causal cost")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2),
            "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup,
            # the measured time of one step's sample; `value` is extrapolated
            # from it to the whole layer
            "ms_per_step": round(statistics.mean(secs) * 1e3, 1),
            "ms_per_step_extrapolated_full_layer": round(B * L / value * 1e3, 1),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded planted-topic prefill)",
            "config": {"workload": f"{args.prefill} + {args.decode}", "L": L, "Hq": Hq, "d": d,
                       "W": xp.W, "k": xp.k},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "kind": "oracle",
                             "cores": cores_used(), "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t_all, 1)}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
