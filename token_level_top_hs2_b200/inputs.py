"""Seeded synthetic inputs shared by the CUDA path, the oracle and the bench.

This module holds no arithmetic of the attention method: it only draws
random tensors, plants retrieval structure in them and stores them in the
formats the library consumes (bf16 rows, or e4m3 codes with a per-token fp32
scale).  Both sides of every parity check consume exactly the bytes made here.

Workloads follow the hot-path description of HySparse2 (onedev.kr/papers/146,
"How it works" / "How to use" sections): one shared KV head (MQA), no
positional encoding, a forced window of W=128 recent tokens plus k=1024 global
tokens, an FP8 KV cache for long contexts.  The pages evaluate on public
long-context suites; none of their items is used here.  Instead the retrieval
structure is synthetic:

* prefill ("planted topics"): n_topics random unit vectors u_c; every query
  segment of `seg` tokens gets a topic and +3*u_c on every head's query; 1% of
  the key positions (drawn without replacement) get +3*u_c of a random topic.
* decode ("needles"): one random unit vector u per sequence; every head's query
  gets +beta*u and 16 keys at uniform depths in [0, T-W) get +beta*u.

Draw order is fixed so that a seed names the bytes: prefill draws Q, K, V,
topic vectors, segment topics, planted key positions, planted key topics, then
each sparse layer's Q'; decode draws K, V, needle vector, needle positions,
q, then each sparse layer's q'.  Values are N(0,1) in fp32, structure is added
in fp32 and the result is rounded once (bf16 round-to-nearest-even, or the
per-token e4m3 quantiser below).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

E4M3_MAX = 448.0

# Named workloads.  Sizes are those of the hot-path configurations: a tiny
# prefill, prefill at 32k and 128k tokens, decode at 256k and 1M tokens.
WORKLOADS = {
    "prefill_tiny_1k": dict(kind="prefill", B=1, L=1024, Hq=4, d=64, W=32, k=128,
                            n_topics=8, seg=128, n_sparse=1, seed_id=0),
    "prefill_32k": dict(kind="prefill", B=1, L=32768, Hq=16, d=128, W=128, k=1024,
                        n_topics=32, seg=256, n_sparse=3, seed_id=1),
    "prefill_128k": dict(kind="prefill", B=1, L=131072, Hq=16, d=128, W=128, k=1024,
                         n_topics=32, seg=256, n_sparse=3, seed_id=2),
    "decode_256k_b16": dict(kind="decode", B=16, T=262144, Hq=16, d=128, W=128, k=1024,
                            n_needles=16, n_sparse=3, kv="e4m3", seed_id=3),
    "decode_1m_b4": dict(kind="decode", B=4, T=1048576, Hq=16, d=128, W=128, k=1024,
                         n_needles=16, n_sparse=3, kv="e4m3", seed_id=4),
}


def seed_for(seed_id: int, repeat: int = 0) -> int:
    return 20260000 + seed_id + 1000 * repeat


@dataclasses.dataclass
class PrefillInputs:
    B: int
    L: int
    Hq: int
    d: int
    W: int
    k: int
    q: torch.Tensor            # [B, L, Hq, d] bf16
    k_: torch.Tensor           # [B, L, d] bf16 (the shared K head)
    v: torch.Tensor            # [B, L, d] bf16
    q_sparse: List[torch.Tensor]  # n_sparse x [B, L, Hq, d] bf16
    segment_topic: torch.Tensor   # [B, n_seg] int64
    planted_pos: torch.Tensor     # [B, n_planted] int64
    planted_topic: torch.Tensor   # [B, n_planted] int64

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclasses.dataclass
class DecodeInputs:
    B: int
    Tmax: int
    Hq: int
    d: int
    W: int
    k: int
    kv: str                     # "e4m3" or "bf16"
    q: torch.Tensor             # [B, Hq, d] bf16
    q_sparse: List[torch.Tensor]  # n_sparse x [B, Hq, d] bf16
    k_cache: torch.Tensor       # [B, Tmax, d] uint8 codes (e4m3) or bf16
    v_cache: torch.Tensor
    k_scale: Optional[torch.Tensor]  # [B, Tmax] fp32 (None for bf16)
    v_scale: Optional[torch.Tensor]
    lengths: torch.Tensor       # [B] int32
    needle_pos: torch.Tensor    # [B, n_needles] int64

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-token e4m3 storage: scale = max|x|/448 (1 for an all-zero row),
    code = round-to-nearest-even(x/scale) saturated to +-448.

    Returns (codes uint8 [..., d], scales fp32 [...]).  The oracle and the
    kernels only ever see the stored codes and scales.
    """
    x = x.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def _unit_rows(g: torch.Generator, n: int, d: int) -> torch.Tensor:
    u = torch.randn(n, d, generator=g, dtype=torch.float32)
    return u / u.norm(dim=-1, keepdim=True)


def make_prefill(B: int, L: int, Hq: int, d: int, W: int, k: int, *, n_topics: int = 8,
                 seg: int = 128, n_sparse: int = 1, seed: int = 0, boost: float = 3.0,
                 planted_frac: float = 0.01) -> PrefillInputs:
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, d, generator=g, dtype=torch.float32)
    kk = torch.randn(B, L, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, L, d, generator=g, dtype=torch.float32)
    n_topics = max(1, n_topics)
    topics = _unit_rows(g, n_topics, d)
    n_seg = (L + seg - 1) // seg
    seg_topic = torch.randint(0, n_topics, (B, n_seg), generator=g)
    n_planted = int(L * planted_frac)
    planted_pos = torch.empty(B, n_planted, dtype=torch.int64)
    for b in range(B):
        planted_pos[b] = torch.randperm(L, generator=g)[:n_planted]
    planted_topic = torch.randint(0, n_topics, (B, n_planted), generator=g)
    # structure, in fp32, before the single rounding to bf16
    seg_of_t = torch.arange(L) // seg
    for b in range(B):
        q[b] += boost * topics[seg_topic[b, seg_of_t]].unsqueeze(1)
        if n_planted:
            kk[b, planted_pos[b]] += boost * topics[planted_topic[b]]
    q_sparse = [torch.randn(B, L, Hq, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
                for _ in range(n_sparse)]
    return PrefillInputs(B=B, L=L, Hq=Hq, d=d, W=W, k=k, q=q.to(torch.bfloat16),
                         k_=kk.to(torch.bfloat16), v=v.to(torch.bfloat16), q_sparse=q_sparse,
                         segment_topic=seg_topic, planted_pos=planted_pos,
                         planted_topic=planted_topic)


def make_decode(B: int, T: int, Hq: int, d: int, W: int, k: int, *, n_needles: int = 16,
                n_sparse: int = 3, kv: str = "e4m3", seed: int = 0, beta: Optional[float] = None,
                lengths: Optional[List[int]] = None, Tmax: Optional[int] = None) -> DecodeInputs:
    """Decode cache of Tmax rows per sequence; sequence b uses lengths[b] rows
    (default: all T).  Needles sit at uniform depths in [0, len-W)."""
    Tmax = T if Tmax is None else Tmax
    if beta is None:
        beta = 12.0 * (d / 128.0) ** 0.25
    g = torch.Generator().manual_seed(seed)
    kk = torch.randn(B, Tmax, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, Tmax, d, generator=g, dtype=torch.float32)
    u = _unit_rows(g, B, d)
    lens = [T] * B if lengths is None else list(lengths)
    needle_pos = torch.zeros(B, n_needles, dtype=torch.int64)
    for b in range(B):
        span = max(1, lens[b] - W)
        n = min(n_needles, span)
        pos = torch.randperm(span, generator=g)[:n]
        needle_pos[b, :n] = pos
        needle_pos[b, n:] = -1
        kk[b, pos] += beta * u[b]
    q = torch.randn(B, Hq, d, generator=g, dtype=torch.float32) + beta * u.unsqueeze(1)
    q_sparse = [torch.randn(B, Hq, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
                for _ in range(n_sparse)]
    if kv == "e4m3":
        kc, ks = quantize_e4m3_per_token(kk)
        vc, vs = quantize_e4m3_per_token(v)
    elif kv == "bf16":
        kc, vc, ks, vs = kk.to(torch.bfloat16), v.to(torch.bfloat16), None, None
    else:
        raise ValueError(f"kv must be 'e4m3' or 'bf16', got {kv!r}")
    del kk, v
    return DecodeInputs(B=B, Tmax=Tmax, Hq=Hq, d=d, W=W, k=k, kv=kv, q=q.to(torch.bfloat16),
                        q_sparse=q_sparse, k_cache=kc, v_cache=vc, k_scale=ks, v_scale=vs,
                        lengths=torch.tensor(lens, dtype=torch.int32), needle_pos=needle_pos)


def make_workload(name: str, repeat: int = 0):
    """Inputs of one named workload (see WORKLOADS), seeded by name and repeat."""
    w = dict(WORKLOADS[name])
    seed = seed_for(w.pop("seed_id"), repeat)
    kind = w.pop("kind")
    if kind == "prefill":
        return make_prefill(seed=seed, **w)
    return make_decode(seed=seed, **w)


def make_selection_pair(B: int, L: int, W: int, k: int, *, seed: int, shuffle: bool = True):
    """Two synthetic selections [B, L, W+k] int32 in the library's idx format,
    for overlap checks.  Row t: the window max(0, t-W+1)..t, then min(k, n)
    distinct global picks from the n = t-W+1 candidates, then -1 padding.
    The picks of the first selection are (a*j + c) mod n for j < min(k, n),
    with a random multiplier a coprime to n; the second uses the same a and
    c + s for a random shift s in [0, k], so rows overlap by every amount
    from all to nothing.  With shuffle, each row's slots are permuted."""
    g = torch.Generator().manual_seed(seed)
    S = W + k
    t = torch.arange(L, dtype=torch.int64).view(1, L, 1).expand(B, L, 1)
    n = (t - W + 1).clamp(min=0)                                   # candidates per row
    primes = torch.tensor([1000003, 999983, 999979, 999961, 999959, 999953], dtype=torch.int64)
    a = primes[torch.randint(0, len(primes), (B, L, 1), generator=g)]
    nn = n.clamp(min=1)
    a = torch.where(torch.gcd(a, nn) == 1, a, torch.ones_like(a))  # coprime: distinct picks
    c = torch.randint(0, 1 << 30, (B, L, 1), generator=g)
    s = torch.randint(0, k + 1, (B, L, 1), generator=g)
    j = torch.arange(k, dtype=torch.int64).view(1, 1, k)
    used = j < n                                                     # min(k, n) picks
    ga = torch.where(used, (a * j + c) % nn, torch.full_like(j, -1))
    gb = torch.where(used, (a * j + c + s) % nn, torch.full_like(j, -1))
    w = torch.arange(W, dtype=torch.int64).view(1, 1, W)
    win = t - W + 1 + w
    win = torch.where(win >= 0, win, torch.full_like(win, -1))
    out = []
    for glob in (ga, gb):
        row = torch.cat([win, glob], dim=2)
        # valid entries first (window, then globals), -1 padding at the tail
        key = torch.where(row >= 0, torch.zeros_like(row), torch.ones_like(row))
        order = torch.argsort(key * (2 * S) + torch.arange(S).view(1, 1, S), dim=2)
        row = torch.gather(row, 2, order)
        if shuffle:
            perm = torch.argsort(torch.rand(B, L, S, generator=g), dim=2)
            row = torch.gather(row, 2, perm)
        out.append(row.to(torch.int32).contiguous())
    return out[0], out[1]
