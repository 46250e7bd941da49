// Sparse-layer kernels: exact softmax attention of each query token over the
// K/V rows its inherited selection names (HySparse2 summary, "How it works":
// the sparse layers reuse the full layer's KV cache and selection indices).
#pragma once

#include <cooperative_groups.h>

#include "gather_attn.cuh"

namespace hs2 {

namespace cg = cooperative_groups;

// Prefill sparse layer: one warp per query token (B*L tokens), heads as rows.
// q [B*L, Hq, D] bf16; kv rows of sequence b start at b*L; idx [B*L, S].
template <int D, bool FP8, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
sparse_prefill_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
                      const uint8_t* __restrict__ vc, const float* __restrict__ ks,
                      const float* __restrict__ vs, const int32_t* __restrict__ idx,
                      __nv_bfloat16* __restrict__ out, int64_t n_tok, int L, int Hq, int S,
                      float qk_scale, unsigned* __restrict__ flags) {
    using R = KvRow<D, FP8>;
    const int lane = lane_id();
    const int64_t tok = (int64_t)blockIdx.x * WARPS + (threadIdx.x >> 5);
    if (tok >= n_tok) return;
    const int64_t b = tok / L;
    const int t = (int)(tok % L);
    const size_t row0 = (size_t)b * L;
    const uint8_t* kb = kc + row0 * D * R::ESZ;
    const uint8_t* vb = vc + row0 * D * R::ESZ;
    const float* ksb = FP8 ? ks + row0 : nullptr;
    const float* vsb = FP8 ? vs + row0 : nullptr;
    const int32_t* my_idx = idx + tok * S;

    WarpAttn<D, FP8> wa;
    if (!wa.load_q(q + tok * Hq * D, Hq)) {
        if (lane == 0) atomicOr(flags, FLAG_Q_RANGE);
    }
    bool bad = false;
    for (int j0 = 0; j0 < S; j0 += 16) {
        int my = -1;
        if (lane < 16 && j0 + lane < S) {
            my = __ldg(my_idx + j0 + lane);
            if (my > t || my < -1) {
                bad = true;
                my = -1;
            }
        }
        if (__ballot_sync(0xffffffffu, my >= 0) == 0) continue;
        int key_k[2], key_v[4];
        distribute_keys(my, key_k, key_v);
        TileRegs<D, FP8> tr;
        wa.load_tile(tr, kb, vb, ksb, vsb, key_k, key_v);
        float s[2][4];
        wa.qk(tr, s);
        wa.scale_mask(tr, s, qk_scale);
        wa.softmax_pv(tr, s);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(flags, FLAG_BAD_INDEX);
    wa.finish_sums();
    wa.store(out + tok * Hq * D, Hq);
}

// Decode sparse layer: one cluster of CLUSTER CTAs per sequence; the S index
// entries are split over CLUSTER*WARPS warps in 16-row tiles.  A warp reads
// the index entries of up to MAXT tiles at once, then issues the K/V loads of
// all of them before any arithmetic (MINB: CTAs per SM the register budget is
// set for).  Partial softmax states (m, l, o) merge first inside the CTA
// (each warp stores its o in fragment order, conflict-free; the CTA sums them
// scaled by per-(warp, row) factors), then across the cluster through
// distributed shared memory, each CTA producing 1/CLUSTER of the outputs.
template <int D, bool FP8, int WARPS, int CLUSTER>
struct DecodeSparseSmem {
    static constexpr int FRAG = 4 * (D / 8);           // o values per lane
    static constexpr int CO = 0;                       // CTA o, fragment order [FRAG][32]
    static constexpr int CM = CO + FRAG * 32;          // CTA m [16]
    static constexpr int CL = CM + 16;                 // CTA l [16]
    static constexpr int WO = CL + 16;                 // warps' o [WARPS][FRAG][32]
    static constexpr int WM = WO + WARPS * FRAG * 32;  // warps' m [WARPS][16]
    static constexpr int WL = WM + WARPS * 16;         // warps' l [WARPS][16]
    static constexpr int RF = WL + WARPS * 16;         // cluster factors [CLUSTER][16], 1/L [16]
    static constexpr int FLOATS = RF + CLUSTER * 16 + 16;
};

template <int D, bool FP8, int WARPS, int CLUSTER, int MAXT, int MINB>
__global__ void __launch_bounds__(WARPS * 32, MINB)
decode_sparse_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
                     const uint8_t* __restrict__ vc, const float* __restrict__ ks,
                     const float* __restrict__ vs, const int32_t* __restrict__ lengths,
                     const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out, int Tmax,
                     int Hq, int S, float qk_scale, unsigned* __restrict__ flags) {
    using R = KvRow<D, FP8>;
    using WA = WarpAttn<D, FP8>;
    using SM = DecodeSparseSmem<D, FP8, WARPS, CLUSTER>;
    constexpr int FRAG = SM::FRAG;
    extern __shared__ float smem_f[];

    // launched with programmatic serialisation: the launch overlaps the
    // previous kernel's tail; every input is read after it completed
    griddep_launch();
    griddep_wait();
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int b = blockIdx.x / CLUSTER;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    int T = __ldg(lengths + b);
    const bool len_ok = T >= 1 && T <= Tmax;
    if (!len_ok && threadIdx.x == 0 && rank == 0) atomicOr(flags, FLAG_BAD_LENGTH);
    const size_t row0 = (size_t)b * Tmax;
    const uint8_t* kb = kc + row0 * D * R::ESZ;
    const uint8_t* vb = vc + row0 * D * R::ESZ;
    const float* ksb = FP8 ? ks + row0 : nullptr;
    const float* vsb = FP8 ? vs + row0 : nullptr;
    const int32_t* my_idx = idx + (size_t)b * S;

    WA wa;
    if (!wa.load_q(q + (size_t)b * Hq * D, Hq)) {
        if (lane == 0) atomicOr(flags, FLAG_Q_RANGE);
    }
    const int n_tiles = (S + 15) / 16;
    const int slice = rank * WARPS + warp, n_slices = CLUSTER * WARPS;
    const int t0 = (int)((int64_t)n_tiles * slice / n_slices);
    const int t1 = (int)((int64_t)n_tiles * (slice + 1) / n_slices);
    bool bad = false;
    for (int base = t0; len_ok && base < t1; base += MAXT) {
        int my[MAXT];
#pragma unroll
        for (int u = 0; u < MAXT; u++) {
            const int j = (base + u) * 16 + lane;
            my[u] = -1;
            if (base + u < t1 && lane < 16 && j < S) {
                my[u] = __ldg(my_idx + j);
                if (my[u] >= T || my[u] < -1) {
                    bad = true;
                    my[u] = -1;
                }
            }
        }
        TileRegs<D, FP8> tr[MAXT];
        bool any[MAXT];
#pragma unroll
        for (int u = 0; u < MAXT; u++) {
            any[u] = __ballot_sync(0xffffffffu, my[u] >= 0) != 0;
            int key_k[2], key_v[4];
            distribute_keys(any[u] ? my[u] : -1, key_k, key_v);
            wa.load_tile(tr[u], kb, vb, ksb, vsb, key_k, key_v);
        }
#pragma unroll
        for (int u = 0; u < MAXT; u++) {
            if (!any[u]) continue;
            float s[2][4];
            wa.qk(tr[u], s);
            wa.scale_mask(tr[u], s, qk_scale);
            wa.softmax_pv(tr[u], s);
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(flags, FLAG_BAD_INDEX);
    wa.finish_sums();

    // ---- merge inside the CTA: o of every warp in fragment order
    float* wo = smem_f + SM::WO + warp * FRAG * 32;
#pragma unroll
    for (int i = 0; i < FRAG; i++) wo[i * 32 + lane] = wa.o[i >> 2][i & 3];
    if ((lane & 3) == 0) {
        const int g = lane >> 2;
        smem_f[SM::WM + warp * 16 + g] = wa.m[0];
        smem_f[SM::WM + warp * 16 + g + 8] = wa.m[1];
        smem_f[SM::WL + warp * 16 + g] = wa.l[0];
        smem_f[SM::WL + warp * 16 + g + 8] = wa.l[1];
    }
    __syncthreads();
    // per row: the CTA's max over its warps, then every warp's factor
    // 2^(m_w - M) kept in WM (warps without keys have l = 0 and o = 0)
    if (threadIdx.x < 16) {
        const int row = threadIdx.x;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; w++) mx = fmaxf(mx, smem_f[SM::WM + w * 16 + row]);
        const float mu = mx == -INFINITY ? 0.f : mx;
        float ls = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; w++) {
            const float mw = smem_f[SM::WM + w * 16 + row];
            const float f = mw == -INFINITY ? 0.f : ex2(mw - mu);
            smem_f[SM::WM + w * 16 + row] = f;
            ls += f * smem_f[SM::WL + w * 16 + row];
        }
        smem_f[SM::CM + row] = mx;
        smem_f[SM::CL + row] = ls;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < FRAG * 32; e += WARPS * 32) {
        const int row = WA::frag_row(e >> 5, e & 31);
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; w++)
            acc += smem_f[SM::WM + w * 16 + row] * smem_f[SM::WO + w * FRAG * 32 + e];
        smem_f[SM::CO + e] = acc;
    }
    cluster.sync();

    // ---- merge across the cluster: per row the factor of every rank, then
    // this rank's slice of the outputs from all ranks' o (independent loads)
    if (threadIdx.x < 16) {
        const int row = threadIdx.x;
        float mr[CLUSTER], lr[CLUSTER];
#pragma unroll
        for (int r = 0; r < CLUSTER; r++) {
            const float* p = cluster.map_shared_rank(smem_f, r);
            mr[r] = p[SM::CM + row];
            lr[r] = p[SM::CL + row];
        }
        float mx = -INFINITY;
#pragma unroll
        for (int r = 0; r < CLUSTER; r++) mx = fmaxf(mx, mr[r]);
        const float mu = mx == -INFINITY ? 0.f : mx;
        float ls = 0.f;
#pragma unroll
        for (int r = 0; r < CLUSTER; r++) {
            const float f = mr[r] == -INFINITY ? 0.f : ex2(mr[r] - mu);
            smem_f[SM::RF + r * 16 + row] = f;
            ls += f * lr[r];
        }
        smem_f[SM::RF + CLUSTER * 16 + row] = ls > 0.f ? WA::kOutScale / ls : 0.f;
    }
    __syncthreads();
    {
        constexpr int PER = FRAG * 32 / CLUSTER;
        for (int e = rank * PER + (int)threadIdx.x; e < (rank + 1) * PER; e += WARPS * 32) {
            const int i = e >> 5, L = e & 31;
            const int row = WA::frag_row(i, L);
            float v[CLUSTER];
#pragma unroll
            for (int r = 0; r < CLUSTER; r++) v[r] = cluster.map_shared_rank(smem_f, r)[SM::CO + e];
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < CLUSTER; r++) acc += smem_f[SM::RF + r * 16 + row] * v[r];
            if (row < Hq)
                out[((size_t)b * Hq + row) * D + WA::frag_col(i, L)] =
                    __float2bfloat16_rn(acc * smem_f[SM::RF + CLUSTER * 16 + row]);
        }
    }
    // no CTA leaves while another may still read its shared memory
    cluster.sync();
}

}  // namespace hs2
