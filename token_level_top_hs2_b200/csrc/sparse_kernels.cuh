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
// entries are split over CLUSTER*WARPS warps; partial softmax states merge in
// shared memory, then across the cluster through distributed shared memory.
template <int D, bool FP8, int WARPS, int CLUSTER>
__global__ void __launch_bounds__(WARPS * 32)
decode_sparse_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
                     const uint8_t* __restrict__ vc, const float* __restrict__ ks,
                     const float* __restrict__ vs, const int32_t* __restrict__ lengths,
                     const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out, int Tmax,
                     int Hq, int S, float qk_scale, unsigned* __restrict__ flags) {
    using R = KvRow<D, FP8>;
    constexpr int PART = 16 * D + 32;  // floats per partial: o[16][D], m[16], l[16]
    extern __shared__ float smem_f[];
    float* wpart = smem_f;                   // WARPS partials
    float* cpart = smem_f + WARPS * PART;    // this CTA's merged partial

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

    WarpAttn<D, FP8> wa;
    if (!wa.load_q(q + (size_t)b * Hq * D, Hq)) {
        if (lane == 0) atomicOr(flags, FLAG_Q_RANGE);
    }
    const int n_tiles = (S + 15) / 16;
    const int slice = rank * WARPS + warp, n_slices = CLUSTER * WARPS;
    const int t0 = (int)((int64_t)n_tiles * slice / n_slices);
    const int t1 = (int)((int64_t)n_tiles * (slice + 1) / n_slices);
    bool bad = false;
    if (len_ok) {
        for (int tile = t0; tile < t1; tile++) {
            const int j = tile * 16 + lane;
            int my = -1;
            if (lane < 16 && j < S) {
                my = __ldg(my_idx + j);
                if (my >= T || my < -1) {
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
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(flags, FLAG_BAD_INDEX);
    wa.finish_sums();
    float* mine = wpart + warp * PART;
    wa.dump(mine + 16 * D, mine + 16 * D + 16, mine);
    __syncthreads();
    merge_partials_block<D>(wpart + 16 * D, wpart + 16 * D + 16, wpart, WARPS, PART, PART, Hq,
                            cpart + 16 * D, cpart + 16 * D + 16, cpart);
    cluster.sync();
    {
        // merge the CLUSTER partials through distributed shared memory; each
        // CTA of the cluster produces its own slice of the Hq x D outputs
        const int per = (Hq * D + CLUSTER - 1) / CLUSTER;
        const int e1 = min(Hq * D, (rank + 1) * per);
        for (int e = rank * per + (int)threadIdx.x; e < e1; e += blockDim.x) {
            const int row = e / D;
            float mx = -INFINITY;
            for (int r = 0; r < CLUSTER; r++) {
                const float* p = cluster.map_shared_rank(cpart, r);
                mx = fmaxf(mx, p[16 * D + row]);
            }
            const float mu = mx == -INFINITY ? 0.f : mx;
            float acc = 0.f, ls = 0.f;
            for (int r = 0; r < CLUSTER; r++) {
                const float* p = cluster.map_shared_rank(cpart, r);
                const float f = ex2(p[16 * D + row] - mu);
                acc += f * p[e];
                ls += f * p[16 * D + 16 + row];
            }
            const float val = ls > 0.f ? acc * WarpAttn<D, FP8>::kOutScale / ls : 0.f;
            out[(size_t)b * Hq * D + e] = __float2bfloat16_rn(val);
        }
    }
    cluster.sync();
}

}  // namespace hs2
