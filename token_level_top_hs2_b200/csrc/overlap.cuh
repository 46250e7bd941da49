// Cross-layer overlap of two token selections.
//
// The IndexCache page (Appendix A, "Cross-Layer Top-(k) Index Overlap")
// measures how far two layers pick the same tokens by the pairwise ratio
// |T(i) ∩ T(j)| / k of their top-k index sets.  Applied to HySparse2 (KV
// Reuse, HySparse2 summary "How it works") it compares the selection a sparse
// layer inherits from its full layer with the exact top-k that layer's own
// queries would pick.
//
// For query row t of an idx row laid out as the selection kernels write it
// (window, global picks, -1 padding), the global picks are the entries s with
// 0 <= s <= t - W.  Per row this kernel counts |G_a ∩ G_b| and writes the
// ratio count / min(k, t - W + 1); rows without global candidates (t < W, or
// k = 0) compare two empty sets and get ratio 1.  Entries outside [-1, t]
// break the idx contract: they are skipped and flagged.
//
// One warp per row: both rows are copied into the warp's shared memory with
// cp.async (the next row's copies in flight while this row is processed).
// For L <= 2^17 the membership test is a bitmap over the positions
// (overlap_bitmap_kernel); longer rows use an open-addressing hash set:
// G_a goes into the set, G_b probes it.  A slot holds (epoch << 21) | (position + 1);
// a slot whose epoch is not the current row's counts as empty, so the set is
// emptied for the next row by advancing the epoch (and wiped only when the
// 11-bit epoch wraps).  Positions must stay below 2^21 - 1.  Reads each idx
// row once (HBM bound).
#pragma once

#include "common.cuh"

namespace hs2 {
namespace ovl {

constexpr int kWarps = 3;
constexpr int kPosBits = 21;
constexpr uint32_t kEpochs = 2047;  // epochs 1..2047; 0 never matches

// hash slots per warp: a power of two >= 2k (load factor <= 1/2), >= 256
__host__ __device__ inline int slot_bits(int k) {
    int b = 8;
    while ((1 << b) < 2 * k) b++;
    return b;
}

// shared memory per CTA: per warp a hash set and two stages of (row a, row b)
__host__ __device__ inline size_t smem_bytes(int S, int k) {
    const int sp = (S + 3) & ~3;
    return (size_t)kWarps * ((1 << slot_bits(k)) + 4 * sp) * sizeof(uint32_t);
}

HS2_DEV uint32_t slot_of(uint32_t key, int bits) { return (key * 0x9E3779B1u) >> (32 - bits); }

HS2_DEV uint32_t shared_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
HS2_DEV void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(shared_addr(smem)), "l"(gmem)
                 : "memory");
}
HS2_DEV void cp_async4(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(shared_addr(smem)), "l"(gmem)
                 : "memory");
}
HS2_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
HS2_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// the warp copies S entries of both rows into its stage (asynchronously)
HS2_DEV void stage_rows(int32_t* dst_a, int32_t* dst_b, const int32_t* ra, const int32_t* rb,
                        int S, bool vec, int lane) {
    if (vec) {
        for (int i = 4 * lane; i < S; i += 128) {
            cp_async16(dst_a + i, ra + i);
            cp_async16(dst_b + i, rb + i);
        }
    } else {
        for (int i = lane; i < S; i += 32) {
            cp_async4(dst_a + i, ra + i);
            cp_async4(dst_b + i, rb + i);
        }
    }
}

__global__ void __launch_bounds__(kWarps * 32)
overlap_kernel(const int32_t* __restrict__ idx_a, const int32_t* __restrict__ idx_b, int B, int L,
               int S, int W, int k, int32_t* __restrict__ inter, float* __restrict__ ratio,
               unsigned* __restrict__ flags) {
    extern __shared__ uint32_t smem_ovl[];
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int sp = (S + 3) & ~3;
    const int bits = slot_bits(k);
    const int n_slots = 1 << bits;
    const uint32_t mask = (uint32_t)n_slots - 1u;
    uint32_t* tab = smem_ovl + warp * (n_slots + 4 * sp);
    int32_t* stage = reinterpret_cast<int32_t*>(tab + n_slots);  // [2][a | b][sp]
    const bool vec = (S & 3) == 0;  // 16-byte rows: every row start is 16-byte aligned
    bool bad = false;
    const long long n_rows = (long long)B * L;
    const long long step = (long long)gridDim.x * kWarps;
    long long r = (long long)blockIdx.x * kWarps + warp;
    if (r < n_rows) stage_rows(stage, stage + sp, idx_a + r * S, idx_b + r * S, S, vec, lane);
    cp_async_commit();
    uint32_t epoch = kEpochs;  // wiped (and reset to 1) before the first row
    for (int it = 0; r < n_rows; r += step, it++) {
        // the next row's copies go out before this row is processed
        const long long rn = r + step;
        int32_t* nxt = stage + ((it + 1) & 1) * 2 * sp;
        if (rn < n_rows) stage_rows(nxt, nxt + sp, idx_a + rn * S, idx_b + rn * S, S, vec, lane);
        cp_async_commit();
        cp_async_wait<1>();
        __syncwarp();
        const int32_t* va = stage + (it & 1) * 2 * sp;
        const int32_t* vb = va + sp;
        if (++epoch > kEpochs) {
            for (int i = lane; i < n_slots; i += 32) tab[i] = 0u;
            __syncwarp();
            epoch = 1;
        }
        const int t = (int)(r % L);
        const int last = t - W;  // global candidates are 0..last
        int found = 0;
        if (last >= 0 && k > 0) {
            // G_a into the set
            for (int i = lane; i < S; i += 32) {
                const int s = va[i];
                bad |= s < -1 || s > t;
                if (s < 0 || s > last) continue;
                const uint32_t e = (epoch << kPosBits) | ((uint32_t)s + 1u);
                uint32_t h = slot_of((uint32_t)s + 1u, bits);
                for (int probe = 0; probe < n_slots;) {
                    const uint32_t prev = tab[h];
                    if ((prev >> kPosBits) != epoch) {
                        if (atomicCAS(&tab[h], prev, e) == prev) break;
                        continue;  // another lane took the slot: look at it again
                    }
                    if (prev == e) break;
                    h = (h + 1u) & mask;
                    probe++;
                }
            }
            __syncwarp();
            // G_b probes it
            for (int i = lane; i < S; i += 32) {
                const int s = vb[i];
                bad |= s < -1 || s > t;
                if (s < 0 || s > last) continue;
                const uint32_t e = (epoch << kPosBits) | ((uint32_t)s + 1u);
                uint32_t h = slot_of((uint32_t)s + 1u, bits);
                for (int probe = 0; probe < n_slots; probe++) {
                    const uint32_t v = tab[h];
                    if ((v >> kPosBits) != epoch) break;
                    if (v == e) {
                        found++;
                        break;
                    }
                    h = (h + 1u) & mask;
                }
            }
        } else {
            for (int i = lane; i < S; i += 32)
                bad |= va[i] < -1 || va[i] > t || vb[i] < -1 || vb[i] > t;
        }
        // every lane is done with this stage before the copies of row it + 2 land in it
        __syncwarp();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) found += __shfl_xor_sync(0xffffffffu, found, o);
        if (lane == 0) {
            const int denom = (last >= 0 && k > 0) ? min(k, last + 1) : 0;
            if (inter) inter[r] = found;
            if (ratio) ratio[r] = denom > 0 ? (float)found / (float)denom : 1.f;
        }
    }
    cp_async_wait<0>();
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(flags, FLAG_BAD_INDEX);
}

// Rows of up to kBitmapMaxL positions: a bitmap over the positions instead of
// the hash set.  G_a sets its bits (atomicOr), G_b tests them, G_a clears its
// words again (plain zero stores: every writer writes 0) -- no probing.
constexpr int kBitmapMaxL = 1 << 17;

__host__ __device__ inline size_t bitmap_smem_bytes(int S, int L) {
    const int sp = (S + 3) & ~3;
    const int words = (L + 31) / 32;
    return (size_t)kWarps * (((words + 3) & ~3) + 4 * sp) * sizeof(uint32_t);
}

__global__ void __launch_bounds__(kWarps * 32)
overlap_bitmap_kernel(const int32_t* __restrict__ idx_a, const int32_t* __restrict__ idx_b,
                      int B, int L, int S, int W, int k, int32_t* __restrict__ inter,
                      float* __restrict__ ratio, unsigned* __restrict__ flags) {
    extern __shared__ uint32_t smem_ovl[];
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int sp = (S + 3) & ~3;
    const int words = ((L + 31) / 32 + 3) & ~3;
    uint32_t* bm = smem_ovl + warp * (words + 4 * sp);
    int32_t* stage = reinterpret_cast<int32_t*>(bm + words);  // [2][a | b][sp]
    const bool vec = (S & 3) == 0;
    for (int i = lane; i < words; i += 32) bm[i] = 0u;
    bool bad = false;
    const long long n_rows = (long long)B * L;
    const long long step = (long long)gridDim.x * kWarps;
    long long r = (long long)blockIdx.x * kWarps + warp;
    if (r < n_rows) stage_rows(stage, stage + sp, idx_a + r * S, idx_b + r * S, S, vec, lane);
    cp_async_commit();
    for (int it = 0; r < n_rows; r += step, it++) {
        const long long rn = r + step;
        int32_t* nxt = stage + ((it + 1) & 1) * 2 * sp;
        if (rn < n_rows) stage_rows(nxt, nxt + sp, idx_a + rn * S, idx_b + rn * S, S, vec, lane);
        cp_async_commit();
        cp_async_wait<1>();
        __syncwarp();
        const int32_t* va = stage + (it & 1) * 2 * sp;
        const int32_t* vb = va + sp;
        const int t = (int)(r % L);
        const int last = t - W;
        int found = 0;
        const bool ranked = last >= 0 && k > 0;
#pragma unroll 4
        for (int i = lane; i < S; i += 32) {
            const int s = va[i];
            bad |= s < -1 || s > t;
            if (ranked && s >= 0 && s <= last) atomicOr(&bm[s >> 5], 1u << (s & 31));
        }
        __syncwarp();
#pragma unroll 4
        for (int i = lane; i < S; i += 32) {
            const int s = vb[i];
            bad |= s < -1 || s > t;
            if (ranked && s >= 0 && s <= last) found += (bm[s >> 5] >> (s & 31)) & 1u;
        }
        __syncwarp();
#pragma unroll 4
        for (int i = lane; i < S; i += 32) {
            const int s = va[i];
            if (ranked && s >= 0 && s <= last) bm[s >> 5] = 0u;
        }
        // every lane is done with this stage (and the bitmap is clear) before
        // the copies of row it + 2 land in the stage
        __syncwarp();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) found += __shfl_xor_sync(0xffffffffu, found, o);
        if (lane == 0) {
            const int denom = ranked ? min(k, last + 1) : 0;
            if (inter) inter[r] = found;
            if (ratio) ratio[r] = denom > 0 ? (float)found / (float)denom : 1.f;
        }
    }
    cp_async_wait<0>();
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(flags, FLAG_BAD_INDEX);
}

}  // namespace ovl
}  // namespace hs2
