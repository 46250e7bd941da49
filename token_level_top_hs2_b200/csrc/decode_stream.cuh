// Decode full layer with token selection: TMA-fed streaming passes.
//
// One new query per sequence at t = T-1 attends exactly to cache rows 0..t and
// selects the window t-W+1..t plus the top-k of 0..t-W by the head-summed
// probability (HySparse2 summary, "What differs").  Each head's global
// log-sum-exp must be known before any score can be ranked, so:
//   pass 1   every CTA streams its chunk of K, V (+ per-token scales) through a
//            4-stage ring of 128-token tiles (TMA, 128-byte swizzle; one
//            producer warp), 8 consumer warps run 16-token tiles with the
//            heads as the MMA M dimension, the CTA's partial (max, sum, O) per
//            head goes to the workspace and the last chunk of a sequence to
//            finish merges them into lse and O;
//   pass 2   re-streams K, writes every candidate's fp32 score (s <= t-W) and
//            a per-sequence histogram of the score bits (1/16-octave bins
//            relative to 2^-8 of the mean score Hq/T);
//   gather   keys above the histogram's boundary bin go straight to the index
//            row; the boundary bin is collected and cut exactly by the last
//            CTA of the sequence, which also writes the window and padding.
// No kernel waits on another CTA: "last to finish" uses atomic counters.
#pragma once

#include "gather_attn.cuh"
#include "tc.cuh"

namespace hs2 {
namespace dec {

using namespace hs2::tc;

constexpr int TOK = 128;      // tokens per stage
constexpr int NST = 4;        // ring depth
constexpr int CWARPS = 8;     // consumer warps, 16 tokens each per stage
constexpr int kThreads = (CWARPS + 1) * 32;
constexpr int kBinShift = 19; // 16 bins per octave
constexpr int BCAP = 4096;    // boundary-bin keys a sequence may collect

template <int D, bool FP8>
struct Stage {
    static constexpr int ESZ = FP8 ? 1 : 2;
    static constexpr int RB = D * ESZ;          // bytes per cache row
    static constexpr int NBLK = RB / 128;       // 128-byte column blocks
    static constexpr int TILE = TOK * RB;       // one K or V tile
    static constexpr int SC = TOK * 4;          // one scale tile
    static constexpr int BOX_X = 128 / ESZ;     // TMA inner box, elements
    // pass 1 stage: K | V | sK | sV ; pass 2 stage: K | sK
    // stage strides: the 128-byte swizzle follows absolute shared-memory
    // address bits, so every stage (and tile) starts on a 1024-byte boundary
    static constexpr int P1 = (2 * TILE + (FP8 ? 2 * SC : 0) + 1023) / 1024 * 1024;
    static constexpr int P2 = (TILE + (FP8 ? SC : 0) + 1023) / 1024 * 1024;
    static constexpr int TX1 = 2 * TILE + (FP8 ? 2 * SC : 0);  // bytes a pass-1 stage receives
    static constexpr int TX2 = TILE + (FP8 ? SC : 0);
    // ring depths that fit shared memory (<= 200 KB of stages)
    static constexpr int NST1 = (200 * 1024 / P1) < NST ? (200 * 1024 / P1) : NST;
    static constexpr int NST2 = NST;
    static constexpr int SMEM1 = NST1 * P1 + 1024;
    static constexpr int SMEM2 = NST2 * P2 + 1024;
    static_assert(NST1 * P1 >= CWARPS * (16 * D + 32) * 4, "partials must fit the ring");
    static_assert(RB % 128 == 0, "cache rows must be whole 128-byte blocks");
};

// byte address of byte e of tile row r in a swizzled [NBLK][TOK][128] tile
HS2_DEV uint32_t sw_off(int r, int e) {
    return (uint32_t)((e >> 7) * (TOK * 128) + r * 128 + ((((e >> 4) & 7) ^ (r & 7)) << 4) +
                      (e & 15));
}

// Fill a TileRegs from a staged tile: this warp's 16 tokens start at tile row
// r0; key i of the warp is valid iff tok0 + i < s_end.  Invalid keys get zero
// operands and scales (rows past the cache length may hold any bytes).
template <int D, bool FP8>
HS2_DEV void load_tile_smem(TileRegs<D, FP8>& t, const uint8_t* ktile, const uint8_t* vtile,
                            const float* kst, const float* vst, int r0, int tok0, int s_end) {
    using R = KvRow<D, FP8>;
    const int lane = lane_id(), g = lane >> 2, c = lane & 3;
    const int kr[2] = {g, 8 + g};
#pragma unroll
    for (int i = 0; i < 2; i++) {
        const bool ok = tok0 + kr[i] < s_end;
#pragma unroll
        for (int j = 0; j < R::KQ_VEC; j++) {
            const uint4 x = *reinterpret_cast<const uint4*>(
                ktile + sw_off(r0 + kr[i], c * R::KQ_BYTES + 16 * j));
            t.k[i][j] = ok ? x : make_uint4(0, 0, 0, 0);
        }
    }
    const int vr[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const bool ok = tok0 + vr[i] < s_end;
        t.kval[i] = ok;
        if (vtile) {
#pragma unroll
            for (int j = 0; j < R::VQ_VEC; j++) {
                const uint4 x = *reinterpret_cast<const uint4*>(
                    vtile + sw_off(r0 + vr[i], g * R::VQ_BYTES + 16 * j));
                t.v[i][j] = ok ? x : make_uint4(0, 0, 0, 0);
            }
        }
        if constexpr (FP8) {
            t.ks[i] = ok ? kst[r0 + vr[i]] : 0.f;
            t.vs[i] = (ok && vst) ? vst[r0 + vr[i]] : 0.f;
        }
    }
}

struct Bars {
    uint64_t full[NST], empty[NST];
    int abort_;
    unsigned last;
};

template <int D, bool FP8>
HS2_DEV void issue_stage(uint8_t* st, const CUtensorMap* mk, const CUtensorMap* mv,
                         const CUtensorMap* mks, const CUtensorMap* mvs, int tok, int b,
                         uint64_t* bar) {
    using SG = Stage<D, FP8>;
    mbar_arrive_expect_tx(bar, mv ? SG::TX1 : SG::TX2);
    for (int blk = 0; blk < SG::NBLK; blk++)
        tma_load_3d(st + blk * (TOK * 128), mk, blk * SG::BOX_X, tok, b, bar);
    int off = SG::TILE;
    if (mv) {
        for (int blk = 0; blk < SG::NBLK; blk++)
            tma_load_3d(st + off + blk * (TOK * 128), mv, blk * SG::BOX_X, tok, b, bar);
        off += SG::TILE;
    }
    if constexpr (FP8) {
        tma_load_2d(st + off, mks, tok, b, bar);
        if (mv) tma_load_2d(st + off + SG::SC, mvs, tok, b, bar);
    }
}

// ------------------------------------------------------------------ pass 1
// grid (n_chunks, B), 288 threads: warps 0-7 consume, warp 8 produces.
template <int D, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
pass1_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
             const __grid_constant__ CUtensorMap map_ks, const __grid_constant__ CUtensorMap map_vs,
             const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lengths, int Tmax,
             int Hq, int chunk_len, int n_chunks, float qk_scale, float* __restrict__ part,
             unsigned* __restrict__ counter, float* __restrict__ lse2_ws,
             float* __restrict__ lse_out, __nv_bfloat16* __restrict__ out,
             unsigned* __restrict__ flags) {
    using SG = Stage<D, FP8>;
    constexpr int PART = 16 * D + 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ Bars bars;
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int T = __ldg(lengths + b);
    const bool len_ok = T >= 1 && T <= Tmax;
    if (!len_ok && threadIdx.x == 0 && chunk == 0) atomicOr(flags, FLAG_BAD_LENGTH);
    const int s_begin = chunk * chunk_len;
    const int s_end = len_ok ? min(s_begin + chunk_len, T) : s_begin;
    const int n_tiles = s_end > s_begin ? (s_end - s_begin + TOK - 1) / TOK : 0;
    volatile int* abort_ = &bars.abort_;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; i++) {
            mbar_init(&bars.full[i], 1);
            mbar_init(&bars.empty[i], CWARPS);
        }
        bars.abort_ = 0;
        fence_mbar_init();
    }
    __syncthreads();

    WarpAttn<D, FP8> wa;
    if (warp == CWARPS) {
        if (lane == 0) {
            int armed = 0;
            constexpr int R = SG::NST1;
            for (int j = 0; j < n_tiles && !*abort_; j++) {
                const int st = j % R, u = j / R;
                if (u > 0 && !mbar_wait(&bars.empty[st], (u - 1) & 1, abort_, flags)) break;
                issue_stage<D, FP8>(smem + st * SG::P1, &map_k, &map_v, &map_ks, &map_vs,
                                    s_begin + j * TOK, b, &bars.full[st]);
                armed++;
            }
            if (*abort_) {
                volatile int no_abort = 0;
                for (int j = max(0, armed - R); j < armed; j++)
                    mbar_wait(&bars.full[j % R], (j / R) & 1, &no_abort, flags);
            }
        }
    } else {
        if (!wa.load_q(q + (size_t)b * Hq * D, Hq) && chunk == 0 && lane == 0 && warp == 0)
            atomicOr(flags, FLAG_Q_RANGE);
        bool bad_scale = false;
        constexpr int R = SG::NST1;
        for (int j = 0; j < n_tiles; j++) {
            const int st = j % R;
            if (!mbar_wait(&bars.full[st], (j / R) & 1, abort_, flags)) break;
            const uint8_t* sb = smem + st * SG::P1;
            const float* kst = reinterpret_cast<const float*>(sb + 2 * SG::TILE);
            const float* vst = kst + TOK;
            const int tok0 = s_begin + j * TOK + 16 * warp;
            TileRegs<D, FP8> tr;
            load_tile_smem<D, FP8>(tr, sb, sb + SG::TILE, FP8 ? kst : nullptr,
                                   FP8 ? vst : nullptr, 16 * warp, tok0, s_end);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.empty[st]);
            if constexpr (FP8) {
#pragma unroll
                for (int i = 0; i < 4; i++) bad_scale |= !(tr.vs[i] <= 255.f);
            }
            float s[2][4];
            wa.qk(tr, s);
            wa.scale_mask(tr, s, qk_scale);
            wa.softmax_pv(tr, s);
        }
        if (__any_sync(0xffffffffu, bad_scale) && lane == 0) atomicOr(flags, FLAG_SCALE_RANGE);
        wa.finish_sums();
    }
    __syncthreads();  // every stage consumed: the ring is reused for the partials
    float* wpart = reinterpret_cast<float*>(smem);
    if (warp < CWARPS) {
        float* mine = wpart + warp * PART;
        wa.dump(mine + 16 * D, mine + 16 * D + 16, mine);
    }
    __syncthreads();
    float* dst = part + ((size_t)b * n_chunks + chunk) * PART;
    merge_partials_block<D>(wpart + 16 * D, wpart + 16 * D + 16, wpart, CWARPS, PART, PART, Hq,
                            dst + 16 * D, dst + 16 * D + 16, dst);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) bars.last = (atomicAdd(counter + b, 1u) == (unsigned)(n_chunks - 1));
    __syncthreads();
    if (!bars.last) return;
    __threadfence();
    const float* pb = part + (size_t)b * n_chunks * PART;
    for (int e = threadIdx.x; e < Hq * D; e += blockDim.x) {
        const int row = e / D;
        float mx = -INFINITY;
        for (int i = 0; i < n_chunks; i++)
            mx = fmaxf(mx, __ldcg(pb + (size_t)i * PART + 16 * D + row));
        const float mu = mx == -INFINITY ? 0.f : mx;
        float acc = 0.f, ls = 0.f;
        for (int i = 0; i < n_chunks; i++) {
            const float* p = pb + (size_t)i * PART;
            const float f = ex2(__ldcg(p + 16 * D + row) - mu);
            acc += f * __ldcg(p + e);
            ls += f * __ldcg(p + 16 * D + 16 + row);
        }
        const float val = ls > 0.f ? acc * WarpAttn<D, FP8>::kOutScale / ls : 0.f;
        out[(size_t)b * Hq * D + e] = __float2bfloat16_rn(val);
        if (e % D == 0) {
            const float l2 = ls > 0.f ? mu + __log2f(ls) : -INFINITY;
            lse2_ws[b * 16 + row] = l2;
            if (lse_out) lse_out[b * Hq + row] = l2 * kLn2;
        }
    }
}

// score-bit bin relative to a base, clamped to [0, 255]
HS2_DEV int score_bin(uint32_t bits, uint32_t base) {
    return bits <= base ? 0 : (int)min((bits - base) >> kBinShift, 255u);
}
HS2_DEV uint32_t seq_base(int Hq, int T) {
    return __float_as_uint((float)Hq / (256.f * (float)T));
}

// ------------------------------------------------------------------ pass 2
template <int D, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
pass2_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_ks,
             const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lengths, int Tmax,
             int Hq, int W, int chunk_len, float qk_scale, const float* __restrict__ lse2_ws,
             float* __restrict__ scores, int score_ld, unsigned* __restrict__ hist_g,
             unsigned* __restrict__ flags) {
    using SG = Stage<D, FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ Bars bars;
    __shared__ unsigned hist[256];
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = lane_id(), g = lane >> 2, c = lane & 3;
    const int T = __ldg(lengths + b);
    const int n_cand = (T >= 1 && T <= Tmax) ? max(0, T - W) : 0;  // candidates 0..T-1-W
    const int s_begin = chunk * chunk_len;
    const int s_end = min(s_begin + chunk_len, n_cand);
    const int n_tiles = s_end > s_begin ? (s_end - s_begin + TOK - 1) / TOK : 0;
    if (n_tiles == 0) return;
    volatile int* abort_ = &bars.abort_;
    const uint32_t base = seq_base(Hq, T);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; i++) {
            mbar_init(&bars.full[i], 1);
            mbar_init(&bars.empty[i], CWARPS);
        }
        bars.abort_ = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == CWARPS) {
        if (lane == 0) {
            int armed = 0;
            for (int j = 0; j < n_tiles && !*abort_; j++) {
                const int st = j % NST, u = j / NST;
                if (u > 0 && !mbar_wait(&bars.empty[st], (u - 1) & 1, abort_, flags)) break;
                issue_stage<D, FP8>(smem + st * SG::P2, &map_k, nullptr, &map_ks, nullptr,
                                    s_begin + j * TOK, b, &bars.full[st]);
                armed++;
            }
            if (*abort_) {
                volatile int no_abort = 0;
                for (int j = max(0, armed - NST); j < armed; j++)
                    mbar_wait(&bars.full[j % NST], (j / NST) & 1, &no_abort, flags);
            }
        }
    } else {
        WarpAttn<D, FP8> wa;
        wa.load_q(q + (size_t)b * Hq * D, Hq);
        float lse2[2];
        lse2[0] = g < Hq ? __ldcg(lse2_ws + b * 16 + g) : INFINITY;
        lse2[1] = g + 8 < Hq ? __ldcg(lse2_ws + b * 16 + g + 8) : INFINITY;
        float* srow = scores + (size_t)b * score_ld;
        for (int j = 0; j < n_tiles; j++) {
            const int st = j % NST;
            if (!mbar_wait(&bars.full[st], (j / NST) & 1, abort_, flags)) break;
            const uint8_t* sb = smem + st * SG::P2;
            const float* kst = reinterpret_cast<const float*>(sb + SG::TILE);
            const int tok0 = s_begin + j * TOK + 16 * warp;
            TileRegs<D, FP8> tr;
            load_tile_smem<D, FP8>(tr, sb, nullptr, FP8 ? kst : nullptr, nullptr, 16 * warp,
                                   tok0, s_end);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.empty[st]);
            float s[2][4];
            wa.qk(tr, s);
            wa.scale_mask(tr, s, qk_scale);
            float cs[4];
#pragma unroll
            for (int jj = 0; jj < 2; jj++)
#pragma unroll
                for (int e = 0; e < 2; e++)
                    cs[2 * jj + e] = ex2(s[jj][e] - lse2[0]) + ex2(s[jj][2 + e] - lse2[1]);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 4);
                cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 8);
                cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 16);
            }
            // lanes with g < 4 take one of their row group's four keys each:
            // lane (g, c) -> key {2c, 2c+1, 2c+8, 2c+9}[g]; equal bins are
            // counted once per warp (match + popc)
            if (g < 4) {
                const int kk = (g < 2) ? 2 * c + g : 2 * c + 8 + (g - 2);
                const float sc = g == 0 ? cs[0] : g == 1 ? cs[1] : g == 2 ? cs[2] : cs[3];
                const bool v = tr.kval[g];
                const int bn = v ? score_bin(__float_as_uint(sc), base) : -1;
                if (v) srow[tok0 + kk] = sc;
                const unsigned grp = __match_any_sync(0x0000ffffu, bn);
                if (v && (lane == __ffs(grp) - 1)) atomicAdd(&hist[bn], (unsigned)__popc(grp));
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (hist[i]) atomicAdd(hist_g + b * 256 + i, hist[i]);
}

// ------------------------------------------------------------------ gather
// The exact cut of one chunk (every thread of the CTA, blockDim.x >= 256):
// the bin of the k-th largest score from the sequence's histogram; the
// chunk's scores above it go into the row, those inside it to the boundary
// buffer; the last CTA of the sequence adds the window, the boundary bin's
// best keys (ties to the lower position) and the padding.  sk: BCAP keys of
// shared memory.
struct GatherShared {
    int bin, above, in_bin;
    unsigned last;
    int hist[260];
};

HS2_DEV void exact_gather_chunk(const float* __restrict__ scores, int score_ld,
                                const unsigned* __restrict__ hist_g, int b, int T, int Tmax,
                                int Hq, int W, int k, int chunk, int chunk_len, int n_chunks,
                                unsigned* __restrict__ out_cnt, unsigned* __restrict__ bnd_cnt,
                                uint64_t* __restrict__ bnd, unsigned* __restrict__ counter,
                                int32_t* __restrict__ idx, uint64_t* sk, GatherShared& sh) {
    const bool ok = T >= 1 && T <= Tmax;
    const int n_cand = ok ? max(0, T - W) : 0;
    const int t = T - 1;
    const int wl = ok ? min(T, W) : 0;
    const int S = W + k;
    const float* srow = scores + (size_t)b * score_ld;  // score_ld % 4 == 0
    int32_t* row = idx + (size_t)b * S;
    const uint32_t base = seq_base(Hq, T);
    const int s_begin = chunk * chunk_len;
    const int s_end = min(s_begin + chunk_len, n_cand);
    if (k > 0 && n_cand > k) {
        if (threadIdx.x < 32) {
            for (int i = threadIdx.x; i < 256; i += 32) sh.hist[i] = (int)__ldcg(hist_g + b * 256 + i);
            __syncwarp();
            int above, in_bin;
            const int j = warp_find_bin(sh.hist, k, &above, &in_bin);
            if (threadIdx.x == 0) {
                sh.bin = j;
                sh.above = above;
                sh.in_bin = in_bin;
            }
        }
        __syncthreads();
        const int j = sh.bin;
        // chunks start on 128-token boundaries: 4 scores per 16-byte load,
        // 4 loads per thread in flight per step
        for (int s0 = s_begin + 4 * threadIdx.x; s0 < s_end; s0 += 16 * blockDim.x) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int s = s0 + u * 4 * blockDim.x;
                v[u] = s < s_end ? __ldcg(reinterpret_cast<const float4*>(srow + s))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int s = s0 + u * 4 * blockDim.x + i;
                    if (s >= s_end) continue;
                    const int bn = score_bin(__float_as_uint(e[i]), base);
                    if (bn > j) {
                        row[wl + atomicAdd(out_cnt + b, 1u)] = s;
                    } else if (bn == j) {
                        const unsigned p = atomicAdd(bnd_cnt + b, 1u);
                        if (p < (unsigned)BCAP)
                            bnd[(size_t)b * BCAP + p] = make_key(e[i], (uint32_t)s);
                    }
                }
            }
        }
    } else if (k > 0) {
        for (int s = s_begin + threadIdx.x; s < s_end; s += blockDim.x) row[wl + s] = s;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sh.last = (atomicAdd(counter + b, 1u) == (unsigned)(n_chunks - 1));
    __syncthreads();
    if (!sh.last) return;
    __threadfence();
    // last CTA of the sequence: window, boundary bin, padding
    for (int i = threadIdx.x; i < wl; i += blockDim.x) row[i] = t - wl + 1 + i;
    int n_glob = min(k, n_cand);
    if (k > 0 && n_cand > k) {
        const int need = k - sh.above;
        const unsigned nb_all = __ldcg(bnd_cnt + b);
        int* hist = sh.hist;
        if (nb_all <= (unsigned)BCAP) {
            const int nb = (int)nb_all;
            for (int i = threadIdx.x; i < nb; i += blockDim.x)
                sk[i] = __ldcg(bnd + (size_t)b * BCAP + i);
            __syncthreads();
            const uint64_t thr =
                block_radix_threshold([&](int i) { return sk[i]; }, nb, need, hist);
            __syncthreads();
            for (int i = threadIdx.x; i < nb; i += blockDim.x)
                if (sk[i] >= thr) row[wl + atomicAdd(out_cnt + b, 1u)] = (int32_t)key_pos(sk[i]);
        } else {
            // the boundary bin overflowed: exact cut over every candidate of it
            const int j = sh.bin;
            auto key_at = [&](int s) {
                const float sc = __ldcg(srow + s);
                return score_bin(__float_as_uint(sc), base) == j ? make_key(sc, (uint32_t)s)
                                                                 : (uint64_t)0;
            };
            const uint64_t thr = block_radix_threshold(key_at, n_cand, need, hist);
            __syncthreads();
            for (int s = threadIdx.x; s < n_cand; s += blockDim.x) {
                const uint64_t key = key_at(s);
                if (key != 0 && key >= thr) row[wl + atomicAdd(out_cnt + b, 1u)] = s;
            }
        }
    }
    __syncthreads();
    for (int i = wl + n_glob + threadIdx.x; i < S; i += blockDim.x) row[i] = -1;
}

// grid (n_chunks, B), 256 threads, dynamic shared memory BCAP keys: the exact
// cut after the exact pass 2.
__global__ void __launch_bounds__(256)
gather_kernel(const float* __restrict__ scores, int score_ld, const unsigned* __restrict__ hist_g,
              const int32_t* __restrict__ lengths, int Tmax, int Hq, int W, int k,
              int chunk_len, int n_chunks, unsigned* __restrict__ out_cnt,
              unsigned* __restrict__ bnd_cnt, uint64_t* __restrict__ bnd,
              unsigned* __restrict__ counter, int32_t* __restrict__ idx) {
    extern __shared__ uint64_t sk[];  // BCAP keys (last CTA)
    __shared__ GatherShared sh;
    // the scores and their histogram come from the kernel before
    griddep_launch();
    griddep_wait();
    const int b = blockIdx.y;
    exact_gather_chunk(scores, score_ld, hist_g, b, __ldg(lengths + b), Tmax, Hq, W, k, blockIdx.x,
                       chunk_len, n_chunks, out_cnt, bnd_cnt, bnd, counter, idx, sk, sh);
}

}  // namespace dec
}  // namespace hs2
