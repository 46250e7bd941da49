// Decode selection from a per-token sketch (FP8 e4m3 cache, d = 128).
//
// HySparse2 summary (onedev.kr/papers/146), 'How it works': the full layer
// ranks every older token by its exact attention score, here the sum over
// query heads of the softmax probability,
//     score(s) = sum_h 2^(x_h(s) - lse2_h),   x_h(s) = scale * log2(e) * <q_h, k_s>,
// and keeps the top k (ties to the lower position) besides the window.
//
// lse2_h needs the whole cache, so a single streaming pass cannot form the
// score.  Instead of reading K a second time, pass 1 leaves behind, for every
// token, one byte per head: the top 8 bits (5 exponent and 3 mantissa bits)
// of the f16 of p_h = 2^(x_h - R_h), rounded toward zero, where R_h is the
// chunk's softmax reference for that 128-token tile (saved per tile).  A code
// c therefore brackets p_h:  F(c) <= p_h < F(c + 1),  F(c) = the f16 with
// bits c << 7.  For a normal F(c), F(c + 1) <= 9/8 F(c); codes below 2^-14
// are subnormal and step by 2^-17.  With w_h = 2^(R_h - lse2_h) <= 2^-6
// (R_h sits kSk = 6 below a running maximum, itself <= lse2_h),
//     L(s) = sum_h w_h F(c_h)  <=  score(s)  <=  9/8 L(s) + Hq 2^-23.
//
// sketch_score_kernel   L(s) for every older token, and a 256-bin histogram
//                       of L per sequence (1/16-octave bins);
// sketch_gather_kernel  the bin holding the k-th largest L gives E, a lower
//                       bound of the k-th largest score.  A token can be in
//                       the top k only if 9/8 L + eps >= E; exactly those are
//                       rescored from their K rows (a warp per 16 tokens, one
//                       16-head x 16-key tensor-core tile); the
//                       last CTA of the sequence bins their exact scores, takes
//                       every key above the bin of the k-th and ranks the
//                       keys inside that bin (ties to the lower position).
// If a sequence's candidates overflow the boundary buffer (many near-equal
// scores, e.g. repeated keys), it is flagged and the exact pass 2 and its
// gather run for that sequence instead (their launches are gated on the flag).
#pragma once

#include "decode_tc.cuh"
#include "gather_attn.cuh"

namespace hs2 {
namespace dsk {

constexpr int TOK = 128;
constexpr int kScoreThreads = 256;
constexpr int kGatherThreads = 512;
constexpr int kCandCap = 2048;  // candidates one CTA may rescore

// ----------------------------------------------------------------------------
// L(s) per token and the per-sequence histogram.  grid (G, B): the CTAs of a
// sequence stride over its 128-token tiles, a warp per tile, two tiles of
// codes in flight per warp.
__global__ void __launch_bounds__(kScoreThreads)
sketch_score_kernel(const uint8_t* __restrict__ sketch, const float* __restrict__ rsnap,
                    int sk_tiles, const int32_t* __restrict__ lengths, int Tmax, int Hq, int W,
                    int k, const float* __restrict__ lse2_ws, float* __restrict__ lrow,
                    int score_ld, unsigned* __restrict__ hist_g) {
    // one counter column per lane: the lanes of a warp never collide
    __shared__ unsigned hist[256 * 32];
    griddep_launch();
    const int b = blockIdx.y;
    const int T = __ldg(lengths + b);
    const int n_cand = (T >= 1 && T <= Tmax) ? max(0, T - W) : 0;
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) hist[i] = 0;
    // the sketch, the tile references and lse2 come from the kernel before
    griddep_wait();
    if (k <= 0 || n_cand <= k) return;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = lane_id();
    constexpr int NW = kScoreThreads / 32;
    const uint32_t base = dec::seq_base(Hq, T);
    const float l2h = (lane & 15) < Hq ? __ldcg(lse2_ws + b * 16 + (lane & 15)) : INFINITY;
    float* srow = lrow + (size_t)b * score_ld;
    const uint8_t* sk_b = sketch + (size_t)b * Tmax * 16;
    const float* rs_b = rsnap + (size_t)b * sk_tiles * 16;
    const int n_tiles = (n_cand + TOK - 1) / TOK;
    const int stride = gridDim.x * NW;
    for (int g0 = blockIdx.x * NW + warp; g0 < n_tiles; g0 += 2 * stride) {
        uint4 cw[2][4];
        float rv[2];
#pragma unroll
        for (int v = 0; v < 2; v++) {
            const int g = g0 + v * stride;
            rv[v] = g < n_tiles ? __ldcg(rs_b + (size_t)g * 16 + (lane & 15)) : 0.f;
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int tok = g * TOK + u * 32 + lane;
                cw[v][u] = (g < n_tiles && tok < n_cand)
                               ? __ldcg(reinterpret_cast<const uint4*>(sk_b + (size_t)tok * 16))
                               : make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int v = 0; v < 2; v++) {
            const int g = g0 + v * stride;
            if (g >= n_tiles) break;
            // tile weights w_h = 2^(R_h - lse2_h), zero for padded heads
            const float wl = ((lane & 15) < Hq && rv[v] != -INFINITY) ? ex2(rv[v] - l2h) : 0.f;
            float w[16];
#pragma unroll
            for (int h = 0; h < 16; h++) w[h] = __shfl_sync(0xffffffffu, wl, h);
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int tok = g * TOK + u * 32 + lane;
                const uint32_t wd[4] = {cw[v][u].x, cw[v][u].y, cw[v][u].z, cw[v][u].w};
                float L = 0.f;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    // codes of heads 4i..4i+3 -> f16 bit patterns c << 7
                    const float2 a = f16x2_to_float2(prmt(wd[i], 0u, 0x1404u) >> 1);
                    const float2 c = f16x2_to_float2(prmt(wd[i], 0u, 0x3424u) >> 1);
                    L = fmaf(w[4 * i], a.x, L);
                    L = fmaf(w[4 * i + 1], a.y, L);
                    L = fmaf(w[4 * i + 2], c.x, L);
                    L = fmaf(w[4 * i + 3], c.y, L);
                }
                if (tok < n_cand) {
                    srow[tok] = L;
                    atomicAdd(&hist[dec::score_bin(__float_as_uint(L), base) * 32 + lane], 1u);
                }
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        unsigned c = 0;
        for (int l = 0; l < 32; l++) c += hist[i * 32 + ((l + i) & 31)];  // banks differ
        if (c) atomicAdd(hist_g + b * 256 + i, c);
    }
}

struct GatherShared {
    int cand[kCandCap];   // this CTA's candidate positions
    int hist[260];
    int bin, above;
    unsigned n_cand, n_out, last;
};

// ----------------------------------------------------------------------------
// Candidates, exact rescoring and the cut.  grid (n_chunks, B), kGatherThreads
// threads, dynamic shared memory BCAP keys (used by the last CTA of each
// sequence).  A warp rescores 16 candidates at a time from their K rows: the
// same expression the exact pass evaluates, sum_h 2^(<q_h, k_s> sK qk2 - lse2_h).
__global__ void __launch_bounds__(kGatherThreads)
sketch_gather_kernel(const float* __restrict__ lrow, int score_ld, const unsigned* __restrict__ hist_g,
                     const uint8_t* __restrict__ kc, const float* __restrict__ ksc,
                     const __nv_bfloat16* __restrict__ q, const float* __restrict__ lse2_ws,
                     float qk2, const int32_t* __restrict__ lengths, int Tmax, int Hq, int W, int k,
                     int chunk_len, int n_chunks, unsigned* __restrict__ bnd_cnt,
                     uint64_t* __restrict__ bnd, unsigned* __restrict__ ovf,
                     unsigned* __restrict__ counter, int32_t* __restrict__ idx) {
    extern __shared__ uint64_t skeys[];
    __shared__ GatherShared sh;
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int T = __ldg(lengths + b);
    const bool ok = T >= 1 && T <= Tmax;
    const int n_cand = ok ? max(0, T - W) : 0;
    const int t = T - 1;
    const int wl = ok ? min(T, W) : 0;
    const int S = W + k;
    int32_t* row = idx + (size_t)b * S;
    const int s_begin = chunk * chunk_len;
    const int s_end = min(s_begin + chunk_len, n_cand);
    const bool ranked = k > 0 && n_cand > k;
    const bool work = ranked && s_end > s_begin;
    griddep_launch();
    // L, its histogram and lse2 come from the kernels before
    griddep_wait();
    if (work) {
        const float* srow = lrow + (size_t)b * score_ld;
        // the first batch of L values is requested before the histogram is
        // known (chunks start on 128-token boundaries; rows are padded to 4)
        constexpr int U = 8;
        float4 v[U];
        auto load_batch = [&](int s0) {
#pragma unroll
            for (int u = 0; u < U; u++) {
                const int s = s0 + u * 4 * kGatherThreads;
                v[u] = s < s_end ? __ldcg(reinterpret_cast<const float4*>(srow + s))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        int s0 = s_begin + 4 * (int)threadIdx.x;
        load_batch(s0);
        if (warp == 0) {
            for (int i = lane; i < 256; i += 32) sh.hist[i] = (int)__ldcg(hist_g + b * 256 + i);
            __syncwarp();
            int above, in_bin;
            const int j = warp_find_bin(sh.hist, k, &above, &in_bin);
            if (lane == 0) {
                sh.bin = j;
                sh.n_cand = 0;
            }
        }
        __syncthreads();
        const int j = sh.bin;
        const uint32_t base = dec::seq_base(Hq, T);
        // E <= the k-th largest L <= the k-th largest score; a token with
        // 9/8 L + eps < E is out.  The factor (1 - 2^-10) absorbs rounding in
        // L, in the pass-1 logits and in the rescored ones.
        const float E = j <= 0 ? 0.f : __uint_as_float(base + ((uint32_t)j << dec::kBinShift));
        const float eps = (float)Hq * 0x1p-23f;
        const float thr = (E - eps) * (8.f / 9.f) * (1.f - 0x1p-10f);
        for (;;) {
#pragma unroll
            for (int u = 0; u < U; u++) {
                const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int s = s0 + u * 4 * kGatherThreads + i;
                    if (s < s_end && e[i] >= thr) {
                        const unsigned p = atomicAdd(&sh.n_cand, 1u);
                        if (p < (unsigned)kCandCap) sh.cand[p] = s;
                    }
                }
            }
            s0 += 4 * U * kGatherThreads;
            if (s0 - 4 * (int)threadIdx.x >= s_end) break;
            load_batch(s0);
        }
        __syncthreads();
        const int nc = (int)sh.n_cand;
        if (nc > kCandCap) {
            if (threadIdx.x == 0) atomicOr(ovf + b, 1u);
        } else {
            // a warp per 16 candidates: their K rows go straight into the
            // fragments of a 16-head x 16-key tensor-core tile (the sparse
            // layers' warp routine), then sum_h 2^(logit_h - lse2_h) per key
            const int g = lane >> 2, c = lane & 3;
            const float l2a = g < Hq ? __ldcg(lse2_ws + b * 16 + g) : INFINITY;
            const float l2b = g + 8 < Hq ? __ldcg(lse2_ws + b * 16 + g + 8) : INFINITY;
            const uint8_t* kb = kc + (size_t)b * Tmax * 128;
            const float* ksb = ksc + (size_t)b * Tmax;
            WarpAttn<128, true> wa;
            wa.load_q(q + (size_t)b * Hq * 128, Hq);  // the range is checked by pass 1
            constexpr int NW = kGatherThreads / 32;
            for (int i0 = warp * 16; i0 < nc; i0 += NW * 16) {
                const int my = (lane < 16 && i0 + lane < nc) ? sh.cand[i0 + lane] : -1;
                int key_k[2], key_v[4];
                distribute_keys(my, key_k, key_v);
                TileRegs<128, true> tr;
                wa.load_tile(tr, kb, kb, ksb, ksb, key_k, key_v);
                float sx[2][4];
                wa.qk(tr, sx);
                wa.scale_mask(tr, sx, qk2 * 256.f);  // e4m3 rows enter as f16 x 2^-8
                // this lane: heads g, g+8 of keys 2c, 2c+1 (tile 0), 8+2c, 9+2c (tile 1)
                float sc[4];
#pragma unroll
                for (int j = 0; j < 2; j++)
#pragma unroll
                    for (int e = 0; e < 2; e++)
                        sc[2 * j + e] = ex2(sx[j][e] - l2a) + ex2(sx[j][2 + e] - l2b);
#pragma unroll
                for (int u = 0; u < 4; u++)
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1)
                        sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
                // lanes 0..3 hold the sums of the tile's 16 keys; one
                // boundary-buffer reservation per tile
                const int n_tile = min(16, nc - i0);
                unsigned basep = 0;
                if (lane == 0) basep = atomicAdd(bnd_cnt + b, (unsigned)n_tile);
                basep = __shfl_sync(0xffffffffu, basep, 0);
                if (lane < 4) {
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const int col = (u < 2) ? 2 * c + u : 8 + 2 * c + (u - 2);
                        if (col >= n_tile) continue;
                        const int pos = sh.cand[i0 + col];
                        const unsigned p = basep + (unsigned)col;
                        if (p < (unsigned)dec::BCAP)
                            bnd[(size_t)b * dec::BCAP + p] = make_key(sc[u], (uint32_t)pos);
                        else
                            atomicOr(ovf + b, 1u);
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
    const int n_glob = min(k, n_cand);
    if (ranked) {
        const unsigned nb_all = __ldcg(bnd_cnt + b);
        if (__ldcg(ovf + b) != 0u || nb_all < (unsigned)k || nb_all > (unsigned)dec::BCAP) {
            // the exact pass and its gather write this sequence's row
            if (threadIdx.x == 0) atomicOr(ovf + b, 1u);
            return;
        }
        // the exact top k of the candidates' keys: bin them by score, take
        // every key above the bin of the k-th, rank the keys inside that bin
        const int nb = (int)nb_all;
        const uint32_t base = dec::seq_base(Hq, T);
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.hist[i] = 0;
        if (threadIdx.x == 0) {
            sh.n_cand = 0;  // boundary keys gathered
            sh.n_out = 0;   // keys written
        }
        __syncthreads();
        constexpr int PER = dec::BCAP / kGatherThreads;
        uint64_t kv[PER];
#pragma unroll
        for (int u = 0; u < PER; u++) {
            const int i = threadIdx.x + u * kGatherThreads;
            kv[u] = i < nb ? __ldcg(bnd + (size_t)b * dec::BCAP + i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < PER; u++) {
            const int i = threadIdx.x + u * kGatherThreads;
            const int bn = i < nb ? dec::score_bin((uint32_t)(kv[u] >> 32), base) : -1;
            const unsigned grp = __match_any_sync(0xffffffffu, bn);
            if (bn >= 0 && lane == __ffs(grp) - 1) atomicAdd(&sh.hist[bn], __popc(grp));
        }
        __syncthreads();
        if (warp == 0) {
            int above, in_bin;
            const int j = warp_find_bin(sh.hist, k, &above, &in_bin);
            if (lane == 0) {
                sh.bin = j;
                sh.above = above;
            }
        }
        __syncthreads();
        const int jb = sh.bin, need = k - sh.above;
        // keys above the boundary bin are in; the boundary bin's go to skeys
#pragma unroll
        for (int u = 0; u < PER; u++) {
            const int i = threadIdx.x + u * kGatherThreads;
            if (i >= nb) continue;
            const int bn = dec::score_bin((uint32_t)(kv[u] >> 32), base);
            if (bn > jb)
                row[wl + atomicAdd(&sh.n_out, 1u)] = (int32_t)key_pos(kv[u]);
            else if (bn == jb)
                skeys[atomicAdd(&sh.n_cand, 1u)] = kv[u];
        }
        __syncthreads();
        // keys are unique: the rank of a boundary key among its bin decides
        const int m = (int)sh.n_cand;
        for (int i = threadIdx.x; i < m; i += blockDim.x) {
            const uint64_t key = skeys[i];
            int rank = 0;
            for (int q = 0; q < m; q++) rank += skeys[q] > key;
            if (rank < need) row[wl + atomicAdd(&sh.n_out, 1u)] = (int32_t)key_pos(key);
        }
    }
    for (int i = threadIdx.x; i < wl; i += blockDim.x) row[i] = t - wl + 1 + i;
    for (int i = wl + n_glob + threadIdx.x; i < S; i += blockDim.x) row[i] = -1;
}

}  // namespace dsk
}  // namespace hs2
