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
// sketch_select_kernel forms L(s) for every older token and a 256-bin
// histogram of L per sequence (1/16-octave bins).  The bin holding the k-th
// largest L gives E, a lower bound of the k-th largest score: a token can be
// in the top k only if 9/8 L + eps >= E, and exactly those are rescored from
// their K rows.  The last CTA of the sequence bins their exact scores, takes
// every key above the bin of the k-th and ranks the keys inside that bin
// (ties to the lower position).
// If a sequence's candidates overflow the boundary buffer (many near-equal
// scores, e.g. repeated keys), the last CTA's verdict sends every CTA of
// that sequence into the exact fallback: the exact score of every token of
// its chunk, a histogram of them, and the exact histogram cut.
#pragma once

#include "decode_tc.cuh"
#include "gather_attn.cuh"

namespace hs2 {
namespace dsk {

constexpr int TOK = 128;
constexpr int kThreads = 512;
constexpr int kCandCap = 2048;  // candidates one CTA may rescore

struct GatherShared {
    int cand[kCandCap];   // this CTA's candidate positions
    int hist[260];
    int bin, above;
    unsigned n_cand, n_out, last;
};

// Buffers of the exact fallback (zeroed before pass 1).
struct ExactArgs {
    unsigned* hist;     // [B][256] histogram of the exact scores
    unsigned* arrive;   // [B] CTAs that added theirs
    unsigned* out_cnt;  // [B] positions written above the boundary bin
    unsigned* bnd_cnt;  // [B] boundary keys
    unsigned* counter;  // [B] CTAs done with the exact cut
    unsigned* verdict;  // [B] 1: the sketch cut stands, 2: the exact fallback runs
};

// Bounded wait until *ctr reaches `target` (one thread); false if it gave up.
HS2_DEV bool wait_count(unsigned* ctr, unsigned target) {
    const uint64_t t0 = tc::globaltimer_ns();
    for (uint32_t i = 0;; i++) {
        unsigned seen;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(ctr) : "memory");
        if (seen >= target) return true;
        if ((i & 63u) == 63u && tc::globaltimer_ns() - t0 > tc::kWaitNs) return false;
        __nanosleep(64);
    }
}

// The exact fallback of a sequence whose candidates overflowed, run by every
// CTA of it on its own chunk: the exact score of each of the chunk's tokens
// (the rescoring routine over consecutive positions) into the score row and
// the sequence's histogram; once every chunk's is in, the exact cut.
HS2_DEV void exact_fallback(float* __restrict__ lrow, int score_ld, const uint8_t* __restrict__ kc,
                            const float* __restrict__ ksc, const __nv_bfloat16* __restrict__ q,
                            const float* __restrict__ lse2_ws, float qk2, int b, int chunk, int T,
                            int Tmax, int Hq, int W, int k, int chunk_len, int n_chunks,
                            uint64_t* __restrict__ bnd, int32_t* __restrict__ idx,
                            const ExactArgs& ex, uint64_t* skeys, GatherShared& sh,
                            dec::GatherShared& gsh, unsigned* flags) {
    const int warp = threadIdx.x >> 5, lane = lane_id();
    constexpr int NW = kThreads / 32;
    const int n_cand = max(0, T - W);
    const int s_begin = chunk * chunk_len;
    const int s_end = min(s_begin + chunk_len, n_cand);
    const uint32_t base = dec::seq_base(Hq, T);
    float* srow = lrow + (size_t)b * score_ld;
    for (int i = threadIdx.x; i < 256; i += kThreads) sh.hist[i] = 0;
    __syncthreads();
    if (s_end > s_begin) {
        const int g = lane >> 2, c = lane & 3;
        const float l2a = g < Hq ? __ldcg(lse2_ws + b * 16 + g) : INFINITY;
        const float l2b = g + 8 < Hq ? __ldcg(lse2_ws + b * 16 + g + 8) : INFINITY;
        const uint8_t* kb = kc + (size_t)b * Tmax * 128;
        const float* ksb = ksc + (size_t)b * Tmax;
        WarpAttn<128, true> wa;
        wa.load_q(q + (size_t)b * Hq * 128, Hq);
        for (int i0 = s_begin + warp * 16; i0 < s_end; i0 += NW * 16) {
            const int my = (lane < 16 && i0 + lane < s_end) ? i0 + lane : -1;
            int key_k[2], key_v[4];
            distribute_keys(my, key_k, key_v);
            TileRegs<128, true> tr;
            wa.load_tile(tr, kb, kb, ksb, ksb, key_k, key_v);
            float sx[2][4];
            wa.qk(tr, sx);
            wa.scale_mask(tr, sx, qk2 * 256.f);  // e4m3 rows enter as f16 x 2^-8
            float sc[4];
#pragma unroll
            for (int jj = 0; jj < 2; jj++)
#pragma unroll
                for (int e = 0; e < 2; e++)
                    sc[2 * jj + e] = ex2(sx[jj][e] - l2a) + ex2(sx[jj][2 + e] - l2b);
#pragma unroll
            for (int u = 0; u < 4; u++)
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
            if (lane < 4) {
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int s = i0 + ((u < 2) ? 2 * c + u : 8 + 2 * c + (u - 2));
                    if (s < s_end) {
                        srow[s] = sc[u];
                        atomicAdd(&sh.hist[dec::score_bin(__float_as_uint(sc[u]), base)], 1);
                    }
                }
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += kThreads)
        if (sh.hist[i]) atomicAdd(ex.hist + b * 256 + i, (unsigned)sh.hist[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        atomicAdd(ex.arrive + b, 1u);
        const bool met = wait_count(ex.arrive + b, (unsigned)n_chunks);
        __threadfence();
        if (!met) atomicOr(flags, FLAG_TIMEOUT);
        sh.last = met ? 0u : 1u;
    }
    __syncthreads();
    if (sh.last) return;
    dec::exact_gather_chunk(lrow, score_ld, ex.hist, b, T, Tmax, Hq, W, k, chunk, chunk_len,
                            n_chunks, ex.out_cnt, ex.bnd_cnt, bnd, ex.counter, idx, skeys, gsh);
}

// ----------------------------------------------------------------------------
// The selection after pass 1, one CTA per chunk of a sequence's cache: grid
// (n_chunks, B) (at most one CTA per SM, all resident at once), kThreads
// threads.  Dynamic shared memory: BCAP keys (phase 1: a histogram column per
// lane; phase 3: this CTA's rescored keys; phase 4: the boundary bin's keys),
// then, with LSM, the chunk's L values (else they go through the score row).
//   1. L(s) for the chunk's tokens from their sketch codes (a warp per
//      128-token tile, four tiles of codes in flight), and a histogram added
//      to the sequence's;
//   2. the CTAs of a sequence meet (a counter, bounded wait): the histogram
//      is complete;
//   3. candidates: tokens of the chunk with 9/8 L + eps >= E, rescored from
//      their K rows (a warp per 16 tokens, one 16-head x 16-key tensor-core
//      tile) with the expression the exact pass evaluates,
//      sum_h 2^(<q_h, k_s> sK qk2 - lse2_h), and appended to the boundary
//      buffer with one reservation per CTA;
//   4. the last CTA of the sequence checks the boundary buffer and gives the
//      verdict the others wait for: the sketch cut (it cuts the exact top k
//      of those keys) or, on an overflow, the exact fallback by all of them.
// A wait that gives up records FLAG_TIMEOUT: the call then reports
// HS2_ERR_TIMEOUT and the sequence's row is not valid.
constexpr int kTilesInFlight = 4;

inline constexpr size_t select_smem_bytes(bool lsm, int chunk_len) {
    return (size_t)dec::BCAP * sizeof(uint64_t) + (lsm ? (size_t)chunk_len * sizeof(float) : 0);
}

template <bool LSM>
__global__ void __launch_bounds__(kThreads)
sketch_select_kernel(const uint8_t* __restrict__ sketch, const float* __restrict__ rsnap,
                     int sk_tiles, float* __restrict__ lrow, int score_ld,
                     unsigned* __restrict__ hist_g, unsigned* __restrict__ arrive,
                     const uint8_t* __restrict__ kc, const float* __restrict__ ksc,
                     const __nv_bfloat16* __restrict__ q, const float* __restrict__ lse2_ws,
                     float qk2, const int32_t* __restrict__ lengths, int Tmax, int Hq, int W, int k,
                     int chunk_len, int n_chunks, unsigned* __restrict__ bnd_cnt,
                     uint64_t* __restrict__ bnd, unsigned* __restrict__ ovf,
                     unsigned* __restrict__ counter, int32_t* __restrict__ idx,
                     const ExactArgs ex, unsigned* __restrict__ flags) {
    extern __shared__ uint64_t skeys[];
    unsigned* hist_l = reinterpret_cast<unsigned*>(skeys);
    float* lsm = reinterpret_cast<float*>(skeys + dec::BCAP);
    __shared__ GatherShared sh;
    __shared__ dec::GatherShared gsh;
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
    constexpr int NW = kThreads / 32;
    float* srow = lrow + (size_t)b * score_ld;
    for (int i = threadIdx.x; i < 256 * 32; i += kThreads) hist_l[i] = 0;
    griddep_launch();
    // the sketch, the tile references and lse2 come from pass 1
    griddep_wait();
    if (ranked) {
        __syncthreads();
        const uint32_t base = dec::seq_base(Hq, T);
        if (work) {
            // ---- 1. L(s) over this chunk's tiles
            const float l2h =
                (lane & 15) < Hq ? __ldcg(lse2_ws + b * 16 + (lane & 15)) : INFINITY;
            const uint8_t* sk_b = sketch + (size_t)b * Tmax * 16;
            const float* rs_b = rsnap + (size_t)b * sk_tiles * 16;
            const int g_end = (s_end + TOK - 1) / TOK;
            const uint64_t pol = l2_evict_first();  // the last read of the sketch
            constexpr int V = kTilesInFlight;
            for (int g0 = s_begin / TOK + warp; g0 < g_end; g0 += V * NW) {
                uint4 cw[V][4];
                float rv[V];
#pragma unroll
                for (int v = 0; v < V; v++) {
                    const int g = g0 + v * NW;
                    rv[v] = g < g_end ? __ldcg(rs_b + (size_t)g * 16 + (lane & 15)) : 0.f;
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const int tok = g * TOK + u * 32 + lane;
                        cw[v][u] = (g < g_end && tok < s_end)
                                       ? ldcg_hint(sk_b + (size_t)tok * 16, pol)
                                       : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
#pragma unroll
                for (int v = 0; v < V; v++) {
                    const int g = g0 + v * NW;
                    if (g >= g_end) break;
                    // tile weights w_h = 2^(R_h - lse2_h), zero for padded heads
                    const float wlh =
                        ((lane & 15) < Hq && rv[v] != -INFINITY) ? ex2(rv[v] - l2h) : 0.f;
                    float w[16];
#pragma unroll
                    for (int h = 0; h < 16; h++) w[h] = __shfl_sync(0xffffffffu, wlh, h);
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
                        if (tok < s_end) {
                            if constexpr (LSM)
                                lsm[tok - s_begin] = L;
                            else
                                srow[tok] = L;
                            atomicAdd(&hist_l[dec::score_bin(__float_as_uint(L), base) * 32 + lane],
                                      1u);
                        }
                    }
                }
            }
            __syncthreads();
            for (int i = threadIdx.x; i < 256; i += kThreads) {
                unsigned c = 0;
                for (int l = 0; l < 32; l++) c += hist_l[i * 32 + ((l + i) & 31)];  // banks differ
                if (c) atomicAdd(hist_g + b * 256 + i, c);
            }
        }
        // ---- 2. every chunk of the sequence has added its histogram
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            atomicAdd(arrive + b, 1u);
            const bool gave_up = !wait_count(arrive + b, (unsigned)n_chunks);
            __threadfence();
            if (gave_up) {
                atomicOr(flags, FLAG_TIMEOUT);
                atomicOr(ovf + b, 1u);
            }
            sh.last = gave_up ? 1u : 0u;  // reused below as the give-up mark
        }
        __syncthreads();
        if (sh.last) return;
    }
    if (work) {
        // ---- 3. candidates of this chunk
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
        // the warps' query fragments meanwhile (the range is checked by pass 1)
        WarpAttn<128, true> wa;
        wa.load_q(q + (size_t)b * Hq * 128, Hq);
        __syncthreads();
        const int j = sh.bin;
        const uint32_t base = dec::seq_base(Hq, T);
        // E <= the k-th largest L <= the k-th largest score; a token with
        // 9/8 L + eps < E is out.  The factor (1 - 2^-10) absorbs rounding in
        // L, in the pass-1 logits and in the rescored ones.
        const float E = j <= 0 ? 0.f : __uint_as_float(base + ((uint32_t)j << dec::kBinShift));
        const float eps = (float)Hq * 0x1p-23f;
        const float thr = (E - eps) * (8.f / 9.f) * (1.f - 0x1p-10f);
        auto take = [&](int s, float e) {
            if (s < s_end && e >= thr) {
                const unsigned p = atomicAdd(&sh.n_cand, 1u);
                if (p < (unsigned)kCandCap) sh.cand[p] = s;
            }
        };
        if constexpr (LSM) {
            const int n = s_end - s_begin;
            constexpr int U = 8;
            for (int i0 = threadIdx.x; i0 < n; i0 += U * kThreads) {
                float e[U];
#pragma unroll
                for (int u = 0; u < U; u++) {
                    const int i = i0 + u * kThreads;
                    e[u] = i < n ? lsm[i] : -1.f;
                }
#pragma unroll
                for (int u = 0; u < U; u++) take(s_begin + i0 + u * kThreads, e[u]);
            }
        } else {
            // chunks start on 128-token boundaries; rows are padded to 4
            constexpr int U = 8;
            for (int s0 = s_begin + 4 * (int)threadIdx.x; s0 < s_end; s0 += 4 * U * kThreads) {
                float4 v[U];
#pragma unroll
                for (int u = 0; u < U; u++) {
                    const int s = s0 + u * 4 * kThreads;
                    v[u] = s < s_end ? __ldcg(reinterpret_cast<const float4*>(srow + s))
                                     : make_float4(-1.f, -1.f, -1.f, -1.f);
                }
#pragma unroll
                for (int u = 0; u < U; u++) {
                    const int s = s0 + u * 4 * kThreads;
                    take(s, v[u].x);
                    take(s + 1, v[u].y);
                    take(s + 2, v[u].z);
                    take(s + 3, v[u].w);
                }
            }
        }
        __syncthreads();
        const int nc = (int)sh.n_cand;
        if (nc > kCandCap) {
            if (threadIdx.x == 0) atomicOr(ovf + b, 1u);
        } else {
            // a warp per 16 candidates: their K rows go straight into the
            // fragments of a 16-head x 16-key tensor-core tile (the sparse
            // layers' warp routine), then sum_h 2^(logit_h - lse2_h) per key,
            // kept at the candidate's slot in shared memory
            const int g = lane >> 2, c = lane & 3;
            const float l2a = g < Hq ? __ldcg(lse2_ws + b * 16 + g) : INFINITY;
            const float l2b = g + 8 < Hq ? __ldcg(lse2_ws + b * 16 + g + 8) : INFINITY;
            const uint8_t* kb = kc + (size_t)b * Tmax * 128;
            const float* ksb = ksc + (size_t)b * Tmax;
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
                for (int jj = 0; jj < 2; jj++)
#pragma unroll
                    for (int e = 0; e < 2; e++)
                        sc[2 * jj + e] = ex2(sx[jj][e] - l2a) + ex2(sx[jj][2 + e] - l2b);
#pragma unroll
                for (int u = 0; u < 4; u++)
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1)
                        sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
                // lanes 0..3 hold the sums of the tile's 16 keys
                if (lane < 4) {
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const int col = (u < 2) ? 2 * c + u : 8 + 2 * c + (u - 2);
                        if (i0 + col < nc)
                            skeys[i0 + col] = make_key(sc[u], (uint32_t)sh.cand[i0 + col]);
                    }
                }
            }
            __syncthreads();
            // one reservation in the sequence's boundary buffer for all of them
            if (threadIdx.x == 0) sh.above = nc > 0 ? (int)atomicAdd(bnd_cnt + b, (unsigned)nc) : 0;
            __syncthreads();
            const int p0 = sh.above;
            if (p0 + nc > dec::BCAP) {
                if (threadIdx.x == 0) atomicOr(ovf + b, 1u);
            } else {
                for (int i = threadIdx.x; i < nc; i += kThreads)
                    bnd[(size_t)b * dec::BCAP + p0 + i] = skeys[i];
            }
        }
    } else if (k > 0 && !ranked) {
        for (int s = s_begin + threadIdx.x; s < s_end; s += blockDim.x) row[wl + s] = s;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sh.last = (atomicAdd(counter + b, 1u) == (unsigned)(n_chunks - 1));
    __syncthreads();
    const bool last = sh.last != 0;
    const int n_glob = min(k, n_cand);
    if (ranked) {
        // ---- the verdict: the last CTA of the sequence checks the boundary
        // buffer; the others wait for it, since an overflow needs them all
        if (threadIdx.x == 0) {
            unsigned v = 0;
            if (last) {
                __threadfence();
                const unsigned nb_all = __ldcg(bnd_cnt + b);
                v = (__ldcg(ovf + b) != 0u || nb_all < (unsigned)k || nb_all > (unsigned)dec::BCAP)
                        ? 2u
                        : 1u;
                asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ex.verdict + b), "r"(v)
                             : "memory");
            } else if (!wait_count(ex.verdict + b, 1u)) {
                atomicOr(flags, FLAG_TIMEOUT);
            } else {
                v = __ldcg(ex.verdict + b);
            }
            __threadfence();
            sh.n_out = v;
        }
        __syncthreads();
        const unsigned verdict = sh.n_out;
        if (verdict == 2u) {
            exact_fallback(lrow, score_ld, kc, ksc, q, lse2_ws, qk2, b, chunk, T, Tmax, Hq, W, k,
                           chunk_len, n_chunks, bnd, idx, ex, skeys, sh, gsh, flags);
            return;
        }
        if (verdict != 1u || !last) return;
        const unsigned nb_all = __ldcg(bnd_cnt + b);
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
        constexpr int PER = dec::BCAP / kThreads;
        uint64_t kv[PER];
#pragma unroll
        for (int u = 0; u < PER; u++) {
            const int i = threadIdx.x + u * kThreads;
            kv[u] = i < nb ? __ldcg(bnd + (size_t)b * dec::BCAP + i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < PER; u++) {
            const int i = threadIdx.x + u * kThreads;
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
            const int i = threadIdx.x + u * kThreads;
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
            for (int qq = 0; qq < m; qq++) rank += skeys[qq] > key;
            if (rank < need) row[wl + atomicAdd(&sh.n_out, 1u)] = (int32_t)key_pos(key);
        }
    }
    if (!last) return;
    __threadfence();
    for (int i = threadIdx.x; i < wl; i += blockDim.x) row[i] = t - wl + 1 + i;
    for (int i = wl + n_glob + threadIdx.x; i < S; i += blockDim.x) row[i] = -1;
}

}  // namespace dsk
}  // namespace hs2
