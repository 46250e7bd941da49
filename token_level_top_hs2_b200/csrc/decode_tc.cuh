// Decode full layer on the 5th-generation tensor cores (e4m3 cache, d = 128).
//
// Same two streaming passes as decode_stream.cuh (exact lse first, scores
// second), but the cached TOKENS are the MMA M dimension, so one 128-token
// tile is one tcgen05 MMA of each kind:
//   S^T[token][head] = K_tile (128 x 128, f16, in TMEM) * Q^T (128 x 16, f16)
//   O^T[dim][head]  += V_tile^T (128 x 128, f16) *  P   (128 tokens x 16, f16)
// e4m3 codes become exact f16 values in shared memory (converter warps), so
// the per-token scales stay in fp32: the logit of token s is multiplied by
// k_scale[s] and its probabilities by v_scale[s] before P is rounded to f16.
// Warp roles (10 warps):
//   warp 0       TMA producer: e4m3 K, V tiles and their scales (raw ring)
//   warp 1       MMA issuer (one thread); TMEM owner
//   warps 2-5    converters: thread = token row = TMEM lane: e4m3 -> f16 K
//                straight into TMEM (the A operand of QK), V into shared
//                memory in the canonical 128-byte-swizzled layout (both double
//                buffered, up to two tiles ahead of the MMAs); Q -> f16 once
//   warps 6-9    softmax: thread = token = TMEM lane of S^T; per-head running
//                max shared by the CTA and raised lazily (a vote over the
//                warpgroup decides when a tile's logit exceeds it by 2^8),
//                per-head partial sums in registers, P written to shared
//                memory (K-major, heads x tokens).
// O^T lives in TMEM (lane = dim); a rare max raise rescales its columns.
#pragma once

#include "decode_stream.cuh"

namespace hs2 {
namespace dtc {

using namespace hs2::tc;

constexpr int TOK = 128;
constexpr int kThreads = 320;
constexpr float kLazy = 8.f;
// Softmax reference offset: probabilities are formed against R = max - kSk,
// so 2^(x - R) lies in (0, 2^14] and its f16 value keeps 3 mantissa bits down
// to 2^-14 before going subnormal (the sketch's 8-bit code range).
constexpr float kSk = 6.f;
constexpr int NRMAX = 12;
// TMEM columns: S^T buffers, O^T, then the two f16 K tiles (A operand of QK:
// lane = token, 64 columns of packed f16 pairs = the 128 dims)
constexpr uint32_t COL_S = 0, COL_O = 32, COL_K = 64;

// Shared-memory plan.  Pass 1 (WITH_V): 4 raw stages of e4m3 K, V and scales
// and double-buffered f16 V tiles.  Pass 2: 12 raw stages of K and its
// scales.  The f16 K tiles live in TMEM.  Every tile starts on 1024 bytes.
template <bool WITH_V>
struct Layout {
    static constexpr int NR = WITH_V ? 4 : 12;
    static constexpr int RAW_K = 0, RAW_V = TOK * 128;
    static constexpr int RAW_SK = (WITH_V ? 2 : 1) * TOK * 128, RAW_SV = RAW_SK + TOK * 4;
    static constexpr int RAW = WITH_V ? 34816 : 17408;   // stage stride, 1024-aligned
    static constexpr int F16T = 2 * TOK * 128;           // f16 tile: 2 blocks x 128 rows x 128 B
    static constexpr int OFF_RAW = 0;
    static constexpr int OFF_VF = OFF_RAW + NR * RAW;    // 2 V tiles (pass 1)
    static constexpr int OFF_QF = OFF_VF + (WITH_V ? 2 * F16T : 0);
    static constexpr int OFF_P = OFF_QF + 2 * 16 * 128;  // 2 P tiles, same shape as Q
    static constexpr int OFF_SC = OFF_P + 2 * 2 * 16 * 128;  // sk[2][128], sv[2][128] floats
    static constexpr int OFF_RED = OFF_SC + 4 * TOK * 4;     // [4][16] floats
    static constexpr int SMEM = OFF_RED + 4 * 16 * 4 + 1024;
    static_assert(RAW >= (WITH_V ? RAW_SV : RAW_SK) + TOK * 4 && RAW % 1024 == 0, "raw stage");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct Bars {
    uint64_t raw_full[NRMAX], raw_empty[NRMAX];
    uint64_t q_ready, kf_full[2], kf_empty[2], vf_full[2], vf_empty[2];
    uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2], o_done, drain;
    uint32_t tmem_base;
    int abort_;
    unsigned last;
};

// f16 x f16 -> f32 instruction descriptor
constexpr uint32_t idesc_f16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

HS2_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

HS2_DEV bool bar_red_or(bool v, int id, int count) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
HS2_DEV void bar_named(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// byte offset of f16 element e of row r in a [2 blocks][rows][128 B] swizzled tile
HS2_DEV uint32_t f16_off(int rows, int r, int e) {
    return (uint32_t)((e >> 6) * (rows * 128) + r * 128 + ((((e & 63) >> 3) ^ (r & 7)) << 4) +
                      (e & 7) * 2);
}

// Convert one 128-byte e4m3 row (raw, swizzled) into f16 row r of a
// [2][128][128 B] swizzled tile; zeros when !valid.
HS2_DEV void convert_row(const uint8_t* raw, uint8_t* f16t, int r, bool valid) {
#pragma unroll
    for (int c = 0; c < 8; c++) {
        uint4 x = *reinterpret_cast<const uint4*>(raw + r * 128 + ((c ^ (r & 7)) << 4));
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            h[2 * i] = valid ? e4m3x2_lo_to_f16x2(w[i]) : 0u;
            h[2 * i + 1] = valid ? e4m3x2_lo_to_f16x2(w[i] >> 16) : 0u;
        }
        // elements 16c..16c+15: block c>>2, 16-byte chunks 2(c&3), 2(c&3)+1
        uint8_t* dst = f16t + (c >> 2) * (TOK * 128) + r * 128;
        *reinterpret_cast<uint4*>(dst + (((2 * (c & 3)) ^ (r & 7)) << 4)) =
            make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(dst + (((2 * (c & 3) + 1) ^ (r & 7)) << 4)) =
            make_uint4(h[4], h[5], h[6], h[7]);
    }
}

// Convert one 128-byte e4m3 row (raw, swizzled) of token row r into 64
// packed f16 pairs stored along TMEM lane r (this warp's lane quarter) from
// column address `taddr` on; zeros when !valid.  Column c holds dims 2c, 2c+1.
HS2_DEV void convert_row_tmem(const uint8_t* raw, int r, bool valid, uint32_t taddr) {
#pragma unroll
    for (int half = 0; half < 4; half++) {
        uint32_t h[16];
#pragma unroll
        for (int cc = 0; cc < 2; cc++) {
            const int c = 2 * half + cc;
            const uint4 x = *reinterpret_cast<const uint4*>(raw + r * 128 + ((c ^ (r & 7)) << 4));
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                h[8 * cc + 2 * i] = valid ? e4m3x2_lo_to_f16x2(w[i]) : 0u;
                h[8 * cc + 2 * i + 1] = valid ? e4m3x2_lo_to_f16x2(w[i] >> 16) : 0u;
            }
        }
        tmem_st16(taddr + 16 * half, h);
    }
}

// Q [Hq][128] bf16 -> f16 [2][16][128 B] swizzled (rows >= Hq zero).  128
// threads: thread t converts head t/8, elements 16*(t%8) .. +15.
HS2_DEV bool convert_q(const __nv_bfloat16* q, int Hq, uint8_t* qf, int t) {
    const int h = t >> 3, e0 = 16 * (t & 7);
    uint32_t w[8];
    bool ok = true;
    if (h < Hq) {
        const uint4* p = reinterpret_cast<const uint4*>(q + h * 128 + e0);
        const uint4 a = ldg_nc(p), b = ldg_nc(p + 1);
        const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float lo = bf16_lo(in[i]), hi = bf16_hi(in[i]);
            ok &= fabsf(lo) <= 65504.f && fabsf(hi) <= 65504.f;
            w[i] = pack_f16(lo, hi);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) w[i] = 0;
    }
    *reinterpret_cast<uint4*>(qf + f16_off(16, h, e0)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(qf + f16_off(16, h, e0 + 8)) = make_uint4(w[4], w[5], w[6], w[7]);
    return ok;
}

template <bool WITH_V>
HS2_DEV void issue_raw(uint8_t* st, const CUtensorMap* mk, const CUtensorMap* mv,
                       const CUtensorMap* mks, const CUtensorMap* mvs, int tok, int b,
                       uint64_t* bar) {
    using LY = Layout<WITH_V>;
    mbar_arrive_expect_tx(bar, WITH_V ? 2 * (TOK * 128 + TOK * 4) : TOK * 128 + TOK * 4);
    tma_load_3d(st + LY::RAW_K, mk, 0, tok, b, bar);
    tma_load_2d(st + LY::RAW_SK, mks, tok, b, bar);
    if constexpr (WITH_V) {
        tma_load_3d(st + LY::RAW_V, mv, 0, tok, b, bar);
        tma_load_2d(st + LY::RAW_SV, mvs, tok, b, bar);
    }
}

// ----------------------------------------------------------------------------
// Pass 1: exact lse and O for one chunk of one sequence; the last chunk of the
// sequence to finish merges the partials.  grid (n_chunks, B), 320 threads.
__global__ void __launch_bounds__(kThreads, 1)
pass1_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                const __grid_constant__ CUtensorMap map_ks,
                const __grid_constant__ CUtensorMap map_vs, const __nv_bfloat16* __restrict__ q,
                const int32_t* __restrict__ lengths, int Tmax, int Hq, int chunk_len,
                int n_chunks, float qk_scale, float* __restrict__ part,
                unsigned* __restrict__ counter, float* __restrict__ lse2_ws,
                float* __restrict__ lse_out, __nv_bfloat16* __restrict__ out,
                uint8_t* __restrict__ sketch, float* __restrict__ rsnap, int sk_tiles,
                unsigned* __restrict__ flags) {
    constexpr int D = 128;
    constexpr int PART = 16 * D + 32;
    using LY = Layout<true>;
    constexpr int NR = LY::NR;
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
    const int n = s_end > s_begin ? (s_end - s_begin + TOK - 1) / TOK : 0;
    volatile int* abort_ = &bars.abort_;
    float* skb = reinterpret_cast<float*>(smem + LY::OFF_SC);  // [2][128]
    float* svb = skb + 2 * TOK;                                // [2][128]
    float* red = reinterpret_cast<float*>(smem + LY::OFF_RED); // [4][16]

    if (threadIdx.x == 0) {
        for (int i = 0; i < NR; i++) {
            mbar_init(&bars.raw_full[i], 1);
            mbar_init(&bars.raw_empty[i], 4);
        }
        mbar_init(&bars.q_ready, 4);
        for (int i = 0; i < 2; i++) {
            mbar_init(&bars.kf_full[i], 4);
            mbar_init(&bars.kf_empty[i], 1);
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.s_empty[i], 4);
            mbar_init(&bars.p_full[i], 4);
            mbar_init(&bars.p_empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&bars.vf_full[i], 4);
            mbar_init(&bars.vf_empty[i], 1);
        }
        mbar_init(&bars.o_done, 1);
        mbar_init(&bars.drain, 1);
        bars.abort_ = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars.tmem_base, 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = bars.tmem_base;

    if (warp == 0) {
        if (lane == 0 && n > 0) {
            // ------------------------------------------------------ producer
            int armed = 0;
            for (int j = 0; j < n && !*abort_; j++) {
                const int st = j % NR, u = j / NR;
                if (u > 0 && !mbar_wait(&bars.raw_empty[st], (u - 1) & 1, abort_, flags)) break;
                issue_raw<true>(smem + LY::OFF_RAW + st * LY::RAW, &map_k, &map_v, &map_ks,
                                &map_vs, s_begin + j * TOK, b, &bars.raw_full[st]);
                armed++;
            }
            if (*abort_) {
                volatile int no_abort = 0;
                for (int j = max(0, armed - NR); j < armed; j++)
                    mbar_wait(&bars.raw_full[j % NR], (j / NR) & 1, &no_abort, flags);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && n > 0) {
            // ---------------------------------------------------------- MMA
            constexpr uint32_t id_qk = idesc_f16(128, 16, false, false);
            constexpr uint32_t id_pv = idesc_f16(128, 16, true, false);
            const uint32_t vf = smem_u32(smem + LY::OFF_VF);
            const uint32_t qf = smem_u32(smem + LY::OFF_QF), pf = smem_u32(smem + LY::OFF_P);
            auto qk = [&](int j) {
                const int buf = j & 1;
#pragma unroll
                for (int ks = 0; ks < 8; ks++) {
                    const uint32_t kb = qf + (ks >> 2) * (16 * 128) + (ks & 3) * 32;
                    mma_ts(tmem + COL_S + buf * 16, tmem + COL_K + buf * 64 + ks * 8,
                           sdesc_sw128(kb, 16, 1024), id_qk, ks > 0);
                }
                mma_commit(&bars.s_full[buf]);
                mma_commit(&bars.kf_empty[buf]);
            };
            bool ok = mbar_wait(&bars.q_ready, 0, abort_, flags) &&
                      mbar_wait(&bars.kf_full[0], 0, abort_, flags);
            if (ok) {
                fence_after_sync();
                qk(0);
            }
            for (int j = 0; ok && j < n; j++) {
                if (j + 1 < n) {
                    const int b1 = (j + 1) & 1, u1 = (j + 1) >> 1;
                    if (!mbar_wait(&bars.kf_full[b1], u1 & 1, abort_, flags)) break;
                    if (u1 > 0 && !mbar_wait(&bars.s_empty[b1], (u1 - 1) & 1, abort_, flags))
                        break;
                    fence_after_sync();
                    qk(j + 1);
                }
                const int buf = j & 1, u = j >> 1;
                if (!mbar_wait(&bars.p_full[buf], u & 1, abort_, flags)) break;
                if (!mbar_wait(&bars.vf_full[buf], u & 1, abort_, flags)) break;
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ks++) {
                    const uint32_t va = vf + buf * LY::F16T + ks * (16 * 128);
                    const uint32_t pb = pf + buf * (2 * 16 * 128) + (ks >> 2) * (16 * 128) +
                                        (ks & 3) * 32;
                    mma_ss(tmem + COL_O, sdesc_sw128(va, TOK * 128, 1024),
                           sdesc_sw128(pb, 16, 1024), id_pv, (j > 0 || ks > 0) ? 1u : 0u);
                }
                mma_commit(&bars.o_done);
                mma_commit(&bars.vf_empty[buf]);
                mma_commit(&bars.p_empty[buf]);
            }
            mma_commit(&bars.drain);
            volatile int no_abort = 0;
            mbar_wait(&bars.drain, 0, &no_abort, flags);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------- converters
        const int t = (warp & 3) * 32 + lane;  // token row = TMEM lane of this warp
        const uint32_t k_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16) + COL_K;
        const bool qok = convert_q(q + (size_t)b * Hq * D, Hq, smem + LY::OFF_QF, t);
        if (!__all_sync(0xffffffffu, qok) && lane == 0 && chunk == 0) atomicOr(flags, FLAG_Q_RANGE);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_ready);
        bool bad_scale = false;
        for (int j = 0; j < n; j++) {
            const int st = j % NR, buf = j & 1, u = j >> 1;
            if (!mbar_wait(&bars.raw_full[st], (j / NR) & 1, abort_, flags)) break;
            // buffer `buf` last held tile j-2: its K and V tiles must be consumed
            // by the MMAs and its scales read by the softmax warps (they read
            // them before releasing S(j-2))
            if (u > 0 && (!mbar_wait(&bars.kf_empty[buf], (u - 1) & 1, abort_, flags) ||
                          !mbar_wait(&bars.s_empty[buf], (u - 1) & 1, abort_, flags) ||
                          !mbar_wait(&bars.vf_empty[buf], (u - 1) & 1, abort_, flags)))
                break;
            const uint8_t* raw = smem + LY::OFF_RAW + st * LY::RAW;
            const bool valid = s_begin + j * TOK + t < s_end;
            fence_after_sync();
            convert_row_tmem(raw + LY::RAW_K, t, valid, k_lane + buf * 64);
            const float sk = reinterpret_cast<const float*>(raw + LY::RAW_SK)[t];
            const float sv = reinterpret_cast<const float*>(raw + LY::RAW_SV)[t];
            skb[buf * TOK + t] = valid ? sk : 0.f;
            svb[buf * TOK + t] = valid ? sv : 0.f;
            bad_scale |= valid && !(sv <= 255.f);
            tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.kf_full[buf]);
            convert_row(raw + LY::RAW_V, smem + LY::OFF_VF + buf * LY::F16T, t, valid);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.vf_full[buf]);
                mbar_arrive(&bars.raw_empty[st]);
            }
        }
        if (__any_sync(0xffffffffu, bad_scale) && lane == 0) atomicOr(flags, FLAG_SCALE_RANGE);
    } else {
        // ----------------------------------------------------------- softmax
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const int t = wq * 32 + lane;            // token row = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        uint8_t* pf = smem + LY::OFF_P;
        // R = running max - kSk: probabilities are formed as 2^(x - R), in
        // (0, 2^(kLazy + kSk)], which is the range the sketch codes cover
        float R[16], l[16];
#pragma unroll
        for (int h = 0; h < 16; h++) {
            R[h] = -INFINITY;
            l[h] = 0.f;
        }
        bool ok = true;
        for (int j = 0; j < n; j++) {
            const int buf = j & 1, u = j >> 1;
            if (!mbar_wait(&bars.s_full[buf], u & 1, abort_, flags)) {
                ok = false;
                break;
            }
            fence_after_sync();
            uint32_t r[16];
            tmem_ld16(lane_addr + COL_S + buf * 16, r);
            tmem_ld_wait();
            const float ks = skb[buf * TOK + t] * qk_scale;
            const float sv = svb[buf * TOK + t] * (1.f / 64.f);
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.s_empty[buf]);
            const bool valid = s_begin + j * TOK + t < s_end;
            float x[16];
            bool over = false;
#pragma unroll
            for (int h = 0; h < 16; h++) {
                x[h] = valid ? __uint_as_float(r[h]) * ks : -INFINITY;
                over |= x[h] > R[h] + (kLazy + kSk);
            }
            if (bar_red_or(over, 1, 128)) {
                // raise the per-head running max to this tile's max
                float mx[16];
#pragma unroll
                for (int h = 0; h < 16; h++) {
                    float v = x[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    mx[h] = v;
                }
                if (lane < 16) {
                    float v = mx[0];
#pragma unroll
                    for (int h = 1; h < 16; h++)
                        if (lane == h) v = mx[h];
                    red[wq * 16 + lane] = v;
                }
                bar_named(2, 128);
                float alpha[16];
                bool any_scale = false;
#pragma unroll
                for (int h = 0; h < 16; h++) {
                    const float tm = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
                    const float nm = fmaxf(R[h], tm - kSk);
                    alpha[h] = (R[h] == -INFINITY || nm == R[h]) ? 1.f : ex2(R[h] - nm);
                    any_scale |= alpha[h] != 1.f;
                    R[h] = nm;
                    l[h] *= alpha[h];
                }
                bar_named(2, 128);  // red[] is read by everyone before it is reused
                if (j > 0 && any_scale) {
                    // O^T holds tiles 0..j-1: wait for that PV, scale its columns
                    if (!mbar_wait(&bars.o_done, (j - 1) & 1, abort_, flags)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    uint32_t o[16];
                    tmem_ld16(lane_addr + COL_O, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 16; h++) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                    tmem_st16(lane_addr + COL_O, o);
                    tmem_st_wait();
                    fence_before_sync();
                }
            }
            uint32_t pw[16];
            float pr[16];
#pragma unroll
            for (int h = 0; h < 16; h++) {
                pr[h] = (valid && R[h] != -INFINITY) ? ex2(x[h] - R[h]) : 0.f;
                l[h] += pr[h];
                pw[h] = __half_as_ushort(__float2half_rn(pr[h] * sv));
            }
            if (sketch != nullptr) {
                const int tok = s_begin + j * TOK + t;
                if (valid) {
                    uint32_t hw[8];
#pragma unroll
                    for (int i = 0; i < 8; i++) hw[i] = f16x2_rz(pr[2 * i], pr[2 * i + 1]);
                    uint4 cw;
                    cw.x = prmt(hw[0] >> 7, hw[1] >> 7, 0x6420u);
                    cw.y = prmt(hw[2] >> 7, hw[3] >> 7, 0x6420u);
                    cw.z = prmt(hw[4] >> 7, hw[5] >> 7, 0x6420u);
                    cw.w = prmt(hw[6] >> 7, hw[7] >> 7, 0x6420u);
                    *reinterpret_cast<uint4*>(sketch + ((size_t)b * Tmax + tok) * 16) = cw;
                }
                if (wq == 0 && lane < 16) {
                    float rv = R[0];
#pragma unroll
                    for (int h = 1; h < 16; h++)
                        if (lane == h) rv = R[h];
                    rsnap[((size_t)b * sk_tiles + (s_begin / TOK + j)) * 16 + lane] = rv;
                }
            }
            if (u > 0 && !mbar_wait(&bars.p_empty[buf], (u - 1) & 1, abort_, flags)) {
                ok = false;
                break;
            }
            uint8_t* pt = pf + buf * (2 * 16 * 128);
#pragma unroll
            for (int h = 0; h < 16; h++)
                *reinterpret_cast<uint16_t*>(pt + f16_off(16, h, t)) = (uint16_t)pw[h];
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.p_full[buf]);
        }
        // chunk partial: l summed over the tile rows, O^T from TMEM (lane = dim)
#pragma unroll
        for (int h = 0; h < 16; h++) {
            float v = l[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            l[h] = v;
        }
        if (lane < 16) {
            float v = l[0];
#pragma unroll
            for (int h = 1; h < 16; h++)
                if (lane == h) v = l[h];
            red[wq * 16 + lane] = v;
        }
        bar_named(2, 128);
        float* dst = part + ((size_t)b * n_chunks + chunk) * PART;
        if (t < 16) {
            float mt = R[0];
#pragma unroll
            for (int h = 1; h < 16; h++)
                if (t == h) mt = R[h];
            // O is relative to R + kSk (the P tiles carry sv / 64), so is the sum
            dst[16 * D + t] = mt + kSk;
            dst[16 * D + 16 + t] =
                (red[t] + red[16 + t] + red[32 + t] + red[48 + t]) * (1.f / 64.f);
        }
        if (ok && n > 0 && mbar_wait(&bars.o_done, (n - 1) & 1, abort_, flags)) {
            fence_after_sync();
            uint32_t o[16];
            tmem_ld16(lane_addr + COL_O, o);
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < 16; h++) dst[h * D + t] = __uint_as_float(o[h]);
        } else {
#pragma unroll
            for (int h = 0; h < 16; h++) dst[h * D + t] = 0.f;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tmem_dealloc(tmem, 256);
    }
    // ---- the last chunk of the sequence merges every chunk's partial
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
        out[(size_t)b * Hq * D + e] = __float2bfloat16_rn(ls > 0.f ? acc / ls : 0.f);
        if (e % D == 0) {
            const float l2 = ls > 0.f ? mu + __log2f(ls) : -INFINITY;
            lse2_ws[b * 16 + row] = l2;
            if (lse_out) lse_out[b * Hq + row] = l2 * kLn2;
        }
    }
}

// ----------------------------------------------------------------------------
// Pass 2: the candidates' exact scores and the per-sequence histogram (the
// fallback of the sketch selection, for sequences flagged in `gate`).
__global__ void __launch_bounds__(kThreads, 1)
pass2_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_ks,
                const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lengths, int Tmax,
                int Hq, int W, int chunk_len, float qk_scale, const float* __restrict__ lse2_ws,
                float* __restrict__ scores, int score_ld, unsigned* __restrict__ hist_g,
                const unsigned* __restrict__ gate, unsigned* __restrict__ flags) {
    constexpr int D = 128;
    using LY = Layout<false>;
    constexpr int NR = LY::NR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ Bars bars;
    __shared__ unsigned hist[256];
    const int b = blockIdx.y, chunk = blockIdx.x;
    // run only for the sequences the sketch selection handed over, if gated
    if (gate != nullptr && __ldg(gate + b) == 0u) return;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int T = __ldg(lengths + b);
    const int n_cand = (T >= 1 && T <= Tmax) ? max(0, T - W) : 0;
    const int s_begin = chunk * chunk_len;
    const int s_end = min(s_begin + chunk_len, n_cand);
    const int n = s_end > s_begin ? (s_end - s_begin + TOK - 1) / TOK : 0;
    if (n == 0) return;
    volatile int* abort_ = &bars.abort_;
    float* skb = reinterpret_cast<float*>(smem + LY::OFF_SC);
    const uint32_t base = dec::seq_base(Hq, T);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NR; i++) {
            mbar_init(&bars.raw_full[i], 1);
            mbar_init(&bars.raw_empty[i], 4);
        }
        mbar_init(&bars.q_ready, 4);
        for (int i = 0; i < 2; i++) {
            mbar_init(&bars.kf_full[i], 4);
            mbar_init(&bars.kf_empty[i], 1);
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.s_empty[i], 4);
        }
        mbar_init(&bars.drain, 1);
        bars.abort_ = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars.tmem_base, 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = bars.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            int armed = 0;
            for (int j = 0; j < n && !*abort_; j++) {
                const int st = j % NR, u = j / NR;
                if (u > 0 && !mbar_wait(&bars.raw_empty[st], (u - 1) & 1, abort_, flags)) break;
                issue_raw<false>(smem + LY::OFF_RAW + st * LY::RAW, &map_k, nullptr, &map_ks,
                                 nullptr, s_begin + j * TOK, b, &bars.raw_full[st]);
                armed++;
            }
            if (*abort_) {
                volatile int no_abort = 0;
                for (int j = max(0, armed - NR); j < armed; j++)
                    mbar_wait(&bars.raw_full[j % NR], (j / NR) & 1, &no_abort, flags);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_f16(128, 16, false, false);
            const uint32_t qf = smem_u32(smem + LY::OFF_QF);
            bool ok = mbar_wait(&bars.q_ready, 0, abort_, flags);
            for (int j = 0; ok && j < n; j++) {
                const int buf = j & 1, u = j >> 1;
                if (!mbar_wait(&bars.kf_full[buf], u & 1, abort_, flags)) break;
                if (u > 0 && !mbar_wait(&bars.s_empty[buf], (u - 1) & 1, abort_, flags)) break;
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ks++) {
                    const uint32_t kb = qf + (ks >> 2) * (16 * 128) + (ks & 3) * 32;
                    mma_ts(tmem + COL_S + buf * 16, tmem + COL_K + buf * 64 + ks * 8,
                           sdesc_sw128(kb, 16, 1024), id_qk, ks > 0);
                }
                mma_commit(&bars.s_full[buf]);
                mma_commit(&bars.kf_empty[buf]);
            }
            mma_commit(&bars.drain);
            volatile int no_abort = 0;
            mbar_wait(&bars.drain, 0, &no_abort, flags);
        }
    } else if (warp < 6) {
        const int t = (warp & 3) * 32 + lane;
        const uint32_t k_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16) + COL_K;
        convert_q(q + (size_t)b * Hq * D, Hq, smem + LY::OFF_QF, t);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_ready);
        for (int j = 0; j < n; j++) {
            const int st = j % NR, buf = j & 1, u = j >> 1;
            if (!mbar_wait(&bars.raw_full[st], (j / NR) & 1, abort_, flags)) break;
            if (u > 0 && (!mbar_wait(&bars.kf_empty[buf], (u - 1) & 1, abort_, flags) ||
                          !mbar_wait(&bars.s_empty[buf], (u - 1) & 1, abort_, flags)))
                break;
            const uint8_t* raw = smem + LY::OFF_RAW + st * LY::RAW;
            const bool valid = s_begin + j * TOK + t < s_end;
            fence_after_sync();
            convert_row_tmem(raw + LY::RAW_K, t, valid, k_lane + buf * 64);
            skb[buf * TOK + t] = valid ? reinterpret_cast<const float*>(raw + LY::RAW_SK)[t] : 0.f;
            tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.kf_full[buf]);
                mbar_arrive(&bars.raw_empty[st]);
            }
        }
    } else {
        const int wq = warp & 3;
        const int t = wq * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        float l2[16];
#pragma unroll
        for (int h = 0; h < 16; h++) l2[h] = h < Hq ? __ldcg(lse2_ws + b * 16 + h) : INFINITY;
        float* srow = scores + (size_t)b * score_ld;
        for (int j = 0; j < n; j++) {
            const int buf = j & 1, u = j >> 1;
            if (!mbar_wait(&bars.s_full[buf], u & 1, abort_, flags)) break;
            fence_after_sync();
            uint32_t r[16];
            tmem_ld16(lane_addr + COL_S + buf * 16, r);
            tmem_ld_wait();
            const float ks = skb[buf * TOK + t] * qk_scale;
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.s_empty[buf]);
            const int tok = s_begin + j * TOK + t;
            const bool valid = tok < s_end;
            float sc = 0.f;
#pragma unroll
            for (int h = 0; h < 16; h++) sc += ex2(fmaf(__uint_as_float(r[h]), ks, -l2[h]));
            const int bn = valid ? dec::score_bin(__float_as_uint(sc), base) : -1;
            if (valid) srow[tok] = sc;
            const unsigned grp = __match_any_sync(0xffffffffu, bn);
            if (valid && lane == __ffs(grp) - 1) atomicAdd(&hist[bn], (unsigned)__popc(grp));
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tmem_dealloc(tmem, 256);
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (hist[i]) atomicAdd(hist_g + b * 256 + i, hist[i]);
}

}  // namespace dtc
}  // namespace hs2
