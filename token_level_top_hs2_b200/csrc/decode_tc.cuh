// Decode on the 5th-generation tensor cores (e4m3 cache, d = 128): shared
// pieces of the decode passes and the exact score pass.
//
// The cached TOKENS are the MMA M dimension, so one 128-token tile is one
// tcgen05 MMA: S^T[token][head] = K_tile (128 x 128, f16, in TMEM) *
// Q^T (128 x 16, f16).  e4m3 codes become exact f16 values (converter warps
// write them straight into TMEM, the A operand), so the per-token scales stay
// in fp32: the logit of token s is multiplied by k_scale[s] afterwards.
//
// pass2_tc_kernel: every older token's exact head-summed probability score
// and a per-sequence histogram of the scores; it runs only for the sequences
// the sketch selection could not settle (gate flag).  Warp roles (10 warps):
//   warp 0       TMA producer: e4m3 K tiles and their scales (raw ring)
//   warp 1       MMA issuer (one thread); TMEM owner
//   warps 2-5    converters: thread = token row = TMEM lane; Q -> f16 once
//   warps 6-9    scorers: thread = token = TMEM lane of S^T
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
// TMEM columns of pass 2: S^T buffers, then the two f16 K tiles (A operand
// of QK: lane = token, 64 columns of packed f16 pairs = the 128 dims)
constexpr uint32_t COL_S = 0, COL_K = 64;

// Pass-2 shared-memory plan: 12 raw stages of e4m3 K and its scales, Q, the
// two K scale slots.  Every tile starts on 1024 bytes.
struct Layout {
    static constexpr int NR = 12;
    static constexpr int RAW_K = 0, RAW_SK = TOK * 128;
    static constexpr int RAW = 17408;                     // stage stride, 1024-aligned
    static constexpr int OFF_RAW = 0;
    static constexpr int OFF_QF = OFF_RAW + NR * RAW;
    static constexpr int OFF_SC = OFF_QF + 2 * 16 * 128;  // sk[2][128] floats
    static constexpr int SMEM = OFF_SC + 2 * TOK * 4 + 1024;
    static_assert(RAW >= RAW_SK + TOK * 4 && RAW % 1024 == 0, "raw stage");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct Bars {
    uint64_t raw_full[Layout::NR], raw_empty[Layout::NR];
    uint64_t q_ready, kf_full[2], kf_empty[2], s_full[2], s_empty[2], drain;
    uint32_t tmem_base;
    int abort_;
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

HS2_DEV void issue_raw_k(uint8_t* st, const CUtensorMap* mk, const CUtensorMap* mks, int tok,
                         int b, uint64_t* bar) {
    mbar_arrive_expect_tx(bar, TOK * 128 + TOK * 4);
    tma_load_3d(st + Layout::RAW_K, mk, 0, tok, b, bar);
    tma_load_2d(st + Layout::RAW_SK, mks, tok, b, bar);
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
    using LY = Layout;
    constexpr int NR = LY::NR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ Bars bars;
    __shared__ unsigned hist[256];
    const int b = blockIdx.y, chunk = blockIdx.x;
    // run only for the sequences the sketch selection handed over, if gated;
    // the gate (and lse2) come from the kernels before
    griddep_launch();
    griddep_wait();
    if (gate != nullptr && __ldcg(gate + b) == 0u) return;
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
                issue_raw_k(smem + LY::OFF_RAW + st * LY::RAW, &map_k, &map_ks, s_begin + j * TOK,
                            b, &bars.raw_full[st]);
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
