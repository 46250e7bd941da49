// Prefill full-attention layer on the 5th-generation tensor cores (tcgen05).
//
// Pass 1 (this file, prefill_fwd_tc_kernel): exact causal attention for one
// block of 128 query rows and TWO heads per CTA.  With one shared KV head
// (MQA, HySparse2 summary "How to use") both heads consume the same K/V tiles,
// so each 128-key tile is fetched once (TMA, 128-byte swizzle) for 2 x 2
// GEMMs.  Warp roles:
//   warp 0        TMA producer (Q once, K/V through a 2-stage ring); TMEM owner
//   warp 1        MMA issuer (one thread): S_h = Q_h K^T into TMEM, then
//                 O_h += P_h V with P_h read from TMEM (it overwrites S_h)
//   warps 4-7     softmax of head 0 (thread = query row = TMEM lane)
//   warps 8-11    softmax of head 1
// TMEM: S0 | S1 | O0 | O1.  The two heads are issued ping-pong so one head's
// softmax overlaps the other head's GEMMs.  The running max is raised lazily
// (only when a tile's max exceeds it by more than 2^8), so O is rescaled in
// TMEM rarely.  Output: O (bf16) and the natural-log lse per (row, head).
#pragma once

#include "tc.cuh"

namespace hs2 {
namespace tcfa {

using namespace hs2::tc;

constexpr int BM = 128;        // query rows per CTA
constexpr int BN = 128;        // keys per tile
constexpr int NSTAGE = 2;      // K/V ring depth
constexpr float kRescaleLog2 = 8.f;

template <int D>
struct Fwd {
    static constexpr int QT = BM * D * 2;   // bytes of one head's Q tile
    static constexpr int KT = BN * D * 2;   // bytes of one K or V tile
    static constexpr int DB = D / 64;       // 64-element (128-byte) column blocks
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = 2 * QT;
    static constexpr int OFF_V = OFF_K + NSTAGE * KT;
    static constexpr int SMEM = OFF_V + NSTAGE * KT + 1024;  // + alignment slack
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
};

struct FwdBars {
    uint64_t q_full;
    uint64_t k_full[NSTAGE], k_empty[NSTAGE], v_full[NSTAGE], v_empty[NSTAGE];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort_;
};

HS2_DEV void setmaxnreg_dec56() { asm volatile("setmaxnreg.dec.sync.aligned.u32 56;"); }
HS2_DEV void setmaxnreg_inc224() { asm volatile("setmaxnreg.inc.sync.aligned.u32 224;"); }

// grid (ceil(L/128), Hq/2, B), 384 threads.  Query blocks run longest first.
template <int D>
__global__ void __launch_bounds__(384, 1)
prefill_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, __nv_bfloat16* __restrict__ o,
                      float* __restrict__ lse, int L, int Hq, float scale2,
                      unsigned* __restrict__ flags) {
    using F = Fwd<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ FwdBars bars;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int nqb = (L + BM - 1) / BM;
    const int qb = nqb - 1 - (int)blockIdx.x;
    const int h0 = 2 * (int)blockIdx.y;
    const int b = blockIdx.z;
    const int n_kt = qb + 1;  // key tiles 0..qb (BN == BM)
    volatile int* abort_ = &bars.abort_;

    if (threadIdx.x == 0) {
        mbar_init(&bars.q_full, 1);
        for (int i = 0; i < NSTAGE; i++) {
            mbar_init(&bars.k_full[i], 1);
            mbar_init(&bars.k_empty[i], 1);
            mbar_init(&bars.v_full[i], 1);
            mbar_init(&bars.v_empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.p_full[i], 4);
            mbar_init(&bars.o_done[i], 1);
        }
        mbar_init(&bars.mma_drain, 1);
        bars.abort_ = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars.tmem_base, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = bars.tmem_base;

    if (warp < 4) {
        setmaxnreg_dec56();
        if (warp == 0 && lane == 0) {
            // ---------------------------------------------------- producer
            tma_prefetch_map(&map_q);
            tma_prefetch_map(&map_k);
            tma_prefetch_map(&map_v);
            mbar_arrive_expect_tx(&bars.q_full, 2 * F::QT);
            for (int hh = 0; hh < 2; hh++)
                for (int db = 0; db < F::DB; db++)
                    tma_load_4d(smem + F::OFF_Q + hh * F::QT + db * (BM * 128), &map_q, 64 * db,
                                h0 + hh, qb * BM, b, &bars.q_full);
            int k_armed = 0, v_armed = 0;  // loads issued so far
            for (int j = 0; j < n_kt && !*abort_; j++) {
                const int st = j % NSTAGE, u = j / NSTAGE;
                if (u > 0 && !mbar_wait(&bars.k_empty[st], (u - 1) & 1, abort_, flags)) break;
                mbar_arrive_expect_tx(&bars.k_full[st], F::KT);
                for (int db = 0; db < F::DB; db++)
                    tma_load_3d(smem + F::OFF_K + st * F::KT + db * (BN * 128), &map_k, 64 * db,
                                j * BN, b, &bars.k_full[st]);
                k_armed++;
                if (u > 0 && !mbar_wait(&bars.v_empty[st], (u - 1) & 1, abort_, flags)) break;
                mbar_arrive_expect_tx(&bars.v_full[st], F::KT);
                for (int db = 0; db < F::DB; db++)
                    tma_load_3d(smem + F::OFF_V + st * F::KT + db * (BN * 128), &map_v, 64 * db,
                                j * BN, b, &bars.v_full[st]);
                v_armed++;
            }
            if (*abort_) {
                // let the copies still in flight land before the CTA leaves
                volatile int no_abort = 0;
                mbar_wait(&bars.q_full, 0, &no_abort, flags);
                for (int j = max(0, k_armed - NSTAGE); j < k_armed; j++)
                    mbar_wait(&bars.k_full[j % NSTAGE], (j / NSTAGE) & 1, &no_abort, flags);
                for (int j = max(0, v_armed - NSTAGE); j < v_armed; j++)
                    mbar_wait(&bars.v_full[j % NSTAGE], (j / NSTAGE) & 1, &no_abort, flags);
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA issuer
            constexpr uint32_t id_qk = idesc_bf16_f32(BM, BN, false, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(BM, D, false, true);
            const uint32_t sq = smem_u32(smem + F::OFF_Q);
            auto issue_qk = [&](int hh, int st) {
                const uint32_t a0 = sq + hh * F::QT;
                const uint32_t b0 = smem_u32(smem + F::OFF_K + st * F::KT);
                const uint32_t dcol = tmem + (hh ? F::COL_S1 : F::COL_S0);
#pragma unroll
                for (int ks = 0; ks < D / 16; ks++) {
                    const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
                    mma_ss(dcol, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024),
                           id_qk, ks > 0);
                }
            };
            auto issue_pv = [&](int hh, int st, bool acc) {
                const uint32_t vb = smem_u32(smem + F::OFF_V + st * F::KT);
                const uint32_t pcol = tmem + (hh ? F::COL_S1 : F::COL_S0);
                const uint32_t dcol = tmem + (hh ? F::COL_O1 : F::COL_O0);
#pragma unroll
                for (int ks = 0; ks < BN / 16; ks++)
                    mma_ts(dcol, pcol + ks * 8, sdesc_sw128(vb + ks * 2048, BN * 128, 1024), id_pv,
                           (acc || ks > 0) ? 1u : 0u);
            };
            bool ok = mbar_wait(&bars.q_full, 0, abort_, flags) &&
                      mbar_wait(&bars.k_full[0], 0, abort_, flags);
            if (ok) {
                fence_after_sync();
                issue_qk(0, 0);
                mma_commit(&bars.s_full[0]);
                issue_qk(1, 0);
                mma_commit(&bars.s_full[1]);
                mma_commit(&bars.k_empty[0]);
            }
            for (int j = 0; ok && j < n_kt; j++) {
                const int st = j % NSTAGE, u = j / NSTAGE;
                const int st1 = (j + 1) % NSTAGE, u1 = (j + 1) / NSTAGE;
                const bool more = j + 1 < n_kt;
                if (!mbar_wait(&bars.v_full[st], u & 1, abort_, flags)) break;
                if (!mbar_wait(&bars.p_full[0], j & 1, abort_, flags)) break;
                fence_after_sync();
                issue_pv(0, st, j > 0);
                mma_commit(&bars.o_done[0]);
                if (more) {
                    if (!mbar_wait(&bars.k_full[st1], u1 & 1, abort_, flags)) break;
                    fence_after_sync();
                    issue_qk(0, st1);
                    mma_commit(&bars.s_full[0]);
                }
                if (!mbar_wait(&bars.p_full[1], j & 1, abort_, flags)) break;
                fence_after_sync();
                issue_pv(1, st, j > 0);
                mma_commit(&bars.o_done[1]);
                mma_commit(&bars.v_empty[st]);
                if (more) {
                    issue_qk(1, st1);
                    mma_commit(&bars.s_full[1]);
                    mma_commit(&bars.k_empty[st1]);
                }
            }
            // every MMA issued must finish before TMEM is released
            mma_commit(&bars.mma_drain);
            volatile int no_abort = 0;
            mbar_wait(&bars.mma_drain, 0, &no_abort, flags);
        }
    } else {
        setmaxnreg_inc224();
        // -------------------------------------------------------- softmax
        const int hh = (warp >> 2) - 1;           // 0 for warps 4-7, 1 for 8-11
        const int row = (warp & 3) * 32 + lane;    // query row in the block = TMEM lane
        const int t = qb * BM + row;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_col = lane_base + (hh ? F::COL_S1 : F::COL_S0);
        const uint32_t o_col = lane_base + (hh ? F::COL_O1 : F::COL_O0);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kt; j++) {
            if (!mbar_wait(&bars.s_full[hh], j & 1, abort_, flags)) {
                ok = false;
                break;
            }
            fence_after_sync();
            float x[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; c++) {
                uint32_t r[32];
                tmem_ld32(s_col + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i++) x[c * 32 + i] = __uint_as_float(r[i]) * scale2;
            }
            if (j == n_kt - 1) {  // diagonal tile: keys j*128 + i, row t = qb*128 + row
#pragma unroll
                for (int i = 0; i < BN; i++)
                    if (i > row) x[i] = -INFINITY;
            }
            float mx = x[0];
#pragma unroll
            for (int i = 1; i < BN; i++) mx = fmaxf(mx, x[i]);
            if (mx > m + kRescaleLog2) {
                if (j > 0) {
                    const float alpha = ex2(m - mx);
                    l *= alpha;
                    // O holds the sum up to tile j-1: wait for that PV, rescale in TMEM
                    if (!mbar_wait(&bars.o_done[hh], (j - 1) & 1, abort_, flags)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
#pragma unroll
                    for (int c = 0; c < D / 32; c++) {
                        uint32_t r[32];
                        tmem_ld32(o_col + c * 32, r);
                        tmem_ld_wait();
                        uint32_t w0[16], w1[16];
#pragma unroll
                        for (int i = 0; i < 16; i++) {
                            w0[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                            w1[i] = __float_as_uint(__uint_as_float(r[16 + i]) * alpha);
                        }
                        tmem_st16(o_col + c * 32, w0);
                        tmem_st16(o_col + c * 32 + 16, w1);
                    }
                }
                m = mx;
            }
            uint32_t pk[BN / 2];
            float rs = 0.f;
#pragma unroll
            for (int i = 0; i < BN / 2; i++) {
                const float p0 = ex2(x[2 * i] - m), p1 = ex2(x[2 * i + 1] - m);
                rs += p0 + p1;
                pk[i] = pack_bf16(p0, p1);
            }
            l += rs;
#pragma unroll
            for (int c = 0; c < BN / 32; c++) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++) w[i] = pk[c * 16 + i];
                tmem_st16(s_col + c * 16, w);
            }
            tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.p_full[hh]);
        }
        // epilogue: O / l and lse
        if (ok && mbar_wait(&bars.o_done[hh], (n_kt - 1) & 1, abort_, flags)) {
            fence_after_sync();
            const int h = h0 + hh;
            const float inv = 1.f / l;
            const bool store = t < L;
            __nv_bfloat16* orow = o + (((size_t)b * L + (store ? t : 0)) * Hq + h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; c++) {
                uint32_t r[32];
                tmem_ld32(o_col + c * 32, r);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; i++)
                    w[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv,
                                     __uint_as_float(r[2 * i + 1]) * inv);
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
            if (store) lse[((size_t)b * L + t) * Hq + h] = (m + __log2f(l)) * kLn2;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tcfa
}  // namespace hs2
