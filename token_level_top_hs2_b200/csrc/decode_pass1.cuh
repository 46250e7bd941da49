// Decode pass 1 on the tensor cores (FP8 e4m3 cache, d = 128): exact lse and
// O of one query per sequence over a chunk of its cache, plus the per-token
// selection sketch (decode_sketch.cuh).
//
// HySparse2 summary (onedev.kr/papers/146), 'How it works': the full layer is
// exact attention; each cached row is dequantised as s_x * e4m3(x) with its
// per-token scale.  The e4m3 -> f16 conversion is exact, and the scales are
// folded in afterwards (logit * sK, p * sV), so the MMAs see exact operands.
//
// Per 128-token tile, with the tokens as the MMA M dimension:
//   S^T[token][head] = K_tile (128 x 128, f16, TMEM) * Q^T (128 x 16, f16)
//   O^T[dim][head]  += V_tile^T (128 x 128, f16, TMEM) * P (128 x 16, f16)
// Roles (19 warps):
//   warp 0       TMA producer: raw e4m3 K, V tiles and both scale rows into a
//                ring of kNR stages;
//   warp 1       QK issuer (one thread); TMEM owner;
//   warp 2       PV issuer (one thread): a single thread issues one tcgen05.mma
//                per ~130 cycles whatever its N, so the 16 N=16 MMAs of a tile
//                are spread over two issuers;
//   warps 3-6    K converters: thread = token row = TMEM lane; e4m3 -> f16
//                straight into one of kDK TMEM K buffers; copy both scales;
//   warps 7-14   softmax, two groups of 4 warps owning heads 0-7 and 8-15:
//                thread = token = TMEM lane of S^T; per group, lazily raised
//                running maxima shared by its 128 threads; P (f16, K-major)
//                into one of kDP shared buffers; the per-token sketch bytes;
//   warps 15-18  V converters: e4m3 -> f16 V^T straight into one of kDV TMEM
//                tiles (lane = dim), the A operand of PV, through transposing
//                16 x 16 byte shared-memory loads.
// K and V conversion run in separate warps so that the QK/softmax chain of
// later tiles proceeds while an older tile's PV is still pending.
#pragma once

#include "decode_tc.cuh"

namespace hs2 {
namespace dtc {

// warp roles
constexpr int kWProd = 0, kWQK = 1, kWPV = 2;
constexpr int kWK0 = 3;                 // 4 K-converter warps: lane quarters 3, 0, 1, 2
constexpr int kWS0 = kWK0 + 4;          // 2 x 4 softmax warps (heads 0-7, 8-15)
constexpr int kWV0 = kWS0 + 8;          // V-converter warps
constexpr int kVW = 4;                  // V-converter warps, one per TMEM lane quarter
constexpr int kP1Threads = 32 * (kWV0 + kVW);
constexpr int kNR = 5;  // raw stages
constexpr int kDK = 4;  // K tiles in TMEM = S^T buffers = scale slots
constexpr int kDV = 2;  // f16 V^T tiles in TMEM
constexpr int kDP = 4;  // P tiles in shared memory
// TMEM columns (512 allocated, one CTA per SM): S^T buffers, O^T, K tiles
// TMEM columns: S^T buffers, O^T, K tiles (lane = token), V^T tiles (lane = dim)
constexpr uint32_t P1_COL_S = 0, P1_COL_O = 16 * kDK, P1_COL_K = 128,
                   P1_COL_V = P1_COL_K + 64 * kDK;
static_assert(P1_COL_O + 16 <= P1_COL_K && P1_COL_V + 64 * kDV <= 512, "TMEM plan");

struct P1Layout {
    static constexpr int RAW_K = 0, RAW_V = TOK * 128;
    static constexpr int RAW_SK = 2 * TOK * 128, RAW_SV = RAW_SK + TOK * 4;
    static constexpr int RAW = 34816;                      // stage stride, 1024-aligned
    static constexpr int PT = 2 * 16 * 128;                // P tile: 2 blocks of 16 x 128 B
    static constexpr int OFF_RAW = 0;
    static constexpr int OFF_QF = OFF_RAW + kNR * RAW;
    static constexpr int OFF_P = OFF_QF + PT;
    static constexpr int OFF_SC = OFF_P + kDP * PT;        // sk[kDK][128], sv[kDK][128]
    static constexpr int OFF_RED = OFF_SC + 2 * kDK * TOK * 4;  // [2][4][8] floats
    static constexpr int SMEM = OFF_RED + 4 * 16 * 4 + 1024;
    static_assert(RAW >= RAW_SV + TOK * 4 && RAW % 1024 == 0, "raw stage");
    static_assert(OFF_QF % 1024 == 0 && OFF_P % 1024 == 0, "alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct P1Bars {
    uint64_t raw_full[kNR], raw_empty[kNR];
    uint64_t q_ready, kf_full[kDK], kf_empty[kDK], s_full[kDK], s_empty[kDK];
    uint64_t vf_full[kDV], vf_empty[kDV], p_full[kDP], p_empty[kDP], drain_qk, drain_pv;
    uint32_t tmem_base;
    int abort_;
    unsigned last;
};

HS2_DEV void p1_issue_raw(uint8_t* st, const CUtensorMap* mk, const CUtensorMap* mv,
                          const CUtensorMap* mks, const CUtensorMap* mvs, int tok, int b,
                          uint64_t* bar, uint64_t policy) {
    mbar_arrive_expect_tx(bar, 2 * (TOK * 128 + TOK * 4));
    tma_load_3d_hint(st + P1Layout::RAW_K, mk, 0, tok, b, bar, policy);
    tma_load_3d_hint(st + P1Layout::RAW_V, mv, 0, tok, b, bar, policy);
    tma_load_2d_hint(st + P1Layout::RAW_SK, mks, tok, b, bar, policy);
    tma_load_2d_hint(st + P1Layout::RAW_SV, mvs, tok, b, bar, policy);
}

// grid (n_chunks, B), kP1Threads threads; the last chunk of a sequence to finish
// merges every chunk's partial into O and lse.
__global__ void __launch_bounds__(kP1Threads, 1)
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
    using LY = P1Layout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ P1Bars bars;
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int T = __ldg(lengths + b);
    const bool len_ok = T >= 1 && T <= Tmax;
    if (!len_ok && threadIdx.x == 0 && chunk == 0) atomicOr(flags, FLAG_BAD_LENGTH);
    const int s_begin = chunk * chunk_len;
    const int s_end = len_ok ? min(s_begin + chunk_len, T) : s_begin;
    const int n = s_end > s_begin ? (s_end - s_begin + TOK - 1) / TOK : 0;
    volatile int* abort_ = &bars.abort_;
    float* skb = reinterpret_cast<float*>(smem + LY::OFF_SC);  // [kDK][128]
    float* svb = skb + kDK * TOK;                              // [kDK][128]
    float* red = reinterpret_cast<float*>(smem + LY::OFF_RED); // [4][16]
    // the selection kernel that follows may launch now; it waits for this
    // grid to complete before reading what it writes
    griddep_launch();

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNR; i++) {
            mbar_init(&bars.raw_full[i], 1);
            mbar_init(&bars.raw_empty[i], 4 + kVW);  // K- and V-converter warps
        }
        mbar_init(&bars.q_ready, 4);
        for (int i = 0; i < kDK; i++) {
            mbar_init(&bars.kf_full[i], 4);
            mbar_init(&bars.kf_empty[i], 1);
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.s_empty[i], 8);
        }
        for (int i = 0; i < kDV; i++) {
            mbar_init(&bars.vf_full[i], kVW);
            mbar_init(&bars.vf_empty[i], 1);
        }
        for (int i = 0; i < kDP; i++) {
            mbar_init(&bars.p_full[i], 8);
            mbar_init(&bars.p_empty[i], 1);
        }
        mbar_init(&bars.drain_qk, 1);
        mbar_init(&bars.drain_pv, 1);
        bars.abort_ = 0;
        fence_mbar_init();
    }
    if (warp == kWQK) {
        tmem_alloc(&bars.tmem_base, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = bars.tmem_base;

    if (warp == kWProd) {
        if (lane == 0 && n > 0) {
            // ------------------------------------------------------ producer
            // the cache is read once: its lines leave L2 first, so that the
            // sketch written meanwhile stays there for the selection
            const uint64_t pol = l2_evict_first();
            int armed = 0;
            for (int j = 0; j < n && !*abort_; j++) {
                const int st = j % kNR, u = j / kNR;
                if (u > 0 && !mbar_wait(&bars.raw_empty[st], (u - 1) & 1, abort_, flags)) break;
                p1_issue_raw(smem + LY::OFF_RAW + st * LY::RAW, &map_k, &map_v, &map_ks, &map_vs,
                             s_begin + j * TOK, b, &bars.raw_full[st], pol);
                armed++;
            }
            if (*abort_) {
                volatile int no_abort = 0;
                for (int j = max(0, armed - kNR); j < armed; j++)
                    mbar_wait(&bars.raw_full[j % kNR], (j / kNR) & 1, &no_abort, flags);
            }
        }
    } else if (warp == kWQK) {
        if (lane == 0 && n > 0) {
            // -------------------------------------------------- QK issuer
            constexpr uint32_t id_qk = idesc_f16(128, 16, false, false);
            const uint32_t qf = smem_u32(smem + LY::OFF_QF);
            bool ok = mbar_wait(&bars.q_ready, 0, abort_, flags);
            for (int j = 0; ok && j < n; j++) {
                const int kb = j % kDK, ku = j / kDK;
                if (!mbar_wait(&bars.kf_full[kb], ku & 1, abort_, flags)) break;
                if (ku > 0 && !mbar_wait(&bars.s_empty[kb], (ku - 1) & 1, abort_, flags)) break;
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ks++) {
                    const uint32_t kbq = qf + (ks >> 2) * (16 * 128) + (ks & 3) * 32;
                    mma_ts(tmem + P1_COL_S + kb * 16, tmem + P1_COL_K + kb * 64 + ks * 8,
                           sdesc_sw128(kbq, 16, 1024), id_qk, ks > 0);
                }
                mma_commit(&bars.s_full[kb]);
                mma_commit(&bars.kf_empty[kb]);
            }
            mma_commit(&bars.drain_qk);
            volatile int no_abort = 0;
            mbar_wait(&bars.drain_qk, 0, &no_abort, flags);
        }
    } else if (warp == kWPV) {
        if (lane == 0 && n > 0) {
            // -------------------------------------------------- PV issuer
            constexpr uint32_t id_pv = idesc_f16(128, 16, false, false);
            const uint32_t pf = smem_u32(smem + LY::OFF_P);
            for (int j = 0; j < n; j++) {
                const int vb = j % kDV, vu = j / kDV, pbf = j % kDP, pu = j / kDP;
                if (!mbar_wait(&bars.p_full[pbf], pu & 1, abort_, flags)) break;
                if (!mbar_wait(&bars.vf_full[vb], vu & 1, abort_, flags)) break;
                fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ks++) {
                    const uint32_t pb = pf + pbf * LY::PT + (ks >> 2) * (16 * 128) + (ks & 3) * 32;
                    mma_ts(tmem + P1_COL_O, tmem + P1_COL_V + vb * 64 + ks * 8,
                           sdesc_sw128(pb, 16, 1024), id_pv, (j > 0 || ks > 0) ? 1u : 0u);
                }
                mma_commit(&bars.vf_empty[vb]);
                mma_commit(&bars.p_empty[pbf]);
            }
            mma_commit(&bars.drain_pv);
            volatile int no_abort = 0;
            mbar_wait(&bars.drain_pv, 0, &no_abort, flags);
        }
    } else if (warp < kWS0) {
        // ---------------------------------------------------- K converters
        const int t = (warp & 3) * 32 + lane;  // token row = TMEM lane of this warp
        const uint32_t k_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16) + P1_COL_K;
        const bool qok = convert_q(q + (size_t)b * Hq * D, Hq, smem + LY::OFF_QF, t);
        if (!__all_sync(0xffffffffu, qok) && lane == 0 && chunk == 0) atomicOr(flags, FLAG_Q_RANGE);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_ready);
        bool bad_scale = false;
        for (int j = 0; j < n; j++) {
            const int st = j % kNR, kb = j % kDK, ku = j / kDK;
            if (!mbar_wait(&bars.raw_full[st], (j / kNR) & 1, abort_, flags)) break;
            // slot kb last held tile j - kDK: its QK must be done and the
            // softmax must have read its scores and scales
            if (ku > 0 && (!mbar_wait(&bars.kf_empty[kb], (ku - 1) & 1, abort_, flags) ||
                           !mbar_wait(&bars.s_empty[kb], (ku - 1) & 1, abort_, flags)))
                break;
            const uint8_t* raw = smem + LY::OFF_RAW + st * LY::RAW;
            const bool valid = s_begin + j * TOK + t < s_end;
            fence_after_sync();
            convert_row_tmem(raw + LY::RAW_K, t, valid, k_lane + kb * 64);
            const float sk = reinterpret_cast<const float*>(raw + LY::RAW_SK)[t];
            const float sv = reinterpret_cast<const float*>(raw + LY::RAW_SV)[t];
            skb[kb * TOK + t] = valid ? sk : 0.f;
            svb[kb * TOK + t] = valid ? sv : 0.f;
            bad_scale |= valid && !(sv <= 255.f);
            tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.kf_full[kb]);
                mbar_arrive(&bars.raw_empty[st]);
            }
        }
        if (__any_sync(0xffffffffu, bad_scale) && lane == 0) atomicOr(flags, FLAG_SCALE_RANGE);
    } else if (warp >= kWV0) {
        // ---------------------------------------------------- V converters
        // V^T into TMEM, lane = dim: this warp owns dims 32 q4 .. 32 q4 + 31.
        // A transposing 16 x 16 byte load gives thread (g = lane/4, tq = lane%4)
        // dims g and g + 8 of a 16-dim block, tokens 4 tq .. 4 tq + 3 of a
        // 16-token block; converted, they are exactly what a 16x256b TMEM
        // store puts in lanes g, g + 8 and columns 2 tq, 2 tq + 1 (column c
        // holds tokens 2c, 2c + 1).
        const int q4 = warp & 3;
        const int tq = lane & 3;
        const uint32_t v_base = tmem + ((uint32_t)(q4 * 32) << 16) + P1_COL_V;
        for (int j = 0; j < n; j++) {
            const int st = j % kNR, vb = j % kDV, vu = j / kDV;
            if (!mbar_wait(&bars.raw_full[st], (j / kNR) & 1, abort_, flags)) break;
            if (vu > 0 && !mbar_wait(&bars.vf_empty[vb], (vu - 1) & 1, abort_, flags)) break;
            fence_after_sync();
            const uint8_t* raw = smem + LY::OFF_RAW + st * LY::RAW + LY::RAW_V;
            const int row0 = s_begin + j * TOK;
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int c = 2 * q4 + h;  // 16-byte chunk = dims 16c .. 16c + 15
#pragma unroll
                for (int kb = 0; kb < 8; kb++) {
                    const int r = kb * 16 + (lane & 15);
                    uint32_t b0, b1;
                    ldmatrix_t16_b8(smem_u32(raw + r * 128 + ((c ^ (r & 7)) << 4)), b0, b1);
                    // tokens past the chunk end (e.g. beyond the length) become zeros
                    const int nv = s_end - (row0 + kb * 16 + 4 * tq);
                    if (nv < 4) {
                        const uint32_t m = nv <= 0 ? 0u : (1u << (8 * nv)) - 1u;
                        b0 &= m;
                        b1 &= m;
                    }
                    tmem_st_16x256b(v_base + ((uint32_t)(16 * h) << 16) + vb * 64 + kb * 8,
                                    e4m3x2_lo_to_f16x2(b0), e4m3x2_lo_to_f16x2(b0 >> 16),
                                    e4m3x2_lo_to_f16x2(b1), e4m3x2_lo_to_f16x2(b1 >> 16));
                }
            }
            tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars.vf_full[vb]);
                mbar_arrive(&bars.raw_empty[st]);
            }
        }
    } else {
        // ----------------------------------------------------------- softmax
        // group g owns heads 8g .. 8g+7 for all 128 tokens of a tile: its own
        // running references, partial sums, votes and O^T columns
        constexpr int NH = 8;
        const int g = (warp - kWS0) >> 2;
        const int h0 = NH * g;
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const int t = wq * 32 + lane;            // token row = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        float* gred = red + g * (4 * NH);        // [4][NH]
        const int bar_vote = 1 + 2 * g, bar_red = 2 + 2 * g;
        uint8_t* pf = smem + LY::OFF_P;
        // the sketch is read back by the next kernel: keep it in L2
        const uint64_t sk_pol = l2_evict_last();
        // R = running max - kSk: probabilities are formed as 2^(x - R), in
        // (0, 2^(kLazy + kSk)], which is the range the sketch codes cover
        float R[NH], l[NH];
#pragma unroll
        for (int h = 0; h < NH; h++) {
            R[h] = -INFINITY;
            l[h] = 0.f;
        }
        bool ok = true;
        for (int j = 0; j < n; j++) {
            const int kb = j % kDK, pbf = j % kDP, pu = j / kDP;
            if (!mbar_wait(&bars.s_full[kb], (j / kDK) & 1, abort_, flags)) {
                ok = false;
                break;
            }
            fence_after_sync();
            uint32_t r[NH];
            tmem_ld8(lane_addr + P1_COL_S + kb * 16 + h0, r);
            tmem_ld_wait();
            const float ks = skb[kb * TOK + t] * qk_scale;
            const float sv = svb[kb * TOK + t] * (1.f / 64.f);
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.s_empty[kb]);
            const bool valid = s_begin + j * TOK + t < s_end;
            float x[NH];
            bool over = false;
#pragma unroll
            for (int h = 0; h < NH; h++) {
                x[h] = valid ? __uint_as_float(r[h]) * ks : -INFINITY;
                over |= x[h] > R[h] + (kLazy + kSk);
            }
            if (bar_red_or(over, bar_vote, 128)) {
                // raise this group's running maxima to the tile's maxima
                float mx[NH];
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    float v = x[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    mx[h] = v;
                }
                if (lane < NH) {
                    float v = mx[0];
#pragma unroll
                    for (int h = 1; h < NH; h++)
                        if (lane == h) v = mx[h];
                    gred[wq * NH + lane] = v;
                }
                bar_named(bar_red, 128);
                float alpha[NH];
                bool any_scale = false;
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    const float tm = fmaxf(fmaxf(gred[h], gred[NH + h]),
                                           fmaxf(gred[2 * NH + h], gred[3 * NH + h]));
                    const float nm = fmaxf(R[h], tm - kSk);
                    alpha[h] = (R[h] == -INFINITY || nm == R[h]) ? 1.f : ex2(R[h] - nm);
                    any_scale |= alpha[h] != 1.f;
                    R[h] = nm;
                    l[h] *= alpha[h];
                }
                bar_named(bar_red, 128);  // gred[] is read by everyone before it is reused
                if (j > 0 && any_scale) {
                    // O^T holds tiles 0..j-1: wait for PV(j-1), scale this group's columns
                    const int pb1 = (j - 1) % kDP, pu1 = (j - 1) / kDP;
                    if (!mbar_wait(&bars.p_empty[pb1], pu1 & 1, abort_, flags)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    uint32_t o[NH];
                    tmem_ld8(lane_addr + P1_COL_O + h0, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < NH; h++) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                    tmem_st8(lane_addr + P1_COL_O + h0, o);
                    tmem_st_wait();
                    fence_before_sync();
                }
            }
            float pr[NH];
            uint32_t pw[NH / 2];
#pragma unroll
            for (int h = 0; h < NH; h++) {
                pr[h] = (valid && R[h] != -INFINITY) ? ex2(x[h] - R[h]) : 0.f;
                l[h] += pr[h];
            }
#pragma unroll
            for (int i = 0; i < NH / 2; i++) pw[i] = pack_f16(pr[2 * i] * sv, pr[2 * i + 1] * sv);
            if (sketch != nullptr) {
                const int tok = s_begin + j * TOK + t;
                if (valid) {
                    uint32_t hw[NH / 2];
#pragma unroll
                    for (int i = 0; i < NH / 2; i++) hw[i] = f16x2_rz(pr[2 * i], pr[2 * i + 1]);
                    const uint2 cw = make_uint2(prmt(hw[0] >> 7, hw[1] >> 7, 0x6420u),
                                                prmt(hw[2] >> 7, hw[3] >> 7, 0x6420u));
                    st_hint_v2(sketch + ((size_t)b * Tmax + tok) * 16 + h0, cw, sk_pol);
                }
                if (wq == 0 && lane < NH) {
                    float rv = R[0];
#pragma unroll
                    for (int h = 1; h < NH; h++)
                        if (lane == h) rv = R[h];
                    rsnap[((size_t)b * sk_tiles + (s_begin / TOK + j)) * 16 + h0 + lane] = rv;
                }
            }
            if (pu > 0 && !mbar_wait(&bars.p_empty[pbf], (pu - 1) & 1, abort_, flags)) {
                ok = false;
                break;
            }
            uint8_t* pt = pf + pbf * LY::PT;
#pragma unroll
            for (int h = 0; h < NH; h++)
                *reinterpret_cast<uint16_t*>(pt + f16_off(16, h0 + h, t)) =
                    (uint16_t)(pw[h >> 1] >> (16 * (h & 1)));
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.p_full[pbf]);
        }
        // chunk partial: l summed over the tile rows, O^T from TMEM (lane = dim)
#pragma unroll
        for (int h = 0; h < NH; h++) {
            float v = l[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            l[h] = v;
        }
        if (lane < NH) {
            float v = l[0];
#pragma unroll
            for (int h = 1; h < NH; h++)
                if (lane == h) v = l[h];
            gred[wq * NH + lane] = v;
        }
        bar_named(bar_red, 128);
        float* dst = part + ((size_t)b * n_chunks + chunk) * PART;
        if (t < NH) {
            float mt = R[0];
#pragma unroll
            for (int h = 1; h < NH; h++)
                if (t == h) mt = R[h];
            // O is relative to R + kSk (the P tiles carry sv / 64), so is the sum
            dst[16 * D + h0 + t] = mt + kSk;
            dst[16 * D + 16 + h0 + t] =
                (gred[t] + gred[NH + t] + gred[2 * NH + t] + gred[3 * NH + t]) * (1.f / 64.f);
        }
        // the last PV (and with it every earlier one) has completed once its
        // P buffer is released
        if (ok && n > 0 &&
            mbar_wait(&bars.p_empty[(n - 1) % kDP], ((n - 1) / kDP) & 1, abort_, flags)) {
            fence_after_sync();
            uint32_t o[NH];
            tmem_ld8(lane_addr + P1_COL_O + h0, o);
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < NH; h++) dst[(h0 + h) * D + t] = __uint_as_float(o[h]);
        } else {
#pragma unroll
            for (int h = 0; h < NH; h++) dst[(h0 + h) * D + t] = 0.f;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == kWQK) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
    // ---- the last chunk of the sequence merges every chunk's partial
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        // the per-call counters are zeroed by the kernel launched before this one
        griddep_wait();
        bars.last = (atomicAdd(counter + b, 1u) == (unsigned)(n_chunks - 1));
    }
    __syncthreads();
    if (!bars.last) return;
    __threadfence();
    // every chunk's maximum and sum once (the pipeline buffers are free now),
    // then per row the merged maximum M, the chunks' factors 2^(m_i - M) and
    // the sum; then the O sums, their loads independent of one another
    const float* pb = part + (size_t)b * n_chunks * PART;
    float* fm = reinterpret_cast<float*>(smem);  // [n_chunks][16] m_i, then 2^(m_i - M)
    float* fl = fm + n_chunks * 16;              // [n_chunks][16] l_i
    float* rs = fl + n_chunks * 16;              // [16] merged sums
    for (int i = threadIdx.x; i < n_chunks * 16; i += blockDim.x) {
        const float* p = pb + (size_t)(i >> 4) * PART + 16 * D + (i & 15);
        fm[i] = __ldcg(p);
        fl[i] = __ldcg(p + 16);
    }
    __syncthreads();
    if (threadIdx.x < Hq) {
        const int row = threadIdx.x;
        float mx = -INFINITY;
        for (int i = 0; i < n_chunks; i++) mx = fmaxf(mx, fm[i * 16 + row]);
        const float mu = mx == -INFINITY ? 0.f : mx;
        float ls = 0.f;
        for (int i = 0; i < n_chunks; i++) {
            const float f = ex2(fm[i * 16 + row] - mu);
            fm[i * 16 + row] = f;
            ls += f * fl[i * 16 + row];
        }
        rs[row] = ls;
        const float l2 = ls > 0.f ? mu + __log2f(ls) : -INFINITY;
        lse2_ws[b * 16 + row] = l2;
        if (lse_out) lse_out[b * Hq + row] = l2 * kLn2;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < Hq * D; e += blockDim.x) {
        const int row = e / D;
        float acc = 0.f;
        int i = 0;
        for (; i + 4 <= n_chunks; i += 4) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; u++) v[u] = __ldcg(pb + (size_t)(i + u) * PART + e);
#pragma unroll
            for (int u = 0; u < 4; u++) acc += fm[(i + u) * 16 + row] * v[u];
        }
        for (; i < n_chunks; i++) acc += fm[i * 16 + row] * __ldcg(pb + (size_t)i * PART + e);
        const float ls = rs[row];
        out[(size_t)b * Hq * D + e] = __float2bfloat16_rn(ls > 0.f ? acc / ls : 0.f);
    }
}

}  // namespace dtc
}  // namespace hs2
