// Warp-level attention of ONE query token (its Hq heads as the 16 rows of the
// MMA M dimension; MQA, so every head reads the same K/V row) over a list of
// key rows, in tiles of 16 rows.  Used by the sparse layer (rows named by the
// inherited selection -- KV Reuse in the HySparse2 summary, "How it works")
// and by the decode full layer (rows 0..T-1 streamed in order).
//
// Each lane loads whole 16-byte pieces of K and V rows from global memory
// straight into MMA fragments (no shared-memory staging):
//   QK^T: k-step ks of lane (g,c) covers row elements c*D/4 + 4ks .. +3, so a
//         lane reads the contiguous quarter [c*D/4, (c+1)*D/4) of the K row of
//         tile key g (n-tile 0) and 8+g (n-tile 1); Q's A fragments use the
//         same element order.
//   PV:   output n-tile jj, column g is element g*D/8 + jj; the lane reads the
//         contiguous eighth [g*D/8, (g+1)*D/8) of the V rows of tile keys
//         2c, 2c+1, 2c+8, 2c+9 and regroups them with byte permutes.
// e4m3 K rows become exact f16 values times 2^-8 by a bit move (common.cuh),
// e4m3 V rows exact f16 values by the hardware conversion, and the MMA runs
// in f16 (Q is converted once; |q| <= 65504 is checked); per-token scales
// multiply the logit (K) and the probability (V) in fp32.  Probabilities are
// relative to a running max raised lazily, so they stay <= 2^8 and
// p * v_scale fits f16 for v_scale <= 255.
#pragma once

#include "common.cuh"

namespace hs2 {

template <int D, bool FP8>
struct KvRow {
    static constexpr int ESZ = FP8 ? 1 : 2;
    static constexpr int KQ_BYTES = D / 4 * ESZ;  // per lane, per K row
    static constexpr int VQ_BYTES = D / 8 * ESZ;  // per lane, per V row
    static constexpr int KQ_VEC = KQ_BYTES / 16;
    static constexpr int VQ_VEC = VQ_BYTES / 16;
    static_assert(KQ_BYTES % 16 == 0 && VQ_BYTES % 16 == 0, "row slice must be 16-byte pieces");
};

// Loaded operands of one 16-key tile for one lane.
template <int D, bool FP8>
struct TileRegs {
    using R = KvRow<D, FP8>;
    uint4 k[2][R::KQ_VEC];  // K rows of tile keys g, 8+g
    uint4 v[4][R::VQ_VEC];  // V rows of tile keys 2c, 2c+1, 2c+8, 2c+9
    float ks[4], vs[4];     // scales of tile keys 2c, 2c+1, 2c+8, 2c+9 (FP8)
    bool kval[4];           // validity of those four keys (lane's S columns)
};

constexpr float kLazyLog2 = 8.f;

template <int D, bool FP8>
struct WarpAttn {
    static constexpr int KS = D / 16;
    static constexpr int NT = D / 8;
    using R = KvRow<D, FP8>;

    uint32_t qa[KS][4];
    float o[NT][4];
    float m[2], l[2];  // log2-domain running max and lane-partial sum, rows g, g+8

    // q: [Hq, D] bf16 row block of one token. Returns false if a value is
    // beyond the f16 range (FP8 path).
    HS2_DEV bool load_q(const __nv_bfloat16* q, int Hq) {
        const int lane = lane_id(), g = lane >> 2, c = lane & 3;
        bool ok = true;
#pragma unroll
        for (int half = 0; half < 2; half++) {
            const int row = g + 8 * half;
            uint32_t w[D / 8];  // D/4 bf16 = D/8 words
            if (row < Hq) {
                const uint4* p = reinterpret_cast<const uint4*>(q + row * D + c * (D / 4));
#pragma unroll
                for (int i = 0; i < D / 32; i++) {
                    uint4 x = ldg_nc(p + i);
                    w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < D / 8; i++) w[i] = 0;
            }
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
                uint32_t lo = w[2 * ks], hi = w[2 * ks + 1];
                if constexpr (FP8) {
                    float a0 = bf16_lo(lo), a1 = bf16_hi(lo), a2 = bf16_lo(hi), a3 = bf16_hi(hi);
                    ok &= fabsf(a0) <= 65504.f && fabsf(a1) <= 65504.f && fabsf(a2) <= 65504.f &&
                          fabsf(a3) <= 65504.f;
                    lo = pack_f16(a0, a1);
                    hi = pack_f16(a2, a3);
                }
                qa[ks][half] = lo;      // a0 / a1: elements 4ks, 4ks+1
                qa[ks][2 + half] = hi;  // a2 / a3: elements 4ks+2, 4ks+3
            }
        }
#pragma unroll
        for (int j = 0; j < NT; j++) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
        return ok;
    }

    // Issue the loads of one tile.  key_k[i]: row index (>= 0) of the lane's K
    // rows (tile keys g, 8+g); key_v[i]: rows of tile keys 2c,2c+1,2c+8,2c+9;
    // invalid keys pass -1 (nothing is loaded, the operand is zero).
    HS2_DEV void load_tile(TileRegs<D, FP8>& t, const uint8_t* kbase, const uint8_t* vbase,
                           const float* kscale, const float* vscale, const int (&key_k)[2],
                           const int (&key_v)[4]) const {
        const int lane = lane_id(), g = lane >> 2, c = lane & 3;
#pragma unroll
        for (int i = 0; i < 2; i++) {
            const uint8_t* p = kbase + (size_t)key_k[i] * (D * R::ESZ) + c * R::KQ_BYTES;
#pragma unroll
            for (int j = 0; j < R::KQ_VEC; j++)
                t.k[i][j] = key_k[i] >= 0 ? ldg_nc(p + 16 * j) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const uint8_t* p = vbase + (size_t)key_v[i] * (D * R::ESZ) + g * R::VQ_BYTES;
#pragma unroll
            for (int j = 0; j < R::VQ_VEC; j++)
                t.v[i][j] = key_v[i] >= 0 ? ldg_nc(p + 16 * j) : make_uint4(0, 0, 0, 0);
            t.kval[i] = key_v[i] >= 0;
            if constexpr (FP8) {
                t.ks[i] = key_v[i] >= 0 ? __ldg(kscale + key_v[i]) : 0.f;
                t.vs[i] = key_v[i] >= 0 ? __ldg(vscale + key_v[i]) : 0.f;
            }
        }
    }

    // S (16 heads x 16 keys) = Q K^T for the tile; s[j][*] is n-tile j.
    HS2_DEV void qk(const TileRegs<D, FP8>& t, float (&s)[2][4]) const {
#pragma unroll
        for (int j = 0; j < 2; j++) {
            s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&t.k[j][0]);
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
                uint32_t b0, b1;
                if constexpr (FP8) {
                    e4m3x4_to_f16(w[ks], b0, b1);
                } else {
                    b0 = w[2 * ks];
                    b1 = w[2 * ks + 1];
                }
                mma<FP8>(s[j], qa[ks], b0, b1);
            }
        }
    }

    // Scaled log2-domain logits with invalid keys masked.  Lane columns:
    // s[0][0..1] -> keys 2c,2c+1; s[1][0..1] -> keys 8+2c, 9+2c (same for rows g+8).
    HS2_DEV void scale_mask(const TileRegs<D, FP8>& t, float (&s)[2][4], float qk_scale) const {
#pragma unroll
        for (int j = 0; j < 2; j++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int kk = 2 * j + (e & 1);  // index into the lane's 4 keys
                float x = s[j][e] * qk_scale;
                if constexpr (FP8) x *= t.ks[kk];
                s[j][e] = t.kval[kk] ? x : -INFINITY;
            }
    }

    // Online-softmax update with the tile's logits, then O += P V.
    HS2_DEV void softmax_pv(const TileRegs<D, FP8>& t, float (&s)[2][4]) {
        float mx[2];
        mx[0] = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        mx[1] = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
#pragma unroll
        for (int r = 0; r < 2; r++) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        }
        // The running max is raised only when a tile's max exceeds it by more
        // than 2^8 (log2 units); until then probabilities are taken relative
        // to the older max and stay <= 2^8, and O/l need no rescale.
        const bool up0 = mx[0] > m[0] + kLazyLog2, up1 = mx[1] > m[1] + kLazyLog2;
        if (__any_sync(0xffffffffu, up0 || up1)) {
            const float a0 = up0 ? ex2(m[0] - mx[0]) : 1.f;
            const float a1 = up1 ? ex2(m[1] - mx[1]) : 1.f;
            if (up0) m[0] = mx[0];
            if (up1) m[1] = mx[1];
            l[0] *= a0;
            l[1] *= a1;
#pragma unroll
            for (int jj = 0; jj < NT; jj++) {
                o[jj][0] *= a0; o[jj][1] *= a0;
                o[jj][2] *= a1; o[jj][3] *= a1;
            }
        }
        float mu[2];
        mu[0] = (m[0] == -INFINITY) ? 0.f : m[0];
        mu[1] = (m[1] == -INFINITY) ? 0.f : m[1];
        float p[2][4];
#pragma unroll
        for (int j = 0; j < 2; j++)
#pragma unroll
            for (int e = 0; e < 4; e++) p[j][e] = ex2(s[j][e] - mu[e >> 1]);
        l[0] += (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
        l[1] += (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
        if constexpr (FP8) {
#pragma unroll
            for (int j = 0; j < 2; j++)
#pragma unroll
                for (int e = 0; e < 4; e++) p[j][e] *= t.vs[2 * j + (e & 1)];
        }
        uint32_t pa[4];
        pa[0] = pack2<FP8>(p[0][0], p[0][1]);
        pa[1] = pack2<FP8>(p[0][2], p[0][3]);
        pa[2] = pack2<FP8>(p[1][0], p[1][1]);
        pa[3] = pack2<FP8>(p[1][2], p[1][3]);
#pragma unroll
        for (int jj = 0; jj < NT; jj++) {
            uint32_t b0, b1;
            if constexpr (FP8) {
                // byte bi of two V rows -> the low 16 bits -> hardware e4m3x2 -> f16x2
                const int wi = jj >> 2, bi = jj & 3;
                const uint32_t sel = ((4u + bi) << 4) | bi;
                const uint32_t* v0 = reinterpret_cast<const uint32_t*>(&t.v[0][0]);
                const uint32_t* v1 = reinterpret_cast<const uint32_t*>(&t.v[1][0]);
                const uint32_t* v2 = reinterpret_cast<const uint32_t*>(&t.v[2][0]);
                const uint32_t* v3 = reinterpret_cast<const uint32_t*>(&t.v[3][0]);
                b0 = e4m3x2_lo_to_f16x2(prmt(v0[wi], v1[wi], sel));
                b1 = e4m3x2_lo_to_f16x2(prmt(v2[wi], v3[wi], sel));
            } else {
                const int wi = jj >> 1;
                const uint32_t sel = (jj & 1) ? 0x7632u : 0x5410u;
                const uint32_t* v0 = reinterpret_cast<const uint32_t*>(&t.v[0][0]);
                const uint32_t* v1 = reinterpret_cast<const uint32_t*>(&t.v[1][0]);
                const uint32_t* v2 = reinterpret_cast<const uint32_t*>(&t.v[2][0]);
                const uint32_t* v3 = reinterpret_cast<const uint32_t*>(&t.v[3][0]);
                b0 = prmt(v0[wi], v1[wi], sel);
                b1 = prmt(v2[wi], v3[wi], sel);
            }
            mma<FP8>(o[jj], pa, b0, b1);
        }
    }

    // Reduce the lane-partial sums across the 4 lanes of a row group.
    HS2_DEV void finish_sums() {
#pragma unroll
        for (int r = 0; r < 2; r++) {
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
        }
    }

    // Output scale of the accumulated V values (e4m3 V rows are converted
    // exactly by the hardware conversion, so none is needed).
    static constexpr float kOutScale = 1.f;

    // Store normalised O rows (< Hq) as bf16 into out [Hq, D].  Call finish_sums first.
    HS2_DEV void store(__nv_bfloat16* out, int Hq) const {
        const int lane = lane_id(), g = lane >> 2, c = lane & 3;
#pragma unroll
        for (int r = 0; r < 2; r++) {
            const int row = g + 8 * r;
            if (row >= Hq) continue;
            const float inv = l[r] > 0.f ? kOutScale / l[r] : 0.f;
#pragma unroll
            for (int col = 0; col < 2; col++) {
                // columns 2c+col of every n-tile = elements (2c+col)*D/8 + jj
                uint32_t w[NT / 2];
#pragma unroll
                for (int jj = 0; jj < NT; jj += 2)
                    w[jj / 2] = pack_bf16(o[jj][2 * r + col] * inv, o[jj + 1][2 * r + col] * inv);
                uint4* dst = reinterpret_cast<uint4*>(out + row * D + (2 * c + col) * (D / 8));
#pragma unroll
                for (int i = 0; i < NT / 8; i++)
                    dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            }
        }
    }

    // Fragment order of the o accumulator: value i (0..4D/8-1) of lane L is
    // o[i / 4][i % 4], i.e. row (L >> 2) + 8 * ((i >> 1) & 1) and column
    // (2 * (L & 3) + (i & 1)) * (D / 8) + (i >> 2).  Storing value i of every
    // lane at po[i * 32 + L] makes the 32 lanes of a store hit 32 banks.
    HS2_DEV static int frag_row(int i, int L) { return (L >> 2) + 8 * ((i >> 1) & 1); }
    HS2_DEV static int frag_col(int i, int L) { return (2 * (L & 3) + (i & 1)) * (D / 8) + (i >> 2); }
    static constexpr int FRAG = NT * 4;  // values per lane

    // Write the unnormalised partial state (m, l, o) of rows < 16 into
    // shared/global arrays: pm[16], pl[16], po[16][D] (o in natural element order).
    HS2_DEV void dump(float* pm, float* pl, float* po) const {
        const int lane = lane_id(), g = lane >> 2, c = lane & 3;
#pragma unroll
        for (int r = 0; r < 2; r++) {
            const int row = g + 8 * r;
            if (c == 0) {
                pm[row] = m[r];
                pl[row] = l[r];
            }
#pragma unroll
            for (int col = 0; col < 2; col++)
#pragma unroll
                for (int jj = 0; jj < NT; jj++)
                    po[row * D + (2 * c + col) * (D / 8) + jj] = o[jj][2 * r + col];
        }
    }
};

// Tile key distribution: given this lane's candidate row (lane < 16 holds tile
// key `lane`; other lanes ignored), fetch the rows each lane needs.
HS2_DEV void distribute_keys(int my_row, int (&key_k)[2], int (&key_v)[4]) {
    const int lane = lane_id(), g = lane >> 2, c = lane & 3;
    key_k[0] = __shfl_sync(0xffffffffu, my_row, g);
    key_k[1] = __shfl_sync(0xffffffffu, my_row, 8 + g);
    key_v[0] = __shfl_sync(0xffffffffu, my_row, 2 * c);
    key_v[1] = __shfl_sync(0xffffffffu, my_row, 2 * c + 1);
    key_v[2] = __shfl_sync(0xffffffffu, my_row, 2 * c + 8);
    key_v[3] = __shfl_sync(0xffffffffu, my_row, 2 * c + 9);
}

// Merge NP partial states (m, l, o over 16 rows) into the first; arrays laid
// out as in WarpAttn::dump with stride `stride` floats between partials.
// Executed by a whole block; rows < Hq.
template <int D>
HS2_DEV void merge_partials_block(const float* pm, const float* pl, const float* po, int np,
                                  size_t stride_m, size_t stride_o, int Hq, float* out_m,
                                  float* out_l, float* out_o) {
    for (int e = threadIdx.x; e < Hq * D; e += blockDim.x) {
        const int row = e / D;
        float mx = -INFINITY;
        for (int i = 0; i < np; i++) mx = fmaxf(mx, pm[i * stride_m + row]);
        const float mu = mx == -INFINITY ? 0.f : mx;
        float acc = 0.f, ls = 0.f;
        for (int i = 0; i < np; i++) {
            const float f = ex2(pm[i * stride_m + row] - mu);
            acc += f * po[i * stride_o + e];
            ls += f * pl[i * stride_m + row];
        }
        out_o[e] = acc;
        if (e % D == 0) {
            out_m[row] = mx;
            out_l[row] = ls;
        }
    }
}

}  // namespace hs2
