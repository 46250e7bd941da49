// Prefill full-attention layer with token selection (warp-MMA version).
//
// HySparse2 summary ("What differs"): the full-attention layer scores every
// older token with exact attention and, per query token, keeps the recent
// window plus the top-k tokens outside it.  Two passes over the keys:
//   pass 1  causal flash attention per (64 query rows, 2 heads): O and the
//           per-(token, head) log-sum-exp;
//   pass 2  per 16 query rows and ALL heads: score(t,s) = sum_h 2^(l2_h(t,s) -
//           lse2_h(t)) for candidates s <= t-W, tile by tile, feeding a
//           streaming per-row top-k: keys above the row's running threshold are
//           appended to the row's buffer in the workspace; a full buffer is cut
//           back to its k best by a warp radix select, which raises the
//           threshold.  The L x L probability matrix never leaves the chip.
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int PF_BM = 64;  // pass-1 query rows per CTA
constexpr int PF_BN = 64;  // keys per tile
constexpr int PS_BM = 16;  // pass-2 query rows per CTA

// byte offset of 16-byte chunk `ch` of row `r` in a swizzled [rows][D] bf16 tile
template <int D>
HS2_DEV uint32_t swz(int r, int ch) {
    return (uint32_t)(r * (D * 2) + ((ch ^ (r & 7)) << 4));
}

// Async copy of rows [row0, row0+64) of a [*, D] bf16 matrix into a swizzled
// tile; rows >= n_rows are zero-filled.
template <int D, int NTHREADS>
HS2_DEV void load_tile_async(uint8_t* tile, const __nv_bfloat16* src, int row0, int n_rows) {
    constexpr int CH = D / 8;
    for (int i = threadIdx.x; i < PF_BN * CH; i += NTHREADS) {
        const int r = i / CH, ch = i % CH;
        const int gr = row0 + r;
        const bool ok = gr < n_rows;
        const __nv_bfloat16* p = src + (size_t)(ok ? gr : 0) * D + ch * 8;
        cp_async16(tile + swz<D>(r, ch), p, ok);
    }
}

// A fragments of a 16-row block of Q straight from global (rows >= valid -> 0).
// q points at row 0 of the block; rows are `stride` elements apart.
template <int D>
HS2_DEV void load_q_frags(uint32_t (&qa)[D / 16][4], const __nv_bfloat16* q, size_t stride,
                          int valid) {
    const int lane = lane_id(), g = lane >> 2, c = lane & 3;
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(q + g * stride);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(q + (g + 8) * stride);
#pragma unroll
    for (int ks = 0; ks < D / 16; ks++) {
        qa[ks][0] = g < valid ? __ldg(r0 + ks * 8 + c) : 0u;
        qa[ks][1] = g + 8 < valid ? __ldg(r1 + ks * 8 + c) : 0u;
        qa[ks][2] = g < valid ? __ldg(r0 + ks * 8 + 4 + c) : 0u;
        qa[ks][3] = g + 8 < valid ? __ldg(r1 + ks * 8 + 4 + c) : 0u;
    }
}

// B fragments of n-tiles (2*jp, 2*jp+1) at k-step ks from a swizzled K tile.
template <int D>
HS2_DEV void ldsm_k(uint32_t (&b)[4], const uint8_t* tile, int jp, int ks) {
    const int lane = lane_id();
    const int mi = lane >> 3, ri = lane & 7;
    const int r = 16 * jp + 8 * (mi >> 1) + ri;
    const int ch = 2 * ks + (mi & 1);
    ldsm_x4(b, tile + swz<D>(r, ch));
}

// B fragments of output n-tiles (2*jp, 2*jp+1) at key step p from a swizzled V tile.
template <int D>
HS2_DEV void ldsm_v(uint32_t (&b)[4], const uint8_t* tile, int jp, int p) {
    const int lane = lane_id();
    const int mi = lane >> 3, ri = lane & 7;
    const int r = 16 * p + 8 * (mi & 1) + ri;
    const int ch = 2 * jp + (mi >> 1);
    ldsm_x4_t(b, tile + swz<D>(r, ch));
}

// ------------------------------------------------------------------ pass 1
// grid (ceil(L/64), Hq/2, B), 8 warps: warp w -> head 2*blockIdx.y + w/4,
// query rows 16*(w%4)..+15 of the block.  Query blocks run longest first.
template <int D>
__global__ void __launch_bounds__(256)
prefill_pass1_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ o,
                     float* __restrict__ lse, int L, int Hq, float scale2) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int TILE = PF_BN * D * 2;
    uint8_t* ks_[2] = {smem, smem + TILE};
    uint8_t* vs_[2] = {smem + 2 * TILE, smem + 3 * TILE};
    const int nqb = (L + PF_BM - 1) / PF_BM;
    const int qb = nqb - 1 - blockIdx.x;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = lane_id(), g = lane >> 2, c = lane & 3;
    const int h = 2 * blockIdx.y + (warp >> 2);
    const int m0 = qb * PF_BM + 16 * (warp & 3);  // first query row of this warp
    const __nv_bfloat16* kb = k + (size_t)b * L * D;
    const __nv_bfloat16* vb = v + (size_t)b * L * D;

    uint32_t qa[D / 16][4];
    const size_t qstride = (size_t)Hq * D;
    load_q_frags<D>(qa, q + ((size_t)b * L + m0) * qstride + (size_t)h * D, qstride,
                    max(0, min(16, L - m0)));
    float oacc[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; j++) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const int row_t[2] = {m0 + g, m0 + g + 8};

    const int n_kt = qb + 1;  // key tiles 0..qb (PF_BN == PF_BM)
    load_tile_async<D, 256>(ks_[0], kb, 0, L);
    load_tile_async<D, 256>(vs_[0], vb, 0, L);
    cp_async_commit();
    for (int kt = 0; kt < n_kt; kt++) {
        const int st = kt & 1;
        if (kt + 1 < n_kt) {
            load_tile_async<D, 256>(ks_[st ^ 1], kb, (kt + 1) * PF_BN, L);
            load_tile_async<D, 256>(vs_[st ^ 1], vb, (kt + 1) * PF_BN, L);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        float s[PF_BN / 8][4];
#pragma unroll
        for (int j = 0; j < PF_BN / 8; j++) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ks++) {
#pragma unroll
            for (int jp = 0; jp < PF_BN / 16; jp++) {
                uint32_t bf[4];
                ldsm_k<D>(bf, ks_[st], jp, ks);
                mma_bf16(s[2 * jp], qa[ks], bf[0], bf[1]);
                mma_bf16(s[2 * jp + 1], qa[ks], bf[2], bf[3]);
            }
        }
        const bool diag = kt == qb;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < PF_BN / 8; j++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int key = kt * PF_BN + 8 * j + 2 * c + (e & 1);
                float x = s[j][e] * scale2;
                if (diag && key > row_t[e >> 1]) x = -INFINITY;
                s[j][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        float alpha[2], mu[2];
#pragma unroll
        for (int r = 0; r < 2; r++) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float mn = fmaxf(mrow[r], mx[r]);
            mu[r] = mn == -INFINITY ? 0.f : mn;
            alpha[r] = ex2(mrow[r] - mu[r]);
            mrow[r] = mn;
            lrow[r] *= alpha[r];
        }
#pragma unroll
        for (int j = 0; j < D / 8; j++) {
            oacc[j][0] *= alpha[0]; oacc[j][1] *= alpha[0];
            oacc[j][2] *= alpha[1]; oacc[j][3] *= alpha[1];
        }
#pragma unroll
        for (int p = 0; p < PF_BN / 16; p++) {
            float pr[2][4];
#pragma unroll
            for (int jj = 0; jj < 2; jj++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    pr[jj][e] = ex2(s[2 * p + jj][e] - mu[e >> 1]);
                    lrow[e >> 1] += pr[jj][e];
                }
            uint32_t pa[4];
            pa[0] = pack_bf16(pr[0][0], pr[0][1]);
            pa[1] = pack_bf16(pr[0][2], pr[0][3]);
            pa[2] = pack_bf16(pr[1][0], pr[1][1]);
            pa[3] = pack_bf16(pr[1][2], pr[1][3]);
#pragma unroll
            for (int jp = 0; jp < D / 16; jp++) {
                uint32_t bf[4];
                ldsm_v<D>(bf, vs_[st], jp, p);
                mma_bf16(oacc[2 * jp], pa, bf[0], bf[1]);
                mma_bf16(oacc[2 * jp + 1], pa, bf[2], bf[3]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 2; r++) {
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
        lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
    }
#pragma unroll
    for (int r = 0; r < 2; r++) {
        const int t = row_t[r];
        if (t >= L) continue;
        const float inv = 1.f / lrow[r];
        __nv_bfloat16* orow = o + (((size_t)b * L + t) * Hq + h) * D;
#pragma unroll
        for (int j = 0; j < D / 8; j++)
            *reinterpret_cast<uint32_t*>(orow + 8 * j + 2 * c) =
                pack_bf16(oacc[j][2 * r] * inv, oacc[j][2 * r + 1] * inv);
        if (c == 0) lse[((size_t)b * L + t) * Hq + h] = (mrow[r] + __log2f(lrow[r])) * kLn2;
    }
}

// ------------------------------------------------------------------ pass 2
struct RowState {
    uint64_t thr;  // keys >= thr may still enter the row's top-k
    int cnt;       // entries in the row's buffer
};

// Cut a row buffer of `cnt` unique keys back to its k best, in place; returns
// the new threshold.  One warp.
HS2_DEV uint64_t warp_compact(uint64_t* buf, int cnt, int k, int* hist) {
    const int lane = lane_id();
    const uint64_t thr =
        warp_radix_threshold([&](int i) { return __ldcg(buf + i); }, cnt, k, hist);
    int wp = 0;
    for (int i0 = 0; i0 < cnt; i0 += 32) {
        const int i = i0 + lane;
        const uint64_t key = i < cnt ? __ldcg(buf + i) : 0;
        const bool keep = i < cnt && key >= thr;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (keep) __stcg(buf + wp + __popc(bal & ((1u << lane) - 1)), key);
        wp += __popc(bal);
    }
    __syncwarp();
    return thr;
}

// grid (ceil(L/16), B), 8 warps.  Warp w owns heads w, w+8 (those < Hq) for the
// MMA and query rows 2w, 2w+1 of the block for the top-k bookkeeping.
template <int D>
__global__ void __launch_bounds__(256)
prefill_pass2_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const float* __restrict__ lse, int L, int Hq, int W, int kk, int S, int cap,
                     float scale2, uint64_t* __restrict__ wsbuf, int32_t* __restrict__ idx) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int TILE = PF_BN * D * 2;
    uint8_t* kt_[2] = {smem, smem + TILE};
    float* part = reinterpret_cast<float*>(smem + 2 * TILE);      // [8][16][64]
    float* score = part + 8 * PS_BM * PF_BN;                        // [16][64]
    int* hist = reinterpret_cast<int*>(score + PS_BM * PF_BN);      // [8][256]
    RowState* rs = reinterpret_cast<RowState*>(hist + 8 * 256);     // [16]

    const int nqb = (L + PS_BM - 1) / PS_BM;
    const int qb = nqb - 1 - blockIdx.x;
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = lane_id(), g = lane >> 2, c = lane & 3;
    const int m0 = qb * PS_BM;
    const __nv_bfloat16* kb = k + (size_t)b * L * D;
    const int valid_rows = min(PS_BM, L - m0);

    // this warp's heads
    const int h0 = warp, h1 = warp + 8;
    const bool has0 = h0 < Hq, has1 = h1 < Hq;
    uint32_t qa0[D / 16][4], qa1[D / 16][4];
    const size_t qstride = (size_t)Hq * D;
    const __nv_bfloat16* qrow = q + ((size_t)b * L + m0) * qstride;
    load_q_frags<D>(qa0, qrow + (size_t)(has0 ? h0 : 0) * D, qstride, has0 ? valid_rows : 0);
    load_q_frags<D>(qa1, qrow + (size_t)(has1 ? h1 : 0) * D, qstride, has1 ? valid_rows : 0);
    float l2a[2], l2b[2];
#pragma unroll
    for (int r = 0; r < 2; r++) {
        const int t = m0 + g + 8 * r;
        const size_t li = ((size_t)b * L + min(t, L - 1)) * Hq;
        l2a[r] = (has0 && t < L) ? __ldg(lse + li + h0) * kLog2e : INFINITY;
        l2b[r] = (has1 && t < L) ? __ldg(lse + li + h1) * kLog2e : INFINITY;
    }
    if (threadIdx.x < PS_BM) {
        rs[threadIdx.x].thr = 0;
        rs[threadIdx.x].cnt = 0;
    }
    // candidates of the block: keys 0 .. m0+15-W
    const int last_key = min(m0 + PS_BM, L) - 1 - W;
    const int n_kt = (kk > 0 && last_key >= 0) ? last_key / PF_BN + 1 : 0;
    int* my_hist = hist + warp * 256;

    if (n_kt > 0) {
        load_tile_async<D, 256>(kt_[0], kb, 0, L);
        cp_async_commit();
    }
    for (int kt = 0; kt < n_kt; kt++) {
        const int st = kt & 1;
        if (kt + 1 < n_kt) load_tile_async<D, 256>(kt_[st ^ 1], kb, (kt + 1) * PF_BN, L);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        float s0[PF_BN / 8][4], s1[PF_BN / 8][4];
#pragma unroll
        for (int j = 0; j < PF_BN / 8; j++)
#pragma unroll
            for (int e = 0; e < 4; e++) s0[j][e] = s1[j][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ks++) {
#pragma unroll
            for (int jp = 0; jp < PF_BN / 16; jp++) {
                uint32_t bf[4];
                ldsm_k<D>(bf, kt_[st], jp, ks);
                mma_bf16(s0[2 * jp], qa0[ks], bf[0], bf[1]);
                mma_bf16(s0[2 * jp + 1], qa0[ks], bf[2], bf[3]);
                if (has1) {
                    mma_bf16(s1[2 * jp], qa1[ks], bf[0], bf[1]);
                    mma_bf16(s1[2 * jp + 1], qa1[ks], bf[2], bf[3]);
                }
            }
        }
        // head-partial probabilities of this warp's heads
        float* wp = part + warp * PS_BM * PF_BN;
#pragma unroll
        for (int j = 0; j < PF_BN / 8; j++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int r = e >> 1;
                float p = ex2(s0[j][e] * scale2 - l2a[r]);
                if (has1) p += ex2(s1[j][e] * scale2 - l2b[r]);
                wp[(g + 8 * r) * PF_BN + 8 * j + 2 * c + (e & 1)] = p;
            }
        __syncthreads();
        // sum over the 8 warps (all heads), mask non-candidates
        for (int i = threadIdx.x; i < PS_BM * PF_BN; i += 256) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < 8; w++) acc += part[w * PS_BM * PF_BN + i];
            score[i] = acc;
        }
        __syncthreads();
        // streaming top-k: warp w updates rows 2w, 2w+1
#pragma unroll
        for (int rr = 0; rr < 2; rr++) {
            const int r = 2 * warp + rr;
            const int t = m0 + r;
            if (t >= L) continue;
            const int maxkey = t - W;  // candidates 0..t-W
            uint64_t* buf = wsbuf + ((size_t)b * L + t) * cap;
            RowState st_ = rs[r];
#pragma unroll
            for (int half = 0; half < 2; half++) {
                const int key = kt * PF_BN + 32 * half + lane;
                const bool cand = key <= maxkey;
                const uint64_t kv = make_key(score[r * PF_BN + 32 * half + lane], (uint32_t)key);
                bool take = cand && kv >= st_.thr;
                unsigned bal = __ballot_sync(0xffffffffu, take);
                if (st_.cnt + __popc(bal) > cap) {
                    st_.thr = warp_compact(buf, st_.cnt, kk, my_hist);
                    st_.cnt = kk;
                    take = cand && kv >= st_.thr;
                    bal = __ballot_sync(0xffffffffu, take);
                }
                if (take) __stcg(buf + st_.cnt + __popc(bal & ((1u << lane) - 1)), kv);
                st_.cnt += __popc(bal);
            }
            __syncwarp();
            if (lane == 0) rs[r] = st_;
        }
        __syncthreads();
    }
    __syncthreads();
    // final selection rows: window ascending, top-k of the buffer, -1 padding
#pragma unroll
    for (int rr = 0; rr < 2; rr++) {
        const int r = 2 * warp + rr;
        const int t = m0 + r;
        if (t >= L) continue;
        uint64_t* buf = wsbuf + ((size_t)b * L + t) * cap;
        int cnt = rs[r].cnt;
        if (cnt > kk) {
            warp_compact(buf, cnt, kk, my_hist);
            cnt = kk;
        }
        const int w0 = max(0, t - W + 1);
        const int wl = t - w0 + 1;
        int32_t* row = idx + ((size_t)b * L + t) * S;
        for (int i = lane; i < S; i += 32) {
            int32_t val = -1;
            if (i < wl)
                val = w0 + i;
            else if (i < wl + cnt)
                val = (int32_t)key_pos(__ldcg(buf + (i - wl)));
            row[i] = val;
        }
    }
}

}  // namespace hs2
