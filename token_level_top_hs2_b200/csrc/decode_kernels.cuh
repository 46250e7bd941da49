// Decode full layer with token selection, split over the cache length.
//
// One new query per sequence at position t = T-1 attends exactly to cache rows
// 0..t (HySparse2 summary, "What differs": the full layer scores tokens with
// exact attention), and selects the window t-W+1..t plus the top-k of 0..t-W
// by the head-summed probability.  Exact selection needs each head's global
// log-sum-exp before any score can be ranked, hence two streaming passes:
//   pass 1  (per chunk of CH1 rows)  partial (max, sum, O) per head over K and V;
//           the last chunk of a sequence to finish merges them into lse and O;
//   pass 2  (per chunk of CH2 rows)  re-reads K, forms score(s) = sum_h
//           2^(l2_h(s) - lse2_h) for the chunk's candidates and keeps the
//           chunk's k best (radix select on the score bits, ties -> lower s);
//   merge   groups of chunk winners are reduced to k; the last group of a
//           sequence merges the groups and writes window + winners.
// "Last to finish" uses an atomic counter, never a wait.
#pragma once

#include "gather_attn.cuh"

namespace hs2 {

template <int D>
struct DecodePart {
    static constexpr int FLOATS = 16 * D + 32;  // o[16][D], m[16], l[16]
};

// ------------------------------------------------------------------ pass 1
template <int D, bool FP8, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
decode_pass1_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
                    const uint8_t* __restrict__ vc, const float* __restrict__ ks,
                    const float* __restrict__ vs, const int32_t* __restrict__ lengths, int Tmax,
                    int Hq, int ch1, int n_chunks, float qk_scale, float* __restrict__ part,
                    unsigned* __restrict__ counter, float* __restrict__ lse2_ws,
                    float* __restrict__ lse_out, __nv_bfloat16* __restrict__ out,
                    unsigned* __restrict__ flags) {
    using R = KvRow<D, FP8>;
    constexpr int PART = DecodePart<D>::FLOATS;
    extern __shared__ float smem_f[];
    __shared__ unsigned s_last;
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int T = __ldg(lengths + b);
    const bool len_ok = T >= 1 && T <= Tmax;
    if (!len_ok && threadIdx.x == 0 && chunk == 0) atomicOr(flags, FLAG_BAD_LENGTH);
    const int s_begin = chunk * ch1;
    const int s_end = len_ok ? min(s_begin + ch1, T) : s_begin;
    const size_t row0 = (size_t)b * Tmax;
    const uint8_t* kb = kc + row0 * D * R::ESZ;
    const uint8_t* vb = vc + row0 * D * R::ESZ;
    const float* ksb = FP8 ? ks + row0 : nullptr;
    const float* vsb = FP8 ? vs + row0 : nullptr;

    WarpAttn<D, FP8> wa;
    if (!wa.load_q(q + (size_t)b * Hq * D, Hq) && chunk == 0 && lane == 0 && warp == 0)
        atomicOr(flags, FLAG_Q_RANGE);
    if constexpr (FP8) {
        // p*scale_v is held in f16 with p <= 2^8: per-token V scales must stay <= 255
        bool bad = false;
        for (int s = s_begin + threadIdx.x; s < s_end; s += blockDim.x) bad |= !(vsb[s] <= 255.f);
        if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(flags, FLAG_SCALE_RANGE);
    }
    // tiles of 16 consecutive rows, interleaved over warps, one tile prefetched
    int tile = s_begin + warp * 16;
    TileRegs<D, FP8> cur, nxt;
    auto fetch = [&](TileRegs<D, FP8>& tr, int base) {
        const int my = (lane < 16 && base + lane < s_end) ? base + lane : -1;
        int key_k[2], key_v[4];
        distribute_keys(my, key_k, key_v);
        wa.load_tile(tr, kb, vb, ksb, vsb, key_k, key_v);
    };
    if (tile < s_end) fetch(cur, tile);
    for (; tile < s_end; tile += WARPS * 16) {
        const int nt = tile + WARPS * 16;
        if (nt < s_end) fetch(nxt, nt);
        float s[2][4];
        wa.qk(cur, s);
        wa.scale_mask(cur, s, qk_scale);
        wa.softmax_pv(cur, s);
        cur = nxt;
    }
    wa.finish_sums();
    float* mine = smem_f + warp * PART;
    wa.dump(mine + 16 * D, mine + 16 * D + 16, mine);
    __syncthreads();
    float* dst = part + ((size_t)b * n_chunks + chunk) * PART;
    merge_partials_block<D>(smem_f + 16 * D, smem_f + 16 * D + 16, smem_f, WARPS, PART, PART, Hq,
                            dst + 16 * D, dst + 16 * D + 16, dst);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(counter + b, 1u) == (unsigned)(n_chunks - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // last chunk of sequence b: merge every chunk's partial
    const float* pb = part + (size_t)b * n_chunks * PART;
    for (int e = threadIdx.x; e < Hq * D; e += blockDim.x) {
        const int row = e / D;
        float mx = -INFINITY;
        for (int i = 0; i < n_chunks; i++) mx = fmaxf(mx, __ldcg(pb + (size_t)i * PART + 16 * D + row));
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
    if (threadIdx.x == 0) counter[b] = 0;
}

// ------------------------------------------------------------------ pass 2
// Scores of the chunk's candidates into shared memory, then the chunk's k best.
template <int D, bool FP8, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
decode_pass2_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
                    const float* __restrict__ ks, const int32_t* __restrict__ lengths, int Tmax,
                    int Hq, int W, int k, int ch2, int n_chunks, float qk_scale,
                    const float* __restrict__ lse2_ws, uint64_t* __restrict__ cand,
                    int* __restrict__ cand_cnt) {
    using R = KvRow<D, FP8>;
    extern __shared__ float sc[];  // [ch2] scores
    __shared__ int hist[260];
    __shared__ int s_cnt;
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int lane = lane_id(), warp = threadIdx.x >> 5, g = lane >> 2, c = lane & 3;
    const int T = __ldg(lengths + b);
    const int n_total = (T >= 1 && T <= Tmax) ? max(0, T - W) : 0;  // candidates 0..T-1-W
    const int s_begin = chunk * ch2;
    const int s_end = min(s_begin + ch2, n_total);
    const int n = max(0, s_end - s_begin);
    uint64_t* my_cand = cand + ((size_t)b * n_chunks + chunk) * k;
    if (n == 0) {
        if (threadIdx.x == 0) cand_cnt[b * n_chunks + chunk] = 0;
        return;
    }
    const size_t row0 = (size_t)b * Tmax;
    const uint8_t* kb = kc + row0 * D * R::ESZ;
    const float* ksb = FP8 ? ks + row0 : nullptr;
    WarpAttn<D, FP8> wa;
    wa.load_q(q + (size_t)b * Hq * D, Hq);
    float lse2[2];
    lse2[0] = g < Hq ? __ldcg(lse2_ws + b * 16 + g) : INFINITY;
    lse2[1] = g + 8 < Hq ? __ldcg(lse2_ws + b * 16 + g + 8) : INFINITY;

    TileRegs<D, FP8> cur, nxt;
    auto fetch = [&](TileRegs<D, FP8>& tr, int base) {
        const int my = (lane < 16 && base + lane < s_end) ? base + lane : -1;
        int key_k[2], key_v[4];
        distribute_keys(my, key_k, key_v);
        // K rows and K scales only
#pragma unroll
        for (int i = 0; i < 2; i++) {
            const uint8_t* p = kb + (size_t)key_k[i] * (D * R::ESZ) + c * R::KQ_BYTES;
#pragma unroll
            for (int j = 0; j < R::KQ_VEC; j++)
                tr.k[i][j] = key_k[i] >= 0 ? ldg_stream(p + 16 * j) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
            tr.kval[i] = key_v[i] >= 0;
            if constexpr (FP8) tr.ks[i] = key_v[i] >= 0 ? __ldg(ksb + key_v[i]) : 0.f;
        }
    };
    int tile = s_begin + warp * 16;
    if (tile < s_end) fetch(cur, tile);
    for (; tile < s_end; tile += WARPS * 16) {
        const int nt = tile + WARPS * 16;
        if (nt < s_end) fetch(nxt, nt);
        float s[2][4];
        wa.qk(cur, s);
        wa.scale_mask(cur, s, qk_scale);
        // column sums over the 16 head rows: rows g and g+8 in-lane, then over g
        float cs[4];
#pragma unroll
        for (int j = 0; j < 2; j++)
#pragma unroll
            for (int e = 0; e < 2; e++)
                cs[2 * j + e] = ex2(s[j][e] - lse2[0]) + ex2(s[j][2 + e] - lse2[1]);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 4);
            cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 8);
            cs[i] += __shfl_xor_sync(0xffffffffu, cs[i], 16);
        }
        if (g == 0) {
            const int base = tile - s_begin;
            // lane keys: 2c, 2c+1, 2c+8, 2c+9
            if (base + 2 * c < n) sc[base + 2 * c] = cs[0];
            if (base + 2 * c + 1 < n) sc[base + 2 * c + 1] = cs[1];
            if (base + 2 * c + 8 < n) sc[base + 2 * c + 8] = cs[2];
            if (base + 2 * c + 9 < n) sc[base + 2 * c + 9] = cs[3];
        }
        cur = nxt;
    }
    __syncthreads();
    auto key_at = [&](int i) { return make_key(sc[i], (uint32_t)(s_begin + i)); };
    if (threadIdx.x == 0) s_cnt = 0;
    if (n <= k) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) my_cand[i] = key_at(i);
        if (threadIdx.x == 0) cand_cnt[b * n_chunks + chunk] = n;
        return;
    }
    const uint64_t thr = block_radix_threshold(key_at, n, k, hist);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const uint64_t key = key_at(i);
        if (key >= thr) my_cand[atomicAdd(&s_cnt, 1)] = key;
    }
    __syncthreads();
    if (threadIdx.x == 0) cand_cnt[b * n_chunks + chunk] = s_cnt;
}

// ------------------------------------------------------------------- merge
// Reduce `cnt` keys in buf (shared) to their top k in place; returns the new count.
HS2_DEV int block_keep_topk(uint64_t* buf, int cnt, int k, int* hist, int* s_cnt,
                            uint64_t* tmp) {
    if (cnt <= k) return cnt;
    const uint64_t thr = block_radix_threshold([&](int i) { return buf[i]; }, cnt, k, hist);
    if (threadIdx.x == 0) *s_cnt = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
        const uint64_t key = buf[i];
        if (key >= thr) tmp[atomicAdd(s_cnt, 1)] = key;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < k; i += blockDim.x) buf[i] = tmp[i];
    __syncthreads();
    return k;
}

// grid (n_groups, B); each CTA merges up to G chunks of winners.  Shared:
// buf[cap] + tmp[k] keys, cap >= G*k.
__global__ void __launch_bounds__(256)
decode_merge_kernel(const uint64_t* __restrict__ cand, const int* __restrict__ cand_cnt,
                    int n_chunks, int G, int n_groups, int k, int W, int S,
                    const int32_t* __restrict__ lengths, int Tmax, uint64_t* __restrict__ gcand,
                    int* __restrict__ gcnt, unsigned* __restrict__ counter,
                    int32_t* __restrict__ idx) {
    extern __shared__ uint64_t sk[];
    __shared__ int hist[260];
    __shared__ int s_cnt;
    __shared__ unsigned s_last;
    const int cap = G * k;
    uint64_t* buf = sk;
    uint64_t* tmp = sk + cap;
    const int b = blockIdx.y, grp = blockIdx.x;
    // 1) this group's chunks
    int cnt = 0;
    for (int ch = grp * G; ch < min((grp + 1) * G, n_chunks); ch++) {
        const int m = __ldcg(cand_cnt + b * n_chunks + ch);
        const uint64_t* src = cand + ((size_t)b * n_chunks + ch) * k;
        for (int i = threadIdx.x; i < m; i += blockDim.x) buf[cnt + i] = __ldcg(src + i);
        cnt += m;
    }
    __syncthreads();
    cnt = block_keep_topk(buf, cnt, k, hist, &s_cnt, tmp);
    if (n_groups > 1) {
        uint64_t* dst = gcand + ((size_t)b * n_groups + grp) * k;
        for (int i = threadIdx.x; i < cnt; i += blockDim.x) dst[i] = buf[i];
        if (threadIdx.x == 0) gcnt[b * n_groups + grp] = cnt;
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = (atomicAdd(counter + b, 1u) == (unsigned)(n_groups - 1));
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        // 2) last group of the sequence: stream every group's winners through buf
        cnt = 0;
        for (int gi = 0; gi < n_groups; gi++) {
            const int m = __ldcg(gcnt + b * n_groups + gi);
            if (cnt + m > cap) {
                cnt = block_keep_topk(buf, cnt, k, hist, &s_cnt, tmp);
            }
            const uint64_t* src = gcand + ((size_t)b * n_groups + gi) * k;
            for (int i = threadIdx.x; i < m; i += blockDim.x) buf[cnt + i] = __ldcg(src + i);
            cnt += m;
            __syncthreads();
        }
        cnt = block_keep_topk(buf, cnt, k, hist, &s_cnt, tmp);
        if (threadIdx.x == 0) counter[b] = 0;
    }
    // 3) selection row: window ascending, winners, -1 padding
    const int T = __ldg(lengths + b);
    const bool ok = T >= 1 && T <= Tmax;
    const int t = ok ? T - 1 : -1;
    const int w0 = max(0, t - W + 1);
    const int wl = ok ? t - w0 + 1 : 0;
    int32_t* row = idx + (size_t)b * S;
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
        int32_t v = -1;
        if (i < wl)
            v = w0 + i;
        else if (i < wl + cnt)
            v = (int32_t)key_pos(buf[i - wl]);
        row[i] = v;
    }
}

}  // namespace hs2
