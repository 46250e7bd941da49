// Device helpers shared by the hs2 kernels (sm_100a).
//
// Fragment conventions for the warp-level m16n8k16 MMA (PTX ISA, "Matrix
// fragments for mma.m16n8k16"): lane = 4*g + c (g = lane/4, c = lane%4).
//   A (16x16): a0 (row g, k 2c..2c+1), a1 (row g+8, k 2c..), a2 (row g, k 2c+8..),
//              a3 (row g+8, k 2c+8..)
//   B (16x8):  b0 (k 2c..2c+1, col g), b1 (k 2c+8..2c+9, col g)
//   C (16x8):  c0,c1 (row g, cols 2c, 2c+1), c2,c3 (row g+8, cols 2c, 2c+1)
// A contraction is invariant under any permutation of k applied to A and B
// alike, and output columns may be permuted if the store undoes it; the gather
// kernels use both freedoms so that every lane loads whole 16-byte pieces of a
// K or V row straight from global memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#define HS2_DEV __device__ __forceinline__

namespace hs2 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device-side data flags (reported by hs2_get_last_device_error).
enum : unsigned {
    FLAG_BAD_LENGTH = 1u,   // decode length outside [1, Tmax]
    FLAG_Q_RANGE = 2u,      // |q| beyond the fp16 range on an e4m3 path
    FLAG_BAD_INDEX = 4u,    // a selection index outside [0, t]
    FLAG_SCALE_RANGE = 8u,  // a V scale beyond 255 on an e4m3 path
    FLAG_TIMEOUT = 16u,     // a bounded wait inside a kernel gave up
};

HS2_DEV uint32_t lane_id() { return threadIdx.x & 31; }

// Three-input maximum (sm_100): one instruction for two comparisons.
HS2_DEV float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialisation may start while the kernel before it in the stream still
// runs: griddep_wait() returns once that kernel has completed and its memory
// is visible; griddep_launch() lets the next kernel of the stream start
// launching.  Both are no-ops in a kernel launched the plain way.
HS2_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
HS2_DEV void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

HS2_DEV float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, for kernels whose exponentials outrun the MUFU pipe:
// part of them go through this routine instead of ex2.
//   * Cody and Waite's range reduction x = n + f, n an integer, |f| <= 1/2:
//     adding 1.5 * 2^23 rounds x to an integer held in the low mantissa bits
//     of the sum (exact for |x| < 2^22), and subtracting it back gives n as
//     a float;
//   * 2^f by a degree-5 polynomial (Horner, fused multiply-adds) whose
//     coefficients were fitted here for least maximum relative error on
//     [-1/2, 1/2] by Lawson's iteratively reweighted least squares; the
//     fp32 evaluation stays within 2.2e-7 relative of 2^f;
//   * 2^n enters by adding n to the exponent field of the result.
// x is clamped to >= -125 so that the exponent cannot wrap: results below
// 2^-125 come out as about 2^-125 instead of 0 (ex2.approx.ftz flushes
// them); callers sum such values into much larger ones.
HS2_DEV float ex2_fma(float x) {
    const float xc = fmaxf(x, -125.f);
    const float t = xc + 12582912.f;  // 1.5 * 2^23
    const float n = t - 12582912.f;
    const float f = xc - n;
    float p = 1.32764713e-3f;
    p = fmaf(p, f, 9.67554096e-3f);
    p = fmaf(p, f, 5.55071309e-2f);
    p = fmaf(p, f, 2.40221202e-1f);
    p = fmaf(p, f, 6.93146944e-1f);
    p = fmaf(p, f, 1.00000012e+0f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

HS2_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

HS2_DEV void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <bool F16>
HS2_DEV void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (F16)
        mma_f16(d, a, b0, b1);
    else
        mma_bf16(d, a, b0, b1);
}

HS2_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Transposing load of a 16 x 16 byte block (threads 0..15 give the 16 row
// addresses, 16-byte aligned): thread L receives column L/4 (r0) and column
// L/4 + 8 (r1), rows 4(L%4) .. 4(L%4)+3 in bytes 0..3 of each.
HS2_DEV void ldmatrix_t16_b8(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x1.trans.shared.b8 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(addr));
}

// Two floats -> f16x2 rounded toward zero: lo in bits 0..15, hi in bits 16..31.
HS2_DEV uint32_t f16x2_rz(float lo, float hi) {
    uint32_t r;
    asm("cvt.rz.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// f16x2 bit pattern -> the two values as floats (exact).
HS2_DEV float2 f16x2_to_float2(uint32_t h) {
    __half2 v = *reinterpret_cast<__half2*>(&h);
    return __half22float2(v);
}

// Two e4m3 codes sitting in the HIGH bytes of the two 16-bit halves of t
// (low bytes ignored) -> f16x2 whose values are exactly e4m3 * 2^-8.
// e4m3 is s.eeee.mmm with bias 7; f16 is s.eeeee.mmmmmmmmmm with bias 15.
// Moving the 7 magnitude bits down by one places eeee.mmm at exponent bits
// 13..10 and mantissa bits 9..7: a normal code becomes 2^(e-15)(1+m/8) and a
// subnormal one (e = 0) (m/8)2^-14, i.e. the e4m3 value times 2^-8 in both
// cases; the sign bit stays in place.
HS2_DEV uint32_t e4m3_hi_to_f16x2(uint32_t t) {
    return (t & 0x80008000u) | ((t >> 1) & 0x3F803F80u);
}

// Four e4m3 codes (bytes 0..3 of w) -> two f16x2: (byte0, byte1), (byte2, byte3),
// each value = e4m3 * 2^-8.
HS2_DEV void e4m3x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
    lo = e4m3_hi_to_f16x2(prmt(w, 0u, 0x1404u));  // bytes [0, b0, 0, b1]
    hi = e4m3_hi_to_f16x2(prmt(w, 0u, 0x3424u));  // bytes [0, b2, 0, b3]
}

// Two e4m3 codes in the low 16 bits of w -> f16x2 of their exact values
// (byte 0 -> low half).
HS2_DEV uint32_t e4m3x2_lo_to_f16x2(uint32_t w) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(r)
        : "r"(w));
    return r;
}

HS2_DEV uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

HS2_DEV uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <bool F16>
HS2_DEV uint32_t pack2(float lo, float hi) {
    if constexpr (F16)
        return pack_f16(lo, hi);
    else
        return pack_bf16(lo, hi);
}

HS2_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
HS2_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Loads that bypass L1 allocation for data read once.
HS2_DEV uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

HS2_DEV uint4 ldg_nc(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// L2 eviction-priority policies: a stream read once goes first, a small
// intermediate the next kernel reads stays.
HS2_DEV uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
HS2_DEV uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
HS2_DEV void st_hint_v2(void* p, uint2 v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" ::"l"(p), "r"(v.x),
                 "r"(v.y), "l"(policy)
                 : "memory");
}
// a coherent (L2) 16-byte load under a policy
HS2_DEV uint4 ldcg_hint(const void* p, uint64_t policy) {
    uint4 r;
    asm volatile("ld.global.cg.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(policy));
    return r;
}

HS2_DEV void cp_async16(void* smem, const void* gmem, bool valid = true) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n));
}
HS2_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
HS2_DEV void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N));
}

HS2_DEV void ldsm_x4(uint32_t (&r)[4], const void* p) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(s));
}
HS2_DEV void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(s));
}

// Selection key: larger is better.  High word = the score's fp32 bits (scores
// are >= 0, so the bit pattern orders like the value); low word = ~position,
// so that among equal scores the lower position wins.  Keys are unique.
HS2_DEV uint64_t make_key(float score, uint32_t pos) {
    return ((uint64_t)__float_as_uint(score) << 32) | (uint64_t)(~pos);
}
HS2_DEV uint32_t key_pos(uint64_t key) { return ~(uint32_t)key; }

// ---------------------------------------------------------------------------
// Suffix search over a 256-bin histogram held by one warp (hist[0..256)):
// finds the highest bin j with sum_{i >= j} hist[i] >= need.  Returns j (or
// -1 if the total is below need) and sets *above = sum_{i > j} hist[i],
// *in_bin = hist[j].  Bins are read after a __syncwarp by the caller.
HS2_DEV int warp_find_bin(const int* hist, int need, int* above_out, int* in_bin_out) {
    const int lane = lane_id();
    int loc[8];
    int tot = 0;
#pragma unroll
    for (int i = 7; i >= 0; i--) {
        loc[i] = hist[lane * 8 + i];
        tot += loc[i];
    }
    int suf = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
    }
    int above = suf - tot;
    int sel = -1, sab = 0, scnt = 0;
#pragma unroll
    for (int i = 7; i >= 0; i--) {
        if (sel < 0 && above < need && above + loc[i] >= need) {
            sel = lane * 8 + i;
            sab = above;
            scnt = loc[i];
        }
        above += loc[i];
    }
    const unsigned who = __ballot_sync(0xffffffffu, sel >= 0);
    if (!who) {
        *above_out = 0;
        *in_bin_out = 0;
        return -1;
    }
    const int src = __ffs(who) - 1;
    *above_out = __shfl_sync(0xffffffffu, sab, src);
    *in_bin_out = __shfl_sync(0xffffffffu, scnt, src);
    return __shfl_sync(0xffffffffu, sel, src);
}

// ---------------------------------------------------------------------------
// Radix select over unique 64-bit keys: returns T such that exactly `kk` keys
// of keys[0..n) are >= T (requires 0 < kk <= n).  Most-significant 8-bit digit
// first; stops as soon as the keys sharing the selected prefix are all taken.
//
// One histogram update per distinct digit of the warp (candidate keys share
// their leading digits, so per-key atomics would serialise on one bin).  All
// 32 lanes call it.
HS2_DEV void count_digit(int* hist, uint64_t key, bool in, uint64_t mask, uint64_t prefix,
                         int shift) {
    const int d = (in && (key & mask) == prefix) ? (int)((key >> shift) & 255) : -1;
    const unsigned grp = __match_any_sync(0xffffffffu, d);
    if (d >= 0 && lane_id() == __ffs(grp) - 1) atomicAdd(&hist[d], __popc(grp));
}

// Warp version: one warp, hist = 256 ints of shared memory owned by the warp.
template <class Get>
HS2_DEV uint64_t warp_radix_threshold(Get get, int n, int kk, int* hist) {
    const int lane = lane_id();
    uint64_t prefix = 0, mask = 0;
    int need = kk;
    for (int shift = 56; shift >= 0; shift -= 8) {
#pragma unroll
        for (int i = 0; i < 8; i++) hist[lane * 8 + i] = 0;
        __syncwarp();
        for (int i0 = 0; i0 < n; i0 += 32) {
            count_digit(hist, i0 + lane < n ? get(i0 + lane) : 0, i0 + lane < n, mask, prefix,
                        shift);
        }
        __syncwarp();
        // lane owns digits 8*lane .. 8*lane+7; suffix sums from the top digit down
        int loc[8];
        int tot = 0;
#pragma unroll
        for (int i = 7; i >= 0; i--) {
            loc[i] = hist[lane * 8 + i];
            tot += loc[i];
        }
        // inclusive suffix scan over lanes (higher lanes = higher digits)
        int suf = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += v;
        }
        int above = suf - tot;  // count of keys with digit > 8*lane+7
        int sel_digit = -1, sel_above = 0, sel_cnt = 0;
#pragma unroll
        for (int i = 7; i >= 0; i--) {
            if (sel_digit < 0 && above < need && above + loc[i] >= need) {
                sel_digit = lane * 8 + i;
                sel_above = above;
                sel_cnt = loc[i];
            }
            above += loc[i];
        }
        unsigned who = __ballot_sync(0xffffffffu, sel_digit >= 0);
        int src = __ffs(who) - 1;
        sel_digit = __shfl_sync(0xffffffffu, sel_digit, src);
        sel_above = __shfl_sync(0xffffffffu, sel_above, src);
        sel_cnt = __shfl_sync(0xffffffffu, sel_cnt, src);
        __syncwarp();
        need -= sel_above;
        prefix |= (uint64_t)sel_digit << shift;
        mask |= (uint64_t)255 << shift;
        if (sel_cnt == need) break;
    }
    return prefix;
}

// Block version (all threads of the block call it; blockDim.x multiple of 32,
// >= 256).  hist = 256 ints + 4 ints of scratch in shared memory.
template <class Get>
HS2_DEV uint64_t block_radix_threshold(Get get, int n, int kk, int* hist) {
    const int tid = threadIdx.x;
    int* sel = hist + 256;  // [digit, above, count]
    uint64_t prefix = 0, mask = 0;
    int need = kk;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += blockDim.x) {
            const int i = i0 + tid;
            count_digit(hist, i < n ? get(i) : 0, i < n, mask, prefix, shift);
        }
        __syncthreads();
        if (tid < 32) {
            const int lane = tid;
            int loc[8];
            int tot = 0;
#pragma unroll
            for (int i = 7; i >= 0; i--) {
                loc[i] = hist[lane * 8 + i];
                tot += loc[i];
            }
            int suf = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int v = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += v;
            }
            int above = suf - tot;
#pragma unroll
            for (int i = 7; i >= 0; i--) {
                if (above < need && above + loc[i] >= need) {
                    sel[0] = lane * 8 + i;
                    sel[1] = above;
                    sel[2] = loc[i];
                }
                above += loc[i];
            }
        }
        __syncthreads();
        int digit = sel[0], sab = sel[1], scnt = sel[2];
        __syncthreads();
        need -= sab;
        prefix |= (uint64_t)digit << shift;
        mask |= (uint64_t)255 << shift;
        if (scnt == need) break;
    }
    return prefix;
}

}  // namespace hs2
