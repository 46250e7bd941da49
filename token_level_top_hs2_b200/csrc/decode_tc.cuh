// Decode on the 5th-generation tensor cores (e4m3 cache, d = 128): pieces
// of the decode pass 1 (decode_pass1.cuh).
//
// The cached TOKENS are the MMA M dimension, so one 128-token tile is one
// tcgen05 MMA: S^T[token][head] = K_tile (128 x 128, f16, in TMEM) *
// Q^T (128 x 16, f16).  e4m3 codes become exact f16 values (converter warps
// write them straight into TMEM, the A operand), so the per-token scales stay
// in fp32: the logit of token s is multiplied by k_scale[s] afterwards.
#pragma once

#include "decode_stream.cuh"

namespace hs2 {
namespace dtc {

using namespace hs2::tc;

constexpr int TOK = 128;
constexpr float kLazy = 8.f;
// Softmax reference offset: probabilities are formed against R = max - kSk,
// so 2^(x - R) lies in (0, 2^14] and its f16 value keeps 3 mantissa bits down
// to 2^-14 before going subnormal (the sketch's 8-bit code range).
constexpr float kSk = 6.f;

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

}  // namespace dtc
}  // namespace hs2
