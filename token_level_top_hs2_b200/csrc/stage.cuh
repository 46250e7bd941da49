// Decode step with the selected rows staged once (KV Reuse: every sparse layer
// of a hybrid block reads the same K/V rows, HySparse2 summary "How it works").
//
// stage_rows_kernel copies, per sequence, the K and V rows and the per-token
// scales that the selection names into a compact buffer, in the order of the
// idx row; entry i of the staged map is i (or -1 for padding / an index
// outside [0, length-1], which is also flagged).  The staged sequence has
// length S, so the decode sparse layers run unchanged on it with the map as
// their index row: the same rows in the same order, hence bit-identical
// outputs, read from one contiguous, L2-resident 4.9 MB block (B = 16,
// S = 1152, e4m3) instead of gathered from the whole cache each layer.
//
// Staged layout (one device buffer, 256-byte aligned parts):
//   K [B, S, D*esz], V [B, S, D*esz], sK [B, S] fp32, sV [B, S] fp32,
//   map [B, S] int32, len [B] int32 (= S).
#pragma once

#include "common.cuh"

namespace hs2 {
namespace stg {

struct Layout {
    size_t k_off, v_off, sk_off, sv_off, map_off, len_off, total;
};

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

__host__ __device__ inline Layout layout(int B, int S, int row_bytes) {
    Layout l;
    const size_t rows = (size_t)B * S;
    l.k_off = 0;
    l.v_off = round256(rows * row_bytes);
    l.sk_off = l.v_off + round256(rows * row_bytes);
    l.sv_off = l.sk_off + round256(rows * 4);
    l.map_off = l.sv_off + round256(rows * 4);
    l.len_off = l.map_off + round256(rows * 4);
    l.total = l.len_off + round256((size_t)B * 4);
    return l;
}

constexpr int kWarps = 8;

// grid (ceil(S / (kWarps * RPW)), B); a warp copies RPW rows, 16 bytes per lane
template <int ROW_BYTES>
__global__ void __launch_bounds__(kWarps * 32)
stage_rows_kernel(const uint8_t* __restrict__ kc, const uint8_t* __restrict__ vc,
                  const float* __restrict__ ks, const float* __restrict__ vs,
                  const int32_t* __restrict__ lengths, const int32_t* __restrict__ idx, int Tmax,
                  int S, uint8_t* __restrict__ staged, unsigned* __restrict__ flags) {
    constexpr int CH = ROW_BYTES / 16;   // 16-byte chunks per row
    constexpr int RPI = 32 / CH;         // rows per warp instruction
    static_assert(ROW_BYTES % 16 == 0 && 32 % CH == 0, "row size");
    griddep_launch();
    griddep_wait();  // the selection comes from the kernel before
    const int b = blockIdx.y;
    const int B = gridDim.y;
    const Layout l = layout(B, S, ROW_BYTES);
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int T = __ldg(lengths + b);
    const bool len_ok = T >= 1 && T <= Tmax;
    const int32_t* row_idx = idx + (size_t)b * S;
    const size_t base = (size_t)b * S;
    const int sub = lane / CH, ch = lane % CH;
    bool bad = false;
    const int per_cta = kWarps * RPI * 4;
    const int r0 = blockIdx.x * per_cta + warp * RPI * 4;
#pragma unroll
    for (int u = 0; u < 4; u++) {
        const int i = r0 + u * RPI + sub;
        if (i >= S) break;
        const int p = __ldg(row_idx + i);
        const bool valid = len_ok && p >= 0 && p < T;
        bad |= len_ok && (p < -1 || p >= T);
        uint4 kw = make_uint4(0u, 0u, 0u, 0u), vw = kw;
        if (valid) {
            const size_t src = ((size_t)b * Tmax + p) * ROW_BYTES + ch * 16;
            kw = __ldg(reinterpret_cast<const uint4*>(kc + src));
            vw = __ldg(reinterpret_cast<const uint4*>(vc + src));
        }
        const size_t dst = (base + i) * ROW_BYTES + ch * 16;
        *reinterpret_cast<uint4*>(staged + l.k_off + dst) = kw;
        *reinterpret_cast<uint4*>(staged + l.v_off + dst) = vw;
        if (ch == 0) {
            float sk = 0.f, sv = 0.f;
            if (valid && ks != nullptr) {
                sk = __ldg(ks + (size_t)b * Tmax + p);
                sv = __ldg(vs + (size_t)b * Tmax + p);
            }
            reinterpret_cast<float*>(staged + l.sk_off)[base + i] = sk;
            reinterpret_cast<float*>(staged + l.sv_off)[base + i] = sv;
            reinterpret_cast<int32_t*>(staged + l.map_off)[base + i] = valid ? i : -1;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0)
        reinterpret_cast<int32_t*>(staged + l.len_off)[b] = S;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(flags, FLAG_BAD_INDEX);
}

}  // namespace stg
}  // namespace hs2
