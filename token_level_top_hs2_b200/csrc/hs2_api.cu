// C ABI of the hs2 library (declared in include/hs2.h): argument validation,
// workspace layout and kernel launches.  All kernels live in the headers
// included below; this file is the library's single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>

#include <algorithm>
#include <mutex>

#include "../../include/hs2.h"
#include "decode_kernels.cuh"
#include "decode_stream.cuh"
#include "decode_pass1.cuh"
#include "decode_sketch.cuh"
#include "decode_tc.cuh"
#include "overlap.cuh"
#include "stage.cuh"
#include "prefill_tc.cuh"
#include "sparse_kernels.cuh"

using namespace hs2;

namespace {

// Device-side data flags (FLAG_* in common.cuh); one word per device.
__device__ unsigned g_device_flags;

constexpr int kMaxDevices = 64;
unsigned* g_flag_ptr[kMaxDevices];
// guards the per-device address caches (g_flag_ptr, g_noalloc_ptr): host
// threads may make their first calls on a device at the same time
std::mutex g_addr_mutex;

unsigned* device_flags() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    if (!g_flag_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_flags) != cudaSuccess) return nullptr;
        g_flag_ptr[dev] = static_cast<unsigned*>(p);
    }
    return g_flag_ptr[dev];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

hs2_status check_common(int Hq, int d, int W, int k, float scale) {
    if (!(scale > 0.f) || !isfinite(scale) || W < 1 || k < 0) return HS2_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return HS2_ERR_UNSUPPORTED;
    if (Hq != 4 && Hq != 8 && Hq != 16) return HS2_ERR_UNSUPPORTED;
    if ((long long)W + k > 2048) return HS2_ERR_UNSUPPORTED;
    return HS2_OK;
}

hs2_status check_prefill(const hs2_prefill_shape* s) {
    if (!s) return HS2_ERR_INVALID_ARG;
    if (s->B < 1 || s->L < 1 || s->B > 65535) return HS2_ERR_INVALID_ARG;
    return check_common(s->Hq, s->d, s->W, s->k, s->scale);
}

hs2_status check_decode(const hs2_decode_shape* s) {
    if (!s) return HS2_ERR_INVALID_ARG;
    if (s->B < 1 || s->Tmax < 1 || s->B > 65535) return HS2_ERR_INVALID_ARG;
    if (s->kv != HS2_KV_BF16 && s->kv != HS2_KV_E4M3) return HS2_ERR_INVALID_ARG;
    return check_common(s->Hq, s->d, s->W, s->k, s->scale);
}

hs2_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device) and
// size increase, so repeated calls -- including calls under stream capture --
// make no further attribute calls.
struct SmemLimit {
    const void* fn;
    int dev;
    size_t bytes;
};
SmemLimit g_smem_limits[512];
int g_n_smem_limits = 0;
std::mutex g_smem_mutex;

template <class K>
bool set_smem(K kernel, size_t bytes) {
    // (static + dynamic shared memory above 48 KiB needs the opt-in, so any
    // nonzero request is registered; the table makes it once per kernel/device)
    if (bytes == 0) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const void* fn = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lock(g_smem_mutex);
    SmemLimit* e = nullptr;
    for (int i = 0; i < g_n_smem_limits; i++)
        if (g_smem_limits[i].fn == fn && g_smem_limits[i].dev == dev) e = &g_smem_limits[i];
    if (e && e->bytes >= bytes) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return false;
    if (!e) {
        if (g_n_smem_limits == 512) return true;  // table full: set again next time
        e = &g_smem_limits[g_n_smem_limits++];
        e->fn = fn;
        e->dev = dev;
    }
    e->bytes = bytes;
    return true;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel of the stream drains (its prologue overlaps that
// kernel's tail); it calls griddep_wait() before reading that kernel's
// results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Check of the error path every pipelined kernel shares: one thread waits on
// an mbarrier that nothing arrives at, through the same bounded wait the
// pipelines use, with a short limit.  No copy or MMA is in flight, so the
// wait giving up leaves nothing behind; it records FLAG_TIMEOUT.
__global__ void bounded_wait_check_kernel(unsigned* __restrict__ flags, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        abort_ = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, &abort_, flags, limit_ns);
}

// Zeroes n16 16-byte words; lets the next kernel of the stream launch at once.
__global__ void zero16_kernel(uint4* __restrict__ p, int n16) {
    griddep_launch();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += gridDim.x * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// ------------------------------------------------------------ tensor maps
// cuTensorMapEncodeTiled through the runtime's driver entry point (no direct
// libcuda link).  bf16 tensors, 128-byte swizzle, 64-element inner box.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool map_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Q [B, L, Hq, D]: box of `rows` positions x 64 columns of one head.
bool map_q(CUtensorMap* m, const void* q, int B, int L, int Hq, int D, int rows) {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2,
                                   (cuuint64_t)L * Hq * D * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    return map_bf16(m, q, 4, dims, strides, box);
}

// Decode cache [B, Tmax, D] (e4m3 codes or bf16): box of 128 tokens x 128 bytes.
bool map_cache(CUtensorMap* m, const void* x, int B, int Tmax, int D, bool fp8) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int esz = fp8 ? 1 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Tmax, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)Tmax * D * esz};
    const cuuint32_t box[3] = {(cuuint32_t)(128 / esz), (cuuint32_t)dec::TOK, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void*>(x), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-token scales [B, Tmax] fp32: box of 128 tokens (needs Tmax % 4 == 0).
bool map_scales(CUtensorMap* m, const float* x, int B, int Tmax) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)Tmax, (cuuint64_t)B};
    const cuuint64_t strides[1] = {(cuuint64_t)Tmax * 4};
    const cuuint32_t box[2] = {(cuuint32_t)dec::TOK, 1};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(x), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K or V [B, L, D]: box of `rows` positions x 64 columns.
bool map_kv(CUtensorMap* m, const void* x, int B, int L, int D, int rows) {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)L * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    return map_bf16(m, x, 3, dims, strides, box);
}

// ---------------------------------------------------------------- prefill
// entries per (query row, key slice) candidate stream
int pf_cap(int k) { return (int)round_up((size_t)2 * k + 128, 32); }

struct PrefillWs {
    size_t lse_off, fail_off, fail_bytes, buf_off, total;
};
PrefillWs prefill_ws(const hs2_prefill_shape* s) {
    PrefillWs w;
    const size_t rows = (size_t)s->B * s->L;
    w.lse_off = 0;
    // per query block: the speculative selection's check failed (zeroed per call)
    w.fail_off = round_up(rows * s->Hq * sizeof(float), 256);
    w.fail_bytes = (size_t)s->B * ((s->L + tcfa::BM - 1) / tcfa::BM) * sizeof(unsigned);
    w.buf_off = round_up(w.fail_off + w.fail_bytes, 256);
    w.total = w.buf_off +
              (s->k > 0 ? rows * tcfa::kSlices * pf_cap(s->k) * sizeof(uint64_t) : 0);
    return w;
}

// Block-level selector workspace: lse (when the caller passes none), then the
// attention mass of every (row, 64-key block).
struct BlockWs {
    size_t lse_off, mass_off, nblk, total;
};
BlockWs block_ws(const hs2_prefill_shape* s) {
    BlockWs w;
    const size_t rows = (size_t)s->B * s->L;
    w.lse_off = 0;
    w.nblk = (size_t)(s->L + tcfa::kBlock - 1) / tcfa::kBlock;
    w.mass_off = round_up(rows * s->Hq * sizeof(float), 256);
    w.total = w.mass_off + rows * w.nblk * sizeof(float);
    return w;
}

template <int D>
hs2_status run_full_select(const hs2_prefill_shape* s, const void* q, const void* k,
                           const void* v, void* o, float* lse, int32_t* idx, uint8_t* ws,
                           cudaStream_t st, unsigned* flags, bool blocks = false,
                           int phases = 3, int row0 = 0, int row1 = -1) {
    // phases: 1 = exact attention (O, lse), 2 = the selection from lse;
    // query rows [row0, row1) of every sequence (row0 a multiple of 128)
    if (row1 < 0) row1 = s->L;
    const int qb0 = row0 / tcfa::BM, qb1 = (row1 + tcfa::BM - 1) / tcfa::BM;
    const PrefillWs w = prefill_ws(s);
    const BlockWs bw = block_ws(s);  // same lse area (offset 0) as the token path
    float* lse_p = lse ? lse : reinterpret_cast<float*>(ws + w.lse_off);
    const float scale2 = s->scale * kLog2e;
    if (phases & 1) {
        CUtensorMap mq, mk, mv;
        if (!map_q(&mq, q, s->B, s->L, s->Hq, D, tcfa::BM) ||
            !map_kv(&mk, k, s->B, s->L, D, tcfa::BN) || !map_kv(&mv, v, s->B, s->L, D, tcfa::BN))
            return HS2_ERR_CUDA;
        const size_t smem = tcfa::Fwd<D>::SMEM;
        auto kern = tcfa::prefill_fwd_tc_kernel<D>;
        if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
        dim3 grid(qb1 - qb0, s->Hq / 2, s->B);
        kern<<<grid, tcfa::kThreads, smem, st>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(o), lse_p,
                                                 s->L, qb1, s->Hq, scale2, flags);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    }
    if (phases & 2) {
        CUtensorMap mq, mk;
        if (!map_q(&mq, q, s->B, s->L, s->Hq, D, tcfa::BM) ||
            !map_kv(&mk, k, s->B, s->L, D, tcfa::SBN))
            return HS2_ERR_CUDA;
        const size_t smem = tcfa::Sel<D>::SMEM;
        dim3 grid(qb1 - qb0, s->B);
        if (blocks) {
            // block masses, then the choice of blocks per row
            auto kb = tcfa::prefill_select_tc_kernel<D, true>;
            if (!set_smem(kb, smem)) return HS2_ERR_CUDA;
            float* mass = reinterpret_cast<float*>(ws + bw.mass_off);
            kb<<<grid, tcfa::kSelThreads, smem, st>>>(mq, mk, lse_p, s->L, qb1, s->Hq, s->W, s->k,
                                                   s->W + s->k, 0, scale2, nullptr, idx, 0,
                                                   nullptr, nullptr, flags, mass, (int)bw.nblk);
            if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
            const long long rows = (long long)s->B * s->L;
            const long long want = (rows + tcfa::kBlkWarps - 1) / tcfa::kBlkWarps;
            const int g2 = (int)std::min<long long>(want, 148LL * 16);
            tcfa::block_select_kernel<<<g2, tcfa::kBlkWarps * 32, 0, st>>>(
                mass, s->B, s->L, s->W, s->k / tcfa::kBlock, s->W + s->k, (int)bw.nblk, idx);
            return launch_status();
        }
        auto kern = tcfa::prefill_select_tc_kernel<D>;
        if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
        unsigned* fail = reinterpret_cast<unsigned*>(ws + w.fail_off);
        uint64_t* buf = reinterpret_cast<uint64_t*>(ws + w.buf_off);
        if (cudaMemsetAsync(fail, 0, w.fail_bytes, st) != cudaSuccess) return HS2_ERR_CUDA;
        // speculative thresholds, then the exact selection for the query blocks
        // whose rows failed the check (a gated launch: the others return at once)
        kern<<<grid, tcfa::kSelThreads, smem, st>>>(mq, mk, lse_p, s->L, qb1, s->Hq, s->W, s->k,
                                                    s->W + s->k, pf_cap(s->k), scale2, buf, idx, 1,
                                                    nullptr, fail, flags, nullptr, 0);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
        kern<<<grid, tcfa::kSelThreads, smem, st>>>(mq, mk, lse_p, s->L, qb1, s->Hq, s->W, s->k,
                                                    s->W + s->k, pf_cap(s->k), scale2, buf, idx, 0,
                                                    fail, nullptr, flags, nullptr, 0);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    }
    return HS2_OK;
}

template <int D, bool FP8>
hs2_status run_sparse(const hs2_prefill_shape* s, const void* q, const void* k, const void* v,
                      const float* ks, const float* vs, const int32_t* idx, void* o,
                      cudaStream_t st, unsigned* flags) {
    constexpr int WARPS = 4;
    const int64_t n_tok = (int64_t)s->B * s->L;
    const float qk_scale = s->scale * kLog2e * (FP8 ? 256.f : 1.f);
    const int64_t blocks = (n_tok + WARPS - 1) / WARPS;
    if (blocks > 0x7fffffff) return HS2_ERR_UNSUPPORTED;
    sparse_prefill_kernel<D, FP8, WARPS><<<(unsigned)blocks, WARPS * 32, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(k),
        static_cast<const uint8_t*>(v), ks, vs, idx, static_cast<__nv_bfloat16*>(o), n_tok, s->L,
        s->Hq, s->W + s->k, qk_scale, flags);
    return launch_status();
}

// ----------------------------------------------------------------- decode
constexpr int kDecCh1 = 4096;   // pass-1 rows per CTA
constexpr int kDecCh2 = 8192;   // pass-2 rows per CTA
constexpr int kDecGroup = 8;    // chunk winners merged per CTA
constexpr int kDecWarps = 8;

struct DecodeWs {
    int n1, n2, ng;
    size_t cnt_off, lse2_off, part_off, cand_off, ccnt_off, gcand_off, gcnt_off, total;
};
DecodeWs decode_ws(const hs2_decode_shape* s) {
    DecodeWs w;
    const size_t B = s->B;
    const int kk = s->k > 0 ? s->k : 1;
    w.n1 = (s->Tmax + kDecCh1 - 1) / kDecCh1;
    w.n2 = (s->Tmax + kDecCh2 - 1) / kDecCh2;
    w.ng = (w.n2 + kDecGroup - 1) / kDecGroup;
    const size_t part_floats = (size_t)16 * s->d + 32;
    size_t off = 0;
    w.cnt_off = off;  off = round_up(off + 2 * B * sizeof(unsigned), 256);
    w.lse2_off = off; off = round_up(off + B * 16 * sizeof(float), 256);
    w.part_off = off; off = round_up(off + B * w.n1 * part_floats * sizeof(float), 256);
    w.cand_off = off; off = round_up(off + B * w.n2 * kk * sizeof(uint64_t), 256);
    w.ccnt_off = off; off = round_up(off + B * w.n2 * sizeof(int), 256);
    w.gcand_off = off; off = round_up(off + B * w.ng * kk * sizeof(uint64_t), 256);
    w.gcnt_off = off; off = round_up(off + B * w.ng * sizeof(int), 256);
    w.total = off;
    return w;
}

bool decode_streamable(const hs2_decode_shape* s);
struct DecodeWs2;
size_t decode_ws2_total(const hs2_decode_shape* s);
size_t decode_ws_bytes(const hs2_decode_shape* s) {
    return decode_streamable(s) ? decode_ws2_total(s) : decode_ws(s).total;
}

// TMA-fed decode path: usable unless e4m3 scales rows break TMA's 16-byte
// stride rule (Tmax % 4 != 0 with more than one sequence).
bool decode_streamable(const hs2_decode_shape* s) {
    return !(s->kv == HS2_KV_E4M3 && (s->Tmax % 4) != 0 && s->B > 1);
}

struct DecodeWs2 {
    int n_chunks, chunk_len, score_ld, sk_tiles;
    size_t zero_off, zero_bytes, lse2_off, part_off, score_off, bnd_off, sketch_off, rsnap_off,
        total;
};

// The sketch selection (FP8 cache, d = 128, k > 0) replaces the exact pass 2.
bool decode_uses_sketch(const hs2_decode_shape* s) {
    return s->kv == HS2_KV_E4M3 && s->d == 128 && s->k > 0;
}
DecodeWs2 decode_ws2(const hs2_decode_shape* s) {
    DecodeWs2 w;
    const size_t B = s->B;
    // at most one CTA per SM in total (a single wave), whole 128-token tiles per chunk
    const int tiles = (s->Tmax + dec::TOK - 1) / dec::TOK;
    int per_seq = 148 / s->B;
    per_seq = per_seq < 1 ? 1 : (per_seq > tiles ? tiles : per_seq);
    const int tiles_per_chunk = (tiles + per_seq - 1) / per_seq;
    w.chunk_len = tiles_per_chunk * dec::TOK;
    w.n_chunks = (s->Tmax + w.chunk_len - 1) / w.chunk_len;
    const size_t part_floats = (size_t)16 * s->d + 32;
    size_t off = 0;
    // zeroed per call: pass-1 counter, gather counter, out count, boundary count,
    // histogram; then the sketch selection's counter, arrival counter, boundary
    // count, overflow flag and histogram; then its verdict and the exact
    // fallback's arrival counter
    w.zero_off = off;
    w.zero_bytes = B * (8 + 512 + 8) * sizeof(unsigned);
    off = round_up(off + w.zero_bytes, 256);
    w.lse2_off = off;  off = round_up(off + B * 16 * sizeof(float), 256);
    w.part_off = off;  off = round_up(off + B * w.n_chunks * part_floats * sizeof(float), 256);
    w.score_ld = (s->Tmax + 3) / 4 * 4;  // 16-byte rows
    w.score_off = off; off = round_up(off + B * (size_t)w.score_ld * sizeof(float), 256);
    w.bnd_off = off;   off = round_up(off + B * dec::BCAP * sizeof(uint64_t), 256);
    w.sk_tiles = (s->Tmax + dec::TOK - 1) / dec::TOK;
    w.sketch_off = off;
    w.rsnap_off = off;
    if (decode_uses_sketch(s)) {
        off = round_up(off + B * (size_t)s->Tmax * 16, 256);
        w.rsnap_off = off;
        off = round_up(off + B * (size_t)w.sk_tiles * 16 * sizeof(float), 256);
    }
    w.total = off;
    return w;
}

size_t decode_ws2_total(const hs2_decode_shape* s) { return decode_ws2(s).total; }

template <int D, bool FP8>
hs2_status run_decode_stream(const hs2_decode_shape* s, const void* q, const void* kc,
                             const void* vc, const float* ks, const float* vs,
                             const int32_t* lengths, void* o, float* lse, int32_t* idx,
                             uint8_t* ws, cudaStream_t st, unsigned* flags) {
    using SG = dec::Stage<D, FP8>;
    const DecodeWs2 w = decode_ws2(s);
    const size_t B = s->B;
    unsigned* zero = reinterpret_cast<unsigned*>(ws + w.zero_off);
    unsigned* cnt1 = zero;
    unsigned* cnt3 = zero + B;
    unsigned* out_cnt = zero + 2 * B;
    unsigned* bnd_cnt = zero + 3 * B;
    unsigned* hist = zero + 4 * B;
    unsigned* sk_cnt = zero + 260 * B;
    unsigned* sk_arrive = zero + 261 * B;
    unsigned* verdict = zero + 520 * B;
    unsigned* ex_arrive = zero + 521 * B;
    unsigned* sk_bnd = zero + 262 * B;
    unsigned* sk_ovf = zero + 263 * B;
    unsigned* sk_hist = zero + 264 * B;
    float* lse2 = reinterpret_cast<float*>(ws + w.lse2_off);
    float* part = reinterpret_cast<float*>(ws + w.part_off);
    float* scores = reinterpret_cast<float*>(ws + w.score_off);
    uint64_t* bnd = reinterpret_cast<uint64_t*>(ws + w.bnd_off);
    const float qk_scale = s->scale * kLog2e * (FP8 ? 256.f : 1.f);
    CUtensorMap mk, mv, mks, mvs;
    if (!map_cache(&mk, kc, s->B, s->Tmax, D, FP8) || !map_cache(&mv, vc, s->B, s->Tmax, D, FP8))
        return HS2_ERR_CUDA;
    if (FP8) {
        if (!map_scales(&mks, ks, s->B, s->Tmax) || !map_scales(&mvs, vs, s->B, s->Tmax))
            return HS2_ERR_CUDA;
    } else {
        mks = mk;  // unused placeholders
        mvs = mk;
    }
    const auto* qp = static_cast<const __nv_bfloat16*>(q);
    if constexpr (FP8 && D == 128) {
        if (decode_uses_sketch(s) && w.n_chunks > 1) {
            // the sketch selection's CTAs of a sequence wait for one another:
            // the grid must be resident at once (one CTA per SM)
            int dev = 0, sms = 0;
            if (cudaGetDevice(&dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return HS2_ERR_CUDA;
            if ((long long)w.n_chunks * s->B > sms) return HS2_ERR_UNSUPPORTED;
        }
        // a chain of launches with programmatic serialisation: each kernel's
        // launch and prologue overlap the tail of the one before
        const int n16 = (int)(w.zero_bytes / 16);  // zero_bytes = B * 2112
        zero16_kernel<<<(n16 + 255) / 256, 256, 0, st>>>(reinterpret_cast<uint4*>(zero), n16);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
        // tensor-memory path: tokens as the MMA M dimension, exact f16 K/V
        const float qk2 = s->scale * kLog2e;
        using LY = dtc::P1Layout;
        const bool sketch = decode_uses_sketch(s);
        uint8_t* skt = sketch ? ws + w.sketch_off : nullptr;
        float* rsnap = reinterpret_cast<float*>(ws + w.rsnap_off);
        if (!set_smem(dtc::pass1_tc_kernel, LY::SMEM)) return HS2_ERR_CUDA;
        if (launch_pdl(dtc::pass1_tc_kernel, dim3(w.n_chunks, s->B), dim3(dtc::kP1Threads),
                       LY::SMEM, st, mk, mv, mks, mvs, qp, lengths, s->Tmax, s->Hq, w.chunk_len,
                       w.n_chunks, qk2, part, cnt1, lse2, lse, static_cast<__nv_bfloat16*>(o),
                       skt, rsnap, w.sk_tiles, flags) != cudaSuccess)
            return HS2_ERR_CUDA;
        if (sketch) {
            // one CTA per chunk, the grid of pass 1: a single wave, so that the
            // CTAs of a sequence can meet after adding their histograms; the
            // chunk's L values stay in shared memory where they fit
            static_assert(dec::BCAP * sizeof(uint64_t) >= 256 * 32 * sizeof(unsigned),
                          "the histogram columns share the key buffer");
            static_assert(dec::BCAP >= dsk::kCandCap, "a CTA's keys fit the key buffer");
            const bool lsm = dsk::select_smem_bytes(true, w.chunk_len) +
                                 sizeof(dsk::GatherShared) <= (size_t)227 * 1024;
            auto kern = lsm ? dsk::sketch_select_kernel<true> : dsk::sketch_select_kernel<false>;
            const dsk::ExactArgs ex{hist, ex_arrive, out_cnt, bnd_cnt, cnt3, verdict};
            const size_t smem = dsk::select_smem_bytes(lsm, w.chunk_len);
            if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
            if (launch_pdl(kern, dim3(w.n_chunks, s->B), dim3(dsk::kThreads), smem, st,
                           static_cast<const uint8_t*>(skt), static_cast<const float*>(rsnap),
                           w.sk_tiles, scores, w.score_ld, sk_hist, sk_arrive,
                           static_cast<const uint8_t*>(kc), ks, qp, lse2, qk2, lengths, s->Tmax,
                           s->Hq, s->W, s->k, w.chunk_len, w.n_chunks, sk_bnd, bnd, sk_ovf,
                           sk_cnt, idx, ex, flags) != cudaSuccess)
                return HS2_ERR_CUDA;
            // the kernel writes every row, through its exact fallback where
            // a sequence's candidates overflow
            return HS2_OK;
        }
    } else {
        if (cudaMemsetAsync(zero, 0, w.zero_bytes, st) != cudaSuccess) return HS2_ERR_CUDA;
        auto kern = dec::pass1_kernel<D, FP8>;
        if (!set_smem(kern, SG::SMEM1)) return HS2_ERR_CUDA;
        kern<<<dim3(w.n_chunks, s->B), dec::kThreads, SG::SMEM1, st>>>(
            mk, mv, mks, mvs, qp, lengths, s->Tmax, s->Hq, w.chunk_len, w.n_chunks, qk_scale, part,
            cnt1, lse2, lse, static_cast<__nv_bfloat16*>(o), flags);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
        if (s->k > 0) {
            auto kern2 = dec::pass2_kernel<D, FP8>;
            if (!set_smem(kern2, SG::SMEM2)) return HS2_ERR_CUDA;
            kern2<<<dim3(w.n_chunks, s->B), dec::kThreads, SG::SMEM2, st>>>(
                mk, mks, qp, lengths, s->Tmax, s->Hq, s->W, w.chunk_len, qk_scale, lse2, scores,
                w.score_ld, hist, flags);
            if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
        }
    }
    {
        const size_t smem = (size_t)dec::BCAP * sizeof(uint64_t);
        if (!set_smem(dec::gather_kernel, smem)) return HS2_ERR_CUDA;
        // waits for the kernel before at its top, whichever path launched it
        if (launch_pdl(dec::gather_kernel, dim3(w.n_chunks, s->B), dim3(256), smem, st, scores,
                       w.score_ld, static_cast<const unsigned*>(hist), lengths, s->Tmax, s->Hq,
                       s->W, s->k, w.chunk_len, w.n_chunks, out_cnt, bnd_cnt, bnd, cnt3,
                       idx) != cudaSuccess)
            return HS2_ERR_CUDA;
    }
    return HS2_OK;
}

template <int D, bool FP8>
hs2_status run_decode_select(const hs2_decode_shape* s, const void* q, const void* kc,
                             const void* vc, const float* ks, const float* vs,
                             const int32_t* lengths, void* o, float* lse, int32_t* idx,
                             uint8_t* ws, cudaStream_t st, unsigned* flags) {
    const DecodeWs w = decode_ws(s);
    unsigned* counters = reinterpret_cast<unsigned*>(ws + w.cnt_off);
    float* lse2 = reinterpret_cast<float*>(ws + w.lse2_off);
    float* part = reinterpret_cast<float*>(ws + w.part_off);
    uint64_t* cand = reinterpret_cast<uint64_t*>(ws + w.cand_off);
    int* ccnt = reinterpret_cast<int*>(ws + w.ccnt_off);
    uint64_t* gcand = reinterpret_cast<uint64_t*>(ws + w.gcand_off);
    int* gcnt = reinterpret_cast<int*>(ws + w.gcnt_off);
    const float qk_scale = s->scale * kLog2e * (FP8 ? 256.f : 1.f);
    const auto* qp = static_cast<const __nv_bfloat16*>(q);
    const auto* kp = static_cast<const uint8_t*>(kc);
    const auto* vp = static_cast<const uint8_t*>(vc);

    if (cudaMemsetAsync(counters, 0, 2 * (size_t)s->B * sizeof(unsigned), st) != cudaSuccess)
        return HS2_ERR_CUDA;
    {
        const size_t smem = (size_t)kDecWarps * DecodePart<D>::FLOATS * sizeof(float);
        auto kern = decode_pass1_kernel<D, FP8, kDecWarps>;
        if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
        kern<<<dim3(w.n1, s->B), kDecWarps * 32, smem, st>>>(
            qp, kp, vp, ks, vs, lengths, s->Tmax, s->Hq, kDecCh1, w.n1, qk_scale, part, counters,
            lse2, lse, static_cast<__nv_bfloat16*>(o), flags);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    }
    int n2 = w.n2, ng = w.ng;
    if (s->k > 0) {
        const size_t smem = (size_t)kDecCh2 * sizeof(float);
        auto kern = decode_pass2_kernel<D, FP8, kDecWarps>;
        if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
        kern<<<dim3(n2, s->B), kDecWarps * 32, smem, st>>>(qp, kp, ks, lengths, s->Tmax, s->Hq,
                                                           s->W, s->k, kDecCh2, n2, qk_scale,
                                                           lse2, cand, ccnt);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    } else {
        n2 = 0;
        ng = 1;
    }
    {
        const int kk = s->k > 0 ? s->k : 1;
        const size_t smem = ((size_t)kDecGroup * kk + kk) * sizeof(uint64_t);
        if (!set_smem(decode_merge_kernel, smem)) return HS2_ERR_CUDA;
        decode_merge_kernel<<<dim3(ng, s->B), 256, smem, st>>>(
            cand, ccnt, n2, kDecGroup, ng, s->k, s->W, s->W + s->k, lengths, s->Tmax, gcand, gcnt,
            counters + s->B, idx);
        if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    }
    return HS2_OK;
}

// Decode select: the TMA-fed streaming path, or the register path for the
// shapes TMA cannot describe.
template <int D, bool FP8>
hs2_status run_decode(const hs2_decode_shape* s, const void* q, const void* kc, const void* vc,
                      const float* ks, const float* vs, const int32_t* lengths, void* o,
                      float* lse, int32_t* idx, uint8_t* ws, cudaStream_t st, unsigned* flags) {
    if (decode_streamable(s))
        return run_decode_stream<D, FP8>(s, q, kc, vc, ks, vs, lengths, o, lse, idx, ws, st,
                                         flags);
    return run_decode_select<D, FP8>(s, q, kc, vc, ks, vs, lengths, o, lse, idx, ws, st, flags);
}

template <int D, bool FP8>
hs2_status run_decode_sparse(const hs2_decode_shape* s, const void* q, const void* kc,
                             const void* vc, const float* ks, const float* vs,
                             const int32_t* lengths, const int32_t* idx, void* o,
                             cudaStream_t st, unsigned* flags) {
    // two CTAs per SM where the registers allow it without spills (the bf16
    // d = 128 tile needs more)
    constexpr int WARPS = 6, CLUSTER = 8, MAXT = 1, MINB = (FP8 || D == 64) ? 2 : 1;
    const size_t smem = (size_t)DecodeSparseSmem<D, FP8, WARPS, CLUSTER>::FLOATS * sizeof(float);
    auto kern = decode_sparse_kernel<D, FP8, WARPS, CLUSTER, MAXT, MINB>;
    if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(s->B * CLUSTER);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CLUSTER;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the launch may overlap the previous kernel's tail (the kernel waits
    // for it before reading anything)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const float qk_scale = s->scale * kLog2e * (FP8 ? 256.f : 1.f);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(q),
                                       static_cast<const uint8_t*>(kc),
                                       static_cast<const uint8_t*>(vc), ks, vs, lengths, idx,
                                       static_cast<__nv_bfloat16*>(o), s->Tmax, s->Hq,
                                       s->W + s->k, qk_scale, flags);
    return e == cudaSuccess ? launch_status() : HS2_ERR_CUDA;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* hs2_status_string(hs2_status s) {
    switch (s) {
        case HS2_OK: return "ok";
        case HS2_ERR_INVALID_ARG: return "invalid argument";
        case HS2_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case HS2_ERR_WORKSPACE: return "workspace too small";
        case HS2_ERR_CUDA: return "CUDA error";
        case HS2_ERR_DEVICE_DATA: return "out-of-contract data met on the device";
        case HS2_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
    }
    return "unknown status";
}

int hs2_version(void) { return 100; }

size_t hs2_full_attn_select_workspace(const hs2_prefill_shape* shape) {
    if (check_prefill(shape) != HS2_OK) return 0;
    return prefill_ws(shape).total;
}

hs2_status hs2_full_attn_select(const hs2_prefill_shape* shape, const void* q, const void* k,
                                const void* v, void* o, float* lse, int32_t* idx,
                                void* workspace, size_t workspace_bytes, hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (!q || !k || !v || !o || !idx || !workspace) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(idx) ||
        !aligned16(workspace) || (lse && !aligned16(lse)))
        return HS2_ERR_INVALID_ARG;
    if ((int64_t)shape->B * shape->L > 0x7fffffffLL) return HS2_ERR_UNSUPPORTED;
    if (workspace_bytes < prefill_ws(shape).total) return HS2_ERR_WORKSPACE;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (shape->d == 128) return run_full_select<128>(shape, q, k, v, o, lse, idx, ws, st, flags);
    return run_full_select<64>(shape, q, k, v, o, lse, idx, ws, st, flags);
}

hs2_status hs2_full_attn(const hs2_prefill_shape* shape, const void* q, const void* k,
                         const void* v, void* o, float* lse, hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (!q || !k || !v || !o || !lse) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return HS2_ERR_INVALID_ARG;
    if ((int64_t)shape->B * shape->L > 0x7fffffffLL) return HS2_ERR_UNSUPPORTED;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (shape->d == 128)
        return run_full_select<128>(shape, q, k, v, o, lse, nullptr, nullptr, st, flags, false, 1);
    return run_full_select<64>(shape, q, k, v, o, lse, nullptr, nullptr, st, flags, false, 1);
}

hs2_status hs2_select(const hs2_prefill_shape* shape, const void* q, const void* k,
                      const float* lse, int32_t* idx, void* workspace, size_t workspace_bytes,
                      hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (!q || !k || !lse || !idx || !workspace) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(lse) || !aligned16(idx) ||
        !aligned16(workspace))
        return HS2_ERR_INVALID_ARG;
    if ((int64_t)shape->B * shape->L > 0x7fffffffLL) return HS2_ERR_UNSUPPORTED;
    if (workspace_bytes < prefill_ws(shape).total) return HS2_ERR_WORKSPACE;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* l = const_cast<float*>(lse);  // read only by the selection
    if (shape->d == 128)
        return run_full_select<128>(shape, q, k, nullptr, nullptr, l, idx, ws, st, flags, false, 2);
    return run_full_select<64>(shape, q, k, nullptr, nullptr, l, idx, ws, st, flags, false, 2);
}

}  // extern "C"

namespace {
// A query-row range [row0, row1) of every sequence: row0 on a 128-row query
// block boundary, row1 on one or at L.
bool rows_ok(const hs2_prefill_shape* s, int row0, int row1) {
    return row0 >= 0 && row0 < row1 && row1 <= s->L && row0 % tcfa::BM == 0 &&
           (row1 % tcfa::BM == 0 || row1 == s->L);
}
}  // namespace

extern "C" {

hs2_status hs2_full_attn_rows(const hs2_prefill_shape* shape, int row0, int row1, const void* q,
                              const void* k, const void* v, void* o, float* lse,
                              hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (!rows_ok(shape, row0, row1)) return HS2_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !lse) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return HS2_ERR_INVALID_ARG;
    if ((int64_t)shape->B * shape->L > 0x7fffffffLL) return HS2_ERR_UNSUPPORTED;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (shape->d == 128)
        return run_full_select<128>(shape, q, k, v, o, lse, nullptr, nullptr, st, flags, false, 1,
                                    row0, row1);
    return run_full_select<64>(shape, q, k, v, o, lse, nullptr, nullptr, st, flags, false, 1,
                               row0, row1);
}

hs2_status hs2_select_rows(const hs2_prefill_shape* shape, int row0, int row1, const void* q,
                           const void* k, const float* lse, int32_t* idx, void* workspace,
                           size_t workspace_bytes, hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (!rows_ok(shape, row0, row1)) return HS2_ERR_INVALID_ARG;
    if (!q || !k || !lse || !idx || !workspace) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(lse) || !aligned16(idx) ||
        !aligned16(workspace))
        return HS2_ERR_INVALID_ARG;
    if ((int64_t)shape->B * shape->L > 0x7fffffffLL) return HS2_ERR_UNSUPPORTED;
    if (workspace_bytes < prefill_ws(shape).total) return HS2_ERR_WORKSPACE;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* l = const_cast<float*>(lse);  // read only by the selection
    if (shape->d == 128)
        return run_full_select<128>(shape, q, k, nullptr, nullptr, l, idx, ws, st, flags, false, 2,
                                    row0, row1);
    return run_full_select<64>(shape, q, k, nullptr, nullptr, l, idx, ws, st, flags, false, 2,
                               row0, row1);
}

size_t hs2_full_attn_select_blocks_workspace(const hs2_prefill_shape* shape, int block) {
    if (check_prefill(shape) != HS2_OK || block != tcfa::kBlock) return 0;
    return block_ws(shape).total;
}

hs2_status hs2_full_attn_select_blocks(const hs2_prefill_shape* shape, int block, const void* q,
                                       const void* k, const void* v, void* o, float* lse,
                                       int32_t* idx, void* workspace, size_t workspace_bytes,
                                       hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (block != tcfa::kBlock) return HS2_ERR_UNSUPPORTED;
    if (shape->k < block || shape->k % block != 0) return HS2_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !idx || !workspace) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(idx) ||
        !aligned16(workspace) || (lse && !aligned16(lse)))
        return HS2_ERR_INVALID_ARG;
    if ((int64_t)shape->B * shape->L > 0x7fffffffLL) return HS2_ERR_UNSUPPORTED;
    if (workspace_bytes < block_ws(shape).total) return HS2_ERR_WORKSPACE;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (shape->d == 128)
        return run_full_select<128>(shape, q, k, v, o, lse, idx, ws, st, flags, true);
    return run_full_select<64>(shape, q, k, v, o, lse, idx, ws, st, flags, true);
}

hs2_status hs2_sparse_attn(const hs2_prefill_shape* shape, const void* q, const void* k,
                           const void* v, hs2_kv_dtype kv, const float* k_scale,
                           const float* v_scale, const int32_t* idx, void* o,
                           hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (kv != HS2_KV_BF16 && kv != HS2_KV_E4M3) return HS2_ERR_INVALID_ARG;
    if (!q || !k || !v || !o || !idx) return HS2_ERR_INVALID_ARG;
    if (kv == HS2_KV_E4M3 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(idx))
        return HS2_ERR_INVALID_ARG;
    if (kv == HS2_KV_E4M3 && shape->d != 128) return HS2_ERR_UNSUPPORTED;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (kv == HS2_KV_E4M3)
        return run_sparse<128, true>(shape, q, k, v, k_scale, v_scale, idx, o, st, flags);
    if (shape->d == 128)
        return run_sparse<128, false>(shape, q, k, v, nullptr, nullptr, idx, o, st, flags);
    return run_sparse<64, false>(shape, q, k, v, nullptr, nullptr, idx, o, st, flags);
}

size_t hs2_decode_select_workspace(const hs2_decode_shape* shape) {
    if (check_decode(shape) != HS2_OK) return 0;
    return decode_ws_bytes(shape);
}

hs2_status hs2_decode_select(const hs2_decode_shape* shape, const void* q, const void* k_cache,
                             const void* v_cache, const float* k_scale, const float* v_scale,
                             const int32_t* lengths, void* o, float* lse, int32_t* idx,
                             void* workspace, size_t workspace_bytes, hs2_stream_t stream) {
    hs2_status e = check_decode(shape);
    if (e != HS2_OK) return e;
    if (!q || !k_cache || !v_cache || !lengths || !o || !idx || !workspace)
        return HS2_ERR_INVALID_ARG;
    const bool fp8 = shape->kv == HS2_KV_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned16(idx) || !aligned16(workspace) || (lse && !aligned16(lse)))
        return HS2_ERR_INVALID_ARG;
    if (fp8 && shape->d != 128) return HS2_ERR_UNSUPPORTED;
    if (workspace_bytes < decode_ws_bytes(shape)) return HS2_ERR_WORKSPACE;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (fp8)
        return run_decode<128, true>(shape, q, k_cache, v_cache, k_scale, v_scale, lengths,
                                            o, lse, idx, ws, st, flags);
    if (shape->d == 128)
        return run_decode<128, false>(shape, q, k_cache, v_cache, nullptr, nullptr,
                                             lengths, o, lse, idx, ws, st, flags);
    return run_decode<64, false>(shape, q, k_cache, v_cache, nullptr, nullptr, lengths, o,
                                        lse, idx, ws, st, flags);
}

hs2_status hs2_decode_sparse(const hs2_decode_shape* shape, const void* q, const void* k_cache,
                             const void* v_cache, const float* k_scale, const float* v_scale,
                             const int32_t* lengths, const int32_t* idx, void* o,
                             hs2_stream_t stream) {
    hs2_status e = check_decode(shape);
    if (e != HS2_OK) return e;
    if (!q || !k_cache || !v_cache || !lengths || !idx || !o) return HS2_ERR_INVALID_ARG;
    const bool fp8 = shape->kv == HS2_KV_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned16(idx))
        return HS2_ERR_INVALID_ARG;
    if (fp8 && shape->d != 128) return HS2_ERR_UNSUPPORTED;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (fp8)
        return run_decode_sparse<128, true>(shape, q, k_cache, v_cache, k_scale, v_scale, lengths,
                                            idx, o, st, flags);
    if (shape->d == 128)
        return run_decode_sparse<128, false>(shape, q, k_cache, v_cache, nullptr, nullptr,
                                             lengths, idx, o, st, flags);
    return run_decode_sparse<64, false>(shape, q, k_cache, v_cache, nullptr, nullptr, lengths,
                                        idx, o, st, flags);
}

size_t hs2_decode_stage_workspace(const hs2_decode_shape* shape) {
    if (check_decode(shape) != HS2_OK) return 0;
    const int esz = shape->kv == HS2_KV_E4M3 ? 1 : 2;
    return stg::layout(shape->B, shape->W + shape->k, shape->d * esz).total;
}

hs2_status hs2_decode_stage(const hs2_decode_shape* shape, const void* k_cache,
                            const void* v_cache, const float* k_scale, const float* v_scale,
                            const int32_t* lengths, const int32_t* idx, void* staged,
                            size_t staged_bytes, hs2_stream_t stream) {
    hs2_status e = check_decode(shape);
    if (e != HS2_OK) return e;
    const bool fp8 = shape->kv == HS2_KV_E4M3;
    if (!k_cache || !v_cache || !lengths || !idx || !staged) return HS2_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(staged))
        return HS2_ERR_INVALID_ARG;
    if (staged_bytes < hs2_decode_stage_workspace(shape)) return HS2_ERR_WORKSPACE;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int S = shape->W + shape->k;
    const int row_bytes = shape->d * (fp8 ? 1 : 2);
    const auto* kc = static_cast<const uint8_t*>(k_cache);
    const auto* vc = static_cast<const uint8_t*>(v_cache);
    auto* out = static_cast<uint8_t*>(staged);
    const float* ks = fp8 ? k_scale : nullptr;
    const float* vs = fp8 ? v_scale : nullptr;
    if (row_bytes == 128) {
        const int per_cta = stg::kWarps * (32 / 8) * 4;
        dim3 grid((S + per_cta - 1) / per_cta, shape->B);
        if (launch_pdl(stg::stage_rows_kernel<128>, grid, dim3(stg::kWarps * 32), 0, st, kc, vc,
                       ks, vs, lengths, idx, shape->Tmax, S, out, flags) != cudaSuccess)
            return HS2_ERR_CUDA;
    } else {
        const int per_cta = stg::kWarps * (32 / 16) * 4;
        dim3 grid((S + per_cta - 1) / per_cta, shape->B);
        if (launch_pdl(stg::stage_rows_kernel<256>, grid, dim3(stg::kWarps * 32), 0, st, kc, vc,
                       ks, vs, lengths, idx, shape->Tmax, S, out, flags) != cudaSuccess)
            return HS2_ERR_CUDA;
    }
    return launch_status();
}

hs2_status hs2_decode_sparse_staged(const hs2_decode_shape* shape, const void* q,
                                    const void* staged, void* o, hs2_stream_t stream) {
    hs2_status e = check_decode(shape);
    if (e != HS2_OK) return e;
    if (!q || !staged || !o) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(staged) || !aligned16(o)) return HS2_ERR_INVALID_ARG;
    const bool fp8 = shape->kv == HS2_KV_E4M3;
    if (fp8 && shape->d != 128) return HS2_ERR_UNSUPPORTED;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int S = shape->W + shape->k;
    const stg::Layout l = stg::layout(shape->B, S, shape->d * (fp8 ? 1 : 2));
    const auto* base = static_cast<const uint8_t*>(staged);
    // the staged rows are a cache of S rows per sequence, the map its index row
    hs2_decode_shape s2 = *shape;
    s2.Tmax = S;
    const void* kc = base + l.k_off;
    const void* vc = base + l.v_off;
    const float* ks = reinterpret_cast<const float*>(base + l.sk_off);
    const float* vs = reinterpret_cast<const float*>(base + l.sv_off);
    const auto* map = reinterpret_cast<const int32_t*>(base + l.map_off);
    const auto* len = reinterpret_cast<const int32_t*>(base + l.len_off);
    if (fp8) return run_decode_sparse<128, true>(&s2, q, kc, vc, ks, vs, len, map, o, st, flags);
    if (shape->d == 128)
        return run_decode_sparse<128, false>(&s2, q, kc, vc, nullptr, nullptr, len, map, o, st,
                                             flags);
    return run_decode_sparse<64, false>(&s2, q, kc, vc, nullptr, nullptr, len, map, o, st, flags);
}

hs2_status hs2_selection_overlap(const hs2_prefill_shape* shape, const int32_t* idx_a,
                                 const int32_t* idx_b, int32_t* inter, float* ratio,
                                 hs2_stream_t stream) {
    hs2_status e = check_prefill(shape);
    if (e != HS2_OK) return e;
    if (!idx_a || !idx_b || (!inter && !ratio)) return HS2_ERR_INVALID_ARG;
    if (!aligned16(idx_a) || !aligned16(idx_b) || (inter && !aligned16(inter)) ||
        (ratio && !aligned16(ratio)))
        return HS2_ERR_INVALID_ARG;
    if (shape->L >= (1 << ovl::kPosBits) - 1) return HS2_ERR_UNSUPPORTED;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long rows = (long long)shape->B * shape->L;
    const bool use_bitmap = shape->L <= ovl::kBitmapMaxL;
    auto kern = use_bitmap ? ovl::overlap_bitmap_kernel : ovl::overlap_kernel;
    const size_t smem = use_bitmap ? ovl::bitmap_smem_bytes(shape->W + shape->k, shape->L)
                                   : ovl::smem_bytes(shape->W + shape->k, shape->k);
    if (!set_smem(kern, smem)) return HS2_ERR_CUDA;
    // per warp a bitmap (or hash set) and two stages of both rows; each warp
    // walks many rows
    const size_t per_sm_smem = 228 * 1024;  // shared memory of one SM (1 KB per CTA reserved)
    const long long per_sm = std::max<long long>(1, (long long)(per_sm_smem / (smem + 1024)));
    const long long want = (rows + ovl::kWarps - 1) / ovl::kWarps;
    const int grid = (int)std::min<long long>(want, per_sm * sms);
    kern<<<grid, ovl::kWarps * 32, smem, st>>>(idx_a, idx_b, shape->B, shape->L, shape->W + shape->k,
                                               shape->W, shape->k, inter, ratio, flags);
    return launch_status();
}

hs2_status hs2_check_bounded_wait(unsigned limit_us, hs2_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return HS2_ERR_INVALID_ARG;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    bounded_wait_check_kernel<<<1, 32, 0, st>>>(flags, (uint64_t)limit_us * 1000ull);
    return launch_status();
}

hs2_status hs2_get_last_device_error(hs2_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return HS2_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return HS2_ERR_CUDA;
    unsigned host = 0;
    if (cudaMemcpyFromSymbol(&host, g_device_flags, sizeof host) != cudaSuccess)
        return HS2_ERR_CUDA;
    if (host) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_device_flags, &zero, sizeof zero) != cudaSuccess)
            return HS2_ERR_CUDA;
        return (host & FLAG_TIMEOUT) ? HS2_ERR_TIMEOUT : HS2_ERR_DEVICE_DATA;
    }
    return HS2_OK;
}

}  // extern "C"

// ====================================================== no-allocation variant
// hs2_decode_select_noalloc: decode select whose workspace is a fixed
// file-scope device array instead of caller memory, for hosts that cannot
// allocate device memory (see include/hs2.h).
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HS2_NOALLOC_SCRATCH_BYTES];

uint8_t* g_noalloc_ptr[kMaxDevices];

// Device address of the scratch on the current device, looked up once per
// device.  In host code g_noalloc_scratch names a host-side stand-in, never
// the device memory, so only this address may be handed to kernels.
uint8_t* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    if (!g_noalloc_ptr[dev]) {
        uint8_t* ptr = nullptr;
        if (cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" hs2_status hs2_decode_select_noalloc(const hs2_decode_shape* shape, const void* q,
                                                const void* k_cache, const void* v_cache,
                                                const float* k_scale, const float* v_scale,
                                                const int32_t* lengths, void* o, float* lse,
                                                int32_t* idx, hs2_stream_t stream) {
    hs2_status e = check_decode(shape);
    if (e != HS2_OK) return e;
    if (!q || !k_cache || !v_cache || !lengths || !o || !idx) return HS2_ERR_INVALID_ARG;
    const bool fp8 = shape->kv == HS2_KV_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return HS2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
        !aligned16(idx) || (lse && !aligned16(lse)))
        return HS2_ERR_INVALID_ARG;
    if (fp8 && shape->d != 128) return HS2_ERR_UNSUPPORTED;
    // the whole workspace layout of hs2_decode_select must fit the fixed scratch
    if (decode_ws_bytes(shape) > (size_t)HS2_NOALLOC_SCRATCH_BYTES) return HS2_ERR_WORKSPACE;
    uint8_t* ws = noalloc_scratch();
    if (!ws) return HS2_ERR_CUDA;
    unsigned* flags = device_flags();
    if (!flags) return HS2_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // run_decode_select clears the per-call counters at the start of every call
    if (fp8)
        return run_decode<128, true>(shape, q, k_cache, v_cache, k_scale, v_scale, lengths,
                                            o, lse, idx, ws, st, flags);
    if (shape->d == 128)
        return run_decode<128, false>(shape, q, k_cache, v_cache, nullptr, nullptr,
                                             lengths, o, lse, idx, ws, st, flags);
    return run_decode<64, false>(shape, q, k_cache, v_cache, nullptr, nullptr, lengths, o,
                                        lse, idx, ws, st, flags);
}
