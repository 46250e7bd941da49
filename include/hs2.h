/*
 * hs2.h -- C ABI of a B200 (sm_100a) library for HySparse2's token-level
 * KV Reuse hot path.
 *
 * The method (HySparse2 summary, onedev.kr/papers/146):
 *   - "What differs": a full-attention layer computes exact attention and, per
 *     query token, selects individual tokens: the recent-token window is always
 *     taken first, then the highest-scoring tokens outside it.  The sparse
 *     layers that follow reuse the selected tokens' KV entries.
 *   - "How it works": inside a hybrid block the sparse layers reuse the full
 *     layer's KV cache and selection indices unchanged (KV Reuse).
 *   - "How to use": one shared KV head (MQA), no positional encoding in full
 *     or sparse attention, W = 128 forced local tokens plus k = 1,024 global
 *     tokens; efficiency quoted on an FP8 KV cache.
 * Readings of what the page leaves open:
 *   - score(t,s) = sum over the Hq query heads of softmax probability
 *     exp(l_h(t,s) - lse_h(t)), l_h(t,s) = scale * <q_{t,h}, k_s>;
 *   - window = positions max(0,t-W+1)..t (the query itself included);
 *   - global candidates = positions 0..t-W; the k best by (score descending,
 *     position ascending); all of them when there are at most k;
 *   - the full layer's own output is full causal attention;
 *   - decode: the new token sits at position T-1 of a cache of length T that
 *     already holds its K/V;
 *   - FP8 KV: x = scale_row * e4m3(code), one fp32 scale per token for K and
 *     one for V.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, row-major, last dim contiguous,
 *     16-byte aligned.  The caller owns every buffer; the library allocates,
 *     frees and synchronises nothing (hs2_get_last_device_error excepted).
 *   - Every call is asynchronous on `stream`.  Arguments are validated on the
 *     host before anything is launched; on failure a non-zero status is
 *     returned and no kernel runs.  Launch failures map to HS2_ERR_CUDA.
 *   - Supported: head dim d in {64, 128}; Hq in {4, 8, 16} query heads sharing
 *     one KV head; W >= 1, k >= 0, W + k <= 2048; scale finite and > 0.
 *   - Index output format (`idx`, W+k int32 per query): the window positions
 *     ascending first, then the global picks in no particular order, then -1
 *     padding.  |selection| = min(t+1, W+k).  Treat it as a set.
 *   - Device-side data checks (decode lengths outside [1, Tmax], a query value
 *     beyond the fp16 range +-65504 or a V scale above 255 on an e4m3 path, an
 *     index outside [0, t])
 *     do not fault: the kernel skips the offending work and records a flag that
 *     hs2_get_last_device_error reports as HS2_ERR_DEVICE_DATA.
 */
#ifndef HS2_H
#define HS2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* hs2_stream_t;

typedef enum {
    HS2_OK = 0,
    HS2_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size, bad scale */
    HS2_ERR_UNSUPPORTED = 2,  /* valid but not implemented (d, Hq, W+k, dtype) */
    HS2_ERR_WORKSPACE = 3,    /* workspace smaller than the *_workspace() size */
    HS2_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
    HS2_ERR_DEVICE_DATA = 5,  /* a kernel met out-of-contract data (see above) */
    HS2_ERR_TIMEOUT = 6       /* a bounded in-kernel wait gave up; results invalid */
} hs2_status;

typedef enum { HS2_KV_BF16 = 0, HS2_KV_E4M3 = 1 } hs2_kv_dtype;

/* Prefill shape: B sequences of L tokens, Hq query heads, one KV head. */
typedef struct {
    int B, L, Hq, d, W, k;
    float scale; /* softmax scale, normally 1/sqrt(d) */
} hs2_prefill_shape;

/* Decode shape: B sequences, caches of Tmax rows, one query token each. */
typedef struct {
    int B, Tmax, Hq, d, W, k;
    float scale;
    hs2_kv_dtype kv;
} hs2_decode_shape;

/* Human-readable name of a status code (static string). */
const char* hs2_status_string(hs2_status s);

/* Library version, major*10000 + minor*100 + patch. */
int hs2_version(void);

/*
 * Bytes of device workspace hs2_full_attn_select needs for `shape`
 * (0 for an invalid shape): the lse (when the caller passes none), one flag
 * word per 128-row query block, and per query row four candidate streams of
 * round_up(2k+128, 32) 8-byte (score, position) keys.
 */
size_t hs2_full_attn_select_workspace(const hs2_prefill_shape* shape);

/*
 * Full-attention layer with token selection (prefill).
 * Defined by the "What differs" section of the HySparse2 summary: exact causal
 * attention whose scores select, per query token, the window plus the top-k
 * older tokens.
 *   q   [B, L, Hq, d] bf16      queries
 *   k,v [B, L, d]     bf16      the layer's single KV head (the cache the sparse
 *                               layers reuse)
 *   o   [B, L, Hq, d] bf16      out: full causal attention output
 *   lse [B, L, Hq]    fp32      out: natural-log log-sum-exp of the scaled
 *                               logits per (token, head); may be NULL
 *   idx [B, L, W+k]   int32     out: selection, format above
 *   workspace: device buffer of at least hs2_full_attn_select_workspace()
 *   bytes; contents need no initialisation and are garbage afterwards.
 * Calls on the same workspace must not overlap in time.
 */
hs2_status hs2_full_attn_select(const hs2_prefill_shape* shape, const void* q, const void* k,
                                const void* v, void* o, float* lse, int32_t* idx,
                                void* workspace, size_t workspace_bytes, hs2_stream_t stream);

/*
 * The two halves of hs2_full_attn_select, for callers that use the full
 * layer's output before its selection is done (O and lse are final when
 * hs2_full_attn returns on the stream; the selection then runs from q, k and
 * lse): e.g. the next layer, or the copy of O to the host, overlaps the
 * selection on another stream.  Results equal hs2_full_attn_select's.
 *   hs2_full_attn: q, k, v, o as hs2_full_attn_select; lse [B, L, Hq] fp32 out
 *     (required here).
 *   hs2_select: q, k and the lse hs2_full_attn wrote; idx out; workspace of at
 *     least hs2_full_attn_select_workspace() bytes.
 */
hs2_status hs2_full_attn(const hs2_prefill_shape* shape, const void* q, const void* k,
                         const void* v, void* o, float* lse, hs2_stream_t stream);
hs2_status hs2_select(const hs2_prefill_shape* shape, const void* q, const void* k,
                      const float* lse, int32_t* idx, void* workspace, size_t workspace_bytes,
                      hs2_stream_t stream);

/*
 * hs2_full_attn and hs2_select for the query rows [row0, row1) of every
 * sequence only (same "What differs" computation, restricted to those rows):
 * row0 a multiple of 128, row1 a multiple of 128 or L, 0 <= row0 < row1 <= L.
 * A query row t reads only K/V rows 0..t, so these calls read K and V rows
 * 0..row1-1, q rows [row0, row1) and (hs2_select_rows) lse rows [row0, row1),
 * and write o, lse or idx rows [row0, row1) only; the tensors keep their
 * full [B, L, ...] shapes.  Results equal those rows of the full calls.  A
 * caller streaming a long prompt in can run the rows that have arrived while
 * the rest is still being copied, and copy finished rows out while later ones
 * compute.  The same workspace size as hs2_full_attn_select; calls on one
 * workspace must not overlap in time.
 */
hs2_status hs2_full_attn_rows(const hs2_prefill_shape* shape, int row0, int row1, const void* q,
                              const void* k, const void* v, void* o, float* lse,
                              hs2_stream_t stream);
hs2_status hs2_select_rows(const hs2_prefill_shape* shape, int row0, int row1, const void* q,
                           const void* k, const float* lse, int32_t* idx, void* workspace,
                           size_t workspace_bytes, hs2_stream_t stream);

/*
 * Block-level selector variant: the full layer of HySparse, the predecessor
 * the HySparse2 summary compares against ("Limits": 64-token blocks, 1,024
 * global tokens, a separate 128-token local window).  Same exact attention
 * (o, lse) as hs2_full_attn_select; the selection takes whole blocks:
 *   - blocks are the aligned `block`-token ranges [block*j, block*j+block-1];
 *   - a block is a candidate if it holds a position <= t - W; its attention
 *     mass is the sum of score(t,s) over its positions s <= t - W (the
 *     head-summed probability, as for the token selector);
 *   - the k / block candidate blocks of largest mass are chosen, ties to the
 *     lower block, all of them when there are at most k / block;
 *   - idx row: the window ascending, then the positions <= t - W of the chosen
 *     blocks (ascending block order), then -1.  Same [B, L, W+k] format, so
 *     hs2_sparse_attn consumes it unchanged.
 * block must be 64; k a positive multiple of it.  The workspace holds the lse
 * (when lse is NULL) and one fp32 mass per (row, block): 4 * B * L * ceil(L/64)
 * bytes, 1 GiB at L = 128k.
 */
size_t hs2_full_attn_select_blocks_workspace(const hs2_prefill_shape* shape, int block);
hs2_status hs2_full_attn_select_blocks(const hs2_prefill_shape* shape, int block, const void* q,
                                       const void* k, const void* v, void* o, float* lse,
                                       int32_t* idx, void* workspace, size_t workspace_bytes,
                                       hs2_stream_t stream);

/*
 * Sparse layer (prefill): each query token attends, with its own queries, only
 * to the K/V rows its inherited index set names (KV Reuse, "How it works").
 *   q   [B, L, Hq, d] bf16      this sparse layer's queries
 *   k,v [B, L, d]               the full layer's cache: bf16, or e4m3 codes (one
 *                               byte each) when kv == HS2_KV_E4M3
 *   k_scale, v_scale [B, L] fp32  per-token scales for e4m3 (NULL for bf16)
 *   idx [B, L, S] int32, S = shape->W + shape->k: per token a set of positions
 *                               in [0, t], -1 entries ignored, no repeats
 *   o   [B, L, Hq, d] bf16      out; a token whose set is empty gets zeros
 * e4m3 additionally needs |q| <= 65504 and per-token V scales <= 255.
 */
hs2_status hs2_sparse_attn(const hs2_prefill_shape* shape, const void* q, const void* k,
                           const void* v, hs2_kv_dtype kv, const float* k_scale,
                           const float* v_scale, const int32_t* idx, void* o,
                           hs2_stream_t stream);

/*
 * Bytes of device workspace hs2_decode_select needs (0 for an invalid shape).
 */
size_t hs2_decode_select_workspace(const hs2_decode_shape* shape);

/*
 * Decode full layer with selection: one new query per sequence at position
 * t = lengths[b]-1; exact attention over cache rows 0..t, and per query the
 * recent-token window first, then the highest-scoring tokens outside it
 * (HySparse2 summary, "What differs": token-level selection from exact
 * attention scores), on the FP8 KV cache the "How to use" section quotes
 * from 1k to 1M tokens.  Split over the cache length (split-KV).
 *   q        [B, Hq, d] bf16
 *   k_cache, v_cache [B, Tmax, d]  e4m3 codes (kv == HS2_KV_E4M3) or bf16
 *   k_scale, v_scale [B, Tmax] fp32 (e4m3 only; NULL for bf16)
 *   lengths  [B] int32, device, each in [1, Tmax]
 *   o        [B, Hq, d] bf16  out: full attention output
 *   lse      [B, Hq] fp32     out, may be NULL
 *   idx      [B, W+k] int32   out: selection, format above
 *   workspace: >= hs2_decode_select_workspace() bytes, no initialisation
 *   needed; calls on the same workspace must not overlap in time.
 * With the e4m3 cache at d = 128 the cache is split into chunks of whole
 * 128-token tiles, at most one per SM (n_chunks = ceil(Tmax / chunk) with
 * n_chunks * B <= 148), and the CTAs of a sequence wait for one another
 * (bounded waits) in the selection: when a sequence spans several chunks the
 * call returns HS2_ERR_UNSUPPORTED on a device with fewer SMs than
 * n_chunks * B, before any kernel runs.
 */
hs2_status hs2_decode_select(const hs2_decode_shape* shape, const void* q, const void* k_cache,
                             const void* v_cache, const float* k_scale, const float* v_scale,
                             const int32_t* lengths, void* o, float* lse, int32_t* idx,
                             void* workspace, size_t workspace_bytes, hs2_stream_t stream);

/*
 * Decode sparse layer: sequence b's query attends to the cache rows idx[b]
 * names -- the sparse layers of a hybrid block reuse the full layer's KV
 * cache and its token selection unchanged (HySparse2 summary, "How it works",
 * KV Reuse; "What differs": the sparse layers attend to the tokens the full
 * layer selected).
 *   q [B, Hq, d] bf16; caches/scales as hs2_decode_select; idx [B, W+k] int32
 *   with entries in [0, lengths[b]-1] or -1; o [B, Hq, d] bf16 out.
 */
hs2_status hs2_decode_sparse(const hs2_decode_shape* shape, const void* q, const void* k_cache,
                             const void* v_cache, const float* k_scale, const float* v_scale,
                             const int32_t* lengths, const int32_t* idx, void* o,
                             hs2_stream_t stream);

/*
 * Cross-layer selection overlap: how far two selections of the same shape
 * pick the same global tokens.  The IndexCache page (Appendix A,
 * "Cross-Layer Top-(k) Index Overlap") compares layers by |T(i) ∩ T(j)| / k of
 * their top-k sets; here T is the set of global picks of a query row, the
 * entries s of its idx row with 0 <= s <= t - W (window entries and -1
 * padding are not part of it).  Typical use: idx_a = the selection a sparse
 * layer inherits from its full layer, idx_b = the exact selection that layer's
 * own queries give (hs2_full_attn_select with them).
 *   shape                 B, L, W, k of both idx tensors (Hq, d, scale are
 *                         checked as for the other prefill calls but unused);
 *                         L < 2^21 - 1
 *   idx_a, idx_b [B, L, W+k] int32   selections in the hs2_full_attn_select
 *                         format (any slot order); entries outside [-1, t]
 *                         are skipped and flagged as HS2_ERR_DEVICE_DATA
 *   inter [B, L] int32    out: |T_a(t) ∩ T_b(t)| (may be NULL)
 *   ratio [B, L] fp32     out: inter / min(k, t - W + 1); 1 for rows without
 *                         global candidates (t < W or k = 0) (may be NULL)
 * At least one of inter, ratio must be given.  Exact integer counting: the
 * ratio is one correctly rounded fp32 division.
 */
hs2_status hs2_selection_overlap(const hs2_prefill_shape* shape, const int32_t* idx_a,
                                 const int32_t* idx_b, int32_t* inter, float* ratio,
                                 hs2_stream_t stream);

/*
 * Decode step with the selected rows staged once.  Every sparse layer of a
 * hybrid block reads the K/V rows its full layer selected (KV Reuse, "How it
 * works"); hs2_decode_stage copies them, per sequence and in idx order, into
 * a compact buffer, and hs2_decode_sparse_staged runs a decode sparse layer
 * on it.  Results are bit-identical to hs2_decode_sparse with the same idx.
 *   hs2_decode_stage_workspace: bytes of the staged buffer for `shape`
 *     (B * (W+k) * (2 * d * esz + 12) plus alignment; 4.9 MB at B = 16,
 *     W + k = 1152, e4m3).
 *   hs2_decode_stage: caches, scales and lengths as hs2_decode_select;
 *     idx [B, W+k] as it returns (entries in [0, lengths[b]-1] or -1; others
 *     are skipped and flagged as HS2_ERR_DEVICE_DATA); staged: out.
 *   hs2_decode_sparse_staged: q [B, Hq, d] bf16 of one sparse layer, the
 *     staged buffer, o [B, Hq, d] bf16 out.  Any number of layers may reuse
 *     one staged buffer.
 */
size_t hs2_decode_stage_workspace(const hs2_decode_shape* shape);
hs2_status hs2_decode_stage(const hs2_decode_shape* shape, const void* k_cache,
                            const void* v_cache, const float* k_scale, const float* v_scale,
                            const int32_t* lengths, const int32_t* idx, void* staged,
                            size_t staged_bytes, hs2_stream_t stream);
hs2_status hs2_decode_sparse_staged(const hs2_decode_shape* shape, const void* q,
                                    const void* staged, void* o, hs2_stream_t stream);

/* Size of the fixed device scratch used by hs2_decode_select_noalloc. */
#define HS2_NOALLOC_SCRATCH_BYTES (96u << 20)

/*
 * hs2_decode_select_noalloc: hs2_decode_select for callers that cannot
 * allocate device memory.  The paper has no counterpart; this is a deployment
 * convenience of this library.
 *
 * Some hosts own every byte of device memory: an inference server that
 * reserves nearly all HBM for its KV-cache pool up front, a plugin whose host
 * application exposes no allocator, or a latency-critical loop in which a
 * cudaMalloc (which can synchronise the device) is not allowed.  Such callers
 * cannot provide the workspace hs2_decode_select needs.  This entry point
 * takes the same arguments minus the workspace and uses a fixed scratch area
 * of HS2_NOALLOC_SCRATCH_BYTES that the library keeps in device memory
 * (a file-scope __device__ array).  It allocates and frees nothing.
 *
 * Limits and behaviour:
 *   - shapes whose hs2_decode_select_workspace() exceeds
 *     HS2_NOALLOC_SCRATCH_BYTES are rejected with HS2_ERR_WORKSPACE before
 *     anything is launched (B=16 x 256k and B=4 x 1M tokens fit);
 *   - every GPU that loads the library holds the scratch until the process
 *     exits;
 *   - the first call on a device looks up the scratch address on that device
 *     (it must be the current device); make that first call before any stream
 *     capture;
 *   - all calls on a device share the one scratch area and it keeps the last
 *     call's contents (the parts that must start at zero are cleared by every
 *     call), so calls whose execution overlaps on the GPU -- e.g. on two
 *     streams without ordering -- race and give wrong results.  Serialise them.
 * Results equal hs2_decode_select's for the same inputs.
 */
hs2_status hs2_decode_select_noalloc(const hs2_decode_shape* shape, const void* q,
                                     const void* k_cache, const void* v_cache,
                                     const float* k_scale, const float* v_scale,
                                     const int32_t* lengths, void* o, float* lse, int32_t* idx,
                                     hs2_stream_t stream);

/*
 * hs2_check_bounded_wait: a check of the library's own error path, with no
 * counterpart in the pages.  Every pipelined kernel waits on its pipeline
 * stages with a time limit and, when a wait gives up, records a timeout flag
 * and leaves instead of hanging.  This call launches one warp whose thread 0
 * waits, through that same bounded wait, on a barrier nothing ever arrives
 * at, with a limit of `limit_us` microseconds (1 .. 1,000,000); no copy or
 * tensor-core operation is in flight.  After it, hs2_get_last_device_error
 * reports HS2_ERR_TIMEOUT once, and the device stays usable.
 */
hs2_status hs2_check_bounded_wait(unsigned limit_us, hs2_stream_t stream);

/*
 * Synchronises `stream`, then reports (and clears) the first error met since
 * the last call: a CUDA error (HS2_ERR_CUDA), a pipeline wait inside a kernel
 * that gave up after its time limit (HS2_ERR_TIMEOUT), or a device-side data
 * flag (HS2_ERR_DEVICE_DATA).  Returns HS2_OK when there is none.
 */
hs2_status hs2_get_last_device_error(hs2_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H */
