/*
 * hs2.h -- C ABI of the HySparse2 hybrid sparse attention step on NVIDIA B200 (sm_100a).
 *
 * What the step computes
 * ----------------------
 * HySparse2 places hybrid sparse attention in the cross-decoder: a full-attention
 * layer over the shared KV cache, followed by sparse layers ("HySparse2 Cuts the
 * Prefill Path for Tool-Using Agents", section "One Cache Plan, Two Sharing Layers").
 * Each sparse layer reuses that layer's KV cache and its per-token selection,
 * and the most recent tokens are always part of the selection (KV Reuse; "HySparse2
 * od Xiaomi zkracuje zpracovani dlouheho kontextu", section "Proc neni nutne znovu
 * zpracovat cely dlouhy vstup", third paragraph; DAIR.AI newsletter, HySparse2
 * bullets "Two levels of KV sharing" and "Prefill exits early").
 *
 * Notation: batch B, query heads Hq, kv heads Hkv, G = Hq / Hkv query heads per kv
 * head (query head hq reads kv head hq / G), head dim d, cached tokens N, queries T
 * per batch row, query position pos[b][t] (0 <= pos < N; key j is visible iff j <= pos),
 * selection size k, forced window W, scale = d^-1/2.
 *
 *   full attention:   l_j = scale <q_full, k_j>,  LSE_full = ln sum_{j<=pos} e^{l_j},
 *                     O_full = sum_{j<=pos} e^{l_j - LSE_full} v_j
 *   selection score:  s_j = max over the G heads of kv head h of (l_j - LSE_full),
 *                     for j in the pool [0, pos - W]   (the pages leave the score
 *                     open; this library fixes it to the GQA-max log-softmax)
 *   selection:        the min(k, |pool|) pool keys of largest s (ties: lower index)
 *                     plus the window [max(0, pos - W + 1), pos]
 *   sparse attention: the full-attention formula with Q_sparse over the selected
 *                     keys only; all G heads of kv head h share the selection.
 *
 * Conventions (all entry points)
 * ------------------------------
 *  - Every tensor pointer is DEVICE memory owned by the caller, contiguous row-major
 *    in the layout given, 16-byte aligned.  bf16 tensors are passed as const void*
 *    holding IEEE bfloat16 bit patterns.
 *      Q_full, Q_sparse, O_full, O_sparse : bf16  [B][Hq][T][d]
 *      K, V                               : bf16  [B][Hkv][N][d]
 *      pos                                : int32 [B][T]
 *      LSE_full, LSE_sparse               : fp32  [B][Hq][T]   (natural log)
 *      idx                                : int32 [B][Hkv][T][k + W]
 *      cnt                                : int32 [B][Hkv][T]
 *  - idx row r holds cnt[r] valid key indices followed by -1 padding.  The order of
 *    the valid entries is unspecified (attention does not depend on key order).  When
 *    k + W = 0 idx has no elements and may be NULL.
 *  - ws is a device workspace of at least hs2_workspace_size(dims) bytes, 256-byte
 *    aligned, owned by the caller; its contents need no initialisation and are
 *    overwritten by every call.  The library allocates no memory of its own.
 *  - stream is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous on that stream: no host synchronisation, no device->host copy.
 *  - Host-side argument checks run before any launch: a failing check returns an
 *    error and launches nothing.  Launch failures return HS2_ERR_CUDA.
 *  - Problems the host cannot see (a pos outside [0, N), an index outside [0, pos]
 *    passed to hs2_sparse_attn, a non-finite score) set bits in a device status
 *    word inside ws; kernels clamp or skip the offending element and continue.  Read
 *    the word with hs2_read_device_status.  Each entry point clears it when it starts.
 *  - Supported shapes: d in {64, 128}; G in {1, 2, 4, 8, 16}; B, Hq, Hkv, T, N >= 1;
 *    T <= N; k >= 0; W >= 0; k + W < 2^31.  Anything else is HS2_ERR_UNSUPPORTED or
 *    HS2_ERR_INVALID_ARG.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HS2_API __attribute__((visibility("default")))
#else
#define HS2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hs2_status {
    HS2_OK = 0,
    HS2_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned pointer, pos/shape mismatch */
    HS2_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes (d, G) */
    HS2_ERR_WORKSPACE = 3,    /* ws is null or smaller than hs2_workspace_size(dims), or misaligned */
    HS2_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    HS2_ERR_DEVICE = 5        /* returned only by hs2_read_device_status when status bits are set */
} hs2_status;

/* Bits of the device status word (see hs2_read_device_status). */
#define HS2_DEV_BAD_POS       0x1u  /* a pos[b][t] outside [0, N): clamped into range */
#define HS2_DEV_BAD_INDEX     0x2u  /* hs2_sparse_attn got an index outside [0, pos]: key skipped */
#define HS2_DEV_NONFINITE     0x4u  /* a selection score was NaN: ranked below every finite score */
#define HS2_DEV_TIMEOUT       0x8u  /* a pipeline wait exceeded its bound: kernel gave up, outputs invalid */
#define HS2_DEV_CAND_OVERFLOW 0x10u /* informational: top-k threshold bucket overflowed its buffer; slow exact path used */
#define HS2_DEV_BAD_PAGE      0x20u /* a page id outside [0, num_pages) in the page table: its tokens read as zeros
                                       (gathers skip them); hs2_kv_append skipped the token */

/* Problem shape.  The attention scale is fixed to d^-1/2. */
typedef struct hs2_dims {
    int32_t B, Hq, Hkv, T, N, d, k, W;
} hs2_dims;

/* Bytes of device workspace every entry point below needs for these dims (a multiple of
 * 256).  Returns 0 if the dims are invalid or unsupported.  Pure host computation. */
HS2_API size_t hs2_workspace_size(const hs2_dims* dims);

/* Full-attention layer: O_full and LSE_full for every (b, hq, t), keys 0..pos[b][t].
 * Source: the full-attention layer of the hybrid block ("HySparse2 Cuts the Prefill
 * Path...", "One Cache Plan, Two Sharing Layers"); split-K flash-decode with a
 * log-sum-exp combine (as in "Simplified Sparse Attention via Gist Tokens", section
 * 3.6, "three-kernel split-K sparse flash-decode"). */
HS2_API hs2_status hs2_full_attn(const hs2_dims* dims, const void* Q_full, const void* K, const void* V,
                         const int32_t* pos, void* O_full, float* LSE_full,
                         void* ws, size_t ws_bytes, void* stream);

/* Token-level selection: scores every pool key with the GQA-max log-softmax score (using
 * the caller's LSE_full, as produced by hs2_full_attn), keeps the min(k, |pool|) best
 * (ties to the lower index) and adds the forced window.  Writes idx and cnt
 * (cnt = min(k, |pool|) + min(W, pos + 1)).  Source: token-level selection with forced
 * recent tokens ("HySparse2 od Xiaomi...", third paragraph; DAIR.AI newsletter,
 * "Prefill exits early"). */
HS2_API hs2_status hs2_select(const hs2_dims* dims, const void* Q_full, const void* K,
                      const float* LSE_full, const int32_t* pos, int32_t* idx, int32_t* cnt,
                      void* ws, size_t ws_bytes, void* stream);

/* Sparse layer with KV Reuse: attention of Q_sparse over the keys listed in idx/cnt
 * (the same list for all G query heads of a kv head).  Any idx/cnt the caller supplies
 * is accepted; entries outside [0, pos] are skipped and flag HS2_DEV_BAD_INDEX, and
 * cnt is clamped to [0, k + W].  A row with no keys gives O = 0, LSE = -inf.
 * Source: KV Reuse ("HySparse2 od Xiaomi...", third paragraph; DAIR.AI newsletter,
 * "Two levels of KV sharing"). */
HS2_API hs2_status hs2_sparse_attn(const hs2_dims* dims, const void* Q_sparse, const void* K,
                           const void* V, const int32_t* pos, const int32_t* idx,
                           const int32_t* cnt, void* O_sparse, float* LSE_sparse,
                           void* ws, size_t ws_bytes, void* stream);

/* The whole hybrid step: hs2_full_attn, hs2_select and hs2_sparse_attn in order on one
 * stream, sharing intermediates through ws.  When T*G <= 16 the full-attention pass keeps its
 * logits so the selection does not read K a second time; when T*G > 64 (128-row query tiles:
 * chunked prefill, multi-query decode) the full-attention and score sweeps run on the tcgen05
 * tensor cores.  Environment variables change the execution plan (results are the same up to
 * rounding order; the workspace size depends on them, so query hs2_workspace_size under the same
 * environment): HS2_UMMA=0 keeps the warp-level MMA sweeps for 128-row tiles;
 * HS2_PREFILL_BRACKET=0 stores every selection key for many rows over long caches instead of
 * filtering candidates; HS2_TRANSPOSED=0 keeps the 16-row warp attention for decode row blocks;
 * HS2_DYN_SWEEP=1 / 0 forces the counter-scheduled sweep on / off (default: on for at least 128
 * key tiles per CTA); HS2_FUSED_DECODE=1 / 0 forces the one-launch decode step (T = 1) on / off
 * (default: caches of at most 8192 tokens).  The plan, and so the workspace size, also follows
 * the current device's SM count. */
HS2_API hs2_status hs2_step(const hs2_dims* dims, const void* Q_full, const void* Q_sparse,
                    const void* K, const void* V, const int32_t* pos,
                    void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse,
                    int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream);

/* Size of the fixed device array that hs2_sparse_attn_static uses as its scratch. */
#define HS2_STATIC_SCRATCH_BYTES (4u << 20)

/* hs2_sparse_attn without a workspace argument, for callers that cannot allocate device
 * memory at the point of the call (an engine serving requests from fixed memory pools, a
 * plugin inside a program that owns all device memory, a path that cannot afford an
 * allocation or a size query per call).  The pages have no counterpart: this is a convenience
 * of this library.  Same arguments, layouts and results as hs2_sparse_attn, minus ws/ws_bytes.
 *
 *  - Scratch: one file-scope device array of HS2_STATIC_SCRATCH_BYTES (4 MiB) that every GPU
 *    loading the library holds until the process exits.  The call allocates nothing (no
 *    cudaMalloc / cudaFree, no allocating library routine).
 *  - Limit: shapes whose scratch (per-row counters plus split partials, about
 *    B*Hq*T * ceil((k+W)/C) * (d+2) * 4 bytes for the library's split size C) exceeds the array
 *    are rejected with HS2_ERR_WORKSPACE before anything is launched; decode shapes up to a
 *    few hundred query-head rows fit.
 *  - Set-up: the first call on each device looks up the array's device address (while that
 *    device is current); make that first call before any stream capture.  The address is kept
 *    for the life of the process: do not call this entry point after cudaDeviceReset, which
 *    frees the array and leaves the kept address dangling.
 *  - Sharing: every call on a device uses the same array and leaves its contents behind; each
 *    call clears what must start at zero.  Calls whose GPU work overlaps (other streams, other
 *    host threads) race on the array and give undefined results: serialise them.
 *  - Device status bits go to the array's first word; hs2_read_device_status cannot reach it,
 *    so problems are reported only through the outputs (skipped indices, clamped positions). */
HS2_API hs2_status hs2_sparse_attn_static(const hs2_dims* dims, const void* Q_sparse, const void* K,
                                          const void* V, const int32_t* pos, const int32_t* idx,
                                          const int32_t* cnt, void* O_sparse, float* LSE_sparse,
                                          void* stream);

/* ---------------------------------------------------------------------------------------------
 * The KV cache in other storage formats and layouts, and the decode loop.
 *
 * The pages give the shared cache's size (2.69 GB at 1M tokens) without its storage precision
 * ("HySparse2 od Xiaomi...", section "Co rikaji vysledky -- a co z nich neplyne"), and serving an
 * agent's long context means a cache that grows by one token per decode step ("HySparse2 Cuts
 * the Prefill Path for Tool-Using Agents", section "Tool Responses Turn Prefill Into the
 * Bottleneck").  These entry points take the cache as a descriptor instead of two contiguous
 * bf16 tensors: bf16 or FP8 E4M3 codes with per-(b, kv head) scales, contiguous or in a paged
 * pool.  The method is unchanged: every stored token is first read back to its value (code x
 * scale for FP8) and the four definitions at the top of this file apply to those values.
 * ------------------------------------------------------------------------------------------- */

typedef enum hs2_kv_dtype {
    HS2_KV_BF16 = 0,      /* bfloat16 values */
    HS2_KV_FP8_E4M3 = 1   /* FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
                             S.1111.111 is NaN); value = code x scale of the token's (b, kv head) */
} hs2_kv_dtype;

/* Where and how the shared cache is stored.  All pointers are device memory owned by the caller.
 *  - dtype: hs2_kv_dtype.  Element size: 2 bytes (bf16) or 1 byte (FP8).
 *  - page_size = 0: contiguous, K and V are [B][Hkv][N][d] (16-byte aligned).
 *  - page_size > 0 (a power of two, 8 .. 65536): paged, K and V are pools
 *    [num_pages][Hkv][page_size][d] (16-byte aligned) and token j of batch row b is stored in page
 *    page_table[b * max_pages + j / page_size], at slot j % page_size.  max_pages >= ceil(N /
 *    page_size); num_pages * Hkv * page_size < 2^31.  Pages may be shared between batch rows and
 *    appear in any order.  A page id outside [0, num_pages) for a token the kernels read sets
 *    HS2_DEV_BAD_PAGE, and the token reads as zeros (gathered keys are skipped).
 *  - k_scale, v_scale: FP8 only, fp32 [B][Hkv]; NULL for bf16.
 * K and V are const for every entry point except hs2_kv_append and hs2_decode_step, which write
 * new tokens into them. */
typedef struct hs2_kv_cache {
    int32_t dtype;
    int32_t page_size;
    int32_t num_pages;
    int32_t max_pages;
    void* K;
    void* V;
    const int32_t* page_table;
    const float* k_scale;
    const float* v_scale;
} hs2_kv_cache;

/* hs2_workspace_size for a cache described by `cache` (its dtype and layout change the plan).
 * Returns 0 if the dims or the cache description are invalid or unsupported. */
HS2_API size_t hs2_workspace_size_kv(const hs2_dims* dims, const hs2_kv_cache* cache);

/* hs2_full_attn, hs2_select, hs2_sparse_attn and hs2_step over a cache descriptor; same
 * arguments, layouts, results and status bits otherwise.  A bf16 contiguous descriptor gives
 * exactly the calls above.  FP8 caches run the warp-level MMA path on f16 operands (every E4M3
 * value is exact in f16; queries are scaled by a power of two per row into the f16 range); FP8
 * and paged caches run 128-row query tiles on the warp-level MMA sweeps, not tcgen05. */
HS2_API hs2_status hs2_full_attn_kv(const hs2_dims* dims, const void* Q_full, const hs2_kv_cache* cache,
                                    const int32_t* pos, void* O_full, float* LSE_full, void* ws, size_t ws_bytes,
                                    void* stream);
HS2_API hs2_status hs2_select_kv(const hs2_dims* dims, const void* Q_full, const hs2_kv_cache* cache,
                                 const float* LSE_full, const int32_t* pos, int32_t* idx, int32_t* cnt, void* ws,
                                 size_t ws_bytes, void* stream);
HS2_API hs2_status hs2_sparse_attn_kv(const hs2_dims* dims, const void* Q_sparse, const hs2_kv_cache* cache,
                                      const int32_t* pos, const int32_t* idx, const int32_t* cnt, void* O_sparse,
                                      float* LSE_sparse, void* ws, size_t ws_bytes, void* stream);
HS2_API hs2_status hs2_step_kv(const hs2_dims* dims, const void* Q_full, const void* Q_sparse,
                               const hs2_kv_cache* cache, const int32_t* pos, void* O_full, void* O_sparse,
                               float* LSE_full, float* LSE_sparse, int32_t* idx, int32_t* cnt, void* ws,
                               size_t ws_bytes, void* stream);

/* Writes new tokens into the cache: for every (b, kv head, t), the bf16 rows K_new[b][h][t][:] and
 * V_new[b][h][t][:] ([B][Hkv][T][d]) become token pos[b][t] of the cache -- stored as they are
 * (bf16) or as the E4M3 code of value / scale (one fp32 division, rounded to nearest even,
 * magnitudes past 448 saturating to 448) for an FP8 cache.  A pos outside [0, N) (HS2_DEV_BAD_POS)
 * or an unmapped page (HS2_DEV_BAD_PAGE) skips that token.  ws: at least 256 bytes (the status
 * word, cleared by the call).  Two (b, t) naming the same token: one of them wins. */
HS2_API hs2_status hs2_kv_append(const hs2_dims* dims, const hs2_kv_cache* cache, const void* K_new,
                                 const void* V_new, const int32_t* pos, void* ws, size_t ws_bytes, void* stream);

/* One decode step of the loop (T = 1): for every batch row b, the new token (K_new/V_new
 * [B][Hkv][1][d], bf16) is written into the cache at position pos[b] + 1 as hs2_kv_append does,
 * pos[b] is advanced to that position on the device, and the hybrid step (hs2_step_kv) runs
 * for a query at that position.  pos (int32 [B], device) is the loop's state: on entry the
 * newest cached position of each row (-1 for an empty row), on exit the new one.  Nothing
 * is read or written by the host, so a CUDA graph of one call replays the loop step after step.
 * A row whose cache is full (pos[b] + 1 >= N) sets HS2_DEV_BAD_POS, appends nothing, keeps
 * pos[b], and its step runs at position N - 1.  ws: hs2_workspace_size_kv(dims, cache) bytes. */
HS2_API hs2_status hs2_decode_step(const hs2_dims* dims, const hs2_kv_cache* cache, const void* Q_full,
                                   const void* Q_sparse, const void* K_new, const void* V_new, int32_t* pos,
                                   void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse, int32_t* idx,
                                   int32_t* cnt, void* ws, size_t ws_bytes, void* stream);

/* Copies the device status word out of ws and waits for the stream (the only synchronising
 * call).  *bits receives the HS2_DEV_* bits; returns HS2_ERR_DEVICE if any bit other than
 * HS2_DEV_CAND_OVERFLOW is set, else HS2_OK. */
HS2_API hs2_status hs2_read_device_status(const void* ws, void* stream, uint32_t* bits);

/* Failure-detection self-test (not from the pages; a property of this library).  Every
 * pipeline wait inside the kernels is bounded (2 s): when the bound runs out the kernel sets
 * HS2_DEV_TIMEOUT in the status word and returns, so a stalled pipeline leaves an error instead
 * of a hung GPU.  This call runs that same bounded wait, with the bound limit_ns (1 us .. 2 s), on
 * a barrier that nothing ever arrives on, on `stream`.  Afterwards hs2_read_device_status(ws)
 * returns HS2_ERR_DEVICE with exactly HS2_DEV_TIMEOUT set, after about limit_ns; the device stays
 * usable.  ws: at least 256 bytes (the status word), 256-byte aligned. */
HS2_API hs2_status hs2_selftest_wait_bound(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream);

/* Static, human-readable name of a status code. */
HS2_API const char* hs2_status_string(hs2_status status);

/* Per-kernel timing (tracing).  hs2_trace_enable(1) creates a fixed pool of CUDA events
 * (host-side driver objects; no device memory) on the current device and starts recording:
 * every entry point then records an event on its stream when it starts and after each kernel
 * it launches.  hs2_trace_enable(0) stops recording.  Either call clears the record.
 * hs2_trace_collect waits for the recorded events and writes, for each kernel name seen since
 * the last collect, its summed duration in milliseconds and its launch count (at most
 * max_entries names; names point to static strings).  It returns the number of names, -1 on
 * a CUDA error, or -(n + 1) if the event pool ran out (the record is then incomplete).
 * Process-global, not thread-safe: meant for profiling and benchmark runs.  Not from the
 * pages: tracing support of this library. */
HS2_API hs2_status hs2_trace_enable(int enable);
HS2_API int hs2_trace_collect(const char** names, double* total_ms, int64_t* launches, int max_entries);

/* Number of CUDA kernels this library has launched in this process (tracing on or off). */
HS2_API uint64_t hs2_launch_count(void);

/* Library version, (major << 16) | minor. */
HS2_API uint32_t hs2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H_ */
