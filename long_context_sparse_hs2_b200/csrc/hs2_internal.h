// Internal (host + device) declarations of the HySparse2 library: the execution plan of
// one call, kernel argument blocks, and the host launchers each kernel file exports.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "hs2.h"

namespace hs2 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kKeyTile = 64;                      // keys per K/V shared-memory tile
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bound on any single pipeline wait (2 s)
constexpr int kHistBins = 2048;      // top-k histogram buckets (see score_bin)
constexpr int kTopkChunk = 4096;     // pool keys per CTA in the histogram / emit passes
constexpr int kMetaInts = 8;

// Per-row bookkeeping in the workspace (ints; zeroed before each use, see Plan::off_meta).
//   kMetaBin / kMetaAbove: threshold bucket of the k-th best key and the count above it
//   kMetaDef / kMetaCand: emit counters (adjacent, 8-byte aligned: reserved together);
//   kMetaDone: score/histogram CTAs finished
//   kMetaSelDone: selection CTAs finished;     kMetaSparseDone: sparse-attention CTAs finished
//   kMetaBarrier: unused
enum TopkMeta { kMetaBin = 0, kMetaAbove = 1, kMetaDef = 2, kMetaCand = 3, kMetaDone = 4, kMetaSelDone = 5,
                kMetaSparseDone = 6, kMetaBarrier = 7 };  // kMetaDef/kMetaCand share one 8-byte word
constexpr int kSmemCand = 4096;      // candidates the final select keeps in shared memory
constexpr int kFusedKeyCap = 16384;  // pool keys per split of the one-launch decode step
constexpr int kFusedMaxN = 8192;     // the one-launch decode step by default up to this cache length
constexpr int kMaxKW = 1 << 22;      // largest supported k + W
constexpr int kSparseMaxC4 = 4096;         // most selected keys one sparse-attention CTA takes
constexpr int kRowsPerCtaTopkPerSM = 4;   // from 4 x (SMs) selection rows on, one top-k CTA per row
constexpr int kSampleTileStride = 16;      // bracketed path: one 128-key tile in 16 is sampled
constexpr int kBracketMinPool = 32768;     // bracketed path: only for caches of at least this many keys
constexpr int kMaxSegments = 64;          // candidate-list segments per row on the bracketed path

// How the kernels find a token's K/V row in the cache (see hs2_kv_cache in hs2.h).
//   contiguous: row (b*Hkv + h)*N + j of [B][Hkv][N][d]
//   paged:      row (page*Hkv + h)*page_size + j % page_size of the pool, page =
//               page_table[b*max_pages + j / page_size]; a page id outside [0, num_pages)
//               (or a page index past max_pages) reads as zeros and flags HS2_DEV_BAD_PAGE
// fp8: rows hold E4M3 codes (d bytes); k_scale/v_scale[b*Hkv + h] turn codes into values.
struct KvSrc {
    int fp8;
    int page_shift;              // log2(page_size), or -1 for the contiguous layout
    int max_pages, num_pages;
    const int32_t* page_table;   // [B][max_pages]
    const float* k_scale;        // [B*Hkv] (fp8 only)
    const float* v_scale;
};

// Everything one call needs to know about shapes, grids and workspace offsets.
struct Plan {
    int B, Hq, Hkv, T, N, d, k, W, G;
    int64_t rows_q;     // B*Hq*T   query-head rows
    int64_t rows_kv;    // B*Hkv*T  selection rows
    int RT;             // 16-row MMA tiles per attention row block (1, 2, 4, 8)
    int TQ;             // queries per row block = 16*RT/G
    int QB;             // row blocks per (b, kv head) = ceil(T / TQ)
    int S1;             // split partials per row written by the full-attention sweep
    int S2;             // split-K factor of the score sweep (second K pass)
    bool umma;          // 128-row tiles: the full sweep runs on tcgen05 (k_umma_attn.cu)
    bool umma_split_keys;  // tcgen05 sweep: one query tile per CTA, its two streams split the keys
    int SU;             // tcgen05 sweep: key-range splits (S1 = SU, or 2 SU when the keys are split)
    int SS;             // tcgen05 score sweep: key-range splits
    bool mat_logits;    // hs2_step keeps the full layer's logits instead of re-reading K
    int C4;             // selected keys per sparse-attention CTA
    int S4;             // sparse-attention splits per row = ceil((k+W)/C4)
    int64_t cand_cap;   // per-row capacity of the top-k candidate buffer
    int topk_ctas;      // CTAs per row of the multi-CTA top-k kernels (each takes every topk_ctas-th chunk)
    int64_t kstride;    // row stride (elements) of the score-key buffer: N rounded up to 64
    bool fp8;           // the cache holds FP8 E4M3 codes
    bool paged;         // the cache is a paged pool
    int page_size, max_pages, num_pages;
    int sms;            // streaming multiprocessors of the device the plan was made for
    // Many rows on the tcgen05 score sweep with large pools: the sweep never stores every key.
    // A pass over a 1/16 sample of the key tiles brackets each row's threshold bucket, and the
    // full pass appends only the keys at or above it to the row's candidate list.
    bool bracketed;
    int nseg, seg_cap;  // bracketed: candidate-list segments per row (4 per score split) and their size
    bool fused;         // decode (T = 1): the one-launch step (k_decode_fused.cu), where its grid fits
    int64_t sstride;    // sample keys per row (a multiple of 128)
    int64_t bcap;       // candidate-list capacity per row
    // workspace byte offsets
    size_t off_status, off_tilectr, init_bytes, off_pos, off_meta, meta_end, off_hist, off_pf_ml, off_pf_acc, off_ps_ml, off_ps_acc, off_keys, off_cand, off_segcnt,
        off_logits, zero_bytes, total;
};

// Cache description the plan depends on (dtype and layout only; pointers are checked per call).
struct KvShape {
    int fp8 = 0;
    int page_size = 0;   // 0: contiguous
    int max_pages = 0;
    int num_pages = 0;
};

bool make_plan(const hs2_dims* dims, Plan* p, hs2_status* why, const KvShape& kv = KvShape());

// ------------------------------------------------------------------ kernel arguments

struct AttnArgs {
    const uint16_t* Q;     // [B][Hq][T][D]
    uint4* zero;           // optional region the full sweep clears for the kernels after it
    int64_t zero_vec;      // its size in 16-byte words
    const int32_t* pos;    // [B][T]
    int B, Hq, Hkv, T, N, G, W;
    int TQ, QB, S;
    float scale_log2;      // d^-1/2 * log2(e)
    int stream_kv;         // 1: every K/V tile is read once (decode) -> load it evict-first
    int* tilectr;          // [units] tiles handed out so far (the mma.sync full sweep's CTAs of a row
                           // block take chunks of its key tiles from it); cleared by init
    float2* part_ml;       // [S][rows_q]
    float* part_acc;       // [S][rows_q][D]
    float* logits;         // optional [rows_kv][N][G] base-2 logits (full sweep only)
    const float* lse;      // [rows_q] natural-log LSE_full (score sweep only)
    uint32_t* keys;        // [rows_kv][kstride] order-preserving score keys (score sweep only)
    int64_t kstride;
    int k;
    // tcgen05 score sweep: 0 stores every pool key's score key in keys; 1 scores every
    // kSampleTileStride-th 128-key tile and stores them compactly in keys (the sample); 2 writes
    // the composite (key, ~j) of every pool key whose bucket is at most the row's bracket
    // (meta[row][kMetaBin]) to the candidate list cand[row] (row stride cand_cap): each epilogue
    // warp of each split fills its own segment of seg_cap entries, and segcnt[row][segment]
    // receives the segment's count (which may exceed seg_cap: the list then overflowed)
    int score_mode;
    unsigned long long* cand;
    int64_t cand_cap;
    int seg_cap;
    int* segcnt;
    int* meta;
    KvSrc kv;              // cache layout / dtype (TMA producer and scales)
    unsigned* status;
};

struct SparseArgs {
    const uint16_t* Q;     // Q_sparse [B][Hq][T][D]
    const uint16_t* K;     // [B][Hkv][N][D]
    const uint16_t* V;
    const int32_t* pos;    // [B][T]
    const int32_t* idx;    // [rows_kv][k+W]
    const int32_t* cnt;    // [rows_kv]
    int B, Hq, Hkv, T, N, G, kw;  // kw = k + W (row stride of idx)
    int C4, S4;
    int stages;            // gather ring depth (set by the launcher)
    KvSrc kv;              // cache layout / dtype
    float scale_log2;
    float2* part_ml;       // [S4][rows_q]
    float* part_acc;       // [S4][rows_q][D]
    int* meta;             // [rows_kv][kMetaInts] (completion counter kMetaSparseDone)
    uint16_t* O;           // O_sparse [B][Hq][T][D]
    float* LSE;            // LSE_sparse [B][Hq][T]
    unsigned* status;
};

struct CombineArgs {
    const float2* part_ml;
    const float* part_acc;
    int S;
    int64_t rows;
    uint16_t* O;           // bf16 [rows][D]
    float* LSE;            // [rows] natural log
};

struct ScoreArgs {         // scores + histogram from kept logits, with the full-attention combine
    const float* logits;   // [rows_kv][N][G] base-2 logits
    const float2* part_ml; // full-attention split partials [S1][rows_q]
    const float* part_acc; // [S1][rows_q][D]
    int S1;
    const int32_t* pos;
    int B, Hq, Hkv, T, N, G, k, W;
    uint16_t* O;           // O_full [B][Hq][T][D]
    float* LSE;            // LSE_full [B][Hq][T]
    uint32_t* keys;        // [rows_kv][kstride]
    int64_t kstride;
    unsigned* hist;        // [rows_kv][kHistBins]
    int* meta;             // [rows_kv][kMetaInts]
    unsigned* status;
};

struct FusedArgs {          // the selection and sparse layer of the one-launch decode step
    const uint16_t* Qs;    // Q_sparse [B][Hq][1][D]
    const void* K;         // the cache (contiguous or pool), bf16 or E4M3 codes
    const void* V;
    int k;
    uint16_t* O_full;      // [B][Hq][1][D]
    float* LSE_full;       // [B][Hq][1]
    uint16_t* O_sparse;
    float* LSE_sparse;
    int32_t* idx;          // [rows_kv][k+W]
    int32_t* cnt;          // [rows_kv]
    unsigned* hist;        // [rows_kv][kHistBins], cleared before the launch
    int* meta;             // [rows_kv][kMetaInts], cleared before the launch
    unsigned long long* cand;  // [rows_kv][cand_cap] threshold-bucket candidates (cand_cap >= N)
    int64_t cand_cap;
    float2* ps_ml;         // sparse split partials [S][rows_q]
    float* ps_acc;         // [S][rows_q][D]
};

struct TopkArgs {
    const uint32_t* keys;  // [rows][kstride] (the sample keys for the bracket kernel)
    int64_t kstride;
    // the exact fallback of the bracketed path rescores a row from Q, K and LSE (contiguous bf16)
    const uint16_t* Q;     // Q_full [B][Hq][T][d]
    const uint16_t* K;     // [B][Hkv][N][d]
    const float* lse;      // LSE_full [B][Hq][T]
    int Hq, G, d;
    float scale_log2;
    const int* segcnt;     // bracketed path: candidates per segment [rows][nseg], seg_cap per segment
    int nseg, seg_cap;
    const int32_t* pos;    // [B][T]
    int Hkv, T, N, k, W;
    int64_t rows;
    unsigned* hist;        // [rows][kHistBins]
    int* meta;             // [rows][kMetaInts]
    unsigned long long* cand;  // [rows][cand_cap] composite (key << 32 | ~index)
    int64_t cand_cap;
    int32_t* idx;          // [rows][k+W]
    int32_t* cnt;          // [rows]
    unsigned* status;
};

// ------------------------------------------------------------------ tracing (hs2_trace.cu)

void trace_call_begin(cudaStream_t st);              // once at the start of every entry point
void trace_mark(const char* name, cudaStream_t st, bool kernel = true);  // after every launch / memset

// ------------------------------------------------------------------ launch helper

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger) -- or, with
// pdl = false, as an ordinary launch that starts only after everything before it completed.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_opt(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    return launch_pdl_opt(true, kern, grid, block, smem, st, static_cast<Args&&>(args)...);
}

// ------------------------------------------------------------------ launchers (return cudaGetLastError())

int num_sms();  // streaming multiprocessors of the current device (queried once per device)

cudaError_t launch_init(void* ws, size_t bytes, cudaStream_t st);  // clears ws[0, bytes) once the stream's previous kernel is done

// New tokens into the cache (hs2_kv_append / hs2_decode_step).  pos_in[b*T + t] (+1 when advance)
// is the token's position; with advance (T = 1) the position is also written to pos_out[b] and
// pos_new[b].  Ordinary launch.
struct AppendArgs {
    const uint16_t* K_new;  // [B][Hkv][T][d] bf16
    const uint16_t* V_new;
    void* K;                // cache (contiguous or pool)
    void* V;
    KvSrc kv;
    const int32_t* pos_in;
    int32_t* pos_out;       // advance: the caller's pos, updated
    int32_t* pos_new;       // advance: the position the step runs at (workspace copy)
    int B, Hkv, T, N, d;
    int advance;
    unsigned* status;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t st);

cudaError_t launch_full_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st, bool pdl = true);  // pdl = false: an ordinary launch
cudaError_t launch_umma_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st);  // tensor maps with 128-key boxes
cudaError_t launch_umma_score(const Plan& p, const CUtensorMap& tmK, const AttnArgs& a,
                              cudaStream_t st);  // tensor map with 128-key boxes
cudaError_t launch_topk_rows(const Plan& p, const TopkArgs& a, cudaStream_t st);  // one CTA per row
cudaError_t launch_score_sweep(const Plan& p, int splits, const CUtensorMap& tmK, const AttnArgs& a, cudaStream_t st);
cudaError_t launch_score_hist(const Plan& p, const ScoreArgs& a, cudaStream_t st);
cudaError_t launch_combine(int d, const CombineArgs& a, cudaStream_t st);
cudaError_t launch_sparse_attn(const Plan& p, const SparseArgs& a, cudaStream_t st);
cudaError_t launch_topk_hist(const Plan& p, const TopkArgs& a, cudaStream_t st);
// The bracketed path: per row, the sample's bucket bracket (into meta[row][kMetaBin]) ...
cudaError_t launch_topk_bracket(const Plan& p, const TopkArgs& a, cudaStream_t st);
// ... and, after the filtering sweep, the exact selection from the candidate list (an exact
// rescoring of the row where the bracket did not hold).
cudaError_t launch_topk_finalize(const Plan& p, const TopkArgs& a, cudaStream_t st);
cudaError_t launch_topk_select(const Plan& p, const TopkArgs& a, cudaStream_t st);
// The one-launch decode step (T = 1): sweep, selection and sparse layer in one cooperative grid
// of p.S1 x rows_kv CTAs.  *launched = false (nothing launched, cudaSuccess) when the grid does
// not fit on the device at once; the caller then runs the kernel chain.
cudaError_t launch_decode_fused(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                                const FusedArgs& f, cudaStream_t st, bool pdl, bool* launched);

}  // namespace hs2
