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
constexpr int kSMs = 148;            // B200 streaming multiprocessors
constexpr int kHistBins = 2048;      // top-k histogram buckets (see score_bin)
constexpr int kTopkChunk = 4096;     // pool keys per CTA in the histogram / emit passes
constexpr int kMetaInts = 8;

// Per-row bookkeeping in the workspace (ints; zeroed before each use, see Plan::off_meta).
//   kMetaBin / kMetaAbove: threshold bucket of the k-th best key and the count above it
//   kMetaDef / kMetaCand: emit counters (adjacent, 8-byte aligned: reserved together);
//   kMetaDone: score/histogram CTAs finished
//   kMetaSelDone: selection CTAs finished;     kMetaSparseDone: sparse-attention CTAs finished
//   kMetaBarrier: the fused decode step's per-row barrier counter
enum TopkMeta { kMetaBin = 0, kMetaAbove = 1, kMetaDef = 2, kMetaCand = 3, kMetaDone = 4, kMetaSelDone = 5,
                kMetaSparseDone = 6, kMetaBarrier = 7 };  // kMetaDef/kMetaCand share one 8-byte word
constexpr int kSmemCand = 4096;      // candidates the final select keeps in shared memory
constexpr int kMaxKW = 1 << 22;      // largest supported k + W
constexpr int kSparseMaxC4 = 4096;         // most selected keys one sparse-attention CTA takes
constexpr int kRowsPerCtaTopk = 4 * kSMs;  // from this many selection rows on, one top-k CTA per row

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
    bool fused;         // hs2_step runs the single fused decode-step kernel (T = 1, see k_decode.cu)
    // workspace byte offsets
    size_t off_status, off_meta, meta_end, off_hist, off_pf_ml, off_pf_acc, off_ps_ml, off_ps_acc, off_keys, off_cand,
        off_logits, zero_bytes, total;
};

bool make_plan(const hs2_dims* dims, Plan* p, hs2_status* why);

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
    float2* part_ml;       // [S][rows_q]
    float* part_acc;       // [S][rows_q][D]
    float* logits;         // optional [rows_kv][N][G] base-2 logits (full sweep only)
    const float* lse;      // [rows_q] natural-log LSE_full (score sweep only)
    uint32_t* keys;        // [rows_kv][kstride] order-preserving score keys (score sweep only)
    int64_t kstride;
    int k;
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
    float scale_log2;
    float2* part_ml;       // [S4][rows_q]
    float* part_acc;       // [S4][rows_q][D]
    int* meta;             // [rows_kv][kMetaInts] (completion counter kMetaSparseDone)
    uint16_t* O;           // O_sparse [B][Hq][T][D]
    float* LSE;            // LSE_sparse [B][Hq][T]
    unsigned* status;
};

struct DecodeArgs {        // the fused decode step (T = 1)
    AttnArgs attn;         // full sweep: Q_full, pos, shapes, full partials, kept logits
    const uint16_t* Qs;    // Q_sparse [B][Hq][1][D]
    const uint16_t* K;     // [B][Hkv][N][D] (gathered by the sparse phase)
    const uint16_t* V;
    int k, W;
    float2* ps_ml;         // sparse partials [S1][rows_q]
    float* ps_acc;         // [S1][rows_q][D]
    unsigned* hist;        // [rows][kHistBins]
    int* meta;             // [rows][kMetaInts]
    unsigned long long* cand;  // [rows][cand_cap]
    int64_t cand_cap;
    int32_t* idx;          // [rows][k+W]
    int32_t* cnt;          // [rows]
    uint16_t* O_full;
    float* LSE_full;
    uint16_t* O_sparse;
    float* LSE_sparse;
};

// Shared-memory plan of the fused decode step's phases after the sweep (byte offsets from the
// 1 KB-aligned base; the sweep ring below is 96 KB).
constexpr int kFusedLseOff = 0;          // 16 floats: per-head base-2 LSE
constexpr int kFusedWbufOff = 1024;      // 256 floats: combine weights
constexpr int kFusedHistOff = 2048;      // kHistBins u32 (phases A, B); then 2 x 64 gather slots (D)
constexpr int kFusedKeysOff = 10240;     // this split's pool keys (u32), phases A and B
constexpr int kFusedCandOff = 10240;     // phase C: candidates held in shared memory
constexpr int kFusedRingOff = 32768;     // phase D: gather ring, 2 tiles of K and V
constexpr int kFusedSmemCand = (kFusedRingOff - kFusedCandOff) / 8;
constexpr int kFusedMaxKeys = (96 * 1024 - kFusedKeysOff) / 4;
constexpr int kFusedMaxSlice = 4096;

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

struct TopkArgs {
    const uint32_t* keys;  // [rows][kstride]
    int64_t kstride;
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

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// ------------------------------------------------------------------ launchers (return cudaGetLastError())

cudaError_t launch_init(void* ws, size_t bytes, cudaStream_t st);  // clears ws[0, bytes) (normal launch)

cudaError_t launch_full_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st);
cudaError_t launch_umma_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st);  // tensor maps with 128-key boxes
cudaError_t launch_umma_score(const Plan& p, const CUtensorMap& tmK, const AttnArgs& a,
                              cudaStream_t st);  // tensor map with 128-key boxes
cudaError_t launch_topk_rows(const Plan& p, const TopkArgs& a, cudaStream_t st);  // one CTA per row
cudaError_t launch_score_sweep(const Plan& p, int splits, const CUtensorMap& tmK, const AttnArgs& a, cudaStream_t st);
cudaError_t launch_score_hist(const Plan& p, const ScoreArgs& a, cudaStream_t st);
cudaError_t launch_combine(int d, const CombineArgs& a, cudaStream_t st);
cudaError_t launch_sparse_attn(const Plan& p, const SparseArgs& a, cudaStream_t st);
// The fused decode step; returns cudaErrorCooperativeLaunchTooLarge if its grid cannot be
// co-resident (the caller then runs the multi-kernel path).
cudaError_t launch_decode_step(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a,
                               cudaStream_t st);
cudaError_t launch_topk_hist(const Plan& p, const TopkArgs& a, cudaStream_t st);
cudaError_t launch_topk_select(const Plan& p, const TopkArgs& a, cudaStream_t st);

}  // namespace hs2
