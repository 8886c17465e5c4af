// C ABI of the HySparse2 hybrid sparse attention step: argument checks, the execution
// plan (grids, split factors, workspace layout), TMA descriptors and launch order.
// Declared and documented in include/hs2.h.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "hs2_internal.h"

namespace hs2 {

namespace {

constexpr int64_t kUmmaCtaCost = 8;  // per-CTA cost of the tcgen05 sweeps, in 128-key tiles

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Split-K factor minimising waves x (tiles per split + a fixed per-CTA cost in tiles: the
// prologue, pipeline fill and partial write-out of one CTA), with a tiny penalty per split.
int choose_splits(int64_t units, int64_t tiles, int64_t slots, int max_splits, int64_t cta_cost = 0) {
    int best = 1;
    double best_cost = 1e300;
    const int limit = static_cast<int>(std::min<int64_t>(max_splits, std::max<int64_t>(tiles, 1)));
    for (int s = 1; s <= limit; ++s) {
        const int64_t waves = (units * s + slots - 1) / slots;
        const int64_t per = (tiles + s - 1) / s + cta_cost;
        const double cost = static_cast<double>(waves * per) + 0.01 * s;
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

}  // namespace

int num_sms() {
    // queried once per device; 148 (a B200) when no device can be queried (host-only use)
    constexpr int kMaxDev = 64;
    static int cached[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        cudaGetLastError();
        return 148;
    }
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

bool make_plan(const hs2_dims* dm, Plan* p, hs2_status* why, const KvShape& kv) {
    *why = HS2_ERR_INVALID_ARG;
    if (!dm) return false;
    const hs2_dims& x = *dm;
    if (x.B < 1 || x.Hq < 1 || x.Hkv < 1 || x.T < 1 || x.N < 1 || x.k < 0 || x.W < 0) return false;
    if (x.T > x.N || x.Hq % x.Hkv != 0) return false;
    if (static_cast<int64_t>(x.k) + x.W >= (int64_t(1) << 31)) return false;
    if (x.N > (int64_t(1) << 30)) return false;
    const int64_t rows_q = static_cast<int64_t>(x.B) * x.Hq * x.T;
    const int64_t rows_kv = static_cast<int64_t>(x.B) * x.Hkv * x.T;
    if (rows_q >= (int64_t(1) << 31) || static_cast<int64_t>(x.B) * x.Hkv >= (int64_t(1) << 31)) return false;
    if (kv.fp8 != 0 && kv.fp8 != 1) return false;
    if (kv.page_size != 0) {  // paged pool: power-of-two pages of 8 .. 65536 tokens
        const int ps = kv.page_size;
        if (ps < 8 || ps > 65536 || (ps & (ps - 1)) != 0) return false;
        if (kv.num_pages < 1 || kv.max_pages < (static_cast<int64_t>(x.N) + ps - 1) / ps) return false;
        if (static_cast<int64_t>(kv.num_pages) * x.Hkv * ps >= (int64_t(1) << 31)) return false;
    }
    *why = HS2_ERR_UNSUPPORTED;
    const int G = x.Hq / x.Hkv;
    if (x.d != 64 && x.d != 128) return false;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return false;
    if (rows_kv > 65535) return false;  // grid.y of the per-row kernels
    if (static_cast<int64_t>(x.k) + x.W > kMaxKW) return false;

    const int sms = num_sms();
    Plan& P = *p;
    P.B = x.B; P.Hq = x.Hq; P.Hkv = x.Hkv; P.T = x.T; P.N = x.N; P.d = x.d; P.k = x.k; P.W = x.W; P.G = G;
    P.rows_q = rows_q;
    P.rows_kv = rows_kv;
    P.fp8 = kv.fp8 != 0;
    P.paged = kv.page_size != 0;
    P.page_size = kv.page_size;
    P.max_pages = kv.max_pages;
    P.num_pages = kv.num_pages;
    P.sms = sms;
    const int64_t rows = static_cast<int64_t>(x.T) * G;
    P.RT = 1;
    while (P.RT < 8 && 16 * P.RT < rows) P.RT *= 2;
    P.TQ = 16 * P.RT / G;
    P.QB = (x.T + P.TQ - 1) / P.TQ;
    P.mat_logits = (P.RT == 1 && P.QB == 1);
    const int64_t units = static_cast<int64_t>(x.B) * x.Hkv * P.QB;
    if (units > 65535) return false;  // grid.y of the streaming kernels
    const int64_t tiles = (x.N + kKeyTile - 1) / kKeyTile;
    // resident sweep CTAs: two per SM for 16-row blocks (three for the transposed FP8 form), else one
    const char* want_tr = std::getenv("HS2_TRANSPOSED");
    const bool tr = x.T * G <= 8 && !(want_tr && want_tr[0] == '0');
    const int64_t slots = (P.RT == 1 ? (P.fp8 && tr ? 3 : 2) : 1) * int64_t(sms);
    P.S1 = choose_splits(units, tiles, slots, 256);
    P.S2 = P.S1;
    // 128-row query tiles: the full sweep runs on the tcgen05 tensor cores (HS2_UMMA=0 keeps the
    // mma.sync sweep), one CTA per SM, two query tiles per CTA -- or one, with the key range
    // split between the CTA's two streams, when a kv head has a single query tile.  The tcgen05
    // kernels read contiguous bf16 caches only; FP8 and paged caches take the mma.sync sweeps.
    const char* want_umma = std::getenv("HS2_UMMA");
    P.umma = P.RT == 8 && !(want_umma && want_umma[0] == '0') && !P.fp8 && !P.paged;
    P.umma_split_keys = P.QB == 1;
    P.SU = 1;
    P.SS = 1;
    if (P.umma) {
        const int64_t uunits = static_cast<int64_t>(x.B) * x.Hkv * (P.umma_split_keys ? P.QB : (P.QB + 1) / 2);
        const int64_t tiles128 = (x.N + 127) / 128;
        P.SU = choose_splits(uunits, tiles128, sms, 128, kUmmaCtaCost);
        P.S1 = P.SU * (P.umma_split_keys ? 2 : 1);
        P.SS = choose_splits(uunits, tiles128, sms, 256, kUmmaCtaCost);
    }

    // sparse attention: about one CTA per SM, each gathering C4 keys (a multiple of 64, <= 1024)
    // -- or, with many rows, a whole row (up to kSparseMaxC4 keys) per CTA, no split partials.
    // (One 128-key step per CTA at two CTAs per SM measured slower for the decode shapes.)
    const int64_t kw = static_cast<int64_t>(x.k) + x.W;
    const int64_t s4_target = std::max<int64_t>(1, sms / rows_kv);
    const int64_t c4 = ((std::max<int64_t>(1, (kw + s4_target - 1) / s4_target) + 63) / 64) * 64;
    const int64_t c4_cap = rows_kv >= 2 * sms ? kSparseMaxC4 : 1024;
    P.C4 = static_cast<int>(std::min<int64_t>(c4_cap, std::max<int64_t>(64, c4)));
    P.S4 = static_cast<int>(std::max<int64_t>(1, (kw + P.C4 - 1) / P.C4));
    // combine scratch: the sparse combine keeps G * S4 weights in the gather ring, the score
    // kernel's combine CTA G * S1 weights in its histogram scratch
    if (static_cast<int64_t>(G) * P.S4 > 8192 || static_cast<int64_t>(G) * P.S1 > 4096) return false;
    P.cand_cap = std::min<int64_t>(x.N, std::max<int64_t>(2048, (int64_t(1) << 24) / rows_kv));
    // one-launch decode step: one selection row per row block, kept logits, every candidate list
    // able to hold a whole pool, a split's pool keys within the kernel's shared-memory key buffer.
    // Taken for short caches, where the kernel chain is all launch and dependency latency (it
    // measured faster at N = 2K, slower from N = 32K on: its row barriers and per-CTA latency
    // chains then cost more than the launches they save); HS2_FUSED_DECODE=1 / 0 forces it on / off
    const char* want_fused = std::getenv("HS2_FUSED_DECODE");
    const int64_t tiles64 = (static_cast<int64_t>(x.N) + kKeyTile - 1) / kKeyTile;
    const bool fused_ok = x.T == 1 && P.RT == 1 && P.mat_logits && !P.umma && P.cand_cap >= x.N &&
                          ((tiles64 + P.S1 - 1) / P.S1) * kKeyTile <= kFusedKeyCap;
    P.fused = fused_ok && (want_fused ? want_fused[0] == '1' : x.N <= kFusedMaxN);
    if (P.fused && P.S1 * units > 2 * int64_t(sms)) {  // the one-launch kernel holds two CTAs per SM
        P.S1 = P.S2 = choose_splits(units, tiles, 2 * int64_t(sms), 256);
        P.fused = ((tiles64 + P.S1 - 1) / P.S1) * kKeyTile <= kFusedKeyCap;
    }
    const int64_t sparse_slots = P.fused ? std::max<int64_t>(P.S4, P.S1) : P.S4;
    P.kstride = ((static_cast<int64_t>(x.N) + 63) / 64) * 64;
    // bracketed selection (tcgen05 score sweep, many rows, large pools): a 1/16 tile sample per
    // row instead of every key, and candidate lists of max(4096, 3 k) (never more than N)
    const char* want_bracket = std::getenv("HS2_PREFILL_BRACKET");
    P.bracketed = P.umma && rows_kv >= int64_t(kRowsPerCtaTopkPerSM) * sms && x.N >= kBracketMinPool &&
                  4 * P.SS <= kMaxSegments && !(want_bracket && want_bracket[0] == '0');
    P.sstride = ((static_cast<int64_t>(x.N) + 128 * kSampleTileStride - 1) / (128 * kSampleTileStride)) * 128;
    P.bcap = std::min<int64_t>(x.N, std::max<int64_t>(4096, 3 * static_cast<int64_t>(x.k)));
    // the filtering sweep's epilogue warps (four per split) each fill their own segment of a
    // row's list: no atomics, and the keys of a tile are spread evenly over the four
    P.nseg = 4 * P.SS;
    P.seg_cap = static_cast<int>(P.bcap / P.nseg);
    // multi-CTA top-k: one chunk per CTA while that is a few waves; with many chunks in all
    // (1M keys x 64 rows) each CTA takes several, so launch and completion costs amortise
    const int64_t nchunks = (static_cast<int64_t>(x.N) + kTopkChunk - 1) / kTopkChunk;
    P.topk_ctas = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(nchunks, std::max<int64_t>(1, (12 * int64_t(sms) + rows_kv - 1) / rows_kv))));

    size_t off = 0;
    P.off_status = off; off += 256;
    P.off_tilectr = off; off = align_up(off + size_t(units) * 4, 256);  // cleared by every call's init
    P.init_bytes = off;
    P.off_pos = off; off = align_up(off + size_t(x.B) * 4, 256);  // decode step: the positions it runs at
    P.off_meta = off; off = align_up(off + rows_kv * kMetaInts * 4, 256);
    P.meta_end = off;
    // per-row global histograms: the multi-CTA top-k (few rows) and the kept-logits score kernel only
    const bool need_hist = P.mat_logits || rows_kv < int64_t(kRowsPerCtaTopkPerSM) * sms;
    P.off_hist = off; off = align_up(off + (need_hist ? rows_kv * kHistBins * 4 : 0), 256);
    P.zero_bytes = off;
    P.off_pf_ml = off; off = align_up(off + size_t(P.S1) * rows_q * 8, 256);
    P.off_pf_acc = off; off = align_up(off + size_t(P.S1) * rows_q * x.d * 4, 256);
    P.off_ps_ml = off; off = align_up(off + size_t(sparse_slots) * rows_q * 8, 256);
    P.off_ps_acc = off; off = align_up(off + size_t(sparse_slots) * rows_q * x.d * 4, 256);
    P.off_keys = off; off = align_up(off + size_t(rows_kv) * (P.bracketed ? P.sstride : P.kstride) * 4, 256);
    P.off_cand = off; off = align_up(off + size_t(rows_kv) * (P.bracketed ? P.bcap : P.cand_cap) * 8, 256);
    P.off_segcnt = off; off = align_up(off + (P.bracketed ? size_t(rows_kv) * P.nseg * 4 : 0), 256);
    P.off_logits = off;
    if (P.mat_logits) off = align_up(off + size_t(rows_kv) * x.N * G * 4, 256);
    P.total = off;
    *why = HS2_OK;
    return true;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// The cache as the kernels see it: base pointers plus layout and dtype.
struct KvView {
    const void* K;
    const void* V;
    KvSrc src;
};

KvView bf16_view(const void* K, const void* V) {
    KvView v{K, V, KvSrc{}};
    v.src.page_shift = -1;
    return v;
}

// Tensor map of a K or V cache for tiles of `rows` keys: contiguous caches as a 3-D view
// [B*Hkv][N][d], paged pools as 4-D [num_pages][Hkv][page_size][d] with boxes of
// min(page_size, rows) slots.  bf16: boxes of 64 dims (128 bytes), 128-byte swizzle; FP8: one box
// of d bytes per row, 128-byte swizzle for d = 128 and 64-byte for d = 64.  Zero fill out of range.
bool make_kv_map(CUtensorMap* m, const void* base, const Plan& p, int rows = kKeyTile) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t eb = p.fp8 ? 1 : 2;
    const CUtensorMapDataType dt = p.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = (p.fp8 && p.d == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    const cuuint32_t inner = p.fp8 ? cuuint32_t(p.d) : 64;
    const cuuint32_t es[4] = {1, 1, 1, 1};
    if (!p.paged) {
        const cuuint64_t dims[3] = {cuuint64_t(p.d), cuuint64_t(p.N), cuuint64_t(p.B) * p.Hkv};
        const cuuint64_t strides[2] = {cuuint64_t(p.d) * eb, cuuint64_t(p.N) * p.d * eb};
        const cuuint32_t box[3] = {inner, cuuint32_t(rows), 1};
        return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const cuuint64_t ps = cuuint64_t(p.page_size);
    const cuuint64_t dims[4] = {cuuint64_t(p.d), ps, cuuint64_t(p.Hkv), cuuint64_t(p.num_pages)};
    const cuuint64_t strides[3] = {cuuint64_t(p.d) * eb, ps * p.d * eb, cuuint64_t(p.Hkv) * ps * p.d * eb};
    const cuuint32_t box[4] = {inner, cuuint32_t(std::min<cuuint64_t>(ps, cuuint64_t(rows))), 1, 1};
    return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Ws {
    uint8_t* base;
    template <class T>
    T* at(size_t off) const { return reinterpret_cast<T*>(base + off); }
};

hs2_status check_ws(const Plan& p, void* ws, size_t ws_bytes) {
    if (!ws || !aligned(ws, 256) || ws_bytes < p.total) return HS2_ERR_WORKSPACE;
    return HS2_OK;
}

hs2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA; }

#define HS2_TRY(expr)                                 \
    do {                                              \
        const hs2_status s_ = cuda_status(expr);      \
        if (s_ != HS2_OK) return s_;                  \
    } while (0)

float scale_log2(const Plan& p) { return kLog2e / sqrtf(static_cast<float>(p.d)); }

AttnArgs attn_args(const Plan& p, const void* Q, const int32_t* pos, const KvView& kv, const Ws& w) {
    AttnArgs a{};
    a.Q = static_cast<const uint16_t*>(Q);
    a.pos = pos;
    a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.T = p.T; a.N = p.N; a.G = p.G; a.W = p.W;
    a.TQ = p.TQ; a.QB = p.QB; a.S = p.S1;
    a.scale_log2 = scale_log2(p);
    a.stream_kv = p.QB == 1 ? 1 : 0;  // one row block per kv head: each K/V tile is read once
    a.part_ml = w.at<float2>(p.off_pf_ml);
    a.part_acc = w.at<float>(p.off_pf_acc);
    a.kv = kv.src;
    a.status = w.at<unsigned>(p.off_status);
    a.tilectr = w.at<int>(p.off_tilectr);
    return a;
}

// Full-attention sweep.  combine: merge the splits here (otherwise the score kernel does it);
// zero_from/zero_to: workspace bytes the sweep clears for the kernels after it; pdl = false makes
// the sweep an ordinary launch (it then also sees what the kernel just before it wrote to pos).
hs2_status run_full(const Plan& p, const void* Qf, const KvView& kv, const int32_t* pos, void* O_full,
                    float* LSE_full, const Ws& w, bool keep_logits, bool combine, size_t zero_from, size_t zero_to,
                    cudaStream_t st, bool pdl = true) {
    CUtensorMap tmK, tmV;
    const int box_rows = p.umma ? 128 : kKeyTile;
    if (!make_kv_map(&tmK, kv.K, p, box_rows) || !make_kv_map(&tmV, kv.V, p, box_rows)) return HS2_ERR_CUDA;
    AttnArgs a = attn_args(p, Qf, pos, kv, w);
    a.logits = keep_logits ? w.at<float>(p.off_logits) : nullptr;
    if (zero_to > zero_from) {
        a.zero = w.at<uint4>(zero_from);
        a.zero_vec = static_cast<int64_t>((zero_to - zero_from) / 16);
    }
    if (p.umma)
        HS2_TRY(launch_umma_attn(p, tmK, tmV, a, st));
    else
        HS2_TRY(launch_full_attn(p, tmK, tmV, a, st, pdl));
    if (combine) {
        CombineArgs c{a.part_ml, a.part_acc, p.S1, p.rows_q, static_cast<uint16_t*>(O_full), LSE_full};
        HS2_TRY(launch_combine(p.d, c, st));
    }
    return HS2_OK;
}

TopkArgs topk_args(const Plan& p, const int32_t* pos, int32_t* idx, int32_t* cnt, const Ws& w) {
    TopkArgs t{};
    t.keys = w.at<uint32_t>(p.off_keys);
    t.kstride = p.kstride;
    t.pos = pos;
    t.Hkv = p.Hkv; t.T = p.T; t.N = p.N; t.k = p.k; t.W = p.W;
    t.rows = p.rows_kv;
    t.hist = w.at<unsigned>(p.off_hist);
    t.meta = w.at<int>(p.off_meta);
    t.cand = w.at<unsigned long long>(p.off_cand);
    t.cand_cap = p.cand_cap;
    t.idx = idx;
    t.cnt = cnt;
    t.status = w.at<unsigned>(p.off_status);
    return t;
}

// Selection from a second K sweep (needs LSE_full): keys, histogram + threshold, select.
hs2_status run_select_sweep(const Plan& p, const void* Qf, const KvView& kv, const float* LSE_full,
                            const int32_t* pos, int32_t* idx, int32_t* cnt, const Ws& w, cudaStream_t st) {
    CUtensorMap tmK;
    if (!make_kv_map(&tmK, kv.K, p, p.umma ? 128 : kKeyTile)) return HS2_ERR_CUDA;
    AttnArgs a = attn_args(p, Qf, pos, kv, w);
    a.lse = LSE_full;
    a.keys = w.at<uint32_t>(p.off_keys);
    a.kstride = p.kstride;
    a.k = p.k;
    a.S = p.S2;
    if (p.bracketed) {
        // sample -> bracket -> filtering sweep -> exact selection from the candidates
        TopkArgs t = topk_args(p, pos, idx, cnt, w);
        t.kstride = p.sstride;
        t.cand_cap = p.bcap;
        t.Q = static_cast<const uint16_t*>(Qf);
        t.K = static_cast<const uint16_t*>(kv.K);
        t.lse = LSE_full;
        t.Hq = p.Hq; t.G = p.G; t.d = p.d;
        t.scale_log2 = scale_log2(p);
        t.segcnt = w.at<int>(p.off_segcnt);
        t.nseg = p.nseg;
        t.seg_cap = p.seg_cap;
        a.score_mode = 1;
        a.kstride = p.sstride;
        HS2_TRY(launch_umma_score(p, tmK, a, st));
        HS2_TRY(launch_topk_bracket(p, t, st));
        a.score_mode = 2;
        a.cand = w.at<unsigned long long>(p.off_cand);
        a.cand_cap = p.bcap;
        a.seg_cap = p.seg_cap;
        a.segcnt = w.at<int>(p.off_segcnt);
        a.meta = w.at<int>(p.off_meta);
        HS2_TRY(launch_umma_score(p, tmK, a, st));
        HS2_TRY(launch_topk_finalize(p, t, st));
        return HS2_OK;
    }
    if (p.umma)
        HS2_TRY(launch_umma_score(p, tmK, a, st));
    else
        HS2_TRY(launch_score_sweep(p, p.S2, tmK, a, st));
    const TopkArgs t = topk_args(p, pos, idx, cnt, w);
    if (p.rows_kv >= int64_t(kRowsPerCtaTopkPerSM) * p.sms) {  // many rows: one CTA finishes each row
        HS2_TRY(launch_topk_rows(p, t, st));
    } else {
        HS2_TRY(launch_topk_hist(p, t, st));
        HS2_TRY(launch_topk_select(p, t, st));
    }
    return HS2_OK;
}

// Selection from the kept logits, with the full-attention combine folded in.
hs2_status run_select_kept(const Plan& p, const int32_t* pos, void* O_full, float* LSE_full, int32_t* idx,
                           int32_t* cnt, const Ws& w, cudaStream_t st) {
    ScoreArgs s{};
    s.logits = w.at<float>(p.off_logits);
    s.part_ml = w.at<float2>(p.off_pf_ml);
    s.part_acc = w.at<float>(p.off_pf_acc);
    s.S1 = p.S1;
    s.pos = pos;
    s.B = p.B; s.Hq = p.Hq; s.Hkv = p.Hkv; s.T = p.T; s.N = p.N; s.G = p.G; s.k = p.k; s.W = p.W;
    s.O = static_cast<uint16_t*>(O_full);
    s.LSE = LSE_full;
    s.keys = w.at<uint32_t>(p.off_keys);
    s.kstride = p.kstride;
    s.hist = w.at<unsigned>(p.off_hist);
    s.meta = w.at<int>(p.off_meta);
    s.status = w.at<unsigned>(p.off_status);
    HS2_TRY(launch_score_hist(p, s, st));
    HS2_TRY(launch_topk_select(p, topk_args(p, pos, idx, cnt, w), st));
    return HS2_OK;
}

hs2_status run_sparse(const Plan& p, const void* Qs, const KvView& kv, const int32_t* pos, const int32_t* idx,
                      const int32_t* cnt, void* O_sparse, float* LSE_sparse, const Ws& w, cudaStream_t st) {
    SparseArgs s{};
    s.Q = static_cast<const uint16_t*>(Qs);
    s.K = static_cast<const uint16_t*>(kv.K);
    s.V = static_cast<const uint16_t*>(kv.V);
    s.kv = kv.src;
    s.pos = pos;
    s.idx = idx;
    s.cnt = cnt;
    s.B = p.B; s.Hq = p.Hq; s.Hkv = p.Hkv; s.T = p.T; s.N = p.N; s.G = p.G; s.kw = p.k + p.W;
    s.C4 = p.C4; s.S4 = p.S4;
    s.scale_log2 = scale_log2(p);
    s.part_ml = w.at<float2>(p.off_ps_ml);
    s.part_acc = w.at<float>(p.off_ps_acc);
    s.meta = w.at<int>(p.off_meta);
    s.O = static_cast<uint16_t*>(O_sparse);
    s.LSE = LSE_sparse;
    s.status = w.at<unsigned>(p.off_status);
    HS2_TRY(launch_sparse_attn(p, s, st));
    return HS2_OK;
}

// The one-launch decode step; *done = false when its grid does not fit on the device at once
// (nothing launched).  The counters and histograms must have been cleared before.
hs2_status run_fused(const Plan& p, const void* Qf, const void* Qs, const KvView& kv, const int32_t* pos,
                     void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse, int32_t* idx, int32_t* cnt,
                     const Ws& w, cudaStream_t st, bool pdl, bool* done) {
    *done = false;
    CUtensorMap tmK, tmV;
    if (!make_kv_map(&tmK, kv.K, p, kKeyTile) || !make_kv_map(&tmV, kv.V, p, kKeyTile)) return HS2_ERR_CUDA;
    AttnArgs a = attn_args(p, Qf, pos, kv, w);
    a.logits = w.at<float>(p.off_logits);
    FusedArgs f{};
    f.Qs = static_cast<const uint16_t*>(Qs);
    f.K = kv.K;
    f.V = kv.V;
    f.k = p.k;
    f.O_full = static_cast<uint16_t*>(O_full);
    f.LSE_full = LSE_full;
    f.O_sparse = static_cast<uint16_t*>(O_sparse);
    f.LSE_sparse = LSE_sparse;
    f.idx = idx;
    f.cnt = cnt;
    f.hist = w.at<unsigned>(p.off_hist);
    f.meta = w.at<int>(p.off_meta);
    f.cand = w.at<unsigned long long>(p.off_cand);
    f.cand_cap = p.cand_cap;
    f.ps_ml = w.at<float2>(p.off_ps_ml);
    f.ps_acc = w.at<float>(p.off_ps_acc);
    HS2_TRY(launch_decode_fused(p, tmK, tmV, a, f, st, pdl, done));
    return HS2_OK;
}

// The whole step after the status word is clear; pos is where the kernels read positions.
hs2_status run_step(const Plan& p, const void* Qf, const void* Qs, const KvView& kv, const int32_t* pos,
                    void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse, int32_t* idx, int32_t* cnt,
                    const Ws& w, cudaStream_t st, bool first_pdl) {
    if (p.fused) {  // the caller cleared the counters and histograms (init over zero_bytes)
        bool done = false;
        const hs2_status s = run_fused(p, Qf, Qs, kv, pos, O_full, O_sparse, LSE_full, LSE_sparse, idx, cnt, w, st,
                                       first_pdl, &done);
        if (s != HS2_OK || done) return s;
    }
    hs2_status s = run_full(p, Qf, kv, pos, O_full, LSE_full, w, p.mat_logits, !p.mat_logits, p.off_meta,
                            p.zero_bytes, st, first_pdl);
    if (s != HS2_OK) return s;
    s = p.mat_logits ? run_select_kept(p, pos, O_full, LSE_full, idx, cnt, w, st)
                     : run_select_sweep(p, Qf, kv, LSE_full, pos, idx, cnt, w, st);
    if (s != HS2_OK) return s;
    return run_sparse(p, Qs, kv, pos, idx, cnt, O_sparse, LSE_sparse, w, st);
}

bool ok16(const void* p) { return p && aligned(p, 16); }
bool ok4(const void* p) { return p && aligned(p, 4); }
// idx has k + W entries per row; with k + W = 0 it is empty and may be null.
bool ok_idx(const void* p, const Plan& P) { return (P.k + P.W == 0 && !p) || ok4(p); }

KvShape kv_shape(const hs2_kv_cache* c) {
    KvShape s;
    if (c) {
        s.fp8 = c->dtype == HS2_KV_FP8_E4M3 ? 1 : (c->dtype == HS2_KV_BF16 ? 0 : -1);
        s.page_size = c->page_size;
        s.max_pages = c->max_pages;
        s.num_pages = c->num_pages;
    }
    return s;
}

// Plan for a cache descriptor, and its pointer checks; *view receives the kernels' view.
bool plan_kv(const hs2_dims* dims, const hs2_kv_cache* c, Plan* p, KvView* view, hs2_status* why) {
    *why = HS2_ERR_INVALID_ARG;
    if (!c) return false;
    if (!make_plan(dims, p, why, kv_shape(c))) return false;
    *why = HS2_ERR_INVALID_ARG;
    if (!ok16(c->K) || !ok16(c->V)) return false;
    if (p->paged && !ok4(c->page_table)) return false;
    if (p->fp8 && (!ok4(c->k_scale) || !ok4(c->v_scale))) return false;
    view->K = c->K;
    view->V = c->V;
    view->src = KvSrc{};
    view->src.fp8 = p->fp8 ? 1 : 0;
    view->src.page_shift = -1;
    if (p->paged) {
        int sh = 0;
        while ((1 << sh) < p->page_size) ++sh;
        view->src.page_shift = sh;
        view->src.max_pages = p->max_pages;
        view->src.num_pages = p->num_pages;
        view->src.page_table = c->page_table;
    }
    if (p->fp8) {
        view->src.k_scale = c->k_scale;
        view->src.v_scale = c->v_scale;
    }
    *why = HS2_OK;
    return true;
}

hs2_status full_attn_impl(const Plan& p, const KvView& kv, const void* Q_full, const int32_t* pos, void* O_full,
                          float* LSE_full, void* ws, size_t ws_bytes, void* stream) {
    if (!ok16(Q_full) || !ok4(pos) || !ok16(O_full) || !ok4(LSE_full)) return HS2_ERR_INVALID_ARG;
    if (check_ws(p, ws, ws_bytes) != HS2_OK) return HS2_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Ws w{static_cast<uint8_t*>(ws)};
    trace_call_begin(st);
    HS2_TRY(launch_init(ws, p.init_bytes, st));  // status word and the sweep's tile counters
    return run_full(p, Q_full, kv, pos, O_full, LSE_full, w, false, true, 0, 0, st);
}

hs2_status select_impl(const Plan& p, const KvView& kv, const void* Q_full, const float* LSE_full,
                       const int32_t* pos, int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
    if (!ok16(Q_full) || !ok4(LSE_full) || !ok4(pos) || !ok_idx(idx, p) || !ok4(cnt)) return HS2_ERR_INVALID_ARG;
    if (check_ws(p, ws, ws_bytes) != HS2_OK) return HS2_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Ws w{static_cast<uint8_t*>(ws)};
    trace_call_begin(st);
    HS2_TRY(launch_init(ws, p.zero_bytes, st));
    return run_select_sweep(p, Q_full, kv, LSE_full, pos, idx, cnt, w, st);
}

hs2_status sparse_impl(const Plan& p, const KvView& kv, const void* Q_sparse, const int32_t* pos, const int32_t* idx,
                       const int32_t* cnt, void* O_sparse, float* LSE_sparse, void* ws, size_t ws_bytes,
                       void* stream) {
    if (!ok16(Q_sparse) || !ok4(pos) || !ok_idx(idx, p) || !ok4(cnt) || !ok16(O_sparse) || !ok4(LSE_sparse))
        return HS2_ERR_INVALID_ARG;
    if (check_ws(p, ws, ws_bytes) != HS2_OK) return HS2_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Ws w{static_cast<uint8_t*>(ws)};
    trace_call_begin(st);
    HS2_TRY(launch_init(ws, p.meta_end, st));
    return run_sparse(p, Q_sparse, kv, pos, idx, cnt, O_sparse, LSE_sparse, w, st);
}

bool step_outputs_ok(const Plan& p, const void* Q_full, const void* Q_sparse, const void* O_full,
                     const void* O_sparse, const float* LSE_full, const float* LSE_sparse, const int32_t* idx,
                     const int32_t* cnt) {
    return ok16(Q_full) && ok16(Q_sparse) && ok16(O_full) && ok16(O_sparse) && ok4(LSE_full) && ok4(LSE_sparse) &&
           ok_idx(idx, p) && ok4(cnt);
}

hs2_status step_impl(const Plan& p, const KvView& kv, const void* Q_full, const void* Q_sparse, const int32_t* pos,
                     void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse, int32_t* idx, int32_t* cnt,
                     void* ws, size_t ws_bytes, void* stream) {
    if (!step_outputs_ok(p, Q_full, Q_sparse, O_full, O_sparse, LSE_full, LSE_sparse, idx, cnt) || !ok4(pos))
        return HS2_ERR_INVALID_ARG;
    if (check_ws(p, ws, ws_bytes) != HS2_OK) return HS2_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Ws w{static_cast<uint8_t*>(ws)};
    trace_call_begin(st);
    // status word and the sweep's tile counters (and, for the one-launch decode step, the per-row
    // counters and histograms; otherwise the full sweep clears those for the kernels after it)
    HS2_TRY(launch_init(ws, p.fused ? p.zero_bytes : p.init_bytes, st));
    return run_step(p, Q_full, Q_sparse, kv, pos, O_full, O_sparse, LSE_full, LSE_sparse, idx, cnt, w, st, true);
}

AppendArgs append_args(const Plan& p, const KvView& kv, const void* K_new, const void* V_new, const int32_t* pos,
                       const Ws& w) {
    AppendArgs a{};
    a.K_new = static_cast<const uint16_t*>(K_new);
    a.V_new = static_cast<const uint16_t*>(V_new);
    a.K = const_cast<void*>(kv.K);
    a.V = const_cast<void*>(kv.V);
    a.kv = kv.src;
    a.pos_in = pos;
    a.B = p.B; a.Hkv = p.Hkv; a.T = p.T; a.N = p.N; a.d = p.d;
    a.status = w.at<unsigned>(p.off_status);
    return a;
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" {

size_t hs2_workspace_size(const hs2_dims* dims) {
    Plan p;
    hs2_status why;
    return make_plan(dims, &p, &why) ? p.total : 0;
}

size_t hs2_workspace_size_kv(const hs2_dims* dims, const hs2_kv_cache* cache) {
    Plan p;
    hs2_status why;
    if (!cache) return 0;
    return make_plan(dims, &p, &why, kv_shape(cache)) ? p.total : 0;
}

hs2_status hs2_full_attn(const hs2_dims* dims, const void* Q_full, const void* K, const void* V, const int32_t* pos,
                         void* O_full, float* LSE_full, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    hs2_status why;
    if (!make_plan(dims, &p, &why)) return why;
    if (!ok16(K) || !ok16(V)) return HS2_ERR_INVALID_ARG;
    return full_attn_impl(p, bf16_view(K, V), Q_full, pos, O_full, LSE_full, ws, ws_bytes, stream);
}

hs2_status hs2_full_attn_kv(const hs2_dims* dims, const void* Q_full, const hs2_kv_cache* cache, const int32_t* pos,
                            void* O_full, float* LSE_full, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    KvView kv;
    hs2_status why;
    if (!plan_kv(dims, cache, &p, &kv, &why)) return why;
    return full_attn_impl(p, kv, Q_full, pos, O_full, LSE_full, ws, ws_bytes, stream);
}

hs2_status hs2_select(const hs2_dims* dims, const void* Q_full, const void* K, const float* LSE_full,
                      const int32_t* pos, int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    hs2_status why;
    if (!make_plan(dims, &p, &why)) return why;
    if (!ok16(K)) return HS2_ERR_INVALID_ARG;
    return select_impl(p, bf16_view(K, K), Q_full, LSE_full, pos, idx, cnt, ws, ws_bytes, stream);
}

hs2_status hs2_select_kv(const hs2_dims* dims, const void* Q_full, const hs2_kv_cache* cache, const float* LSE_full,
                         const int32_t* pos, int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    KvView kv;
    hs2_status why;
    if (!plan_kv(dims, cache, &p, &kv, &why)) return why;
    return select_impl(p, kv, Q_full, LSE_full, pos, idx, cnt, ws, ws_bytes, stream);
}

hs2_status hs2_sparse_attn(const hs2_dims* dims, const void* Q_sparse, const void* K, const void* V,
                           const int32_t* pos, const int32_t* idx, const int32_t* cnt, void* O_sparse,
                           float* LSE_sparse, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    hs2_status why;
    if (!make_plan(dims, &p, &why)) return why;
    if (!ok16(K) || !ok16(V)) return HS2_ERR_INVALID_ARG;
    return sparse_impl(p, bf16_view(K, V), Q_sparse, pos, idx, cnt, O_sparse, LSE_sparse, ws, ws_bytes, stream);
}

hs2_status hs2_sparse_attn_kv(const hs2_dims* dims, const void* Q_sparse, const hs2_kv_cache* cache,
                              const int32_t* pos, const int32_t* idx, const int32_t* cnt, void* O_sparse,
                              float* LSE_sparse, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    KvView kv;
    hs2_status why;
    if (!plan_kv(dims, cache, &p, &kv, &why)) return why;
    return sparse_impl(p, kv, Q_sparse, pos, idx, cnt, O_sparse, LSE_sparse, ws, ws_bytes, stream);
}

hs2_status hs2_step(const hs2_dims* dims, const void* Q_full, const void* Q_sparse, const void* K, const void* V,
                    const int32_t* pos, void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse,
                    int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    hs2_status why;
    if (!make_plan(dims, &p, &why)) return why;
    if (!ok16(K) || !ok16(V)) return HS2_ERR_INVALID_ARG;
    return step_impl(p, bf16_view(K, V), Q_full, Q_sparse, pos, O_full, O_sparse, LSE_full, LSE_sparse, idx, cnt, ws,
                     ws_bytes, stream);
}

hs2_status hs2_step_kv(const hs2_dims* dims, const void* Q_full, const void* Q_sparse, const hs2_kv_cache* cache,
                       const int32_t* pos, void* O_full, void* O_sparse, float* LSE_full, float* LSE_sparse,
                       int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    KvView kv;
    hs2_status why;
    if (!plan_kv(dims, cache, &p, &kv, &why)) return why;
    return step_impl(p, kv, Q_full, Q_sparse, pos, O_full, O_sparse, LSE_full, LSE_sparse, idx, cnt, ws, ws_bytes,
                     stream);
}

hs2_status hs2_kv_append(const hs2_dims* dims, const hs2_kv_cache* cache, const void* K_new, const void* V_new,
                         const int32_t* pos, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    KvView kv;
    hs2_status why;
    if (!plan_kv(dims, cache, &p, &kv, &why)) return why;
    if (!ok16(K_new) || !ok16(V_new) || !ok4(pos)) return HS2_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, 256) || ws_bytes < 256) return HS2_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Ws w{static_cast<uint8_t*>(ws)};
    trace_call_begin(st);
    HS2_TRY(launch_init(ws, 256, st));
    AppendArgs a = append_args(p, kv, K_new, V_new, pos, w);
    a.status = static_cast<unsigned*>(ws);
    HS2_TRY(launch_append(a, st));
    return HS2_OK;
}

hs2_status hs2_decode_step(const hs2_dims* dims, const hs2_kv_cache* cache, const void* Q_full, const void* Q_sparse,
                           const void* K_new, const void* V_new, int32_t* pos, void* O_full, void* O_sparse,
                           float* LSE_full, float* LSE_sparse, int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes,
                           void* stream) {
    Plan p;
    KvView kv;
    hs2_status why;
    if (!plan_kv(dims, cache, &p, &kv, &why)) return why;
    if (p.T != 1) return HS2_ERR_INVALID_ARG;
    if (!step_outputs_ok(p, Q_full, Q_sparse, O_full, O_sparse, LSE_full, LSE_sparse, idx, cnt) || !ok16(K_new) ||
        !ok16(V_new) || !ok4(pos))
        return HS2_ERR_INVALID_ARG;
    if (check_ws(p, ws, ws_bytes) != HS2_OK) return HS2_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Ws w{static_cast<uint8_t*>(ws)};
    trace_call_begin(st);
    HS2_TRY(launch_init(ws, p.fused ? p.zero_bytes : p.init_bytes, st));  // as in step_impl
    // the new tokens go in and pos advances; the step then reads the positions from ws.  The full
    // sweep is an ordinary launch, so it starts after the append has completed and every kernel
    // after it sees the new tokens and positions.
    AppendArgs a = append_args(p, kv, K_new, V_new, pos, w);
    a.advance = 1;
    a.pos_out = pos;
    a.pos_new = w.at<int32_t>(p.off_pos);
    HS2_TRY(launch_append(a, st));
    return run_step(p, Q_full, Q_sparse, kv, w.at<int32_t>(p.off_pos), O_full, O_sparse, LSE_full, LSE_sparse, idx,
                    cnt, w, st, false);
}

hs2_status hs2_read_device_status(const void* ws, void* stream, uint32_t* bits) {
    if (!ws || !bits || !aligned(ws, 256)) return HS2_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    HS2_TRY(cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st));
    HS2_TRY(cudaStreamSynchronize(st));
    *bits = v;
    return (v & ~HS2_DEV_CAND_OVERFLOW) ? HS2_ERR_DEVICE : HS2_OK;
}

const char* hs2_status_string(hs2_status s) {
    switch (s) {
        case HS2_OK: return "ok";
        case HS2_ERR_INVALID_ARG: return "invalid argument";
        case HS2_ERR_UNSUPPORTED: return "unsupported shape";
        case HS2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case HS2_ERR_CUDA: return "CUDA error";
        case HS2_ERR_DEVICE: return "device status bits set";
    }
    return "unknown status";
}

uint32_t hs2_version(void) { return (1u << 16) | 1u; }

}  // extern "C"
