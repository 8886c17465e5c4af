// Full-attention layer and selection-score sweeps over the shared KV cache (sm_100a), for bf16
// or FP8 E4M3 caches, contiguous or paged (the TMA producer in attn_sweep.cuh).
//
// full_attn_kernel: the split-K flash-decode sweep (attn_sweep.cuh) as a kernel of its own.
//
// score_sweep_kernel: the second K sweep used when logits are not kept.  It recomputes
// QK^T tile by tile, subtracts each head's LSE and takes the max over the G heads of the
// kv head: the GQA-max log-softmax selection score (in base-2 units), written as an
// order-preserving uint32 key for every pool key j <= pos - W.
//
// combine_kernel: split partials -> bf16 O and natural-log LSE (used when the combine is not
// fused into the next kernel).
#include <algorithm>
#include <cstdlib>

#include "attn_sweep.cuh"
#include "combine.cuh"
#include "topk_common.cuh"
#include "hs2_internal.h"

namespace hs2 {

// ====================================================================== full attention

template <int D, int RT, int NC, int STAGES, bool KEEP_LOGITS, bool FP8, bool TR, bool DYN>
__global__ void __launch_bounds__((NC + 1) * 32)
    full_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    pdl_trigger();
    if (a.zero) {  // clear the next kernels' per-row counters and histograms, spread over all CTAs
        const int64_t cta = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
        const int64_t nthr = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
        for (int64_t i = cta * blockDim.x + threadIdx.x; i < a.zero_vec; i += nthr)
            a.zero[i] = make_uint4(0, 0, 0, 0);
    }
    int2 range;
    full_sweep<D, RT, NC, STAGES, KEEP_LOGITS, FP8, TR, DYN>(&tmK, &tmV, a, smem, blockIdx.x, blockIdx.y, &range);
    // The sweep reads nothing its predecessor writes, but it must not complete before the
    // predecessor does (later kernels rely on that chain).
    pdl_wait();
}

// ====================================================================== score sweep (second K pass)
//
// MMA row m of 16-row tile rt holds query rt*Q8 + t_in, head g, with Q8 = 16/G queries per tile
// and, for m < 8: t_in = m % Q8, g = m / Q8; for m >= 8: the same query and head g + G/2 (G = 1:
// query m).  A lane's two accumulator rows m and m+8 are then two heads of one query, so the max
// over the G heads is one local max plus log2(G/2) lane shuffles (instead of log2(G)).

template <int D, int RT, int NC, int STAGES, bool FP8>
__global__ void __launch_bounds__((NC + 1) * 32)
    score_sweep_kernel(const __grid_constant__ CUtensorMap tmK, const AttnArgs a) {
    constexpr int NKS = NC / RT;
    constexpr int KW = kKeyTile / NKS;
    using L = StreamSmem<D, STAGES, 1, FP8 ? 1 : 2>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
    int* s_pos = reinterpret_cast<int*>(smem + L::kMiscOff + 16);  // per query of the block
    __shared__ int s_row[16 * RT], s_rank[16 * RT];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, unit = blockIdx.y;
    const int bh = unit / a.QB, qb = unit % a.QB;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const int G = a.G;
    const int Q8 = G >= 2 ? 16 / G : 16;
    const int nq = a.TQ;  // queries in this row block (the last block may have fewer valid)
    pdl_trigger();

    for (int q = tid; q < nq; q += blockDim.x) {
        const int t = qb * a.TQ + q;
        int p = -1, rank = 0;
        if (t < a.T) {
            p = clamp_pos(a.pos[b * a.T + t], a.N, nullptr);
            const int P = max(0, p - a.W + 1);
            const int keff = min(a.k, P);
            rank = keff > 0 && keff < P;  // only these rows need ranked keys
        }
        s_pos[q] = p;
        s_row[q] = bh * a.T + t;
        s_rank[q] = rank;
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    // only pool keys (j <= pos - W) of rows that need ranking are scored
    int jmax = -1;
    for (int q = 0; q < nq; ++q)
        if (s_pos[q] >= 0 && s_rank[q]) jmax = max(jmax, s_pos[q] - a.W);
    const int ntiles = jmax >= 0 ? (jmax + kKeyTile) / kKeyTile : 0;
    const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.S);
    const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.S);
    const int nt = t_end - t_begin;

    if (warp == NC) {
        if (lane == 0)
            produce_tiles<D, STAGES, 1, FP8>(&tmK, &tmK, ring, full, empty, abort_flag, t_begin, nt, bh, a.Hkv, a.kv,
                                             a.status, a.stream_kv != 0);
        __syncwarp();
    }
    const int rt = warp % RT, ks = warp / RT;
    const int m_lo = lane >> 2, c = lane & 3;
    // (query in block, head) of MMA rows m_lo and m_lo + 8 of tile rt
    int tq_lo, g_lo, tq_hi, g_hi;
    if (G >= 2) {
        tq_lo = tq_hi = rt * Q8 + m_lo % Q8;
        g_lo = m_lo / Q8;
        g_hi = g_lo + G / 2;
    } else {
        tq_lo = rt * 16 + m_lo;
        tq_hi = tq_lo + 8;
        g_lo = g_hi = 0;
    }
    auto row_q = [&](int tq, int gg) -> int {
        const int t = qb * a.TQ + tq;
        if (tq >= a.TQ || t >= a.T) return -1;
        return (b * a.Hq + h * G + gg) * a.T + t;
    };
    const bool writer = G >= 2 ? (m_lo < Q8) : true;
    bool nonfinite = false;
    if (warp < NC) {
        QTileOf<D, FP8> q;
        const int rq_lo = row_q(tq_lo, g_lo), rq_hi = row_q(tq_hi, g_hi);
        q.load(a.Q, rq_lo >= 0 ? static_cast<int64_t>(rq_lo) * D : -1, rq_hi >= 0 ? static_cast<int64_t>(rq_hi) * D : -1);
        const float kscale = FP8 ? a.kv.k_scale[bh] : 1.f;
        const float f2[2] = {logit_factor<D, FP8>(q, 0, a.scale_log2, kscale),
                             logit_factor<D, FP8>(q, 1, a.scale_log2, kscale)};
        pdl_wait();  // LSE_full comes from the previous kernel
        // base-2 LSE of the two rows (+inf for padding rows so their scores are -inf)
        const float lse_lo = rq_lo >= 0 ? a.lse[rq_lo] * kLog2e : INFINITY;
        const float lse_hi = rq_hi >= 0 ? a.lse[rq_hi] * kLog2e : INFINITY;
        // last pool key of each row's query (-1: nothing to rank)
        const int pl_lo = (rq_lo >= 0 && s_rank[tq_lo]) ? s_pos[tq_lo] - a.W : -1;
        const int pl_hi = (rq_hi >= 0 && s_rank[tq_hi]) ? s_pos[tq_hi] - a.W : -1;
        uint32_t* key_lo = rq_lo >= 0 ? a.keys + static_cast<int64_t>(s_row[tq_lo]) * a.kstride : nullptr;
        uint32_t* key_hi = rq_hi >= 0 ? a.keys + static_cast<int64_t>(s_row[tq_hi]) * a.kstride : nullptr;
        const int key0 = ks * KW;
        for (int i = 0; i < nt; ++i) {
            const int stage = i % STAGES;
            if (!mbar_wait(&full[stage], (i / STAGES) & 1, a.status)) {
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            const uint32_t kbase = smem_u32(ring + stage * L::kStageBytes);
            float sc[KW / 8][4];
            qk_any<D, KW, FP8>(q, kbase, key0, sc);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            const int jb = (t_begin + i) * kKeyTile + key0 + 2 * c;
#pragma unroll
            for (int n = 0; n < KW / 8; ++n) {
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) v[e] = sc[n][e] * f2[e >> 1] - ((e < 2) ? lse_lo : lse_hi);
                if (G >= 2) {
                    v[0] = nan_max(v[0], v[2]);  // heads g and g + G/2 of the same query
                    v[1] = nan_max(v[1], v[3]);
                    for (int off = 4 * Q8; off < 32; off <<= 1) {
                        v[0] = nan_max(v[0], __shfl_xor_sync(0xffffffffu, v[0], off));
                        v[1] = nan_max(v[1], __shfl_xor_sync(0xffffffffu, v[1], off));
                    }
                }
                if (writer) {
                    const int nrow = G >= 2 ? 1 : 2;
                    for (int r = 0; r < nrow; ++r) {
                        const int pl = r == 0 ? pl_lo : pl_hi;
                        uint32_t* kr = r == 0 ? key_lo : key_hi;
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int j = jb + n * 8 + e;
                            if (j <= pl) {
                                const float sv = v[2 * r + e];
                                nonfinite |= (sv != sv);
                                kr[j] = score_key(sv);
                            }
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    if (__syncthreads_or(nonfinite) && tid == 0) set_status(a.status, HS2_DEV_NONFINITE);
}

// ====================================================================== combine

template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
    __shared__ float wbuf[8][256];
    const int warp = threadIdx.x >> 5;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp;
    pdl_trigger();
    pdl_wait();
    if (row >= a.rows) return;
    warp_combine_row<D>(a.part_ml, a.part_acc, a.S, a.rows, row, wbuf[warp], a.O, a.LSE);
}

// ====================================================================== launchers

namespace {

constexpr int64_t kDynMinTiles = 128;  // key tiles per CTA from which the sweep is scheduled dynamically

// HS2_TRANSPOSED=0 keeps the query-rows-as-M warp attention for decode row blocks
bool transposed_decode() {
    const char* env = std::getenv("HS2_TRANSPOSED");
    return !(env && env[0] == '0');
}

template <class Kern>
cudaError_t set_smem(Kern kern, int bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, int RT, bool KEEP, bool FP8, bool TR = false, int DYN = -1>
cudaError_t full_attn_variant(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                              cudaStream_t st, bool pdl) {
    // Long key ranges per CTA (at least kDynMinTiles tiles: the 1M-token decode) are handed out in
    // chunks from a counter, so that CTAs slowed by memory contention take fewer of them (4-5 %
    // faster there); shorter ranges keep a fixed split (the counter cost more than it saved at
    // the 32K-token batch and broke even at 128K), which also keeps their summation order fixed.
    // HS2_DYN_SWEEP=1 / 0 forces either.
    if constexpr (DYN < 0) {
        const char* env = std::getenv("HS2_DYN_SWEEP");
        const int64_t tiles = (static_cast<int64_t>(p.N) + kKeyTile - 1) / kKeyTile;
        const bool dyn = env ? env[0] == '1' : (tiles + p.S1 - 1) / p.S1 >= kDynMinTiles;
        return dyn ? full_attn_variant<D, RT, KEEP, FP8, TR, 1>(p, tmK, tmV, a, st, pdl)
                   : full_attn_variant<D, RT, KEEP, FP8, TR, 0>(p, tmK, tmV, a, st, pdl);
    }
    // at most 8 query-head rows per row block: the transposed warp attention
    if constexpr (RT == 1 && !TR)
        if (p.T * p.G <= 8 && transposed_decode())
            return full_attn_variant<D, RT, KEEP, FP8, true, DYN>(p, tmK, tmV, a, st, pdl);
    constexpr int NC = RT >= 8 ? 8 : 4;
    // ring of 96 KB (bf16: 3 stages at d = 128, 6 at d = 64; FP8 twice as many), two CTAs per SM;
    // the transposed FP8 form (96 registers) takes a 64 KB ring and three CTAs per SM
    constexpr int STAGES = (TR && FP8) ? (D == 128 ? 4 : 8) : (D == 128 ? 3 : 6) * (FP8 ? 2 : 1);
    using L = StreamSmem<D, STAGES, 2, FP8 ? 1 : 2>;
    static_assert(L::kRingBytes >= RT * merge_floats<D, NC / RT>() * 4, "merge scratch must fit in the ring");
    auto kern = full_attn_kernel<D, RT, NC, STAGES, KEEP, FP8, TR, (DYN == 1)>;
    cudaError_t e = set_smem(kern, L::kBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(p.S1, p.B * p.Hkv * p.QB);
    e = launch_pdl_opt(pdl, kern, grid, dim3((NC + 1) * 32), L::kBytes, st, tmK, tmV, a);
    trace_mark(KEEP ? "full_attn_keep_logits" : "full_attn", st);
    return e;
}

template <int D, int RT, bool FP8>
cudaError_t score_sweep_variant(const Plan& p, int splits, const CUtensorMap& tmK, const AttnArgs& a,
                                cudaStream_t st) {
    constexpr int NC = RT >= 8 ? 8 : 4;
    constexpr int STAGES = (D == 128 ? 6 : 12) * (FP8 ? 2 : 1);
    using L = StreamSmem<D, STAGES, 1, FP8 ? 1 : 2>;
    auto kern = score_sweep_kernel<D, RT, NC, STAGES, FP8>;
    cudaError_t e = set_smem(kern, L::kBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(splits, p.B * p.Hkv * p.QB);
    e = launch_pdl(kern, grid, dim3((NC + 1) * 32), L::kBytes, st, tmK, a);
    trace_mark("score_sweep", st);
    return e;
}

}  // namespace

cudaError_t launch_full_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st, bool pdl) {
    const bool keep = a.logits != nullptr;
#define HS2_FA(D_, RT_, F_)                                                                              \
    if (p.d == D_ && p.RT == RT_ && p.fp8 == F_)                                                         \
        return (keep && RT_ == 1) ? full_attn_variant<D_, RT_, (RT_ == 1), F_>(p, tmK, tmV, a, st, pdl)  \
                                  : full_attn_variant<D_, RT_, false, F_>(p, tmK, tmV, a, st, pdl);
    HS2_FA(64, 1, false) HS2_FA(64, 2, false) HS2_FA(64, 4, false) HS2_FA(64, 8, false)
    HS2_FA(128, 1, false) HS2_FA(128, 2, false) HS2_FA(128, 4, false) HS2_FA(128, 8, false)
    HS2_FA(64, 1, true) HS2_FA(64, 2, true) HS2_FA(64, 4, true) HS2_FA(64, 8, true)
    HS2_FA(128, 1, true) HS2_FA(128, 2, true) HS2_FA(128, 4, true) HS2_FA(128, 8, true)
#undef HS2_FA
    return cudaErrorInvalidValue;
}

cudaError_t launch_score_sweep(const Plan& p, int splits, const CUtensorMap& tmK, const AttnArgs& a,
                               cudaStream_t st) {
#define HS2_SS(D_, RT_, F_) \
    if (p.d == D_ && p.RT == RT_ && p.fp8 == F_) return score_sweep_variant<D_, RT_, F_>(p, splits, tmK, a, st);
    HS2_SS(64, 1, false) HS2_SS(64, 2, false) HS2_SS(64, 4, false) HS2_SS(64, 8, false)
    HS2_SS(128, 1, false) HS2_SS(128, 2, false) HS2_SS(128, 4, false) HS2_SS(128, 8, false)
    HS2_SS(64, 1, true) HS2_SS(64, 2, true) HS2_SS(64, 4, true) HS2_SS(64, 8, true)
    HS2_SS(128, 1, true) HS2_SS(128, 2, true) HS2_SS(128, 4, true) HS2_SS(128, 8, true)
#undef HS2_SS
    return cudaErrorInvalidValue;
}

// Clears the start of the workspace (status word, counters) for the call that launches it.  It is
// launched with programmatic serialisation, so it is resident while the stream's previous kernel
// drains; it writes only after that kernel has completed (pdl_wait -- and since every kernel of
// this library waits for its predecessor before it ends, the whole previous call has completed),
// and lets the call's next kernel launch only after its own writes (the trigger comes last), so
// nothing of this call touches the workspace while the previous call might still use it.
__global__ void __launch_bounds__(256) init_kernel(uint4* p, int64_t n) {
    pdl_wait();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = make_uint4(0, 0, 0, 0);
    pdl_trigger();
}

cudaError_t launch_init(void* ws, size_t bytes, cudaStream_t st) {
    const int64_t n = static_cast<int64_t>(bytes / 16);
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(8 * num_sms(), std::max<int64_t>(1, (n + 255) / 256)));
    const cudaError_t e = launch_pdl(init_kernel, dim3(blocks), dim3(256), 0, st, static_cast<uint4*>(ws), n);
    trace_mark("init", st);
    return e;
}

cudaError_t launch_combine(int d, const CombineArgs& a, cudaStream_t st) {
    const unsigned blocks = static_cast<unsigned>((a.rows + 7) / 8);
    const cudaError_t e = d == 128 ? launch_pdl(combine_kernel<128>, dim3(blocks), dim3(256), 0, st, a)
                                   : launch_pdl(combine_kernel<64>, dim3(blocks), dim3(256), 0, st, a);
    trace_mark("combine", st);
    return e;
}

}  // namespace hs2
