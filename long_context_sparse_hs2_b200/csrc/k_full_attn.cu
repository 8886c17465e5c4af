// Full-attention layer and selection-score sweeps over the shared KV cache (sm_100a).
//
// full_attn_kernel: split-K flash-decode.  One CTA owns one row block (the G query
// heads of one kv head for TQ consecutive queries = 16*RT MMA rows) and one contiguous
// range of 64-key tiles.  A producer warp streams K and V tiles into a STAGES-deep
// shared-memory ring with TMA (3-D tensor map, 128-byte swizzle, no multicast), signalled
// through mbarriers; NC consumer warps compute QK^T and PV with bf16 mma.sync and keep an
// online softmax in base-2 units.  The CTA writes one split partial (m, l, O) per row;
// combine_kernel merges the splits with the log-sum-exp correction ("Simplified Sparse
// Attention via Gist Tokens", section 3.6, "three-kernel split-K sparse flash-decode").
// With KEEP_LOGITS the sweep also stores every visible base-2 logit, [row][key][head], so
// the selection score can be formed without reading K a second time.
//
// score_sweep_kernel: the second K sweep used when logits are not kept.  It recomputes
// QK^T tile by tile, subtracts each head's LSE and takes the max over the G heads of the
// kv head: the GQA-max log-softmax selection score (in base-2 units), written as an
// order-preserving uint32 key for every pool key j <= pos - W.
//
// combine_kernel: split partials -> bf16 O and natural-log LSE (used when the combine is not
// fused into the next kernel).
#include <algorithm>

#include "attn_core.cuh"
#include "combine.cuh"
#include "hs2_internal.h"

namespace hs2 {

namespace {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ int clamp_pos(int p, int N, unsigned* status) {
    if (p < 0 || p >= N) {
        set_status(status, HS2_DEV_BAD_POS);
        p = p < 0 ? 0 : N - 1;
    }
    return p;
}

// Shared-memory layout of the streaming kernels (after 1 KB alignment).
template <int D, int STAGES, int TENSORS>
struct StreamSmem {
    static constexpr int kTileBytes = kKeyTile * D * 2;                 // one tensor, one tile
    static constexpr int kStageBytes = TENSORS * kTileBytes;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kBarOff = kRingBytes;                           // full[STAGES], empty[STAGES]
    static constexpr int kMiscOff = kBarOff + 2 * STAGES * 8;            // abort flag + row positions
    static constexpr int kBytes = kMiscOff + 16 + 128 * 4 + 1024;        // + alignment slack
};

// Producer side of the TMA ring: stream tiles [t_begin, t_begin + nt) of kv slice bh.
template <int D, int STAGES, int TENSORS>
__device__ void produce_tiles(const CUtensorMap* tmK, const CUtensorMap* tmV, uint8_t* ring, uint64_t* full,
                              uint64_t* empty, volatile int* abort_flag, int t_begin, int nt, int bh,
                              unsigned* status) {
    using L = StreamSmem<D, STAGES, TENSORS>;
    prefetch_tensormap(tmK);
    if (TENSORS == 2) prefetch_tensormap(tmV);
    int issued = 0;
    for (int i = 0; i < nt; ++i) {
        const int stage = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[stage], ((i / STAGES) - 1) & 1, status)) {
            *abort_flag = 1;
            break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
        const int j0 = (t_begin + i) * kKeyTile;
        uint8_t* dst = ring + stage * L::kStageBytes;
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
            tma_load_3d(dst + half * (kKeyTile * 128), tmK, &full[stage], half * 64, j0, bh);
            if (TENSORS == 2)
                tma_load_3d(dst + L::kTileBytes + half * (kKeyTile * 128), tmV, &full[stage], half * 64, j0, bh);
        }
        ++issued;
    }
    // Drain: wait (bounded) for the last load issued into every stage, so no copy is still
    // landing in shared memory when the CTA retires (matters only after an abort).
    for (int st = 0; st < STAGES && st < issued; ++st) {
        const int last = st + ((issued - 1 - st) / STAGES) * STAGES;
        mbar_wait(&full[st], (last / STAGES) & 1, status);
    }
}

}  // namespace

// ====================================================================== full attention

template <int D, int RT, int NC, int STAGES, bool KEEP_LOGITS>
__global__ void __launch_bounds__((NC + 1) * 32)
    full_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const AttnArgs a) {
    constexpr int NKS = NC / RT;          // warps sharing one row tile (each a key slice)
    constexpr int KW = kKeyTile / NKS;    // keys per warp per tile
    static_assert(NC % RT == 0 && KW % 16 == 0, "bad warp split");
    using L = StreamSmem<D, STAGES, 2>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
    int* s_pos = reinterpret_cast<int*>(smem + L::kMiscOff + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x;
    const int unit = blockIdx.y;
    const int bh = unit / a.QB, qb = unit % a.QB;
    const int b = bh / a.Hkv, h = bh % a.Hkv;

    if (a.zero) {  // clear the next kernels' per-row counters and histograms, spread over all CTAs
        const int64_t cta = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
        const int64_t nthr = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
        for (int64_t i = cta * blockDim.x + tid; i < a.zero_vec; i += nthr) a.zero[i] = make_uint4(0, 0, 0, 0);
    }
    for (int r = tid; r < 16 * RT; r += blockDim.x) {
        const int tq = r / a.G, t = qb * a.TQ + tq;
        s_pos[r] = (tq < a.TQ && t < a.T) ? clamp_pos(a.pos[b * a.T + t], a.N, a.status) : -1;
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

    int jmax = -1;
    for (int r = 0; r < 16 * RT; ++r) jmax = max(jmax, s_pos[r]);
    const int ntiles = jmax >= 0 ? (jmax + kKeyTile) / kKeyTile : 0;
    const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.S);
    const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.S);
    const int nt = t_end - t_begin;

    OnlineSoftmax<D> st;
    st.init();
    const int rt = warp % RT, ks = warp / RT;
    const int g = lane >> 2, c = lane & 3;
    const int r_lo = rt * 16 + g, r_hi = r_lo + 8;
    auto row_q = [&](int r) -> int {  // global query-head row of local row r, or -1
        const int tq = r / a.G, t = qb * a.TQ + tq;
        if (tq >= a.TQ || t >= a.T) return -1;
        return (b * a.Hq + h * a.G + (r % a.G)) * a.T + t;
    };

    if (warp == NC) {
        if (lane == 0)
            produce_tiles<D, STAGES, 2>(&tmK, &tmV, ring, full, empty, abort_flag, t_begin, nt, bh, a.status);
        __syncwarp();
    } else {
        QTile<D> q;
        const int rq_lo = row_q(r_lo), rq_hi = row_q(r_hi);
        q.load(a.Q, rq_lo >= 0 ? static_cast<int64_t>(rq_lo) * D : -1, rq_hi >= 0 ? static_cast<int64_t>(rq_hi) * D : -1);
        const int p_lo = s_pos[r_lo], p_hi = s_pos[r_hi];
        const int key0 = ks * KW;
        float* lg_lo = nullptr;
        float* lg_hi = nullptr;
        if (KEEP_LOGITS) {
            // [row_kv][N][G]: row_kv = (b*Hkv + h)*T + t
            if (p_lo >= 0)
                lg_lo = a.logits + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + r_lo / a.G) * a.N * a.G + (r_lo % a.G);
            if (p_hi >= 0)
                lg_hi = a.logits + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + r_hi / a.G) * a.N * a.G + (r_hi % a.G);
        }
        for (int i = 0; i < nt; ++i) {
            const int stage = i % STAGES;
            if (!mbar_wait(&full[stage], (i / STAGES) & 1, a.status)) {
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            const uint32_t kbase = smem_u32(ring + stage * L::kStageBytes);
            const uint32_t vbase = kbase + L::kTileBytes;
            float sc[KW / 8][4];
            qk_tile<D, KW>(q, kbase, key0, sc);
            const int jb = (t_begin + i) * kKeyTile + key0 + 2 * c;
#pragma unroll
            for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = jb + n * 8 + (e & 1);
                    const int p = (e < 2) ? p_lo : p_hi;
                    const float v = sc[n][e] * a.scale_log2;
                    sc[n][e] = (j <= p) ? v : -INFINITY;
                    if (KEEP_LOGITS && j <= p) {
                        float* lg = (e < 2) ? lg_lo : lg_hi;
                        lg[static_cast<int64_t>(j) * a.G] = v;
                    }
                }
            }
            st.template update<KW>(sc, vbase, key0);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
        st.finish_rows();
    }
    __syncthreads();
    if (*abort_flag) return;

    const PartialRef out{a.part_ml + static_cast<int64_t>(split) * (a.B * a.Hq * a.T),
                         a.part_acc + static_cast<int64_t>(split) * (a.B * a.Hq * a.T) * D};
    if (NKS == 1) {
        if (warp < NC) store_partial<D>(st, out, [&](int r) { return row_q(rt * 16 + r); });
    } else {
        float* red = reinterpret_cast<float*>(ring);  // the ring is idle now
        if (warp < NC) stash_state<D, NKS>(st, ks, red + rt * merge_floats<D, NKS>());
        __syncthreads();
        // threads of the CTA split evenly over the RT tiles
        const int per = blockDim.x / RT;
        const int my_rt = tid / per;
        if (my_rt < RT)
            merge_states<D, NKS>(red + my_rt * merge_floats<D, NKS>(), tid - my_rt * per, per, out,
                                 [&](int r) { return row_q(my_rt * 16 + r); });
    }
}

// ====================================================================== score sweep (second K pass)

template <int D, int RT, int NC, int STAGES>
__global__ void __launch_bounds__((NC + 1) * 32)
    score_sweep_kernel(const __grid_constant__ CUtensorMap tmK, const AttnArgs a) {
    constexpr int NKS = NC / RT;
    constexpr int KW = kKeyTile / NKS;
    using L = StreamSmem<D, STAGES, 1>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
    int* s_pos = reinterpret_cast<int*>(smem + L::kMiscOff + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, unit = blockIdx.y;
    const int bh = unit / a.QB, qb = unit % a.QB;
    const int b = bh / a.Hkv, h = bh % a.Hkv;

    for (int r = tid; r < 16 * RT; r += blockDim.x) {
        const int tq = r / a.G, t = qb * a.TQ + tq;
        s_pos[r] = (tq < a.TQ && t < a.T) ? clamp_pos(a.pos[b * a.T + t], a.N, nullptr) : -1;
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

    // only pool keys (j <= pos - W) are scored
    int jmax = -1;
    for (int r = 0; r < 16 * RT; ++r)
        if (s_pos[r] >= 0) jmax = max(jmax, s_pos[r] - a.W);
    const int ntiles = jmax >= 0 ? (jmax + kKeyTile) / kKeyTile : 0;  // 0 when every pool is empty
    const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.S);
    const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.S);
    const int nt = t_end - t_begin;

    if (warp == NC) {
        if (lane == 0)
            produce_tiles<D, STAGES, 1>(&tmK, &tmK, ring, full, empty, abort_flag, t_begin, nt, bh, a.status);
        __syncwarp();
    } else {
        const int rt = warp % RT, ks = warp / RT;
        const int g = lane >> 2, c = lane & 3;
        const int r_lo = rt * 16 + g, r_hi = r_lo + 8;
        auto row_q = [&](int r) -> int {
            const int tq = r / a.G, t = qb * a.TQ + tq;
            if (tq >= a.TQ || t >= a.T) return -1;
            return (b * a.Hq + h * a.G + (r % a.G)) * a.T + t;
        };
        QTile<D> q;
        const int rq_lo = row_q(r_lo), rq_hi = row_q(r_hi);
        q.load(a.Q, rq_lo >= 0 ? static_cast<int64_t>(rq_lo) * D : -1, rq_hi >= 0 ? static_cast<int64_t>(rq_hi) * D : -1);
        // base-2 LSE of the two rows (+inf for padding rows so their scores are -inf)
        const float lse_lo = rq_lo >= 0 ? a.lse[rq_lo] * kLog2e : INFINITY;
        const float lse_hi = rq_hi >= 0 ? a.lse[rq_hi] * kLog2e : INFINITY;
        // last pool key of each row's query (-1: empty pool / padding)
        const int pl_lo = s_pos[r_lo] >= 0 ? s_pos[r_lo] - a.W : -1;
        const int pl_hi = s_pos[r_hi] >= 0 ? s_pos[r_hi] - a.W : -1;
        // group of G consecutive rows = one query; reduce over the lane bits that index g
        constexpr int kMaxGroupLanes = 8;  // rows g = lane>>2 span 8 values per half
        const int gl = a.G < kMaxGroupLanes ? a.G : kMaxGroupLanes;
        const bool writer_lo = (g % gl) == 0;
        const bool writer_hi = writer_lo && a.G < 16;  // with G = 16 rows g and g+8 share a query
        uint32_t* key_lo = nullptr;
        uint32_t* key_hi = nullptr;
        if (rq_lo >= 0) key_lo = a.keys + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + r_lo / a.G) * a.kstride;
        if (rq_hi >= 0) key_hi = a.keys + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + r_hi / a.G) * a.kstride;
        const int key0 = ks * KW;
        bool nonfinite = false;
        for (int i = 0; i < nt; ++i) {
            const int stage = i % STAGES;
            if (!mbar_wait(&full[stage], (i / STAGES) & 1, a.status)) {
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            const uint32_t kbase = smem_u32(ring + stage * L::kStageBytes);
            float sc[KW / 8][4];
            qk_tile<D, KW>(q, kbase, key0, sc);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            const int jb = (t_begin + i) * kKeyTile + key0 + 2 * c;
#pragma unroll
            for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lse = (e < 2) ? lse_lo : lse_hi;
                    sc[n][e] = sc[n][e] * a.scale_log2 - lse;
                }
                // max over the G heads of each query
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    if (off < 4 * gl) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) sc[n][e] = nan_max(sc[n][e], __shfl_xor_sync(0xffffffffu, sc[n][e], off));
                    }
                }
                if (a.G >= 16) {
                    sc[n][0] = nan_max(sc[n][0], sc[n][2]);
                    sc[n][1] = nan_max(sc[n][1], sc[n][3]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = jb + n * 8 + (e & 1);
                    const bool lo = e < 2;
                    const int pl = lo ? pl_lo : pl_hi;
                    if ((lo ? writer_lo : writer_hi) && j <= pl) {
                        nonfinite |= (sc[n][e] != sc[n][e]);
                        (lo ? key_lo : key_hi)[j] = score_key(sc[n][e]);
                    }
                }
            }
        }
        if (__any_sync(0xffffffffu, nonfinite) && lane == 0) set_status(a.status, HS2_DEV_NONFINITE);
    }
    __syncthreads();
}

// ====================================================================== combine

template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
    __shared__ float wbuf[8][256];
    const int warp = threadIdx.x >> 5;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp;
    if (row >= a.rows) return;
    warp_combine_row<D>(a.part_ml, a.part_acc, a.S, a.rows, row, wbuf[warp], a.O, a.LSE);
}

// ====================================================================== launchers

namespace {

template <class Kern>
cudaError_t set_smem(Kern kern, int bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, int RT, bool KEEP>
cudaError_t full_attn_variant(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                              cudaStream_t st) {
    constexpr int NC = RT >= 8 ? 8 : 4;
    constexpr int STAGES = D == 128 ? 3 : 6;
    using L = StreamSmem<D, STAGES, 2>;
    auto kern = full_attn_kernel<D, RT, NC, STAGES, KEEP>;
    cudaError_t e = set_smem(kern, L::kBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(p.S1, p.B * p.Hkv * p.QB);
    kern<<<grid, (NC + 1) * 32, L::kBytes, st>>>(tmK, tmV, a);
    trace_mark(KEEP ? "full_attn_keep_logits" : "full_attn", st);
    return cudaGetLastError();
}

template <int D, int RT>
cudaError_t score_sweep_variant(const Plan& p, const CUtensorMap& tmK, const AttnArgs& a, cudaStream_t st) {
    constexpr int NC = RT >= 8 ? 8 : 4;
    constexpr int STAGES = D == 128 ? 6 : 12;
    using L = StreamSmem<D, STAGES, 1>;
    auto kern = score_sweep_kernel<D, RT, NC, STAGES>;
    cudaError_t e = set_smem(kern, L::kBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(p.S1, p.B * p.Hkv * p.QB);
    kern<<<grid, (NC + 1) * 32, L::kBytes, st>>>(tmK, a);
    trace_mark("score_sweep", st);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_full_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st) {
    const bool keep = a.logits != nullptr;
#define HS2_FA(D_, RT_)                                                                                  \
    if (p.d == D_ && p.RT == RT_)                                                                        \
        return (keep && RT_ == 1) ? full_attn_variant<D_, RT_, (RT_ == 1)>(p, tmK, tmV, a, st)           \
                                  : full_attn_variant<D_, RT_, false>(p, tmK, tmV, a, st);
    HS2_FA(64, 1) HS2_FA(64, 2) HS2_FA(64, 4) HS2_FA(64, 8)
    HS2_FA(128, 1) HS2_FA(128, 2) HS2_FA(128, 4) HS2_FA(128, 8)
#undef HS2_FA
    return cudaErrorInvalidValue;
}

cudaError_t launch_score_sweep(const Plan& p, const CUtensorMap& tmK, const AttnArgs& a, cudaStream_t st) {
#define HS2_SS(D_, RT_) \
    if (p.d == D_ && p.RT == RT_) return score_sweep_variant<D_, RT_>(p, tmK, a, st);
    HS2_SS(64, 1) HS2_SS(64, 2) HS2_SS(64, 4) HS2_SS(64, 8)
    HS2_SS(128, 1) HS2_SS(128, 2) HS2_SS(128, 4) HS2_SS(128, 8)
#undef HS2_SS
    return cudaErrorInvalidValue;
}

cudaError_t launch_combine(int d, const CombineArgs& a, cudaStream_t st) {
    const unsigned blocks = static_cast<unsigned>((a.rows + 7) / 8);
    if (d == 128)
        combine_kernel<128><<<blocks, 256, 0, st>>>(a);
    else
        combine_kernel<64><<<blocks, 256, 0, st>>>(a);
    trace_mark("combine", st);
    return cudaGetLastError();
}

}  // namespace hs2
