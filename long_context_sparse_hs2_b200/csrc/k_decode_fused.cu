// The decode step (T = 1) in one cooperative launch (sm_100a): full attention, GQA-max
// log-softmax selection, token-level top-k with the forced window, and the sparse layer with KV
// Reuse, for every selection row at once.
//
// Grid: S splits x B*Hkv selection rows, all CTAs resident together (two per SM).  CTA (s, row)
//   1. runs the split-K flash-decode sweep over its key range (attn_sweep.cuh): the split
//      partial (m, l, O) of the row's G heads and the kept base-2 logits of its keys;
//   -- row barrier: every split of the row has published its partial --
//   2. merges the G heads' LSE from the S partials (every CTA, the same fixed order, so all get
//      bit-identical values) and writes its 1/S share of the O_full / LSE_full columns;
//   3. scores its own pool keys from the kept logits (max over heads of logit - LSE, as
//      order-preserving keys in shared memory) and adds its histogram to the row's;
//   -- row barrier: the row's histogram is complete --
//   4. finds the threshold bucket b1 of the keff-th best key from the row histogram (every CTA),
//      writes its keys of better buckets to the index list and its keys of b1 to the row's
//      candidate list (one 64-bit atomic per CTA reserves both ranges);
//   -- row barrier: the candidate list is complete --
//   5. ranks each of its own candidates against the whole list (a candidate is selected iff
//      fewer than keff - above others beat it, and that rank is its slot), or, for a long list,
//      radix-selects the exact threshold composite (every CTA, identical) and writes its own
//      candidates at or above it;
//   -- row barrier: the row's index list (window, selection, padding) is complete --
//   6. runs the sparse layer over an equal share of the index list: the rows gathered with
//      16-byte cp.async into the swizzled tile layout (two 64-key stages), the same warp
//      attention core as the sweep, one split partial per CTA;
//   -- row barrier: every sparse partial is written --
//   7. merges its share of the outputs' columns from the S sparse partials.
// The selection rule is that of the kernel chain (ties to the lower index, NaN ranked last); the
// split-K partials and the log-sum-exp merges are those of "Simplified Sparse Attention via Gist
// Tokens", section 3.6.  A row barrier is an arrival counter per row and a bounded spin
// (HS2_DEV_TIMEOUT after kWaitLimitNs; a CTA that gave up only arrives at the later barriers).
// The counters and histograms are cleared by the kernel before this one.  The next kernel is
// let launch only after the first barrier, when every CTA of this grid is resident, so it
// cannot take the place of a CTA that the others wait for.
#include "attn_sweep.cuh"
#include "combine.cuh"
#include "hs2_internal.h"
#include "topk_common.cuh"

namespace hs2 {

namespace {

constexpr int kFNC = 4;                    // consumer warps (four 16-key slices of a 64-key tile)
constexpr int kFWarps = kFNC + 1;          // + the TMA producer of the sweep
constexpr int kFThreads = kFWarps * 32;
constexpr int kFKeyCap = kFusedKeyCap;     // pool keys of one split kept in shared memory
constexpr int kFCandCap = 2048;            // a row's candidates radix-selected from shared memory
constexpr int kFOwnCap = 1024;             // a CTA's own candidates kept in shared memory

template <int D, int STAGES, bool FP8>
struct FSmem {
    using R = StreamSmem<D, STAGES, 2, FP8 ? 1 : 2>;
    static constexpr int kSweepBytes = R::kMiscOff + 16 + 128 * 4;  // ring, barriers, positions
    // selection phases
    static constexpr int kKeysOff = 0;                               // u32 [kFKeyCap]
    static constexpr int kHistOff = kKeysOff + kFKeyCap * 4;         // u32 [kHistBins]
    static constexpr int kCandOff = kHistOff + kHistBins * 4;        // u64 [kFCandCap]; first the
    static constexpr int kSelBytes = kCandOff + kFCandCap * 8;       //   O_full merge weights
    // sparse phase: two stages of gathered K and V (64 keys), their cache rows
    static constexpr int kGTile = kKeyTile * D * (FP8 ? 1 : 2);
    static constexpr int kGStage = 2 * kGTile;
    static constexpr int kRowOff = 2 * kGStage;
    static constexpr int kSparseBytes = kRowOff + 2 * kKeyTile * 4;
    static constexpr int kMergeBytes = merge_floats<D, kFNC>() * 4;  // after the loop, from offset 0
    static constexpr int kMax1 = kSweepBytes > kSelBytes ? kSweepBytes : kSelBytes;
    static constexpr int kUsed = kMax1 > kSparseBytes ? kMax1 : kSparseBytes;
    static_assert(kMergeBytes <= kUsed && kMergeBytes <= kCandOff, "merge scratch inside the layout");
    static constexpr int kBytes = kUsed + 1024;  // + alignment slack
};

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrive at the row barrier and (if wait) spin until `target` arrivals, for at most
// kWaitLimitNs.  Returns whether the CTA may go on (false after a timeout, and whenever wait is
// false).  Call from all threads.
__device__ __forceinline__ bool row_barrier(int* ctr, int target, unsigned* status, bool wait, int* s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1);
        int go = wait ? 1 : 0;
        if (wait && ld_acquire(ctr) < target) {
            const uint64_t t0 = global_ns();
            while (ld_acquire(ctr) < target) {
                if (global_ns() - t0 > kWaitLimitNs) {
                    set_status(status, HS2_DEV_TIMEOUT);
                    go = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        *s_flag = go;
    }
    __syncthreads();
    return *s_flag != 0;
}

// Exclusive prefix of v over the block and the block total (blockDim.x a multiple of 32).
__device__ __forceinline__ unsigned block_scan_total(unsigned v, unsigned* s_warp, unsigned* total) {
    const unsigned e = block_exclusive_scan(v, s_warp);
    __shared__ unsigned s_tot;
    if (threadIdx.x == blockDim.x - 1) s_tot = e + v;
    __syncthreads();
    *total = s_tot;
    __syncthreads();
    return e;
}

// Gathers the cache rows of index-list slots slot0 .. slot0 + nvalid - 1 (at most 64) into one
// stage: K then V, each in the swizzled 64-key tile layout.  Invalid entries (outside [0, pos],
// or on an unmapped page) load zeros and are marked -1 in s_row.  Call from all threads.
template <int D, bool FP8>
__device__ __forceinline__ void gather_stage(const void* K, const void* V, const KvSrc& kv, const int32_t* idx_row,
                                             int slot0, int nvalid, int pos, int b, int h, int Hkv, int N,
                                             uint8_t* stage, int* s_row, bool* bad, bool* bad_page) {
    using L = FSmem<D, 1, FP8>;
    const int tid = threadIdx.x;
    if (tid < kKeyTile) {
        int j = -1;
        if (tid < nvalid) {
            j = __ldcg(idx_row + slot0 + tid);
            if (j < 0 || j > pos) {
                *bad = true;
                j = -1;
            } else if (kv.page_shift >= 0) {  // the token's row in the page pool
                const int page = kv.page_table[static_cast<int64_t>(b) * kv.max_pages + (j >> kv.page_shift)];
                if (page < 0 || page >= kv.num_pages) {
                    *bad_page = true;
                    j = -1;
                } else {
                    j = (page * Hkv + h) * (1 << kv.page_shift) + (j & ((1 << kv.page_shift) - 1));
                }
            }
        }
        s_row[tid] = j;
    }
    __syncthreads();
    constexpr int RB = D * (FP8 ? 1 : 2);  // bytes per cache row
    constexpr int CH = RB / 16;
    const int64_t kv_base = kv.page_shift >= 0 ? 0 : static_cast<int64_t>(b * Hkv + h) * N;
    const uint8_t* Kb = static_cast<const uint8_t*>(K);
    const uint8_t* Vb = static_cast<const uint8_t*>(V);
    for (int e = tid; e < kKeyTile * CH; e += blockDim.x) {
        const int r = e / CH, c16 = e % CH;
        const int j = s_row[r];
        const int64_t off = (kv_base + (j >= 0 ? j : 0)) * RB + c16 * 16;
        const uint32_t nbytes = j >= 0 ? 16u : 0u;
        uint8_t* dst = stage + kv_chunk_offset<D, FP8>(r, c16);
        cp_async16(dst, Kb + off, nbytes);
        cp_async16(dst + L::kGTile, Vb + off, nbytes);
    }
}

// Merges the S split partials (m, l, acc) of the G query-head rows row0 .. row0 + G - 1 (every CTA
// computes the same per-split weights, in one fixed order) and writes this CTA's contiguous share
// of the outputs' float4 columns (split of S): bf16 O and, with a row's first column, its
// natural-log LSE; s_lse2 receives each head's base-2 LSE.  Every (column, split) product is
// loaded by its own thread, and the products are summed in a fixed order, so the result does not
// depend on timing.  scratch: G * S float2 + G * S floats + ceil(G*D/4 / S) * S float4 bytes of
// shared memory.  Call from all threads.
template <int D, int G>
__device__ __forceinline__ void merge_share(const float2* __restrict__ part_ml, const float* __restrict__ part_acc,
                                            int S, int64_t rows, int64_t row0, int split, uint8_t* scratch,
                                            float2* s_ml, float* s_lse2, uint16_t* O, float* LSE) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    float2* s_pml = reinterpret_cast<float2*>(scratch);               // [G][S]
    float* s_w = reinterpret_cast<float*>(s_pml + G * S);              // [G][S]
    float4* s_prod = reinterpret_cast<float4*>(s_w + ((G * S + 3) & ~3));  // [columns of this CTA][S]
    for (int e = tid; e < G * S; e += blockDim.x) {
        const int g = e / S, sp = e % S;
        s_pml[e] = __ldcg(&part_ml[static_cast<int64_t>(sp) * rows + row0 + g]);
    }
    __syncthreads();
    for (int g = warp; g < G; g += nw) {
        const float2* pm = s_pml + g * S;
        float m = -INFINITY;
        for (int sp = lane; sp < S; sp += 32) m = fmaxf(m, pm[sp].x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        if (m != -INFINITY)
            for (int sp = lane; sp < S; sp += 32)
                if (pm[sp].x != -INFINITY) l += fast_exp2(pm[sp].x - m) * pm[sp].y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        const float inv = l > 0.f ? 1.f / l : 0.f;
        for (int sp = lane; sp < S; sp += 32)
            s_w[g * S + sp] = (pm[sp].x == -INFINITY || m == -INFINITY) ? 0.f : fast_exp2(pm[sp].x - m) * inv;
        if (lane == 0) {
            s_ml[g] = make_float2(m, l);
            s_lse2[g] = lse2_of(make_float2(m, l));
        }
    }
    __syncthreads();
    constexpr int C4 = D / 4;
    const int ncol = G * C4;
    const int c_lo = static_cast<int>((static_cast<int64_t>(split) * ncol) / S);
    const int c_hi = static_cast<int>((static_cast<int64_t>(split + 1) * ncol) / S);
    const int nc = c_hi - c_lo;
    for (int e = tid; e < nc * S; e += blockDim.x) {
        const int cl = e / S, sp = e % S;
        const int col = c_lo + cl, g = col / C4, c = col % C4;
        const float wt = s_w[g * S + sp];
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (wt != 0.f) {
            x = __ldcg(reinterpret_cast<const float4*>(part_acc + ((static_cast<int64_t>(sp) * rows + row0 + g) * D + c * 4)));
            x = make_float4(wt * x.x, wt * x.y, wt * x.z, wt * x.w);
        }
        s_prod[e] = x;
    }
    __syncthreads();
    for (int cl = tid; cl < nc; cl += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < S; ++sp) {
            const float4 x = s_prod[cl * S + sp];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        const int col = c_lo + cl, g = col / C4, c = col % C4;
        const int64_t row = row0 + g;
        *reinterpret_cast<uint2*>(O + row * D + c * 4) =
            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        if (c == 0) LSE[row] = s_lse2[g] * kLn2;
    }
    __syncthreads();
}

}  // namespace

template <int D, int G, int STAGES, bool FP8>
__global__ void __launch_bounds__(kFThreads, 2)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const AttnArgs a, const FusedArgs f) {
    using L = FSmem<D, STAGES, FP8>;
    using R = StreamSmem<D, STAGES, 2, FP8 ? 1 : 2>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ float2 s_ml[G];
    __shared__ float s_lse2[G];
    __shared__ unsigned s_hh[256];
    __shared__ unsigned s_small[2];
    __shared__ unsigned s_warp[32];
    __shared__ unsigned long long s_base2;
    __shared__ int s_int[8];  // 0 barrier flag, 1 b1, 2 above, 4 reserved base, 5 own candidates

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, row = blockIdx.y, S = gridDim.x;  // row = b * Hkv + h
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int64_t rows_q = static_cast<int64_t>(a.B) * a.Hq;
    const int64_t rq0 = static_cast<int64_t>(b) * a.Hq + h * G;  // query-head row of head g: rq0 + g
    int* meta = f.meta + static_cast<int64_t>(row) * kMetaInts;
    int* bar_ctr = meta + kMetaBarrier;
    int arrivals = 0;

    // ---- 1. the sweep of this split: partials and kept logits
    int2 range;
    constexpr bool TR = G <= 8;  // the transposed warp attention (at most 8 query-head rows)
    bool ok = full_sweep<D, 1, kFNC, STAGES, true, FP8, TR>(&tmK, &tmV, a, smem, split, row, &range);
    if (tid == 0) {
        uint64_t* bars = reinterpret_cast<uint64_t*>(smem + R::kBarOff);
        for (int i = 0; i < 2 * STAGES; ++i) mbar_inval(&bars[i]);  // the memory is reused below
    }
    pdl_wait();  // the kernel before cleared the counters, histograms and status word
    ok = row_barrier(bar_ctr, (++arrivals) * S, a.status, ok, &s_int[0]);
    pdl_trigger();  // every CTA of the grid is resident and past its sweep

    // ---- 2. the G heads' LSE (every CTA) and this CTA's share of the O_full combine
    if (ok)
        merge_share<D, G>(a.part_ml, a.part_acc, S, rows_q, rq0, split, smem + L::kKeysOff, s_ml, s_lse2, f.O_full,
                          f.LSE_full);

    const int pos = clamp_pos(a.pos[b], a.N, nullptr);  // a bad position was flagged by the sweep
    const int P = max(0, pos - a.W + 1);                 // pool: keys 0 .. pos - W
    const int keff = min(f.k, P), wcnt = min(a.W, pos + 1);
    const bool ranked = keff > 0 && keff < P;
    const int j_lo = range.x * kKeyTile;
    const int nown = max(0, min(range.y * kKeyTile, P) - j_lo);  // this CTA's pool keys
    const int kw = f.k + a.W;
    int32_t* idx = f.idx + static_cast<int64_t>(row) * kw;
    uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + L::kKeysOff);
    unsigned* s_hist = reinterpret_cast<unsigned*>(smem + L::kHistOff);
    // this CTA's candidates (the threshold bucket's keys), over the histogram once b1 is known
    unsigned long long* s_own = reinterpret_cast<unsigned long long*>(smem + L::kHistOff);

    if (ranked) {
        // ---- 3. scores of this CTA's pool keys, local histogram into the row's
        unsigned* gh = f.hist + static_cast<int64_t>(row) * kHistBins;
        if (ok) {
            for (int i = tid; i < kHistBins; i += kFThreads) s_hist[i] = 0u;
            __syncthreads();
            float lse[G];
#pragma unroll
            for (int g = 0; g < G; ++g) lse[g] = s_lse2[g];
            const float* lg = a.logits + static_cast<int64_t>(row) * a.N * G;
            bool nonfinite = false;
            constexpr int U = G >= 16 ? 4 : 8;  // keys in flight per thread
            for (int base = tid; base < nown; base += U * kFThreads) {
                float v[U][G];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = base + u * kFThreads;
                    if (i < nown) {
                        const float* src = lg + static_cast<int64_t>(j_lo + i) * G;
                        if constexpr (G % 4 == 0) {
#pragma unroll
                            for (int q = 0; q < G / 4; ++q) {
                                const float4 x = __ldcs(reinterpret_cast<const float4*>(src) + q);
                                v[u][4 * q] = x.x;
                                v[u][4 * q + 1] = x.y;
                                v[u][4 * q + 2] = x.z;
                                v[u][4 * q + 3] = x.w;
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < G; ++q) v[u][q] = __ldcs(src + q);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = base + u * kFThreads;
                    if (i < nown) {
                        float sv = v[u][0] - lse[0];
#pragma unroll
                        for (int g = 1; g < G; ++g) sv = nan_max(sv, v[u][g] - lse[g]);
                        nonfinite |= (sv != sv);
                        const uint32_t key = score_key(sv);
                        s_keys[i] = key;
                        atomicAdd(&s_hist[score_bin(key)], 1u);
                    }
                }
            }
            if (__syncthreads_or(nonfinite) && tid == 0) set_status(a.status, HS2_DEV_NONFINITE);
            for (int i = tid; i < kHistBins; i += kFThreads)
                if (s_hist[i]) atomicAdd(&gh[i], s_hist[i]);
        }
        ok = row_barrier(bar_ctr, (++arrivals) * S, a.status, ok, &s_int[0]);

        // ---- 4. threshold bucket (identical in every CTA); better buckets out, b1 to the candidates
        if (ok) {
            for (int i = tid; i < kHistBins; i += kFThreads) s_hist[i] = __ldcg(gh + i);
            if (tid == 0) {
                s_int[1] = kHistBins - 1;
                s_int[2] = 0;
            }
            __syncthreads();
            {  // the bucket holding the keff-th best key: 16 buckets per thread over 128 threads
                constexpr int PER = kHistBins / 128;
                unsigned v = 0;
                if (tid < 128)
                    for (int i = 0; i < PER; ++i) v += s_hist[tid * PER + i];
                const unsigned excl = block_exclusive_scan(v, s_warp);
                const unsigned need = static_cast<unsigned>(keff);
                if (tid < 128 && excl < need && need <= excl + v) {
                    unsigned cum = excl;
                    for (int i = 0; i < PER; ++i) {
                        const unsigned x = s_hist[tid * PER + i];
                        if (cum + x >= need) {
                            s_int[1] = tid * PER + i;
                            s_int[2] = static_cast<int>(cum);
                            break;
                        }
                        cum += x;
                    }
                }
                __syncthreads();
            }
            const int b1 = s_int[1], above = s_int[2];
            unsigned nd = 0, nc = 0;
            for (int i = tid; i < nown; i += kFThreads) {
                const int bin = score_bin(s_keys[i]);
                nd += bin < b1;
                nc += bin == b1;
            }
            unsigned tot;
            const unsigned ex = block_scan_total(nd | (nc << 16), s_warp, &tot);  // both < 2^16 per CTA
            const int td = static_cast<int>(tot & 0xFFFFu), tc = static_cast<int>(tot >> 16);
            const int2 base = block_reserve2(td, tc, meta + kMetaDef, &s_base2);
            int od = base.x + static_cast<int>(ex & 0xFFFFu), oc = base.y + static_cast<int>(ex >> 16);
            int lo_own = static_cast<int>(ex >> 16);
            unsigned long long* gc = f.cand + static_cast<int64_t>(row) * f.cand_cap;
            for (int i = tid; i < nown; i += kFThreads) {
                const uint32_t key = s_keys[i];
                const int bin = score_bin(key);
                if (bin < b1) {
                    if (od < above) idx[wcnt + od] = j_lo + i;
                    ++od;
                } else if (bin == b1) {
                    const unsigned long long c = composite(key, j_lo + i);
                    if (oc < f.cand_cap) gc[oc] = c;
                    if (lo_own < kFOwnCap) s_own[lo_own] = c;
                    ++oc;
                    ++lo_own;
                }
            }
            if (tid == 0) s_int[5] = tc;
        }
        ok = row_barrier(bar_ctr, (++arrivals) * S, a.status, ok, &s_int[0]);

        // ---- 5. the winners among the candidates: a candidate is selected iff fewer than
        // need = keff - above candidates beat it (composites are distinct), and its rank is its
        // slot.  Every CTA ranks its own candidates against the whole list; a longer list (heavy
        // ties) takes the exact radix threshold instead, in every CTA of the row alike.
        if (ok) {
            const int above = s_int[2], b1 = s_int[1], own = min(s_int[5], kFOwnCap);
            const unsigned need = static_cast<unsigned>(keff - above);
            const int64_t ncand = __ldcg(meta + kMetaCand);
            const int n = static_cast<int>(ncand < f.cand_cap ? ncand : f.cand_cap);
            const unsigned long long* gc = f.cand + static_cast<int64_t>(row) * f.cand_cap;
            unsigned long long* s_cand = reinterpret_cast<unsigned long long*>(smem + L::kCandOff);
            if (n <= kFOwnCap) {  // row-uniform: then every CTA holds all its own candidates
                for (int i = tid; i < n; i += kFThreads) s_cand[i] = __ldcg(gc + i);
                __syncthreads();
                for (int o = warp; o < own; o += kFWarps) {
                    const unsigned long long c = s_own[o];
                    int r = 0;
                    for (int i = lane; i < n; i += 32) r += s_cand[i] > c;
#pragma unroll
                    for (int x = 16; x > 0; x >>= 1) r += __shfl_xor_sync(0xffffffffu, r, x);
                    if (lane == 0 && r < static_cast<int>(need)) idx[wcnt + above + r] = composite_index(c);
                }
            } else {
                unsigned long long thr;
                if (n <= kFCandCap) {
                    for (int i = tid; i < n; i += kFThreads) s_cand[i] = __ldcg(gc + i);
                    __syncthreads();
                    thr = radix_threshold(SmemSource{s_cand, n}, need, s_hh, s_small);
                } else {
                    thr = radix_threshold(GlobalSource{gc, n}, need, s_hh, s_small);
                }
                unsigned ns = 0;
                for (int i = tid; i < nown; i += kFThreads) {
                    const uint32_t key = s_keys[i];
                    ns += score_bin(key) == b1 && composite(key, j_lo + i) >= thr;
                }
                unsigned ts;
                const unsigned es = block_scan_total(ns, s_warp, &ts);
                int o = block_reserve(static_cast<int>(ts), meta + kMetaAbove, &s_int[4]) + static_cast<int>(es);
                for (int i = tid; i < nown; i += kFThreads) {
                    const uint32_t key = s_keys[i];
                    if (score_bin(key) == b1 && composite(key, j_lo + i) >= thr) {
                        if (o < static_cast<int>(need)) idx[wcnt + above + o] = j_lo + i;
                        ++o;
                    }
                }
            }
        }
    } else if (ok && keff > 0) {  // the whole pool is selected, in index order
        for (int i = tid; i < nown; i += kFThreads) idx[wcnt + j_lo + i] = j_lo + i;
    }
    if (ok && split == 0) {  // window first, then the selection, then -1 padding
        for (int i = tid; i < wcnt; i += kFThreads) idx[i] = pos - wcnt + 1 + i;
        for (int i = wcnt + keff + tid; i < kw; i += kFThreads) idx[i] = -1;
        if (tid == 0) f.cnt[row] = wcnt + keff;
    }
    ok = row_barrier(bar_ctr, (++arrivals) * S, a.status, ok, &s_int[0]);

    // ---- 6. the sparse layer over this CTA's share of the index list
    const int nsel = wcnt + keff;
    const int C = (nsel + S - 1) / S;
    const int lo = split * C;
    const int nk = ok ? max(0, min(nsel, lo + C) - lo) : 0;
    const PartialRef out{f.ps_ml + static_cast<int64_t>(split) * rows_q,
                         f.ps_acc + static_cast<int64_t>(split) * rows_q * D};
    auto row_q = [&](int r) -> int { return r < G ? static_cast<int>(rq0 + r) : -1; };
    if (nk <= 0) {  // empty share: m = -inf, l = 0, O = 0
        for (int e = tid; e < G * D; e += kFThreads) {
            const int r = e / D, dc = e % D;
            out.acc[static_cast<int64_t>(row_q(r)) * D + dc] = 0.f;
            if (dc == 0) out.ml[row_q(r)] = make_float2(-INFINITY, 0.f);
        }
    } else {
        int* s_row = reinterpret_cast<int*>(smem + L::kRowOff);
        const int ntl = (nk + kKeyTile - 1) / kKeyTile;
        bool bad = false, bad_page = false;
        __syncthreads();  // the selection's shared memory is free
        for (int i = 0; i < min(ntl, 2); ++i) {
            gather_stage<D, FP8>(f.K, f.V, a.kv, idx, lo + i * kKeyTile, min(kKeyTile, nk - i * kKeyTile), pos, b, h,
                                 a.Hkv, a.N, smem + i * L::kGStage, s_row + i * kKeyTile, &bad, &bad_page);
            cp_async_commit();
        }
        const float kscale = FP8 ? a.kv.k_scale[row] : 1.f;
        const float vscale = FP8 ? a.kv.v_scale[row] : 1.f;
        OnlineSoftmax<D, FP8> st;
        st.init();
        const int g8 = lane >> 2, c = lane & 3;
        const int key0 = warp * 16;
        QTileOf<D, FP8> q;
        float f_lo = 0.f, f_hi = 0.f;
        if (warp < kFNC) {
            const int r0 = row_q(g8), r1 = row_q(g8 + 8);
            q.load(f.Qs, r0 >= 0 ? static_cast<int64_t>(r0) * D : -1, r1 >= 0 ? static_cast<int64_t>(r1) * D : -1);
            f_lo = logit_factor<D, FP8>(q, 0, a.scale_log2, kscale);
            f_hi = logit_factor<D, FP8>(q, 1, a.scale_log2, kscale);
        }
        for (int i = 0; i < ntl; ++i) {
            if (i + 1 < ntl)
                cp_async_wait<1>();
            else
                cp_async_wait<0>();
            __syncthreads();
            const int stg = i & 1;
            if (warp < kFNC) {
                const uint32_t kbase = smem_u32(smem + stg * L::kGStage);
                const uint32_t vbase = kbase + L::kGTile;
                float sc[2][4];
                qk_any<D, 16, FP8>(q, kbase, key0, sc);
                const int* rows = s_row + stg * kKeyTile;
#pragma unroll
                for (int nn = 0; nn < 2; ++nn)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = key0 + nn * 8 + 2 * c + (e & 1);
                        const bool valid = i * kKeyTile + r < nk && rows[r] >= 0;
                        sc[nn][e] = valid ? sc[nn][e] * (e < 2 ? f_lo : f_hi) : -INFINITY;
                    }
                st.template update<16>(sc, vbase, key0);
            }
            __syncthreads();  // everyone is done with this stage before it is refilled
            if (i + 2 < ntl) {
                gather_stage<D, FP8>(f.K, f.V, a.kv, idx, lo + (i + 2) * kKeyTile,
                                     min(kKeyTile, nk - (i + 2) * kKeyTile), pos, b, h, a.Hkv, a.N,
                                     smem + stg * L::kGStage, s_row + stg * kKeyTile, &bad, &bad_page);
                cp_async_commit();
            }
        }
        if (__syncthreads_or(bad) && tid == 0) set_status(a.status, HS2_DEV_BAD_INDEX);
        if (__syncthreads_or(bad_page) && tid == 0) set_status(a.status, HS2_DEV_BAD_PAGE);
        float* red = reinterpret_cast<float*>(smem);
        if (warp < kFNC) {
            st.finish_rows();
            stash_state<D, kFNC, FP8>(st, warp, red, vscale);
        }
        __syncthreads();
        merge_states<D, kFNC>(red, tid, kFThreads, out, row_q);
    }
    ok = row_barrier(bar_ctr, (++arrivals) * S, a.status, ok, &s_int[0]);

    // ---- 7. every CTA merges its share of the sparse partials
    if (ok)
        merge_share<D, G>(f.ps_ml, f.ps_acc, S, rows_q, rq0, split, smem, s_ml, s_lse2, f.O_sparse, f.LSE_sparse);
}

// ====================================================================== launcher

namespace {

template <int D, int G, int STAGES, bool FP8>
cudaError_t fused_variant(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                          const FusedArgs& f, cudaStream_t st, bool pdl, bool* launched) {
    using L = FSmem<D, STAGES, FP8>;
    auto kern = decode_fused_kernel<D, G, STAGES, FP8>;
    struct Fit {
        int dev = -1;
        int per_sm = 0;
    };
    static Fit fit[8];  // per device (the query runs once)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    Fit& ft = fit[dev & 7];
    if (ft.dev != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFThreads, L::kBytes);
        if (e != cudaSuccess) return e;
        ft.per_sm = per_sm;
        ft.dev = dev;
    }
    const int64_t ctas = static_cast<int64_t>(p.S1) * p.rows_kv;
    if (ctas > static_cast<int64_t>(ft.per_sm) * p.sms) {
        *launched = false;
        return cudaSuccess;
    }
    AttnArgs x = a;
    x.S = p.S1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.S1, static_cast<unsigned>(p.rows_kv));
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = L::kBytes;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, tmK, tmV, x, f);
    if (e != cudaSuccess && pdl) {  // a launch without programmatic serialisation is always valid
        (void)cudaGetLastError();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, tmK, tmV, x, f);
    }
    trace_mark("decode_fused", st);
    *launched = e == cudaSuccess;
    return e;
}

template <int D, bool FP8>
cudaError_t fused_g(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                    const FusedArgs& f, cudaStream_t st, bool pdl, bool* launched) {
    constexpr int STG = FP8 ? 6 : 3;
    switch (p.G) {
        case 1: return fused_variant<D, 1, STG, FP8>(p, tmK, tmV, a, f, st, pdl, launched);
        case 2: return fused_variant<D, 2, STG, FP8>(p, tmK, tmV, a, f, st, pdl, launched);
        case 4: return fused_variant<D, 4, STG, FP8>(p, tmK, tmV, a, f, st, pdl, launched);
        case 8: return fused_variant<D, 8, STG, FP8>(p, tmK, tmV, a, f, st, pdl, launched);
        case 16: return fused_variant<D, 16, STG, FP8>(p, tmK, tmV, a, f, st, pdl, launched);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_fused(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                                const FusedArgs& f, cudaStream_t st, bool pdl, bool* launched) {
    *launched = false;
    if (p.d == 128) return p.fp8 ? fused_g<128, true>(p, tmK, tmV, a, f, st, pdl, launched)
                                 : fused_g<128, false>(p, tmK, tmV, a, f, st, pdl, launched);
    if (p.d == 64) return p.fp8 ? fused_g<64, true>(p, tmK, tmV, a, f, st, pdl, launched)
                                : fused_g<64, false>(p, tmK, tmV, a, f, st, pdl, launched);
    return cudaErrorInvalidValue;
}

}  // namespace hs2
