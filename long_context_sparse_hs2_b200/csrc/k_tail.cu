// The decode step after the full-attention sweep, in one thread-block cluster per selection row
// (sm_100a): GQA-max log-softmax scores from the kept logits, the exact token-level top-k with
// the forced window, and the sparse layer with KV Reuse -- one kernel instead of a score, a
// select and a sparse-attention launch.
//
// The full layer's selection is what the sparse layers reuse ("HySparse2 od Xiaomi zkracuje
// zpracovani dlouheho kontextu", section "Proc neni nutne znovu zpracovat cely dlouhy vstup",
// third paragraph); the score (max over the G heads of l - LSE) and the tie rule (lower index)
// are this library's reading (see hs2.h).
//
// A selection row (b, kv head, t) is handled by a cluster of C CTAs (C up to 16), which the
// hardware schedules together, so the CTAs can exchange data through distributed shared memory
// and meet at cluster barriers -- no global atomics, no completion counters, no waiting on
// another kernel:
//   1. every CTA merges the G heads' LSE from the sweep's split partials, scores its share of
//      the pool (base-2 log-softmax, order-preserving uint32 keys kept in shared memory) and
//      bins the keys in a shared-memory histogram (score_bin buckets);
//   2. CTA c sums slice c of all C histograms (DSMEM reads); every CTA then reads the summed
//      histogram and finds the bucket b1 of the keff-th best key and the count above it;
//   3. every CTA counts its keys in better buckets (winners) and in b1 (candidates); from the
//      other CTAs' counts it knows exactly where to write its winners in the index row and its
//      candidates in the row's candidate list;
//   4. CTA 0 radix-selects the exact composite (key, ~index) threshold among the candidates
//      and writes the remaining winners, the window, the -1 padding and cnt; meanwhile CTAs
//      1 .. C-1 merge the full layer's split partials into O_full and LSE_full;
//   5. CTA c gathers its share of the selected K/V rows (16-byte cp.async into swizzled tiles)
//      and runs the warp attention core for the G heads of the row (KV Reuse);
//   6. each CTA stores its partial (m, l, O) of head g into the shared memory of head g's owner
//      (remote stores), which merges the C partials into O_sparse and LSE_sparse.
// Every CTA executes every cluster barrier (no early exit); remote shared-memory reads and writes
// all happen before the last barrier.
#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "combine.cuh"
#include "sparse_core.cuh"
#include "topk_common.cuh"

namespace hs2 {

namespace {

constexpr int kTailThreads = kSparseThreads;  // 8 warps
constexpr int kTailMaxChunk = 16384;          // pool keys one CTA keeps in shared memory
constexpr int kTailMaxSlots = 1024;           // selected keys one CTA gathers
constexpr int kTailStageBytes = 64 * 1024;    // kept logits streamed into shared memory per stage

// ------------------------------------------------------------------ cluster primitives

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// All threads of all CTAs of the cluster; writes before it (shared and global) are visible to
// every thread of the cluster after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The address of the shared variable p in the CTA of the cluster with the given rank.
__device__ __forceinline__ uint32_t dsmem(const void* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}
__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t a) { return __uint_as_float(ld_dsmem_u32(a)); }
__device__ __forceinline__ void st_dsmem_f32(uint32_t a, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void st_dsmem_f4(uint32_t a, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// max of two floats that is NaN when either is (PTX max.NaN): the score of a key with a NaN logit
// stays NaN, is flagged and ranks below every finite score.
__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Shared-memory plan (bytes from the 1 KB-aligned base).  The selection phase and the sparse
// phase use the same space one after the other.
template <int D, bool FP8>
struct TailSmem {
    using S = SparseSmem<D, FP8>;
    // selection phase
    static constexpr int kKeysOff = 0;                                    // u32 [kTailMaxChunk]
    static constexpr int kHistOff = kKeysOff + kTailMaxChunk * 4;         // u32 [kHistBins] local
    static constexpr int kHsumOff = kHistOff + kHistBins * 4;             // u32 [kHistBins] slice sums
    static constexpr int kWbufOff = kHsumOff + kHistBins * 4;             // O_full combine: S1 <= 256 weights + 8 x D
    static constexpr int kBarOff = kWbufOff + (256 + 8 * 128) * 4;        // 2 mbarriers of the logit stream
    static constexpr int kStageOff = kBarOff + 1024;                      // 2 logit stages (1 KB aligned)
    static constexpr int kCandOff = kStageOff;                            // u64 [kSmemCand] (CTA 0, after scoring)
    static constexpr int kSelectEnd = kStageOff + 2 * kTailStageBytes;
    static_assert(kSmemCand * 8 <= 2 * kTailStageBytes, "candidates reuse the stages");
    // sparse phase
    static constexpr int ring_end(int stages) { return S::idx_off(stages); }
    static constexpr int row_off(int stages) { return ring_end(stages); }  // int [kTailMaxSlots + kSparseTile]
    static constexpr int part_off(int stages) { return row_off(stages) + (kTailMaxSlots + kSparseTile) * 4; }
    // this CTA's partial [G][D] + [G] (m, l), then (16-byte aligned) the inbox of the heads it owns:
    // ceil(G / C) * C partials of D + 4 floats (O, m, l, padding; at most G + 15 of them)
    static constexpr int inbox_off(int stages, int G) { return part_off(stages) + ((G * (D + 2) + 3) / 4) * 16; }
    static constexpr int sparse_end(int stages, int G) { return inbox_off(stages, G) + (G + 15) * (D + 4) * 4; }
    static constexpr int bytes(int stages, int G) {
        return (kSelectEnd > sparse_end(stages, G) ? kSelectEnd : sparse_end(stages, G)) + 1024;
    }
};

}  // namespace

template <int D, int G, bool FP8>
__global__ void __launch_bounds__(kTailThreads, 1) tail_kernel(const TailArgs a) {
    using L = TailSmem<D, FP8>;
    using S = SparseSmem<D, FP8>;
    constexpr int KW = 16;  // keys per warp per sparse step
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + L::kKeysOff);
    unsigned* s_hist = reinterpret_cast<unsigned*>(smem + L::kHistOff);
    unsigned* s_hsum = reinterpret_cast<unsigned*>(smem + L::kHsumOff);
    unsigned long long* s_cand = reinterpret_cast<unsigned long long*>(smem + L::kCandOff);
    float* s_wbuf = reinterpret_cast<float*>(smem + L::kWbufOff);
    uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    float* s_stage = reinterpret_cast<float*>(smem + L::kStageOff);
    __shared__ float s_lse2[G];
    __shared__ unsigned s_warp[32];
    __shared__ int s_bin[2], s_below[2];
    __shared__ int s_cnt[2];      // this CTA's winners / candidates
    __shared__ int s_off[3];      // winners / candidates of the CTAs before this one, all candidates
    __shared__ unsigned s_radix[256];
    __shared__ unsigned s_small[2];
    __shared__ int s_count;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = static_cast<int>(gridDim.x);  // the cluster spans the grid's x dimension
    const int c = static_cast<int>(cluster_rank());
    const int row = blockIdx.y;  // (b*Hkv + h)*T + t
    const int t = row % a.T, bh = row / a.T;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const int64_t rows_q = static_cast<int64_t>(a.B) * a.Hq * a.T;
    auto row_q = [&](int r) -> int { return r < G ? (b * a.Hq + h * G + r) * a.T + t : -1; };
    pdl_trigger();

    // ---- prologue (inputs only): position, row geometry, the sparse layer's query fragments
    int pos = a.pos[b * a.T + t];
    const bool bad_pos = pos < 0 || pos >= a.N;
    pos = pos < 0 ? 0 : (pos >= a.N ? a.N - 1 : pos);
    const int P = max(0, pos - a.W + 1);        // pool [0, P)
    const int keff = min(a.k, P);
    const int wcnt = min(a.W, pos + 1);
    const int kw = a.k + a.W;
    const bool ranked = keff > 0 && keff < P;
    const int per = (P + C - 1) / C;            // pool keys per CTA (<= kTailMaxChunk: checked by the launcher)
    const int j0 = min(P, c * per), j1 = min(P, j0 + per);
    const int g8 = lane >> 2, cq = lane & 3;
    int32_t* idx = a.idx + static_cast<int64_t>(row) * kw;
    // this thread's keys in phases 3-4: an odd-length contiguous run (odd: conflict-free smem reads)
    const int run = ((j1 - j0 + kTailThreads - 1) / kTailThreads) | 1;
    const int r0 = min(j1, j0 + tid * run), r1 = min(j1, r0 + run);
    if (tid == 0) {
        mbar_init(&s_bar[0], 1);
        mbar_init(&s_bar[1], 1);
        fence_barrier_init();
    }
    pdl_wait();  // split partials and kept logits of the sweep
    if (bad_pos && tid == 0 && c == 0) set_status(a.status, HS2_DEV_BAD_POS);

    // ---- 1. LSE of the G heads, scores of this CTA's pool keys, local histogram
    for (int g = warp; g < G; g += kTailThreads / 32) {
        const float2 ML = warp_row_ml(a.pf_ml, a.S1, rows_q, row_q(g));
        if (lane == 0) s_lse2[g] = lse2_of(ML);
    }
    for (int i = tid; i < kHistBins; i += kTailThreads) s_hist[i] = 0u;
    __syncthreads();
    bool nonfinite = false;
    if (ranked) {
        // The chunk's kept logits stream into two shared-memory stages with bulk copies (the copy
        // engine keeps them in flight, no registers); the threads score one stage while the next
        // one lands.  The copy window is widened to 16-byte boundaries (inside the workspace).
        float lse[G];
#pragma unroll
        for (int g = 0; g < G; ++g) lse[g] = s_lse2[g];
        const uint8_t* lrow = reinterpret_cast<const uint8_t*>(a.logits + static_cast<int64_t>(row) * a.N * G);
        constexpr int kStageKeys = (kTailStageBytes - 32) / (G * 4);  // room for the widening
        const int nstage = (j1 - j0 + kStageKeys - 1) / kStageKeys;
        auto issue = [&](int s) {
            const int ja = j0 + s * kStageKeys, jb = min(j1, ja + kStageKeys);
            const uintptr_t from = reinterpret_cast<uintptr_t>(lrow + static_cast<int64_t>(ja) * G * 4) & ~uintptr_t(15);
            const uintptr_t to = (reinterpret_cast<uintptr_t>(lrow + static_cast<int64_t>(jb) * G * 4) + 15) & ~uintptr_t(15);
            mbar_arrive_expect_tx(&s_bar[s & 1], static_cast<uint32_t>(to - from));
            bulk_load(reinterpret_cast<uint8_t*>(s_stage) + (s & 1) * kTailStageBytes,
                      reinterpret_cast<const void*>(from), static_cast<uint32_t>(to - from), &s_bar[s & 1]);
        };
        if (tid == 0) {
            issue(0);
            if (nstage > 1) issue(1);
        }
        bool ok = true;
        for (int s = 0; s < nstage; ++s) {
            ok = ok && mbar_wait(&s_bar[s & 1], (s >> 1) & 1, a.status);
            const int ja = j0 + s * kStageKeys, jb = min(j1, ja + kStageKeys);
            const int lead = static_cast<int>((reinterpret_cast<uintptr_t>(lrow + static_cast<int64_t>(ja) * G * 4) & 15) / 4);
            const float* st = s_stage + (s & 1) * (kTailStageBytes / 4) + lead;
            constexpr int U = 8;  // keys per thread in flight: independent chains hide the latencies
            for (int jb0 = ja + tid; jb0 < jb && ok; jb0 += U * kTailThreads) {
                float v[U][G];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int j = jb0 + u * kTailThreads;
                    const float* src = st + (min(j, jb - 1) - ja) * G;
                    if constexpr (G % 4 == 0) {  // 16-byte aligned: the row and the stage start are
#pragma unroll
                        for (int qd = 0; qd < G / 4; ++qd) {
                            const float4 f = reinterpret_cast<const float4*>(src)[qd];
                            v[u][4 * qd] = f.x;
                            v[u][4 * qd + 1] = f.y;
                            v[u][4 * qd + 2] = f.z;
                            v[u][4 * qd + 3] = f.w;
                        }
                    } else {
#pragma unroll
                        for (int g = 0; g < G; ++g) v[u][g] = src[g];
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int j = jb0 + u * kTailThreads;
                    // max over the heads as a tree (log2 G dependent steps)
#pragma unroll
                    for (int g = 0; g < G; ++g) v[u][g] -= lse[g];
#pragma unroll
                    for (int w2 = 1; w2 < G; w2 *= 2)
#pragma unroll
                        for (int g = 0; g + w2 < G; g += 2 * w2) v[u][g] = max_nan(v[u][g], v[u][g + w2]);
                    const float sc = v[u][0];
                    if (j < jb) {
                        nonfinite |= (sc != sc);
                        const uint32_t key = score_key(sc);
                        s_keys[j - j0] = key;
                        atomicAdd(&s_hist[score_bin(key)], 1u);
                    }
                }
            }
            __syncthreads();  // stage s consumed
            if (tid == 0 && s + 2 < nstage) issue(s + 2);
        }
    }
    if (__syncthreads_or(nonfinite) && tid == 0) set_status(a.status, HS2_DEV_NONFINITE);
    if (tid == 0) {  // every copy has landed (each stage was waited for): the barriers' memory is reused later
        mbar_inval(&s_bar[0]);
        mbar_inval(&s_bar[1]);
    }
    cluster_sync();  // #1 every CTA's histogram is complete

    // ---- 2. slice sums, then the whole summed histogram -> threshold bucket b1, count above it
    const int slice = (kHistBins + C - 1) / C;  // bins summed by each CTA (the last slice may be short)
    if (ranked) {
        for (int i = tid; i < slice && c * slice + i < kHistBins; i += kTailThreads) {
            const int bin = c * slice + i;
            unsigned v[16];  // all C remote loads in flight before the first use
            for (int r = 0; r < C; ++r) v[r] = ld_dsmem_u32(dsmem(&s_hist[bin], r));
            unsigned sum = 0;
            for (int r = 0; r < C; ++r) sum += v[r];
            s_hsum[bin] = sum;
        }
    }
    cluster_sync();  // #2 slice sums complete (and nobody reads a local histogram any more)
    if (ranked) {
        constexpr int PB = kHistBins / kTailThreads;
        unsigned v[PB];
#pragma unroll
        for (int i = 0; i < PB; ++i) {
            const int bin = tid + i * kTailThreads;
            v[i] = ld_dsmem_u32(dsmem(&s_hsum[bin], bin / slice));
        }
#pragma unroll
        for (int i = 0; i < PB; ++i) s_hist[tid + i * kTailThreads] = v[i];
        if (tid == 0) {
            s_bin[0] = s_bin[1] = kHistBins - 1;
            s_below[0] = s_below[1] = 0;
        }
        __syncthreads();
        const unsigned cnts[2] = {static_cast<unsigned>(keff), static_cast<unsigned>(keff)};
        buckets_at_counts<kTailThreads>(s_hist, cnts, s_warp, s_bin, s_below);
    }
    __syncthreads();
    const int b1 = s_bin[0], above = s_below[0];

    // ---- 3. winners (better buckets) and candidates (bucket b1): each thread counts its run, a
    // block scan gives every thread its place, and the other CTAs' totals give the CTA's place
    unsigned mine_cnt = 0;  // winners | candidates << 16 (a run is < 2^16 keys)
    if (ranked) {
        int nd = 0, nc = 0;
#pragma unroll 4
        for (int j = r0; j < r1; ++j) {
            const int bin = score_bin(s_keys[j - j0]);
            nd += bin < b1;
            nc += bin == b1;
        }
        mine_cnt = static_cast<unsigned>(nd) | (static_cast<unsigned>(nc) << 16);
    }
    const unsigned excl = block_exclusive_scan(mine_cnt, s_warp);
    if (tid == kTailThreads - 1) {
        s_cnt[0] = static_cast<int>((excl + mine_cnt) & 0xFFFFu);
        s_cnt[1] = static_cast<int>((excl + mine_cnt) >> 16);
    }
    cluster_sync();  // #3 every CTA's counts are known
    int def_off = 0, cnd_off = 0, ncand = 0;
    if (ranked) {
        // lane r of warp 0 reads CTA r's two counts; prefix and total by shuffles; broadcast in smem
        if (warp == 0) {
            const int nd = lane < C ? static_cast<int>(ld_dsmem_u32(dsmem(&s_cnt[0], lane))) : 0;
            const int nc = lane < C ? static_cast<int>(ld_dsmem_u32(dsmem(&s_cnt[1], lane))) : 0;
            int pd = nd, pc = nc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int yd = __shfl_up_sync(0xffffffffu, pd, o), yc = __shfl_up_sync(0xffffffffu, pc, o);
                if (lane >= o) {
                    pd += yd;
                    pc += yc;
                }
            }
            if (lane == c) {
                s_off[0] = pd - nd;
                s_off[1] = pc - nc;
            }
            if (lane == 31) s_off[2] = pc;
        }
        __syncthreads();
        def_off = s_off[0];
        cnd_off = s_off[1];
        ncand = s_off[2];
        int od = def_off + static_cast<int>(excl & 0xFFFFu), oc = cnd_off + static_cast<int>(excl >> 16);
        int32_t* out = idx + wcnt;
        unsigned long long* cand = a.cand + static_cast<int64_t>(row) * a.cand_cap;
#pragma unroll 4
        for (int j = r0; j < r1; ++j) {
            const uint32_t key = s_keys[j - j0];
            const int bin = score_bin(key);
            if (bin < b1) {
                if (od < above) out[od] = j;
                ++od;
            } else if (bin == b1) {
                if (oc < a.cand_cap) cand[oc] = composite(key, j);
                ++oc;
            }
        }
    } else if (keff > 0) {  // the whole pool is selected
        for (int j = j0 + tid; j < j1; j += kTailThreads) idx[wcnt + j] = j;
    }
    __threadfence();
    cluster_sync();  // #4 winners and candidates are in memory

    // ---- 4. CTA 0: the exact remainder, window, padding, cnt.  CTAs 1..C-1: O_full, LSE_full
    if (c == 0) {
        for (int i = tid; i < wcnt; i += kTailThreads) idx[i] = pos - wcnt + 1 + i;
        for (int i = wcnt + keff + tid; i < kw; i += kTailThreads) idx[i] = -1;
        if (tid == 0) {
            a.cnt[row] = wcnt + keff;
            s_count = 0;
        }
        __syncthreads();
        if (ranked && above >= 0 && above < keff) {  // always, for a consistent histogram
            const unsigned need = static_cast<unsigned>(keff - above);
            int32_t* tail = idx + wcnt + above;
            const unsigned long long* gc = a.cand + static_cast<int64_t>(row) * a.cand_cap;
            const int nc = static_cast<int>(min(static_cast<int64_t>(ncand), a.cand_cap));
            if (nc <= kSmemCand) {
                for (int i = tid; i < nc; i += kTailThreads) s_cand[i] = __ldcg(gc + i);
                __syncthreads();
                const SmemSource src{s_cand, nc};
                emit_at_least(src, radix_threshold(src, need, s_radix, s_small), need, tail, &s_count);
            } else {
                const GlobalSource src{gc, nc};
                emit_at_least(src, radix_threshold(src, need, s_radix, s_small), need, tail, &s_count);
            }
        }
    }
    if (c > 0 || C == 1) {
        // heads c - 1, c - 1 + (C - 1), ... (all of them when C == 1), the whole CTA on each
        const int first = C == 1 ? 0 : c - 1, stride = C == 1 ? 1 : C - 1;
        for (int g = first; g < G; g += stride)
            block_combine_row<D>(a.pf_ml, a.pf_acc, a.S1, rows_q, row_q(g), s_wbuf, s_wbuf + 256, a.O_full,
                                 a.LSE_full);
    }
    __threadfence();
    cluster_sync();  // #5 the index row is complete

    // ---- 5. sparse layer over this CTA's share of the selection
    const int n = wcnt + keff;
    const int lo = static_cast<int>((static_cast<int64_t>(c) * n) / C);
    const int nk = static_cast<int>((static_cast<int64_t>(c + 1) * n) / C) - lo;
    const int stages = a.stages;
    int* s_row = reinterpret_cast<int*>(smem + L::row_off(stages));
    float* s_part = reinterpret_cast<float*>(smem + L::part_off(stages));  // [G][D] O, then [G] (m, l)
    const PartialRef mine{reinterpret_cast<float2*>(s_part + G * D), s_part};
    const int ntl = (nk + kSparseTile - 1) / kSparseTile;
    const bool paged = a.kv.page_shift >= 0;
    bool bad_page = false;
    for (int i = tid; i < ntl * kSparseTile; i += kTailThreads) {
        int j = -1;
        if (i < nk) {
            j = __ldcg(idx + lo + i);
            if (j < 0 || j > pos) {
                j = -1;  // cannot happen: the row was just written
            } else if (paged) {
                const int page = a.kv.page_table[static_cast<int64_t>(b) * a.kv.max_pages + (j >> a.kv.page_shift)];
                if (page < 0 || page >= a.kv.num_pages) {
                    bad_page = true;
                    j = -1;
                } else {
                    j = (page * a.Hkv + h) * (1 << a.kv.page_shift) + (j & ((1 << a.kv.page_shift) - 1));
                }
            }
        }
        s_row[i] = j;
    }
    if (__syncthreads_or(bad_page) && tid == 0) set_status(a.status, HS2_DEV_BAD_PAGE);
    const int64_t kv_base = paged ? 0 : static_cast<int64_t>(bh) * a.N;
    const int prime = min(ntl, stages);
    for (int i = 0; i < prime; ++i) {
        gather_tile<D, FP8>(a.K, a.V, s_row, i, smem + i * S::kStageBytes, kv_base);
        cp_async_commit();
    }
    QTileOf<D, FP8> q;
    {
        const int q0 = row_q(g8), q1 = row_q(g8 + 8);
        q.load(a.Qs, q0 >= 0 ? static_cast<int64_t>(q0) * D : -1, q1 >= 0 ? static_cast<int64_t>(q1) * D : -1);
    }
    const float kscale = FP8 ? a.kv.k_scale[bh] : 1.f;
    const float vscale = FP8 ? a.kv.v_scale[bh] : 1.f;
    const float f_lo = logit_factor<D, FP8>(q, 0, a.scale_log2, kscale);
    const float f_hi = logit_factor<D, FP8>(q, 1, a.scale_log2, kscale);
    OnlineSoftmax<D, FP8> st;
    st.init();
    const int sub = warp >> 2;
    const int key0 = (warp & 3) * KW;
    for (int i = 0; i < ntl; ++i) {
        cp_async_wait_upto(min(ntl, i + stages) - (i + 1));  // step i has landed
        __syncthreads();
        const int stage = i % stages;
        const uint32_t kbase = smem_u32(smem + stage * S::kStageBytes + sub * S::kSubBytes);
        const uint32_t vbase = kbase + S::kTileBytes;
        float sc[KW / 8][4];
        qk_any<D, KW, FP8>(q, kbase, key0, sc);
        const int slot0 = i * kSparseTile + sub * kKeyTile + key0 + 2 * cq;
#pragma unroll
        for (int nn = 0; nn < KW / 8; ++nn)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool ok = s_row[slot0 + nn * 8 + (e & 1)] >= 0;
                sc[nn][e] = ok ? sc[nn][e] * (e < 2 ? f_lo : f_hi) : -INFINITY;
            }
        st.template update<KW>(sc, vbase, key0);
        __syncthreads();  // everyone is done with this stage before it is refilled
        if (i + stages < ntl) {
            gather_tile<D, FP8>(a.K, a.V, s_row, i + stages, smem + stage * S::kStageBytes, kv_base);
            cp_async_commit();
        }
    }
    st.finish_rows();
    float* red = reinterpret_cast<float*>(smem);  // the ring is idle now
    stash_state<D, kSparseWarps, FP8>(st, warp, red, vscale);
    __syncthreads();
    merge_states<D, kSparseWarps>(red, tid, kTailThreads, mine, [&](int r) { return r < G ? r : -1; });
    __syncthreads();
    // push this CTA's partial of head g into the inbox of head g's owner (CTA g % C), slot c
    float* inbox = reinterpret_cast<float*>(smem + L::inbox_off(stages, G));  // [heads owned][C][D + 4]
    for (int e = tid; e < G * (D / 4); e += kTailThreads) {
        const int g = e / (D / 4), q4 = e % (D / 4);
        const int slot = ((g / C) * C + c) * (D + 4);
        st_dsmem_f4(dsmem(inbox + slot + 4 * q4, g % C), reinterpret_cast<const float4*>(mine.acc + g * D)[q4]);
    }
    for (int g = tid; g < G; g += kTailThreads) {
        const int slot = ((g / C) * C + c) * (D + 4);
        st_dsmem_f32(dsmem(inbox + slot + D, g % C), mine.ml[g].x);
        st_dsmem_f32(dsmem(inbox + slot + D + 1, g % C), mine.ml[g].y);
    }
    cluster_sync();  // #6 every head's C partials are in its owner's inbox

    // ---- 6. the owner of head g (CTA g % C) merges its C partials, one warp per head
    for (int g = c + C * warp; g < G; g += C * (kTailThreads / 32)) {
        constexpr int PER = D / 32;
        const float* box = inbox + (g / C) * C * (D + 4);
        float M = -INFINITY;
        for (int r = 0; r < C; ++r) M = fmaxf(M, box[r * (D + 4) + D]);
        float Ls = 0.f;
        float acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.f;
        for (int r = 0; r < C; ++r) {
            const float* pr = box + r * (D + 4);
            const float m = pr[D];
            const float wgt = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
            Ls += wgt * pr[D + 1];
#pragma unroll
            for (int e = 0; e < PER; ++e) acc[e] += wgt * pr[lane * PER + e];
        }
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] *= inv;
        store_row<D>(acc, make_float2(M, Ls), row_q(g), a.O_sparse, a.LSE_sparse);
    }
    // nothing reads another CTA's shared memory after barrier #6: the CTAs may leave independently
}

// ====================================================================== launcher

namespace {

// The launch decision for one shape (cluster size C, 0 = the shape does not fit; ring depth),
// cached per (kernel variant, device, rows, N, k + W, W): the occupancy query is a host call
// too slow to repeat on every step.
struct TailChoice {
    int C, stages, bytes;
};

struct TailKey {
    const void* kern;
    int dev, rows, N, kw, W;
    bool force;
    bool operator==(const TailKey& o) const {
        return kern == o.kern && dev == o.dev && rows == o.rows && N == o.N && kw == o.kw && W == o.W &&
               force == o.force;
    }
};

std::mutex g_tail_mutex;
std::vector<std::pair<TailKey, TailChoice>> g_tail_cache;

// Cluster size: the largest C (16 at most, any integer) that keeps every row's cluster resident at once,
// with each CTA's share of the pool and of the selection within its shared-memory plan.
template <int D, int G, bool FP8, class Kern>
cudaError_t choose_tail(const Plan& p, Kern kern, bool force, TailChoice* out) {
    using L = TailSmem<D, FP8>;
    const int64_t kw = static_cast<int64_t>(p.k) + p.W;
    const int64_t pool_max = std::max<int64_t>(0, p.N - p.W);
    for (int C = 16; C >= 1; --C) {
        if ((pool_max + C - 1) / C > kTailMaxChunk || (kw + C - 1) / C > kTailMaxSlots) break;
        const int stages =
            static_cast<int>(std::min<int64_t>(kSparseMaxStages, ((kw + C - 1) / C + kSparseTile - 1) / kSparseTile));
        const int s = std::max(1, stages);
        const int bytes = L::bytes(s, G);
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        if (C > 8) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) {
                cudaGetLastError();
                continue;
            }
        }
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(C, static_cast<unsigned>(p.rows_kv));
        cfg.blockDim = dim3(kTailThreads);
        cfg.dynamicSmemBytes = bytes;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = C;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int active = 0;
        e = cudaOccupancyMaxActiveClusters(&active, kern, &cfg);
        if (e != cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        if (static_cast<int64_t>(active) < p.rows_kv && C > 1) continue;  // not one wave: try smaller clusters
        if (active < 1) return cudaSuccess;                               // cannot run: keep the kernel chain
        // Measured on B200: the cluster tail once beat the kernel chain where its grid covered most
        // SMs (batched decode, 32 rows x 4 CTAs: 0.1425 against 0.1459 ms) and lost where it left
        // them idle (long-context decode, 8 rows x 10 CTAs: 0.1306 against 0.1292 ms); since the
        // chain's scoring and final selection were sped up it loses there too (0.1421 against
        // 0.1381 ms), so it runs only when forced.
        if (!force) return cudaSuccess;
        *out = TailChoice{C, s, bytes};
        return cudaSuccess;
    }
    return cudaSuccess;  // not applicable: the caller runs the kernel chain
}

template <int D, int G, bool FP8>
cudaError_t tail_variant(const Plan& p, const TailArgs& x, cudaStream_t st, bool force, bool* launched) {
    using L = TailSmem<D, FP8>;
    auto kern = tail_kernel<D, G, FP8>;
    const int64_t kw = static_cast<int64_t>(p.k) + p.W;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    const TailKey key{reinterpret_cast<const void*>(kern), dev, static_cast<int>(p.rows_kv), p.N, static_cast<int>(kw),
                      p.W, force};
    TailChoice ch{-1, 0, 0};
    {
        std::lock_guard<std::mutex> lock(g_tail_mutex);
        for (const auto& e : g_tail_cache)
            if (e.first == key) ch = e.second;
    }
    if (ch.C < 0) {
        ch = TailChoice{0, 0, 0};
        const cudaError_t e = choose_tail<D, G, FP8>(p, kern, force, &ch);
        if (e != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(g_tail_mutex);
        g_tail_cache.emplace_back(key, ch);
    }
    if (ch.C == 0) return cudaSuccess;  // not applicable: the caller runs the kernel chain
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, ch.bytes);
    if (e != cudaSuccess) return e;
    if (ch.C > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ch.C, static_cast<unsigned>(p.rows_kv));
    cfg.blockDim = dim3(kTailThreads);
    cfg.dynamicSmemBytes = ch.bytes;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = ch.C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    TailArgs y = x;
    y.stages = ch.stages;
    e = cudaLaunchKernelEx(&cfg, kern, y);
    trace_mark("select_sparse_cluster", st);
    *launched = e == cudaSuccess;
    return e;
}

template <int D, bool FP8>
cudaError_t tail_g(const Plan& p, const TailArgs& x, cudaStream_t st, bool force, bool* launched) {
    switch (p.G) {
        case 1: return tail_variant<D, 1, FP8>(p, x, st, force, launched);
        case 2: return tail_variant<D, 2, FP8>(p, x, st, force, launched);
        case 4: return tail_variant<D, 4, FP8>(p, x, st, force, launched);
        case 8: return tail_variant<D, 8, FP8>(p, x, st, force, launched);
        case 16: return tail_variant<D, 16, FP8>(p, x, st, force, launched);
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_tail(const Plan& p, const TailArgs& a, cudaStream_t st, bool force, bool* launched) {
    *launched = false;
    if (p.d == 128)
        return p.fp8 ? tail_g<128, true>(p, a, st, force, launched) : tail_g<128, false>(p, a, st, force, launched);
    if (p.d == 64)
        return p.fp8 ? tail_g<64, true>(p, a, st, force, launched) : tail_g<64, false>(p, a, st, force, launched);
    return cudaSuccess;
}

}  // namespace hs2
