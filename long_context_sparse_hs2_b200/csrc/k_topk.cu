// Token-level top-k with a forced window (sm_100a).
//
// HySparse2 selects individual tokens (not blocks) and always includes the most recent
// ones ("HySparse2 od Xiaomi zkracuje zpracovani dlouheho kontextu", section "Proc neni
// nutne znovu zpracovat cely dlouhy vstup", third paragraph; DAIR.AI newsletter, HySparse2
// bullet "Prefill exits early").  Per selection row (b, kv head, t) the library keeps the
// min(k, |pool|) pool keys [0, pos - W] of largest score, ties to the lower index, and
// writes them after the window [max(0, pos - W + 1), pos].
//
// The scores arrive as order-preserving keys with a per-row histogram of a monotone
// bucketing and the threshold bucket b1 already found (score_hist_kernel, or
// topk_hist_kernel below after a K re-sweep).  topk_select_kernel then:
//   * selects every key in a better bucket than b1 outright and appends the keys of b1 to a
//     candidate list (warp ballot + one atomic per warp; order arbitrary -- the compaction
//     pattern of "Simplified Sparse Attention via Gist Tokens", section 3.6);
//   * the row's last CTA (completion counter; nothing waits) radix-selects, 8 bits per pass,
//     the exact 64-bit composite threshold among the candidates, emits the winners, and
//     writes the window, the -1 padding and cnt.  If the candidate list overflowed its
//     capacity it re-scans the row's keys instead (exact, slower, flagged).
#include "topk_common.cuh"

namespace hs2 {

// ====================================================================== histogram of stored keys

__global__ void __launch_bounds__(256) topk_hist_kernel(const TopkArgs a) {
    __shared__ unsigned sh[kHistBins];
    __shared__ unsigned s_warp[32];
    __shared__ int s_last;
    const int64_t row = blockIdx.y;
    pdl_trigger();
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
    pdl_wait();  // keys from the score sweep (every CTA waits before it can finish)
    const RowInfo ri = make_row_info(a.pos, row, a.Hkv, a.T, a.N, a.k, a.W);
    if (ri.keff == 0 || ri.keff == ri.P) return;
    const int participants = (ri.P + kTopkChunk - 1) / kTopkChunk;
    if (static_cast<int>(blockIdx.x) >= participants) return;
    __syncthreads();
    const int j0 = blockIdx.x * kTopkChunk, j1 = min(j0 + kTopkChunk, ri.P);
    const uint32_t* keys = a.keys + row * a.kstride;
    // 4 keys per thread per 16-byte load (rows are 256-byte aligned, j0 a multiple of 4)
    for (int j = j0 + 4 * static_cast<int>(threadIdx.x); j < j1; j += 4 * blockDim.x) {
        const uint4 q = __ldcs(reinterpret_cast<const uint4*>(keys + j));
        const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (j + e < j1) atomicAdd(&sh[score_bin(kk[e])], 1u);
    }
    __syncthreads();
    hist_flush_and_threshold(sh, a.hist + row * kHistBins, a.meta + row * kMetaInts, participants, ri.keff, s_warp,
                             &s_last);
}

// ====================================================================== exact threshold among candidates

namespace {

struct SmemSource {
    const unsigned long long* c;
    int n;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const { v = c[i]; return true; }
};
struct GlobalSource {
    const unsigned long long* c;
    int n;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const { v = __ldcg(c + i); return true; }
};
struct KeyScanSource {  // overflow path: every pool key of the row whose bucket is b1
    const uint32_t* keys;
    int n, b1;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const {
        const uint32_t k = __ldcg(keys + i);
        v = composite(k, i);
        return score_bin(k) == b1;
    }
};

// The composite T such that exactly `need` source elements are >= T (8-bit radix digits,
// most significant first; stops as soon as the remaining digits are free).
template <class Src>
__device__ unsigned long long radix_threshold(const Src& src, unsigned need, unsigned* h, unsigned* s_small) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // Bits every element shares need no pass: start at the highest digit where they differ.
    __shared__ unsigned long long s_and[32], s_or[32];
    unsigned long long all_and = ~0ull, any_or = 0ull;
    for (int i = threadIdx.x; i < src.size(); i += blockDim.x) {
        unsigned long long c;
        if (src.get(i, c)) {
            all_and &= c;
            any_or |= c;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        all_and &= __shfl_xor_sync(0xffffffffu, all_and, o);
        any_or |= __shfl_xor_sync(0xffffffffu, any_or, o);
    }
    if (lane == 0) {
        s_and[warp] = all_and;
        s_or[warp] = any_or;
    }
    __syncthreads();
    all_and = ~0ull;
    any_or = 0ull;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
        all_and &= s_and[w];
        any_or |= s_or[w];
    }
    __syncthreads();
    const unsigned long long differ = all_and ^ any_or;
    if (differ == 0ull) return all_and;  // a single element (composites are distinct)
    const int top = 63 - __clzll(static_cast<long long>(differ));
    const int first_shift = (top / 8) * 8;
    unsigned long long prefix = first_shift >= 56 ? 0ull : (all_and & (~0ull << (first_shift + 8)));
    for (int shift = first_shift; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0u;
        if (threadIdx.x == 0) s_small[0] = s_small[1] = 0u;
        __syncthreads();
        const unsigned long long mask_hi = (shift == 56) ? 0ull : (~0ull << (shift + 8));
        const int n = src.size();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            unsigned long long c;
            if (src.get(i, c) && (c & mask_hi) == (prefix & mask_hi))
                atomicAdd(&h[static_cast<int>((c >> shift) & 255ull)], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane covers digits 255-8*lane down to 248-8*lane (best first)
            unsigned cnts[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnts[i] = h[255 - 8 * lane - i];
                sum += cnts[i];
            }
            unsigned incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned excl = incl - sum;
            if (excl < need && need <= incl) {
                unsigned cum = excl;
                for (int i = 0; i < 8; ++i) {
                    if (cum + cnts[i] >= need) {
                        s_small[0] = 255 - 8 * lane - i;
                        s_small[1] = cum;
                        break;
                    }
                    cum += cnts[i];
                }
            }
        }
        __syncthreads();
        const unsigned d = s_small[0];
        need -= s_small[1];
        prefix |= static_cast<unsigned long long>(d) << shift;
        const bool done = (h[d] == need);
        __syncthreads();
        if (done) break;
    }
    return prefix;
}

// Writes the source elements >= thr; never more than `need` slots whatever the inputs.
template <class Src>
__device__ void emit_at_least(const Src& src, unsigned long long thr, unsigned need, int32_t* out, int* s_count) {
    const int n = src.size();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        unsigned long long c;
        if (src.get(i, c) && c >= thr) {
            const int slot = atomicAdd(s_count, 1);
            if (slot < static_cast<int>(need)) out[slot] = composite_index(c);
        }
    }
}

}  // namespace

// ====================================================================== select: emit, then exact threshold

__global__ void __launch_bounds__(256, 3) topk_select_kernel(const TopkArgs a) {
    __shared__ unsigned long long s_cand[kSmemCand];
    __shared__ unsigned h[256];
    __shared__ unsigned s_small[2];
    __shared__ int s_count, s_last;
    __shared__ unsigned long long s_base2;
    __shared__ int s_cnt[2];
    static_assert(kTopkChunk % (4 * 256) == 0, "whole 16-byte key loads per thread");
    const int64_t row = blockIdx.y;
    const RowInfo ri = make_row_info(a.pos, row, a.Hkv, a.T, a.N, a.k, a.W);
    const int participants = max(1, (ri.P + kTopkChunk - 1) / kTopkChunk);
    pdl_trigger();
    pdl_wait();  // keys, histogram threshold and cleared counters from the kernels before
    if (static_cast<int>(blockIdx.x) >= participants) return;
    const int kw = a.k + a.W;
    int32_t* idx = a.idx + row * kw;
    int32_t* out = idx + ri.wcnt;  // the pool's winners follow the window
    int* meta = a.meta + row * kMetaInts;
    const int j0 = blockIdx.x * kTopkChunk, j1 = min(j0 + kTopkChunk, ri.P);
    const bool ranked = ri.keff > 0 && ri.keff < ri.P;
    const int b1 = ranked ? meta[kMetaBin] : 0;
    const int above = ranked ? meta[kMetaAbove] : 0;

    if (ri.keff > 0 && ri.keff == ri.P) {  // the whole pool is selected
        for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) out[j] = j;
    } else if (ranked) {
        const uint32_t* keys = a.keys + row * a.kstride;
        unsigned long long* cand = a.cand + row * a.cand_cap;
        // 16 keys per thread as four 16-byte loads; pass 1 counts, one global atomic per CTA
        // reserves the CTA's slots, pass 2 writes with shared-memory slot counters.
        constexpr int V4 = kTopkChunk / (4 * 256);
        uint32_t kk[V4][4];
        int bins[V4][4], ndef = 0, ncnd = 0;
#pragma unroll
        for (int v = 0; v < V4; ++v) {
            const int j = j0 + 4 * (static_cast<int>(threadIdx.x) + 256 * v);
            uint4 q = make_uint4(0, 0, 0, 0);
            if (j < j1) q = __ldcs(reinterpret_cast<const uint4*>(keys + j));
            kk[v][0] = q.x; kk[v][1] = q.y; kk[v][2] = q.z; kk[v][3] = q.w;
        }
#pragma unroll
        for (int v = 0; v < V4; ++v)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = j0 + 4 * (static_cast<int>(threadIdx.x) + 256 * v) + e;
                bins[v][e] = j < j1 ? score_bin(kk[v][e]) : kHistBins;
                ndef += bins[v][e] < b1;
                ncnd += bins[v][e] == b1;
            }
        if (threadIdx.x == 0) s_cnt[0] = s_cnt[1] = 0;
        __syncthreads();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ndef += __shfl_xor_sync(0xffffffffu, ndef, o);
            ncnd += __shfl_xor_sync(0xffffffffu, ncnd, o);
        }
        if ((threadIdx.x & 31) == 0) {
            atomicAdd(&s_cnt[0], ndef);
            atomicAdd(&s_cnt[1], ncnd);
        }
        __syncthreads();
        const int2 bases = block_reserve2(s_cnt[0], s_cnt[1], &meta[kMetaDef], &s_base2);
        const int def_base = bases.x, cnd_base = bases.y;
        if (threadIdx.x == 0) s_cnt[0] = s_cnt[1] = 0;
        __syncthreads();
#pragma unroll
        for (int v = 0; v < V4; ++v)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = j0 + 4 * (static_cast<int>(threadIdx.x) + 256 * v) + e;
                const bool def = bins[v][e] < b1;
                const bool cnd = bins[v][e] == b1;
                const int sd = warp_append(def, &s_cnt[0]);
                if (def && def_base + sd < above) out[def_base + sd] = j;
                const int sc = warp_append(cnd, &s_cnt[1]);
                if (cnd && cnd_base + sc < a.cand_cap) cand[cnd_base + sc] = composite(kk[v][e], j);
            }
    }

    // completion: the row's last CTA finishes the row
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&meta[kMetaSelDone], 1) == participants - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    for (int i = threadIdx.x; i < ri.wcnt; i += blockDim.x) idx[i] = ri.pos - ri.wcnt + 1 + i;
    for (int i = ri.wcnt + ri.keff + threadIdx.x; i < kw; i += blockDim.x) idx[i] = -1;
    if (threadIdx.x == 0) {
        a.cnt[row] = ri.wcnt + ri.keff;
        s_count = 0;
    }
    if (!ranked || above < 0 || above >= ri.keff) return;  // the last two tests hold for a consistent histogram
    const unsigned need = static_cast<unsigned>(ri.keff - above);
    const int ncand = __ldcg(&meta[kMetaCand]);
    int32_t* tail = out + above;
    __syncthreads();
    if (ncand <= a.cand_cap) {
        const unsigned long long* gc = a.cand + row * a.cand_cap;
        if (ncand <= kSmemCand) {
            for (int i = threadIdx.x; i < ncand; i += blockDim.x) s_cand[i] = __ldcg(gc + i);
            __syncthreads();
            const SmemSource src{s_cand, ncand};
            emit_at_least(src, radix_threshold(src, need, h, s_small), need, tail, &s_count);
        } else {
            const GlobalSource src{gc, ncand};
            emit_at_least(src, radix_threshold(src, need, h, s_small), need, tail, &s_count);
        }
    } else {
        if (threadIdx.x == 0) set_status(a.status, HS2_DEV_CAND_OVERFLOW);
        const KeyScanSource src{a.keys + row * a.kstride, ri.P, b1};
        emit_at_least(src, radix_threshold(src, need, h, s_small), need, tail, &s_count);
    }
}

// ====================================================================== one CTA per row (many rows)
//
// With thousands of selection rows (chunked prefill) one CTA finishes a whole row: it builds
// the row's histogram in shared memory, finds the threshold bucket with a block scan, then
// reads the row's keys again (mostly from L2) to write the keys of better buckets and collect
// the threshold bucket's candidates in shared memory, and radix-selects the exact remainder.
// No cross-CTA counters or global histograms.

template <int NT>
__global__ void __launch_bounds__(NT) topk_rows_kernel(const TopkArgs a) {
    __shared__ unsigned sh[kHistBins];
    __shared__ unsigned long long s_cand[kSmemCand];
    __shared__ unsigned h[256];
    __shared__ unsigned s_small[2];
    __shared__ unsigned s_warp[32];
    __shared__ int s_b1, s_above, s_ndef, s_ncand, s_count;
    static_assert(kHistBins % NT == 0 && NT % 32 == 0, "bins per thread");
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_trigger();
    for (int i = tid; i < kHistBins; i += NT) sh[i] = 0u;
    if (tid == 0) {
        s_ndef = s_ncand = s_count = 0;
        s_b1 = kHistBins;
        s_above = -1;
    }
    const RowInfo ri = make_row_info(a.pos, row, a.Hkv, a.T, a.N, a.k, a.W);
    const int kw = a.k + a.W;
    int32_t* idx = a.idx + row * kw;
    int32_t* out = idx + ri.wcnt;
    pdl_wait();  // keys from the score sweep
    for (int i = tid; i < ri.wcnt; i += NT) idx[i] = ri.pos - ri.wcnt + 1 + i;
    for (int i = ri.wcnt + ri.keff + tid; i < kw; i += NT) idx[i] = -1;
    if (tid == 0) a.cnt[row] = ri.wcnt + ri.keff;
    if (ri.keff == 0) return;
    if (ri.keff == ri.P) {  // the whole pool is selected
        for (int j = tid; j < ri.P; j += NT) out[j] = j;
        return;
    }
    const uint32_t* keys = a.keys + row * a.kstride;
    __syncthreads();
    // pass 1: histogram (rows are 256-byte aligned: 16-byte loads, 4 keys each)
    for (int base = 0; base < ri.P; base += 4 * NT) {
        const int j = base + 4 * tid;
        if (j < ri.P) {
            const uint4 q = __ldcg(reinterpret_cast<const uint4*>(keys + j));
            const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (j + e < ri.P) atomicAdd(&sh[score_bin(kk[e])], 1u);
        }
    }
    __syncthreads();
    {
        constexpr int PER = kHistBins / NT;
        unsigned vals[PER], sum = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            vals[i] = sh[tid * PER + i];
            sum += vals[i];
        }
        const unsigned excl = block_exclusive_scan(sum, s_warp);
        const unsigned need = static_cast<unsigned>(ri.keff);
        if (excl < need && need <= excl + sum) {
            unsigned cum = excl;
            for (int i = 0; i < PER; ++i) {
                if (cum + vals[i] >= need) {
                    s_b1 = tid * PER + i;
                    s_above = static_cast<int>(cum);
                    break;
                }
                cum += vals[i];
            }
        }
    }
    __syncthreads();
    const int b1 = s_b1, above = s_above;
    if (above < 0 || above >= ri.keff) return;  // cannot happen for a consistent histogram
    // pass 2: keys of better buckets go straight out, the threshold bucket's are candidates.
    // Each thread has 4 keys; a warp with any hit scans its per-lane counts (packed: defs in the
    // low, candidates in the high half-word) and reserves its slots with one shared-memory
    // atomic per list.
    const int lane = tid & 31;
    for (int base = 0; base < ri.P; base += 4 * NT) {  // warp-uniform trip count (shuffles inside)
        const int j = base + 4 * tid;
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (j < ri.P) q = __ldcg(reinterpret_cast<const uint4*>(keys + j));
        const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
        unsigned dmask = 0u, cmask = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int bin = j + e < ri.P ? score_bin(kk[e]) : kHistBins;
            dmask |= static_cast<unsigned>(bin < b1) << e;
            cmask |= static_cast<unsigned>(bin == b1) << e;
        }
        if (!__any_sync(0xffffffffu, (dmask | cmask) != 0u)) continue;
        const unsigned mine = __popc(dmask) | (__popc(cmask) << 16);  // <= 128 per warp: no carry
        unsigned incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int bdef = 0, bcnd = 0;
        if (lane == 31) {
            if (incl & 0xFFFFu) bdef = atomicAdd(&s_ndef, static_cast<int>(incl & 0xFFFFu));
            if (incl >> 16) bcnd = atomicAdd(&s_ncand, static_cast<int>(incl >> 16));
        }
        bdef = __shfl_sync(0xffffffffu, bdef, 31);
        bcnd = __shfl_sync(0xffffffffu, bcnd, 31);
        const unsigned excl = incl - mine;
        int od = bdef + static_cast<int>(excl & 0xFFFFu);
        int oc = bcnd + static_cast<int>(excl >> 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (dmask >> e & 1u) {
                if (od < above) out[od] = j + e;
                ++od;
            }
            if (cmask >> e & 1u) {
                if (oc < kSmemCand) s_cand[oc] = composite(kk[e], j + e);
                ++oc;
            }
        }
    }
    __syncthreads();
    const unsigned need = static_cast<unsigned>(ri.keff - above);
    const int ncand = s_ncand;
    int32_t* tail = out + above;
    if (ncand <= kSmemCand) {
        const SmemSource src{s_cand, ncand};
        emit_at_least(src, radix_threshold(src, need, h, s_small), need, tail, &s_count);
    } else {  // more ties in one bucket than shared memory holds: scan the row's keys again
        const KeyScanSource src{keys, ri.P, b1};
        emit_at_least(src, radix_threshold(src, need, h, s_small), need, tail, &s_count);
    }
}

cudaError_t launch_topk_rows(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    const cudaError_t e =
        launch_pdl(topk_rows_kernel<512>, dim3(static_cast<unsigned>(p.rows_kv)), dim3(512), 0, st, a);
    trace_mark("topk_rows", st);
    return e;
}

cudaError_t launch_topk_hist(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    dim3 grid((p.N + kTopkChunk - 1) / kTopkChunk, static_cast<unsigned>(p.rows_kv));
    const cudaError_t e = launch_pdl(topk_hist_kernel, grid, dim3(256), 0, st, a);
    trace_mark("topk_hist", st);
    return e;
}

cudaError_t launch_topk_select(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    dim3 grid((p.N + kTopkChunk - 1) / kTopkChunk, static_cast<unsigned>(p.rows_kv));
    const cudaError_t e = launch_pdl(topk_select_kernel, grid, dim3(256), 0, st, a);
    trace_mark("topk_select", st);
    return e;
}

}  // namespace hs2
