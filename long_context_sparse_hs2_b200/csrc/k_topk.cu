// Token-level top-k with a forced window (sm_100a).
//
// HySparse2 selects individual tokens (not blocks) and always includes the most recent
// ones ("HySparse2 od Xiaomi zkracuje zpracovani dlouheho kontextu", section "Proc neni
// nutne znovu zpracovat cely dlouhy vstup", third paragraph; DAIR.AI newsletter, HySparse2
// bullet "Prefill exits early").  Per selection row (b, kv head, t) this file picks the
// min(k, |pool|) pool keys [0, pos - W] of largest score, ties to the lower index, and
// writes them after the window [max(0, pos - W + 1), pos].
//
// Exactness: ranking uses the 64-bit composite c = (key << 32) | (2^32 - 1 - j), where key
// is the order-preserving image of the fp32 score.  Composites are distinct, and c_a > c_b
// iff s_a > s_b or (s_a == s_b and a < b), so "the k largest composites" is exactly the
// selection rule.  Three passes:
//   1. topk_hist_kernel: per-row histogram of a monotone bucketing of the score
//      (1/128 base-2 unit per bin, bin 0 = best); the last CTA of each row (a completion
//      counter, no waiting) finds the bucket b1 holding the k-th best key.
//   2. topk_emit_kernel: keys in better buckets are selected outright; keys in b1 are
//      appended to a candidate list (warp ballot + one atomic per warp, order arbitrary,
//      the compaction pattern of "Simplified Sparse Attention via Gist Tokens", section 3.6).
//   3. topk_final_kernel: one CTA per row radix-selects (8 bits per pass) the composite
//      threshold among the candidates and emits the winners; writes the window, the -1
//      padding and cnt.  If the candidate list overflowed, it re-scans the row's keys.
#include "hs2_device.cuh"
#include "hs2_internal.h"

namespace hs2 {

namespace {

constexpr int kSmemCand = 8192;  // candidates held in shared memory by the final pass

__device__ __forceinline__ int score_bin(uint32_t key) {
    if (key == 0u) return kHistBins - 1;  // NaN ranks last
    const float x = -key_score(key) * kBinsPerUnit;
    if (!(x > 0.f)) return 0;
    if (x >= static_cast<float>(kHistBins - 1)) return kHistBins - 1;
    return static_cast<int>(x);
}

__device__ __forceinline__ unsigned long long composite(uint32_t key, int j) {
    return (static_cast<unsigned long long>(key) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(j));
}
__device__ __forceinline__ int composite_index(unsigned long long c) {
    return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(c & 0xFFFFFFFFull));
}

struct RowInfo {
    int pos, P, keff, wcnt;
};

__device__ __forceinline__ RowInfo row_info(const TopkArgs& a, int64_t row) {
    const int t = static_cast<int>(row % a.T);
    const int b = static_cast<int>(row / (static_cast<int64_t>(a.Hkv) * a.T));
    int p = a.pos[b * a.T + t];
    p = p < 0 ? 0 : (p >= a.N ? a.N - 1 : p);
    RowInfo r;
    r.pos = p;
    r.P = max(0, p - a.W + 1);
    r.keff = min(a.k, r.P);
    r.wcnt = min(a.W, p + 1);
    return r;
}

// Appends the lanes with pred set to a global list; returns the lane's slot (or -1).
__device__ __forceinline__ int warp_append(bool pred, int* counter) {
    const unsigned mask = __ballot_sync(0xffffffffu, pred);
    if (mask == 0u) return -1;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(mask) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(counter, __popc(mask));
    base = __shfl_sync(0xffffffffu, base, leader);
    return pred ? base + __popc(mask & ((1u << lane) - 1u)) : -1;
}

// Exclusive block-wide prefix sum of one value per thread (blockDim.x multiple of 32, <= 1024).
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    unsigned incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        unsigned w = lane < nw ? s_warp[lane] : 0u;
        unsigned wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nw) s_warp[lane] = wi - w;
    }
    __syncthreads();
    const unsigned r = s_warp[warp] + incl - v;
    __syncthreads();
    return r;
}

}  // namespace

// ====================================================================== pass 1: histogram + threshold bucket

__global__ void __launch_bounds__(256) topk_hist_kernel(const TopkArgs a) {
    __shared__ unsigned sh[kHistBins];
    __shared__ unsigned s_warp[32];
    __shared__ int s_last;
    const int64_t row = blockIdx.y;
    const RowInfo ri = row_info(a, row);
    if (ri.keff == 0 || ri.keff == ri.P) return;  // nothing to rank
    const int nchunks = (ri.P + kTopkChunk - 1) / kTopkChunk;
    if (static_cast<int>(blockIdx.x) >= nchunks) return;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    const int j0 = blockIdx.x * kTopkChunk, j1 = min(j0 + kTopkChunk, ri.P);
    const uint32_t* keys = a.keys + row * a.N;
    for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) atomicAdd(&sh[score_bin(keys[j])], 1u);
    __syncthreads();
    unsigned* hist = a.hist + row * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
        if (sh[i]) atomicAdd(&hist[i], sh[i]);
    __threadfence();
    __syncthreads();
    int* meta = a.meta + row * kMetaInts;
    if (threadIdx.x == 0) s_last = (atomicAdd(&meta[kMetaDone], 1) == nchunks - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // Bucket of the keff-th best key: smallest b1 with count(bins <= b1) >= keff.
    constexpr int PER = kHistBins / 256;
    unsigned vals[PER];
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        vals[i] = __ldcg(&hist[threadIdx.x * PER + i]);
        sum += vals[i];
    }
    const unsigned excl = block_exclusive_scan(sum, s_warp);
    const unsigned need = static_cast<unsigned>(ri.keff);
    if (excl < need && need <= excl + sum) {
        unsigned cum = excl;
        for (int i = 0; i < PER; ++i) {
            if (cum + vals[i] >= need) {
                meta[kMetaBin] = threadIdx.x * PER + i;
                meta[kMetaAbove] = static_cast<int>(cum);
                break;
            }
            cum += vals[i];
        }
    }
}

// ====================================================================== pass 2: emit winners, compact candidates

__global__ void __launch_bounds__(256) topk_emit_kernel(const TopkArgs a) {
    const int64_t row = blockIdx.y;
    const RowInfo ri = row_info(a, row);
    if (ri.keff == 0) return;
    const int j0 = blockIdx.x * kTopkChunk;
    if (j0 >= ri.P) return;
    const int j1 = min(j0 + kTopkChunk, ri.P);
    int32_t* out = a.idx + row * (a.k + a.W) + ri.wcnt;
    if (ri.keff == ri.P) {  // the whole pool is selected
        for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) out[j] = j;
        return;
    }
    int* meta = a.meta + row * kMetaInts;
    const int b1 = meta[kMetaBin];
    const int above = meta[kMetaAbove];
    const uint32_t* keys = a.keys + row * a.N;
    unsigned long long* cand = a.cand + row * a.cand_cap;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int base = j0 + warp * 32; base < j1; base += blockDim.x) {
        const int j = base + lane;
        const bool valid = j < j1;
        const uint32_t key = valid ? keys[j] : 0u;
        const int bin = valid ? score_bin(key) : kHistBins;
        const bool def = valid && bin < b1;
        const bool cnd = valid && bin == b1;
        const int sd = warp_append(def, &meta[kMetaDef]);
        if (def && sd < above) out[sd] = j;
        const int sc = warp_append(cnd, &meta[kMetaCand]);
        if (cnd && sc < a.cand_cap) cand[sc] = composite(key, j);
    }
}

// ====================================================================== pass 3: exact threshold among candidates

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
        const uint32_t k = keys[i];
        v = composite(k, i);
        return score_bin(k) == b1;
    }
};

// Largest composite threshold T such that exactly `need` source elements are >= T.
template <class Src>
__device__ unsigned long long radix_threshold(const Src& src, unsigned need, unsigned* h, unsigned* s_small) {
    unsigned long long prefix = 0ull;
    const int lane = threadIdx.x & 31;
    for (int shift = 56; shift >= 0; shift -= 8) {
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

// Writes the elements >= thr; at most `need` slots are written whatever the inputs.
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

__global__ void __launch_bounds__(512) topk_final_kernel(const TopkArgs a) {
    extern __shared__ unsigned long long s_cand[];
    __shared__ unsigned h[256];
    __shared__ unsigned s_small[2];
    __shared__ int s_count;
    const int64_t row = blockIdx.x;
    const RowInfo ri = row_info(a, row);
    const int kw = a.k + a.W;
    int32_t* idx = a.idx + row * kw;
    for (int i = threadIdx.x; i < ri.wcnt; i += blockDim.x) idx[i] = ri.pos - ri.wcnt + 1 + i;
    for (int i = ri.wcnt + ri.keff + threadIdx.x; i < kw; i += blockDim.x) idx[i] = -1;
    if (threadIdx.x == 0) {
        a.cnt[row] = ri.wcnt + ri.keff;
        s_count = 0;
    }
    if (ri.keff == 0 || ri.keff == ri.P) return;
    const int* meta = a.meta + row * kMetaInts;
    const int b1 = meta[kMetaBin];
    const int above = meta[kMetaAbove];
    if (above < 0 || above >= ri.keff) return;  // cannot happen with a consistent histogram
    const unsigned need = static_cast<unsigned>(ri.keff - above);
    const int ncand = meta[kMetaCand];
    int32_t* out = idx + ri.wcnt + above;
    __syncthreads();
    if (ncand <= a.cand_cap) {
        const unsigned long long* gc = a.cand + row * a.cand_cap;
        if (ncand <= kSmemCand) {
            for (int i = threadIdx.x; i < ncand; i += blockDim.x) s_cand[i] = __ldcg(gc + i);
            __syncthreads();
            const SmemSource src{s_cand, ncand};
            const unsigned long long thr = radix_threshold(src, need, h, s_small);
            emit_at_least(src, thr, need, out, &s_count);
        } else {
            const GlobalSource src{gc, ncand};
            const unsigned long long thr = radix_threshold(src, need, h, s_small);
            emit_at_least(src, thr, need, out, &s_count);
        }
    } else {
        if (threadIdx.x == 0) set_status(a.status, HS2_DEV_CAND_OVERFLOW);
        const KeyScanSource src{a.keys + row * a.N, ri.P, b1};
        const unsigned long long thr = radix_threshold(src, need, h, s_small);
        emit_at_least(src, thr, need, out, &s_count);
    }
}

cudaError_t launch_topk(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    const unsigned chunks = static_cast<unsigned>((p.N + kTopkChunk - 1) / kTopkChunk);
    dim3 grid(chunks, static_cast<unsigned>(p.rows_kv));
    topk_hist_kernel<<<grid, 256, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    topk_emit_kernel<<<grid, 256, 0, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int bytes = kSmemCand * 8;
    e = cudaFuncSetAttribute(topk_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    topk_final_kernel<<<static_cast<unsigned>(p.rows_kv), 512, bytes, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hs2
