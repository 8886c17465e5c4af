// Pieces of the exact token-level top-k shared by the scoring and selection kernels.
//
// Keys: the fp32 score s (base-2 units) maps to an order-preserving uint32 (score_key).
// Buckets: score_bin is a monotone, non-increasing function of the score, read straight from
// the key's bits: a selection score is a log-probability (<= 0), and for s < 0 the key is
// 0x7FFFFFFF - bits(|s|), so bits(|s|) >> 15 (exponent and 8 mantissa bits) is a logarithmic
// bucket of |s| with 256 buckets per octave.  Buckets 0 .. 2047 cover |s| in [1/4, 64) (1/32
// of a unit per bucket around |s| = 8); |s| < 1/4 and s >= 0 share bucket 0, |s| >= 64 and
// NaN (key 0) the last one.  Every key in a better bucket than the bucket holding the k-th
// best key is selected outright.  Composite: (key << 32) | (2^32 - 1 - j) is distinct per
// key and orders by (score desc, index asc) -- exactly the selection rule with ties to the
// lower index.
#pragma once

#include "hs2_device.cuh"

namespace hs2 {

__device__ __forceinline__ int score_bin(uint32_t key) {
    constexpr int kFirst = (125 << 8);  // bits(0.25) >> 15
    const int v = (static_cast<int>(0x7FFFFFFFu - key) >> 15) - kFirst;  // negative for s >= 0
    return min(max(v, 0), kHistBins - 1);
}

__device__ __forceinline__ unsigned long long composite(uint32_t key, int j) {
    return (static_cast<unsigned long long>(key) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(j));
}
__device__ __forceinline__ int composite_index(unsigned long long c) {
    return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(c & 0xFFFFFFFFull));
}

struct RowInfo {
    int pos;   // query position (clamped into [0, N))
    int P;     // pool size: keys 0 .. pos-W
    int keff;  // min(k, P) keys come from the pool
    int wcnt;  // min(W, pos+1) window keys
};

__device__ __forceinline__ RowInfo make_row_info(const int32_t* pos, int64_t row, int Hkv, int T, int N, int k,
                                                 int W) {
    const int t = static_cast<int>(row % T);
    const int b = static_cast<int>(row / (static_cast<int64_t>(Hkv) * T));
    int p = pos[b * T + t];
    p = p < 0 ? 0 : (p >= N ? N - 1 : p);
    RowInfo r;
    r.pos = p;
    r.P = max(0, p - W + 1);
    r.keff = min(k, r.P);
    r.wcnt = min(W, p + 1);
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

// Reserves `n` consecutive slots of a global list for the whole CTA with one atomic: call from
// all threads with the CTA's total; returns the base slot (broadcast through *s_base).
__device__ __forceinline__ int block_reserve(int n, int* counter, int* s_base) {
    if (threadIdx.x == 0) *s_base = n > 0 ? atomicAdd(counter, n) : 0;
    __syncthreads();
    const int base = *s_base;
    __syncthreads();
    return base;
}

// Reserves n0 and n1 slots of two adjacent list counters (ctr[0], ctr[1], 8-byte aligned) with
// one 64-bit atomic for the whole CTA; returns both bases.  Call from all threads.
__device__ __forceinline__ int2 block_reserve2(int n0, int n1, int* ctr, unsigned long long* s_base) {
    if (threadIdx.x == 0) {
        const unsigned long long add = (static_cast<unsigned long long>(static_cast<unsigned>(n1)) << 32) |
                                       static_cast<unsigned>(n0);
        *s_base = add ? atomicAdd(reinterpret_cast<unsigned long long*>(ctr), add) : 0ull;  // nothing to reserve: unused
    }
    __syncthreads();
    const unsigned long long v = *s_base;
    __syncthreads();
    return make_int2(static_cast<int>(v & 0xFFFFFFFFull), static_cast<int>(v >> 32));
}

// Exclusive block-wide prefix sum of one value per thread (blockDim.x a multiple of 32).
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
        const unsigned w = lane < nw ? s_warp[lane] : 0u;
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

// Adds this CTA's shared-memory histogram to the row's global one; the last of the row's
// `participants` CTAs (a completion counter -- nothing waits) then finds the bucket b1 of the
// keff-th best key and the number of keys above it, and stores them in meta.
// blockDim.x must be 256.
__device__ __forceinline__ void hist_flush_and_threshold(const unsigned* sh, unsigned* hist, int* meta,
                                                         int participants, int keff, unsigned* s_warp,
                                                         int* s_last) {
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
        if (sh[i]) atomicAdd(&hist[i], sh[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *s_last = (atomicAdd(&meta[kMetaDone], 1) == participants - 1);
    __syncthreads();
    if (!*s_last) return;
    __threadfence();
    constexpr int PER = kHistBins / 256;
    unsigned vals[PER];
    unsigned sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        vals[i] = __ldcg(&hist[threadIdx.x * PER + i]);
        sum += vals[i];
    }
    const unsigned excl = block_exclusive_scan(sum, s_warp);
    const unsigned need = static_cast<unsigned>(keff);
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

// ------------------------------------------------------------------ exact threshold among candidates

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


// After a histogram in sh: for each of the two counts c[0], c[1] (>= 1), the smallest bucket b
// whose cumulative count (buckets 0 .. b) reaches c, and the count below it, into
// s_bin[i] / s_below[i] (bucket kHistBins - 1 and the count below it if c exceeds the total).
// Call from all threads (NT of them).
template <int NT>
__device__ __forceinline__ void buckets_at_counts(const unsigned* sh, const unsigned (&c)[2], unsigned* s_warp,
                                                  int* s_bin, int* s_below) {
    constexpr int PER = kHistBins / NT;
    const int tid = threadIdx.x;
    unsigned vals[PER], sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        vals[i] = sh[tid * PER + i];
        sum += vals[i];
    }
    const unsigned excl = block_exclusive_scan(sum, s_warp);
    const bool last_thread = tid == NT - 1;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        if (excl < c[k] && c[k] <= excl + sum) {
            unsigned cum = excl;
            for (int i = 0; i < PER; ++i) {
                if (cum + vals[i] >= c[k]) {
                    s_bin[k] = tid * PER + i;
                    s_below[k] = static_cast<int>(cum);
                    break;
                }
                cum += vals[i];
            }
        } else if (last_thread && c[k] > excl + sum) {  // beyond the total
            s_bin[k] = kHistBins - 1;
            s_below[k] = static_cast<int>(excl + sum - vals[PER - 1]);
        }
    }
}

}  // namespace hs2
