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
// topk_hist_kernel below after a K re-sweep); each CTA takes every gridDim.x-th 4096-key
// chunk of its row.  topk_select_kernel then:
//   * selects every key in a better bucket than b1 outright and appends the keys of b1 to a
//     candidate list (warp ballot + one atomic per warp; order arbitrary -- the compaction
//     pattern of "Simplified Sparse Attention via Gist Tokens", section 3.6);
//   * the row's last CTA (completion counter; nothing waits) radix-selects, 8 bits per pass,
//     the exact 64-bit composite threshold among the candidates, emits the winners, and
//     writes the window, the -1 padding and cnt.  If the candidate list overflowed its
//     capacity it re-scans the row's keys instead (exact, slower, flagged).
// With thousands of rows topk_rows_kernel (further below) finishes each row in one CTA.
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
    // the row's chunks are shared out over at most gridDim.x CTAs
    const int nchunks = (ri.P + kTopkChunk - 1) / kTopkChunk;
    const int participants = min(nchunks, static_cast<int>(gridDim.x));
    if (static_cast<int>(blockIdx.x) >= participants) return;
    __syncthreads();
    const uint32_t* keys = a.keys + row * a.kstride;
    for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
        const int j0 = c * kTopkChunk, j1 = min(j0 + kTopkChunk, ri.P);
        // 4 keys per thread per 16-byte load (rows are 256-byte aligned, j0 a multiple of 4)
        for (int j = j0 + 4 * static_cast<int>(threadIdx.x); j < j1; j += 4 * blockDim.x) {
            const uint4 q = __ldcs(reinterpret_cast<const uint4*>(keys + j));
            const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (j + e < j1) atomicAdd(&sh[score_bin(kk[e])], 1u);
        }
    }
    __syncthreads();
    hist_flush_and_threshold(sh, a.hist + row * kHistBins, a.meta + row * kMetaInts, participants, ri.keff, s_warp,
                             &s_last);
}

// ====================================================================== select: emit, then exact threshold

constexpr int kRankCand = 1024;  // up to this many threshold-bucket candidates are ranked directly

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
    // the row's chunks are shared out over at most gridDim.x CTAs
    const int nchunks = max(1, (ri.P + kTopkChunk - 1) / kTopkChunk);
    const int participants = min(nchunks, static_cast<int>(gridDim.x));
    pdl_trigger();
    pdl_wait();  // keys, histogram threshold and cleared counters from the kernels before
    if (static_cast<int>(blockIdx.x) >= participants) return;
    const int kw = a.k + a.W;
    int32_t* idx = a.idx + row * kw;
    int32_t* out = idx + ri.wcnt;  // the pool's winners follow the window
    int* meta = a.meta + row * kMetaInts;
    const bool ranked = ri.keff > 0 && ri.keff < ri.P;
    const int b1 = ranked ? meta[kMetaBin] : 0;
    const int above = ranked ? meta[kMetaAbove] : 0;

    for (int chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
        const int j0 = chunk * kTopkChunk, j1 = min(j0 + kTopkChunk, ri.P);
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
            __syncthreads();  // the slot counters are reset for the next chunk
        }

    }  // chunks

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
            if (ncand <= kRankCand) {
                // few candidates: each one's rank among them (composites are distinct) is its slot,
                // and it is selected iff that rank is below need -- one pass, no radix passes
                for (int i = threadIdx.x; i < ncand; i += blockDim.x) {
                    const unsigned long long c = s_cand[i];
                    unsigned r = 0;
                    for (int j = 0; j < ncand; ++j) r += s_cand[j] > c;
                    if (r < need) tail[r] = composite_index(c);
                }
            } else {
                const SmemSource src{s_cand, ncand};
                emit_at_least(src, radix_threshold(src, need, h, s_small), need, tail, &s_count);
            }
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
// With thousands of selection rows (chunked prefill) one CTA finishes a whole row, with no
// cross-CTA counters or global histograms.  Bucket ranges bracket the threshold:
//   1. a histogram of a 1/16 sample of the row's keys (one 16-byte group in sixteen) gives
//      buckets b_lo <= b_hi around the sample's estimate of the keff-th best key, with a
//      margin of several standard deviations;
//   2. one pass over all keys writes the keys of buckets < b_lo to the output and collects the
//      keys of buckets b_lo .. b_hi as candidates in shared memory;
//   3. if #(bucket < b_lo) <= keff <= #(bucket <= b_hi) and the candidates fit, the selection is
//      exactly those keys plus the best (keff - #(bucket < b_lo)) candidates by radix select
//      (a better bucket means a strictly better score);
//   4. otherwise (an unlucky sample, heavy ties, small pools) the exact two-pass method runs:
//      full histogram, threshold bucket, emit, radix select.
// Either way the result is the exact top-keff with ties to the lower index.

namespace {

constexpr int kSampleStride = 16;        // sample one 4-key group in 16
constexpr int kSampleMinPool = 32768;    // smaller pools go straight to the two-pass method

// Writes the keys of buckets < lo to out (the first `cap` of them) and collects the keys of
// buckets lo .. hi as candidates in s_cand (the first kSmemCand); counts both in *s_ndef and
// *s_ncand.  Each thread takes 4 keys per step; a warp with any hit scans its lanes' counts
// (packed: defs low, candidates high half-word) and reserves slots with one shared atomic per
// list.  Call from all threads.
template <int NT>
__device__ __forceinline__ void emit_bucket_range(const uint32_t* keys, int P, int lo, int hi, int cap, int32_t* out,
                                                  unsigned long long* s_cand, int* s_ndef, int* s_ncand) {
    const int lane = threadIdx.x & 31;
    for (int base = 0; base < P; base += 4 * NT) {  // warp-uniform trip count (shuffles inside)
        const int j = base + 4 * static_cast<int>(threadIdx.x);
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (j < P) q = __ldcg(reinterpret_cast<const uint4*>(keys + j));
        const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
        unsigned dmask = 0u, cmask = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int bin = j + e < P ? score_bin(kk[e]) : kHistBins;
            dmask |= static_cast<unsigned>(bin < lo) << e;
            cmask |= static_cast<unsigned>(bin >= lo && bin <= hi) << e;
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
            if (incl & 0xFFFFu) bdef = atomicAdd(s_ndef, static_cast<int>(incl & 0xFFFFu));
            if (incl >> 16) bcnd = atomicAdd(s_ncand, static_cast<int>(incl >> 16));
        }
        bdef = __shfl_sync(0xffffffffu, bdef, 31);
        bcnd = __shfl_sync(0xffffffffu, bcnd, 31);
        const unsigned excl = incl - mine;
        int od = bdef + static_cast<int>(excl & 0xFFFFu);
        int oc = bcnd + static_cast<int>(excl >> 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (dmask >> e & 1u) {
                if (od < cap) out[od] = j + e;
                ++od;
            }
            if (cmask >> e & 1u) {
                if (oc < kSmemCand) s_cand[oc] = composite(kk[e], j + e);
                ++oc;
            }
        }
    }
}

}  // namespace

template <int NT>
__global__ void __launch_bounds__(NT) topk_rows_kernel(const TopkArgs a) {
    __shared__ unsigned sh[kHistBins];
    __shared__ unsigned long long s_cand[kSmemCand];
    __shared__ unsigned h[256];
    __shared__ unsigned s_small[2];
    __shared__ unsigned s_warp[32];
    __shared__ int s_bin[2], s_below[2], s_ndef, s_ncand, s_count, s_nsample;
    static_assert(kHistBins % NT == 0 && NT % 32 == 0, "bins per thread");
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_trigger();
    for (int i = tid; i < kHistBins; i += NT) sh[i] = 0u;
    if (tid == 0) {
        s_ndef = s_ncand = s_count = s_nsample = 0;
        s_bin[0] = s_bin[1] = kHistBins - 1;
        s_below[0] = s_below[1] = 0;
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
    const uint32_t* keys = a.keys + row * a.kstride;  // rows are 256-byte aligned: 16-byte loads
    __syncthreads();

    if (ri.P >= kSampleMinPool) {
        // 1. sample histogram
        int mine = 0;
        const int groups = (ri.P + 3) / 4;
        for (int g = tid * kSampleStride; g < groups; g += NT * kSampleStride) {
            const int j = 4 * g;
            const uint4 q = __ldcg(reinterpret_cast<const uint4*>(keys + j));
            const uint32_t kk[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (j + e < ri.P) {
                    atomicAdd(&sh[score_bin(kk[e])], 1u);
                    ++mine;
                }
        }
        if (mine) atomicAdd(&s_nsample, mine);
        __syncthreads();
        const float ns = static_cast<float>(s_nsample);
        const float r = static_cast<float>(ri.keff) * ns / static_cast<float>(ri.P);  // expected sample rank
        const float margin = 4.f * sqrtf(r) + 16.f;
        const unsigned c[2] = {static_cast<unsigned>(fmaxf(r - margin, 0.f)) + 1u,
                               static_cast<unsigned>(fminf(r + margin, ns)) + 1u};
        buckets_at_counts<NT>(sh, c, s_warp, s_bin, s_below);
        __syncthreads();
        // 2. one pass: buckets < lo out, lo .. hi candidates
        const int lo = s_bin[0], hi = s_bin[1];
        emit_bucket_range<NT>(keys, ri.P, lo, hi, ri.keff, out, s_cand, &s_ndef, &s_ncand);
        __syncthreads();
        // 3. bracketed?
        const int ndef = s_ndef, ncand = s_ncand;
        if (ndef <= ri.keff && ri.keff <= ndef + ncand && ncand <= kSmemCand) {
            const unsigned need = static_cast<unsigned>(ri.keff - ndef);
            if (need > 0) {
                const SmemSource src{s_cand, ncand};
                emit_at_least(src, radix_threshold(src, need, h, s_small), need, out + ndef, &s_count);
            }
            return;
        }
        // 4. not bracketed: start over with the exact two-pass method
        for (int i = tid; i < kHistBins; i += NT) sh[i] = 0u;
        if (tid == 0) {
            s_ndef = s_ncand = 0;
            s_bin[0] = s_bin[1] = kHistBins - 1;
            s_below[0] = s_below[1] = 0;
        }
        __syncthreads();
    }

    // exact two-pass method: full histogram
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
        const unsigned c[2] = {static_cast<unsigned>(ri.keff), static_cast<unsigned>(ri.keff)};
        buckets_at_counts<NT>(sh, c, s_warp, s_bin, s_below);
    }
    __syncthreads();
    const int b1 = s_bin[0], above = s_below[0];
    if (above < 0 || above >= ri.keff) return;  // cannot happen for a consistent histogram
    // keys of better buckets go straight out, the threshold bucket's are candidates
    emit_bucket_range<NT>(keys, ri.P, b1, b1, above, out, s_cand, &s_ndef, &s_ncand);
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

// ====================================================================== bracketed selection (unstored keys)
//
// With long pools and many rows (prefill) the keys are never stored.  The tcgen05 score sweep
// first scores one 128-key tile in kSampleTileStride (keys compacted per row); topk_bracket
// turns each row's sample into a bucket bracket b_hi -- the bucket of the sample key at rank
// (expected rank of the keff-th best key) + margin; a second, filtering sweep writes every key
// of bucket <= b_hi to the row's candidate list (each epilogue warp of the sweep fills its own
// segment, so no atomics); topk_finalize radix-selects the exact top-keff among them.  A key of a bucket above b_hi scores strictly below every candidate, so the
// result is exact whenever the list holds at least keff keys and nothing overflowed; where it
// did not (an unlucky sample, heavy ties) topk_finalize rescores the row from Q, K and LSE on
// the CUDA cores and selects exactly (flagged HS2_DEV_CAND_OVERFLOW, informational).

__global__ void __launch_bounds__(256) topk_bracket_kernel(const TopkArgs a) {
    __shared__ unsigned sh[kHistBins];
    __shared__ unsigned s_warp[32];
    __shared__ int s_bin[2], s_below[2];
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_trigger();
    for (int i = tid; i < kHistBins; i += blockDim.x) sh[i] = 0u;
    if (tid == 0) {
        s_bin[0] = s_bin[1] = kHistBins - 1;
        s_below[0] = s_below[1] = 0;
    }
    const RowInfo ri = make_row_info(a.pos, row, a.Hkv, a.T, a.N, a.k, a.W);
    int* meta = a.meta + row * kMetaInts;
    pdl_wait();  // sample keys from the sampling sweep; the previous readers of meta are done
    if (ri.keff == 0 || ri.keff == ri.P) {  // nothing to rank: the filter takes no key
        if (tid == 0) meta[kMetaBin] = -1;
        return;
    }
    constexpr int kSpan = kSampleTileStride * 128;  // pool keys per sample tile
    const int nv = (ri.P + kSpan - 1) / kSpan;      // sample tiles (the last one may be short)
    const int ns = 128 * (nv - 1) + min(128, ri.P - kSpan * (nv - 1));
    const float r = static_cast<float>(ri.keff) * static_cast<float>(ns) / static_cast<float>(ri.P);
    const float margin = 4.f * sqrtf(r) + 16.f;
    if (ns < 256 || r + margin >= static_cast<float>(ns)) {  // too small a sample: every key is a candidate
        if (tid == 0) meta[kMetaBin] = kHistBins - 1;
        return;
    }
    __syncthreads();
    const uint32_t* keys = a.keys + row * a.kstride;
    for (int i = tid; i < nv * 128; i += blockDim.x) {
        const int v = i >> 7, rr = i & 127;
        if (rr < ri.P - kSpan * v) atomicAdd(&sh[score_bin(__ldcs(keys + i))], 1u);
    }
    __syncthreads();
    const unsigned c = static_cast<unsigned>(r + margin) + 1u;
    const unsigned cc[2] = {c, c};
    buckets_at_counts<256>(sh, cc, s_warp, s_bin, s_below);
    __syncthreads();
    if (tid == 0) meta[kMetaBin] = s_bin[0];
}

namespace {

// The selection key of pool key j for one row, recomputed on the CUDA cores: max over the G
// heads of (q_g . k_j - u_g) scaled to base 2 (u_g = LSE_g sqrt(d), q in shared memory as fp32).
struct Rescorer {
    const uint16_t* K;  // this (b, kv head)'s keys [N][d]
    const float* q;     // [G][d]
    const float* u;     // [G]
    int G, d;
    float c2;
    __device__ uint32_t key(int j) const {
        const uint4* kr = reinterpret_cast<const uint4*>(K + static_cast<int64_t>(j) * d);
        float best = -INFINITY;
        bool nan = false;
        for (int g = 0; g < G; ++g) {
            const float* qg = q + g * d;
            float x = 0.f;
            for (int c = 0; c < d / 8; ++c) {
                const uint4 w = __ldg(kr + c);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x = fmaf(qg[8 * c + 2 * e], __uint_as_float(ww[e] << 16), x);
                    x = fmaf(qg[8 * c + 2 * e + 1], __uint_as_float(ww[e] & 0xFFFF0000u), x);
                }
            }
            const float v = x - u[g];
            nan |= v != v;
            best = fmaxf(best, v);
        }
        return nan ? 0u : score_key(best * c2);  // NaN ranks below every score
    }
};

struct SegmentSource {  // the candidates of a row's list segments (seg_start: nseg + 1 prefix offsets)
    const unsigned long long* c;
    const int* seg_start;
    int nseg, seg_cap, n;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const {
        int sg = 0;
        while (sg + 1 < nseg && i >= seg_start[sg + 1]) ++sg;
        v = __ldcg(c + sg * seg_cap + (i - seg_start[sg]));
        return true;
    }
};

struct RescoreSource {  // the pool keys of bucket b1, recomputed
    Rescorer rs;
    int n, b1;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const {
        const uint32_t k = rs.key(i);
        v = composite(k, i);
        return score_bin(k) == b1;
    }
};

}  // namespace

template <int NT>
__global__ void __launch_bounds__(NT) topk_finalize_kernel(const TopkArgs a) {
    __shared__ unsigned long long s_cand[kSmemCand];  // candidates; the fallback keeps Q here
    __shared__ unsigned sh[kHistBins];
    __shared__ unsigned h[256];
    __shared__ unsigned s_small[2];
    __shared__ unsigned s_warp[32];
    __shared__ float s_u[16];
    __shared__ int s_bin[2], s_below[2], s_ndef, s_ncand, s_count;
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_trigger();
    if (tid == 0) {
        s_ndef = s_ncand = s_count = 0;
        s_bin[0] = s_bin[1] = kHistBins - 1;
        s_below[0] = s_below[1] = 0;
    }
    const RowInfo ri = make_row_info(a.pos, row, a.Hkv, a.T, a.N, a.k, a.W);
    const int kw = a.k + a.W;
    int32_t* idx = a.idx + row * kw;
    int32_t* out = idx + ri.wcnt;
    pdl_wait();  // candidates from the filtering sweep
    for (int i = tid; i < ri.wcnt; i += NT) idx[i] = ri.pos - ri.wcnt + 1 + i;
    for (int i = ri.wcnt + ri.keff + tid; i < kw; i += NT) idx[i] = -1;
    if (tid == 0) a.cnt[row] = ri.wcnt + ri.keff;
    if (ri.keff == 0) return;
    if (ri.keff == ri.P) {  // the whole pool is selected
        for (int j = tid; j < ri.P; j += NT) out[j] = j;
        return;
    }
    unsigned long long* gcand = a.cand + row * a.cand_cap;
    // the candidates: nseg segments of the row's list, each filled by one epilogue warp
    __shared__ int s_seg[kMaxSegments + 1];
    __shared__ int s_over;
    if (tid == 0) {
        int total = 0, over = 0;
        for (int sg = 0; sg < a.nseg; ++sg) {
            const int c = __ldcg(a.segcnt + row * a.nseg + sg);
            over |= c > a.seg_cap;
            s_seg[sg] = total;
            total += min(c, a.seg_cap);
        }
        s_seg[a.nseg] = total;
        s_over = over;
    }
    __syncthreads();
    const int n = s_seg[a.nseg];
    if (!s_over && n >= ri.keff) {  // bracketed: the exact top-keff among the candidates
        const unsigned need = static_cast<unsigned>(ri.keff);
        if (n <= kSmemCand) {
            for (int sg = 0; sg < a.nseg; ++sg) {
                const int c = s_seg[sg + 1] - s_seg[sg];
                for (int i = tid; i < c; i += NT) s_cand[s_seg[sg] + i] = __ldcg(gcand + sg * a.seg_cap + i);
            }
            __syncthreads();
            const SmemSource src{s_cand, n};
            emit_at_least(src, radix_threshold(src, need, h, s_small), need, out, &s_count);
        } else {
            const SegmentSource src{gcand, s_seg, a.nseg, a.seg_cap, n};
            emit_at_least(src, radix_threshold(src, need, h, s_small), need, out, &s_count);
        }
        return;
    }

    // not bracketed: rescore the row (exact two-pass method on recomputed keys)
    if (tid == 0) set_status(a.status, HS2_DEV_CAND_OVERFLOW);
    const int t = static_cast<int>(row % a.T);
    const int64_t bh = row / a.T;  // b * Hkv + kv head
    const int b = static_cast<int>(bh / a.Hkv), hk = static_cast<int>(bh % a.Hkv);
    float* s_q = reinterpret_cast<float*>(s_cand);  // G * d <= 2048 floats
    const float sqrt_d = sqrtf(static_cast<float>(a.d));
    for (int i = tid; i < a.G * a.d; i += NT) {
        const int g = i / a.d, c = i % a.d;
        const int64_t hq = static_cast<int64_t>(b) * a.Hq + hk * a.G + g;
        s_q[i] = __uint_as_float(static_cast<uint32_t>(a.Q[(hq * a.T + t) * a.d + c]) << 16);
    }
    for (int g = tid; g < a.G; g += NT) s_u[g] = a.lse[(static_cast<int64_t>(b) * a.Hq + hk * a.G + g) * a.T + t] * sqrt_d;
    for (int i = tid; i < kHistBins; i += NT) sh[i] = 0u;
    __syncthreads();
    const Rescorer rs{a.K + bh * a.N * a.d, s_q, s_u, a.G, a.d, a.scale_log2};
    for (int j = tid; j < ri.P; j += NT) atomicAdd(&sh[score_bin(rs.key(j))], 1u);
    __syncthreads();
    {
        const unsigned c[2] = {static_cast<unsigned>(ri.keff), static_cast<unsigned>(ri.keff)};
        buckets_at_counts<NT>(sh, c, s_warp, s_bin, s_below);
    }
    __syncthreads();
    const int b1 = s_bin[0], above = s_below[0];
    if (above < 0 || above >= ri.keff) return;  // cannot happen for a consistent histogram
    // better buckets go straight out; the threshold bucket's keys become the row's candidates
    for (int j = tid; j < ri.P; j += NT) {
        const uint32_t k = rs.key(j);
        const int bin = score_bin(k);
        if (bin < b1) {
            const int slot = atomicAdd(&s_ndef, 1);
            if (slot < above) out[slot] = j;
        } else if (bin == b1) {
            const int slot = atomicAdd(&s_ncand, 1);
            if (slot < a.cand_cap) gcand[slot] = composite(k, j);
        }
    }
    __syncthreads();
    const unsigned need = static_cast<unsigned>(ri.keff - above);
    const int ncand = s_ncand;
    if (ncand <= a.cand_cap) {
        const GlobalSource src{gcand, ncand};
        emit_at_least(src, radix_threshold(src, need, h, s_small), need, out + above, &s_count);
    } else {  // more ties in one bucket than the list holds: recompute them on every pass
        const RescoreSource src{rs, ri.P, b1};
        emit_at_least(src, radix_threshold(src, need, h, s_small), need, out + above, &s_count);
    }
}

cudaError_t launch_topk_bracket(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    const cudaError_t e =
        launch_pdl(topk_bracket_kernel, dim3(static_cast<unsigned>(p.rows_kv)), dim3(256), 0, st, a);
    trace_mark("topk_bracket", st);
    return e;
}

cudaError_t launch_topk_finalize(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    const cudaError_t e =
        launch_pdl(topk_finalize_kernel<512>, dim3(static_cast<unsigned>(p.rows_kv)), dim3(512), 0, st, a);
    trace_mark("topk_finalize", st);
    return e;
}

cudaError_t launch_topk_rows(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    const cudaError_t e =
        launch_pdl(topk_rows_kernel<512>, dim3(static_cast<unsigned>(p.rows_kv)), dim3(512), 0, st, a);
    trace_mark("topk_rows", st);
    return e;
}

cudaError_t launch_topk_hist(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    dim3 grid(p.topk_ctas, static_cast<unsigned>(p.rows_kv));
    const cudaError_t e = launch_pdl(topk_hist_kernel, grid, dim3(256), 0, st, a);
    trace_mark("topk_hist", st);
    return e;
}

cudaError_t launch_topk_select(const Plan& p, const TopkArgs& a, cudaStream_t st) {
    dim3 grid(p.topk_ctas, static_cast<unsigned>(p.rows_kv));
    const cudaError_t e = launch_pdl(topk_select_kernel, grid, dim3(256), 0, st, a);
    trace_mark("topk_select", st);
    return e;
}

}  // namespace hs2
