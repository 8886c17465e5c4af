// Selection score from the full layer's kept logits, fused with the first top-k pass and
// with the full-attention split combine (sm_100a).
//
// The score of pool key j for selection row (b, kv head h, t) is the max over the G query
// heads of h of the log-softmax probability, s_j = max_g (l_gj - LSE_g) -- the full
// layer's own logits and LSE, which is how its selection feeds the sparse layers that
// reuse it (KV Reuse: "HySparse2 od Xiaomi zkracuje zpracovani dlouheho kontextu", section
// "Proc neni nutne znovu zpracovat cely dlouhy vstup", third paragraph).  The pages leave
// the score open; this library fixes it to the GQA-max log-softmax.
//
// Grid (x, y = selection row):
//   x < nscore: one kTopkChunk-key chunk of the row's pool.  The CTA merges the G heads' LSE from
//     the split partials, forms every key's score (base-2 units, NaN-propagating max), writes
//     the order-preserving key, and bins it in a shared-memory histogram that is added to
//     the row's global histogram; the row's last CTA finds the threshold bucket.
//   x == nscore: merges the split partials of the row's G query heads into O_full and
//     LSE_full (the full-attention combine, off the critical path of the scoring CTAs).
#include "combine.cuh"
#include "topk_common.cuh"

namespace hs2 {

template <int G, int D>
__global__ void __launch_bounds__(256) score_hist_kernel(const ScoreArgs a) {
    constexpr int kScratch = kHistBins > 16 * 256 + 64 ? kHistBins : 16 * 256 + 64;
    __shared__ unsigned sh[kScratch];  // histogram, or the combine CTA's weights (G * S1 <= 4096)
    __shared__ unsigned s_warp[32];
    __shared__ int s_last;
    __shared__ float s_lse2[G];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.y;  // (b*Hkv + h)*T + t
    const int t = static_cast<int>(row % a.T);
    const int bh = static_cast<int>(row / a.T);
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const int64_t rows_q = static_cast<int64_t>(a.B) * a.Hq * a.T;
    auto row_q = [&](int g) -> int64_t { return (static_cast<int64_t>(b) * a.Hq + h * G + g) * a.T + t; };
    const int nscore = (a.N + kTopkChunk - 1) / kTopkChunk;
    pdl_trigger();

    if (static_cast<int>(blockIdx.x) >= nscore) {  // the full-attention combine of this row's G heads
        pdl_wait();
        float* s_w = reinterpret_cast<float*>(sh);
        float2* s_ml = reinterpret_cast<float2*>(sh + 16 * 256);
        block_combine_rows<D, 8>(a.part_ml, a.part_acc, a.S1, rows_q, row_q(0), a.T, G, s_w, s_ml, a.O, a.LSE);
        return;
    }

    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
    // Every CTA waits for the full sweep (partials, kept logits, cleared histograms) before it
    // can finish, so this kernel's completion implies the sweep's.
    pdl_wait();
    const RowInfo ri = make_row_info(a.pos, row, a.Hkv, a.T, a.N, a.k, a.W);
    if (ri.keff == 0 || ri.keff == ri.P) return;  // nothing to rank: the selection kernel takes all or none
    const int participants = (ri.P + kTopkChunk - 1) / kTopkChunk;
    const int chunk = blockIdx.x;
    if (chunk >= participants) return;
    for (int g = warp; g < G; g += 8) {
        const float2 ML = warp_row_ml(a.part_ml, a.S1, rows_q, row_q(g));
        if (lane == 0) s_lse2[g] = lse2_of(ML);
    }
    __syncthreads();
    float lse[G];
#pragma unroll
    for (int g = 0; g < G; ++g) lse[g] = s_lse2[g];

    const int j0 = chunk * kTopkChunk, j1 = min(j0 + kTopkChunk, ri.P);
    const float* lg = a.logits + row * static_cast<int64_t>(a.N) * G;
    uint32_t* keys = a.keys + row * a.kstride;
    bool nonfinite = false;
    constexpr int U = G >= 16 ? 4 : 8;  // keys in flight per thread
    for (int base = j0 + threadIdx.x; base < j1; base += U * 256) {
        float v[U][G];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = base + u * 256;
            if (j < j1) {
                const float* src = lg + static_cast<int64_t>(j) * G;
                if constexpr (G % 4 == 0) {
#pragma unroll
                    for (int q = 0; q < G / 4; ++q) {
                        const float4 f = __ldcs(reinterpret_cast<const float4*>(src) + q);
                        v[u][4 * q] = f.x;
                        v[u][4 * q + 1] = f.y;
                        v[u][4 * q + 2] = f.z;
                        v[u][4 * q + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < G; ++q) v[u][q] = __ldcs(src + q);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = base + u * 256;
            if (j < j1) {
                float s = v[u][0] - lse[0];
#pragma unroll
                for (int g = 1; g < G; ++g) s = nan_max(s, v[u][g] - lse[g]);
                nonfinite |= (s != s);
                const uint32_t key = score_key(s);
                keys[j] = key;
                atomicAdd(&sh[score_bin(key)], 1u);
            }
        }
    }
    if (__syncthreads_or(nonfinite) && threadIdx.x == 0) set_status(a.status, HS2_DEV_NONFINITE);
    hist_flush_and_threshold(sh, a.hist + row * kHistBins, a.meta + row * kMetaInts, participants, ri.keff, s_warp,
                             &s_last);
}

cudaError_t launch_score_hist(const Plan& p, const ScoreArgs& a, cudaStream_t st) {
    const int nscore = (p.N + kTopkChunk - 1) / kTopkChunk;
    const int ncomb = 1;
    dim3 grid(nscore + ncomb, static_cast<unsigned>(p.rows_kv));
#define HS2_SH(G_)                                                                                          \
    case G_:                                                                                                \
        e = p.d == 128 ? launch_pdl(score_hist_kernel<G_, 128>, grid, dim3(256), 0, st, a)                  \
                       : launch_pdl(score_hist_kernel<G_, 64>, grid, dim3(256), 0, st, a);                  \
        break;
    cudaError_t e = cudaErrorInvalidValue;
    switch (p.G) {
        HS2_SH(1) HS2_SH(2) HS2_SH(4) HS2_SH(8) HS2_SH(16)
        default: return cudaErrorInvalidValue;
    }
#undef HS2_SH
    trace_mark("score_hist", st);
    return e;
}

}  // namespace hs2
