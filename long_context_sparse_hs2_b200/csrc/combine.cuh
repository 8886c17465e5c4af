// Log-sum-exp merge of split-K partials (m, l, O) -- used inside the kernels that consume
// them (no separate combine launch on the decode path).
//
// A partial of one query-head row is (m, l, acc[D]) in base-2 units: m the max logit of the
// split, l = sum 2^(logit - m), acc = sum 2^(logit - m) v.  Merging S of them:
// M = max m_s, L = sum 2^(m_s - M) l_s, O = sum 2^(m_s - M) acc_s / L, LSE = (M + log2 L) ln 2
// -- exact in real arithmetic ("Simplified Sparse Attention via Gist Tokens", section 3.6,
// combine phase).  Every function reduces in one fixed order, so all CTAs that need the same
// row's LSE get bit-identical values.
#pragma once

#include "hs2_device.cuh"

namespace hs2 {

// Warp-cooperative (M, L) of one row over S splits; every lane returns the same values.
// Each partial is loaded once (up to 64 splits are held in registers).
__device__ __forceinline__ float2 warp_row_ml(const float2* __restrict__ part_ml, int S, int64_t rows, int64_t row) {
    const int lane = threadIdx.x & 31;
    const float2 none = make_float2(-INFINITY, 0.f);
    const float2 v0 = lane < S ? __ldcg(&part_ml[lane * rows + row]) : none;
    const float2 v1 = lane + 32 < S ? __ldcg(&part_ml[(lane + 32) * rows + row]) : none;
    float m = fmaxf(v0.x, v1.x);
    for (int s = lane + 64; s < S; s += 32) m = fmaxf(m, __ldcg(&part_ml[s * rows + row]).x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    if (m != -INFINITY) {
        if (v0.x != -INFINITY) l += fast_exp2(v0.x - m) * v0.y;
        if (v1.x != -INFINITY) l += fast_exp2(v1.x - m) * v1.y;
        for (int s = lane + 64; s < S; s += 32) {
            const float2 ml = __ldcg(&part_ml[s * rows + row]);
            if (ml.x != -INFINITY) l += fast_exp2(ml.x - m) * ml.y;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    return make_float2(m, l);
}

// Base-2 LSE from (M, L); -inf for an empty row.
__device__ __forceinline__ float lse2_of(float2 ml) { return ml.y > 0.f ? ml.x + log2f(ml.y) : -INFINITY; }

// Per-split merge weights 2^(m_s - M) / L of one row into wbuf[0..S) (shared memory), every
// partial (m, l) read once; returns (M, L).  Warp-cooperative.
__device__ __forceinline__ float2 warp_row_weights(const float2* __restrict__ part_ml, int S, int64_t rows, int64_t row,
                                                   float* wbuf) {
    const int lane = threadIdx.x & 31;
    const float2 ML = warp_row_ml(part_ml, S, rows, row);
    const float inv = ML.y > 0.f ? 1.f / ML.y : 0.f;
    for (int s = lane; s < S; s += 32) {
        const float2 ml = __ldcg(&part_ml[s * rows + row]);  // L2 hit: just read by warp_row_ml
        wbuf[s] = (ml.x == -INFINITY || ML.x == -INFINITY) ? 0.f : fast_exp2(ml.x - ML.x) * inv;
    }
    __syncwarp();
    return ML;
}

// acc[PER] += sum over splits s = s0, s0 + stride, ... < S of wbuf[s] * part_acc[s][row][lane's dims],
// 16 loads in flight per lane.
template <int D>
__device__ __forceinline__ void accumulate_splits(const float* __restrict__ part_acc, int S, int s0, int stride,
                                                  int64_t rows, int64_t row, const float* wbuf, float* acc) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const float* src = part_acc + row * D + lane * PER;
    for (int base = s0; base < S; base += 16 * stride) {
        float x[16][PER];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int s = base + u * stride;
            if (s < S) {
                if constexpr (PER == 4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(src + s * rows * D));
                    x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
                } else {
                    const float2 v = __ldcg(reinterpret_cast<const float2*>(src + s * rows * D));
                    x[u][0] = v.x; x[u][1] = v.y;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int s = base + u * stride;
            if (s < S) {
                const float wgt = wbuf[s];
#pragma unroll
                for (int e = 0; e < PER; ++e) acc[e] += wgt * x[u][e];
            }
        }
    }
}

template <int D>
__device__ __forceinline__ void store_row(const float* acc, float2 ML, int64_t row, uint16_t* O, float* LSE) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    uint32_t packed[PER / 2];
#pragma unroll
    for (int e = 0; e < PER / 2; ++e) packed[e] = pack_bf16x2(acc[2 * e], acc[2 * e + 1]);
    uint16_t* dst = O + row * D + lane * PER;
    if constexpr (PER == 4)
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    else
        *reinterpret_cast<uint32_t*>(dst) = packed[0];
    if (lane == 0) LSE[row] = lse2_of(ML) * kLn2;
}

// One warp merges one row: writes O (bf16, D values) and LSE (natural log).
// wbuf: this warp's shared scratch of at least S floats.
template <int D>
__device__ __forceinline__ void warp_combine_row(const float2* __restrict__ part_ml, const float* __restrict__ part_acc,
                                                 int S, int64_t rows, int64_t row, float* wbuf, uint16_t* O,
                                                 float* LSE) {
    const float2 ML = warp_row_weights(part_ml, S, rows, row, wbuf);
    float acc[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
    accumulate_splits<D>(part_acc, S, 0, 1, rows, row, wbuf, acc);
    store_row<D>(acc, ML, row, O, LSE);
}

// The whole CTA merges one row: every warp takes every nw-th split, then the warps' sums are
// added in shared memory.  red: blockDim/32 * D floats; wbuf: S floats.  Contains barriers:
// call from all threads.
template <int D>
__device__ __forceinline__ void block_combine_row(const float2* __restrict__ part_ml, const float* __restrict__ part_acc,
                                                  int S, int64_t rows, int64_t row, float* wbuf, float* red,
                                                  uint16_t* O, float* LSE) {
    constexpr int PER = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    float2 ML = make_float2(0.f, 0.f);
    if (warp == 0) ML = warp_row_weights(part_ml, S, rows, row, wbuf);
    __syncthreads();
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    accumulate_splits<D>(part_acc, S, warp, nw, rows, row, wbuf, acc);
#pragma unroll
    for (int e = 0; e < PER; ++e) red[warp * D + lane * PER + e] = acc[e];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            float t = 0.f;
            for (int w = 0; w < nw; ++w) t += red[w * D + lane * PER + e];
            acc[e] = t;
        }
        store_row<D>(acc, ML, row, O, LSE);
    }
    __syncthreads();
}

// Merge, for float4 columns col0, col0 + cstep, ... of nh rows (rows row0 + g * stride, D/4
// columns each), the S split partials with the per-split weights s_w[g * S + s] and (M, L)
// s_ml[g] already computed; writes bf16 O and (with a row's first column) the natural-log LSE.
// Up to U loads in flight per column.  No barriers.
template <int D, int U = 32>
__device__ __forceinline__ void combine_columns(const float* __restrict__ part_acc, int S, int64_t rows, int64_t row0,
                                                int64_t stride, int nh, const float* s_w, const float2* s_ml,
                                                uint16_t* O, float* LSE, int col0, int cstep) {
    constexpr int C4 = D / 4;  // float4 columns per row
    for (int col = col0; col < nh * C4; col += cstep) {
        const int g = col / C4, c = col % C4;
        const int64_t row = row0 + g * stride;
        const float* src = part_acc + row * D + c * 4;
        const float* w = s_w + g * S;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int base = 0; base < S; base += U) {
            float4 x[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + u < S) x[u] = __ldcg(reinterpret_cast<const float4*>(src + (base + u) * rows * D));
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + u < S) {
                    const float wt = w[base + u];
                    acc.x += wt * x[u].x;
                    acc.y += wt * x[u].y;
                    acc.z += wt * x[u].z;
                    acc.w += wt * x[u].w;
                }
        }
        *reinterpret_cast<uint2*>(O + row * D + c * 4) =
            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        if (c == 0) LSE[row] = lse2_of(s_ml[g]) * kLn2;
    }
}

// The whole CTA merges the split partials of nh rows at once (the G query heads of one
// selection row: rows row0 + g * stride).  Warps first turn each row's (m, l) into per-split
// weights (s_w[g * S + s]); then every thread owns float4 columns (row, 4 dims) and sums its
// splits with up to U loads in flight.  s_w: nh * S floats, s_ml: nh float2.  Call from all
// threads (contains barriers).
template <int D, int U = 32>
__device__ __forceinline__ void block_combine_rows(const float2* __restrict__ part_ml,
                                                   const float* __restrict__ part_acc, int S, int64_t rows,
                                                   int64_t row0, int64_t stride, int nh, float* s_w, float2* s_ml,
                                                   uint16_t* O, float* LSE) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int g = warp; g < nh; g += nw) {
        const float2 ML = warp_row_weights(part_ml, S, rows, row0 + g * stride, s_w + g * S);
        if (lane == 0) s_ml[g] = ML;
    }
    __syncthreads();
    combine_columns<D, U>(part_acc, S, rows, row0, stride, nh, s_w, s_ml, O, LSE, threadIdx.x, blockDim.x);
    __syncthreads();
}

// NaN-propagating max (fmaxf drops NaN operands; a NaN score must stay NaN).
__device__ __forceinline__ float nan_max(float a, float b) { return (a > b || a != a) ? a : b; }

}  // namespace hs2
