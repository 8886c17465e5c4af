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
__device__ __forceinline__ float2 warp_row_ml(const float2* __restrict__ part_ml, int S, int64_t rows, int64_t row) {
    const int lane = threadIdx.x & 31;
    float m = -INFINITY;
    for (int s = lane; s < S; s += 32) m = fmaxf(m, __ldcg(&part_ml[s * rows + row]).x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    if (m != -INFINITY)
        for (int s = lane; s < S; s += 32) {
            const float2 ml = __ldcg(&part_ml[s * rows + row]);
            if (ml.x != -INFINITY) l += fast_exp2(ml.x - m) * ml.y;
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    return make_float2(m, l);
}

// Base-2 LSE from (M, L); -inf for an empty row.
__device__ __forceinline__ float lse2_of(float2 ml) { return ml.y > 0.f ? ml.x + log2f(ml.y) : -INFINITY; }

// One warp merges one row: writes O (bf16, D values) and LSE (natural log).
// wbuf: this warp's shared scratch of at least S floats.
template <int D>
__device__ __forceinline__ void warp_combine_row(const float2* __restrict__ part_ml, const float* __restrict__ part_acc,
                                                 int S, int64_t rows, int64_t row, float* wbuf, uint16_t* O,
                                                 float* LSE) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const float2 ML = warp_row_ml(part_ml, S, rows, row);
    const float inv = ML.y > 0.f ? 1.f / ML.y : 0.f;
    for (int s = lane; s < S; s += 32) {
        const float2 ml = __ldcg(&part_ml[s * rows + row]);
        wbuf[s] = (ml.x == -INFINITY || ML.x == -INFINITY) ? 0.f : fast_exp2(ml.x - ML.x) * inv;
    }
    __syncwarp();
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    const float* src = part_acc + row * D + lane * PER;
#pragma unroll 8
    for (int s = 0; s < S; ++s) {
        const float wgt = wbuf[s];
        if constexpr (PER == 4) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(src + s * rows * D));
            acc[0] += wgt * x.x;
            acc[1] += wgt * x.y;
            acc[2] += wgt * x.z;
            acc[3] += wgt * x.w;
        } else {
            const float2 x = __ldcg(reinterpret_cast<const float2*>(src + s * rows * D));
            acc[0] += wgt * x.x;
            acc[1] += wgt * x.y;
        }
    }
    __syncwarp();
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

// NaN-propagating max (fmaxf drops NaN operands; a NaN score must stay NaN).
__device__ __forceinline__ float nan_max(float a, float b) { return (a > b || a != a) ? a : b; }

}  // namespace hs2
