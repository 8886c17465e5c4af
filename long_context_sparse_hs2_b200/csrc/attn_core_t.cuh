// Transposed warp attention for a row block of at most 8 query-head rows (decode, T * G <= 8),
// over a bf16 or an FP8 E4M3 cache.
//
// With keys as the MMA's M dimension and the query rows as N (m16n8k16), S^T = K Q^T takes one
// MMA per 16 keys x 16 dims where the query-rows-as-M form takes two (half of its 16 rows are
// padding), and O^T = V^T P^T one MMA per 16 keys x 16 dims of output: the MMAs, the
// exponentials and the O registers halve.
//   S^T: A = the K tile read with ldmatrix (bf16: a lane holds dims 2c, 2c+1 and 2c+8, 2c+9 of
//        keys g and g+8; E4M3: byte pairs, a lane holds dims 4c .. 4c+3 and the reduction order
//        is permuted to match, as in the query-rows-as-M form), B = Q^T (E4M3: f16, each query
//        row scaled by a power of two into f16 range).  Lane (g, c) gets the scores of keys g
//        and g+8 for query rows 2c and 2c+1.
//   softmax: online, per query row (a column here): maxima and sums over the key rows of the
//        fragment and the 8 lanes of a column.
//   O^T: A = V^T (ldmatrix.trans: bf16 gives dims g, g+8 of a 16-dim chunk for keys 2c, 2c+1;
//        E4M3 byte pairs give dims 2g, 2g+1, split by a byte permute, so the MMA's rows are the
//        even dims then the odd dims of the chunk), B = P^T (the score fragment packed to
//        bf16 / f16 and transposed in registers with movmatrix).
// The per-warp state is merged across warps through the same shared-memory layout as the
// query-rows-as-M form (merge_states in attn_core.cuh).
#pragma once

#include "attn_core.cuh"

namespace hs2 {

// Q^T B fragments for query rows 0..7 of the row block (lane (g, c) loads row g) and, for an
// E4M3 cache, the power-of-two scales of the lane's two score columns (rows 2c, 2c+1).
template <int D, bool FP8>
struct QTileT {
    uint32_t b[D / 16][2];
    float col_scale[2];

    __device__ __forceinline__ void load(const uint16_t* __restrict__ Q, int64_t off) {
        const int lane = threadIdx.x & 31, c = lane & 3;
        if constexpr (!FP8) {
#pragma unroll
            for (int kc = 0; kc < D / 16; ++kc) {  // k = 2c, 2c+1 and 2c+8, 2c+9 of chunk kc
                b[kc][0] = off >= 0 ? *reinterpret_cast<const uint32_t*>(Q + off + kc * 16 + 2 * c) : 0u;
                b[kc][1] = off >= 0 ? *reinterpret_cast<const uint32_t*>(Q + off + kc * 16 + 2 * c + 8) : 0u;
            }
            col_scale[0] = col_scale[1] = 1.f;
            return;
        }
        float x[D / 4];
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
            uint2 v = make_uint2(0u, 0u);
            if (off >= 0) v = *reinterpret_cast<const uint2*>(Q + off + kc * 16 + 4 * c);
            x[4 * kc + 0] = __uint_as_float(v.x << 16);
            x[4 * kc + 1] = __uint_as_float(v.x & 0xFFFF0000u);
            x[4 * kc + 2] = __uint_as_float(v.y << 16);
            x[4 * kc + 3] = __uint_as_float(v.y & 0xFFFF0000u);
        }
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < D / 4; ++i) mx = fmaxf(mx, fabsf(x[i]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // 2^e <= mx < 2^(e+1)  ->  scale by 2^(14 - e): the row's largest |q| in [2^14, 2^15)
        const int e = (mx > 0.f && mx < INFINITY) ? ilogbf(mx) : 14;
        const int sh = 14 - e;
        const float rs = exp2f(static_cast<float>(-sh));
#pragma unroll
        for (int i = 0; i < D / 4; ++i) x[i] = ldexpf(x[i], sh);
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
            b[kc][0] = pack_f16x2(x[4 * kc + 0], x[4 * kc + 1]);  // MMA k = 2c, 2c+1  <- dims 4c, 4c+1
            b[kc][1] = pack_f16x2(x[4 * kc + 2], x[4 * kc + 3]);  // MMA k = 2c+8, 2c+9 <- dims 4c+2, 4c+3
        }
        // row r's scale lives in the lanes 4r .. 4r+3
        col_scale[0] = __shfl_sync(0xffffffffu, rs, 8 * c);
        col_scale[1] = __shfl_sync(0xffffffffu, rs, 8 * c + 4);
    }
};

// S^T for keys key0 .. key0+15 of the K tile at smem address kbase: s[0] = (key g, row 2c),
// s[1] = (key g, row 2c+1), s[2] = (key g+8, row 2c), s[3] = (key g+8, row 2c+1).
template <int D, bool FP8>
__device__ __forceinline__ void qk_t(const QTileT<D, FP8>& q, uint32_t kbase, int key0, float (&s)[4]) {
    const int lane = threadIdx.x & 31;
    const int mi = lane >> 3;
    s[0] = s[1] = s[2] = s[3] = 0.f;
    const int row = key0 + (lane & 7) + ((mi & 1) << 3);
    if constexpr (!FP8) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];  // (keys 0-7, dims 0-7), (8-15, 0-7), (0-7, 8-15), (8-15, 8-15) of chunk kk
            ldsm_x4(kbase + tile_chunk_offset(row, 2 * kk + (mi >> 1)), a[0], a[1], a[2], a[3]);
            mma_bf16(s, a, q.b[kk][0], q.b[kk][1]);
        }
        return;
    }
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
        uint32_t r0, r1, r2, r3;  // (keys 0-7, chunk 2kk), (8-15, 2kk), (0-7, 2kk+1), (8-15, 2kk+1)
        ldsm_x4(kbase + fp8_chunk_offset<D>(row, 2 * kk + (mi >> 1)), r0, r1, r2, r3);
        const uint32_t a0[4] = {e4m3x2_to_f16x2(r0), e4m3x2_to_f16x2(r1), e4m3x2_to_f16x2(r0 >> 16),
                                e4m3x2_to_f16x2(r1 >> 16)};
        mma_f16(s, a0, q.b[2 * kk][0], q.b[2 * kk][1]);
        const uint32_t a1[4] = {e4m3x2_to_f16x2(r2), e4m3x2_to_f16x2(r3), e4m3x2_to_f16x2(r2 >> 16),
                                e4m3x2_to_f16x2(r3 >> 16)};
        mma_f16(s, a1, q.b[2 * kk + 1][0], q.b[2 * kk + 1][1]);
    }
}

// Running softmax of the lane's two query rows (columns 2c, 2c+1) and O^T: o[ch][0], o[ch][1]
// hold (rows 2c, 2c+1) dim odim(ch, 0) and o[ch][2], o[ch][3] dim odim(ch, 1), with
// odim = 16 ch + g + 8 i (bf16) or 16 ch + 2g + i (E4M3).
template <int D, bool FP8>
struct OnlineSoftmaxT {
    __device__ __forceinline__ static int odim(int ch, int i) {
        const int g = (threadIdx.x & 31) >> 2;
        return FP8 ? 16 * ch + 2 * g + i : 16 * ch + g + 8 * i;
    }
    float o[D / 16][4];
    float m[2];  // running max (base-2 logits) of rows 2c, 2c+1
    float l[2];  // this lane's partial sum (summed over the column's 8 lanes at the end)

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int ch = 0; ch < D / 16; ++ch) o[ch][0] = o[ch][1] = o[ch][2] = o[ch][3] = 0.f;
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
    }

    // Fold in 16 keys' base-2 logits s (masked with -inf); V codes from the tile at vbase.  The
    // reference max is raised lazily, as in OnlineSoftmax (exact: l and O share it).
    __device__ __forceinline__ void update(float (&s)[4], uint32_t vbase, int key0) {
        constexpr float kLazyRescale = 8.f;
        const int lane = threadIdx.x & 31;
        float corr[2], p[4];
        bool bumped = false;
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
            float mx = fmaxf(s[ci], s[2 + ci]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const bool bump = mx > m[ci] + kLazyRescale;  // false while both are -inf
            const float m_new = bump ? mx : m[ci];
            const float base = (m_new == -INFINITY) ? 0.f : m_new;
            corr[ci] = bump ? fast_exp2(m[ci] - base) : 1.f;  // 0 when m was -inf
            bumped |= bump;
            p[ci] = fast_exp2(s[ci] - base);
            p[2 + ci] = fast_exp2(s[2 + ci] - base);
            l[ci] = l[ci] * corr[ci] + p[ci] + p[2 + ci];
            m[ci] = m_new;
        }
        if (__any_sync(0xffffffffu, bumped)) {
#pragma unroll
            for (int ch = 0; ch < D / 16; ++ch) {
                o[ch][0] *= corr[0];
                o[ch][1] *= corr[1];
                o[ch][2] *= corr[0];
                o[ch][3] *= corr[1];
            }
        }
        // P^T fragments: (keys 2c, 2c+1 | 2c+8, 2c+9; query row g)
        const int mi = lane >> 3;
        if constexpr (!FP8) {
            const uint32_t b0 = movmatrix_t(pack_bf16x2(p[0], p[1]));
            const uint32_t b1 = movmatrix_t(pack_bf16x2(p[2], p[3]));
            // V^T fragments: (keys 0-7, dims 0-7), (0-7, 8-15), (8-15, 0-7), (8-15, 8-15) of a chunk,
            // transposed: lane (g, c) gets dim g (or g + 8) of keys 2c, 2c+1 (or 2c+8, 2c+9)
            const int row = key0 + (lane & 7) + ((mi >> 1) << 3);
#pragma unroll
            for (int ch = 0; ch < D / 16; ++ch) {
                uint32_t a[4];
                ldsm_x4_t(vbase + tile_chunk_offset(row, 2 * ch + (mi & 1)), a[0], a[1], a[2], a[3]);
                mma_bf16(o[ch], a, b0, b1);
            }
        } else {
            const uint32_t b0 = movmatrix_t(pack_f16x2(p[0], p[1]));
            const uint32_t b1 = movmatrix_t(pack_f16x2(p[2], p[3]));
            const int row = key0 + (lane & 7) + ((mi & 1) << 3);
#pragma unroll
            for (int dc2 = 0; dc2 < D / 32; ++dc2) {
                uint32_t r0, r1, r2, r3;  // (keys 0-7, chunk 2 dc2), (8-15, 2 dc2), (0-7, +1), (8-15, +1)
                ldsm_x4_t(vbase + fp8_chunk_offset<D>(row, 2 * dc2 + (mi >> 1)), r0, r1, r2, r3);
                const uint32_t p0 = __byte_perm(r0, 0u, 0x3120), p1 = __byte_perm(r1, 0u, 0x3120);
                const uint32_t p2 = __byte_perm(r2, 0u, 0x3120), p3 = __byte_perm(r3, 0u, 0x3120);
                const uint32_t a0[4] = {e4m3x2_to_f16x2(p0), e4m3x2_to_f16x2(p0 >> 16), e4m3x2_to_f16x2(p1),
                                        e4m3x2_to_f16x2(p1 >> 16)};
                mma_f16(o[2 * dc2], a0, b0, b1);
                const uint32_t a1[4] = {e4m3x2_to_f16x2(p2), e4m3x2_to_f16x2(p2 >> 16), e4m3x2_to_f16x2(p3),
                                        e4m3x2_to_f16x2(p3 >> 16)};
                mma_f16(o[2 * dc2 + 1], a1, b0, b1);
            }
        }
    }

    // Sum l over the 8 lanes of each column.
    __device__ __forceinline__ void finish_rows() {
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
            l[ci] += __shfl_xor_sync(0xffffffffu, l[ci], 4);
            l[ci] += __shfl_xor_sync(0xffffffffu, l[ci], 8);
            l[ci] += __shfl_xor_sync(0xffffffffu, l[ci], 16);
        }
    }
};

// Park this warp's state in shared-memory slot ks in the layout merge_states reads (query rows
// 0..7; O times vscale, natural dim order).
template <int D, int NKS, bool FP8>
__device__ __forceinline__ void stash_state_t(const OnlineSoftmaxT<D, FP8>& st, int ks, float* red, float vscale) {
    constexpr int LD = merge_ld<D>();
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    float* red_ml = red + NKS * 16 * LD;
#pragma unroll
    for (int ci = 0; ci < 2; ++ci) {
        const int r = 2 * c + ci;
        float* dst = red + (ks * 16 + r) * LD;
#pragma unroll
        for (int ch = 0; ch < D / 16; ++ch) {
            dst[OnlineSoftmaxT<D, FP8>::odim(ch, 0)] = st.o[ch][ci] * vscale;
            dst[OnlineSoftmaxT<D, FP8>::odim(ch, 1)] = st.o[ch][2 + ci] * vscale;
        }
        if (g == 0) {
            red_ml[(ks * 16 + r) * 2] = st.m[ci];
            red_ml[(ks * 16 + r) * 2 + 1] = st.l[ci];
        }
    }
}

}  // namespace hs2
