// Warp-level attention on one 16-row query tile against a shared-memory K/V tile.
//
// The query rows of one kv head (its G query heads, for one or more queries) form
// 16-row tiles.  A warp owns one such tile and a slice of KW keys of the current
// 64-key K/V tile, computes S = Q K^T with bf16 mma.sync (fp32 accumulate), applies
// the causal / validity mask, and folds the slice into a running online softmax
// (m, l, O) in base-2 units: logits are pre-multiplied by d^-1/2 * log2(e) so every
// exponential is one ex2.  The split-K partial results (m, l, O) merge exactly with
// the log-sum-exp correction, as in the split-K flash-decode of "Simplified Sparse
// Attention via Gist Tokens", section 3.6 ("three-kernel split-K sparse flash-decode").
//
// Register fragments follow the m16n8k16 layout: lane = 4*g + c holds rows g and g+8
// and, per 8-key n-tile, columns 2c and 2c+1.
#pragma once

#include <type_traits>

#include "hs2_device.cuh"

namespace hs2 {

// A fragments of a 16 x D bf16 query tile (row-major), kept in registers for the whole sweep.
template <int D>
struct QTile {
    uint32_t a[D / 16][4];

    // rows: global element offsets of tile rows g and g+8 for this lane (-1 = padding row)
    __device__ __forceinline__ void load(const uint16_t* __restrict__ Q, int64_t off_lo, int64_t off_hi) {
        const int c = threadIdx.x & 3;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int col = kk * 16 + 2 * c;
            a[kk][0] = off_lo >= 0 ? *reinterpret_cast<const uint32_t*>(Q + off_lo + col) : 0u;
            a[kk][1] = off_hi >= 0 ? *reinterpret_cast<const uint32_t*>(Q + off_hi + col) : 0u;
            a[kk][2] = off_lo >= 0 ? *reinterpret_cast<const uint32_t*>(Q + off_lo + col + 8) : 0u;
            a[kk][3] = off_hi >= 0 ? *reinterpret_cast<const uint32_t*>(Q + off_hi + col + 8) : 0u;
        }
    }
};

// The query tile for an FP8 cache: f16 A fragments.  The K tile is read with ldmatrix as b16
// pairs, so a lane gets four consecutive E4M3 dims 4c..4c+3 of a key per 16-dim chunk; the
// reduction order inside a chunk is permuted to match (MMA column 2c <-> dim 4c, 2c+1 <-> 4c+1,
// 2c+8 <-> 4c+2, 2c+9 <-> 4c+3), which leaves the dot product unchanged.  Each row is scaled by a
// power of two 2^a (exact) that brings its largest |q| into [2^14, 2^15), so bf16 queries fit the
// f16 range; row_scale[i] = 2^-a undoes it on the logits.
template <int D>
struct QTileF16 {
    uint32_t a[D / 16][4];
    float row_scale[2];

    __device__ __forceinline__ void load(const uint16_t* __restrict__ Q, int64_t off_lo, int64_t off_hi) {
        const int c = threadIdx.x & 3;
        float x[2][D / 4];
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
            const int64_t off = ri == 0 ? off_lo : off_hi;
#pragma unroll
            for (int kc = 0; kc < D / 16; ++kc) {
                uint2 v = make_uint2(0u, 0u);
                if (off >= 0) v = *reinterpret_cast<const uint2*>(Q + off + kc * 16 + 4 * c);
                x[ri][4 * kc + 0] = __uint_as_float(v.x << 16);
                x[ri][4 * kc + 1] = __uint_as_float(v.x & 0xFFFF0000u);
                x[ri][4 * kc + 2] = __uint_as_float(v.y << 16);
                x[ri][4 * kc + 3] = __uint_as_float(v.y & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
            float mx = 0.f;
#pragma unroll
            for (int i = 0; i < D / 4; ++i) mx = fmaxf(mx, fabsf(x[ri][i]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            // 2^e <= mx < 2^(e+1)  ->  scale by 2^(14 - e)
            const int e = (mx > 0.f && mx < INFINITY) ? ilogbf(mx) : 14;
            const int sh = 14 - e;
            row_scale[ri] = exp2f(static_cast<float>(-sh));
#pragma unroll
            for (int i = 0; i < D / 4; ++i) x[ri][i] = ldexpf(x[ri][i], sh);
        }
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
            a[kc][0] = pack_f16x2(x[0][4 * kc + 0], x[0][4 * kc + 1]);
            a[kc][1] = pack_f16x2(x[1][4 * kc + 0], x[1][4 * kc + 1]);
            a[kc][2] = pack_f16x2(x[0][4 * kc + 2], x[0][4 * kc + 3]);
            a[kc][3] = pack_f16x2(x[1][4 * kc + 2], x[1][4 * kc + 3]);
        }
    }
};

// S[16 x KW] = Q[16 x D] * K^T for an FP8 E4M3 K tile (codes, not yet scaled): ldmatrix reads
// four 8-key x 16-dim blocks, each lane's 4 codes become two f16x2 B fragments.
template <int D, int KW>
__device__ __forceinline__ void qk_tile_fp8(const QTileF16<D>& q, uint32_t kbase, int key0, float (&s)[KW / 8][4]) {
    const int lane = threadIdx.x & 31;
    const int mi = lane >> 3;
#pragma unroll
    for (int n = 0; n < KW / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kg = 0; kg < KW / 16; ++kg) {
        const int row = key0 + kg * 16 + (lane & 7) + ((mi >> 1) << 3);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
            uint32_t r0, r1, r2, r3;
            ldsm_x4(kbase + fp8_chunk_offset<D>(row, 2 * kk + (mi & 1)), r0, r1, r2, r3);
            mma_f16(s[2 * kg], q.a[2 * kk], e4m3x2_to_f16x2(r0), e4m3x2_to_f16x2(r0 >> 16));
            mma_f16(s[2 * kg], q.a[2 * kk + 1], e4m3x2_to_f16x2(r1), e4m3x2_to_f16x2(r1 >> 16));
            mma_f16(s[2 * kg + 1], q.a[2 * kk], e4m3x2_to_f16x2(r2), e4m3x2_to_f16x2(r2 >> 16));
            mma_f16(s[2 * kg + 1], q.a[2 * kk + 1], e4m3x2_to_f16x2(r3), e4m3x2_to_f16x2(r3 >> 16));
        }
    }
}

// Query tile and QK^T of the cache's element type.
template <int D, bool FP8>
using QTileOf = typename std::conditional<FP8, QTileF16<D>, QTile<D>>::type;

template <int D, int KW, bool FP8>
__device__ __forceinline__ void qk_any(const QTileOf<D, FP8>& q, uint32_t kbase, int key0, float (&s)[KW / 8][4]);

// S[16 x KW] = Q[16 x D] * K[key0 .. key0+KW)^T, K read from a swizzled tile at smem address kbase.
template <int D, int KW>
__device__ __forceinline__ void qk_tile(const QTile<D>& q, uint32_t kbase, int key0, float (&s)[KW / 8][4]) {
    const int lane = threadIdx.x & 31;
    const int mi = lane >> 3;
#pragma unroll
    for (int n = 0; n < KW / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kg = 0; kg < KW / 16; ++kg) {
        const int row = key0 + kg * 16 + (lane & 7) + ((mi >> 1) << 3);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + tile_chunk_offset(row, 2 * kk + (mi & 1)), b0, b1, b2, b3);
            mma_bf16(s[2 * kg], q.a[kk], b0, b1);
            mma_bf16(s[2 * kg + 1], q.a[kk], b2, b3);
        }
    }
}

template <int D, int KW, bool FP8>
__device__ __forceinline__ void qk_any(const QTileOf<D, FP8>& q, uint32_t kbase, int key0, float (&s)[KW / 8][4]) {
    if constexpr (FP8)
        qk_tile_fp8<D, KW>(q, kbase, key0, s);
    else
        qk_tile<D, KW>(q, kbase, key0, s);
}

// Logit multiplier of tile rows g (i = 0) and g + 8 (i = 1): d^-1/2 log2(e), times the K scale
// and the query's power-of-two scale for an FP8 cache.
template <int D, bool FP8>
__device__ __forceinline__ float logit_factor(const QTileOf<D, FP8>& q, int i, float scale_log2, float k_scale) {
    if constexpr (FP8)
        return scale_log2 * k_scale * q.row_scale[i];
    else
        return scale_log2;
}

// Output dims held by accumulator o[n][e] (e = 0, 1 for row g; 2, 3 for row g + 8) of this
// lane, as the first of two adjacent dims stored together: bf16 V gives dims 8n + 2c, +1 in
// o[n][e], o[n][e+1]; FP8 V (see OnlineSoftmax::update) gives dims 16(n/2) + 4c + 2e + {0, 1}
// in o[n][e] (n even) and o[n+1][e].  PairOut hides the difference for the stores.
template <int D, bool FP8>
struct PairOut {
    // visits (dim, value of dim, value of dim + 1) for the lane's values of row ri
    template <class F>
    __device__ __forceinline__ static void each(const float (&o)[D / 8][4], int ri, F f) {
        const int c = threadIdx.x & 3;
        if constexpr (FP8) {
#pragma unroll
            for (int dc = 0; dc < D / 16; ++dc)
#pragma unroll
                for (int e = 0; e < 2; ++e) f(16 * dc + 4 * c + 2 * e, o[2 * dc][2 * ri + e], o[2 * dc + 1][2 * ri + e]);
        } else {
#pragma unroll
            for (int n = 0; n < D / 8; ++n) f(n * 8 + 2 * c, o[n][2 * ri], o[n][2 * ri + 1]);
        }
    }
};

// Running softmax state of one warp's 16-row tile.
template <int D, bool FP8 = false>
struct OnlineSoftmax {
    float o[D / 8][4];
    float m[2];  // running max (base-2 logits) of rows g, g+8
    float l[2];  // this lane's partial sum of 2^(logit - m) (summed over the quad at the end)

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
    }

    // Fold in a slice of base-2 logits s (already masked with -inf); V from the swizzled tile at vbase.
    // The reference max m is raised only when the slice's max exceeds it by more than
    // kLazyRescale (base 2): exponentials stay <= 2^kLazyRescale, and the O rescale (D/4
    // multiplies per lane) is skipped by the whole warp unless some row raised its max.  Exact:
    // l and O always share the same reference m.
    template <int KW>
    __device__ __forceinline__ void update(float (&s)[KW / 8][4], uint32_t vbase, int key0) {
        constexpr float kLazyRescale = 8.f;
        const int lane = threadIdx.x & 31;
        float corr[2];
        bool bumped = false;
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
            float mx = -INFINITY;
#pragma unroll
            for (int n = 0; n < KW / 8; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * ri], s[n][2 * ri + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const bool bump = mx > m[ri] + kLazyRescale;  // false while both are -inf
            const float m_new = bump ? mx : m[ri];
            const float base = (m_new == -INFINITY) ? 0.f : m_new;
            corr[ri] = bump ? fast_exp2(m[ri] - base) : 1.f;  // 0 when m was -inf
            bumped |= bump;
            float sum = 0.f;
#pragma unroll
            for (int n = 0; n < KW / 8; ++n) {
                s[n][2 * ri] = fast_exp2(s[n][2 * ri] - base);
                s[n][2 * ri + 1] = fast_exp2(s[n][2 * ri + 1] - base);
                sum += s[n][2 * ri] + s[n][2 * ri + 1];
            }
            l[ri] = l[ri] * corr[ri] + sum;
            m[ri] = m_new;
        }
        if (__any_sync(0xffffffffu, bumped)) {
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                o[n][0] *= corr[0];
                o[n][1] *= corr[0];
                o[n][2] *= corr[1];
                o[n][3] *= corr[1];
            }
        }
        // O += P V
        const int mi = lane >> 3;
#pragma unroll
        for (int kg = 0; kg < KW / 16; ++kg) {
            const int row = key0 + kg * 16 + (lane & 7) + ((mi & 1) << 3);
            if constexpr (FP8) {
                // P in f16; V codes read transposed as b16 pairs: a lane gets, for keys 2c and 2c+1,
                // the codes of dims 2g and 2g+1; a byte permute splits them into the B fragment of
                // the even dim and that of the odd dim, so each 16-dim chunk takes two MMAs (even
                // dims into o[2 dc], odd dims into o[2 dc + 1]).
                uint32_t a[4];
                a[0] = pack_f16x2(s[2 * kg][0], s[2 * kg][1]);
                a[1] = pack_f16x2(s[2 * kg][2], s[2 * kg][3]);
                a[2] = pack_f16x2(s[2 * kg + 1][0], s[2 * kg + 1][1]);
                a[3] = pack_f16x2(s[2 * kg + 1][2], s[2 * kg + 1][3]);
#pragma unroll
                for (int dc2 = 0; dc2 < D / 32; ++dc2) {
                    uint32_t r0, r1, r2, r3;  // (keys 0-7, chunk 2 dc2), (8-15, 2 dc2), (0-7, +1), (8-15, +1)
                    ldsm_x4_t(vbase + fp8_chunk_offset<D>(row, 2 * dc2 + (mi >> 1)), r0, r1, r2, r3);
                    const uint32_t p0 = __byte_perm(r0, 0u, 0x3120), p1 = __byte_perm(r1, 0u, 0x3120);
                    const uint32_t p2 = __byte_perm(r2, 0u, 0x3120), p3 = __byte_perm(r3, 0u, 0x3120);
                    const int dc = 2 * dc2;
                    mma_f16(o[2 * dc], a, e4m3x2_to_f16x2(p0), e4m3x2_to_f16x2(p1));
                    mma_f16(o[2 * dc + 1], a, e4m3x2_to_f16x2(p0 >> 16), e4m3x2_to_f16x2(p1 >> 16));
                    mma_f16(o[2 * dc + 2], a, e4m3x2_to_f16x2(p2), e4m3x2_to_f16x2(p3));
                    mma_f16(o[2 * dc + 3], a, e4m3x2_to_f16x2(p2 >> 16), e4m3x2_to_f16x2(p3 >> 16));
                }
            } else {
                uint32_t a[4];
                a[0] = pack_bf16x2(s[2 * kg][0], s[2 * kg][1]);
                a[1] = pack_bf16x2(s[2 * kg][2], s[2 * kg][3]);
                a[2] = pack_bf16x2(s[2 * kg + 1][0], s[2 * kg + 1][1]);
                a[3] = pack_bf16x2(s[2 * kg + 1][2], s[2 * kg + 1][3]);
#pragma unroll
                for (int dn = 0; dn < D / 16; ++dn) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vbase + tile_chunk_offset(row, 2 * dn + (mi >> 1)), b0, b1, b2, b3);
                    mma_bf16(o[2 * dn], a, b0, b1);
                    mma_bf16(o[2 * dn + 1], a, b2, b3);
                }
            }
        }
    }

    // Sum l over the 4 lanes of each row.
    __device__ __forceinline__ void finish_rows() {
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
            l[ri] += __shfl_xor_sync(0xffffffffu, l[ri], 1);
            l[ri] += __shfl_xor_sync(0xffffffffu, l[ri], 2);
        }
    }
};

// Split-K partial of one row: (m, l) in base-2 units and the unnormalised O.
struct PartialRef {
    float2* ml;   // [rows] (m, l)
    float* acc;   // [rows][D]
};

// Write a warp's tile straight to the partial buffers (one warp per tile, no merge).
// row_out(r) gives the global partial row of tile row r, or -1 to skip it.  vscale multiplies O
// (the V scale of an FP8 cache; 1 otherwise).
template <int D, bool FP8, class RowOut>
__device__ __forceinline__ void store_partial(const OnlineSoftmax<D, FP8>& st, const PartialRef& out, RowOut row_out,
                                              float vscale = 1.f) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
        const int grow = row_out(g + 8 * ri);
        if (grow < 0) continue;
        float* dst = out.acc + static_cast<int64_t>(grow) * D;
        PairOut<D, FP8>::each(st.o, ri, [&](int dim, float v0, float v1) {
            *reinterpret_cast<float2*>(dst + dim) = make_float2(v0 * vscale, v1 * vscale);
        });
        if (c == 0) out.ml[grow] = make_float2(st.m[ri], st.l[ri]);
    }
}

// Shared scratch for merging the NKS warps that swept disjoint key slices of one tile.
template <int D>
constexpr int merge_ld() { return D + 4; }
template <int D, int NKS>
constexpr int merge_floats() { return NKS * 16 * (merge_ld<D>() + 2); }

// Phase 1 (every warp of the tile): park this warp's state in shared memory slot ks (O times
// vscale, in natural dim order).
template <int D, int NKS, bool FP8>
__device__ __forceinline__ void stash_state(const OnlineSoftmax<D, FP8>& st, int ks, float* red, float vscale = 1.f) {
    constexpr int LD = merge_ld<D>();
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    float* red_ml = red + NKS * 16 * LD;
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
        const int r = g + 8 * ri;
        float* dst = red + (ks * 16 + r) * LD;
        PairOut<D, FP8>::each(st.o, ri, [&](int dim, float v0, float v1) {
            *reinterpret_cast<float2*>(dst + dim) = make_float2(v0 * vscale, v1 * vscale);
        });
        if (c == 0) {
            red_ml[(ks * 16 + r) * 2] = st.m[ri];
            red_ml[(ks * 16 + r) * 2 + 1] = st.l[ri];
        }
    }
}

// Phase 2 (after a barrier; threads tid = 0..nthr-1 of the tile): merge the NKS states
// with the log-sum-exp correction and write the tile's partial.
template <int D, int NKS, class RowOut>
__device__ __forceinline__ void merge_states(const float* red, int tid, int nthr, const PartialRef& out,
                                             RowOut row_out) {
    constexpr int LD = merge_ld<D>();
    const float* red_ml = red + NKS * 16 * LD;
    for (int e = tid; e < 16 * D; e += nthr) {
        const int r = e / D, dcol = e % D;
        const int grow = row_out(r);
        if (grow < 0) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NKS; ++w) M = fmaxf(M, red_ml[(w * 16 + r) * 2]);
        float L = 0.f, A = 0.f;
#pragma unroll
        for (int w = 0; w < NKS; ++w) {
            const float mw = red_ml[(w * 16 + r) * 2];
            const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
            L += f * red_ml[(w * 16 + r) * 2 + 1];
            A += f * red[(w * 16 + r) * LD + dcol];
        }
        out.acc[static_cast<int64_t>(grow) * D + dcol] = A;
        if (dcol == 0) out.ml[grow] = make_float2(M, L);
    }
}

}  // namespace hs2
