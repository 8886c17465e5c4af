// New tokens into the shared KV cache (sm_100a): hs2_kv_append and the first kernel of
// hs2_decode_step.
//
// An agent's context grows one token per decode step, and that token's K/V join the cache every
// later query reads ("HySparse2 Cuts the Prefill Path for Tool-Using Agents", section "Tool
// Responses Turn Prefill Into the Bottleneck").  Each (b, kv head, t) row of K_new / V_new (bf16)
// becomes token j of the cache: copied as it is for a bf16 cache, or stored as the E4M3 code of
// value / scale (one IEEE fp32 division, then round to nearest even with saturation to +-448, the
// conversion instruction's satfinite mode) for an FP8 cache.  The row goes to the contiguous
// slice or to slot j % page_size of page page_table[b][j / page_size] of the pool.
//
// advance (decode loop, T = 1): j = pos[b] + 1; one CTA per batch row reads pos[b] before any
// thread of that CTA writes it back, so the update needs no cross-CTA ordering.
#include <cuda_fp8.h>

#include "hs2_device.cuh"

namespace hs2 {

namespace {

constexpr int kAppendThreads = 256;
constexpr int kAppendRows = 32;  // (kv head, t) rows per CTA without advance

// Cache row of token j of (b, h), or -1 (and a status bit) when it cannot be stored.
__device__ __forceinline__ int64_t cache_row(const AppendArgs& a, int b, int h, int j) {
    if (j < 0 || j >= a.N) {
        set_status(a.status, HS2_DEV_BAD_POS);
        return -1;
    }
    if (a.kv.page_shift < 0) return (static_cast<int64_t>(b) * a.Hkv + h) * a.N + j;
    const int page = a.kv.page_table[static_cast<int64_t>(b) * a.kv.max_pages + (j >> a.kv.page_shift)];
    if (page < 0 || page >= a.kv.num_pages) {
        set_status(a.status, HS2_DEV_BAD_PAGE);
        return -1;
    }
    return (static_cast<int64_t>(page) * a.Hkv + h) * (int64_t(1) << a.kv.page_shift) + (j & ((1 << a.kv.page_shift) - 1));
}

// Copies (bf16) or quantises (FP8) 16 elements: chunk q of one K or V row.
__device__ __forceinline__ void store16(const AppendArgs& a, const uint16_t* src_row, void* cache, int64_t row, int q,
                                        float scale) {
    const uint4* src = reinterpret_cast<const uint4*>(src_row + q * 16);
    const uint4 x0 = src[0], x1 = src[1];
    if (!a.kv.fp8) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(cache) + row * a.d + q * 16);
        dst[0] = x0;
        dst[1] = x1;
        return;
    }
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const uint32_t pair = w[2 * i + e];
            const float2 v = make_float2(__fdiv_rn(__uint_as_float(pair << 16), scale),
                                         __fdiv_rn(__uint_as_float(pair & 0xFFFF0000u), scale));
            const uint32_t two = __nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3);  // v.x -> low byte
            packed |= (two & 0xFFFFu) << (16 * e);
        }
        out[i] = packed;
    }
    *reinterpret_cast<uint4*>(static_cast<uint8_t*>(cache) + row * a.d + q * 16) =
        make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendArgs a) {
    const int b = blockIdx.x;
    const int chunks = a.d / 16;  // 16 elements per thread and tensor
    if (a.advance) {
        __shared__ int s_j;
        if (threadIdx.x == 0) {
            const int j = a.pos_in[b] + 1;
            s_j = j;
            a.pos_new[b] = j < 0 ? 0 : (j >= a.N ? a.N - 1 : j);
        }
        __syncthreads();
        const int j = s_j;
        for (int i = threadIdx.x; i < a.Hkv * chunks; i += blockDim.x) {
            const int h = i / chunks, q = i % chunks;
            const int64_t row = cache_row(a, b, h, j);
            if (row < 0) continue;
            const int64_t src = (static_cast<int64_t>(b) * a.Hkv + h) * a.d;
            store16(a, a.K_new + src, a.K, row, q, a.kv.fp8 ? a.kv.k_scale[b * a.Hkv + h] : 1.f);
            store16(a, a.V_new + src, a.V, row, q, a.kv.fp8 ? a.kv.v_scale[b * a.Hkv + h] : 1.f);
        }
        __syncthreads();  // every thread has read pos[b] (through s_j) before it changes
        if (threadIdx.x == 0 && j >= 0 && j < a.N) a.pos_out[b] = j;
        return;
    }
    const int r0 = blockIdx.y * kAppendRows;
    const int nrows = min(kAppendRows, a.Hkv * a.T - r0);
    for (int i = threadIdx.x; i < nrows * chunks; i += blockDim.x) {
        const int r = r0 + i / chunks, q = i % chunks;
        const int h = r / a.T, t = r % a.T;
        const int64_t row = cache_row(a, b, h, a.pos_in[b * a.T + t]);
        if (row < 0) continue;
        const int64_t src = ((static_cast<int64_t>(b) * a.Hkv + h) * a.T + t) * a.d;
        store16(a, a.K_new + src, a.K, row, q, a.kv.fp8 ? a.kv.k_scale[b * a.Hkv + h] : 1.f);
        store16(a, a.V_new + src, a.V, row, q, a.kv.fp8 ? a.kv.v_scale[b * a.Hkv + h] : 1.f);
    }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t st) {
    const unsigned ys = a.advance ? 1u : static_cast<unsigned>((a.Hkv * a.T + kAppendRows - 1) / kAppendRows);
    append_kernel<<<dim3(static_cast<unsigned>(a.B), ys), kAppendThreads, 0, st>>>(a);
    trace_mark("kv_append", st);
    return cudaGetLastError();
}

}  // namespace hs2
