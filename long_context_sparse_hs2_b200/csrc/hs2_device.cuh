// Device-side building blocks shared by the HySparse2 kernels (sm_100a).
//
// Everything here is a thin wrapper over one PTX instruction or a small, exact
// integer/bit manipulation: shared-memory addresses, mbarriers with bounded waits,
// TMA tile loads (no multicast), cp.async gathers, ldmatrix, warp-level bf16 MMA,
// the order-preserving float->uint32 key used by the top-k, and the device status
// word.  No kernel logic lives here.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "hs2_internal.h"

namespace hs2 {

// ------------------------------------------------------------------ status word

__device__ __forceinline__ void set_status(unsigned* status, unsigned bits) {
    if (status) atomicOr(status, bits);
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ programmatic dependent launch
//
// Kernels of one call are launched with programmatic stream serialisation: a kernel may start
// while its predecessor drains, runs its prologue, and calls pdl_wait() before it touches
// anything the predecessor writes (pdl_wait returns once the predecessor has completed and its
// memory is visible; without the launch attribute it returns at once).  pdl_trigger() lets the
// next kernel launch as soon as every CTA of this one has started.

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ shared memory

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Ends an mbarrier's life (before its shared memory is used for anything else).
__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed, for at most limit_ns (kWaitLimitNs,
// 2 s, unless a shorter bound is given).  Returns false (and flags HS2_DEV_TIMEOUT) if the bound
// ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) {
            pdl_wait();  // the status word is cleared by the call's first kernel
            set_status(status, HS2_DEV_TIMEOUT);
            return false;
        }
    }
}

// Makes this thread's ordinary shared-memory stores visible to the async proxy (TMA, tensor
// core) before a following barrier arrive.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------ L2 cache policies

// A stream read once (the K/V sweep) is loaded evict-first; short-lived intermediates the next
// phase reads back (kept logits, split partials) are stored evict-last, and dropped from L2
// with discard once consumed so they are never written back to HBM.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void st_f32_policy(float* p, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}
// Invalidates (without write-back) the 128-byte L2 line holding p: its data becomes undefined.
__device__ __forceinline__ void discard_l2_line(const void* p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// ------------------------------------------------------------------ TMA (no multicast)

// 3-D tiled bulk tensor load global -> shared, completing on an mbarrier, with an L2 cache
// policy.  Coordinates are (c0 = innermost element, c1, c2).  c0 must be a multiple of 8 for bf16.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 4-D tiled load (paged pool [num_pages][Hkv][page_size][d]: c0 = element, c1 = slot in the page,
// c2 = kv head, c3 = page).  An out-of-range coordinate reads as zeros.
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Untiled bulk copy global -> shared of `bytes` (a multiple of 16; both addresses 16-byte
// aligned), completing on an mbarrier; no multicast.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ cp.async (gather)

// 16-byte async copy; src_bytes = 0 zero-fills the destination without reading src.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ ldmatrix / mma

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulate.
// Transpose of an 8x8 matrix of b16 elements held one row per lane quad (lane 4r + c holds
// elements (r, 2c) and (r, 2c + 1)); afterwards the lane holds (2c, r) and (2c + 1, r).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t r;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A(16x16, row) * B(16x8, col) + D, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two fp32 -> packed f16x2 (round to nearest even); lo goes to the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two FP8 E4M3 codes (the low byte first) -> f16x2, exact (every E4M3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    uint32_t r;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(r) : "r"(two_codes));
    return r;
}

// Two fp32 -> packed bf16x2 (round to nearest even); lo goes to the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2^x on the SFU (ex2.approx, flush-to-zero); -inf -> +0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ swizzled K/V tiles
//
// A tile of kKeyTile keys x D dims (bf16) is stored as D/64 "halves"; half h holds
// dims [64h, 64h+64) of every key as 128-byte rows, with the 16-byte chunks of row r
// permuted by XOR with (r & 7).  This is exactly the layout a TMA load with
// CU_TENSOR_MAP_SWIZZLE_128B and a 64-element inner box writes, and what the gather
// path writes by hand, so ldmatrix reads are bank-conflict free in both.
__device__ __forceinline__ uint32_t tile_chunk_offset(int row, int chunk16) {
    // chunk16 = 16-byte chunk index across the full row (0 .. D/8-1)
    const int half = chunk16 >> 3;
    const int c = chunk16 & 7;
    return static_cast<uint32_t>(half * (kKeyTile * 128) + row * 128 + ((c ^ (row & 7)) << 4));
}

// FP8 E4M3 tiles hold one D-byte row per key: D = 128 uses the same 128-byte swizzled rows as a
// 64-dim bf16 half (TMA CU_TENSOR_MAP_SWIZZLE_128B); D = 64 uses 64-byte rows with the 64-byte
// swizzle (16-byte chunk c of row r stored at chunk c ^ ((r >> 1) & 3), as TMA writes with
// CU_TENSOR_MAP_SWIZZLE_64B).  chunk16 indexes 16-byte chunks (16 dims) of the row.
template <int D>
__device__ __forceinline__ uint32_t fp8_chunk_offset(int row, int chunk16) {
    if constexpr (D == 128)
        return static_cast<uint32_t>(row * 128 + ((chunk16 ^ (row & 7)) << 4));
    else
        return static_cast<uint32_t>(row * 64 + ((chunk16 ^ ((row >> 1) & 3)) << 4));
}

// Byte offset of 16-byte chunk `chunk16` of key `row` in a K/V tile of the cache's element type.
template <int D, bool FP8>
__device__ __forceinline__ uint32_t kv_chunk_offset(int row, int chunk16) {
    if constexpr (FP8)
        return fp8_chunk_offset<D>(row, chunk16);
    else
        return tile_chunk_offset(row, chunk16);
}

// ------------------------------------------------------------------ top-k keys

// Order-preserving map float -> uint32 (larger float -> larger key).  NaN maps to 0
// (below every other value); -0 is treated as +0.
__device__ __forceinline__ uint32_t score_key(float s) {
    if (s != s) return 0u;
    if (s == 0.0f) s = 0.0f;
    const uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t u) {
    const uint32_t b = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
    return __uint_as_float(b);
}

}  // namespace hs2
