// The gathered-attention core of the sparse layer (sm_100a), used by the sparse-attention
// kernel: selected K/V rows are gathered with 16-byte cp.async into the
// same swizzled tile layout the TMA path writes (bf16 or FP8 E4M3 tiles), a ring of up to three
// 128-key steps in flight, and 8 warps run the warp attention core on them (warps 0-3 take the
// first 64-key sub-tile of a step, warps 4-7 the second).
#pragma once

#include "attn_core_t.cuh"

namespace hs2 {

constexpr int kSparseWarps = 8;
constexpr int kSparseThreads = kSparseWarps * 32;
constexpr int kSparseTile = 2 * kKeyTile;  // keys per pipeline step: two 64-key sub-tiles

constexpr int kSparseMaxStages = 3;  // ring depth for long rows; short rows use fewer (less smem)

template <int D, bool FP8>
struct SparseSmem {
    static constexpr int kTileBytes = kKeyTile * D * (FP8 ? 1 : 2);  // one 64-key sub-tile of K (or V)
    static constexpr int kSubBytes = 2 * kTileBytes;       // K + V of one sub-tile
    static constexpr int kStageBytes = 2 * kSubBytes;      // two sub-tiles = one 128-key step
    // After the main loop the ring is reused as scratch: the warps' softmax states are merged
    // there (merge_states) and the row's last CTA keeps its combine weights there; the region
    // before the index list is at least as large as either.
    static constexpr int kMergeBytes = merge_floats<D, kSparseWarps>() * 4;
    static constexpr int kCombineBytes = (8192 / 2 + 1 + 16) * 8;  // G * S4 <= 8192 weights, then G <= 16 (m, l)
    static constexpr int kScratchBytes = kMergeBytes > kCombineBytes ? kMergeBytes : kCombineBytes;
    static constexpr int idx_off(int stages) {
        return stages * kStageBytes > kScratchBytes ? stages * kStageBytes : kScratchBytes;
    }
    static constexpr int bytes(int stages, int C4) { return idx_off(stages) + (C4 + kSparseTile) * 4 + 16 + 1024; }
};

// Wait until at most `pending` of this thread's cp.async groups are still in flight.
__device__ __forceinline__ void cp_async_wait_upto(int pending) {
    static_assert(kSparseMaxStages <= 3, "extend the wait ladder");
    if (pending <= 0)
        cp_async_wait<0>();
    else if (pending == 1)
        cp_async_wait<1>();
    else
        cp_async_wait<2>();
}

// Gathers the K and V rows of 128-key step `tile` into a stage: sub-tile u (keys 64u..64u+63
// of the step) at u * kSubBytes, K then V, each in the swizzled 64-key tile layout of the cache's
// element type.  Thread t copies 16-byte chunk t mod CH of rows t / CH, + 256/CH, ... of both
// sub-tiles, K and V alike: one index load and one address per row for two copies.  s_row holds
// the cache row of every slot (-1: empty or skipped); kv_base is added for a contiguous cache.
template <int D, bool FP8>
__device__ __forceinline__ void gather_tile(const void* K, const void* V, const int* s_row, int tile, uint8_t* stage,
                                            int64_t kv_base) {
    using L = SparseSmem<D, FP8>;
    constexpr int RB = D * (FP8 ? 1 : 2);           // bytes per cache row
    constexpr int CH = RB / 16;                     // 16-byte chunks per row
    constexpr int RSTEP = kSparseThreads / CH;      // rows covered per pass
    const int c16 = threadIdx.x % CH, r0 = threadIdx.x / CH;
    const uint8_t* Kb = reinterpret_cast<const uint8_t*>(K);
    const uint8_t* Vb = reinterpret_cast<const uint8_t*>(V);
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
#pragma unroll
        for (int rr = r0; rr < kKeyTile; rr += RSTEP) {
            const int j = s_row[tile * kSparseTile + sub * kKeyTile + rr];
            const int64_t off = (kv_base + (j >= 0 ? j : 0)) * RB + c16 * 16;
            const uint32_t nbytes = j >= 0 ? 16u : 0u;
            uint8_t* dst = stage + sub * L::kSubBytes + kv_chunk_offset<D, FP8>(rr, c16);
            cp_async16(dst, Kb + off, nbytes);
            cp_async16(dst + L::kTileBytes, Vb + off, nbytes);
        }
    }
}

}  // namespace hs2
