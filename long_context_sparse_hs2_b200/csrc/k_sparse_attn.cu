// Sparse layer with KV Reuse: attention of Q_sparse over the selected keys only (sm_100a), from a
// bf16 or FP8 E4M3 cache, contiguous or paged (the gather resolves each index to its pool row).
//
// Each sparse layer of a hybrid block reuses the preceding full-attention layer's KV
// cache and its token selection ("HySparse2 od Xiaomi zkracuje zpracovani dlouheho
// kontextu", section "Proc neni nutne znovu zpracovat cely dlouhy vstup", third
// paragraph; DAIR.AI newsletter, HySparse2 bullet "Two levels of KV sharing").  All G
// query heads of a kv head share one index list, so a CTA gathers each selected K/V row
// once into shared memory and reuses it for the G heads -- the group-shared tile idea of
// "Simplified Sparse Attention via Gist Tokens", section 3.3 ("Grouped Unfolding for GQA")
// and section 3.6 (split-K partial attention over a compact list).
//
// Grid: (S4 splits, B*Hkv*T rows).  A CTA reads its C4 slots of the row's index list,
// validates them (0 <= j <= pos; others are skipped and flagged), gathers the rows with
// 16-byte cp.async into the same 128-byte-swizzled tile layout the TMA path uses -- a ring
// of up to three 128-key steps in flight -- and runs the shared warp attention core.  The
// row's last CTA to finish (a completion counter; nothing waits) merges the S4 split
// partials into O_sparse and LSE_sparse.
#include <algorithm>
#include <cstdlib>

#include "combine.cuh"
#include "hs2_internal.h"
#include "sparse_core.cuh"

namespace hs2 {

namespace {

__device__ __forceinline__ int64_t out_rows_q_base(const SparseArgs& a, int b, int h, int t) {
    return (static_cast<int64_t>(b) * a.Hq + h * a.G) * a.T + t;  // row of head g is base + g*T
}

// The row's last split CTA merges all S4 partials of the row's G heads (one warp per head).
template <int D>
__device__ __forceinline__ void finish_row(const SparseArgs& a, int row, int64_t rq_base, uint8_t* smem) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&a.meta[static_cast<int64_t>(row) * kMetaInts + kMetaSparseDone], 1) ==
                                    a.S4 - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int64_t rows_q = static_cast<int64_t>(a.B) * a.Hq * a.T;
    float* s_w = reinterpret_cast<float*>(smem);                       // G * S4 weights
    float2* s_ml = reinterpret_cast<float2*>(smem) + a.G * a.S4 / 2 + 1;  // after the weights
    block_combine_rows<D, 16>(a.part_ml, a.part_acc, a.S4, rows_q, rq_base, a.T, a.G, s_w, s_ml, a.O, a.LSE);
}

}  // namespace

// MINB: CTAs per SM the register allocation must allow (2 for one-step CTAs, whose ring is a
// single 64 KB stage; 1 for the deep-ring variant, which also gets the registers to avoid spills).
// TR: at most 8 query heads per kv head -- the transposed warp attention of attn_core_t.cuh
// (keys as the MMA's M dimension, no padded rows).
template <int D, int MINB, bool FP8, bool TR>
__global__ void __launch_bounds__(kSparseThreads, MINB) sparse_attn_kernel(const SparseArgs a) {
    using L = SparseSmem<D, FP8>;
    constexpr int KW = 16;  // keys per warp per step: warps 0-3 take sub-tile 0, warps 4-7 sub-tile 1
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = a.stages;  // ring depth: min(3, 128-key steps of a CTA)
    int* s_idx = reinterpret_cast<int*>(smem + L::idx_off(stages));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x;
    const int row = blockIdx.y;  // (b*Hkv + h)*T + t
    const int t = row % a.T, bh = row / a.T;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    pdl_trigger();
    int pos = a.pos[b * a.T + t];
    pdl_wait();  // idx / cnt (and cleared counters) come from the kernels before
    if (pos < 0 || pos >= a.N) {
        if (tid == 0) set_status(a.status, HS2_DEV_BAD_POS);
        pos = pos < 0 ? 0 : a.N - 1;
    }
    int n = a.cnt[row];
    n = n < 0 ? 0 : (n > a.kw ? a.kw : n);
    const int lo = split * a.C4;
    const int nk = min(lo + a.C4, n) - lo;
    const int64_t rows_q = static_cast<int64_t>(a.B) * a.Hq * a.T;
    auto row_q = [&](int r) -> int { return r < a.G ? (b * a.Hq + h * a.G + r) * a.T + t : -1; };
    const PartialRef out{a.part_ml + split * rows_q, a.part_acc + split * rows_q * D};

    if (nk <= 0) {  // empty split: m = -inf, l = 0, O = 0
        for (int e = tid; e < a.G * D; e += kSparseThreads) {
            const int r = e / D, dc = e % D;
            out.acc[static_cast<int64_t>(row_q(r)) * D + dc] = 0.f;
            if (dc == 0) out.ml[row_q(r)] = make_float2(-INFINITY, 0.f);
        }
        finish_row<D>(a, row, out_rows_q_base(a, b, h, t), smem);
        return;
    }

    const int ntl = (nk + kSparseTile - 1) / kSparseTile;
    const bool paged = a.kv.page_shift >= 0;
    bool bad = false, bad_page = false;
    for (int i = tid; i < ntl * kSparseTile; i += kSparseThreads) {
        int j = -1;
        if (i < nk) {
            j = a.idx[static_cast<int64_t>(row) * a.kw + lo + i];
            if (j < 0 || j > pos) {
                bad = true;
                j = -1;
            } else if (paged) {  // the token's row in the page pool
                const int page = a.kv.page_table[static_cast<int64_t>(b) * a.kv.max_pages + (j >> a.kv.page_shift)];
                if (page < 0 || page >= a.kv.num_pages) {
                    bad_page = true;
                    j = -1;
                } else {
                    j = (page * a.Hkv + h) * (1 << a.kv.page_shift) + (j & ((1 << a.kv.page_shift) - 1));
                }
            }
        }
        s_idx[i] = j;
    }
    if (__syncthreads_or(bad) && tid == 0) set_status(a.status, HS2_DEV_BAD_INDEX);
    if (__syncthreads_or(bad_page) && tid == 0) set_status(a.status, HS2_DEV_BAD_PAGE);

    const int64_t kv_base = paged ? 0 : static_cast<int64_t>(bh) * a.N;
    const int prime = min(ntl, stages);
    for (int i = 0; i < prime; ++i) {
        gather_tile<D, FP8>(a.K, a.V, s_idx, i, smem + i * L::kStageBytes, kv_base);
        cp_async_commit();
    }

    const int g = lane >> 2, c = lane & 3;
    const float kscale = FP8 ? a.kv.k_scale[bh] : 1.f;
    const float vscale = FP8 ? a.kv.v_scale[bh] : 1.f;
    const int sub = warp >> 2;
    const int key0 = (warp & 3) * KW;
    float* red = reinterpret_cast<float*>(smem);
    if constexpr (TR) {
        QTileT<D, FP8> q;
        const int rq = row_q(g);
        q.load(a.Q, rq >= 0 ? static_cast<int64_t>(rq) * D : -1);
        const float f0 = a.scale_log2 * kscale * q.col_scale[0];
        const float f1 = a.scale_log2 * kscale * q.col_scale[1];
        OnlineSoftmaxT<D, FP8> st;
        st.init();
        for (int i = 0; i < ntl; ++i) {
            cp_async_wait_upto(min(ntl, i + stages) - (i + 1));  // step i has landed
            __syncthreads();
            const int stage = i % stages;
            const uint32_t kbase = smem_u32(smem + stage * L::kStageBytes + sub * L::kSubBytes);
            const uint32_t vbase = kbase + L::kTileBytes;
            float sc[4];  // keys g, g + 8 of the warp's 16 for query heads 2c, 2c + 1
            qk_t<D, FP8>(q, kbase, key0, sc);
            const int slot = i * kSparseTile + sub * kKeyTile + key0 + g;
            const bool v_lo = s_idx[slot] >= 0, v_hi = s_idx[slot + 8] >= 0;
            sc[0] = v_lo ? sc[0] * f0 : -INFINITY;
            sc[1] = v_lo ? sc[1] * f1 : -INFINITY;
            sc[2] = v_hi ? sc[2] * f0 : -INFINITY;
            sc[3] = v_hi ? sc[3] * f1 : -INFINITY;
            st.update(sc, vbase, key0);
            __syncthreads();  // everyone is done with this stage before it is refilled
            if (i + stages < ntl) {
                gather_tile<D, FP8>(a.K, a.V, s_idx, i + stages, smem + stage * L::kStageBytes, kv_base);
                cp_async_commit();
            }
        }
        st.finish_rows();
        stash_state_t<D, kSparseWarps, FP8>(st, warp, red, vscale);
    } else {
        QTileOf<D, FP8> q;
        {
            const int r0 = row_q(g), r1 = row_q(g + 8);
            q.load(a.Q, r0 >= 0 ? static_cast<int64_t>(r0) * D : -1, r1 >= 0 ? static_cast<int64_t>(r1) * D : -1);
        }
        const float f_lo = logit_factor<D, FP8>(q, 0, a.scale_log2, kscale);
        const float f_hi = logit_factor<D, FP8>(q, 1, a.scale_log2, kscale);
        OnlineSoftmax<D, FP8> st;
        st.init();
        for (int i = 0; i < ntl; ++i) {
            cp_async_wait_upto(min(ntl, i + stages) - (i + 1));  // step i has landed
            __syncthreads();
            const int stage = i % stages;
            const uint32_t kbase = smem_u32(smem + stage * L::kStageBytes + sub * L::kSubBytes);
            const uint32_t vbase = kbase + L::kTileBytes;
            float sc[KW / 8][4];
            qk_any<D, KW, FP8>(q, kbase, key0, sc);
            const int slot0 = i * kSparseTile + sub * kKeyTile + key0 + 2 * c;
#pragma unroll
            for (int nn = 0; nn < KW / 8; ++nn)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool ok = s_idx[slot0 + nn * 8 + (e & 1)] >= 0;
                    sc[nn][e] = ok ? sc[nn][e] * (e < 2 ? f_lo : f_hi) : -INFINITY;
                }
            st.template update<KW>(sc, vbase, key0);
            __syncthreads();  // everyone is done with this stage before it is refilled
            if (i + stages < ntl) {
                gather_tile<D, FP8>(a.K, a.V, s_idx, i + stages, smem + stage * L::kStageBytes, kv_base);
                cp_async_commit();
            }
        }
        st.finish_rows();
        stash_state<D, kSparseWarps, FP8>(st, warp, red, vscale);
    }
    __syncthreads();
    merge_states<D, kSparseWarps>(red, tid, kSparseThreads, out, row_q);
    finish_row<D>(a, row, out_rows_q_base(a, b, h, t), smem);
}

template <int D, int MINB, bool FP8, bool TR>
cudaError_t sparse_variant(const Plan& p, const SparseArgs& x, cudaStream_t st) {
    auto kern = sparse_attn_kernel<D, MINB, FP8, TR>;
    const int bytes = SparseSmem<D, FP8>::bytes(x.stages, p.C4);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(p.S4, static_cast<unsigned>(p.rows_kv)), dim3(kSparseThreads), bytes, st, x);
    trace_mark("sparse_attn_combine", st);
    return e;
}

template <int D, bool FP8>
cudaError_t sparse_dispatch(const Plan& p, const SparseArgs& x, cudaStream_t st) {
    // at most 8 query heads per kv head: the transposed warp attention (HS2_TRANSPOSED=0: the
    // 16-row form)
    const char* env = std::getenv("HS2_TRANSPOSED");
    if (p.G <= 8 && !(env && env[0] == '0'))
        return x.stages == 1 ? sparse_variant<D, 2, FP8, true>(p, x, st) : sparse_variant<D, 1, FP8, true>(p, x, st);
    return x.stages == 1 ? sparse_variant<D, 2, FP8, false>(p, x, st) : sparse_variant<D, 1, FP8, false>(p, x, st);
}

cudaError_t launch_sparse_attn(const Plan& p, const SparseArgs& a, cudaStream_t st) {
    SparseArgs x = a;
    x.stages = std::min(kSparseMaxStages, (p.C4 + kSparseTile - 1) / kSparseTile);
    if (p.d == 128) return p.fp8 ? sparse_dispatch<128, true>(p, x, st) : sparse_dispatch<128, false>(p, x, st);
    return p.fp8 ? sparse_dispatch<64, true>(p, x, st) : sparse_dispatch<64, false>(p, x, st);
}

}  // namespace hs2
