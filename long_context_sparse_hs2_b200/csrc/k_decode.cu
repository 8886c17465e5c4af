// The whole hybrid step for one decode query per batch row (T = 1) in a single kernel
// (sm_100a).
//
// Grid (S1 splits, B*Hkv rows), launched cooperatively so every CTA is co-resident.  The S1
// CTAs of a row -- one (b, kv head) -- run the split-K full-attention sweep over disjoint key
// ranges (attn_sweep.cuh, keeping the base-2 logits), then walk through the rest of the step
// together, separated by bounded per-row barriers (hs2_device.cuh, cta_barrier):
//
//   B0  every split partial and logit of the row is written.
//   A   each CTA merges the G heads' LSE from the partials, scores the pool keys of its own
//       key range -- s_j = max_g (l_gj - LSE_g), the GQA-max log-softmax probability --
//       keeps their order-preserving keys in shared memory and adds its bucket histogram to
//       the row's.
//   B1  the row's histogram is complete.
//   B   every CTA finds the threshold bucket b1 (redundantly; same result), emits its keys in
//       better buckets straight into idx, appends its b1 keys to the row's candidates, writes
//       its slice of the window, and starts gathering the K/V rows of both (cp.async).
//   B2  the candidate list is complete.
//   C   every CTA radix-selects the same exact 64-bit composite threshold among the
//       candidates and emits the winners of its slice; split 0 writes the -1 padding and cnt.
//   D   each CTA attends with Q_sparse (the row's G heads) over the keys it wrote itself --
//       its definite winners, window slice and final winners, all KV Reuse index-list
//       entries -> a sparse split partial.  No barrier is needed before it.
//   B3  every sparse partial is written.
//   E   split 0 merges the sparse partials of the G heads into O_sparse / LSE_sparse and
//       split 1 the full partials into O_full / LSE_full (each CTA-wide, all heads at once).
//
// Sources: token-level selection with forced recent tokens and KV Reuse ("HySparse2 od
// Xiaomi zkracuje zpracovani dlouheho kontextu", section "Proc neni nutne znovu zpracovat
// cely dlouhy vstup", third paragraph; DAIR.AI newsletter, HySparse2 bullets); split-K
// partials, compaction by warp ballot and a log-sum-exp combine ("Simplified Sparse
// Attention via Gist Tokens", section 3.6).
#include "attn_sweep.cuh"
#include "combine.cuh"
#include "topk_common.cuh"

namespace hs2 {

namespace {

constexpr int kThreads = 160;  // 4 consumer warps + the producer warp

struct SmemCand {
    const unsigned long long* c;
    int n;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const { v = c[i]; return true; }
};
struct GlobalCand {
    const unsigned long long* c;
    int n;
    __device__ int size() const { return n; }
    __device__ bool get(int i, unsigned long long& v) const { v = __ldcg(c + i); return true; }
};

// Exact composite threshold: see k_topk.cu (the same digit walk, duplicated here so the fused
// kernel keeps its shared memory to itself).
template <class Src>
__device__ unsigned long long fused_radix_threshold(const Src& src, unsigned need, unsigned* h, unsigned* s_small,
                                                    unsigned long long* s_and, unsigned long long* s_or) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long all_and = ~0ull, any_or = 0ull;
    for (int i = threadIdx.x; i < src.size(); i += blockDim.x) {
        unsigned long long c;
        if (src.get(i, c)) {
            all_and &= c;
            any_or |= c;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        all_and &= __shfl_xor_sync(0xffffffffu, all_and, o);
        any_or |= __shfl_xor_sync(0xffffffffu, any_or, o);
    }
    if (lane == 0) {
        s_and[warp] = all_and;
        s_or[warp] = any_or;
    }
    __syncthreads();
    all_and = ~0ull;
    any_or = 0ull;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
        all_and &= s_and[w];
        any_or |= s_or[w];
    }
    __syncthreads();
    const unsigned long long differ = all_and ^ any_or;
    if (differ == 0ull) return all_and;
    const int top = 63 - __clzll(static_cast<long long>(differ));
    const int first_shift = (top / 8) * 8;
    unsigned long long prefix = first_shift >= 56 ? 0ull : (all_and & (~0ull << (first_shift + 8)));
    for (int shift = first_shift; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0u;
        if (threadIdx.x == 0) s_small[0] = s_small[1] = 0u;
        __syncthreads();
        const unsigned long long mask_hi = (shift == 56) ? 0ull : (~0ull << (shift + 8));
        for (int i = threadIdx.x; i < src.size(); i += blockDim.x) {
            unsigned long long c;
            if (src.get(i, c) && (c & mask_hi) == (prefix & mask_hi))
                atomicAdd(&h[static_cast<int>((c >> shift) & 255ull)], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            unsigned cnts[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnts[i] = h[255 - 8 * lane - i];
                sum += cnts[i];
            }
            unsigned incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned excl = incl - sum;
            if (excl < need && need <= incl) {
                unsigned cum = excl;
                for (int i = 0; i < 8; ++i) {
                    if (cum + cnts[i] >= need) {
                        s_small[0] = 255 - 8 * lane - i;
                        s_small[1] = cum;
                        break;
                    }
                    cum += cnts[i];
                }
            }
        }
        __syncthreads();
        const unsigned d = s_small[0];
        need -= s_small[1];
        prefix |= static_cast<unsigned long long>(d) << shift;
        const bool done = (h[d] == need);
        __syncthreads();
        if (done) break;
    }
    return prefix;
}

template <int D>
__device__ __forceinline__ void gather_rows(const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
                                            const int* s_idx, int tile, uint8_t* stage, int64_t kv_base) {
    constexpr int CH = D / 8;
    constexpr int PER_T = kKeyTile * CH;
    constexpr int TILE = kKeyTile * D * 2;
    for (int ch = threadIdx.x; ch < 2 * PER_T; ch += blockDim.x) {
        const int tensor = ch / PER_T;
        const int rem = ch - tensor * PER_T;
        const int r = rem / CH, c16 = rem - r * CH;
        const int j = s_idx[tile * kKeyTile + r];
        const uint16_t* src = (tensor ? V : K) + (kv_base + (j >= 0 ? j : 0)) * D + c16 * 8;
        cp_async16(stage + tensor * TILE + tile_chunk_offset(r, c16), src, j >= 0 ? 16u : 0u);
    }
}

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 2) decode_step_kernel(const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               const DecodeArgs a) {
    constexpr int NC = 4;
    constexpr int STAGES = D == 128 ? 3 : 6;
    constexpr int KW = kKeyTile / NC;
    __shared__ unsigned h[256];
    __shared__ unsigned s_small[2];
    __shared__ unsigned long long s_and[32], s_or[32];
    __shared__ unsigned s_warp[32];
    __shared__ int s_flag, s_b1, s_above, s_base;
    __shared__ unsigned long long s_base2;
    __shared__ int s_cnt[2];
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);

    const AttnArgs& at = a.attn;
    const int split = blockIdx.x, S = gridDim.x;
    const int row = blockIdx.y;  // b*Hkv + h (one query per batch row)
    const int b = row / at.Hkv, hk = row % at.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows_q = static_cast<int64_t>(at.B) * at.Hq;
    auto row_q = [&](int g) -> int64_t { return static_cast<int64_t>(b) * at.Hq + hk * G + g; };
    unsigned* status = at.status;

    // ---------------------------------------------------------------- full-attention sweep
    int2 range;
    const bool swept = full_sweep<D, 1, NC, STAGES, true>(&tmK, &tmV, at, smem, split, row, &range);
    pdl_wait();  // the call's first kernel has cleared the status word, counters and histograms
    if (!swept) return;
    int* meta = a.meta + static_cast<int64_t>(row) * kMetaInts;
    unsigned* bar = reinterpret_cast<unsigned*>(meta + kMetaBarrier);
    if (!cta_barrier(bar, 1u * S, status, &s_flag)) return;  // B0

    // ---------------------------------------------------------------- A: LSE, scores, histogram
    const RowInfo ri = make_row_info(at.pos, row, at.Hkv, 1, at.N, a.k, a.W);
    const bool ranked = ri.keff > 0 && ri.keff < ri.P;
    float* s_lse2 = reinterpret_cast<float*>(smem + kFusedLseOff);
    float* wbuf = reinterpret_cast<float*>(smem + kFusedWbufOff);
    unsigned* sh = reinterpret_cast<unsigned*>(smem + kFusedHistOff);
    uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + kFusedKeysOff);
    const int k0 = range.x * kKeyTile;
    const int k1 = min(range.y * kKeyTile, ri.P);
    const int nmine = max(0, k1 - k0);
    if (warp < NC) {
        for (int g = warp; g < G; g += NC) {
            const float2 ML = warp_row_ml(at.part_ml, S, rows_q, row_q(g));
            if (lane == 0) s_lse2[g] = lse2_of(ML);
        }
    }
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    if (ranked && warp < NC) {
        float lse[G];
#pragma unroll
        for (int g = 0; g < G; ++g) lse[g] = s_lse2[g];
        const float* lg = at.logits + static_cast<int64_t>(row) * at.N * G;
        bool nonfinite = false;
        constexpr int U = 8;  // logit rows in flight per thread
        for (int base = threadIdx.x; base < nmine; base += U * NC * 32) {
            float v[U][G];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * NC * 32;
                if (i < nmine) {
                    const float* src = lg + static_cast<int64_t>(k0 + i) * G;
                    if constexpr (G % 4 == 0) {
#pragma unroll
                        for (int q = 0; q < G / 4; ++q) {
                            const float4 f = __ldcg(reinterpret_cast<const float4*>(src) + q);
                            v[u][4 * q] = f.x;
                            v[u][4 * q + 1] = f.y;
                            v[u][4 * q + 2] = f.z;
                            v[u][4 * q + 3] = f.w;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < G; ++q) v[u][q] = __ldcg(src + q);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * NC * 32;
                if (i < nmine) {
                    float s = v[u][0] - lse[0];
#pragma unroll
                    for (int g = 1; g < G; ++g) s = nan_max(s, v[u][g] - lse[g]);
                    nonfinite |= (s != s);
                    const uint32_t key = score_key(s);
                    s_keys[i] = key;
                    atomicAdd(&sh[score_bin(key)], 1u);
                }
            }
        }
        if (__any_sync(0xffffffffu, nonfinite) && lane == 0) set_status(status, HS2_DEV_NONFINITE);
    }
    __syncthreads();
    {  // this split's kept logits are dead now: drop the 128-byte lines wholly inside its range
       // from L2 without write-back (lines shared with a neighbouring range are left alone)
        const uintptr_t lo = reinterpret_cast<uintptr_t>(at.logits + (static_cast<int64_t>(row) * at.N + k0) * G);
        const uintptr_t hi = lo + static_cast<uintptr_t>(max(0, min(range.y * kKeyTile, at.N) - k0)) * G * 4;
        for (uintptr_t p = ((lo + 127) & ~uintptr_t(127)) + threadIdx.x * 128; p + 128 <= hi; p += blockDim.x * 128)
            discard_l2_line(reinterpret_cast<const void*>(p));
    }
    if (ranked) {
        unsigned* hist = a.hist + static_cast<int64_t>(row) * kHistBins;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
            if (sh[i]) atomicAdd(&hist[i], sh[i]);
    }
    if (!cta_barrier(bar, 2u * S, status, &s_flag)) return;  // B1

    // ---------------------------------------------------------------- B: threshold bucket, emit
    // Each CTA's sparse-attention work list is three contiguous segments of idx that it writes
    // itself: its definite winners, its slice of the window, and its share of the final
    // winners -- so no barrier is needed before the gathers, and the first ones are issued
    // before the candidate phase.
    const int kw = a.k + a.W;
    int32_t* idx = a.idx + static_cast<int64_t>(row) * kw;
    int32_t* out = idx + ri.wcnt;
    int def_base = 0, ndef = 0;
    if (ranked) {
        const unsigned* hist = a.hist + static_cast<int64_t>(row) * kHistBins;
        constexpr int PER = kHistBins / (NC * 32);  // bins per consumer thread
        unsigned vals[PER], sum = 0;
        if (warp < NC) {
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                vals[i] = __ldcg(&hist[threadIdx.x * PER + i]);
                sum += vals[i];
            }
        }
        const unsigned excl = block_exclusive_scan(warp < NC ? sum : 0u, s_warp);
        const unsigned need = static_cast<unsigned>(ri.keff);
        if (warp < NC && excl < need && need <= excl + sum) {
            unsigned cum = excl;
            for (int i = 0; i < PER; ++i) {
                if (cum + vals[i] >= need) {
                    s_b1 = threadIdx.x * PER + i;
                    s_above = static_cast<int>(cum);
                    break;
                }
                cum += vals[i];
            }
        }
        __syncthreads();
        const int b1 = s_b1, above = s_above;
        unsigned long long* cand = a.cand + static_cast<int64_t>(row) * a.cand_cap;
        // pass 1: this CTA's counts; one global atomic per CTA reserves its slots
        int nd = 0, nc = 0;
        for (int i = threadIdx.x; i < nmine; i += blockDim.x) {
            const int bin = score_bin(s_keys[i]);
            nd += bin < b1;
            nc += bin == b1;
        }
        if (threadIdx.x == 0) s_cnt[0] = s_cnt[1] = 0;
        __syncthreads();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            nd += __shfl_xor_sync(0xffffffffu, nd, o);
            nc += __shfl_xor_sync(0xffffffffu, nc, o);
        }
        if (lane == 0) {
            atomicAdd(&s_cnt[0], nd);
            atomicAdd(&s_cnt[1], nc);
        }
        __syncthreads();
        ndef = s_cnt[0];
        const int2 bases = block_reserve2(ndef, s_cnt[1], &meta[kMetaDef], &s_base2);
        def_base = bases.x;
        const int cnd_base = bases.y;
        if (threadIdx.x == 0) s_cnt[0] = s_cnt[1] = 0;
        __syncthreads();
        // pass 2: write with CTA-local slots (shared-memory atomics, one per warp per step)
        for (int base = warp * 32; base < nmine; base += blockDim.x) {
            const int i = base + lane;
            const bool valid = i < nmine;
            const uint32_t key = valid ? s_keys[i] : 0u;
            const int bin = valid ? score_bin(key) : kHistBins;
            const bool def = valid && bin < b1;
            const bool cnd = valid && bin == b1;
            const int sd = warp_append(def, &s_cnt[0]);
            if (def && def_base + sd < above) out[def_base + sd] = k0 + i;
            const int sc = warp_append(cnd, &s_cnt[1]);
            if (cnd && cnd_base + sc < a.cand_cap) cand[cnd_base + sc] = composite(key, k0 + i);
        }
        ndef = max(0, min(ndef, above - def_base));
    } else if (ri.keff > 0) {  // the whole pool is selected: this CTA's keys are its winners
        for (int i = threadIdx.x; i < nmine; i += blockDim.x) out[k0 + i] = k0 + i;
        def_base = k0;
        ndef = nmine;
    }
    // window slice of this CTA (its keys are known without any selection)
    const int w0 = static_cast<int>((static_cast<int64_t>(split) * ri.wcnt) / S);
    const int w1 = static_cast<int>((static_cast<int64_t>(split + 1) * ri.wcnt) / S);
    for (int i = w0 + threadIdx.x; i < w1; i += blockDim.x) idx[i] = ri.pos - ri.wcnt + 1 + i;
    __syncthreads();  // idx segments written; s_keys no longer needed

    // work list: pre items [definite winners | window slice] in tiles of 64, then the final
    // winners in tiles of their own (so tiles staged before the candidate phase stay valid)
    const int nwin = w1 - w0;
    int fin_base = 0, nfin = 0;
    int* s_slot = reinterpret_cast<int*>(smem + kFusedHistOff);  // 2 stages x 64 gather slots
    uint8_t* ring = smem + kFusedRingOff;
    constexpr int kStageBytes = 2 * kKeyTile * D * 2;
    const int64_t kv_base = static_cast<int64_t>(row) * at.N;
    const int pre_items = ndef + nwin;
    const int pre_tiles = (pre_items + kKeyTile - 1) / kKeyTile;
    // slot s of tile t -> key index (definite and final winners are read back from idx)
    auto tile_key = [&](int t, int s) -> int {
        if (t < pre_tiles) {
            const int i = t * kKeyTile + s;
            if (i >= pre_items) return -1;
            if (i < ndef) return __ldcg(out + def_base + i);
            return ri.pos - ri.wcnt + 1 + w0 + (i - ndef);
        }
        const int i = (t - pre_tiles) * kKeyTile + s;
        return i < nfin ? __ldcg(out + s_above + fin_base + i) : -1;
    };
    auto stage_tile = [&](int t) {  // resolve the 64 slots of tile t, then gather their K/V rows
        int* slots = s_slot + (t & 1) * kKeyTile;
        if (threadIdx.x < kKeyTile) {
            int j = tile_key(t, threadIdx.x);
            if (j > ri.pos) {  // cannot happen: the CTA wrote these itself
                set_status(status, HS2_DEV_BAD_INDEX);
                j = -1;
            }
            slots[threadIdx.x] = j < 0 ? -1 : j;
        }
        __syncthreads();
        gather_rows<D>(a.K, a.V, slots, 0, ring + (t & 1) * kStageBytes, kv_base);
        cp_async_commit();
    };
    // the definite winners and the window slice are known now: start gathering them
    const int pre_staged = min(2, pre_tiles);
    for (int t = 0; t < pre_staged; ++t) stage_tile(t);
    if (!cta_barrier(bar, 3u * S, status, &s_flag)) return;  // B2: the candidate list is complete

    // ---------------------------------------------------------------- C: exact threshold
    if (ranked) {
        const int above = s_above;
        const unsigned need = static_cast<unsigned>(ri.keff - above);
        const int ncand = min(static_cast<int64_t>(__ldcg(&meta[kMetaCand])), a.cand_cap);
        const unsigned long long* gc = a.cand + static_cast<int64_t>(row) * a.cand_cap;
        unsigned long long thr;
        unsigned long long* sc = reinterpret_cast<unsigned long long*>(smem + kFusedCandOff);
        const bool in_smem = ncand <= kFusedSmemCand;
        if (in_smem) {
            for (int i = threadIdx.x; i < ncand; i += blockDim.x) sc[i] = __ldcg(gc + i);
            __syncthreads();
            thr = fused_radix_threshold(SmemCand{sc, ncand}, need, h, s_small, s_and, s_or);
        } else {
            thr = fused_radix_threshold(GlobalCand{gc, ncand}, need, h, s_small, s_and, s_or);
        }
        // this CTA's slice of the candidates: count its winners, reserve slots once, write
        const int c0 = static_cast<int>((static_cast<int64_t>(split) * ncand) / S);
        const int c1 = static_cast<int>((static_cast<int64_t>(split + 1) * ncand) / S);
        int nw = 0;
        for (int i = c0 + threadIdx.x; i < c1; i += blockDim.x) nw += (in_smem ? sc[i] : __ldcg(gc + i)) >= thr;
        if (threadIdx.x == 0) s_cnt[0] = 0;
        __syncthreads();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nw += __shfl_xor_sync(0xffffffffu, nw, o);
        if (lane == 0) atomicAdd(&s_cnt[0], nw);
        __syncthreads();
        nfin = s_cnt[0];
        fin_base = block_reserve(nfin, &meta[kMetaSelDone], &s_base);
        if (threadIdx.x == 0) s_cnt[0] = 0;
        __syncthreads();
        int32_t* tail = out + above;
        for (int base = c0 + warp * 32; base < c1; base += blockDim.x) {
            const int i = base + lane;
            unsigned long long c = 0ull;
            if (i < c1) c = in_smem ? sc[i] : __ldcg(gc + i);
            const bool win = i < c1 && c >= thr;
            const int slot = warp_append(win, &s_cnt[0]);
            if (win && fin_base + slot < static_cast<int>(need)) tail[fin_base + slot] = composite_index(c);
        }
        nfin = max(0, min(nfin, static_cast<int>(need) - fin_base));
    }
    if (split == 0) {
        for (int i = ri.wcnt + ri.keff + threadIdx.x; i < kw; i += blockDim.x) idx[i] = -1;
        if (threadIdx.x == 0) a.cnt[row] = ri.wcnt + ri.keff;
    }
    __syncthreads();  // this CTA's final winners are written (read back by item_key)

    // ---------------------------------------------------------------- D: sparse attention over the work list
    {
        const int ntl = pre_tiles + (nfin + kKeyTile - 1) / kKeyTile;
        const PartialRef part{a.ps_ml + static_cast<int64_t>(split) * rows_q,
                              a.ps_acc + static_cast<int64_t>(split) * rows_q * D};
        const int g = lane >> 2, c = lane & 3;
        QTile<D> q;
        q.load(a.Qs, g < G ? row_q(g) * D : -1, g + 8 < G ? row_q(g + 8) * D : -1);
        OnlineSoftmax<D> st;
        st.init();
        for (int t = pre_staged; t < min(ntl, 2); ++t) stage_tile(t);
        for (int i = 0; i < ntl; ++i) {
            if (i + 1 < ntl && i + 1 >= 2) stage_tile(i + 1);  // keep one tile ahead
            if (i + 1 < ntl) cp_async_wait<1>(); else cp_async_wait<0>();
            __syncthreads();
            if (warp < NC) {
                const uint32_t kbase = smem_u32(ring + (i & 1) * kStageBytes);
                const uint32_t vbase = kbase + kKeyTile * D * 2;
                const int* slots = s_slot + (i & 1) * kKeyTile;
                float scv[KW / 8][4];
                qk_tile<D, KW>(q, kbase, warp * KW, scv);
                const int slot0 = warp * KW + 2 * c;
#pragma unroll
                for (int nn = 0; nn < KW / 8; ++nn)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        scv[nn][e] = slots[slot0 + nn * 8 + (e & 1)] >= 0 ? scv[nn][e] * at.scale_log2 : -INFINITY;
                st.template update<KW>(scv, vbase, warp * KW);
            }
            __syncthreads();
        }
        if (ntl == 0) {
            for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
                const int gg = e / D, dc = e % D;
                part.acc[row_q(gg) * D + dc] = 0.f;
                if (dc == 0) part.ml[row_q(gg)] = make_float2(-INFINITY, 0.f);
            }
        } else {
            if (warp < NC) st.finish_rows();
            float* red = reinterpret_cast<float*>(ring);
            if (warp < NC) stash_state<D, NC>(st, warp, red);
            __syncthreads();
            merge_states<D, NC>(red, threadIdx.x, blockDim.x, part,
                                [&](int r) -> int { return r < G ? static_cast<int>(row_q(r)) : -1; });
        }
    }
    if (!cta_barrier(bar, 4u * S, status, &s_flag)) return;  // B3: every sparse partial is written

    // ---------------------------------------------------------------- E: combines
    // split 0 merges the sparse partials of all G heads, split 1 (0 if S == 1) the full ones
    {
        float* s_w = reinterpret_cast<float*>(smem + kFusedRingOff);
        float2* s_ml = reinterpret_cast<float2*>(smem + kFusedRingOff + 16 * 256 * 4);
        if (split == 0)
            block_combine_rows<D, 16>(a.ps_ml, a.ps_acc, S, rows_q, row_q(0), 1, G, s_w, s_ml, a.O_sparse,
                                  a.LSE_sparse);
        if (split == (S > 1 ? 1 : 0))
            block_combine_rows<D, 16>(at.part_ml, at.part_acc, S, rows_q, row_q(0), 1, G, s_w, s_ml, a.O_full,
                                  a.LSE_full);
    }
}

cudaError_t launch_decode_step(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a,
                               cudaStream_t st) {
    void (*kern)(CUtensorMap, CUtensorMap, DecodeArgs) = nullptr;
#define HS2_DK(D_, G_) \
    if (p.d == D_ && p.G == G_) kern = decode_step_kernel<D_, G_>;
    HS2_DK(64, 1) HS2_DK(64, 2) HS2_DK(64, 4) HS2_DK(64, 8) HS2_DK(64, 16)
    HS2_DK(128, 1) HS2_DK(128, 2) HS2_DK(128, 4) HS2_DK(128, 8) HS2_DK(128, 16)
#undef HS2_DK
    if (!kern) return cudaErrorInvalidValue;
    const int stages = p.d == 128 ? 3 : 6;
    const int smem = stages * 2 * kKeyTile * p.d * 2 + 2 * stages * 8 + 16 + 128 * 4 + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const dim3 grid(p.S1, static_cast<unsigned>(p.rows_kv));
    if (static_cast<int64_t>(per_sm) * sms < static_cast<int64_t>(grid.x) * grid.y) return cudaErrorCooperativeLaunchTooLarge;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, tmK, tmV, a);
    if (e != cudaSuccess) {  // some drivers refuse the pair of attributes: keep the co-residency one
        (void)cudaGetLastError();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, tmK, tmV, a);
    }
    trace_mark("decode_step_fused", st);
    return e;
}

}  // namespace hs2
