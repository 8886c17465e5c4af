// The full-attention sweep of one CTA (sm_100a), and the TMA producer the score sweep shares.
//
// Split-K flash-decode: a CTA owns one row block (the G query heads of one kv head for TQ
// consecutive queries = 16*RT MMA rows) and one contiguous range of 64-key tiles.  A
// producer warp streams K and V tiles into a STAGES-deep shared-memory ring with TMA (3-D
// tensor map, 128-byte swizzle, no multicast), signalled through mbarriers with bounded
// waits; NC consumer warps compute QK^T and PV with bf16 mma.sync and keep an online softmax
// in base-2 units.  Each CTA writes one split partial (m, l, O) per row; the partials merge
// with the log-sum-exp correction ("Simplified Sparse Attention via Gist Tokens", section
// 3.6, "three-kernel split-K sparse flash-decode").  With KEEP_LOGITS the sweep also stores
// every visible base-2 logit, [row][key][head], so the selection score can be formed
// without reading K a second time.
#pragma once

#include "attn_core_t.cuh"

namespace hs2 {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ int clamp_pos(int p, int N, unsigned* status) {
    if (p < 0 || p >= N) {
        if (status) {
            pdl_wait();  // the status word is cleared by the call's first kernel
            set_status(status, HS2_DEV_BAD_POS);
        }
        p = p < 0 ? 0 : N - 1;
    }
    return p;
}

// Shared-memory layout of the streaming kernels (after 1 KB alignment).  EB: bytes per cache
// element (2 for bf16, 1 for FP8 E4M3).
template <int D, int STAGES, int TENSORS, int EB = 2>
struct StreamSmem {
    static constexpr int kTileBytes = kKeyTile * D * EB;                // one tensor, one tile
    static constexpr int kStageBytes = TENSORS * kTileBytes;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kBarOff = kRingBytes;                           // full[STAGES], empty[STAGES]
    static constexpr int kMiscOff = kBarOff + 2 * STAGES * 8;            // abort flag + row positions
    static constexpr int kTileOff = kMiscOff + 16 + 128 * 4;           // key tile of each stage (dynamic sweep)
    static constexpr int kBytes = kTileOff + 16 * 4 + 1024;              // + alignment slack
};

// Issues the TMA loads of one tile (keys j0 .. j0 + 63 of kv slice bh = b*Hkv + h) of one tensor
// into dst, completing on bar.  Contiguous caches take one 3-D box per 64-dim half (bf16) or one
// box (FP8); a paged pool takes one 4-D box per page the tile touches (per half for bf16), at the
// page's slot range.  Page ids come from the page table; one outside [0, num_pages), or a page
// index past the table's row, loads zeros and flags HS2_DEV_BAD_PAGE (keys past pos are never
// used, so the tail of a row's last tile may be unmapped).
template <int D, bool FP8>
__device__ __forceinline__ void load_kv_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, const KvSrc& kv,
                                             int j0, int bh, int Hkv, uint64_t pol, unsigned* status) {
    constexpr int kHalves = FP8 ? 1 : D / 64;
    constexpr int kRowBytes = FP8 ? D : 128;    // bytes of one key row inside a half
    constexpr int kHalfBytes = kKeyTile * kRowBytes;
    if (kv.page_shift < 0) {
#pragma unroll
        for (int hb = 0; hb < kHalves; ++hb) tma_load_3d(dst + hb * kHalfBytes, map, bar, hb * 64, j0, bh, pol);
        return;
    }
    const int ps = 1 << kv.page_shift;
    const int box = ps < kKeyTile ? ps : kKeyTile;
    const int b = bh / Hkv, h = bh % Hkv;
    for (int r = 0; r < kKeyTile; r += box) {
        const int j = j0 + r;
        const int pi = j >> kv.page_shift;
        int page = pi < kv.max_pages ? kv.page_table[static_cast<int64_t>(b) * kv.max_pages + pi] : -1;
        if (page < 0 || page >= kv.num_pages) {
            if (pi < kv.max_pages) {
                pdl_wait();  // the status word is cleared by the call's first kernel
                set_status(status, HS2_DEV_BAD_PAGE);
            }
            page = -1;  // whole box out of range: zeros
        }
#pragma unroll
        for (int hb = 0; hb < kHalves; ++hb)
            tma_load_4d(dst + hb * kHalfBytes + r * kRowBytes, map, bar, hb * 64, j & (ps - 1), h, page, pol);
    }
}

// Producer side of the TMA ring: stream tiles [t_begin, t_begin + nt) of kv slice bh.
template <int D, int STAGES, int TENSORS, bool FP8>
__device__ void produce_tiles(const CUtensorMap* tmK, const CUtensorMap* tmV, uint8_t* ring, uint64_t* full,
                              uint64_t* empty, volatile int* abort_flag, int t_begin, int nt, int bh, int Hkv,
                              const KvSrc& kv, unsigned* status, bool stream) {
    using L = StreamSmem<D, STAGES, TENSORS, FP8 ? 1 : 2>;
    const uint64_t pol = stream ? l2_evict_first() : l2_evict_normal();
    prefetch_tensormap(tmK);
    if (TENSORS == 2) prefetch_tensormap(tmV);
    int issued = 0;
    for (int i = 0; i < nt; ++i) {
        const int stage = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[stage], ((i / STAGES) - 1) & 1, status)) {
            *abort_flag = 1;
            break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
        const int j0 = (t_begin + i) * kKeyTile;
        uint8_t* dst = ring + stage * L::kStageBytes;
        load_kv_tile<D, FP8>(dst, tmK, &full[stage], kv, j0, bh, Hkv, pol, status);
        if (TENSORS == 2) load_kv_tile<D, FP8>(dst + L::kTileBytes, tmV, &full[stage], kv, j0, bh, Hkv, pol, status);
        ++issued;
    }
    // Drain: wait (bounded) for the last load issued into every stage, so no copy is still
    // landing in shared memory when the CTA retires (matters only after an abort).
    for (int st = 0; st < STAGES && st < issued; ++st) {
        const int last = st + ((issued - 1 - st) / STAGES) * STAGES;
        mbar_wait(&full[st], (last / STAGES) & 1, status);
    }
}


// Producer side of the dynamically scheduled sweep: the CTAs of a row block take chunks of
// `chunk` consecutive key tiles of [0, ntiles) from the counter ctr (one atomic per chunk, the next
// chunk taken while the current one is loading), so that a CTA that finishes early takes more
// and all of them end together.  The tile of each stage goes to s_tile[stage] before its loads;
// a final stage with no loads and tile -1 tells the consumers to stop.
template <int D, int STAGES, bool FP8>
__device__ void produce_tiles_dyn(const CUtensorMap* tmK, const CUtensorMap* tmV, uint8_t* ring, uint64_t* full,
                                  uint64_t* empty, volatile int* abort_flag, int* s_tile, int* ctr, int ntiles,
                                  int chunk, int bh, int Hkv, const KvSrc& kv, unsigned* status, bool stream) {
    using L = StreamSmem<D, STAGES, 2, FP8 ? 1 : 2>;
    const uint64_t pol = stream ? l2_evict_first() : l2_evict_normal();
    prefetch_tensormap(tmK);
    prefetch_tensormap(tmV);
    int i = 0, issued = 0;
    bool ok = true;
    pdl_wait();  // the counter is cleared by the call's first kernel
    int cur = atomicAdd(ctr, chunk);
    // (the counter only grows from 0, so a CTA never takes more than ntiles tiles; the bound on
    // issued makes that explicit)
    while (ok && cur >= 0 && cur < ntiles && issued < ntiles) {
        const int nxt = atomicAdd(ctr, chunk);
        const int end = min(cur + chunk, ntiles);
        for (int t = cur; t < end; ++t, ++i) {
            const int stage = i % STAGES;
            if ((i >= STAGES && !mbar_wait(&empty[stage], ((i / STAGES) - 1) & 1, status)) || *abort_flag) {
                *abort_flag = 1;
                ok = false;
                break;
            }
            s_tile[stage] = t;
            mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
            uint8_t* dst = ring + stage * L::kStageBytes;
            load_kv_tile<D, FP8>(dst, tmK, &full[stage], kv, t * kKeyTile, bh, Hkv, pol, status);
            load_kv_tile<D, FP8>(dst + L::kTileBytes, tmV, &full[stage], kv, t * kKeyTile, bh, Hkv, pol, status);
            ++issued;
        }
        cur = nxt;
    }
    // drain: the last load issued into every stage has landed before the CTA retires (done before
    // the end marker, whose plain arrive completes one more phase of its stage's barrier)
    for (int st = 0; st < STAGES && st < issued; ++st) {
        const int last = st + ((issued - 1 - st) / STAGES) * STAGES;
        mbar_wait(&full[st], (last / STAGES) & 1, status);
    }
    if (ok) {  // the end marker
        const int stage = i % STAGES;
        if (i < STAGES || mbar_wait(&empty[stage], ((i / STAGES) - 1) & 1, status)) {
            s_tile[stage] = -1;
            mbar_arrive(&full[stage]);
        } else {
            *abort_flag = 1;
        }
    }
}

// One CTA's share of the full-attention sweep: row block `unit`, split `split`.  Streams the
// split's K/V tiles through the TMA ring, keeps the online softmax, optionally stores the
// base-2 logits, and writes the split partial of every row of the block.  Returns false if a
// pipeline wait ran out (HS2_DEV_TIMEOUT is then set).  *t_range receives the tile range.
// Ends with the block synchronised; the ring is free again afterwards.  TR (RT = 1, at most 8
// query-head rows in the block): the transposed warp attention of attn_core_t.cuh.  DYN: the
// split's tiles are not a fixed range but chunks taken from a.tilectr[unit] (produce_tiles_dyn);
// *t_range is then empty.
template <int D, int RT, int NC, int STAGES, bool KEEP_LOGITS, bool FP8, bool TR = false, bool DYN = false>
__device__ __forceinline__ bool full_sweep(const CUtensorMap* tmK, const CUtensorMap* tmV, const AttnArgs& a,
                                           uint8_t* smem, int split, int unit, int2* t_range) {
    constexpr int NKS = NC / RT;          // warps sharing one row tile (each a key slice)
    constexpr int KW = kKeyTile / NKS;    // keys per warp per tile
    static_assert(NC % RT == 0 && KW % 16 == 0, "bad warp split");
    static_assert(!TR || (RT == 1 && KW == 16 && NC / RT > 1), "transposed form: one 16-key slice per warp");
    using L = StreamSmem<D, STAGES, 2, FP8 ? 1 : 2>;
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff);
    int* s_pos = reinterpret_cast<int*>(smem + L::kMiscOff + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = unit / a.QB, qb = unit % a.QB;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    for (int r = tid; r < 16 * RT; r += blockDim.x) {
        const int tq = r / a.G, t = qb * a.TQ + tq;
        s_pos[r] = (tq < a.TQ && t < a.T) ? clamp_pos(a.pos[b * a.T + t], a.N, a.status) : -1;
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    int jmax = -1;
    for (int r = 0; r < 16 * RT; ++r) jmax = max(jmax, s_pos[r]);
    const int ntiles = jmax >= 0 ? (jmax + kKeyTile) / kKeyTile : 0;
    const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.S);
    const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.S);
    const int nt = t_end - t_begin;
    *t_range = DYN ? make_int2(0, 0) : make_int2(t_begin, t_end);
    int* s_tile = reinterpret_cast<int*>(smem + L::kTileOff);
    // the key tile of step i: fixed range, or what the producer put in the stage (-1: the end)
    auto tile_of = [&](int i, int stage) -> int { return DYN ? s_tile[stage] : t_begin + i; };

    typename std::conditional<TR, OnlineSoftmaxT<D, FP8>, OnlineSoftmax<D, FP8>>::type st;
    st.init();
    const int rt = warp % RT, ks = warp / RT;
    const int g = lane >> 2, c = lane & 3;
    const int r_lo = rt * 16 + g, r_hi = r_lo + 8;
    auto row_q = [&](int r) -> int {  // global query-head row of local row r, or -1
        const int tq = r / a.G, t = qb * a.TQ + tq;
        if (tq >= a.TQ || t >= a.T) return -1;
        return (b * a.Hq + h * a.G + (r % a.G)) * a.T + t;
    };

    const float kscale = FP8 ? a.kv.k_scale[bh] : 1.f;
    const float vscale = FP8 ? a.kv.v_scale[bh] : 1.f;
    if (warp == NC) {
        if (lane == 0) {
            if (DYN)
                produce_tiles_dyn<D, STAGES, FP8>(tmK, tmV, ring, full, empty, abort_flag, s_tile, a.tilectr + unit,
                                                  ntiles, max(1, ntiles / (a.S * 8)), bh, a.Hkv, a.kv, a.status,
                                                  a.stream_kv != 0);
            else
                produce_tiles<D, STAGES, 2, FP8>(tmK, tmV, ring, full, empty, abort_flag, t_begin, nt, bh, a.Hkv,
                                                 a.kv, a.status, a.stream_kv != 0);
        }
        __syncwarp();
    } else if constexpr (TR) {
        // query rows 0..7: lane (g, c) loads row g of Q and scores rows 2c, 2c+1
        QTileT<D, FP8> q;
        const int rq = row_q(g);
        q.load(a.Q, rq >= 0 ? static_cast<int64_t>(rq) * D : -1);
        const float f0 = a.scale_log2 * kscale * q.col_scale[0];
        const float f1 = a.scale_log2 * kscale * q.col_scale[1];
        const int p0 = s_pos[2 * c], p1 = s_pos[2 * c + 1];
        const int key0 = ks * KW;
        float* lg0 = nullptr;
        float* lg1 = nullptr;
        const uint64_t keep = l2_evict_last();
        if (KEEP_LOGITS) {
            // [row_kv][N][G]: row_kv = (b*Hkv + h)*T + t
            if (p0 >= 0) lg0 = a.logits + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + (2 * c) / a.G) * a.N * a.G + (2 * c) % a.G;
            if (p1 >= 0)
                lg1 = a.logits + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + (2 * c + 1) / a.G) * a.N * a.G + (2 * c + 1) % a.G;
        }
        for (int i = 0; DYN || i < nt; ++i) {
            const int stage = i % STAGES;
            if (!mbar_wait(&full[stage], (i / STAGES) & 1, a.status)) {
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            const uint32_t kbase = smem_u32(ring + stage * L::kStageBytes);
            const uint32_t vbase = kbase + L::kTileBytes;
            const int tile = tile_of(i, stage);
            if (tile < 0) break;  // the end marker of the dynamic sweep
            const int tile_j0 = tile * kKeyTile;
            const bool past_end = tile_j0 + key0 + KW - 1 > jmax;
            if (past_end) {  // as below: zero this warp's V rows of keys past the CTA's last position
                constexpr int CH = D * (FP8 ? 1 : 2) / 16;
                uint8_t* vtile = ring + stage * L::kStageBytes + L::kTileBytes;
                for (int e = lane; e < KW * CH; e += 32) {
                    const int r = key0 + e / CH;
                    if (tile_j0 + r > jmax)
                        *reinterpret_cast<uint4*>(vtile + kv_chunk_offset<D, FP8>(r, e % CH)) = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            float sc[4];
            qk_t<D, FP8>(q, kbase, key0, sc);
            const int j_lo = tile_j0 + key0 + g, j_hi = j_lo + 8;
            sc[0] = j_lo <= p0 ? sc[0] * f0 : -INFINITY;
            sc[1] = j_lo <= p1 ? sc[1] * f1 : -INFINITY;
            sc[2] = j_hi <= p0 ? sc[2] * f0 : -INFINITY;
            sc[3] = j_hi <= p1 ? sc[3] * f1 : -INFINITY;
            if (KEEP_LOGITS) {
                if (j_lo <= p0) st_f32_policy(lg0 + static_cast<int64_t>(j_lo) * a.G, sc[0], keep);
                if (j_lo <= p1) st_f32_policy(lg1 + static_cast<int64_t>(j_lo) * a.G, sc[1], keep);
                if (j_hi <= p0) st_f32_policy(lg0 + static_cast<int64_t>(j_hi) * a.G, sc[2], keep);
                if (j_hi <= p1) st_f32_policy(lg1 + static_cast<int64_t>(j_hi) * a.G, sc[3], keep);
            }
            st.update(sc, vbase, key0);
            if (past_end) fence_async_smem();  // the zeros are ordered before the next TMA write
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
        st.finish_rows();
    } else {
        QTileOf<D, FP8> q;
        const int rq_lo = row_q(r_lo), rq_hi = row_q(r_hi);
        q.load(a.Q, rq_lo >= 0 ? static_cast<int64_t>(rq_lo) * D : -1, rq_hi >= 0 ? static_cast<int64_t>(rq_hi) * D : -1);
        const float f_lo = logit_factor<D, FP8>(q, 0, a.scale_log2, kscale);
        const float f_hi = logit_factor<D, FP8>(q, 1, a.scale_log2, kscale);
        const int p_lo = s_pos[r_lo], p_hi = s_pos[r_hi];
        const int key0 = ks * KW;
        float* lg_lo = nullptr;
        float* lg_hi = nullptr;
        const uint64_t keep = l2_evict_last();
        if (KEEP_LOGITS) {
            // [row_kv][N][G]: row_kv = (b*Hkv + h)*T + t
            if (p_lo >= 0)
                lg_lo = a.logits + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + r_lo / a.G) * a.N * a.G + (r_lo % a.G);
            if (p_hi >= 0)
                lg_hi = a.logits + (static_cast<int64_t>(bh) * a.T + qb * a.TQ + r_hi / a.G) * a.N * a.G + (r_hi % a.G);
        }
        for (int i = 0; DYN || i < nt; ++i) {
            const int stage = i % STAGES;
            if (!mbar_wait(&full[stage], (i / STAGES) & 1, a.status)) {
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            const uint32_t kbase = smem_u32(ring + stage * L::kStageBytes);
            const uint32_t vbase = kbase + L::kTileBytes;
            const int tile = tile_of(i, stage);
            if (tile < 0) break;  // the end marker of the dynamic sweep
            const int tile_j0 = tile * kKeyTile;
            const bool past_end = tile_j0 + key0 + KW - 1 > jmax;
            if (past_end) {
                // Keys past the CTA's last position are masked (P = 0), but their cache slots may hold
                // anything (an unwritten cache, a paged pool's unused slots): 0 x NaN would poison O.
                // Zero this warp's V rows there; only the warp itself reads them.
                constexpr int CH = D * (FP8 ? 1 : 2) / 16;
                uint8_t* vtile = ring + stage * L::kStageBytes + L::kTileBytes;
                for (int e = lane; e < KW * CH; e += 32) {
                    const int r = key0 + e / CH;
                    if (tile_j0 + r > jmax)
                        *reinterpret_cast<uint4*>(vtile + kv_chunk_offset<D, FP8>(r, e % CH)) = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            float sc[KW / 8][4];
            qk_any<D, KW, FP8>(q, kbase, key0, sc);
            const int jb = tile_j0 + key0 + 2 * c;
#pragma unroll
            for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = jb + n * 8 + (e & 1);
                    const int p = (e < 2) ? p_lo : p_hi;
                    const float v = sc[n][e] * ((e < 2) ? f_lo : f_hi);
                    sc[n][e] = (j <= p) ? v : -INFINITY;
                    if (KEEP_LOGITS && j <= p) {
                        float* lg = (e < 2) ? lg_lo : lg_hi;
                        st_f32_policy(lg + static_cast<int64_t>(j) * a.G, v, keep);
                    }
                }
            }
            st.template update<KW>(sc, vbase, key0);
            if (past_end) fence_async_smem();  // the zeros are ordered before the next TMA write
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
        st.finish_rows();
    }
    __syncthreads();
    if (*abort_flag) return false;

    const PartialRef out{a.part_ml + static_cast<int64_t>(split) * (a.B * a.Hq * a.T),
                         a.part_acc + static_cast<int64_t>(split) * (a.B * a.Hq * a.T) * D};
    if constexpr (NKS == 1 && !TR) {
        if (warp < NC) store_partial<D, FP8>(st, out, [&](int r) { return row_q(rt * 16 + r); }, vscale);
    } else {
        float* red = reinterpret_cast<float*>(ring);  // the ring is idle now
        if (warp < NC) {
            if constexpr (TR)
                stash_state_t<D, NKS, FP8>(st, ks, red + rt * merge_floats<D, NKS>(), vscale);
            else
                stash_state<D, NKS, FP8>(st, ks, red + rt * merge_floats<D, NKS>(), vscale);
        }
        __syncthreads();
        // threads of the CTA split evenly over the RT tiles
        const int per = blockDim.x / RT;
        const int my_rt = tid / per;
        if (my_rt < RT)
            merge_states<D, NKS>(red + my_rt * merge_floats<D, NKS>(), tid - my_rt * per, per, out,
                                 [&](int r) { return row_q(my_rt * 16 + r); });
    }
    __syncthreads();
    return true;
}


}  // namespace hs2
