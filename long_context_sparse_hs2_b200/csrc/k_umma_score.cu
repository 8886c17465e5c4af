// Selection-score sweep on the Blackwell tensor cores (tcgen05 / TMEM) for 128-row query tiles.
//
// The second K pass computes, for every query and pool key j <= pos - W, the GQA-max
// log-softmax score s_j = max over the G heads g of (logit_gj - LSE_g) in base-2 units and
// stores it as an order-preserving uint32 key for the top-k.  Here the product is taken
// transposed, S^T = K Q^T: the M dimension is 128 keys (one TMEM lane, one epilogue thread per
// key) and the N dimension the query-head rows of one or two query tiles (row = query * G +
// head, N = 128 or 256).  A thread then holds all G heads of every query for its key in its
// own registers, so the max over heads needs no shuffles, and the 32 threads of a warp write
// 32 consecutive keys of one query (128-byte stores).
//
// With x = q . k (the raw dot product), logit - LSE in base 2 is c * (x - u) for
// c = log2(e) / sqrt(d) and u = LSE * sqrt(d) (natural-log LSE).  The subtraction is folded
// into the MMA: one extra K step multiplies a constant key block (1, 1, 1, 0, ...) with a
// per-row block (-u split into three bf16 parts whose sum is u to about 24 bits), so TMEM
// already holds x - u and the epilogue is a max over heads and one scale per (query, key).
//
// Roles (576 threads): warps 0-15 are four epilogue warpgroups that split the columns of
// every tile between them (a quarter each); two TMEM accumulators (256 columns each) let the
// MMA of tile i + 1 run during the epilogue of tile i, and a warpgroup hands its accumulator
// back as soon as it has read its columns; warp 16 streams K tiles of 128 keys (3-stage TMA
// ring); warp 17 allocates TMEM and one of its lanes issues the MMAs.  Every wait is bounded; on expiry the CTA flags HS2_DEV_TIMEOUT, drains
// and exits.
#include "attn_sweep.cuh"
#include "topk_common.cuh"
#include "umma.cuh"

namespace hs2 {

namespace {

constexpr int kSTile = 128;      // keys per K tile (= TMEM lanes = M)
constexpr int kURowsPerTile = 128;  // query-head rows per query tile
constexpr int kSStages = 3;
constexpr int kSEpiWarps = 16;  // four epilogue warpgroups
constexpr int kSProducer = kSEpiWarps, kSMma = kSEpiWarps + 1;
constexpr int kSThreads = (kSEpiWarps + 2) * 32;
constexpr int kSMaxCols = 256;   // query-head rows per CTA (two query tiles)

template <int D>
struct SSmem {
    static constexpr int kQBytes = kSMaxCols * D * 2;    // both query tiles, [D/64][256 rows][128 B]
    static constexpr int kQHalf = kSMaxCols * 128;
    static constexpr int kTileBytes = kSTile * D * 2;
    static constexpr int kBlock = kSTile * 128;          // one 64-column block of a K tile
    static constexpr int kQOff = 0;
    static constexpr int kQcOff = kQBytes;               // -u parts per row: [256 rows][128 B] (16 B used)
    static constexpr int kKcOff = kQcOff + kSMaxCols * 128;  // ones per key: [128 keys][128 B]
    static constexpr int kKOff = kKcOff + kSTile * 128;
    static constexpr int kBarOff = kKOff + kSStages * kTileBytes;
    static constexpr int kNumBars = 2 * kSStages + 5;    // kfull, kempty, sfull[2], tfree[2], done
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kPlOff = kMiscOff + 16;         // last pool key per query (-1: not ranked)
    static constexpr int kThrOff = kPlOff + kSMaxCols * 4;  // filter mode: each query's score bound
    static constexpr int kCntOff = kThrOff + kSMaxCols * 4;  // filter mode: [warp][query] segment counts
    static constexpr int kBytes = kCntOff + kSEpiWarps * (kSMaxCols / 4) * 4 + 1024;
};

__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float max_nan3(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// NaN-propagating max of the G values v[0 .. G-1] (three-input maxes)
template <int G>
__device__ __forceinline__ float head_max(const float* v) {
    if constexpr (G == 1) {
        return v[0];
    } else if constexpr (G == 2) {
        return max_nan(v[0], v[1]);
    } else if constexpr (G == 4) {
        return max_nan(max_nan3(v[0], v[1], v[2]), v[3]);
    } else if constexpr (G == 8) {
        return max_nan3(max_nan3(v[0], v[1], v[2]), max_nan3(v[3], v[4], v[5]), max_nan(v[6], v[7]));
    } else {
        static_assert(G == 16, "G in {1, 2, 4, 8, 16}");
        const float a = max_nan3(max_nan3(v[0], v[1], v[2]), max_nan3(v[3], v[4], v[5]), max_nan3(v[6], v[7], v[8]));
        const float b = max_nan3(max_nan3(v[9], v[10], v[11]), max_nan3(v[12], v[13], v[14]), v[15]);
        return max_nan(a, b);
    }
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(r) : "f"(x));
    return static_cast<uint16_t>(r & 0xFFFFu);
}
__device__ __forceinline__ float bf16_value(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kSThreads, 1)
    umma_score_kernel(const __grid_constant__ CUtensorMap tmK, const AttnArgs a, const int split_keys) {
    using L = SSmem<D>;
    constexpr int TQ = kURowsPerTile / G;  // queries per query tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* kfull = bars;
    uint64_t* kempty = bars + kSStages;
    uint64_t* sfull = bars + 2 * kSStages;
    uint64_t* tfree = sfull + 2;
    uint64_t* done = sfull + 4;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    int* s_pl = reinterpret_cast<int*>(smem + L::kPlOff);
    float* s_thr = reinterpret_cast<float*>(smem + L::kThrOff);
    const int mode = a.score_mode;
    const int tstep = mode == 1 ? kSampleTileStride : 1;  // sample mode: one tile in kSampleTileStride

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();
    const int split = blockIdx.x, unit = blockIdx.y;
    const int QP = split_keys ? a.QB : (a.QB + 1) / 2;
    const int bh = unit / QP, pr = unit % QP;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const int nq = split_keys ? 1 : 2;
    const int ncols = nq * kURowsPerTile;

    // ---- prologue: per-query pool ends, query tiles and the constant key block (swizzled)
    for (int qa = tid; qa < nq * TQ; qa += kSThreads) {
        const int s = qa / TQ, tq = qa % TQ;
        const int qb = split_keys ? pr : 2 * pr + s;
        const int t = qb * TQ + tq;
        int pl = -1;
        if (qb < a.QB && t < a.T) {
            const int p = clamp_pos(a.pos[b * a.T + t], a.N, nullptr);
            const int P = max(0, p - a.W + 1);
            const int keff = min(a.k, P);
            if (keff > 0 && keff < P) pl = p - a.W;  // only these rows need ranked keys
        }
        s_pl[qa] = pl;
    }
    constexpr int CH = D / 8;
    for (int i = tid; i < nq * kURowsPerTile * CH; i += kSThreads) {
        const int R = i / CH, c = i % CH;  // R = s * 128 + r
        const int s = R / kURowsPerTile, r = R % kURowsPerTile;
        const int qb = split_keys ? pr : 2 * pr + s;
        const int tq = r / G, t = qb * TQ + tq;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (qb < a.QB && t < a.T) {
            const int64_t grow = static_cast<int64_t>((b * a.Hq + h * G + r % G)) * a.T + t;
            v = *reinterpret_cast<const uint4*>(a.Q + grow * D + c * 8);
        }
        *reinterpret_cast<uint4*>(smem + L::kQOff + (c >> 3) * L::kQHalf + R * 128 + (((c & 7) ^ (R & 7)) << 4)) = v;
    }
    for (int i = tid; i < kSTile * 8; i += kSThreads) {  // key block: elements 0..2 of every row are 1
        const int r = i >> 3, c = i & 7;
        const uint4 v = c == 0 ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + L::kKcOff + r * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
    if (tid == 0) {
        for (int i = 0; i < L::kNumBars; ++i) {
            const bool is_tfree = i >= 2 * kSStages + 2 && i < 2 * kSStages + 4;
            mbar_init(&bars[i], is_tfree ? kSEpiWarps * 32 : 1);  // tfree: one arrival per epilogue thread
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    pdl_wait();  // LSE_full comes from the previous kernel; TMEM only after it has completed
    if (mode == 2) {
        // The bracket of every query's selection row (the bracket kernel's bucket b_hi) as a bound
        // on the score itself: score_bin(key(s)) <= b_hi exactly when s > -F, F the float whose
        // bits are (b_hi + 1) << 15 above the first bucket's (see score_bin).  b_hi = the last
        // bucket takes every key except NaN and -inf, which rank below all others.
        for (int qa = tid; qa < nq * TQ; qa += kSThreads) {
            const int s = qa / TQ, tq = qa % TQ;
            const int qb = split_keys ? pr : 2 * pr + s;
            const int t = qb * TQ + tq;
            float thr = INFINITY;
            if (s_pl[qa] >= 0) {
                const int bhi = a.meta[(static_cast<int64_t>(bh) * a.T + t) * kMetaInts + kMetaBin];
                if (bhi >= kHistBins - 1)
                    thr = -INFINITY;
                else if (bhi >= 0)
                    thr = -__uint_as_float(static_cast<uint32_t>(bhi + (125 << 8) + 1) << 15);
            }
            s_thr[qa] = thr;
        }
    }
    __syncthreads();  // s_pl (and s_bhi) complete
    const float sqrt_d = sqrtf(static_cast<float>(D));
    for (int i = tid; i < kSMaxCols * 8; i += kSThreads) {  // row block: -u as hi + mid + lo
        const int R = i >> 3, c = i & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c == 0 && R < ncols) {
            const int s = R / kURowsPerTile, r = R % kURowsPerTile;
            const int qa = s * TQ + r / G;
            if (s_pl[qa] >= 0) {  // unranked and padding rows keep u = 0: never written
                const int qb = split_keys ? pr : 2 * pr + s;
                const int t = qb * TQ + r / G;
                const float nu = -a.lse[static_cast<int64_t>(b * a.Hq + h * G + r % G) * a.T + t] * sqrt_d;
                const uint16_t hi = bf16_bits_rn(nu);
                const float r1 = nu - bf16_value(hi);
                const uint16_t mid = bf16_bits_rn(r1);
                const uint16_t lo = bf16_bits_rn(r1 - bf16_value(mid));
                v = make_uint4(static_cast<uint32_t>(hi) | (static_cast<uint32_t>(mid) << 16), lo, 0u, 0u);
            }
        }
        *reinterpret_cast<uint4*>(smem + L::kQcOff + R * 128 + ((c ^ (R & 7)) << 4)) = v;
    }
    fence_async_smem();
    if (warp == kSMma) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;

    int jmax = -1;
    for (int qa = 0; qa < nq * TQ; ++qa) jmax = max(jmax, s_pl[qa]);
    // tiles (of the sample in sample mode: tile v stands for key tile v * tstep)
    const int ntiles = jmax >= 0 ? ((jmax + kSTile) / kSTile + tstep - 1) / tstep : 0;
    const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.S);
    const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.S);
    const int nt = t_end - t_begin;

    bool nonfinite = false;
    if (warp == kSProducer) {
        // ------------------------------------------------------------ TMA producer (K only)
        if (lane == 0) {
            const uint64_t pol = a.stream_kv ? l2_evict_first() : l2_evict_normal();
            prefetch_tensormap(&tmK);
            int issued = 0;
            for (int q = 0; q < nt; ++q) {
                const int st = q % kSStages;
                if (q >= kSStages && !mbar_wait(&kempty[st], ((q / kSStages) - 1) & 1, a.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&kfull[st], L::kTileBytes);
#pragma unroll
                for (int hb = 0; hb < D / 64; ++hb)
                    tma_load_3d(smem + L::kKOff + st * L::kTileBytes + hb * L::kBlock, &tmK, &kfull[st], hb * 64,
                                (t_begin + q) * tstep * kSTile, bh, pol);
                ++issued;
            }
            for (int st = 0; st < kSStages && st < issued; ++st) {
                const int last = st + ((issued - 1 - st) / kSStages) * kSStages;
                mbar_wait(&kfull[st], (last / kSStages) & 1, a.status);
            }
        }
        __syncwarp();
    } else if (warp == kSMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kSTile, ncols, false);
            const uint32_t qb0 = smem_u32(smem + L::kQOff);
            const uint32_t kb0 = smem_u32(smem + L::kKOff);
            const uint64_t kc_desc = sw128_desc(smem_u32(smem + L::kKcOff), 16, 1024);
            const uint64_t qc_desc = sw128_desc(smem_u32(smem + L::kQcOff), 16, 1024);
            bool ok = true;
            for (int i = 0; ok && i < nt; ++i) {
                const int st = i % kSStages, buf = i & 1;
                ok = !*abort_flag && mbar_wait(&kfull[st], (i / kSStages) & 1, a.status);
                if (ok && i >= 2) ok = mbar_wait(&tfree[buf], ((i >> 1) - 1) & 1, a.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kb = kb0 + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * L::kBlock + (kk & 3) * 32;
                    const uint32_t qoff = (kk >> 2) * L::kQHalf + (kk & 3) * 32;
                    umma_ss(tm + 256 * buf, sw128_desc(kb + koff, 16, 1024), sw128_desc(qb0 + qoff, 16, 1024), idesc,
                            kk > 0);
                }
                umma_ss(tm + 256 * buf, kc_desc, qc_desc, idesc, 1u);  // - u
                umma_commit(&kempty[st]);
                umma_commit(&sfull[buf]);
            }
            if (!ok) *abort_flag = 1;
            umma_commit(done);
            mbar_wait(done, 0, a.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (thread = key)
        const int w = warp >> 2, quarter = warp & 3;  // warpgroup, TMEM lane quarter
        const int r = quarter * 32 + lane;
        const int wcols = ncols / (kSEpiWarps / 4);  // columns of this warpgroup: a quarter of the tile
        const int col0 = w * wcols;
        const int s = col0 / kURowsPerTile;    // query tile of these columns
        const int qa0 = col0 / G, nqw = wcols / G;
        const int qb = split_keys ? pr : 2 * pr + s;
        // selection row of query qa0 + i is row0 + i (valid queries only; the others are never written)
        const int64_t row0 = static_cast<int64_t>(bh) * a.T + qb * TQ + (qa0 - s * TQ);
        int plmin = INT_MAX;
        for (int i = 0; i < nqw; ++i) plmin = min(plmin, s_pl[qa0 + i]);  // -1 if any is not ranked
        const uint32_t tbase = tm + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
        const float c2 = a.scale_log2;
        // filter mode: this warp's segment (split, lane quarter) of every query's list, and its
        // running counts (registers for G >= 4, shared memory otherwise)
        int* s_cnt = reinterpret_cast<int*>(smem + L::kCntOff) + warp * (kSMaxCols / 4);
        unsigned long long* seg = a.cand + (split * 4 + quarter) * a.seg_cap;
        constexpr bool kRegCnt = G >= 4;
        int qcnt[2][32 / G];
#pragma unroll
        for (int cq = 0; cq < 2; ++cq)
#pragma unroll
            for (int qq = 0; qq < 32 / G; ++qq) qcnt[cq][qq] = 0;
        if (mode == 2 && !kRegCnt) {
            for (int i = lane; i < nqw; i += 32) s_cnt[i] = 0;
            __syncwarp();
        }
        // filter mode, G >= 8: the warp's query bounds in registers (the same for every tile)
        constexpr bool kRegThr = G >= 8;
        float qthr[2][32 / G];
#pragma unroll
        for (int cq = 0; cq < 2; ++cq)
#pragma unroll
            for (int qq = 0; qq < 32 / G; ++qq) {
                const int ql = (32 * cq) / G + qq;
                qthr[cq][qq] = (kRegThr && mode == 2 && ql < nqw) ? s_thr[qa0 + ql] : INFINITY;
            }
        for (int i = 0; i < nt; ++i) {
            const int buf = i & 1;
            const bool got = mbar_wait(&sfull[buf], (i >> 1) & 1, a.status);
            if (!got) *abort_flag = 1;
            if (!__all_sync(0xffffffffu, got && !*abort_flag)) break;
            tc_fence_after();
            const int jt = (t_begin + i) * tstep * kSTile;  // first key of the tile
            const int j = jt + r;
            const bool fast = jt + kSTile - 1 <= plmin;  // every query of these columns takes every key
            // sample mode stores the tile compactly (tile i of the sample at i * 128)
            uint32_t* kp = a.keys + row0 * a.kstride + (mode == 1 ? (t_begin + i) * kSTile + r : j);
            // read all of this warpgroup's columns, then hand the accumulator back to the MMA
            // before the max / key conversion / stores
            uint32_t x[2][32];
            tmem_ld32(tbase + 256 * buf, x[0]);
            if (wcols > 32) tmem_ld32(tbase + 256 * buf + 32, x[1]);
            tmem_wait_ld();
            tie_regs(x[0]);
            tie_regs(x[1]);
            tc_fence_before();
            mbar_arrive(&tfree[buf]);
#pragma unroll
            for (int cq = 0; cq < 2; ++cq) {
                if (32 * cq >= wcols) break;
                // max over the G heads of each query (three-input maxes, independent queries)
                float m[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) m[e] = __uint_as_float(x[cq][e]);
                float sv[32 / G];
#pragma unroll
                for (int qq = 0; qq < 32 / G; ++qq) {
                    sv[qq] = head_max<G>(m + qq * G) * c2;
                    // only keys that are stored count (past a query's pool the slot may hold anything)
                    nonfinite |= (sv[qq] != sv[qq]) && (fast || j <= s_pl[qa0 + (32 * cq) / G + qq]);
                }
                if (mode == 2) {
                    // each query's keys above its score bound go to this warp's own segment of the
                    // query's candidate list (a running count per warp and query: no atomics)
#pragma unroll
                    for (int qq = 0; qq < 32 / G; ++qq) {
                        const int ql = (32 * cq) / G + qq;  // query of the warpgroup
                        const float thr = kRegThr ? qthr[cq][qq] : s_thr[qa0 + ql];
                        const bool take = sv[qq] > thr && (fast || j <= s_pl[qa0 + ql]);
                        const unsigned bal = __ballot_sync(0xffffffffu, take);
                        if (bal == 0u) continue;
                        const int c0 = kRegCnt ? qcnt[cq][qq] : s_cnt[ql];
                        const int slot = c0 + __popc(bal & ((1u << lane) - 1u));
                        if (take && slot < a.seg_cap)
                            seg[(row0 + ql) * a.cand_cap + slot] = composite(score_key(sv[qq]), j);
                        if (kRegCnt) {
                            qcnt[cq][qq] = c0 + __popc(bal);
                        } else {
                            __syncwarp();
                            if (lane == 0) s_cnt[ql] = c0 + __popc(bal);
                            __syncwarp();
                        }
                    }
                    continue;
                }
                uint32_t key[32 / G];
#pragma unroll
                for (int qq = 0; qq < 32 / G; ++qq) key[qq] = score_key(sv[qq]);
                uint32_t* kq = kp + static_cast<int64_t>((32 * cq) / G) * a.kstride;
                if (fast) {  // every query of these columns takes this key
#pragma unroll
                    for (int qq = 0; qq < 32 / G; ++qq) __stcs(kq + static_cast<int64_t>(qq) * a.kstride, key[qq]);
                } else {
#pragma unroll
                    for (int qq = 0; qq < 32 / G; ++qq)
                        if (j <= s_pl[qa0 + (32 * cq) / G + qq]) __stcs(kq + static_cast<int64_t>(qq) * a.kstride, key[qq]);
                }
            }
        }
        if (mode == 2) {  // the segment counts of the ranked queries
            if (kRegCnt) {
                if (lane == 0) {
#pragma unroll
                    for (int cq = 0; cq < 2; ++cq)
#pragma unroll
                        for (int qq = 0; qq < 32 / G; ++qq) {
                            const int ql = (32 * cq) / G + qq;
                            if (ql < nqw && s_pl[qa0 + ql] >= 0)
                                a.segcnt[(row0 + ql) * (4 * a.S) + split * 4 + quarter] = qcnt[cq][qq];
                        }
                }
            } else {
                __syncwarp();
                for (int i = lane; i < nqw; i += 32)
                    if (s_pl[qa0 + i] >= 0) a.segcnt[(row0 + i) * (4 * a.S) + split * 4 + quarter] = s_cnt[i];
            }
        }
    }

    tc_fence_before();
    if (__syncthreads_or(nonfinite) && tid == 0) set_status(a.status, HS2_DEV_NONFINITE);
    if (warp == kSMma) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// ====================================================================== launcher

template <int D, int G>
cudaError_t umma_score_variant(const Plan& p, const CUtensorMap& tmK, const AttnArgs& a, cudaStream_t st) {
    using L = SSmem<D>;
    auto kern = umma_score_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    const int split_keys = p.umma_split_keys ? 1 : 0;
    const int QP = split_keys ? p.QB : (p.QB + 1) / 2;
    dim3 grid(p.SS, p.B * p.Hkv * QP);
    AttnArgs x = a;
    x.S = p.SS;
    e = launch_pdl(kern, grid, dim3(kSThreads), L::kBytes, st, tmK, x, split_keys);
    trace_mark(a.score_mode == 1 ? "umma_score_sample" : (a.score_mode == 2 ? "umma_score_filter" : "umma_score"), st);
    return e;
}

cudaError_t launch_umma_score(const Plan& p, const CUtensorMap& tmK, const AttnArgs& a, cudaStream_t st) {
#define HS2_US(D_, G_) \
    if (p.d == D_ && p.G == G_) return umma_score_variant<D_, G_>(p, tmK, a, st);
    HS2_US(128, 1) HS2_US(128, 2) HS2_US(128, 4) HS2_US(128, 8) HS2_US(128, 16)
    HS2_US(64, 1) HS2_US(64, 2) HS2_US(64, 4) HS2_US(64, 8) HS2_US(64, 16)
#undef HS2_US
    return cudaErrorInvalidValue;
}

}  // namespace hs2
