// Full-attention sweep on the Blackwell tensor cores (tcgen05 / TMEM) for 128-row query tiles:
// the chunked-prefill and multi-query decode shapes, where Q K^T and P V are dense
// contractions.
//
// A query tile holds the G query heads of one kv head for 128 / G consecutive queries (row
// r = query * G + head), the same row blocks as the mma.sync sweep with RT = 8.  One CTA runs
// two independent "streams", each an online softmax over 128-key tiles with its own TMEM
// accumulators, so that the tensor core works on one stream while the other stream's softmax
// runs:
//   pair mode   two consecutive query tiles share one stream of K/V tiles (chunked prefill:
//               every K/V tile loaded once feeds 256 rows);
//   split mode  one query tile; stream 0 takes the even and stream 1 the odd K/V tiles of the
//               CTA's key range (few query tiles, e.g. 16 decode queries), and each stream
//               writes its own split partial.
//
// Roles (384 threads):
//   warps 0-3   softmax of stream 0 (thread = TMEM lane = tile row), warps 4-7 stream 1
//   warp 8      TMA producer: K and V tiles of 128 keys into two 2-stage rings
//   warp 9      allocates TMEM; one lane issues every tcgen05.mma and commit
//   warps 10-11 zero the V rows of keys past the CTA's last position in its last tile (when
//               that tile reaches past it); with warps 8 and 9 they form the warpgroup that
//               hands registers to the softmax warpgroups (setmaxnreg)
// TMEM (512 columns): stream s has S at columns 256s .. 256s+127 (fp32 logits; the bf16
// probabilities P overwrite its first 64 columns) and O at 256s+128 .. 256s+128+D-1.
//
// Per stream and key tile: S = Q K^T (SS MMA, K-major operands) -> softmax warps read S,
// mask, update the running max with lazy rescaling (O and l are rescaled only when the max
// grows by more than 8 in base-2 units, exact because the final normalisation uses the same
// reference max), write P = 2^(S - m) into TMEM -> O += P V (TS MMA, V MN-major).  The row
// max uses three-input maxes in independent chains, the scaling and the row sum run on packed
// f32x2 pairs.  Every wait is bounded; on expiry the CTA flags HS2_DEV_TIMEOUT, drains and
// exits.
//
// The split partials (m, l, O) and the log-sum-exp combine are those of the mma.sync sweep
// ("Simplified Sparse Attention via Gist Tokens", section 3.6, split-K flash-decode).
#include "attn_sweep.cuh"
#include "umma.cuh"

namespace hs2 {

namespace {

constexpr int kUTile = 128;     // keys per K/V tile
constexpr int kURows = 128;     // rows per query tile (= TMEM lanes)
constexpr int kUStages = 2;     // stages of each of the K and V rings
constexpr int kUThreads = 384;
// Registers per thread: at launch (65536 / 384, rounded down to a multiple of 8), and after the
// split -- the softmax warpgroups hold a whole 128-column row of S; the producer/MMA warpgroup
// needs few.  The split must not exceed the launch total.
constexpr int kURegsLaunch = 168;
constexpr int kURegsSoftmax = 224;
constexpr int kURegsOther = 56;
static_assert(2 * 128 * kURegsSoftmax + 128 * kURegsOther <= kUThreads * kURegsLaunch, "register split");
constexpr float kRescaleBits = 8.f;  // lazy-rescale threshold (base-2 units)

template <int D>
struct USmem {
    static constexpr int kQBytes = kURows * D * 2;       // one query tile
    static constexpr int kTileBytes = kUTile * D * 2;    // one K or V tile
    static constexpr int kBlock = kUTile * 128;          // one 64-column block of a tile
    static constexpr int kQOff = 0;
    static constexpr int kKOff = 2 * kQBytes;
    static constexpr int kVOff = kKOff + kUStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kUStages * kTileBytes;
    static constexpr int kNumBars = 4 * kUStages + 6;    // kfull, kempty, vfull, vempty, sfull[2], pfull[2], done, vfix
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kPosOff = kMiscOff + 16;        // row positions of both streams
    static constexpr int kBytes = kPosOff + 2 * kURows * 4 + 1024;  // + alignment slack
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kUThreads, 1)
    umma_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const AttnArgs a, const int split_keys) {
    using L = USmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* kfull = bars;
    uint64_t* kempty = bars + kUStages;
    uint64_t* vfull = bars + 2 * kUStages;
    uint64_t* vempty = bars + 3 * kUStages;
    uint64_t* sfull = bars + 4 * kUStages;
    uint64_t* pfull = sfull + 2;
    uint64_t* done = sfull + 4;
    uint64_t* vfix = sfull + 5;  // the last V tile with its rows past the last position zeroed
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
    int* s_pos = reinterpret_cast<int*>(smem + L::kPosOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();
    if (a.zero) {  // clear the next kernels' per-row counters and histograms, spread over all CTAs
        const int64_t cta = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
        const int64_t nthr = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
        for (int64_t i = cta * blockDim.x + tid; i < a.zero_vec; i += nthr) a.zero[i] = make_uint4(0, 0, 0, 0);
    }

    const int split = blockIdx.x, unit = blockIdx.y;
    const int QP = split_keys ? a.QB : (a.QB + 1) / 2;  // CTAs (row-block pairs) per (b, kv head)
    const int bh = unit / QP, pr = unit % QP;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const int nq = split_keys ? 1 : 2;  // query tiles held by this CTA
    // global query-head row of row r of query tile s, or -1 for a padding row
    auto row_q = [&](int s, int r) -> int {
        const int qb = split_keys ? pr : 2 * pr + s;
        const int tq = r / a.G, t = qb * a.TQ + tq;
        if (qb >= a.QB || tq >= a.TQ || t >= a.T) return -1;
        return (b * a.Hq + h * a.G + (r % a.G)) * a.T + t;
    };

    // ---- prologue: positions, query tiles (128-byte swizzled, zero padding rows), barriers
    for (int i = tid; i < 2 * kURows; i += kUThreads) {
        const int s = i / kURows, r = i % kURows;
        int p = -1;
        if (s < nq && row_q(s, r) >= 0) {
            const int qb = split_keys ? pr : 2 * pr + s;
            p = clamp_pos(a.pos[b * a.T + qb * a.TQ + r / a.G], a.N, a.status);
        }
        s_pos[i] = p;
    }
    constexpr int CH = D / 8;  // 16-byte chunks per row
    for (int i = tid; i < nq * kURows * CH; i += kUThreads) {
        const int s = i / (kURows * CH), rem = i % (kURows * CH);
        const int r = rem / CH, c = rem % CH;
        const int grow = row_q(s, r);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (grow >= 0) v = *reinterpret_cast<const uint4*>(a.Q + static_cast<int64_t>(grow) * D + c * 8);
        *reinterpret_cast<uint4*>(smem + L::kQOff + s * L::kQBytes + (c >> 3) * (kURows * 128) + r * 128 +
                                  (((c & 7) ^ (r & 7)) << 4)) = v;
    }
    fence_async_smem();
    if (tid == 0) {
        for (int i = 0; i < L::kNumBars; ++i) mbar_init(&bars[i], i >= 4 * kUStages + 2 && i < 4 * kUStages + 4
                                                                      ? kURows   // pfull: one arrival per row
                                                                      : (i == 4 * kUStages + 5 ? 64 : 1));  // vfix: warps 10-11
        *abort_flag = 0;
        fence_barrier_init();
    }
    // TMEM is taken only after the predecessor kernel has completed: a CTA of a later kernel
    // that allocated first could otherwise wait on this one forever.
    pdl_wait();
    if (warp == 9) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;

    // ---- key range of this split (128-key tiles up to the largest row position)
    int jmax = -1;
    for (int i = 0; i < 2 * kURows; ++i) jmax = max(jmax, s_pos[i]);
    const int ntiles = jmax >= 0 ? (jmax + kUTile) / kUTile : 0;
    const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.S);
    const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.S);
    const int nt = t_end - t_begin;
    // steps of each stream; step i of stream s uses the (seq)-th tile of the range
    const int nstep0 = split_keys ? (nt + 1) / 2 : nt;
    const int nstep1 = split_keys ? nt / 2 : nt;
    auto seq_of = [&](int s, int i) { return split_keys ? 2 * i + s : i; };
    // The CTA's last tile reaches past its largest position: those keys are masked (P = 0), but
    // their cache slots may hold anything (an unwritten cache), and 0 x NaN would poison O.  Warps
    // 10-11 zero those V rows once the tile lands; the PV MMA of that tile waits for them.
    const bool fix_last = nt > 0 && t_end == ntiles && ntiles * kUTile - 1 > jmax;

    if (warp >= 8) {
        reg_dealloc<kURegsOther>();
    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol = a.stream_kv ? l2_evict_first() : l2_evict_normal();
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            int k_issued = 0, v_issued = 0;  // tiles whose K (V) load was issued
            for (int q = 0; q < nt; ++q) {
                const int st = q % kUStages;
                const uint32_t ph = ((q / kUStages) - 1) & 1;
                const int j0 = (t_begin + q) * kUTile;
                if (q >= kUStages && !mbar_wait(&kempty[st], ph, a.status)) { *abort_flag = 1; break; }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&kfull[st], L::kTileBytes);
#pragma unroll
                for (int hb = 0; hb < D / 64; ++hb)
                    tma_load_3d(smem + L::kKOff + st * L::kTileBytes + hb * L::kBlock, &tmK, &kfull[st], hb * 64, j0,
                                bh, pol);
                ++k_issued;
                if (q >= kUStages && !mbar_wait(&vempty[st], ph, a.status)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&vfull[st], L::kTileBytes);
#pragma unroll
                for (int hb = 0; hb < D / 64; ++hb)
                    tma_load_3d(smem + L::kVOff + st * L::kTileBytes + hb * L::kBlock, &tmV, &vfull[st], hb * 64, j0,
                                bh, pol);
                ++v_issued;
            }
            // drain: the last load issued into every stage has landed before the CTA retires
            for (int st = 0; st < kUStages && st < k_issued; ++st) {
                const int last = st + ((k_issued - 1 - st) / kUStages) * kUStages;
                mbar_wait(&kfull[st], (last / kUStages) & 1, a.status);
            }
            for (int st = 0; st < kUStages && st < v_issued; ++st) {
                const int last = st + ((v_issued - 1 - st) / kUStages) * kUStages;
                mbar_wait(&vfull[st], (last / kUStages) & 1, a.status);
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_bf16(kURows, kUTile, false);
            constexpr uint32_t kIdescPV = idesc_bf16(kURows, D, true);
            const uint32_t qa0 = smem_u32(smem + L::kQOff);
            const uint32_t kb0 = smem_u32(smem + L::kKOff);
            const uint32_t vb0 = smem_u32(smem + L::kVOff);
            auto issue_qk = [&](int s, int i) -> bool {
                const int q = seq_of(s, i), st = q % kUStages;
                if (!mbar_wait(&kfull[st], (q / kUStages) & 1, a.status)) return false;
                tc_fence_after();
                const uint32_t qa = qa0 + (split_keys ? 0 : s) * L::kQBytes;
                const uint32_t kb = kb0 + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kBlock + (kk & 3) * 32;
                    umma_ss(tm + 256 * s, sw128_desc(qa + off, 16, 1024), sw128_desc(kb + off, 16, 1024), kIdescQK,
                            kk > 0);
                }
                if (split_keys || s == 1) umma_commit(&kempty[st]);  // last reader of this K tile
                umma_commit(&sfull[s]);
                return true;
            };
            auto issue_pv = [&](int s, int i) -> bool {
                if (!mbar_wait(&pfull[s], i & 1, a.status)) return false;
                const int q = seq_of(s, i), st = q % kUStages;
                if (fix_last && q == nt - 1) {
                    if (!mbar_wait(vfix, 0, a.status)) return false;
                } else if (!mbar_wait(&vfull[st], (q / kUStages) & 1, a.status)) {
                    return false;
                }
                tc_fence_after();
                const uint32_t vb = vb0 + st * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kUTile / 16; ++kk)
                    umma_ts(tm + 256 * s + 128, tm + 256 * s + 8 * kk, sw128_desc(vb + kk * 2048, L::kBlock, 1024),
                            kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                if (split_keys || s == 1) umma_commit(&vempty[st]);
                return true;
            };
            bool ok = true;
            if (nstep0 > 0) ok = issue_qk(0, 0);
            if (ok && nstep1 > 0) ok = issue_qk(1, 0);
            for (int i = 0; ok && i < nstep0; ++i) {
                for (int s = 0; ok && s < 2; ++s) {
                    const int ns = s == 0 ? nstep0 : nstep1;
                    if (i >= ns) continue;
                    // (no abort-flag check here: every wait below is bounded, so an aborted CTA
                    // still ends; the flag's shared-memory load sat on the issue path)
                    ok = issue_pv(s, i);
                    if (ok && i + 1 < ns) ok = issue_qk(s, i + 1);
                }
            }
            if (!ok) *abort_flag = 1;
            umma_commit(done);
            mbar_wait(done, 0, a.status);  // nothing of this CTA is left in the tensor core
        }
        __syncwarp();
    } else if (fix_last) {
        // ------------------------------------------------------------ warps 10-11: zero the V rows
        // of keys past jmax in the last tile (rows of 128 bytes in each 64-dim block)
        const int q = nt - 1, st = q % kUStages;
        const bool landed = mbar_wait(&vfull[st], (q / kUStages) & 1, a.status);
        if (landed) {
            uint8_t* vt = smem + L::kVOff + st * L::kTileBytes;
            const int r0 = jmax + 1 - (t_begin + q) * kUTile;  // first row to clear, in [1, 127]
            const int t = (warp - 10) * 32 + lane;
            for (int e = t; e < (kUTile - r0) * (D / 8); e += 64) {
                const int r = r0 + e / (D / 8), c = e % (D / 8);
                *reinterpret_cast<uint4*>(vt + (c >> 3) * L::kBlock + r * 128 + (c & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_async_smem();  // visible to the tensor core before the arrive
            mbar_arrive(vfix);
        } else {
            *abort_flag = 1;
        }
        __syncwarp();
    }
    } else {
        reg_alloc<kURegsSoftmax>();
        // ------------------------------------------------------------ softmax (thread = row)
        const int s = warp >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int p = s_pos[(split_keys ? 0 : s) * kURows + r];
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tm + lane_bits + 256 * s, tO = tS + 128;
        const int nstep = s == 0 ? nstep0 : nstep1;
        const float sc = a.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int i = 0; i < nstep; ++i) {
            // the decision to go on is warp-uniform: TMEM loads and stores are warp-collective
            const bool got = mbar_wait(&sfull[s], i & 1, a.status);
            if (!got) *abort_flag = 1;
            if (!__all_sync(0xffffffffu, got && !*abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t x[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, x[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) tie_regs(x[c]);
            const int j0 = (t_begin + seq_of(s, i)) * kUTile;
            float mx;
            if (j0 + kUTile - 1 > p) {  // tile reaches past this row's position: mask
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0 + 32 * c + e > p) x[c][e] = __float_as_uint(-INFINITY);
            }
            {  // row max: 8 independent chains of three-input maxes (a single chain would
               // serialise 127 dependent ops)
                float m8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) m8[u] = fmaxf(__uint_as_float(x[0][u]), __uint_as_float(x[0][8 + u]));
#pragma unroll
                for (int e = 16; e < 128; e += 16)  // values e .. e + 15: two per chain
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        m8[u] = max3f(m8[u], __uint_as_float(x[(e + u) >> 5][(e + u) & 31]),
                                      __uint_as_float(x[(e + 8 + u) >> 5][(e + 8 + u) & 31]));
                mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
            }
            mx *= sc;  // base-2 units (sc > 0 keeps the order)
            const bool bump = mx > m_ref + kRescaleBits;
            const float corr = bump ? fast_exp2(m_ref - mx) : 1.f;  // 0 when m_ref = -inf
            const bool fix_o = bump && i > 0 && m_ref != -INFINITY;
            if (bump) m_ref = mx;
            if (__any_sync(0xffffffffu, fix_o)) {
                // O holds P V of the earlier steps (complete: this step's S was committed after it)
                const float f = fix_o ? corr : 1.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
                    tie_regs(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                    tmem_st32(tO + 32 * c, o);
                }
            }
            const float base = m_ref == -INFINITY ? 0.f : m_ref;
            // exponents and the row sum on packed pairs: x * sc - base by one f32x2 FMA per pair,
            // the sum as 4 independent chains of f32x2 adds (8 scalar chains)
            const uint64_t sc2 = f2_pack(sc, sc), nb2 = f2_pack(-base, -base);
            uint64_t sum4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) sum4[e] = f2_pack(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float a0, a1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(x[c][2 * e]), __uint_as_float(x[c][2 * e + 1])), sc2, nb2),
                              a0, a1);
                    const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
                    sum4[e & 3] = f2_add(sum4[e & 3], f2_pack(p0, p1));
                    pk[e] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tS + 16 * c, pk);
            }
            float rs;
            {
                const uint64_t s2 = f2_add(f2_add(sum4[0], sum4[1]), f2_add(sum4[2], sum4[3]));
                float s_lo, s_hi;
                f2_unpack(s2, s_lo, s_hi);
                rs = s_lo + s_hi;
            }
            l = l * corr + rs;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&pfull[s]);
        }
        // ---- epilogue: this stream's split partial
        bool fin = ok && !*abort_flag;
        if (fin) fin = mbar_wait(done, 0, a.status);
        if (__all_sync(0xffffffffu, fin && !*abort_flag)) {
            tc_fence_after();
            const int grow = row_q(split_keys ? 0 : s, r);
            const int slot = split_keys ? 2 * split + s : split;
            const int64_t rows = static_cast<int64_t>(a.B) * a.Hq * a.T;
            float* acc = a.part_acc + (static_cast<int64_t>(slot) * rows + (grow >= 0 ? grow : 0)) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                tie_regs(o);
                if (grow >= 0) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        float4 v = nstep > 0 ? make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                                                           __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                        *reinterpret_cast<float4*>(acc + 32 * c + e) = v;
                    }
                }
            }
            if (grow >= 0)
                a.part_ml[static_cast<int64_t>(slot) * rows + grow] =
                    nstep > 0 ? make_float2(m_ref, l) : make_float2(-INFINITY, 0.f);
        }
    }

    // ---- teardown: every TMEM access of the CTA is complete before the columns are freed
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// ====================================================================== launcher

template <int D>
cudaError_t umma_attn_variant(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                              cudaStream_t st) {
    using L = USmem<D>;
    auto kern = umma_attn_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    // the register split is sized for exactly kURegsLaunch registers per thread at launch
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kURegsLaunch) return cudaErrorInvalidConfiguration;
    const int split_keys = p.umma_split_keys ? 1 : 0;
    const int QP = split_keys ? p.QB : (p.QB + 1) / 2;
    dim3 grid(p.SU, p.B * p.Hkv * QP);
    AttnArgs x = a;
    x.S = p.SU;
    e = launch_pdl(kern, grid, dim3(kUThreads), L::kBytes, st, tmK, tmV, x, split_keys);
    trace_mark("umma_attn", st);
    return e;
}

cudaError_t launch_umma_attn(const Plan& p, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnArgs& a,
                             cudaStream_t st) {
    if (p.d == 128) return umma_attn_variant<128>(p, tmK, tmV, a, st);
    if (p.d == 64) return umma_attn_variant<64>(p, tmK, tmV, a, st);
    return cudaErrorInvalidValue;
}

}  // namespace hs2
