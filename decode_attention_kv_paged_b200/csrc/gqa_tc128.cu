// gqa_tc128.cu -- decode attention for groups of up to 32 query heads (MQA and
// wide GQA, d <= 128) on the tcgen05 tensor cores with M = 128 MMAs.
//
// Computes the same as the other GQA kernels (attention-head article, §1
// Attention equation, §2 group rule) for one KV head and its HC <= 32 query
// heads:   S = Q K^T (rows x 64 tokens),   O += P V (rows x d).
//
// Design (B200):
//   * The 128 MMA rows hold 128 / HCP copies of the head group (HCP = 16 or
//     32, the group padded); copy c takes only the token slice
//     [c TPC, (c + 1) TPC) of every 64-token tile (TPC = 64 HCP / 128), so
//     all 128 softmax threads work.  Each copy keeps its own (m, l, O) and
//     writes its own partial, merged with the split partials by the
//     log-sum-exp combine.
//   * Q and P live in tensor memory as the MMAs' A operand (row = TMEM lane,
//     bf16 pairs per 32-bit column): only the K and V tiles are read from
//     shared memory (2-D TMA, 128-byte swizzle, 6-stage ring).  The M = 128
//     accumulators put row r in lane r, so one thread owns one row and the
//     softmax needs no cross-thread reduction.
//   * P = P_hi + P_lo (bf16 rounding remainder) keeps ~16 significant bits;
//     O += P_hi V + P_lo V with V read MN-major from its swizzled tile.
//     S and P are double-buffered, each buffer with its own barriers.
//   * Two threads issue the MMAs: one the S products in tile order, the
//     other the P V products.  The softmax threads write a segment's queries
//     into TMEM when they reach it, after reading the previous segment's O
//     (which waits for that segment's last P V), so the S issuer's wait for
//     new queries depends only on the other issuer: no wait depends on itself.
//   * Lazy rescale: the running max is raised only when it grows by more
//     than 2^8 (exact either way).  Every wait is bounded; TMEM is freed.
#include "attn_decode.h"
#include "gqa_decode.cuh"
#include "gqa_tc.cuh"
#include "tc_common.cuh"
#include "host_state.cuh"

namespace attn {

constexpr int kT2Threads = 256;
constexpr int kT2ThreadsF8 = 384;          // fp8: + warps 8-11 widening the codes
constexpr int kT2Box = 64 * 128;           // [64 rows][64 cols] bf16, swizzled
constexpr float kT2Rescale = 8.0f;         // lazy-rescale headroom, log2 units

template <int D, bool F8 = false>
struct T2Cfg {
    static constexpr int kBoxes = D / 64;
    static constexpr int kStageBytes = 2 * kBoxes * kT2Box;       // K then V (bf16 / f16)
    // fp8: each stage also has a raw stage (K codes, V codes, K and V row
    // scales) that the widening warps convert into it.
    // The raw ring is the deeper one: the codes in flight from HBM are what
    // keeps the memory system busy, the widened stages only feed the MMAs.
    static constexpr int kRawBytes = F8 ? 2 * 64 * D + 512 : 0;
    static constexpr int kScaleBytes = F8 ? 512 : 0;              // widened stage's scales
    static constexpr int kStagesFit = (227 * 1024 - 4096) / kStageBytes;
    static constexpr int kStages = F8 ? (D == 128 ? 4 : 6) : (kStagesFit > 6 ? 6 : kStagesFit);
    static constexpr int kRawFit =
        F8 ? (227 * 1024 - 4096 - kStages * (kStageBytes + kScaleBytes)) / kRawBytes : 0;
    static constexpr int kRaw = kRawFit > 8 ? 8 : kRawFit;         // fp8 raw stages
    static constexpr int kOffRaw = kStages * kStageBytes;
    static constexpr int kOffScale = kOffRaw + kRaw * kRawBytes;
    static constexpr int kOffBar = kOffScale + kStages * kScaleBytes;
    static constexpr int kSmem = kOffBar + 1024 + 1024;           // + alignment slack
    // TMEM columns: O [0, D), S 2 x 64, Q D/2 (bf16 pairs), P 2 x (hi 32, lo 32).
    static constexpr uint32_t kTmemO = 0;
    static constexpr uint32_t kTmemS = D;
    static constexpr uint32_t kTmemQ = D + 128;
    static constexpr uint32_t kTmemP = D + 128 + D / 2;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kTmemP + 128 <= kTmemCols, "TMEM columns");
    static_assert(kStages >= 3, "stages");
    static_assert(!F8 || kRaw >= 4, "raw stages");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct T2Bars {
    uint64_t c_full[6], c_empty[6];
    uint64_t raw_full[8], raw_empty[8];   // fp8: codes landed / widened
    int raw_bad[8];                       // fp8: the stage's block id was invalid
    uint64_t q_full, q_empty;
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], pv_done[2];
    uint64_t o_free, mma_final;
    // Per stage: global positions among the staged block's keys below the
    // window (bit t: key 64 * block + t), written before the stage is armed.
    unsigned long long gmask[6];
    uint32_t tmem_base;
    int abort;
    PlanScratch plan;
};
static_assert(sizeof(T2Bars) <= 1024, "barrier block");

// G: the call has an explicit global set (its masking code is compiled only
// into that instantiation, keeping the common loop as tight as before).
// F8: the cache holds OCP E4M3 codes with one fp32 scale per row (value =
// code x scale); the codes are widened to f16 on the chip (exact) and the
// MMAs run on f16 operands (query converted once per segment, exact within
// f16's range; P one f16 operand of 11 significant bits, so no P_lo
// product); the K row scale multiplies the token's score, the V row scale
// its probability before the P V product (the softmax sums stay unscaled).
template <int D, int HCP, bool G, bool F8>
__global__ void __launch_bounds__(F8 ? kT2ThreadsF8 : kT2Threads, 1)
gqa_tc128_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const GqaParams p, int HC) {
    using C = T2Cfg<D, F8>;
    constexpr int kCopies = 128 / HCP;      // copies of the head group in the rows
    constexpr int kTPC = 64 / kCopies;      // tokens per copy per tile (16 or 8)
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *sC = smem;
    T2Bars *bars = reinterpret_cast<T2Bars *>(smem + C::kOffBar);
    volatile int *abort_flag = &bars->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int units = p.H_kv * p.n_hc;
    PlanArgs pa{p.seq_lens, p.B, units, p.vis, p.max_blocks, p.num_ctas};
    plan_locate(pa, blockIdx.x, &bars->plan, blockIdx.x == 0 ? p.ws_prefix : nullptr, p.err);
    const long long W = bars->plan.total;
    const int P = working_ctas(W, p.num_ctas);
    if ((int)blockIdx.x >= P) return;
    const long long lo = cta_bound(blockIdx.x, W, P);
    const long long hi = cta_bound(blockIdx.x + 1, W, P);
    const int first_seq = bars->plan.seq;
    const long long first_base = bars->plan.base;
    const int n_tiles = (int)(hi - lo);

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->c_full[s], F8 ? 4 : 1);     // widening warps, or the TMA
            mbar_init(&bars->c_empty[s], 1);
        }
        for (int s = 0; s < C::kRaw; ++s) {
            mbar_init(&bars->raw_full[s], 1);
            mbar_init(&bars->raw_empty[s], 4);
        }
        mbar_init(&bars->q_full, 4);        // barriers count warps (one arrival each)
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_free[s], 4);
            mbar_init(&bars->p_full[s], 4);
            mbar_init(&bars->pv_done[s], 1);
        }
        mbar_init(&bars->o_free, 4);
        mbar_init(&bars->mma_final, 2);     // one commit per issuing thread
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ============================================================ TMA
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
            TileCursorT<G> cur;
            cur.init(pa, lo, hi, first_seq, first_base);
            int tile = 0;
            constexpr int kRing = F8 ? C::kRaw : C::kStages;   // the ring this thread fills
            uint64_t *freed = F8 ? bars->raw_empty : bars->c_empty;
            while (!cur.done()) {
                const int kvh = cur.w.unit / p.n_hc;
                const int st = tile % kRing;
                if (tile >= kRing &&
                    !mbar_wait(&freed[st], (uint32_t)(((tile - kRing) / kRing) & 1),
                               p.timeout_ns, p.err, abort_flag))
                    break;
                int phys = p.block_table[(size_t)cur.w.b * p.max_blocks +
                                         cur.table_slot_of_tile()];
                const bool bad = phys < 0 || phys >= p.num_blocks;
                if (bad) {
                    raise_error(p.err, kErrBadBlock);
                    phys = p.num_blocks;                 // wholly out of bounds: zero fill
                }
                const int row = (phys * p.H_kv + kvh) * 64;
                if constexpr (G) {
                    const int blk = cur.logical_block();
                    bars->gmask[st] = blk * 64 < cur.w.lo
                                          ? global_mask_thread(p.vis, cur.w.b, blk) : 0ull;
                }
                if constexpr (F8) {
                    // codes and row scales into the raw stage (the widening
                    // warps release it); a bad block is zeros, never read
                    unsigned char *raw = smem + C::kOffRaw + st * C::kRawBytes;
                    bars->raw_bad[st] = bad ? 1 : 0;
                    if (bad) {
                        mbar_arrive(&bars->raw_full[st]);
                    } else {
                        const size_t off = (size_t)row * D;
                        mbar_arrive_expect_tx(&bars->raw_full[st], C::kRawBytes);
                        bulk_load(raw, static_cast<const uint8_t *>(p.k_cache) + off, 64 * D,
                                  &bars->raw_full[st], pol);
                        bulk_load(raw + 64 * D, static_cast<const uint8_t *>(p.v_cache) + off,
                                  64 * D, &bars->raw_full[st], pol);
                        bulk_load(raw + 128 * D, p.k_scale + row, 256, &bars->raw_full[st], pol);
                        bulk_load(raw + 128 * D + 256, p.v_scale + row, 256, &bars->raw_full[st],
                                  pol);
                    }
                } else {
                    unsigned char *dst = sC + st * C::kStageBytes;
                    mbar_arrive_expect_tx(&bars->c_full[st], C::kStageBytes);
                    for (int j = 0; j < C::kBoxes; ++j) {
                        tma_load_2d(dst + j * kT2Box, &tm_k, 64 * j, row, &bars->c_full[st], pol);
                        tma_load_2d(dst + (C::kBoxes + j) * kT2Box, &tm_v, 64 * j, row,
                                    &bars->c_full[st], pol);
                    }
                }
                cur.next();
                ++tile;
            }
            // Every issued load must have landed before the CTA exits.
            uint64_t *landed = F8 ? bars->raw_full : bars->c_full;
            for (int t = tile - kRing < 0 ? 0 : tile - kRing; t < tile; ++t)
                mbar_wait(&landed[t % kRing], (uint32_t)((t / kRing) & 1), p.timeout_ns, p.err,
                          nullptr);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 2) {
        // ============================================================ MMA
        // Lane 0 of warp 1 issues S(n) = Q K(n)^T for every tile in order,
        // lane 0 of warp 2 issues O += P(i) V(i); each waits only on its own
        // inputs, so the two streams overlap.  A segment's first S waits for
        // its queries, which the softmax threads write only after reading the
        // previous segment's O (after its last P V): that chain runs through
        // the other issuer, never back to this one.  Barriers are polled.
        if (lane == 0) {
            const uint32_t c_base = smem_u32(sC);
            auto wait = [&](uint64_t *bar, uint32_t parity) -> bool {
                unsigned long long t0 = 0;
                for (uint32_t it = 0;; ++it) {
                    if (mbar_test(bar, parity)) return true;
                    if ((it & 15u) == 15u) {
                        if (*abort_flag) return false;
                        __nanosleep(20);
                    }
                    if ((it & 1023u) == 1023u) {
                        const unsigned long long now = global_timer_ns();
                        if (t0 == 0) {
                            t0 = now;
                        } else if (now - t0 > p.timeout_ns) {
                            raise_error(p.err, kErrTimeout);
                            *abort_flag = 1;
                            return false;
                        }
                    }
                }
            };
            if (warp == 1) {
                constexpr uint32_t idesc_s =
                    F8 ? umma_idesc_f16(128, 64, 0, 0) : umma_idesc_bf16(128, 64, 0, 0);
                TileCursorT<G> cs;
                cs.init(pa, lo, hi, first_seq, first_base);
                int seg_s = 0;
                for (int n = 0; n < n_tiles; ++n) {
                    // S(n) into S buffer n % 2; A = Q from TMEM.
                    const bool first = cs.t == 0, last = cs.t == cs.len - 1;
                    const int st = n % C::kStages, sb = n & 1;
                    if (first && !wait(&bars->q_full, (uint32_t)(seg_s & 1))) break;
                    if (!wait(&bars->c_full[st], (uint32_t)((n / C::kStages) & 1))) break;
                    if (n >= 2 && !wait(&bars->s_free[sb], (uint32_t)(((n - 2) >> 1) & 1)))
                        break;
                    tc_fence_after();
                    const uint32_t kst = c_base + st * C::kStageBytes;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint64_t b =
                            umma_desc_sw128(kst + (ks >> 2) * kT2Box + (ks & 3) * 32, 16, 1024);
                        umma_bf16_ts(tmem + C::kTmemS + 64 * sb, tmem + C::kTmemQ + 8 * ks, b,
                                     idesc_s, ks != 0);
                    }
                    umma_commit(&bars->s_full[sb]);
                    if (last) umma_commit(&bars->q_empty);
                    if (first) ++seg_s;
                    cs.next();
                }
            } else {
                constexpr uint32_t idesc_pv =
                    F8 ? umma_idesc_f16(128, D, 0, 1) : umma_idesc_bf16(128, D, 0, 1);
                TileCursorT<G> cv;
                cv.init(pa, lo, hi, first_seq, first_base);
                int seg_v = 0;
                for (int i = 0; i < n_tiles; ++i) {
                    // O += P(i) V(i); A = P from TMEM buffer i % 2 (hi, then lo).
                    const bool first = cv.t == 0;
                    if (!wait(&bars->p_full[i & 1], (uint32_t)((i >> 1) & 1))) break;
                    if (first && seg_v > 0 && !wait(&bars->o_free, (uint32_t)((seg_v - 1) & 1)))
                        break;
                    tc_fence_after();
                    const int st = i % C::kStages;
                    const uint32_t vst = c_base + st * C::kStageBytes + C::kBoxes * kT2Box;
                    const uint32_t pb = tmem + C::kTmemP + 64 * (i & 1);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t b = umma_desc_sw128(vst + ks * 2048, kT2Box, 1024);
                        umma_bf16_ts(tmem + C::kTmemO, pb + 8 * ks, b, idesc_pv,
                                     !(first && ks == 0));
                        if constexpr (!F8)
                            umma_bf16_ts(tmem + C::kTmemO, pb + 32 + 8 * ks, b, idesc_pv, 1);
                    }
                    umma_commit(&bars->c_empty[st]);
                    umma_commit(&bars->pv_done[i & 1]);
                    if (first) ++seg_v;
                    cv.next();
                }
            }
            // Both issuers' MMAs complete before the tensor memory is freed.
            umma_commit(&bars->mma_final);
            mbar_wait(&bars->mma_final, 0, p.timeout_ns, p.err, nullptr);
        }
        __syncwarp();
    } else if (F8 && warp >= 8) {
        // ============================================= fp8 -> f16 widening
        // Each item: 16 codes of one row of K or V -> two 16-byte chunks of
        // the row's swizzled f16 box (the layout the TMA gives bf16 tiles);
        // the hardware conversion is exact (every E4M3 value is an f16).
        if constexpr (F8) {
            const int wt = tid - 256;                 // widening thread 0..127
            constexpr int kGroups = D / 16;           // 16-code groups per row
            for (int tile = 0; tile < n_tiles; ++tile) {
                const int rs = tile % C::kRaw, st = tile % C::kStages;
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&bars->raw_full[rs], (uint32_t)((tile / C::kRaw) & 1),
                                          p.timeout_ns, p.err, abort_flag)))
                    break;
                if (tile >= C::kStages &&
                    !__all_sync(0xffffffffu,
                                mbar_wait(&bars->c_empty[st],
                                          (uint32_t)(((tile - C::kStages) / C::kStages) & 1),
                                          p.timeout_ns, p.err, abort_flag)))
                    break;
                const unsigned char *raw = smem + C::kOffRaw + rs * C::kRawBytes;
                unsigned char *dst = sC + st * C::kStageBytes;
                const bool bad = bars->raw_bad[rs] != 0;
                // kGroups items per thread: all loads first, then convert and store
                uint4 codes[kGroups];
#pragma unroll
                for (int k = 0; k < kGroups; ++k) {
                    const int idx = wt + 128 * k;
                    const int m = idx / (64 * kGroups), r = idx % (64 * kGroups);
                    const int t = r / kGroups, g = r % kGroups;
                    codes[k] = bad ? make_uint4(0u, 0u, 0u, 0u)
                                   : *reinterpret_cast<const uint4 *>(raw + m * 64 * D + t * D +
                                                                      16 * g);
                }
#pragma unroll
                for (int k = 0; k < kGroups; ++k) {
                    const int idx = wt + 128 * k;
                    const int m = idx / (64 * kGroups), r = idx % (64 * kGroups);
                    const int t = r / kGroups, g = r % kGroups;
                    uint32_t w[8];
                    e4m3x4_to_f16x4(codes[k].x, w[0], w[1]);
                    e4m3x4_to_f16x4(codes[k].y, w[2], w[3]);
                    e4m3x4_to_f16x4(codes[k].z, w[4], w[5]);
                    e4m3x4_to_f16x4(codes[k].w, w[6], w[7]);
                    unsigned char *drow = dst + (m * C::kBoxes + g / 4) * kT2Box + t * 128;
                    const int c0 = 2 * (g % 4);
                    *reinterpret_cast<uint4 *>(drow + ((c0 ^ (t & 7)) * 16)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4 *>(drow + (((c0 + 1) ^ (t & 7)) * 16)) =
                        make_uint4(w[4], w[5], w[6], w[7]);
                }
                // row scales of the stage: K [0, 64), V [64, 128)
                float *sc = reinterpret_cast<float *>(smem + C::kOffScale) + st * 128;
                sc[wt] = bad ? 0.f : reinterpret_cast<const float *>(raw + 128 * D)[wt];
                fence_proxy_async_smem();             // the MMAs read the widened stage
                mbar_arrive_warp(&bars->raw_empty[rs]);
                mbar_arrive_warp(&bars->c_full[st]);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ================================================ softmax, epilogue
        // Row r = 32 q + lane lives in TMEM lane r: head r % HCP of copy
        // r / HCP.  Warp q reads the 16-token window [16 q, 16 q + 16) of S
        // and writes P columns [8 q, 8 q + 8); with 8 copies (HCP = 16) the
        // window holds two copies' slices and each lane takes its half.
        const int q4 = warp & 3;
        const int row = 32 * q4 + lane;
        const int copy = row / HCP;
        const int head = row % HCP;
        const bool active = head < HC;
        const int half = kTPC == 16 ? 0 : (lane >> 4);   // own slice in the window
        const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
        auto all = [](bool v) { return __all_sync(0xffffffffu, v); };

        // P columns outside a row's slice must read as zero: clear them once.
        {
            uint32_t z[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) z[j] = 0u;
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_st32(trow + C::kTmemP + 32 * c, z);
        }

        TileCursorT<G> cur;
        cur.init(pa, lo, hi, first_seq, first_base);
        float m_run = kNegInf, l_run = 0.f;
        int q_seg = 0;
        for (int i = 0; i < n_tiles; ++i) {
            const bool first = cur.t == 0, last = cur.t == cur.len - 1;
            const int b = cur.w.b, T = cur.w.T;
            const int lo_tok = cur.w.lo, sink = p.vis.sink;
            if (first) {
                // This segment's queries into TMEM (rows beyond the group: 0),
                // once the previous segment's last S has read the old ones.
                if (q_seg > 0 && !all(mbar_wait(&bars->q_empty, (uint32_t)((q_seg - 1) & 1),
                                                p.timeout_ns, p.err, abort_flag)))
                    break;
                tc_fence_after();
                const int kvh = cur.w.unit / p.n_hc, hc = cur.w.unit % p.n_hc;
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    static_cast<const __nv_bfloat16 *>(p.q) +
                    ((size_t)b * p.H_q + kvh * p.group + hc * HC + (active ? head : 0)) * D);
#pragma unroll
                for (int bx = 0; bx < D / 64; ++bx) {
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 v = active ? __ldg(src + 8 * bx + j) : make_uint4(0, 0, 0, 0);
                        r[4 * j] = v.x; r[4 * j + 1] = v.y; r[4 * j + 2] = v.z; r[4 * j + 3] = v.w;
                    }
                    if constexpr (F8) {
                        // f16 operands: exact within f16's range
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = bf16x2_to_f16x2(r[j]);
                    }
                    tmem_st32(trow + C::kTmemQ + 32 * bx, r);
                }
                tc_fence_before();
                mbar_arrive_warp(&bars->q_full);
                ++q_seg;
            }
            const int sb = i & 1;
            if (!all(mbar_wait(&bars->s_full[sb], (uint32_t)((i >> 1) & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            tc_fence_after();
            float w16[16];
            tmem_ld16(trow + C::kTmemS + 64 * sb + 16 * q4, w16);
            tc_fence_before();
            mbar_arrive_warp(&bars->s_free[sb]);

            // This lane's kTPC tokens: window positions [half kTPC, + kTPC).
            const int blk = cur.logical_block();
            const int tok0 = blk * 64 + 16 * q4 + half * kTPC;
            // Global positions among this block's keys below the window.
            unsigned long long gmask = 0ull;
            if (G && blk * 64 < lo_tok) {
                // The stage of tile i is still armed for it (it is refilled only
                // after this tile's P V), so this wait returns at once and orders
                // the producer's mask before the read.
                const int st = i % C::kStages;
                if (!all(mbar_wait(&bars->c_full[st], (uint32_t)((i / C::kStages) & 1),
                                   p.timeout_ns, p.err, abort_flag)))
                    break;
                gmask = bars->gmask[st];
            }
            float s[kTPC];
#pragma unroll
            for (int j = 0; j < kTPC; ++j) {
                float v = w16[j];
                if constexpr (kTPC == 8) v = half ? w16[8 + j] : w16[j];
                s[j] = v * p.scale_log2;
            }
            // fp8: this lane's tokens' K and V row scales, kept with the
            // stage (armed for tile i until its P V: the wait returns at once
            // and orders the widening warps' writes before the reads)
            const float *tsc = nullptr;
            if constexpr (F8) {
                const int st = i % C::kStages;
                if (!all(mbar_wait(&bars->c_full[st], (uint32_t)((i / C::kStages) & 1),
                                   p.timeout_ns, p.err, abort_flag)))
                    break;
                tsc = reinterpret_cast<const float *>(smem + C::kOffScale) + st * 128 +
                      (tok0 - blk * 64);
#pragma unroll
                for (int j = 0; j < kTPC; ++j) s[j] *= tsc[j];
            }
            if (tok0 + kTPC > T || (tok0 < lo_tok && (tok0 + kTPC > sink || gmask))) {
#pragma unroll
                for (int j = 0; j < kTPC; ++j) {
                    const int pos = tok0 + j;
                    if (pos >= T || (pos < lo_tok && pos >= sink &&
                                     !((gmask >> (pos - blk * 64)) & 1ull)))
                        s[j] = kNegInf;
                }
            }
            float mx = s[0];
#pragma unroll
            for (int j = 1; j < kTPC; ++j) mx = fmaxf(mx, s[j]);
            bool rescale = false;
            float alpha = 1.f;
            if (first) {
                m_run = mx;
                l_run = 0.f;
            } else if (mx > m_run + kT2Rescale) {
                alpha = m_run == kNegInf ? 0.f : exp2_approx(m_run - mx);
                m_run = mx;
                l_run *= alpha;
                rescale = true;
            }
            const float mref = m_run == kNegInf ? 0.f : m_run;
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < kTPC; ++j) {
                s[j] = exp2_approx(s[j] - mref);
                sum += s[j];
            }
            l_run += sum;
            if constexpr (F8) {
#pragma unroll
                for (int j = 0; j < kTPC; ++j) s[j] *= tsc[64 + j];   // V row scales
            }

            // P buffer i % 2 was last read by P V(i - 2).
            if (i >= 2 && !all(mbar_wait(&bars->pv_done[i & 1], (uint32_t)(((i >> 1) - 1) & 1),
                                         p.timeout_ns, p.err, abort_flag)))
                break;
            if constexpr (F8) {
                // f16 pairs of this lane's window: own slice, zeros elsewhere.
                uint32_t w[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) w[k] = 0u;
#pragma unroll
                for (int k = 0; k < kTPC / 2; ++k) {
                    const uint32_t h = pack_f16x2(active ? s[2 * k] : 0.f,
                                                  active ? s[2 * k + 1] : 0.f);
                    if constexpr (kTPC == 16) {
                        w[k] = h;
                    } else {
                        w[k] = half ? 0u : h;
                        w[4 + k] = half ? h : 0u;
                    }
                }
                tmem_st8(trow + C::kTmemP + 64 * (i & 1) + 8 * q4, w);
            } else {
                // bf16 pairs of this lane's window: own slice, zeros elsewhere.
                uint32_t hi_w[8], lo_w[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) { hi_w[k] = 0u; lo_w[k] = 0u; }
#pragma unroll
                for (int k = 0; k < kTPC / 2; ++k) {
                    const float a = active ? s[2 * k] : 0.f, bb = active ? s[2 * k + 1] : 0.f;
                    const uint32_t h = pack_bf16x2(a, bb);
                    const float2 r = __fadd2_rn(make_float2(a, bb),
                                                make_float2(-__uint_as_float(h << 16),
                                                            -__uint_as_float(h & 0xFFFF0000u)));
                    const uint32_t l = pack_bf16x2(r.x, r.y);
                    if constexpr (kTPC == 16) {
                        hi_w[k] = h;
                        lo_w[k] = l;
                    } else {
                        hi_w[k] = half ? 0u : h;
                        lo_w[k] = half ? 0u : l;
                        hi_w[4 + k] = half ? h : 0u;
                        lo_w[4 + k] = half ? l : 0u;
                    }
                }
                const uint32_t pcol = trow + C::kTmemP + 64 * (i & 1) + 8 * q4;
                tmem_st8(pcol, hi_w);
                tmem_st8(pcol + 32, lo_w);
            }
            // O may be rescaled only once P V(i - 1) has completed.
            if (__any_sync(0xffffffffu, rescale)) {
                if (i >= 1 && !all(mbar_wait(&bars->pv_done[(i - 1) & 1],
                                             (uint32_t)(((i - 1) >> 1) & 1), p.timeout_ns, p.err,
                                             abort_flag)))
                    break;
                tc_fence_after();
                const float a = rescale ? alpha : 1.f;
                float o[32];
#pragma unroll 1
                for (int ch = 0; ch < D / 32; ++ch) {
                    tmem_ld32(trow + C::kTmemO + 32 * ch, o);
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(o[j] * a);
                    tmem_st32(trow + C::kTmemO + 32 * ch, r);
                }
            }
            tc_fence_before();
            mbar_arrive_warp(&bars->p_full[i & 1]);

            if (last) {
                if (!all(mbar_wait(&bars->pv_done[i & 1], (uint32_t)((i >> 1) & 1), p.timeout_ns,
                                   p.err, abort_flag)))
                    break;
                tc_fence_after();
                // Partial of copy `copy` of this (unit, CTA) slot; a copy that
                // saw no visible key writes zero weight (lse = -inf).
                const long long slot = (long long)b * units + cur.w.unit + blockIdx.x;
                const long long part = (slot * kCopies + copy) * HC + (active ? head : 0);
                const bool empty = l_run == 0.f;
                const float inv = empty ? 0.f : 1.f / l_run;
                float *dst = p.ws_o + (size_t)part * D;
                float o[32];
#pragma unroll 1
                for (int ch = 0; ch < D / 32; ++ch) {
                    tmem_ld32(trow + C::kTmemO + 32 * ch, o);
                    if (active) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(dst + 32 * ch + j) =
                                make_float4(o[j] * inv, o[j + 1] * inv, o[j + 2] * inv,
                                            o[j + 3] * inv);
                    }
                }
                if (active) p.ws_lse[part] = empty ? kNegInf : m_run + log2f(l_run);
                tc_fence_before();
                mbar_arrive_warp(&bars->o_free);
            }
            cur.next();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// -------------------------------------------------------------- host side
namespace {

template <int D, int HCP, bool G, bool F8>
cudaError_t launch_tc128_g(const GqaLaunch &L, int HC) {
    using C = T2Cfg<D, F8>;
    static PerDeviceFlag configured;   // the attribute is per function and device
    {
        const cudaError_t e = configure_once_per_device(configured, [] {
            return cudaFuncSetAttribute(gqa_tc128_kernel<D, HCP, G, F8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        });
        if (e != cudaSuccess) return e;
    }
    const GqaParams &kp = L.kp;
    CUtensorMap tk{}, tv{};            // fp8: the codes come by bulk copies, no maps
    if (!F8 && (!tc_make_map(&tk, kp.k_cache, D, (uint64_t)kp.num_blocks * kp.H_kv * 64, 64) ||
                !tc_make_map(&tv, kp.v_cache, D, (uint64_t)kp.num_blocks * kp.H_kv * 64, 64)))
        return cudaErrorInvalidValue;
    if (L.ev_start) cudaEventRecord(L.ev_start, L.stream);
    gqa_tc128_kernel<D, HCP, G, F8><<<kp.num_ctas, F8 ? kT2ThreadsF8 : kT2Threads, C::kSmem,
                                      L.stream>>>(tk, tv, kp, HC);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (L.ev_stop) cudaEventRecord(L.ev_stop, L.stream);

    CombineParams cp = L.cp;
    cp.D = D;
    cp.HC = HC;
    cp.copies = 128 / HCP;
    cp.lanes = combine_lanes((int)((kp.num_ctas / (L.units_total > 0 ? L.units_total : 1) + 1) *
                                   cp.copies));
    cp.blocks_per_unit = combine_blocks_per_unit(HC, D, cp.lanes);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)L.units_total * cp.blocks_per_unit));
    cfg.blockDim = dim3(kCombineThreads);
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = L.ev_stop ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel<__nv_bfloat16>, cp);
}

template <int D, int HCP, bool F8>
cudaError_t launch_tc128(const GqaLaunch &L, int HC) {
    return L.kp.vis.n_g > 0 ? launch_tc128_g<D, HCP, true, F8>(L, HC)
                            : launch_tc128_g<D, HCP, false, F8>(L, HC);
}

}  // namespace

bool gqa_tc128_supported(int d, int HC) { return (d == 64 || d == 128) && HC <= 32; }

int gqa_tc128_copies(int HC) { return HC <= 16 ? 8 : 4; }

bool gqa_tc128_fp8_supported(int d, int G) {
    return (d == 64 || d == 128) && (G <= 32 || G % 32 == 0);
}

int gqa_tc128_fp8_heads_per_cta(int G) { return G <= 32 ? G : 32; }

cudaError_t launch_gqa_tc128(const GqaLaunch &L, int d, int HC) {
    const bool wide = HC > 16;
    switch (d) {
        case 64: return wide ? launch_tc128<64, 32, false>(L, HC)
                             : launch_tc128<64, 16, false>(L, HC);
        case 128: return wide ? launch_tc128<128, 32, false>(L, HC)
                              : launch_tc128<128, 16, false>(L, HC);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_gqa_tc128_fp8(const GqaLaunch &L, int d, int HC) {
    const bool wide = HC > 16;
    switch (d) {
        case 64: return wide ? launch_tc128<64, 32, true>(L, HC)
                             : launch_tc128<64, 16, true>(L, HC);
        case 128: return wide ? launch_tc128<128, 32, true>(L, HC)
                              : launch_tc128<128, 16, true>(L, HC);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace attn
