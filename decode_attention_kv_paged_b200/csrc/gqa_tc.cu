// gqa_tc.cu -- decode attention for large query groups (MQA / wide GQA) on
// the tcgen05 tensor cores.
//
// Computes the same as the CUDA-core kernel (attention-head article, §1
// Attention equation, §2 group rule), for one KV head and up to 64 of the
// query heads that share it at a time:
//     S = Q K^T   (heads x 64 tokens)      O += P V   (heads x d)
// With a large group every K/V element feeds many heads, so the two products
// are real dense contractions and belong on the tensor cores; the CUDA-core
// path would need ~G flops per loaded byte.
//
// Design (B200):
//   * One CTA per SM over the split-KV partition (plan.cuh).  Warp 0 issues
//     2-D TMA loads (128-byte swizzle) of each 64-token K and V tile of the
//     paged cache into two rings and of the unit's query rows: a K slot is
//     released by its S product, a V slot only after the softmax and the P V
//     product, so the V ring is the deeper one (at d = 256 the fixed buffers
//     leave room for five 32 KiB slots: two K, three V); one
//     thread of warp 1 issues the S MMAs and one of warp 2 the P V MMAs as
//     their inputs become ready; warps 4-7 run the softmax and the epilogue.
//   * S: M = 64 query rows, N = 64 tokens, K = d, both operands in shared
//     memory, fp32 accumulator in TMEM (double-buffered).  The M = 64
//     accumulator puts row r in TMEM lane (r % 16) + 32 (r / 16), so each
//     row is read by one thread: the softmax needs no cross-thread
//     reductions.  A group of HC <= 32 heads (padded to HCP = 16 or 32) is
//     loaded 64 / HCP times into the 64 rows; copy c of the heads takes only
//     the token slice [c TPC, (c + 1) TPC) of every tile (TPC = HCP), so all
//     four softmax warps work and each thread handles TPC tokens.  Every
//     copy keeps its own (m, l, O) and writes its own partial, merged with
//     the split partials by the log-sum-exp combine.  The running max is only
//     raised when it grows by more than 2^8 (lazy rescale, exact either way).
//   * P is split into bf16 P_hi + P_lo (the rounding remainder) so the
//     weights keep ~16 significant bits; O += P_hi V + P_lo V with V read
//     MN-major from the same swizzled tile; O stays in TMEM for the segment.
//   * Every wait is bounded; TMEM is always freed.
#include <mutex>
#include <vector>

#include "attn_decode.h"
#include "gqa_decode.cuh"
#include "gqa_tc.cuh"
#include "tc_common.cuh"
#include "host_state.cuh"

namespace attn {

constexpr int kTcM = 64;                    // MMA M: query rows per CTA pass
constexpr int kTcThreads = 256;
constexpr int kTcBox = 64 * 128;            // [64 rows][64 cols] bf16, swizzled
constexpr int kTcPBytes = kTcM * 128;       // one P half: [64 heads][64 tokens]
constexpr float kTcRescaleThreshold = 8.0f;

template <int D>
struct TcCfg {
    static constexpr int kBoxes = D / 64;
    static constexpr int kQBytes = kBoxes * kTcBox;
    static constexpr int kSlotBytes = kBoxes * kTcBox;          // one K or V tile
    // P is double-buffered (hi and lo halves each): the softmax of tile i + 1
    // writes while the P V of tile i reads.
    static constexpr int kPBytes = 4 * kTcPBytes;
    static constexpr int kFixed = kQBytes + kPBytes + 1024 /*bars*/ + 1024 /*align*/;
    static constexpr int kSlots = (227 * 1024 - kFixed) / kSlotBytes;
    static constexpr int kKHalf = kSlots / 2 < 2 ? 2 : kSlots / 2;
    static constexpr int kKStages = kKHalf > 6 ? 6 : kKHalf;
    static constexpr int kVStages = kSlots - kKStages > 6 ? 6 : kSlots - kKStages;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kKStages * kSlotBytes;
    static constexpr int kOffP = kOffV + kVStages * kSlotBytes;
    static constexpr int kOffBar = kOffP + kPBytes;
    static constexpr int kSmem = kOffBar + 1024 + 1024;
    static constexpr uint32_t kTmemO = 0, kTmemS = D;            // S buffers at D, D + 64
    static constexpr uint32_t kTmemCols = D + 128 <= 256 ? 256 : 512;
    static_assert(kKStages >= 2 && kVStages >= 2, "at least two stages per ring");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct TcBars {
    uint64_t q_full, q_empty;
    uint64_t k_full[6], k_empty[6], v_full[6], v_empty[6];
    uint64_t s_full[2], s_free[2];
    // One P-ready and one P V-done barrier per P buffer: the softmax can
    // finish two tiles before the MMA thread tests the first, which a single
    // barrier could not tell apart.
    uint64_t p_full[2], pv_done[2], o_free, mma_final;
    // Per V slot (held until the tile's P V, so past the softmax that reads
    // it): global positions among the staged block's keys below the window
    // (bit t: key 64 * block + t), written before the slot is armed.
    unsigned long long gmask[6];
    uint32_t tmem_base;
    int abort;
    PlanScratch plan;
};
static_assert(sizeof(TcBars) <= 1024, "barrier block");

// G: the call has an explicit global set (its masking code is compiled only
// into that instantiation, keeping the common loop as tight as before).
template <int D, int TPC, bool G>
__global__ void __launch_bounds__(kTcThreads, 1)
gqa_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const GqaParams p, int HC) {
    using C = TcCfg<D>;
    constexpr int kCopies = kTcM / TPC;     // copies of the head group in the 64 rows
    constexpr int kHCP = TPC;               // rows per copy (heads, padded)
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *sQ = smem + C::kOffQ;
    unsigned char *sK = smem + C::kOffK;
    unsigned char *sV = smem + C::kOffV;
    unsigned char *sP = smem + C::kOffP;
    TcBars *bars = reinterpret_cast<TcBars *>(smem + C::kOffBar);
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

    // Zero Q (rows beyond the group stay zero) and P (rows beyond the group
    // are never written), then make the zeros visible to the tensor cores.
    for (int i = tid; i < (C::kQBytes + C::kPBytes) / 16; i += kTcThreads) {
        const int off = i * 16;
        uint4 *dst = reinterpret_cast<uint4 *>(off < C::kQBytes ? sQ + off
                                                                : sP + (off - C::kQBytes));
        *dst = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (tid == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < C::kKStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < C::kVStages; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_free[s], 128);
        }
        mbar_init(&bars->p_full[0], 128);
        mbar_init(&bars->p_full[1], 128);
        mbar_init(&bars->pv_done[0], 1);
        mbar_init(&bars->pv_done[1], 1);
        mbar_init(&bars->o_free, 128);
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
            int tile = 0, seg = 0, n_k = 0, n_v = 0;   // tiles; K and V loads issued
            while (!cur.done()) {
                const int kvh = cur.w.unit / p.n_hc, hc = cur.w.unit % p.n_hc;
                if (cur.t == 0) {
                    if (seg > 0 && !mbar_wait(&bars->q_empty, (uint32_t)((seg - 1) & 1),
                                              p.timeout_ns, p.err, abort_flag))
                        break;
                    const int qrow = cur.w.b * p.H_q + kvh * p.group + hc * HC;
                    mbar_arrive_expect_tx(&bars->q_full, kCopies * C::kBoxes * HC * 128);
                    for (int c = 0; c < kCopies; ++c)
                        for (int j = 0; j < C::kBoxes; ++j)
                            tma_load_2d(sQ + j * kTcBox + c * kHCP * 128, &tm_q, 64 * j, qrow,
                                        &bars->q_full, pol);
                    ++seg;
                }
                const int ks = tile % C::kKStages, vs = tile % C::kVStages;
                if (tile >= C::kKStages &&
                    !mbar_wait(&bars->k_empty[ks],
                               (uint32_t)(((tile - C::kKStages) / C::kKStages) & 1), p.timeout_ns,
                               p.err, abort_flag))
                    break;
                int phys = p.block_table[(size_t)cur.w.b * p.max_blocks +
                                         cur.table_slot_of_tile()];
                if (phys < 0 || phys >= p.num_blocks) {
                    raise_error(p.err, kErrBadBlock);
                    phys = p.num_blocks;                 // wholly out of bounds: zero fill
                }
                const int row = (phys * p.H_kv + kvh) * 64;
                mbar_arrive_expect_tx(&bars->k_full[ks], C::kSlotBytes);
                for (int j = 0; j < C::kBoxes; ++j)
                    tma_load_2d(sK + ks * C::kSlotBytes + j * kTcBox, &tm_k, 64 * j, row,
                                &bars->k_full[ks], pol);
                n_k = tile + 1;
                if (tile >= C::kVStages &&
                    !mbar_wait(&bars->v_empty[vs],
                               (uint32_t)(((tile - C::kVStages) / C::kVStages) & 1), p.timeout_ns,
                               p.err, abort_flag))
                    break;
                if constexpr (G) {
                    const int blk = cur.logical_block();
                    bars->gmask[vs] = blk * 64 < cur.w.lo
                                          ? global_mask_thread(p.vis, cur.w.b, blk) : 0ull;
                }
                mbar_arrive_expect_tx(&bars->v_full[vs], C::kSlotBytes);
                for (int j = 0; j < C::kBoxes; ++j)
                    tma_load_2d(sV + vs * C::kSlotBytes + j * kTcBox, &tm_v, 64 * j, row,
                                &bars->v_full[vs], pol);
                n_v = tile + 1;
                cur.next();
                ++tile;
            }
            // Every issued load must have landed before the CTA exits.
            for (int t = n_k - C::kKStages < 0 ? 0 : n_k - C::kKStages; t < n_k; ++t)
                mbar_wait(&bars->k_full[t % C::kKStages], (uint32_t)((t / C::kKStages) & 1),
                          p.timeout_ns, p.err, nullptr);
            for (int t = n_v - C::kVStages < 0 ? 0 : n_v - C::kVStages; t < n_v; ++t)
                mbar_wait(&bars->v_full[t % C::kVStages], (uint32_t)((t / C::kVStages) & 1),
                          p.timeout_ns, p.err, nullptr);
            if (seg > 0)
                mbar_wait(&bars->q_full, (uint32_t)((seg - 1) & 1), p.timeout_ns, p.err, nullptr);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 2) {
        // ============================================================ MMA
        // Two issuing threads: lane 0 of warp 1 issues S(n) = Q K(n)^T for
        // every tile in order, lane 0 of warp 2 issues O += P(i) V(i).  Each
        // chain waits only on its own inputs (S on the staged K tile and a
        // free S buffer, P V on the softmax's P and the staged V tile), so the
        // two streams of MMAs overlap instead of queueing behind one thread.
        // A K slot is released by the commit after S(n), a V slot by the
        // commit after P V(i).  Barriers are polled (a sleeping wait wakes up
        // too late for these chains).
        if (lane == 0) {
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
            const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
            if (warp == 1) {
                constexpr uint32_t idesc_s = umma_idesc_bf16(kTcM, 64, 0, 0);
                const uint32_t q_base = smem_u32(sQ);
                TileCursorT<G> cs;
                cs.init(pa, lo, hi, first_seq, first_base);
                int seg_s = 0;
                for (int n = 0; n < n_tiles; ++n) {
                    // S(n) into S buffer n % 2, once the softmax of tile
                    // n - 2 has read it.
                    const bool first = cs.t == 0, last = cs.t == cs.len - 1;
                    const int ks = n % C::kKStages, sb = n & 1;
                    if (first && !wait(&bars->q_full, (uint32_t)(seg_s & 1))) break;
                    if (!wait(&bars->k_full[ks], (uint32_t)((n / C::kKStages) & 1))) break;
                    if (n >= 2 && !wait(&bars->s_free[sb], (uint32_t)(((n - 2) >> 1) & 1)))
                        break;
                    tc_fence_after();
                    const uint32_t kst = k_base + ks * C::kSlotBytes;
                    for (int j = 0; j < C::kBoxes; ++j)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t a =
                                umma_desc_sw128(q_base + j * kTcBox + k * 32, 16, 1024);
                            const uint64_t b = umma_desc_sw128(kst + j * kTcBox + k * 32, 16, 1024);
                            umma_bf16(tmem + C::kTmemS + 64 * sb, a, b, idesc_s, (j | k) != 0);
                        }
                    umma_commit(&bars->s_full[sb]);
                    umma_commit(&bars->k_empty[ks]);       // K(n) read once S(n) completes
                    if (last) umma_commit(&bars->q_empty);
                    if (first) ++seg_s;
                    cs.next();
                }
            } else {
                constexpr uint32_t idesc_pv = umma_idesc_bf16(kTcM, D, 0, 1);
                const uint32_t p_base = smem_u32(sP);
                TileCursorT<G> cv;
                cv.init(pa, lo, hi, first_seq, first_base);
                int seg_v = 0;
                for (int i = 0; i < n_tiles; ++i) {
                    // O += P(i) V(i), P from buffer i % 2 (hi and lo halves); a
                    // segment's first P V overwrites O once the previous
                    // segment's output has been read.
                    const bool first = cv.t == 0;
                    if (!wait(&bars->p_full[i & 1], (uint32_t)((i >> 1) & 1))) break;
                    if (first && seg_v > 0 && !wait(&bars->o_free, (uint32_t)((seg_v - 1) & 1)))
                        break;
                    tc_fence_after();
                    const int vs = i % C::kVStages;
                    if (!wait(&bars->v_full[vs], (uint32_t)((i / C::kVStages) & 1))) break;
                    const uint32_t vst = v_base + vs * C::kSlotBytes;
                    const uint32_t pb = p_base + (i & 1) * 2 * kTcPBytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t b = umma_desc_sw128(vst + k * 2048, kTcBox, 1024);
                        const uint64_t a_hi = umma_desc_sw128(pb + k * 32, 16, 1024);
                        const uint64_t a_lo = umma_desc_sw128(pb + kTcPBytes + k * 32, 16, 1024);
                        umma_bf16(tmem + C::kTmemO, a_hi, b, idesc_pv, !(first && k == 0));
                        umma_bf16(tmem + C::kTmemO, a_lo, b, idesc_pv, 1);
                    }
                    umma_commit(&bars->v_empty[vs]);
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
    } else if (warp >= 4) {
        // ================================================ softmax, epilogue
        // M = 64 accumulator: row r lives in TMEM lane (r % 16) + 32 (r / 16);
        // warp 4 + q owns rows 16q .. 16q + 15 in its lanes 0..15, which are
        // head rows of copy c (warp-uniform) for the token slice c * TPC.
        const int q4 = warp & 3;
        const int row = 16 * q4 + lane;
        const int copy = (16 * q4) / kHCP;
        const int head = row - copy * kHCP;
        const bool active = lane < 16 && head < HC;
        const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
        unsigned char *prow0 = sP + (lane < 16 ? row : 0) * 128;
        auto all = [](bool v) { return __all_sync(0xffffffffu, v); };
        TileCursorT<G> cur;
        cur.init(pa, lo, hi, first_seq, first_base);
        float m_run = kNegInf, l_run = 0.f;
        for (int i = 0; i < n_tiles; ++i) {
            const bool first = cur.t == 0, last = cur.t == cur.len - 1;
            const int b = cur.w.b, T = cur.w.T;
            const int lo_tok = cur.w.lo, sink = p.vis.sink;
            const int blk = cur.logical_block();
            const int tok0 = blk * 64 + copy * TPC;
            // Global positions among this block's keys below the window.
            unsigned long long gmask = 0ull;
            if (G && blk * 64 < lo_tok) {
                // The V slot of tile i stays armed for it (it is refilled only
                // after this tile's P V), so this wait orders the producer's
                // mask before the read.
                const int vs = i % C::kVStages;
                if (!all(mbar_wait(&bars->v_full[vs], (uint32_t)((i / C::kVStages) & 1),
                                   p.timeout_ns, p.err, abort_flag)))
                    break;
                gmask = bars->gmask[vs];
            }
            const int sb = i & 1;
            if (!all(mbar_wait(&bars->s_full[sb], (uint32_t)((i >> 1) & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            tc_fence_after();
            float s[TPC];
            const uint32_t saddr = trow + C::kTmemS + 64 * sb + copy * TPC;
            if constexpr (TPC == 64) tmem_ld64(saddr, s);
            else if constexpr (TPC == 32) tmem_ld32(saddr, s);
            else tmem_ld16(saddr, s);
            tc_fence_before();
            mbar_arrive(&bars->s_free[sb]);

            // scale to log2 units, mask keys that are not visible
            const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
            for (int j = 0; j < TPC; j += 2) {
                const float2 v = __fmul2_rn(make_float2(s[j], s[j + 1]), sl2);
                s[j] = v.x;
                s[j + 1] = v.y;
            }
            if (tok0 + TPC > T || (tok0 < lo_tok && (tok0 + TPC > sink || gmask))) {
#pragma unroll
                for (int j = 0; j < TPC; ++j) {
                    const int pos = tok0 + j;
                    if (pos >= T || (pos < lo_tok && pos >= sink &&
                                     !((gmask >> (pos - blk * 64)) & 1ull)))
                        s[j] = kNegInf;
                }
            }
            float mx;
            {
                float t[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    t[j] = s[j];
#pragma unroll
                    for (int k = j + 8; k < TPC; k += 8) t[j] = fmaxf(t[j], s[k]);
                }
#pragma unroll
                for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                    for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
                mx = t[0];
            }
            // Raise the running max on the segment's first tile, or when a
            // score exceeds it by more than the headroom.  A slice with no
            // visible key so far keeps m_run = -inf (its probabilities are 0).
            bool rescale = false;
            float alpha = 1.f;
            if (first) {
                m_run = mx;
                l_run = 0.f;
            } else if (mx > m_run + kTcRescaleThreshold) {
                alpha = m_run == kNegInf ? 0.f : exp2_approx(m_run - mx);
                m_run = mx;
                l_run *= alpha;
                rescale = true;
            }
            const float mref = m_run == kNegInf ? 0.f : m_run;
            float2 sum2 = make_float2(0.f, 0.f);
            const float2 m2 = make_float2(-mref, -mref);
#pragma unroll
            for (int j = 0; j < TPC; j += 2) {
                const float2 d = __fadd2_rn(make_float2(s[j], s[j + 1]), m2);
                s[j] = exp2_approx(d.x);
                s[j + 1] = exp2_approx(d.y);
                sum2 = __fadd2_rn(sum2, make_float2(s[j], s[j + 1]));
            }
            l_run += sum2.x + sum2.y;

            // P buffer i % 2 was last read by P V(i - 2).
            if (i >= 2 && !all(mbar_wait(&bars->pv_done[i & 1], (uint32_t)(((i >> 1) - 1) & 1),
                                         p.timeout_ns, p.err, abort_flag)))
                break;
            unsigned char *prow = prow0 + (i & 1) * 2 * kTcPBytes;
            if (active) {
                // This row's 16-byte chunks (8 tokens each) of its slice; the
                // rest of the row stays zero.
#pragma unroll
                for (int cc = 0; cc < TPC / 8; ++cc) {
                    uint32_t hi_w[4], lo_w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float a = s[8 * cc + 2 * k], bb = s[8 * cc + 2 * k + 1];
                        hi_w[k] = pack_bf16x2(a, bb);
                        const float2 r = __fadd2_rn(
                            make_float2(a, bb),
                            make_float2(-__uint_as_float(hi_w[k] << 16),
                                        -__uint_as_float(hi_w[k] & 0xFFFF0000u)));
                        lo_w[k] = pack_bf16x2(r.x, r.y);
                    }
                    const int chunk = copy * (TPC / 8) + cc;
                    const int off = (chunk ^ (row & 7)) * 16;
                    *reinterpret_cast<uint4 *>(prow + off) =
                        make_uint4(hi_w[0], hi_w[1], hi_w[2], hi_w[3]);
                    *reinterpret_cast<uint4 *>(prow + kTcPBytes + off) =
                        make_uint4(lo_w[0], lo_w[1], lo_w[2], lo_w[3]);
                }
            }
            tc_fence_after();
            // O may be rescaled only once P V(i - 1) has completed.
            if (__any_sync(0xffffffffu, active && rescale) && i >= 1 &&
                !all(mbar_wait(&bars->pv_done[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1),
                               p.timeout_ns, p.err, abort_flag)))
                break;
            if (__any_sync(0xffffffffu, active && rescale)) {
                const float a = (active && rescale) ? alpha : 1.f;
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
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full[i & 1]);

            if (last) {
                if (!all(mbar_wait(&bars->pv_done[i & 1], (uint32_t)((i >> 1) & 1), p.timeout_ns,
                                   p.err, abort_flag)))
                    break;
                tc_fence_after();
                // Partial of copy `copy` of this (unit, CTA) slot; a copy
                // that saw no visible key writes zero weight (lse = -inf).
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
                mbar_arrive(&bars->o_free);
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
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn tc_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                 uint32_t box_rows) {
    EncodeTiledFn fn = tc_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int D, int TPC, bool G>
cudaError_t launch_tc_g(const GqaLaunch &L, int HC) {
    using C = TcCfg<D>;
    static PerDeviceFlag configured;   // the attribute is per function and device
    {
        const cudaError_t e = configure_once_per_device(configured, [] {
            return cudaFuncSetAttribute(gqa_tc_kernel<D, TPC, G>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        });
        if (e != cudaSuccess) return e;
    }
    const GqaParams &kp = L.kp;
    CUtensorMap tq, tk, tv;
    if (!tc_make_map(&tq, kp.q, D, (uint64_t)kp.B * kp.H_q, (uint32_t)HC) ||
        !tc_make_map(&tk, kp.k_cache, D, (uint64_t)kp.num_blocks * kp.H_kv * 64, 64) ||
        !tc_make_map(&tv, kp.v_cache, D, (uint64_t)kp.num_blocks * kp.H_kv * 64, 64))
        return cudaErrorInvalidValue;
    if (L.ev_start) cudaEventRecord(L.ev_start, L.stream);
    gqa_tc_kernel<D, TPC, G><<<kp.num_ctas, kTcThreads, C::kSmem, L.stream>>>(tq, tk, tv, kp, HC);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (L.ev_stop) cudaEventRecord(L.ev_stop, L.stream);

    CombineParams cp = L.cp;
    cp.D = D;
    cp.HC = HC;
    cp.copies = kTcM / TPC;
    // Partials per unit: about (CTAs / units + 1) splits, times the copies.
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

template <int D, int TPC>
cudaError_t launch_tc(const GqaLaunch &L, int HC) {
    return L.kp.vis.n_g > 0 ? launch_tc_g<D, TPC, true>(L, HC)
                            : launch_tc_g<D, TPC, false>(L, HC);
}

}  // namespace

bool gqa_tc_supported(int d, int dtype_bf16, int G) {
    return dtype_bf16 && (d == 64 || d == 128 || d == 256) && (G <= kTcM || G % kTcM == 0);
}

int gqa_tc_heads_per_cta(int G) { return G <= kTcM ? G : kTcM; }

int gqa_tc_copies(int HC) { return HC <= 16 ? 4 : (HC <= 32 ? 2 : 1); }

template <int D>
cudaError_t launch_tc_d(const GqaLaunch &L, int HC) {
    switch (gqa_tc_copies(HC)) {
        case 4: return launch_tc<D, 16>(L, HC);
        case 2: return launch_tc<D, 32>(L, HC);
        default: return launch_tc<D, 64>(L, HC);
    }
}

cudaError_t launch_gqa_tc(const GqaLaunch &L, int d, int HC) {
    switch (d) {
        case 64: return launch_tc_d<64>(L, HC);
        case 128: return launch_tc_d<128>(L, HC);
        case 256: return launch_tc_d<256>(L, HC);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace attn
