// mla_decode.cu -- absorbed MLA decode on the tcgen05 tensor cores.
//
// What it computes (xuesongtap "attention-head" article, §5.2-§5.3): for
// sequence b and head h, with cached rows [c_j | kR_j] (512 + 64 bf16),
//     s_j = scale * (<q_lat[b,h], c_j> + <q_rope[b,h], kR_j>)
//     z[b,h] = sum_j softmax_j(s) c_j                      (512 wide)
// one softmax over the summed content + RoPE scores.
//
// Design (B200): a cluster of two CTAs works on one range of the flattened
// (sequence, 64-token block) list.  The latent columns are split between
// them -- rank 0 owns columns [0, 256), rank 1 owns [256, 512) plus the RoPE
// columns [512, 576) -- so each CTA streams only its slice of every block
// with 2-D TMA (128-byte swizzle, 3-stage ring), and no cache byte is read
// twice.
//   * The query slice lives in tensor memory (row = head = TMEM lane, bf16
//     pairs per 32-bit column), written once per sequence by the softmax
//     threads; S = Q C^T is a 128 x 64 (heads x tokens) tcgen05 MMA with A in
//     TMEM and B = the C tile in shared memory, accumulated in TMEM.
//   * The two partial S are exchanged between the CTAs of the cluster by
//     four exchange warps per CTA (one thread per head row): they read S(i)
//     from TMEM as soon as its MMA completes, stage it in shared memory,
//     free the TMEM buffer for S(i + 1), and one thread moves the staged 32
//     KiB to the peer with a single bulk copy (shared::cta ->
//     shared::cluster, completion on the peer's barrier, which the peer
//     arms itself).  The softmax warps only sum the staged and the received
//     halves, so the exchange of tile i + 1 runs while they work on tile i;
//     no cluster-scope fence sits on their path (the consume signal to the
//     peer is a relaxed arrival).  Both CTAs sum the halves identically.
//   * Softmax runs one thread per head row on the TMEM rows (no cross-thread
//     reductions); the running max is only raised when it grows by more than
//     2^8, so O is rescaled rarely (the result is exact either way: numerator
//     and denominator use the same max).
//   * P is split into two bf16 halves, P = P_hi + P_lo (P_lo = the rounding
//     remainder), so the weights keep ~16 significant bits instead of bf16's
//     8; both halves (128 x 64, swizzled like a TMA tile) are A operands of
//     O += P_hi C + P_lo C, 128 x 256 MMAs whose B operand is the same C tile
//     read MN-major.  Each CTA keeps its 256 output columns in TMEM.
//   * Warp 0 issues TMA; one thread of warp 1 issues the S MMAs and one of
//     warp 2 the P V MMAs, each as its inputs become ready; warps 4-11 load
//     Q, run the softmax and the epilogue; warps 12-15 exchange the scores.  Every
//     wait is bounded; TMEM is always freed; the final cluster handshake is a
//     bounded mbarrier exchange.
// Each (sequence, cluster) segment writes an fp32 partial (O/l and log2-sum-
// exp) that a combine kernel reduces in cluster order.
//
// FP8 latent cache (template flag F8): rows stored as OCP E4M3 codes with one
// fp32 scale per row (value = code value x scale).  The TMA loads each tile's
// code boxes and 64 row scales into a raw stage; a widening warpgroup (warps
// 16-19) converts the codes to f16 exactly (every E4M3 value is an f16
// value) into the same swizzled stage layout the MMAs read, and this variant
// runs its MMAs on f16 operands: the query is converted to f16 once per
// sequence (exact within f16's range) and P is one f16 operand (11
// significant bits, so no P_lo product).  The row scale multiplies the
// token's score column (scores) and its probability before the P V product
// (values); the softmax sums use the unscaled probabilities.
#include <mutex>

#include "attn_decode.h"
#include "gqa_decode.cuh"
#include "mla_launch.cuh"
#include "tc_common.cuh"
#include "host_state.cuh"

namespace attn {

constexpr int kMlaH = 128;                 // heads = MMA M
constexpr int kMlaDc = 512, kMlaDr = 64, kMlaWidth = 576;
constexpr int kMlaCBox = 64 * 128;         // [64 tokens][64 cols] bf16
constexpr int kMlaMaxBoxes = 5;
constexpr int kMlaPrefetch = 4;            // blocks pulled into L2 ahead of the ring
constexpr int kMlaStageBytes = kMlaMaxBoxes * kMlaCBox;
constexpr int kMlaThreads = 512;           // warps 0-3 TMA/MMA, 4-11 softmax, 12-15 exchange
constexpr int kMlaThreadsF8 = 640;         // fp8: + warps 16-19 widening the codes
constexpr int kXchgWarps = 4;              // exchange warps: one thread per head row
constexpr int kSoftThreads = 256;
constexpr int kSoftWarps = kSoftThreads / 32;   // barriers count warps (one arrival each)
constexpr int kPBytes = kMlaH * 128;       // one P half: [128 heads][64 tokens] bf16
constexpr int kXBytes = kMlaH * 64 * 4;    // exchange buffer: 16 chunks x [128 rows] x 16 B
constexpr int kRawBox = 64 * 64;           // fp8: one box of codes, [64 tokens][64 columns]

// Shared-memory layout of one variant (bf16 cache, or fp8 codes + row scales).
template <bool F8> struct MlaCfg {
    static constexpr int kStages = F8 ? 2 : 3;      // bf16 stages the MMAs read
    static constexpr int kOffC = 0;
    static constexpr int kOffP = kOffC + kStages * kMlaStageBytes;
    static constexpr int kOffX = kOffP + 2 * kPBytes;   // receives the peer's partial S
    static constexpr int kOffStg = kOffX + kXBytes;     // stages this CTA's partial S
    static constexpr int kOffBar = kOffStg + kXBytes;
    static constexpr int kOffRed = kOffBar + 512;       // [2][2][128] row maxima + sums
    static constexpr int kOffRaw = kOffRed + 4096;      // fp8: raw code stages
    static constexpr int kRawStages = 2;
    static constexpr int kRawStageBytes = kMlaMaxBoxes * kRawBox + 1024;   // + 64 row scales
    static constexpr int kOffScale = kOffRaw + (F8 ? kRawStages * kRawStageBytes : 0);
    static constexpr int kSmemUsed = kOffScale + (F8 ? kStages * 64 * 4 : 0);
    static constexpr int kSmem = kSmemUsed + 1024;     // + alignment slack
    static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
    // Registers per thread by warpgroup (setmaxnreg), within the launch's
    // threads x registers (bf16: 512 x 128; fp8: 640 x 96): TMA/MMA warps,
    // softmax warps (two warpgroups), exchange warps, widening warps.
    static constexpr int kRegCtl = F8 ? 48 : 56;
    static constexpr int kRegSoft = F8 ? 152 : 184;
    static constexpr int kRegX = F8 ? 64 : 80;
    static constexpr int kRegW = 64;
    static_assert(128 * kRegCtl + 256 * kRegSoft + 128 * kRegX + (F8 ? 128 * kRegW : 0) <=
                      (F8 ? 640 * 96 : 512 * 128),
                  "register split");
};
constexpr int kMlaMaxStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 320;   // Q: 32 columns per box
constexpr float kRescaleThreshold = 8.0f;           // log2 units

struct MlaBars {
    uint64_t q_full, q_empty;
    uint64_t c_full[kMlaMaxStages], c_empty[kMlaMaxStages];
    uint64_t raw_full[2], raw_empty[2];   // fp8: code stages landed / widened
    uint64_t s_full, s_free;
    uint64_t p_full, pv_done, o_free;
    uint64_t x_full, x_free, stg_full, stg_free;
    uint64_t red_bar, sum_bar;
    uint64_t end_bar, mma_final;
    uint32_t tmem_base;
    int abort;
    PlanScratch plan;
};
static_assert(sizeof(MlaBars) <= 512, "barrier block");
static_assert(kTmemQ + 32 * kMlaMaxBoxes <= kTmemCols, "TMEM columns");

struct MlaParams {
    const __nv_bfloat16 *q_lat;    // [B][128][512]
    const __nv_bfloat16 *q_rope;   // [B][128][64]
    const void *latent;            // [num_blocks][64][576] bf16, or E4M3 codes (fp8)
    const float *lscale;           // fp8: [num_blocks][64] row scales
    const int32_t *seq_lens;
    const int32_t *block_table;
    float *ws_o;          // [slots][128][512]
    float *ws_lse;        // [slots][128]
    long long *ws_prefix; // [B + 1]
    unsigned *err;
    unsigned long long timeout_ns;
    float scale_log2;
    int B, max_blocks, num_blocks, num_clusters;
};

template <bool F8>
__global__ void __launch_bounds__(F8 ? kMlaThreadsF8 : kMlaThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_c, const MlaParams p) {
    using C = MlaCfg<F8>;
    constexpr int kMlaStages = C::kStages;
    constexpr int kOffC = C::kOffC, kOffP = C::kOffP, kOffX = C::kOffX, kOffStg = C::kOffStg,
                  kOffBar = C::kOffBar, kOffRed = C::kOffRed;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *sC = smem + kOffC;
    unsigned char *sP = smem + kOffP;
    unsigned char *sX = smem + kOffX;
    MlaBars *bars = reinterpret_cast<MlaBars *>(smem + kOffBar);
    volatile int *abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int cluster = (int)cluster_id_x();
    const int nbox = rank == 0 ? 4 : 5;          // 64-column boxes this CTA owns
    const int col0 = rank == 0 ? 0 : 256;

    // Programmatic dependent launch: the launch overlaps the previous kernel;
    // every input is read after the wait.  The combine may be scheduled as
    // soon as SMs free up (it waits for this grid to finish).
    pdl_wait_primary();
    pdl_launch_dependents();

    // ---- plan (both CTAs of the cluster compute the same range)
    PlanArgs pa{p.seq_lens, p.B, 1, Visibility{0, 0, 0}, p.max_blocks, p.num_clusters};
    plan_locate(pa, cluster, &bars->plan,
                (cluster == 0 && rank == 0) ? p.ws_prefix : nullptr, p.err);
    const long long W = bars->plan.total;
    const int P = working_ctas(W, p.num_clusters);
    if (cluster >= P) return;                      // uniform in the cluster
    const long long lo = cta_bound(cluster, W, P);
    const long long hi = cta_bound(cluster + 1, W, P);
    const int first_seq = bars->plan.seq;
    const long long first_base = bars->plan.base;
    const int n_tiles = (int)(hi - lo);

    // ---- set-up: barriers, TMEM, cluster handshake
    if (tid == 0) {
        mbar_init(&bars->q_full, kSoftWarps);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < kMlaStages; ++s) {
            mbar_init(&bars->c_full[s], F8 ? 4 : 1);    // widening warps, or the TMA
            mbar_init(&bars->c_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->raw_full[s], 1);
            mbar_init(&bars->raw_empty[s], 4);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, kXchgWarps);        // the exchange warps read S
        mbar_init(&bars->p_full, kSoftWarps);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_free, kSoftWarps);
        mbar_init(&bars->x_full, 1);               // own arrive.expect_tx + peer's bulk copy
        mbar_init(&bars->x_free, kSoftWarps);      // peer's softmax warps consumed my data
        mbar_init(&bars->stg_full, kXchgWarps);    // exchange warps staged my partial S
        mbar_init(&bars->stg_free, kSoftWarps);    // my softmax warps consumed it
        mbar_init(&bars->red_bar, kSoftWarps);
        mbar_init(&bars->sum_bar, kSoftWarps);
        mbar_init(&bars->end_bar, 1);
        mbar_init(&bars->mma_final, 2);            // one commit per issuing thread
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();   // the peer's barriers exist before any remote arrive
    const uint32_t tmem = bars->tmem_base;

    // Registers are re-split by warpgroup at the top of each role (MlaCfg).
    if (warp == 0) {
        regs_decrease<C::kRegCtl>();
        // ============================================================ TMA
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            constexpr uint32_t kElem = F8 ? 1 : 2;     // bytes per cached value
            tma_prefetch_map(&tm_c);
            TileCursorT<false> cur;
            cur.init(pa, lo, hi, first_seq, first_base);
            // Rank 0 also pulls whole blocks (all 576 columns, contiguous)
            // into L2 kMlaPrefetch tiles ahead, so the ring's loads of both
            // CTAs are served from L2 rather than waiting on HBM.
            TileCursorT<false> pf;
            pf.init(pa, lo, hi, first_seq, first_base);
            auto prefetch_next = [&]() {
                if (rank != 0 || pf.done()) return;
                const int pb = p.block_table[(size_t)pf.w.b * p.max_blocks + pf.logical_block()];
                if (pb >= 0 && pb < p.num_blocks)
                    bulk_prefetch_l2(static_cast<const unsigned char *>(p.latent) +
                                         (size_t)pb * 64 * kMlaWidth * kElem,
                                     64 * kMlaWidth * kElem);
                pf.next();
            };
            for (int k = 0; k < kMlaPrefetch; ++k) prefetch_next();
            // bf16: straight into the stages the MMAs read; fp8: codes and
            // row scales into a raw stage that warp 3 widens.
            constexpr int kRing = F8 ? C::kRawStages : kMlaStages;
            uint64_t *ring_full = F8 ? bars->raw_full : bars->c_full;
            uint64_t *ring_empty = F8 ? bars->raw_empty : bars->c_empty;
            int tile = 0;
            while (!cur.done()) {
                prefetch_next();
                const int st = tile % kRing;
                if (tile >= kRing &&
                    !mbar_wait(&ring_empty[st], (uint32_t)(((tile - kRing) / kRing) & 1),
                               p.timeout_ns, p.err, abort_flag))
                    break;
                int phys = p.block_table[(size_t)cur.w.b * p.max_blocks + cur.logical_block()];
                const bool bad = phys < 0 || phys >= p.num_blocks;
                if (bad) {
                    raise_error(p.err, kErrBadBlock);
                    phys = p.num_blocks;            // wholly out of bounds: zero fill
                }
                if constexpr (F8) {
                    unsigned char *dst = smem + C::kOffRaw + st * C::kRawStageBytes;
                    float *dsc = reinterpret_cast<float *>(dst + kMlaMaxBoxes * kRawBox);
                    if (bad)   // no scale row to copy: zeros (the codes are zero-filled too)
                        for (int t = 0; t < 64; ++t) dsc[t] = 0.f;
                    mbar_arrive_expect_tx(&ring_full[st], nbox * kRawBox + (bad ? 0 : 256));
                    for (int i = 0; i < nbox; ++i)
                        tma_load_2d(dst + i * kRawBox, &tm_c, col0 + i * 64, phys * 64,
                                    &ring_full[st], pol);
                    if (!bad) bulk_load(dsc, p.lscale + (size_t)phys * 64, 256, &ring_full[st]);
                } else {
                    unsigned char *dst = sC + st * kMlaStageBytes;
                    mbar_arrive_expect_tx(&ring_full[st], nbox * kMlaCBox);
                    for (int i = 0; i < nbox; ++i)
                        tma_load_2d(dst + i * kMlaCBox, &tm_c, col0 + i * 64, phys * 64,
                                    &ring_full[st], pol);
                }
                cur.next();
                ++tile;
            }
            // Every issued load must have landed before the CTA exits.
            for (int t = tile - kRing < 0 ? 0 : tile - kRing; t < tile; ++t)
                mbar_wait(&ring_full[t % kRing], (uint32_t)((t / kRing) & 1), p.timeout_ns,
                          p.err, nullptr);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 2) {
        regs_decrease<C::kRegCtl>();
        // ============================================================ MMA
        // Lane 0 of warp 1 issues S(n) = Q C(n)^T for every tile in order,
        // lane 0 of warp 2 issues O += P(i) C(i); each waits only on its own
        // inputs, so the two streams of MMAs overlap.  The stage is released
        // by the commit after P V(i): S(i) has completed by then (the softmax
        // read it before producing P(i)).  Barriers are polled.
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
                TileCursorT<false> cs;
                cs.init(pa, lo, hi, first_seq, first_base);
                int seg_s = 0;
                for (int n = 0; n < n_tiles; ++n) {
                    // S(n) into the S buffer once the softmax has read S(n - 1).
                    const bool first = cs.t == 0, last = cs.t == cs.len - 1;
                    const int st = n % kMlaStages;
                    if (first && !wait(&bars->q_full, (uint32_t)(seg_s & 1))) break;
                    if (!wait(&bars->c_full[st], (uint32_t)((n / kMlaStages) & 1))) break;
                    if (n > 0 && !wait(&bars->s_free, (uint32_t)((n - 1) & 1))) break;
                    tc_fence_after();
                    const uint32_t cst = c_base + st * kMlaStageBytes;
                    for (int bx = 0; bx < nbox; ++bx)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t b =
                                umma_desc_sw128(cst + bx * kMlaCBox + k * 32, 16, 1024);
                            umma_bf16_ts(tmem + kTmemS, tmem + kTmemQ + 32 * bx + 8 * k, b,
                                         idesc_s, (bx | k) != 0);
                        }
                    umma_commit(&bars->s_full);
                    if (last) umma_commit(&bars->q_empty);
                    if (first) ++seg_s;
                    cs.next();
                }
            } else {
                constexpr uint32_t idesc_pv =
                    F8 ? umma_idesc_f16(128, 256, 0, 1) : umma_idesc_bf16(128, 256, 0, 1);
                const uint32_t p_base = smem_u32(sP);
                TileCursorT<false> cv;
                cv.init(pa, lo, hi, first_seq, first_base);
                int seg_v = 0;
                for (int i = 0; i < n_tiles; ++i) {
                    // O += P_hi C + P_lo C (fp8: O += P C, P in f16); a
                    // segment's first P V overwrites O once the previous
                    // segment's output has been read.
                    const bool first = cv.t == 0;
                    if (!wait(&bars->p_full, (uint32_t)(i & 1))) break;
                    if (first && seg_v > 0 && !wait(&bars->o_free, (uint32_t)((seg_v - 1) & 1)))
                        break;
                    tc_fence_after();
                    const int st = i % kMlaStages;
                    const uint32_t cst = c_base + st * kMlaStageBytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t b = umma_desc_sw128(cst + k * 2048, kMlaCBox, 1024);
                        const uint64_t a_hi = umma_desc_sw128(p_base + k * 32, 16, 1024);
                        const uint64_t a_lo = umma_desc_sw128(p_base + kPBytes + k * 32, 16, 1024);
                        umma_bf16(tmem + kTmemO, a_hi, b, idesc_pv, !(first && k == 0));
                        if constexpr (!F8) umma_bf16(tmem + kTmemO, a_lo, b, idesc_pv, 1);
                    }
                    umma_commit(&bars->c_empty[st]);
                    umma_commit(&bars->pv_done);
                    if (first) ++seg_v;
                    cv.next();
                }
            }
            // Both issuers' MMAs complete before TMEM is released.
            umma_commit(&bars->mma_final);
            mbar_wait(&bars->mma_final, 0, p.timeout_ns, p.err, nullptr);
        }
        __syncwarp();
    } else if (warp == 3) {
        regs_decrease<C::kRegCtl>();
    } else if (F8 && warp >= 16) {
        // ================================================ fp8 -> f16 widening
        regs_decrease<C::kRegW>();
        // The codes are widened to f16 with the hardware conversion (exact:
        // every E4M3 value is an f16 value); the fp8 variant runs its MMAs on
        // f16 operands.
        if constexpr (F8) {
            const int wt = tid - 512;            // widening thread 0..127
            for (int tile = 0; tile < n_tiles; ++tile) {
                const int rs = tile % C::kRawStages, st = tile % kMlaStages;
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&bars->raw_full[rs], (uint32_t)((tile / C::kRawStages) & 1),
                                          p.timeout_ns, p.err, abort_flag)))
                    break;
                if (tile >= kMlaStages &&
                    !__all_sync(0xffffffffu,
                                mbar_wait(&bars->c_empty[st],
                                          (uint32_t)(((tile - kMlaStages) / kMlaStages) & 1),
                                          p.timeout_ns, p.err, abort_flag)))
                    break;
                const unsigned char *raw = smem + C::kOffRaw + rs * C::kRawStageBytes;
                unsigned char *dst = sC + st * kMlaStageBytes;
                // item: 16 codes (group g of row t of box bx) -> 2 swizzled chunks
                for (int idx = wt; idx < nbox * 256; idx += 128) {
                    const int bx = idx >> 8, t = (idx >> 2) & 63, g = idx & 3;
                    const uint4 codes =
                        *reinterpret_cast<const uint4 *>(raw + bx * kRawBox + t * 64 + g * 16);
                    const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
                    uint32_t w[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) e4m3x4_to_f16x4(cw[k], w[2 * k], w[2 * k + 1]);
                    unsigned char *drow = dst + bx * kMlaCBox + t * 128;
                    *reinterpret_cast<uint4 *>(drow + (((2 * g) ^ (t & 7)) * 16)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4 *>(drow + (((2 * g + 1) ^ (t & 7)) * 16)) =
                        make_uint4(w[4], w[5], w[6], w[7]);
                }
                const float *rsc = reinterpret_cast<const float *>(raw + kMlaMaxBoxes * kRawBox);
                float *ssc = reinterpret_cast<float *>(smem + C::kOffScale) + st * 64;
                if (wt < 64) ssc[wt] = rsc[wt];
                fence_proxy_async_smem();      // the MMAs read the widened stage
                mbar_arrive_warp(&bars->raw_empty[rs]);
                mbar_arrive_warp(&bars->c_full[st]);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ============================================ Q load, softmax, epilogue
        regs_increase<C::kRegSoft>();
        // Two threads per head row: warps w and w + 4 share TMEM lanes
        // 32*(w%4) .. +31; half h takes tokens [32h, 32h+32) of each tile and
        // output columns [128h, 128h+128) of this CTA's 256.
        const int q4 = warp & 3, h = (warp - 4) >> 2;
        const int row = 32 * q4 + lane;                      // head = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
        const uint32_t x_free_peer = map_to_rank(&bars->x_free, peer);
        const unsigned char *own_row = smem + kOffStg + row * 16;   // staged by the exchange warps
        const unsigned char *peer_row = sX + row * 16;             // received from the peer
        const bool sender = (warp == 4 && lane == 0);              // arms the receive barrier
        unsigned char *prow = sP + row * 128;
        float *red = reinterpret_cast<float *>(smem + kOffRed);   // [2][2][128] then sums
        // Wait outcomes are made warp-uniform: the TMEM loads and stores are
        // warp-collective and must never run in a partial warp.
        auto all = [](bool v) { return __all_sync(0xffffffffu, v); };
        const int box_lo = h == 0 ? 0 : (nbox + 1) / 2;
        const int box_hi = h == 0 ? (nbox + 1) / 2 : nbox;

        // Write this head's query slice (this half's boxes) into TMEM.
        auto load_q = [&](int b, int q_seg) -> bool {
            if (q_seg > 0 && !all(mbar_wait(&bars->q_empty, (uint32_t)((q_seg - 1) & 1),
                                            p.timeout_ns, p.err, abort_flag)))
                return false;
            tc_fence_after();
            for (int bx = box_lo; bx < box_hi; ++bx) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    (rank == 1 && bx == 4)
                        ? p.q_rope + ((size_t)b * kMlaH + row) * kMlaDr
                        : p.q_lat + ((size_t)b * kMlaH + row) * kMlaDc + col0 + 64 * bx);
                uint32_t r[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 v = __ldg(src + j);
                    r[4 * j] = v.x; r[4 * j + 1] = v.y; r[4 * j + 2] = v.z; r[4 * j + 3] = v.w;
                }
                if constexpr (F8) {
                    // f16 operands: the query pairs converted (exact within f16's range)
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = bf16x2_to_f16x2(r[j]);
                }
                tmem_st32(trow + kTmemQ + 32 * bx, r);
            }
            tc_fence_before();
            mbar_arrive_warp(&bars->q_full);
            return true;
        };
        TileCursorT<false> cur, nxt;
        cur.init(pa, lo, hi, first_seq, first_base);
        nxt.init(pa, lo, hi, first_seq, first_base);
        int q_seg = 0, n_seg = 0;
        float m_run = -1e30f, l_run = 0.f;                // l_run: this half's sum
        if (sender && n_tiles > 0) mbar_arrive_expect_tx(&bars->x_full, kXBytes);   // tile 0
        bool ok = load_q(nxt.w.b, q_seg++);
        for (int i = 0; ok && i < n_tiles; ++i) {
            float s[32];
            const bool first = cur.t == 0, last = cur.t == cur.len - 1;
            const int b = cur.w.b, T = cur.w.T;
            const int nvalid = T - (cur.logical_block() * 64 + 32 * h);   // valid in this half

            // this CTA's and the peer's partial scores of tile i, summed and
            // scaled to log2 units
            if (!all(mbar_wait(&bars->stg_full, (uint32_t)(i & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            if (!all(mbar_wait(&bars->x_full, (uint32_t)(i & 1), p.timeout_ns, p.err, abort_flag)))
                break;
            const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
            // fp8: this half's 32 row scales of tile i (kept with its stage)
            const float *tsc = reinterpret_cast<const float *>(smem + C::kOffScale) +
                               (i % kMlaStages) * 64 + 32 * h;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 u =
                    *reinterpret_cast<const float4 *>(own_row + (8 * h + c) * (kMlaH * 16));
                const float4 v =
                    *reinterpret_cast<const float4 *>(peer_row + (8 * h + c) * (kMlaH * 16));
                float2 a = __fadd2_rn(make_float2(u.x, u.y), make_float2(v.x, v.y));
                float2 bb = __fadd2_rn(make_float2(u.z, u.w), make_float2(v.z, v.w));
                a = __fmul2_rn(a, sl2);
                bb = __fmul2_rn(bb, sl2);
                if constexpr (F8) {
                    const float4 r = *reinterpret_cast<const float4 *>(tsc + 4 * c);
                    a = __fmul2_rn(a, make_float2(r.x, r.y));
                    bb = __fmul2_rn(bb, make_float2(r.z, r.w));
                }
                s[4 * c] = a.x; s[4 * c + 1] = a.y; s[4 * c + 2] = bb.x; s[4 * c + 3] = bb.y;
            }
            // arm the receive barrier for tile i + 1 (the peer's copy may
            // land first: the byte count then runs negative until this),
            // then let the exchange warps restage and the peer resend
            if (sender && i + 1 < n_tiles) mbar_arrive_expect_tx(&bars->x_full, kXBytes);
            mbar_arrive_warp(&bars->stg_free);
            mbar_arrive_remote_relaxed_warp(x_free_peer);

            // the next tile's query (a new sequence) into TMEM ahead of its S
            nxt.next();
            if (i + 1 < n_tiles && nxt.t == 0 && !load_q(nxt.w.b, q_seg++)) break;

            if (nvalid < 32) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j >= nvalid) s[j] = kNegInf;
            }
            float mx = s[0];
#pragma unroll
            for (int j = 1; j < 32; ++j) mx = fmaxf(mx, s[j]);
            // row max across the two halves (double-buffered by tile parity)
            float *rb = red + (i & 1) * 256;
            rb[h * 128 + row] = mx;
            mbar_arrive_warp(&bars->red_bar);
            if (!all(mbar_wait(&bars->red_bar, (uint32_t)(i & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            mx = fmaxf(mx, rb[(h ^ 1) * 128 + row]);

            // online softmax (log2 domain), lazy rescale -- same decision in
            // both halves and both CTAs (same scores)
            bool rescale = false;
            float alpha = 1.f;
            if (first) {
                m_run = mx;
                l_run = 0.f;
            } else if (mx > m_run + kRescaleThreshold) {
                alpha = exp2_approx(m_run - mx);
                m_run = mx;
                l_run *= alpha;
                rescale = true;
            }
            float2 sum2 = make_float2(0.f, 0.f);
            const float2 m2 = make_float2(-m_run, -m_run);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const float2 d = __fadd2_rn(make_float2(s[j], s[j + 1]), m2);
                s[j] = exp2_approx(d.x);
                s[j + 1] = exp2_approx(d.y);
                sum2 = __fadd2_rn(sum2, make_float2(s[j], s[j + 1]));
            }
            l_run += sum2.x + sum2.y;
            if constexpr (F8) {
                // the values are code values x row scale: scale each token's weight
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 r = *reinterpret_cast<const float4 *>(tsc + j);
                    s[j] *= r.x; s[j + 1] *= r.y; s[j + 2] *= r.z; s[j + 3] *= r.w;
                }
            }

            // P and O may be touched once the previous P V has completed
            if (i >= 1 && !all(mbar_wait(&bars->pv_done, (uint32_t)((i - 1) & 1),
                                         p.timeout_ns, p.err, abort_flag)))
                break;
            if constexpr (F8) {
                // one f16 P (11 significant bits): no P_lo product needed
#pragma unroll
                for (int c = 0; c < 4; ++c) {      // 8 tokens per 16-byte chunk
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        w[k] = pack_f16x2(s[8 * c + 2 * k], s[8 * c + 2 * k + 1]);
                    const int off = ((4 * h + c) ^ (row & 7)) * 16;
                    *reinterpret_cast<uint4 *>(prow + off) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {          // 8 tokens per 16-byte chunk
                    uint32_t hi_w[4], lo_w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float a = s[8 * c + 2 * k], bb = s[8 * c + 2 * k + 1];
                        hi_w[k] = pack_bf16x2(a, bb);
                        const float2 r = __fadd2_rn(
                            make_float2(a, bb),
                            make_float2(-__uint_as_float(hi_w[k] << 16),
                                        -__uint_as_float(hi_w[k] & 0xFFFF0000u)));
                        lo_w[k] = pack_bf16x2(r.x, r.y);
                    }
                    const int off = ((4 * h + c) ^ (row & 7)) * 16;
                    *reinterpret_cast<uint4 *>(prow + off) =
                        make_uint4(hi_w[0], hi_w[1], hi_w[2], hi_w[3]);
                    *reinterpret_cast<uint4 *>(prow + kPBytes + off) =
                        make_uint4(lo_w[0], lo_w[1], lo_w[2], lo_w[3]);
                }
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, rescale)) {   // rows without a new max use alpha = 1
                float o[32];
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    tmem_ld32(trow + kTmemO + 128 * h + 32 * ch, o);
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(o[j] * alpha);
                    tmem_st32(trow + kTmemO + 128 * h + 32 * ch, r);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive_warp(&bars->p_full);

            if (last) {
                float *sb = red + 512 + (n_seg & 1) * 256;
                sb[h * 128 + row] = l_run;
                mbar_arrive_warp(&bars->sum_bar);
                if (!all(mbar_wait(&bars->sum_bar, (uint32_t)(n_seg & 1), p.timeout_ns, p.err,
                                   abort_flag)))
                    break;
                const float l_tot = l_run + sb[(h ^ 1) * 128 + row];
                ++n_seg;
                if (!all(mbar_wait(&bars->pv_done, (uint32_t)(i & 1), p.timeout_ns, p.err,
                                   abort_flag)))
                    break;
                tc_fence_after();
                const long long slot = (long long)b + cluster;
                float *dst = p.ws_o + ((size_t)slot * kMlaH + row) * kMlaDc + col0 + 128 * h;
                const float inv = 1.f / l_tot;
                float o[32];
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    tmem_ld32(trow + kTmemO + 128 * h + 32 * ch, o);
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(dst + 32 * ch + j) =
                            make_float4(o[j] * inv, o[j + 1] * inv, o[j + 2] * inv,
                                        o[j + 3] * inv);
                }
                if (rank == 0 && h == 0) p.ws_lse[slot * kMlaH + row] = m_run + log2f(l_tot);
                tc_fence_before();
                mbar_arrive_warp(&bars->o_free);
            }
            cur.next();
        }
    }

    if (warp >= 12 && warp < 16) {
        // ============================================= score exchange
        // One thread per head row (TMEM lane) reads this CTA's partial S(i)
        // (64 tokens) from TMEM, stages it in shared memory -- where this
        // CTA's softmax reads it too -- and frees the TMEM buffer for S(i + 1);
        // one thread then sends the staged tile to the peer with a bulk copy.
        // Staging tile i waits until this CTA's softmax has consumed tile
        // i - 1 (stg_free) and the peer has consumed its copy of it (x_free:
        // the copy out of the staging buffer has completed and the peer's
        // receive buffer is free), so the softmax threads never wait on the
        // exchange themselves.
        regs_decrease<C::kRegX>();
        const int q4 = warp & 3;
        const int row = 32 * q4 + lane;
        const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
        const uint32_t x_peer = map_to_rank(sX, peer);
        const uint32_t x_full_peer = map_to_rank(&bars->x_full, peer);
        unsigned char *sStg = smem + kOffStg;
        unsigned char *stg = sStg + row * 16;
        const bool issuer = warp == 12 && lane == 0;
        auto all = [](bool v) { return __all_sync(0xffffffffu, v); };
        for (int i = 0; i < n_tiles; ++i) {
            if (i >= 1 &&
                !all(mbar_wait(&bars->stg_free, (uint32_t)((i - 1) & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            if (i >= 1 &&
                !all(mbar_wait(&bars->x_free, (uint32_t)((i - 1) & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            if (!all(mbar_wait(&bars->s_full, (uint32_t)(i & 1), p.timeout_ns, p.err,
                               abort_flag)))
                break;
            tc_fence_after();
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float v[32];
                tmem_ld32(trow + kTmemS + 32 * hh, v);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<float4 *>(stg + (8 * hh + c) * (kMlaH * 16)) =
                        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
            tc_fence_before();
            mbar_arrive_warp(&bars->s_free);
            fence_proxy_async_smem();          // the bulk copy reads the staging buffer
            mbar_arrive_warp(&bars->stg_full);
            if (issuer &&
                mbar_wait(&bars->stg_full, (uint32_t)(i & 1), p.timeout_ns, p.err, abort_flag))
                bulk_copy_to_peer(x_peer, sStg, kXBytes, x_full_peer);
            __syncwarp();
        }
    }

    // ---- tear-down: release TMEM, then a bounded handshake with the peer so
    // that neither CTA exits while the other may still touch its memory.
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (tid == 0) {
        mbar_arrive_remote(map_to_rank(&bars->end_bar, peer));
        mbar_wait_cluster(&bars->end_bar, 0, p.timeout_ns, p.err, nullptr);
    }
}

// -------------------------------------------------------------- host side
namespace {

// ---- combine of the per-cluster partials, for shapes with few partials per
// sequence (many sequences): z[b, h] = sum_s 2^(lse_s - L) O_s /
// sum_s 2^(lse_s - L) over the partials of sequence b, one per cluster whose
// tile range meets it, in cluster order (fixed, deterministic).  A partial
// with lse = -inf has weight zero.  One CTA makes 8 heads x 512 columns:
// warp w computes head w's weights once (shared memory), then every thread
// accumulates four float4 of output over the partials, so each CTA's set-up
// round trips (sequence length, prefix, log-sum-exps) are paid for 4096
// outputs.  The host picks it when sequences expect few partials; a ragged
// sequence that spans more than kMlaCombMaxW clusters still combines
// correctly (its further weights are recomputed from the log-sum-exps).
// Shapes with many partials per sequence use the generic combine, which
// spreads one output over several threads.
constexpr int kMlaCombThreads = 256;
constexpr int kMlaCombHeads = 8;                 // heads per CTA
constexpr int kMlaCombMaxW = 128;                // weights per head held in shared memory
constexpr int kMlaCombExpected = 8;              // host: expected partials per sequence
constexpr int kMlaCombVec = kMlaCombHeads * kMlaDc / 4 / kMlaCombThreads;   // float4 per thread

struct MlaCombineParams {
    const int32_t *seq_lens;
    const long long *ws_prefix;
    const float *ws_o;      // [slots][128][512]
    const float *ws_lse;    // [slots][128]
    __nv_bfloat16 *out;     // [B][128][512]
    int B, max_blocks, num_clusters;
};

__global__ void __launch_bounds__(kMlaCombThreads)
mla_combine_kernel(const MlaCombineParams p) {
    __shared__ float s_w[kMlaCombHeads][kMlaCombMaxW];
    __shared__ float s_max[kMlaCombHeads], s_inv[kMlaCombHeads];
    __shared__ long long s_first;
    __shared__ int s_n;
    pdl_wait_primary();                           // the partials are the decode's output
    constexpr int kParts = kMlaH / kMlaCombHeads;
    const int b = blockIdx.x / kParts;
    const int h0 = (blockIdx.x % kParts) * kMlaCombHeads;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        int fb, sb;
        bool bad;
        const int nb = visible_blocks<false>(p.seq_lens[b], Visibility{0, 0, 0}, p.max_blocks,
                                             &fb, &sb, &bad, b);
        int n = 0;
        long long first = 0;
        if (nb > 0) {
            const long long W = p.ws_prefix[p.B];
            const int P = working_ctas(W, p.num_clusters);
            const long long s_u = p.ws_prefix[b];
            const int c0 = cta_of(s_u, W, P);
            const int c1 = cta_of(s_u + nb - 1, W, P);
            n = c1 - c0 + 1;
            first = (long long)b + c0;
        }
        s_n = n;
        s_first = first;
    }
    __syncthreads();
    const int n = s_n;
    const long long s0 = s_first;
    // Weights of head h0 + warp over the n partials (lane-strided).
    const float *lse = p.ws_lse + (size_t)s0 * kMlaH + h0;    // [partial][head]
    if (warp < kMlaCombHeads) {
        float L = kNegInf;
        for (int i = lane; i < n; i += 32) L = fmaxf(L, lse[(size_t)i * kMlaH + warp]);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, m));
        float den = 0.f;
        for (int i = lane; i < n; i += 32) {
            const float w = L == kNegInf ? 0.f : exp2f(lse[(size_t)i * kMlaH + warp] - L);
            if (i < kMlaCombMaxW) s_w[warp][i] = w;
            den += w;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) den += __shfl_xor_sync(0xffffffffu, den, m);
        if (lane == 0) {
            s_max[warp] = L;
            s_inv[warp] = den > 0.f ? 1.f / den : 0.f;
        }
    }
    __syncthreads();
    float4 acc[kMlaCombVec];
#pragma unroll
    for (int k = 0; k < kMlaCombVec; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *src = p.ws_o + ((size_t)s0 * kMlaH + h0) * kMlaDc;
    for (int i = 0; i < n; ++i) {
        const float *pi = src + (size_t)i * kMlaH * kMlaDc;
        float4 v[kMlaCombVec];
#pragma unroll
        for (int k = 0; k < kMlaCombVec; ++k)
            v[k] = *reinterpret_cast<const float4 *>(pi + 4 * (tid + k * kMlaCombThreads));
#pragma unroll
        for (int k = 0; k < kMlaCombVec; ++k) {
            const int hh = (tid + k * kMlaCombThreads) / (kMlaDc / 4);
            const float w = i < kMlaCombMaxW ? s_w[hh][i]
                            : s_max[hh] == kNegInf
                                ? 0.f
                                : exp2f(lse[(size_t)i * kMlaH + hh] - s_max[hh]);
            acc[k].x = fmaf(w, v[k].x, acc[k].x);
            acc[k].y = fmaf(w, v[k].y, acc[k].y);
            acc[k].z = fmaf(w, v[k].z, acc[k].z);
            acc[k].w = fmaf(w, v[k].w, acc[k].w);
        }
    }
    __nv_bfloat16 *out = p.out + ((size_t)b * kMlaH + h0) * kMlaDc;
    const bool vec = (reinterpret_cast<uintptr_t>(out) & 7) == 0;
#pragma unroll
    for (int k = 0; k < kMlaCombVec; ++k) {
        const int q = tid + k * kMlaCombThreads;
        const float inv = s_inv[q / (kMlaDc / 4)];
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[k].x * inv, acc[k].y * inv);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[k].z * inv, acc[k].w * inv);
        if (vec) {
            uint2 u;
            u.x = *reinterpret_cast<const uint32_t *>(&lo);
            u.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(out + 4 * q) = u;
        } else {
            out[4 * q] = lo.x;
            out[4 * q + 1] = lo.y;
            out[4 * q + 2] = hi.x;
            out[4 * q + 3] = hi.y;
        }
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// The latent cache as a row-major matrix [num_blocks * 64][576] with boxes of
// [64 rows][64 values]: bf16 with 128-byte swizzle (the MMAs read the boxes
// directly), or fp8 codes unswizzled (widened into the swizzled layout).
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, bool fp8) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t elem = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)kMlaWidth, rows};
    cuuint64_t strides[1] = {kMlaWidth * elem};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              fp8 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Clusters of two that can be resident at once (one CTA per SM), so that the
// persistent ranges all run in a single wave.  Cached per device and variant.
template <bool F8>
int max_resident_clusters(int num_sms) {
    static std::mutex mu;
    static int cache[kMaxDevices] = {};
    const int dev = current_device();
    if (dev < 0) return -1;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(num_sms);
        cfg.blockDim = dim3(F8 ? kMlaThreadsF8 : kMlaThreads);
        cfg.dynamicSmemBytes = MlaCfg<F8>::kSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, mla_decode_kernel<F8>, &cfg) != cudaSuccess ||
            n <= 0)
            n = num_sms / 2;
        cache[dev] = n < num_sms / 2 ? n : num_sms / 2;
        if (cache[dev] <= 0) cache[dev] = 1;
    }
    return cache[dev];
}

template <bool F8>
int mla_launch(const MlaParams &mp, const CUtensorMap &tc, int clusters, cudaStream_t stream,
               cudaEvent_t ev_start, cudaEvent_t ev_stop) {
    static PerDeviceFlag configured;   // the attribute is per function and device
    if (configure_once_per_device(configured, [] {
            return cudaFuncSetAttribute(mla_decode_kernel<F8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        MlaCfg<F8>::kSmem);
        }) != cudaSuccess)
        return ATTN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(F8 ? kMlaThreadsF8 : kMlaThreads);
    cfg.dynamicSmemBytes = MlaCfg<F8>::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (ev_start) cudaEventRecord(ev_start, stream);
    if (cudaLaunchKernelEx(&cfg, mla_decode_kernel<F8>, tc, mp) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (ev_stop) cudaEventRecord(ev_stop, stream);
    return ATTN_OK;
}

}  // namespace

int mla_decode_entry(const void *q_latent, const void *q_rope, const void *latent_cache,
                     const float *latent_scale, const int32_t *seq_lens,
                     const int32_t *block_table, void *out, int B, int H, float scale,
                     cudaStream_t stream, int max_blocks, int num_blocks, int num_sms,
                     int forced_ctas, unsigned *err, const WorkspaceFn &workspace,
                     cudaEvent_t ev_start, cudaEvent_t ev_stop) {
    if (H != kMlaH) return ATTN_ERR_UNSUPPORTED;
    if ((long long)num_blocks * 64 > (1ll << 31) - 64 || (long long)B * kMlaH > (1ll << 31))
        return ATTN_ERR_ARG;
    const bool fp8 = latent_scale != nullptr;
    int clusters = forced_ctas > 0 ? forced_ctas
                                   : (fp8 ? max_resident_clusters<true>(num_sms)
                                          : max_resident_clusters<false>(num_sms));
    if (clusters <= 0) return ATTN_ERR_CUDA;
    const long long slots = (long long)B + clusters;
    const size_t o_bytes = round256((size_t)slots * kMlaH * kMlaDc * sizeof(float));
    const size_t lse_bytes = round256((size_t)slots * kMlaH * sizeof(float));
    const size_t pre_bytes = round256((size_t)(B + 1) * sizeof(long long));
    void *ws = nullptr;
    int rc = workspace(o_bytes + lse_bytes + pre_bytes, &ws);
    if (rc) return rc;
    unsigned char *w = static_cast<unsigned char *>(ws);

    CUtensorMap tc;
    if (!make_map(&tc, latent_cache, (uint64_t)num_blocks * 64, fp8)) return ATTN_ERR_CUDA;

    MlaParams mp{};
    mp.q_lat = static_cast<const __nv_bfloat16 *>(q_latent);
    mp.q_rope = static_cast<const __nv_bfloat16 *>(q_rope);
    mp.latent = latent_cache;
    mp.lscale = latent_scale;
    mp.seq_lens = seq_lens;
    mp.block_table = block_table;
    mp.ws_o = reinterpret_cast<float *>(w);
    mp.ws_lse = reinterpret_cast<float *>(w + o_bytes);
    mp.ws_prefix = reinterpret_cast<long long *>(w + o_bytes + lse_bytes);
    mp.err = err;
    mp.timeout_ns = kDefaultTimeoutNs;
    mp.scale_log2 = scale * 1.4426950408889634f;
    mp.B = B;
    mp.max_blocks = max_blocks;
    mp.num_blocks = num_blocks;
    mp.num_clusters = clusters;
    rc = fp8 ? mla_launch<true>(mp, tc, clusters, stream, ev_start, ev_stop)
             : mla_launch<false>(mp, tc, clusters, stream, ev_start, ev_stop);
    if (rc) return rc;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kCombineThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Few expected partials per sequence and enough sequences to fill the
    // SMs: the 8-head combine; else the generic one.
    if (clusters / B + 1 <= kMlaCombExpected &&
        (long long)B * (kMlaH / kMlaCombHeads) >= num_sms) {
        MlaCombineParams mc{};
        mc.seq_lens = seq_lens;
        mc.ws_prefix = mp.ws_prefix;
        mc.ws_o = mp.ws_o;
        mc.ws_lse = mp.ws_lse;
        mc.out = static_cast<__nv_bfloat16 *>(out);
        mc.B = B;
        mc.max_blocks = max_blocks;
        mc.num_clusters = clusters;
        cfg.gridDim = dim3(B * (kMlaH / kMlaCombHeads));
        cfg.blockDim = dim3(kMlaCombThreads);
        return cudaLaunchKernelEx(&cfg, mla_combine_kernel, mc) == cudaSuccess ? ATTN_OK
                                                                             : ATTN_ERR_CUDA;
    }
    CombineParams cp{};
    cp.seq_lens = seq_lens;
    cp.ws_prefix = mp.ws_prefix;
    cp.ws_o = mp.ws_o;
    cp.ws_lse = mp.ws_lse;
    cp.out = out;
    cp.B = B;
    cp.H_q = kMlaH;
    cp.H_kv = 1;
    cp.group = kMlaH;
    cp.n_hc = 1;
    cp.max_blocks = max_blocks;
    cp.vis = Visibility{0, 0, 0};
    cp.num_ctas = clusters;
    cp.D = kMlaDc;
    cp.HC = kMlaH;
    cp.copies = 1;
    cp.lanes = combine_lanes(clusters / B + 1);
    cp.blocks_per_unit = combine_blocks_per_unit(kMlaH, kMlaDc, cp.lanes);
    cfg.gridDim = dim3(B * cp.blocks_per_unit);
    return cudaLaunchKernelEx(&cfg, combine_kernel<__nv_bfloat16>, cp) == cudaSuccess
               ? ATTN_OK
               : ATTN_ERR_CUDA;
}

}  // namespace attn
