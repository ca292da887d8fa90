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
// with 2-D TMA (128-byte swizzle), and no cache byte is read twice.
//   * S = Q C^T is a 128 x 64 (heads x tokens) tcgen05 MMA with K = 256 or
//     320 per CTA, accumulated in TMEM; the two partial S are exchanged
//     through distributed shared memory and summed identically in both CTAs.
//   * Softmax runs one thread per head row directly on the TMEM rows (no
//     cross-thread reductions); the running max is only raised when it grows
//     by more than 2^8, so O is rescaled rarely (the result is exact either
//     way: numerator and denominator use the same max).
//   * P is split into two bf16 halves, P = P_hi + P_lo (P_lo = the rounding
//     remainder), so the weights keep ~16 significant bits instead of bf16's
//     8; both halves (128 x 64, swizzled like a TMA tile) are A operands of
//     O += P_hi C + P_lo C, 128 x 256 MMAs whose B operand is the same C tile
//     read MN-major.  Each CTA keeps its 256 output columns in TMEM.
//   * Warp 0 issues TMA, warp 1 issues MMAs, warps 4-7 do softmax and the
//     epilogue.  Every wait is bounded; TMEM is always freed; the final
//     cluster handshake is a bounded mbarrier exchange.
// Each (sequence, cluster) segment writes an fp32 partial (O/l and log2-sum-
// exp) that the combine kernel reduces in cluster order.
#include <mutex>
#include <vector>

#include "attn_decode.h"
#include "gqa_decode.cuh"
#include "mla_launch.cuh"
#include "tc_common.cuh"

namespace attn {

constexpr int kMlaH = 128;                 // heads = MMA M
constexpr int kMlaDc = 512, kMlaDr = 64, kMlaWidth = 576;
constexpr int kMlaQBox = 128 * 128;        // [128 heads][64 cols] bf16
constexpr int kMlaCBox = 64 * 128;         // [64 tokens][64 cols] bf16
constexpr int kMlaMaxBoxes = 5;
constexpr int kMlaStages = 2;
constexpr int kMlaThreads = 256;
constexpr int kOffQ = 0;
constexpr int kOffC = kOffQ + kMlaMaxBoxes * kMlaQBox;
constexpr int kOffP = kOffC + kMlaStages * kMlaMaxBoxes * kMlaCBox;
constexpr int kPBytes = kMlaH * 128;       // one P half: [128 heads][64 tokens] bf16
constexpr int kOffX = kOffP + 2 * kPBytes;
constexpr int kOffBar = kOffX + kMlaH * 64 * 4;
constexpr int kMlaSmemUsed = kOffBar + 512;
constexpr int kMlaSmem = kMlaSmemUsed + 1024;       // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS = 256;       // S buffers at 256, 320
constexpr float kRescaleThreshold = 8.0f;           // log2 units

struct MlaBars {
    uint64_t q_full, q_empty;
    uint64_t c_full[kMlaStages], c_empty[kMlaStages];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full, pv_done, o_free;
    uint64_t x_full, x_free;
    uint64_t end_bar, mma_final;
    uint32_t tmem_base;
    int abort;
    PlanScratch plan;
};
static_assert(sizeof(MlaBars) <= 512, "barrier block");
static_assert(kMlaSmem <= 227 * 1024, "shared memory per CTA");

struct MlaParams {
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

__global__ void __launch_bounds__(kMlaThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_qr,
                  const __grid_constant__ CUtensorMap tm_c, const MlaParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *sQ = smem + kOffQ;
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

    // ---- plan (both CTAs of the cluster compute the same range)
    PlanArgs pa{p.seq_lens, p.B, 1, 0, p.max_blocks, p.num_clusters};
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
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < kMlaStages; ++s) {
            mbar_init(&bars->c_full[s], 1);
            mbar_init(&bars->c_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_free[s], 128);
        }
        mbar_init(&bars->p_full, 128);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_free, 128);
        mbar_init(&bars->x_full, 128);
        mbar_init(&bars->x_free, 128);
        mbar_init(&bars->end_bar, 1);
        mbar_init(&bars->mma_final, 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();   // the peer's barriers exist before any remote arrive
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ============================================================ TMA
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            tma_prefetch_map(&tm_c);
            tma_prefetch_map(&tm_q);
            TileCursor cur;
            cur.init(pa, lo, hi, first_seq, first_base);
            int seg = 0, tile = 0, q_issued = 0;
            bool ok = true;
            while (ok && !cur.done()) {
                if (cur.t == 0) {
                    if (seg > 0 && !mbar_wait(&bars->q_empty, (uint32_t)((seg - 1) & 1),
                                              p.timeout_ns, p.err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int row = cur.w.b * kMlaH;
                    mbar_arrive_expect_tx(&bars->q_full, nbox * kMlaQBox);
                    for (int i = 0; i < nbox; ++i) {
                        if (rank == 1 && i == 4)
                            tma_load_2d(sQ + i * kMlaQBox, &tm_qr, 0, row, &bars->q_full, pol);
                        else
                            tma_load_2d(sQ + i * kMlaQBox, &tm_q, col0 + i * 64, row,
                                        &bars->q_full, pol);
                    }
                    ++seg;
                    q_issued = seg;
                }
                const int st = tile % kMlaStages;
                if (tile >= kMlaStages &&
                    !mbar_wait(&bars->c_empty[st], (uint32_t)(((tile - kMlaStages) / kMlaStages) & 1),
                               p.timeout_ns, p.err, abort_flag)) {
                    ok = false;
                    break;
                }
                int phys = p.block_table[(size_t)cur.w.b * p.max_blocks + cur.logical_block()];
                if (phys < 0 || phys >= p.num_blocks) {
                    raise_error(p.err, kErrBadBlock);
                    phys = p.num_blocks;            // wholly out of bounds: zero fill
                }
                unsigned char *dst = sC + st * (kMlaMaxBoxes * kMlaCBox);
                mbar_arrive_expect_tx(&bars->c_full[st], nbox * kMlaCBox);
                for (int i = 0; i < nbox; ++i)
                    tma_load_2d(dst + i * kMlaCBox, &tm_c, col0 + i * 64, phys * 64,
                                &bars->c_full[st], pol);
                cur.next();
                ++tile;
            }
            // Every issued load must have landed before the CTA exits.
            for (int t = tile - kMlaStages < 0 ? 0 : tile - kMlaStages; t < tile; ++t)
                mbar_wait(&bars->c_full[t % kMlaStages], (uint32_t)((t / kMlaStages) & 1),
                          p.timeout_ns, p.err, nullptr);
            if (q_issued > 0)
                mbar_wait(&bars->q_full, (uint32_t)((q_issued - 1) & 1), p.timeout_ns, p.err,
                          nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ============================================================ MMA
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 256, 0, 1);
            const uint32_t q_base = smem_u32(sQ), c_base = smem_u32(sC), p_base = smem_u32(sP);
            TileCursor cs, cv;           // S runs one tile ahead of P V
            cs.init(pa, lo, hi, first_seq, first_base);
            cv.init(pa, lo, hi, first_seq, first_base);
            int seg_s = 0, seg_v = 0;
            bool ok = true;

            auto issue_s = [&](int i) -> bool {
                const bool first = cs.t == 0, last = cs.t == cs.len - 1;
                if (first) {
                    if (!mbar_wait(&bars->q_full, (uint32_t)(seg_s & 1), p.timeout_ns, p.err,
                                   abort_flag))
                        return false;
                }
                const int st = i % kMlaStages, sb = i & 1;
                if (!mbar_wait(&bars->c_full[st], (uint32_t)((i / kMlaStages) & 1),
                               p.timeout_ns, p.err, abort_flag))
                    return false;
                if (i >= 2 && !mbar_wait(&bars->s_free[sb], (uint32_t)(((i - 2) / 2) & 1),
                                         p.timeout_ns, p.err, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t cst = c_base + st * (kMlaMaxBoxes * kMlaCBox);
                for (int bx = 0; bx < nbox; ++bx)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t a = umma_desc_sw128(q_base + bx * kMlaQBox + k * 32, 16, 1024);
                        const uint64_t b = umma_desc_sw128(cst + bx * kMlaCBox + k * 32, 16, 1024);
                        umma_bf16(tmem + kTmemS + 64 * sb, a, b, idesc_s, (bx | k) != 0);
                    }
                umma_commit(&bars->s_full[sb]);
                if (last) umma_commit(&bars->q_empty);
                if (first) ++seg_s;
                cs.next();
                return true;
            };
            auto issue_pv = [&](int i) -> bool {
                const bool first = cv.t == 0;
                if (!mbar_wait(&bars->p_full, (uint32_t)(i & 1), p.timeout_ns, p.err, abort_flag))
                    return false;
                if (first && seg_v > 0 &&
                    !mbar_wait(&bars->o_free, (uint32_t)((seg_v - 1) & 1), p.timeout_ns, p.err,
                               abort_flag))
                    return false;
                tc_fence_after();
                const int st = i % kMlaStages;
                const uint32_t cst = c_base + st * (kMlaMaxBoxes * kMlaCBox);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t b = umma_desc_sw128(cst + k * 2048, kMlaCBox, 1024);
                    const uint64_t a_hi = umma_desc_sw128(p_base + k * 32, 16, 1024);
                    const uint64_t a_lo = umma_desc_sw128(p_base + kPBytes + k * 32, 16, 1024);
                    umma_bf16(tmem + kTmemO, a_hi, b, idesc_pv, !(first && k == 0));
                    umma_bf16(tmem + kTmemO, a_lo, b, idesc_pv, 1);
                }
                umma_commit(&bars->c_empty[st]);
                umma_commit(&bars->pv_done);
                if (first) ++seg_v;
                cv.next();
                return true;
            };

            ok = issue_s(0);
            for (int i = 0; ok && i < n_tiles; ++i) {
                if (i + 1 < n_tiles && !issue_s(i + 1)) { ok = false; break; }
                if (!issue_pv(i)) { ok = false; break; }
            }
            // All MMAs issued so far complete before TMEM is released.
            umma_commit(&bars->mma_final);
            mbar_wait(&bars->mma_final, 0, p.timeout_ns, p.err, nullptr);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ===================================================== softmax
        const int row = tid - 128;                       // head = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t x_peer = map_to_rank(sX, peer);
        const uint32_t x_full_peer = map_to_rank(&bars->x_full, peer);
        const uint32_t x_free_peer = map_to_rank(&bars->x_free, peer);
        float *xrow = reinterpret_cast<float *>(sX) + row * 64;
        unsigned char *prow = sP + row * 128;
        // Every wait outcome is made warp-uniform: the TMEM loads and stores
        // below are warp-collective and must never run in a partial warp.
        auto all = [](bool v) { return __all_sync(0xffffffffu, v); };
        TileCursor cur;
        cur.init(pa, lo, hi, first_seq, first_base);
        float m_run = -1e30f, l_run = 0.f;
        float s[64];
        for (int i = 0; i < n_tiles; ++i) {
            const bool first = cur.t == 0, last = cur.t == cur.len - 1;
            const int b = cur.w.b, T = cur.w.T;
            const int tok0 = cur.logical_block() * 64;
            const int sb = i & 1;
            if (!all(mbar_wait(&bars->s_full[sb], (uint32_t)((i >> 1) & 1), p.timeout_ns,
                               p.err, abort_flag)))
                break;
            tc_fence_after();
            tmem_ld64(trow + kTmemS + 64 * sb, s);
            tc_fence_before();
            mbar_arrive(&bars->s_free[sb]);

            // exchange the partial scores with the other CTA of the cluster
            if (i >= 1 && !all(mbar_wait_cluster(&bars->x_free, (uint32_t)((i - 1) & 1),
                                                 p.timeout_ns, p.err, abort_flag)))
                break;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                st_cluster_v4(x_peer + (uint32_t)(row * 256 + ((c ^ (row & 15)) * 16)),
                              s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
            mbar_arrive_remote(x_full_peer);
            if (!all(mbar_wait_cluster(&bars->x_full, (uint32_t)(i & 1), p.timeout_ns, p.err,
                                       abort_flag)))
                break;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 v = *reinterpret_cast<const float4 *>(
                    reinterpret_cast<const unsigned char *>(xrow) + ((c ^ (row & 15)) * 16));
                s[4 * c] += v.x; s[4 * c + 1] += v.y; s[4 * c + 2] += v.z; s[4 * c + 3] += v.w;
            }
            mbar_arrive_remote(x_free_peer);

            // online softmax (log2 domain), lazy rescale
            const int nvalid = T - tok0 < 64 ? T - tok0 : 64;
            float mx = kNegInf;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                s[j] = j < nvalid ? s[j] * p.scale_log2 : kNegInf;
                mx = fmaxf(mx, s[j]);
            }
            bool rescale = false;
            float alpha = 1.f;
            if (first) {
                m_run = mx;
                l_run = 0.f;
            } else if (mx > m_run + kRescaleThreshold) {
                alpha = exp2f(m_run - mx);
                m_run = mx;
                l_run *= alpha;
                rescale = true;
            }
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                s[j] = exp2f(s[j] - m_run);
                sum += s[j];
            }
            l_run += sum;

            // P and O may be touched once the previous P V has completed
            if (i >= 1 && !all(mbar_wait(&bars->pv_done, (uint32_t)((i - 1) & 1),
                                         p.timeout_ns, p.err, abort_flag)))
                break;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float a = s[8 * c + 2 * k], b = s[8 * c + 2 * k + 1];
                    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                    const float2 hf = __bfloat1622float2(h);
                    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
                    hi[k] = *reinterpret_cast<const uint32_t *>(&h);
                    lo[k] = *reinterpret_cast<const uint32_t *>(&l);
                }
                const int off = (c ^ (row & 7)) * 16;
                *reinterpret_cast<uint4 *>(prow + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(prow + kPBytes + off) =
                    make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, rescale)) {   // rows without a new max use alpha = 1
                float o[64];
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    tmem_ld64(trow + kTmemO + 64 * ch, o);
#pragma unroll
                    for (int j = 0; j < 64; ++j) o[j] *= alpha;
                    tmem_st64(trow + kTmemO + 64 * ch, o);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->p_full);

            if (last) {
                if (!all(mbar_wait(&bars->pv_done, (uint32_t)(i & 1), p.timeout_ns, p.err,
                                   abort_flag)))
                    break;
                tc_fence_after();
                const long long slot = (long long)b + cluster;
                float *dst = p.ws_o + ((size_t)slot * kMlaH + row) * kMlaDc + col0;
                const float inv = 1.f / l_run;
                float o[64];
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    tmem_ld64(trow + kTmemO + 64 * ch, o);
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4 *>(dst + 64 * ch + j) =
                            make_float4(o[j] * inv, o[j + 1] * inv, o[j + 2] * inv,
                                        o[j + 3] * inv);
                }
                if (rank == 0) p.ws_lse[slot * kMlaH + row] = m_run + log2f(l_run);
                tc_fence_before();
                mbar_arrive(&bars->o_free);
            }
            cur.next();
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

// Row-major bf16 matrix [rows][cols] with row stride `stride` bytes, boxes of
// [box_rows][64] with 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
              uint64_t stride, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {stride};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Clusters of two that can be resident at once (one CTA per SM), so that the
// persistent ranges all run in a single wave.  Cached per device.
int max_resident_clusters(int num_sms) {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(num_sms);
        cfg.blockDim = dim3(kMlaThreads);
        cfg.dynamicSmemBytes = kMlaSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, mla_decode_kernel, &cfg) != cudaSuccess || n <= 0)
            n = num_sms / 2;
        cache[dev] = n < num_sms / 2 ? n : num_sms / 2;
        if (cache[dev] <= 0) cache[dev] = 1;
    }
    return cache[dev];
}

}  // namespace

int mla_decode_entry(const void *q_latent, const void *q_rope, const void *latent_cache,
                     const int32_t *seq_lens, const int32_t *block_table, void *out, int B,
                     int H, float scale, cudaStream_t stream, int max_blocks, int num_blocks,
                     int num_sms, int forced_ctas, unsigned *err,
                     const WorkspaceFn &workspace) {
    if (H != kMlaH) return ATTN_ERR_UNSUPPORTED;
    if ((long long)num_blocks * 64 > (1ll << 31) - 64 || (long long)B * kMlaH > (1ll << 31))
        return ATTN_ERR_ARG;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMlaSmem) != cudaSuccess)
            return ATTN_ERR_CUDA;
        configured = true;
    }
    int clusters = forced_ctas > 0 ? forced_ctas : max_resident_clusters(num_sms);
    if (clusters <= 0) return ATTN_ERR_CUDA;
    const long long slots = (long long)B + clusters;
    const size_t o_bytes = round256((size_t)slots * kMlaH * kMlaDc * sizeof(float));
    const size_t lse_bytes = round256((size_t)slots * kMlaH * sizeof(float));
    const size_t pre_bytes = round256((size_t)(B + 1) * sizeof(long long));
    void *ws = nullptr;
    int rc = workspace(o_bytes + lse_bytes + pre_bytes, &ws);
    if (rc) return rc;
    unsigned char *w = static_cast<unsigned char *>(ws);

    CUtensorMap tq, tr, tc;
    if (!make_map(&tq, q_latent, kMlaDc, (uint64_t)B * kMlaH, kMlaDc * 2, 128) ||
        !make_map(&tr, q_rope, kMlaDr, (uint64_t)B * kMlaH, kMlaDr * 2, 128) ||
        !make_map(&tc, latent_cache, kMlaWidth, (uint64_t)num_blocks * 64, kMlaWidth * 2, 64))
        return ATTN_ERR_CUDA;

    MlaParams mp{};
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

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(kMlaThreads);
    cfg.dynamicSmemBytes = kMlaSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mla_decode_kernel, tq, tr, tc, mp) != cudaSuccess)
        return ATTN_ERR_CUDA;

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
    cp.window = 0;
    cp.num_ctas = clusters;
    cp.D = kMlaDc;
    cp.HC = kMlaH;
    cp.blocks_per_unit = kMlaH * kMlaDc / 4 / kCombineThreads;
    combine_kernel<__nv_bfloat16><<<B * cp.blocks_per_unit, kCombineThreads, 0, stream>>>(cp);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
