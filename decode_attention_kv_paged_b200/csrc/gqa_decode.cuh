// gqa_decode.cuh -- split-KV decode attention for MHA / GQA / MQA on CUDA
// cores (sm_100a), plus the log-sum-exp combine of the split partials.
//
// Computes, per sequence b and query head h (attention-head article, §1
// Attention equation; §2 group rule: head h reads KV head floor(h/G)):
//     out[b,h] = sum_{j in [lo_b, T_b)} softmax_j(scale <q[b,h], K[b,g,j]>) V[b,g,j]
//
// Design (B200):
//   * One CTA per SM (persistent range of the flattened block list, see
//     plan.cuh) of 16 warps (4 per SM sub-partition, <= 128 registers each)
//     or, for register-heavy shapes, 8 warps.  Thread 0 also streams each
//     64-token K tile and V
//     tile (64*d contiguous elements each in the paged layout) with 1-D bulk
//     async copies (TMA engine) into a multi-stage shared-memory ring,
//     completion tracked by mbarriers, L2 policy evict-first; it refills a
//     stage one tile after the CTA has released it.
//   * Every warp computes.  Each warp owns 64/NW tokens of a tile and the
//     HC query heads of its unit, so a K/V tile is read from HBM once for the
//     whole GQA group.  Lanes split the head dimension: each lane keeps its
//     slice of the HC queries and of the HC output accumulators in fp32
//     registers; partial dot products are combined with a warp-shuffle
//     reduce-scatter, the warp's running max / sum (online softmax, as in the
//     FlashAttention tiling the toolsku article describes) with shuffles.
//   * Warps keep independent (m, l, O) states and are merged once per
//     segment through shared memory; each (unit, CTA) segment writes an fp32
//     partial (O / l, log2-sum-exp) that the combine kernel reduces in a fixed
//     order (deterministic, no atomics on data).
//   * Every wait is bounded (%globaltimer); a block id outside the pool is
//     skipped and flagged, never dereferenced.
#pragma once

#include "plan.cuh"

namespace attn {

constexpr int kSmemBudget = 227 * 1024 - 1024;
#define kNegInf (__int_as_float(0xff800000u))

constexpr int pow2_floor(int x) {
    int p = 1;
    while (p * 2 <= x) p *= 2;
    return p;
}

// Warps per CTA.  Sixteen (four per SM sub-partition, so one warp's
// dependency chain -- shuffle reductions, exp2, shared-memory round trips --
// overlaps three others) whenever the per-thread state fits the 128
// registers that allows; otherwise eight (up to 255 registers each).
constexpr int gqa_warps(int D, int HC) {
    return (D >= 64 && HC <= 4 && false) ? 16 : 8;
}

// Elements of the head dimension each lane owns: the queries plus the
// accumulators take 2*HC*EPL fp32 registers (at most 64 with 16 warps, 128
// with 8), a warp covers no more rows per instruction than the 64/NW tokens
// it owns, and no fewer than one row per instruction.
constexpr int gqa_epl(int D, int HC, int NW) {
    int e = pow2_floor((NW == 16 ? 32 : 64) / HC);
    const int tpw = 64 / NW;
    if (e > D * tpw / 32) e = D * tpw / 32;
    if (e < D / 32) e = D / 32;
    return e;
}

struct GqaParams {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *seq_lens;
    const int32_t *block_table;
    float *ws_o;          // [slots][HC][D]
    float *ws_lse;        // [slots][HC]  log2-sum-exp of the scaled scores
    long long *ws_prefix; // [B + 1]
    unsigned *err;
    unsigned long long timeout_ns;
    float scale_log2;     // scale * log2(e)
    int B, H_q, H_kv, group, n_hc, max_blocks, num_blocks, window, num_ctas;
    int force_timeout;
};

template <int D, int HC, typename T>
struct GqaCfg {
    static constexpr int kS = (int)sizeof(T);
    static constexpr int kNW = gqa_warps(D, HC);
    static constexpr int kThreads = kNW * 32;
    static constexpr int kTPW = kBlockSize / kNW;                 // tokens/warp
    static constexpr int kEPL = gqa_epl(D, HC, kNW);
    static constexpr int kLE = (16 / kS < kEPL) ? 16 / kS : kEPL; // per load
    static constexpr int kCPL = kEPL / kLE;                       // loads/lane/row
    static constexpr int kLPR = D / kEPL;                         // lanes per row
    static constexpr int kRPW = 32 / kLPR;                        // rows per instr.
    static constexpr int kIters = kTPW / kRPW;
    static constexpr int kCPR = D / kLE;                          // chunks per row
    static constexpr int kHPP = 32 / kTPW;                        // heads/pass
    static constexpr int kPasses = (HC + kHPP - 1) / kHPP;        // softmax passes
    static constexpr int kHCP = (HC == 3) ? 4 : (HC > 4 ? 8 : HC);// padded heads
    static constexpr int kTileBytes = kBlockSize * D * kS;
    static constexpr int kStageBytes = 2 * kTileBytes;
    // shared memory carve-up (bytes)
    static constexpr int kScoreBytes = kNW * kTPW * kHCP * 4;
    static constexpr int kMergeOBytes = kNW * HC * D * 4;
    static constexpr int kMergeMLBytes = 2 * kNW * HC * 4;
    static constexpr int kMiscBytes = 1024;  // barriers + plan scratch + flags
    static constexpr int kOther =
        kScoreBytes + kMergeOBytes + kMergeMLBytes + kMiscBytes;
    static constexpr int kStagesRaw = (kSmemBudget - kOther) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 6 ? 6 : kStagesRaw;
    static_assert(kTPW * kHPP == 32, "softmax lane map");
    static constexpr int kSmemBytes = kStages * kStageBytes + kOther;
    static_assert(kStages >= 2, "not enough shared memory for two stages");
    static_assert(kLPR >= 4 && kLPR <= 32 && (kLPR & (kLPR - 1)) == 0, "LPR");
    static_assert(kIters >= 1 && kIters * kRPW == kTPW, "rows per warp");
    static_assert(kTileBytes % 16 == 0, "bulk copy size");
};

// Load kLE consecutive elements (16 or 8 bytes) and widen to fp32.
template <typename T, int LE>
__device__ __forceinline__ void load_widen(const T *p, float *f) {
    if constexpr (sizeof(T) * LE == 16) {
        uint4 v = *reinterpret_cast<const uint4 *>(p);
        Chunk<T>::unpack(v, f);
    } else {
        static_assert(sizeof(T) * LE == 8, "load width");
        uint2 v = *reinterpret_cast<const uint2 *>(p);
        if constexpr (sizeof(T) == 2) {
            f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
            f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
        } else {
            f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        }
    }
}

// Load kLE consecutive elements and widen them to fp32 pairs (element 2j in
// .x, 2j+1 in .y), ready for packed fp32x2 arithmetic.
template <typename T, int LE>
__device__ __forceinline__ void load_pairs(const T *p, float2 *f) {
    if constexpr (sizeof(T) == 2) {
        if constexpr (LE == 8) {
            const uint4 v = *reinterpret_cast<const uint4 *>(p);
            f[0] = make_float2(bf16lo(v.x), bf16hi(v.x));
            f[1] = make_float2(bf16lo(v.y), bf16hi(v.y));
            f[2] = make_float2(bf16lo(v.z), bf16hi(v.z));
            f[3] = make_float2(bf16lo(v.w), bf16hi(v.w));
        } else {
            static_assert(LE == 4, "load width");
            const uint2 v = *reinterpret_cast<const uint2 *>(p);
            f[0] = make_float2(bf16lo(v.x), bf16hi(v.x));
            f[1] = make_float2(bf16lo(v.y), bf16hi(v.y));
        }
    } else {
        static_assert(LE == 4, "load width");
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = make_float2(v.x, v.y);
        f[1] = make_float2(v.z, v.w);
    }
}

// Read n consecutive fp32 from shared memory with the widest aligned loads
// (rows of the score buffer are n floats, n in {1, 2, 4, 8}).
template <int n>
__device__ __forceinline__ void load_row(const float *p, float *v) {
    if constexpr (n % 4 == 0) {
#pragma unroll
        for (int i = 0; i < n; i += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(p + i);
            v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
        }
    } else if constexpr (n == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x; v[1] = x.y;
    } else {
#pragma unroll
        for (int i = 0; i < n; ++i) v[i] = p[i];
    }
}

// Reduce-scatter of V per-lane values across the L lanes of a row group
// (lanes differing in the low log2(L) bits).  On return vals[0..count) hold
// full sums of the original indices [base, base + count).
template <int V, int L>
struct RowReduce {
    static constexpr __host__ __device__ int final_count() {
        int n = V;
        for (int m = L / 2; m >= 1; m /= 2)
            if (n >= 2 && n % 2 == 0) n /= 2;
        return n;
    }
    static __device__ __forceinline__ int run(float (&vals)[V], int lane) {
        int base = 0;
        int n = V;
#pragma unroll
        for (int m = L / 2; m >= 1; m /= 2) {
            if (n >= 2 && n % 2 == 0) {
                const bool upper = (lane & m) != 0;
                const int h = n / 2;
#pragma unroll
                for (int i = 0; i < V / 2; ++i) {
                    if (i < h) {
                        const float send = upper ? vals[i] : vals[i + h];
                        const float keep = upper ? vals[i + h] : vals[i];
                        vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                    }
                }
                if (upper) base += h;
                n = h;
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (i < n) vals[i] += __shfl_xor_sync(0xffffffffu, vals[i], m);
            }
        }
        return base;
    }
};

// Steps through the tiles (blocks) of a CTA's range in order.
struct TileCursor {
    SegmentWalker w;
    int t, len;
    __device__ void init(const PlanArgs &a, long long lo, long long hi, int seq,
                         long long base) {
        w.init(a, lo, hi, seq, base);
        t = 0;
        len = w.done() ? 0 : w.seg_len();
    }
    __device__ bool done() const { return w.done(); }
    __device__ int logical_block() const { return w.first_blk + w.blk_off + t; }
    __device__ void next() {
        if (++t == len) {
            w.advance(len);
            t = 0;
            len = w.done() ? 0 : w.seg_len();
        }
    }
};

// Producer of warp 0: walks the CTA's tiles and keeps the physical block ids
// of the current segment in registers, 32 at a time (lane i holds tile
// bt0 + i), fetched with one coalesced load and the next batch prefetched
// half a batch early, so no bulk copy waits on a dependent global load.
// All 32 lanes call it together; lane 0 issues the copies.
struct Producer {
    TileCursor cur;
    int id_cur, id_nxt, bt0;
    bool has_next;

    __device__ int fetch(const GqaParams &p, int i, int lane) const {
        const int j = i + lane;
        if (j >= cur.len) return -1;
        return __ldg(p.block_table + (size_t)cur.w.b * p.max_blocks + cur.w.first_blk +
                     cur.w.blk_off + j);
    }

    // Physical block id of the current tile (warp-uniform call).
    __device__ int block_id(const GqaParams &p, int lane) {
        const int t = cur.t;
        if (t == 0) {
            bt0 = 0;
            id_cur = fetch(p, 0, lane);
            has_next = false;
        } else if (t == bt0 + 32) {
            bt0 += 32;
            id_cur = has_next ? id_nxt : fetch(p, bt0, lane);
            has_next = false;
        }
        if (!has_next && t == bt0 + 16 && bt0 + 32 < cur.len) {
            id_nxt = fetch(p, bt0 + 32, lane);
            has_next = true;
        }
        return __shfl_sync(0xffffffffu, id_cur, t - bt0);
    }
};

// Issue the bulk copies of one tile (physical block `phys`, KV head of the
// cursor's unit) into a stage.  Called by one lane.
template <int D, typename T, int kTileBytes>
__device__ __forceinline__ void issue_tile(const GqaParams &p, const TileCursor &cur,
                                          int phys, unsigned char *dst, uint64_t *full,
                                          uint64_t pol) {
    const int kvh = cur.w.unit / p.n_hc;
    if (phys < 0 || phys >= p.num_blocks) {
        raise_error(p.err, kErrBadBlock);
        mbar_arrive(full);
        return;
    }
    const size_t off = ((size_t)phys * p.H_kv + kvh) * kBlockSize * D;
    mbar_arrive_expect_tx(full, 2 * kTileBytes);
    bulk_load(dst, static_cast<const T *>(p.k_cache) + off, kTileBytes, full, pol);
    bulk_load(dst + kTileBytes, static_cast<const T *>(p.v_cache) + off, kTileBytes,
              full, pol);
}

template <int D, int HC, typename T>
__global__ void __launch_bounds__(GqaCfg<D, HC, T>::kThreads, 1)
gqa_split_kernel(const GqaParams p) {
    using C = GqaCfg<D, HC, T>;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *stage_base = smem;
    float *s_scores = reinterpret_cast<float *>(smem + C::kStages * C::kStageBytes);
    float *s_mo = s_scores + C::kScoreBytes / 4;
    float *s_mm = s_mo + C::kMergeOBytes / 4;
    float *s_ml = s_mm + C::kNW * HC;
    unsigned char *misc = reinterpret_cast<unsigned char *>(s_ml + C::kNW * HC);
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(misc);
    uint64_t *empty_bar = full_bar + C::kStages;
    uint64_t *merge_bar = empty_bar + C::kStages;       // [2]
    uint64_t *never_bar = merge_bar + 2;                // fault injection
    PlanScratch *plan_sh = reinterpret_cast<PlanScratch *>(never_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(plan_sh + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], C::kNW);
        }
        mbar_init(&merge_bar[0], C::kNW * 32);
        mbar_init(&merge_bar[1], C::kNW * 32);
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int units = p.H_kv * p.n_hc;
    PlanArgs pa{p.seq_lens, p.B, units, p.window, p.max_blocks, p.num_ctas};
    plan_locate(pa, blockIdx.x, plan_sh, blockIdx.x == 0 ? p.ws_prefix : nullptr,
                p.err);
    const long long W = plan_sh->total;
    const int P = working_ctas(W, p.num_ctas);
    if ((int)blockIdx.x >= P) return;
    const long long lo = cta_bound(blockIdx.x, W, P);
    const long long hi = cta_bound(blockIdx.x + 1, W, P);
    SegmentWalker walk;
    walk.init(pa, lo, hi, plan_sh->seq, plan_sh->base);

    // ------------------------------------------------------------ producer
    // Warp 0 streams the tiles (lane 0 issues); the prologue fills every stage.
    const bool producer = (warp == 0);
    Producer prod;
    long long issued = 0;
    const long long n_tiles = hi - lo;
    uint64_t pol = 0;
    if (producer) {
        pol = l2_policy_evict_first();
        prod.cur.init(pa, lo, hi, plan_sh->seq, plan_sh->base);
        while (issued < C::kStages && issued < n_tiles) {
            const int phys = prod.block_id(p, lane);
            if (lane == 0)
                issue_tile<D, T, C::kTileBytes>(p, prod.cur, phys,
                                                stage_base + issued * C::kStageBytes,
                                                &full_bar[issued], pol);
            prod.cur.next();
            ++issued;
        }
    }

    // ------------------------------------------------------------ consumers
    if (p.force_timeout) {
        // Fault injection: wait on a barrier nobody signals; bounded.
        mbar_wait(never_bar, 0, p.timeout_ns, p.err, abort_flag);
        *abort_flag = 1;
    }

    const int lr = lane % C::kLPR;          // lane within its row group
    const int rg = lane / C::kLPR;          // row group
    const int rot = (C::kLPR < 8) ? (rg % (8 / C::kLPR)) * C::kLPR : 0;
    int col[C::kCPL];
#pragma unroll
    for (int c = 0; c < C::kCPL; ++c)
        col[c] = ((lr + rot + c * C::kLPR) % C::kCPR) * C::kLE;

    const T *qg = static_cast<const T *>(p.q);
    float *sc = s_scores + warp * C::kTPW * C::kHCP;   // [TPW][HCP]
    long long n_tile = 0;
    int n_seg = 0;
    int c_stage = 0, p_stage = 0;          // stage of tile n_tile / n_tile - 1
    uint32_t c_phase = 0, p_phase = 0;     // their use parity

    while (!*abort_flag && !walk.done()) {
        const int len = walk.seg_len();
        const int b = walk.b, unit = walk.unit;
        const int kvh = unit / p.n_hc, hc = unit % p.n_hc;
        const int head0 = kvh * p.group + hc * HC;
        const int Tb = walk.T;
        const int lo_tok = (p.window > 0 && Tb > p.window) ? Tb - p.window : 0;

        constexpr int LP = C::kLE / 2;          // pairs per load
        constexpr int EP = C::kEPL / 2;         // pairs per lane
        float2 q2[HC][EP];
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
        for (int g = 0; g < HC; ++g) {
            const T *qrow = qg + ((size_t)b * p.H_q + head0 + g) * D;
#pragma unroll
            for (int c = 0; c < C::kCPL; ++c) {
                float2 f[LP];
                load_pairs<T, C::kLE>(qrow + col[c], f);
#pragma unroll
                for (int j = 0; j < LP; ++j) q2[g][c * LP + j] = __fmul2_rn(f[j], sc2);
            }
        }
        float2 o2[HC][EP];
#pragma unroll
        for (int g = 0; g < HC; ++g)
#pragma unroll
            for (int j = 0; j < EP; ++j) o2[g][j] = make_float2(0.f, 0.f);
        float m_run[C::kPasses], l_run[C::kPasses];
#pragma unroll
        for (int ps = 0; ps < C::kPasses; ++ps) { m_run[ps] = -1e30f; l_run[ps] = 0.f; }

        bool ok = true;
        for (int t = 0; t < len; ++t) {
            const int stage = c_stage;
            if (!mbar_wait(&full_bar[stage], c_phase, p.timeout_ns, p.err, abort_flag)) {
                ok = false;
                break;
            }
            const T *Ks = reinterpret_cast<const T *>(stage_base + stage * C::kStageBytes);
            const T *Vs = Ks + kBlockSize * D;
            const int tok0 = (walk.first_blk + walk.blk_off + t) * kBlockSize +
                             warp * C::kTPW;

            // ---- scores: partial dot products, then reduce over the row group
            float2 acc[C::kIters * HC];
#pragma unroll
            for (int it = 0; it < C::kIters; ++it) {
                const T *krow = Ks + (warp * C::kTPW + it * C::kRPW + rg) * D;
#pragma unroll
                for (int g = 0; g < HC; ++g) acc[it * HC + g] = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < C::kCPL; ++c) {
                    float2 kp[LP];
                    load_pairs<T, C::kLE>(krow + col[c], kp);
#pragma unroll
                    for (int g = 0; g < HC; ++g)
#pragma unroll
                        for (int j = 0; j < LP; ++j)
                            acc[it * HC + g] =
                                __ffma2_rn(q2[g][c * LP + j], kp[j], acc[it * HC + g]);
                }
            }
            float part[C::kIters * HC];
#pragma unroll
            for (int i = 0; i < C::kIters * HC; ++i) part[i] = acc[i].x + acc[i].y;
            using RR = RowReduce<C::kIters * HC, C::kLPR>;
            const int base = RR::run(part, lane);
#pragma unroll
            for (int i = 0; i < RR::final_count(); ++i) {
                const int v = base + i;
                const int it = v / HC, g = v % HC;
                sc[(it * C::kRPW + rg) * C::kHCP + g] = part[i];
            }
            __syncwarp();

            // ---- online softmax over this warp's 8 tokens (log2 domain)
            float alpha_reg[C::kPasses];
#pragma unroll
            for (int ps = 0; ps < C::kPasses; ++ps) {
                const int gs = lane / C::kTPW + C::kHPP * ps;
                const int tt = lane % C::kTPW;
                const bool active = gs < HC;
                const int pos = tok0 + tt;
                const bool valid = active && pos >= lo_tok && pos < Tb;
                float s = valid ? sc[tt * C::kHCP + gs] : kNegInf;
                float mx = s;
#pragma unroll
                for (int m = 1; m < C::kTPW; m <<= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
                const float m_new = fmaxf(m_run[ps], mx);
                const float pr = exp2f(s - m_new);
                float sum = pr;
#pragma unroll
                for (int m = 1; m < C::kTPW; m <<= 1)
                    sum += __shfl_xor_sync(0xffffffffu, sum, m);
                const float alpha = exp2f(m_run[ps] - m_new);
                l_run[ps] = l_run[ps] * alpha + sum;
                m_run[ps] = m_new;
                alpha_reg[ps] = alpha;
                if (active) sc[tt * C::kHCP + gs] = pr;
            }
            __syncwarp();
#pragma unroll
            for (int g = 0; g < HC; ++g) {
                const float a = __shfl_sync(0xffffffffu, alpha_reg[g / C::kHPP],
                                            (g % C::kHPP) * C::kTPW);
                if (a != 1.f) {
                    const float2 a2 = make_float2(a, a);
#pragma unroll
                    for (int j = 0; j < EP; ++j) o2[g][j] = __fmul2_rn(o2[g][j], a2);
                }
            }

            // ---- P V
#pragma unroll
            for (int it = 0; it < C::kIters; ++it) {
                const int rl = it * C::kRPW + rg;
                const T *vrow = Vs + (warp * C::kTPW + rl) * D;
                float pg[C::kHCP];
                load_row<C::kHCP>(sc + rl * C::kHCP, pg);
                float2 pp[HC];
#pragma unroll
                for (int g = 0; g < HC; ++g) pp[g] = make_float2(pg[g], pg[g]);
#pragma unroll
                for (int c = 0; c < C::kCPL; ++c) {
                    float2 vp[LP];
                    load_pairs<T, C::kLE>(vrow + col[c], vp);
#pragma unroll
                    for (int g = 0; g < HC; ++g)
#pragma unroll
                        for (int j = 0; j < LP; ++j)
                            o2[g][c * LP + j] = __ffma2_rn(pp[g], vp[j], o2[g][c * LP + j]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[stage]);
            // Refill the stage released one tile ago (one-tile lag keeps the
            // producer from waiting on the slowest warp's current tile).
            if (producer && n_tile >= 1 && issued < n_tiles) {
                const int ps = p_stage;
                const bool freed =
                    mbar_wait(&empty_bar[ps], p_phase, p.timeout_ns, p.err, abort_flag);
                if (__all_sync(0xffffffffu, freed)) {
                    const int phys = prod.block_id(p, lane);
                    if (lane == 0)
                        issue_tile<D, T, C::kTileBytes>(p, prod.cur, phys,
                                                        stage_base + ps * C::kStageBytes,
                                                        &full_bar[ps], pol);
                    prod.cur.next();
                    ++issued;
                } else {
                    ok = false;
                }
            }
            p_stage = c_stage;
            p_phase = c_phase;
            if (++c_stage == C::kStages) {
                c_stage = 0;
                c_phase ^= 1u;
            }
            ++n_tile;
            if (!ok) break;
        }
        if (!ok) break;

        // ---- merge the warps' states, write the segment's partial
        // Row groups with a rotated chunk order hold chunk (c + shift) mod CPL
        // in register slot c; put them back in the unrotated order first so
        // the cross-row-group sums below add like columns.
        if constexpr (C::kLPR < 8 && C::kCPL > 1) {
            const int shift = rot / C::kLPR;
#pragma unroll
            for (int sh = 1; sh < 8 / C::kLPR; ++sh) {
                if (shift == sh) {
#pragma unroll
                    for (int g = 0; g < HC; ++g) {
                        float2 tmp[EP];
#pragma unroll
                        for (int c = 0; c < C::kCPL; ++c)
#pragma unroll
                            for (int j = 0; j < LP; ++j)
                                tmp[((c + sh) % C::kCPL) * LP + j] = o2[g][c * LP + j];
#pragma unroll
                        for (int j = 0; j < EP; ++j) o2[g][j] = tmp[j];
                    }
                }
            }
        }
#pragma unroll
        for (int m = C::kLPR; m < 32; m <<= 1)
#pragma unroll
            for (int g = 0; g < HC; ++g)
#pragma unroll
                for (int j = 0; j < EP; ++j) {
                    o2[g][j].x += __shfl_xor_sync(0xffffffffu, o2[g][j].x, m);
                    o2[g][j].y += __shfl_xor_sync(0xffffffffu, o2[g][j].y, m);
                }
        if (rg == 0) {
#pragma unroll
            for (int g = 0; g < HC; ++g)
#pragma unroll
                for (int c = 0; c < C::kCPL; ++c)
#pragma unroll
                    for (int j = 0; j < LP; ++j)
                        *reinterpret_cast<float2 *>(&s_mo[(warp * HC + g) * D + col[c] + 2 * j]) =
                            o2[g][c * LP + j];
        }
        if ((lane % C::kTPW) == 0) {
#pragma unroll
            for (int ps = 0; ps < C::kPasses; ++ps) {
                const int gs = lane / C::kTPW + C::kHPP * ps;
                if (gs < HC) {
                    s_mm[warp * HC + gs] = m_run[ps];
                    s_ml[warp * HC + gs] = l_run[ps];
                }
            }
        }
        mbar_arrive(&merge_bar[0]);
        if (!mbar_wait(&merge_bar[0], (uint32_t)(n_seg & 1), p.timeout_ns, p.err,
                       abort_flag))
            break;
        const long long slot = (long long)b * units + unit + blockIdx.x;
        for (int idx = tid; idx < HC * D; idx += C::kNW * 32) {
            const int g = idx / D, k = idx % D;
            float M = -1e30f;
#pragma unroll
            for (int w = 0; w < C::kNW; ++w) M = fmaxf(M, s_mm[w * HC + g]);
            float num = 0.f, den = 0.f;
#pragma unroll
            for (int w = 0; w < C::kNW; ++w) {
                const float wt = exp2f(s_mm[w * HC + g] - M);
                num = fmaf(wt, s_mo[(w * HC + g) * D + k], num);
                den = fmaf(wt, s_ml[w * HC + g], den);
            }
            p.ws_o[(slot * HC + g) * D + k] = num / den;
            if (k == 0) p.ws_lse[slot * HC + g] = M + log2f(den);
        }
        mbar_arrive(&merge_bar[1]);
        if (!mbar_wait(&merge_bar[1], (uint32_t)(n_seg & 1), p.timeout_ns, p.err,
                       abort_flag))
            break;
        ++n_seg;
        walk.advance(len);
    }

    // Abort path: copies still in flight must land before the CTA exits.
    if (producer && lane == 0) {
        for (long long n = n_tile; n < issued; ++n)
            mbar_wait(&full_bar[n % C::kStages], (uint32_t)((n / C::kStages) & 1),
                      p.timeout_ns, p.err, nullptr);
    }
}

struct CombineParams {
    const int32_t *seq_lens;
    const long long *ws_prefix;
    const float *ws_o;
    const float *ws_lse;
    void *out;
    int B, H_q, H_kv, group, n_hc, max_blocks, window, num_ctas;
    int D, HC;               // head dim, query heads per unit
    int blocks_per_unit;     // CTAs of kCombineThreads per unit
};

constexpr int kCombineThreads = 256;

// out = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L) over the unit's split
// partials, in CTA order (fixed, deterministic).  Each thread produces four
// consecutive outputs of one head; a unit's HC*D outputs are spread over
// blocks_per_unit CTAs.
template <typename T>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const CombineParams p) {
    __shared__ long long s_first_slot;
    __shared__ int s_nsplit, s_nb;
    pdl_wait_primary();
    const int units = p.H_kv * p.n_hc;
    const int u = blockIdx.x / p.blocks_per_unit;
    const int part = blockIdx.x % p.blocks_per_unit;
    const int b = u / units, rem = u % units;
    if (threadIdx.x == 0) {
        int fb;
        bool bad;
        const int nb = visible_blocks(p.seq_lens[b], p.window, p.max_blocks, &fb, &bad);
        s_nb = nb;
        s_nsplit = 0;
        s_first_slot = 0;
        if (nb > 0) {
            const long long W = p.ws_prefix[p.B];
            const int P = working_ctas(W, p.num_ctas);
            const long long s_u = p.ws_prefix[b] + (long long)rem * nb;
            const int c0 = cta_of(s_u, W, P);
            const int c1 = cta_of(s_u + nb - 1, W, P);
            s_nsplit = c1 - c0 + 1;
            s_first_slot = (long long)u + c0;
        }
    }
    __syncthreads();
    const int e = (part * kCombineThreads + threadIdx.x) * 4;   // output index in unit
    if (e >= p.HC * p.D) return;
    const int g = e / p.D, k = e % p.D;
    const int kvh = rem / p.n_hc, hc = rem % p.n_hc;
    T *out = static_cast<T *>(p.out) +
             ((size_t)b * p.H_q + kvh * p.group + hc * p.HC + g) * p.D + k;
    float r[4];
    const int ns = s_nsplit;
    if (s_nb == 0) {
        r[0] = r[1] = r[2] = r[3] = 0.f;
    } else {
        const long long s0 = s_first_slot;
        if (ns == 1) {
            const float4 v = *reinterpret_cast<const float4 *>(
                p.ws_o + ((size_t)s0 * p.HC + g) * p.D + k);
            r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
        } else {
            float L = kNegInf;
            for (int i = 0; i < ns; ++i) L = fmaxf(L, p.ws_lse[(s0 + i) * p.HC + g]);
            float den = 0.f;
            r[0] = r[1] = r[2] = r[3] = 0.f;
            for (int i = 0; i < ns; ++i) {
                const float w = exp2f(p.ws_lse[(s0 + i) * p.HC + g] - L);
                const float4 v = *reinterpret_cast<const float4 *>(
                    p.ws_o + ((size_t)(s0 + i) * p.HC + g) * p.D + k);
                r[0] = fmaf(w, v.x, r[0]);
                r[1] = fmaf(w, v.y, r[1]);
                r[2] = fmaf(w, v.z, r[2]);
                r[3] = fmaf(w, v.w, r[3]);
                den += w;
            }
            const float inv = 1.f / den;
            r[0] *= inv; r[1] *= inv; r[2] *= inv; r[3] *= inv;
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) out[j] = ElemTraits<T>::from_float(r[j]);
}

}  // namespace attn
