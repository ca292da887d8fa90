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
// Headroom of the lazy softmax rescale, log2 units: probabilities <= 2^8.
constexpr float kRescaleLog2 = 8.0f;
#define kNegInf (__int_as_float(0xff800000u))

constexpr int pow2_floor(int x) {
    int p = 1;
    while (p * 2 <= x) p *= 2;
    return p;
}

// Elements of the head dimension each lane owns.  The queries plus the
// accumulators take 2*HC*EPL fp32 registers (at most 128), a warp covers no
// more rows per instruction than the `tpw` tokens it owns, a row is split
// over 4 to 32 lanes.
constexpr int gqa_epl(int D, int HC, int tpw) {
    int e = pow2_floor(64 / HC);
    if (e > D * tpw / 32) e = D * tpw / 32;
    if (e > D / 4) e = D / 4;
    if (e < D / 32) e = D / 32;
    return e;
}

// Row-iterations whose partial dot products are reduced together: the
// largest divisor of `iters` with at most 16 (iteration, head) sums.
constexpr int gqa_chunk(int iters, int HC) {
    int c = 16 / HC;
    if (c < 1) c = 1;
    if (c > iters) c = iters;
    while (iters % c != 0) --c;
    return c;
}

struct GqaParams {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *seq_lens;
    const int32_t *block_table;
    void *out;            // [B][H_q][D]
    float *ws_o;          // [slots][HC][D]
    float *ws_lse;        // [slots][HC]  log2-sum-exp of the scaled scores
    long long *ws_prefix; // [B + 1]
    unsigned *ws_cnt;     // [B * units] split arrival counters, zero between launches
    const float *k_scale; // fp8 cache only: [num_blocks][H_kv][64] row scales
    const float *v_scale;
    unsigned *err;
    unsigned long long timeout_ns;
    float scale_log2;     // scale * log2(e)
    int B, H_q, H_kv, group, n_hc, max_blocks, num_blocks, num_ctas;
    Visibility vis;       // window, sink (global) tokens, ring table
    int force_timeout;
};

// T: query / output element type; TK: cache element type (T, or uint8_t
// for fp8 e4m3 codes with one fp32 scale per cached row).
template <int D, int HC, typename T, typename TK = T>
struct GqaCfg {
    static constexpr int kS = (int)sizeof(TK);                   // cache bytes / element
    static constexpr bool kFp8 = sizeof(TK) == 1;
    // Warp specialisation: warpgroup 0 is the producer (its warp 0 streams
    // the tiles, warps 1-3 run the segment epilogues), warpgroups 1 and 2
    // are the kNW compute warps.  setmaxnreg moves registers from the
    // producer group to the compute groups; the shares add up to the
    // launch's 384 x 168.  200 per compute thread is what their loop needs;
    // the rest keeps the epilogue's merge and combine out of local memory.
    static constexpr int kNW = 8;                                 // compute warps
    static constexpr int kThreads = 32 * (4 + kNW);
    static constexpr int kProducerRegs = 104;
    static constexpr int kConsumerRegs = 200;
    static constexpr int kLaunchRegs = 168;
    static_assert(4 * 32 * kProducerRegs + kNW * 32 * kConsumerRegs <=
                      kThreads * kLaunchRegs, "register split exceeds the launch");
    // A staged tile is a whole 64-token block, or half of one when a block's
    // K and V would take more than 32 KiB (d = 256 bf16, fp32 d = 128).
    static constexpr int kTileTok =
        (kBlockSize * D * kS * 2 > 32768) ? 32768 / (2 * D * kS) : kBlockSize;
    static constexpr int kSub = kBlockSize / kTileTok;            // tiles/block
    // The warps form kNG groups; group g consumes the CTA's tiles n with
    // n % kNG == g, so kNG tiles are in work at once and each warp owns
    // kTPW rows of its group's tiles.
    static constexpr int kNG = 2;
    static constexpr int kWPG = kNW / kNG;                        // warps/group
    static constexpr int kTPW = kTileTok / kWPG;                  // tokens/warp
    static constexpr int kEPL = gqa_epl(D, HC, kTPW);
    static constexpr int kLE = (16 / kS < kEPL) ? 16 / kS : kEPL; // per load
    static constexpr int kCPL = kEPL / kLE;                       // loads/lane/row
    static constexpr int kLPR = D / kEPL;                         // lanes per row
    static constexpr int kRPW = 32 / kLPR;                        // rows per instr.
    static constexpr int kIters = kTPW / kRPW;
    // Score rows are reduced kChunk row-iterations at a time (bounds the
    // live partial sums to 16 fp32x2 registers).
    static constexpr int kChunk = gqa_chunk(kIters, HC);
    static constexpr int kChunks = (kIters + kChunk - 1) / kChunk;
    static constexpr int kCPR = D / kLE;                          // chunks per row
    static constexpr int kHPP = 32 / kTPW;                        // heads/pass
    static constexpr int kPasses = (HC + kHPP - 1) / kHPP;        // softmax passes
    static constexpr int kHCP = (HC == 3) ? 4 : (HC > 4 ? 8 : HC);// padded heads
    static constexpr int kTileBytes = kTileTok * D * kS;
    static constexpr int kScaleBytes = kFp8 ? kTileTok * 4 : 0;   // one fp32 per row
    static constexpr int kStageBytes = 2 * (kTileBytes + kScaleBytes);
    // shared memory carve-up (bytes)
    static constexpr int kScoreBytes = kNW * kTPW * kHCP * 4;
    static constexpr int kMergeOBytes = kNW * HC * D * 4;
    static constexpr int kMergeMLBytes = 2 * kNW * HC * 4;
    static constexpr int kEpiBytes = ((kNW + 2) * HC * 4 + 15) / 16 * 16;  // merge weights
    static constexpr int kEpiThreads = 96;                        // producer WG warps 1-3
    static constexpr int kQBytes = HC * D * (int)sizeof(T);      // one unit's queries
    static constexpr int kQRingBytes = 2 * ((kQBytes + 127) / 128 * 128);
    static constexpr int kMiscBytes = 1024;  // barriers + plan scratch + flags
    static constexpr int kOther =
        kQRingBytes + kScoreBytes + kMergeOBytes + kMergeMLBytes + kEpiBytes + kMiscBytes;
    static constexpr int kStagesRaw = (kSmemBudget - kOther) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static_assert(kTPW * kHPP == 32, "softmax lane map");
    // What the ring leaves over holds up to kPreMax other splits' partials
    // (fp32 O and lse of one unit), prefetched by the epilogue warps.
    static constexpr int kPreUnit = HC * D * 4 + HC * 4;
    static constexpr int kPreRaw = (kSmemBudget - kStages * kStageBytes - kOther) / kPreUnit;
    static constexpr int kPreMax = kPreRaw > 8 ? 8 : kPreRaw;
    static constexpr int kSmemBytes = kStages * kStageBytes + kOther + kPreMax * kPreUnit;
    static_assert(kStages >= kNG + 2, "not enough shared memory for the ring");
    static_assert(kLPR >= 4 && kLPR <= 32 && (kLPR & (kLPR - 1)) == 0, "LPR");
    static_assert(kIters >= 1 && kIters * kRPW == kTPW, "rows per warp");
    static_assert(kChunks * kChunk == kIters, "score chunks");
    static_assert(kTileBytes % 16 == 0, "bulk copy size");
};

// Load kLE consecutive elements and widen them to fp32 pairs (element 2j in
// .x, 2j+1 in .y), ready for packed fp32x2 arithmetic.
// fp8 e4m3 byte I of w as an fp32 equal to its value times 2^-120, exactly
// (subnormals included): the sign and the 7 exponent/mantissa bits placed at
// the top of an fp32, whose exponent bias (127) exceeds e4m3's (7) by 120.
template <int I>
__device__ __forceinline__ float e4m3_scaled(uint32_t w) {
    const uint32_t t = (I == 3) ? w : (w << (24 - 8 * I));
    return __uint_as_float((uint32_t)((int32_t)t >> 4) & 0x87F00000u);
}
constexpr float kE4m3Half = 1.152921504606846976e18f;   // 2^60: half of 2^120

// Load kLE consecutive elements and widen them to fp32 pairs (element 2j in
// .x, 2j+1 in .y), ready for packed fp32x2 arithmetic.  fp8 (e4m3) codes are
// widened times 2^-120 (see e4m3_scaled); the caller folds 2^120 back in.
template <typename T, int LE>
__device__ __forceinline__ void load_pairs(const T *p, float2 *f) {
    if constexpr (sizeof(T) == 1) {
        static_assert(LE == 4 || LE == 8 || LE == 16, "load width");
        uint32_t w[LE / 4];
        if constexpr (LE == 16) {
            const uint4 v = *reinterpret_cast<const uint4 *>(p);
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else if constexpr (LE == 8) {
            const uint2 v = *reinterpret_cast<const uint2 *>(p);
            w[0] = v.x; w[1] = v.y;
        } else {
            w[0] = *reinterpret_cast<const uint32_t *>(p);
        }
#pragma unroll
        for (int k = 0; k < LE / 4; ++k) {
            f[2 * k] = make_float2(e4m3_scaled<0>(w[k]), e4m3_scaled<1>(w[k]));
            f[2 * k + 1] = make_float2(e4m3_scaled<2>(w[k]), e4m3_scaled<3>(w[k]));
        }
    } else if constexpr (sizeof(T) == 2) {
        if constexpr (LE == 8 || LE == 16) {
#pragma unroll
            for (int k = 0; k < LE / 8; ++k) {
                const uint4 v = *reinterpret_cast<const uint4 *>(p + 8 * k);
                f[4 * k] = make_float2(bf16lo(v.x), bf16hi(v.x));
                f[4 * k + 1] = make_float2(bf16lo(v.y), bf16hi(v.y));
                f[4 * k + 2] = make_float2(bf16lo(v.z), bf16hi(v.z));
                f[4 * k + 3] = make_float2(bf16lo(v.w), bf16hi(v.w));
            }
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
template <bool G = true>
struct TileCursorT {
    SegmentWalkerT<G> w;
    int t, len;
    __device__ void init(const PlanArgs &a, long long lo, long long hi, int seq,
                         long long base) {
        w.init(a, lo, hi, seq, base);
        t = 0;
        len = w.done() ? 0 : w.seg_len();
    }
    __device__ bool done() const { return w.done(); }
    __device__ int logical_block() const { return w.logical(w.blk_off + t); }
    __device__ int table_slot_of_tile() const { return w.slot(w.blk_off + t); }
    __device__ void next() {
        if (++t == len) {
            w.advance(len);
            t = 0;
            len = w.done() ? 0 : w.seg_len();
        }
    }
};
using TileCursor = TileCursorT<true>;

// Producer of warp 0: walks the CTA's tiles and keeps the physical block ids
// of the current segment in registers, 32 at a time (lane i holds tile
// bt0 + i), fetched with one coalesced load and the next batch prefetched
// half a batch early, so no bulk copy waits on a dependent global load.
// All 32 lanes call it together; lane 0 issues the copies.
template <bool G>
struct Producer {
    TileCursorT<G> cur;
    int id_cur, id_nxt, bt0;
    bool has_next;

    __device__ int fetch(const GqaParams &p, int i, int lane) const {
        const int j = i + lane;
        if (j >= cur.len) return -1;
        return __ldg(p.block_table + (size_t)cur.w.b * p.max_blocks +
                     cur.w.slot(cur.w.blk_off + j));
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

// Issue the bulk copies of one tile -- tile `sub` (kTileTok tokens) of the
// physical block `phys`, KV head of the cursor's unit -- into a stage.
// Called by one lane.
template <int D, typename T, int kTileTok, bool G>
__device__ __forceinline__ void issue_tile(const GqaParams &p, const TileCursorT<G> &cur,
                                          int phys, int sub, unsigned char *dst,
                                          uint64_t *full, uint64_t pol) {
    constexpr uint32_t kTileBytes = kTileTok * D * sizeof(T);
    constexpr uint32_t kScaleBytes = sizeof(T) == 1 ? kTileTok * 4 : 0;
    const int kvh = cur.w.unit / p.n_hc;
    if (phys < 0 || phys >= p.num_blocks) {
        raise_error(p.err, kErrBadBlock);
        mbar_arrive(full);
        return;
    }
    const size_t off = (((size_t)phys * p.H_kv + kvh) * kBlockSize + (size_t)sub * kTileTok) * D;
    mbar_arrive_expect_tx(full, 2 * (kTileBytes + kScaleBytes));
    bulk_load(dst, static_cast<const T *>(p.k_cache) + off, kTileBytes, full, pol);
    bulk_load(dst + kTileBytes, static_cast<const T *>(p.v_cache) + off, kTileBytes,
              full, pol);
    if constexpr (kScaleBytes > 0) {
        // The tile's row scales (fp8 cache), after the K and V codes.
        const size_t srow = off / D;
        bulk_load(dst + 2 * kTileBytes, p.k_scale + srow, kScaleBytes, full, pol);
        bulk_load(dst + 2 * kTileBytes + kScaleBytes, p.v_scale + srow, kScaleBytes, full, pol);
    }
}

// Arrival of one split of a unit: true for the last of its `ns` splits,
// which also puts the counter back to zero for the next launch.
__device__ __forceinline__ bool unit_arrive(unsigned *cnt, int ns) {
    const unsigned old = atomicAdd(cnt, 1u);
    const bool last = old + 1 == (unsigned)ns;
    if (last) *cnt = 0u;
    return last;
}

// The producer warp: streams the CTA's tiles, numbered n = 0, 1, ... over
// its range (kSub per block), into stage n % S once tile n - S has been
// released by the compute warps; then waits for the copies still in flight
// (the last S issued) so none lands after the CTA exits.  All 32 lanes run
// it; lane 0 issues the copies.
template <int D, int HC, typename T, typename TK, int S, int kTileTok, int kSub, bool G>
__device__ void produce_tiles(const GqaParams &p, const PlanArgs &pa, long long lo,
                              long long hi, int seq, long long base,
                              unsigned char *stage_base, uint64_t *full_bar,
                              uint64_t *empty_bar, unsigned char *q_ring, int q_slot_bytes,
                              uint64_t *q_full, uint64_t *q_empty, int lane,
                              volatile int *abort_flag, unsigned long long *s_gmask) {
    constexpr int kStageBytes =
        2 * (kTileTok * D * (int)sizeof(TK) + (sizeof(TK) == 1 ? kTileTok * 4 : 0));
    constexpr uint32_t kQBytes = HC * D * sizeof(T);
    const uint64_t pol = l2_policy_evict_first();
    Producer<G> prod;
    prod.cur.init(pa, lo, hi, seq, base);
    const long long n_tiles = (hi - lo) * kSub;
    int sub = 0, phys = -1, seg = 0;
    long long m = 0;
    for (; m < n_tiles; ++m) {
        if (sub == 0 && prod.cur.t == 0) {
            // First tile of a segment: its unit's queries go first, into
            // slot seg % 2 once segment seg - 2 has read that slot.
            const int qs = seg & 1;
            if (seg >= 2) {
                const bool fr = mbar_wait(&q_empty[qs], (uint32_t)(((seg >> 1) - 1) & 1),
                                          p.timeout_ns, p.err, abort_flag);
                if (!__all_sync(0xffffffffu, fr)) break;
            }
            if (lane == 0) {
                const int u = prod.cur.w.unit;
                const int head0 = (u / p.n_hc) * p.group + (u % p.n_hc) * HC;
                mbar_arrive_expect_tx(&q_full[qs], kQBytes);
                bulk_load(q_ring + qs * q_slot_bytes,
                          static_cast<const T *>(p.q) +
                              ((size_t)prod.cur.w.b * p.H_q + head0) * D,
                          kQBytes, &q_full[qs]);
            }
            ++seg;
        }
        const int s = (int)(m % S);
        if (m >= S) {
            const bool fr = mbar_wait(&empty_bar[s], (uint32_t)(((m / S) - 1) & 1),
                                      p.timeout_ns, p.err, abort_flag);
            if (!__all_sync(0xffffffffu, fr)) break;
        }
        if (sub == 0) phys = prod.block_id(p, lane);
        if constexpr (G) {
            // The block's global positions, for the masking of keys below
            // the window (ordered before the stage's arrival below).
            const int blk = prod.cur.logical_block();
            const unsigned long long gm = blk * kBlockSize < prod.cur.w.lo
                                              ? global_mask(p.vis, prod.cur.w.b, blk, lane)
                                              : 0ull;
            if (lane == 0) s_gmask[s] = gm;
        }
        if (lane == 0)
            issue_tile<D, TK, kTileTok, G>(p, prod.cur, phys, sub,
                                       stage_base + (size_t)s * kStageBytes, &full_bar[s],
                                       pol);
        if (++sub == kSub) {
            sub = 0;
            prod.cur.next();
        }
    }
    if (lane == 0) {
        for (long long k = m > S ? m - S : 0; k < m; ++k)
            mbar_wait(&full_bar[k % S], (uint32_t)((k / S) & 1), p.timeout_ns, p.err,
                      nullptr);
        for (int j = seg > 2 ? seg - 2 : 0; j < seg; ++j)
            mbar_wait(&q_full[j & 1], (uint32_t)((j >> 1) & 1), p.timeout_ns, p.err,
                      nullptr);
    }
}

// Loads the published partials of a unit's other splits (slots slot0 ..
// slot0 + ns - 1 except this CTA's own, `own`) into shared memory: pf_o
// [ns - 1][HC][D] and pf_lse [ns - 1][HC], other split i at index
// i - (i > own).  Each thread loads the elements it later combines (the same
// thread-to-element map as the combine), so no barrier is needed between.
template <int D, int HC, int NT>
__device__ __forceinline__ void prefetch_splits(const GqaParams &p, int et, long long slot0,
                                                int ns, int own, float *pf_o, float *pf_lse) {
    for (int e = et * 4; e < HC * D; e += NT * 4) {
        for (int i0 = 0; i0 < ns; i0 += 4) {
            float4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (i0 + k < ns && i0 + k != own)
                    v[k] = __ldcg(reinterpret_cast<const float4 *>(
                        p.ws_o + (slot0 + i0 + k) * HC * D + e));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + k;
                if (i < ns && i != own)
                    *reinterpret_cast<float4 *>(pf_o + (size_t)(i - (i > own)) * HC * D + e) =
                        v[k];
            }
        }
    }
    for (int k = et; k < ns * HC; k += NT) {
        const int i = k / HC;
        if (i != own) pf_lse[(i - (i > own)) * HC + k % HC] = __ldcg(p.ws_lse + slot0 * HC + k);
    }
}

// Segment epilogue, run by the kEpiThreads epilogue threads (et = 0 ..) on the
// compute warps' stashed states: s_mo [NW][HC][D] partial outputs, s_mm /
// s_ml [NW][HC] running max / sum of each warp.  Merges them, then writes the
// unit's output (one split) or combines the unit's splits:
//     out = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L),
// over the splits in CTA order (fixed, deterministic).  A split that finds
// every other split of its unit already arrived is the last one: it combines
// at once, taking its own (O, lse) from shared memory, without publishing
// them -- the common case for the last segment of a CTA, whose unit's other
// split ran at the start of the next CTA's range.  `pre` says this thread
// has already loaded the other splits' partials into pf_o / pf_lse (while
// the segment ran).  Otherwise the split publishes its fp32 partial and
// arrives on the unit's counter, and the last split to arrive combines.
// Either way the same values are summed in the same order.
template <int D, int HC, typename T, int NW, int NT, int PRE>
__device__ void segment_epilogue(const GqaParams &p, int et, long long u, int c0, int ns,
                                 long long slot, T *out_u, float *s_mo, const float *s_mm,
                                 const float *s_ml, float *s_w, volatile int *last_flag,
                                 bool pre, float *pf_o, float *pf_lse) {
    float *s_inv = s_w + NW * HC;          // [HC]
    float *s_lse = s_inv + HC;             // [HC]
    // Other splits already arrived?  Read early; used after the merge.
    unsigned seen = 0;
    if (ns > 1 && et == 0) seen = pre ? (unsigned)(ns - 1) : ld_relaxed_gpu(p.ws_cnt + u);
    // Per head: the common max, each warp's weight, the normaliser.
    if (et < HC) {
        const int g = et;
        float M = -1e30f;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, s_mm[w * HC + g]);
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float wt = exp2f(s_mm[w * HC + g] - M);
            s_w[w * HC + g] = wt;
            den = fmaf(wt, s_ml[w * HC + g], den);
        }
        s_inv[g] = 1.f / den;
        s_lse[g] = M + log2f(den);
    }
    named_barrier(1, NT);
    // The merged output; for a split unit it replaces warp 0's stash (each
    // element is read and rewritten by the same thread).
    for (int e = et * 4; e < HC * D; e += NT * 4) {
        const int g = e / D;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float wt = s_w[w * HC + g];
            const float4 v = *reinterpret_cast<const float4 *>(s_mo + (size_t)w * HC * D + e);
            acc.x = fmaf(wt, v.x, acc.x);
            acc.y = fmaf(wt, v.y, acc.y);
            acc.z = fmaf(wt, v.z, acc.z);
            acc.w = fmaf(wt, v.w, acc.w);
        }
        const float iv = s_inv[g];
        acc.x *= iv; acc.y *= iv; acc.z *= iv; acc.w *= iv;
        if (ns == 1) {
            out_u[e] = ElemTraits<T>::from_float(acc.x);
            out_u[e + 1] = ElemTraits<T>::from_float(acc.y);
            out_u[e + 2] = ElemTraits<T>::from_float(acc.z);
            out_u[e + 3] = ElemTraits<T>::from_float(acc.w);
        } else {
            *reinterpret_cast<float4 *>(s_mo + e) = acc;
        }
    }
    if (ns == 1) return;
    // The other splits' (O, lse) fit in the prefetch buffer: the combine
    // reads them from shared memory, and the last split need not publish.
    const bool fits = ns - 1 <= PRE;
    if (et == 0) {
        const bool fast = fits && seen == (unsigned)(ns - 1);
        if (fast) {
            fence_acq_rel_gpu();               // the other splits' partials, then
            st_relaxed_gpu(p.ws_cnt + u, 0u);  // the counter back to zero
        }
        *last_flag = fast ? 2 : 0;
    }
    named_barrier(1, NT);
    if (*last_flag != 2) {
        // Publish this split's partial and arrive.  The barrier orders every
        // thread's stores before thread 0's fence, which publishes them,
        // cumulatively, before the arrival (and orders the last arrival's
        // reads after the other splits' partials).
        for (int e = et * 4; e < HC * D; e += NT * 4)
            *reinterpret_cast<float4 *>(p.ws_o + slot * HC * D + e) =
                *reinterpret_cast<const float4 *>(s_mo + e);
        if (et < HC) p.ws_lse[slot * HC + et] = s_lse[et];
        named_barrier(1, NT);
        if (et == 0) {
            __threadfence();
            const bool last = unit_arrive(p.ws_cnt + u, ns);
            if (last) __threadfence();
            *last_flag = last ? 1 : 0;
        }
        named_barrier(1, NT);
        if (!*last_flag) return;
    }
    const long long slot0 = u + c0;
    const int own = (int)(slot - slot0);
    float *wts = s_mo + HC * D;            // [ns][HC] split weights
    if (fits) {
        // The other splits' (O, lse) in shared memory (loaded here, in one
        // round trip, unless already prefetched), this split's own from the
        // merge; then the split weights 2^(lse - L), and each output is one
        // weighted sum.
        if (!pre) prefetch_splits<D, HC, NT>(p, et, slot0, ns, own, pf_o, pf_lse);
        for (int i = et; i < ns * HC; i += NT) {
            const int si = i / HC;
            wts[i] = si == own ? s_lse[i % HC] : pf_lse[(si - (si > own)) * HC + i % HC];
        }
        named_barrier(1, NT);
        if (et < HC) {
            const int g = et;
            float L = kNegInf;
            for (int i = 0; i < ns; ++i) L = fmaxf(L, wts[i * HC + g]);
            float den = 0.f;
            for (int i = 0; i < ns; ++i) {
                const float w = exp2f(wts[i * HC + g] - L);
                wts[i * HC + g] = w;
                den += w;
            }
            s_inv[g] = 1.f / den;
        }
        named_barrier(1, NT);
        for (int e = et * 4; e < HC * D; e += NT * 4) {
            const int g = e / D;
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
            for (int i = 0; i < ns; ++i) {
                const float w = wts[i * HC + g];
                const float4 v = *reinterpret_cast<const float4 *>(
                    i == own ? s_mo + e : pf_o + (size_t)(i - (i > own)) * HC * D + e);
                r0 = fmaf(w, v.x, r0);
                r1 = fmaf(w, v.y, r1);
                r2 = fmaf(w, v.z, r2);
                r3 = fmaf(w, v.w, r3);
            }
            const float iv = s_inv[g];
            out_u[e] = ElemTraits<T>::from_float(r0 * iv);
            out_u[e + 1] = ElemTraits<T>::from_float(r1 * iv);
            out_u[e + 2] = ElemTraits<T>::from_float(r2 * iv);
            out_u[e + 3] = ElemTraits<T>::from_float(r3 * iv);
        }
    } else if (ns <= (NW - 1) * D) {
        // More splits: weights in shared memory, partials from the
        // published copies (this split's own included), eight loads in flight.
        for (int i = et; i < ns * HC; i += NT) wts[i] = __ldcg(p.ws_lse + slot0 * HC + i);
        named_barrier(1, NT);
        if (et < HC) {
            const int g = et;
            float L = kNegInf;
            for (int i = 0; i < ns; ++i) L = fmaxf(L, wts[i * HC + g]);
            float den = 0.f;
            for (int i = 0; i < ns; ++i) {
                const float w = exp2f(wts[i * HC + g] - L);
                wts[i * HC + g] = w;
                den += w;
            }
            s_inv[g] = 1.f / den;
        }
        named_barrier(1, NT);
        for (int e = et * 4; e < HC * D; e += NT * 4) {
            const int g = e / D;
            const float *src = p.ws_o + slot0 * HC * D + e;
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll 8
            for (int i = 0; i < ns; ++i) {
                const float w = wts[i * HC + g];
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + (size_t)i * HC * D));
                r0 = fmaf(w, v.x, r0);
                r1 = fmaf(w, v.y, r1);
                r2 = fmaf(w, v.z, r2);
                r3 = fmaf(w, v.w, r3);
            }
            const float iv = s_inv[g];
            out_u[e] = ElemTraits<T>::from_float(r0 * iv);
            out_u[e + 1] = ElemTraits<T>::from_float(r1 * iv);
            out_u[e + 2] = ElemTraits<T>::from_float(r2 * iv);
            out_u[e + 3] = ElemTraits<T>::from_float(r3 * iv);
        }
    } else {
        // Many splits: everything from the published partials.
        for (int e = et * 4; e < HC * D; e += NT * 4) {
            const int g = e / D, k = e % D;
            float L = kNegInf;
            for (int i = 0; i < ns; ++i) L = fmaxf(L, __ldcg(p.ws_lse + (slot0 + i) * HC + g));
            float den = 0.f, r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
            for (int i = 0; i < ns; ++i) {
                const float w = exp2f(__ldcg(p.ws_lse + (slot0 + i) * HC + g) - L);
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                    p.ws_o + ((slot0 + i) * HC + g) * D + k));
                r0 = fmaf(w, v.x, r0);
                r1 = fmaf(w, v.y, r1);
                r2 = fmaf(w, v.z, r2);
                r3 = fmaf(w, v.w, r3);
                den += w;
            }
            const float iv = 1.f / den;
            out_u[e] = ElemTraits<T>::from_float(r0 * iv);
            out_u[e + 1] = ElemTraits<T>::from_float(r1 * iv);
            out_u[e + 2] = ElemTraits<T>::from_float(r2 * iv);
            out_u[e + 3] = ElemTraits<T>::from_float(r3 * iv);
        }
    }
}

// G: the call has an explicit global set (p.vis.n_g > 0).  It is a template
// flag so that calls without one run a loop free of its masking code, which
// measurably slowed the common case when present but not taken.
template <int D, int HC, typename T, typename TK, bool G>
__global__ void __launch_bounds__(GqaCfg<D, HC, T, TK>::kThreads, 1)
gqa_split_kernel(const GqaParams p) {
    using C = GqaCfg<D, HC, T, TK>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *stage_base = smem;
    unsigned char *q_ring = smem + S * C::kStageBytes;          // [2][HC][D]
    constexpr int kQSlot = C::kQRingBytes / 2;
    float *s_scores = reinterpret_cast<float *>(q_ring + C::kQRingBytes);
    float *s_mo = s_scores + C::kScoreBytes / 4;
    float *s_mm = s_mo + C::kMergeOBytes / 4;
    float *s_ml = s_mm + C::kNW * HC;
    float *s_w = s_ml + C::kNW * HC;                    // epilogue scratch
    unsigned char *misc = reinterpret_cast<unsigned char *>(s_w + C::kEpiBytes / 4);
    float *pf_o = reinterpret_cast<float *>(misc + C::kMiscBytes);   // [kPreMax][HC][D]
    float *pf_lse = pf_o + C::kPreMax * HC * D;                       // [kPreMax][HC]
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(misc);
    uint64_t *empty_bar = full_bar + S;
    uint64_t *q_full = empty_bar + S;                   // [2]
    uint64_t *q_empty = q_full + 2;                     // [2]
    uint64_t *epi_full = q_empty + 2;                   // stash written
    uint64_t *epi_empty = epi_full + 1;                 // stash consumed
    uint64_t *never_bar = epi_empty + 1;                // fault injection
    PlanScratch *plan_sh = reinterpret_cast<PlanScratch *>(never_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(plan_sh + 1);
    volatile int *last_flag = abort_flag + 1;
    volatile int *epi_vote = last_flag + 1;             // [2][4]: epilogue warps' wait outcomes
    // Per stage: global positions among the staged block's keys below the
    // window (bit t: key 64 * block + t), written by the producer before it
    // arms the stage, read by the compute warps after they wait on it.
    unsigned long long *s_gmask = reinterpret_cast<unsigned long long *>(misc + 768);
    static_assert((2 * S + 7) * 8 + sizeof(PlanScratch) + 8 + 32 <= 768 &&
                      768 + 8 * S <= C::kMiscBytes,
                  "misc shared-memory layout");
    static_assert(C::kEpiThreads % 32 == 0 && C::kEpiThreads / 32 <= 4, "epilogue vote slots");

    const int tid = threadIdx.x;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], C::kWPG);
        }
        mbar_init(epi_full, C::kNW * 32);
        mbar_init(epi_empty, C::kEpiThreads);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], C::kNW);
        }
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    // Programmatic dependent launch: everything above overlaps the previous
    // kernel on the stream; inputs are read only after it has completed.
    pdl_wait_primary();
    pdl_launch_dependents();

    const int units = p.H_kv * p.n_hc;
    PlanArgs pa{p.seq_lens, p.B, units, p.vis, p.max_blocks, p.num_ctas};
    plan_locate(pa, blockIdx.x, plan_sh, blockIdx.x == 0 ? p.ws_prefix : nullptr,
                p.err);
    const long long W = plan_sh->total;
    const int P = working_ctas(W, p.num_ctas);
    if ((int)blockIdx.x >= P) return;
    const long long lo = cta_bound(blockIdx.x, W, P);
    const long long hi = cta_bound(blockIdx.x + 1, W, P);
    SegmentWalkerT<G> walk;
    walk.init(pa, lo, hi, plan_sh->seq, plan_sh->base);

    // ------------------------------------------------------------ producer
    if (tid < 128) {
        regs_decrease<C::kProducerRegs>();
        if (tid < 32) {
            produce_tiles<D, HC, T, TK, S, C::kTileTok, C::kSub, G>(
                p, pa, lo, hi, plan_sh->seq, plan_sh->base, stage_base, full_bar, empty_bar,
                q_ring, kQSlot, q_full, q_empty, lane, abort_flag, s_gmask);
        } else {
            const int et = tid - 32;
            // A sequence without a visible block (empty) has a zero output
            // and no split works on it.
            for (int b = blockIdx.x; b < p.B; b += P) {
                int fb, sb;
                bool bad;
                if (visible_blocks(p.seq_lens[b], p.vis, p.max_blocks, &fb, &sb, &bad, b) == 0) {
                    T *o = static_cast<T *>(p.out) + (size_t)b * p.H_q * D;
                    for (int i = et; i < p.H_q * D; i += C::kEpiThreads)
                        o[i] = ElemTraits<T>::from_float(0.f);
                }
            }
            // The epilogue of every segment, while the compute warps go on
            // with the next one.
            SegmentWalkerT<G> ew;
            ew.init(pa, lo, hi, plan_sh->seq, plan_sh->base);
            for (int es = 0; !ew.done(); ++es) {
                const int len = ew.seg_len();
                const long long u = (long long)ew.b * units + ew.unit;
                const long long s_u = ew.pos - ew.blk_off;     // the unit's first block
                const int c0 = cta_of(s_u, W, P);
                const int ns = cta_of(s_u + ew.nb - 1, W, P) - c0 + 1;
                const int own = (int)blockIdx.x - c0;
                // While the segment runs, watch the unit's counter: once the
                // other splits have all arrived, load their partials.
                bool pre = false;
                const bool watch = ns > 1 && ns - 1 <= C::kPreMax;
                const unsigned *cnt = p.ws_cnt + u;
                auto idle = [&]() {
                    if (watch && !pre && ld_relaxed_gpu(cnt) == (unsigned)(ns - 1)) {
                        fence_acq_rel_gpu();
                        prefetch_splits<D, HC, C::kEpiThreads>(p, et, u + c0, ns, own, pf_o,
                                                                pf_lse);
                        pre = true;
                    }
                };
                const bool got = mbar_wait_watch(epi_full, (uint32_t)(es & 1), p.timeout_ns,
                                                 p.err, abort_flag, idle);
                // The epilogue warps leave that wait separately: a stash that
                // completes just as an abort is raised can end one warp's
                // wait with the phase and another's with the abort.  Every
                // warp reaches this barrier either way (each wait is bounded)
                // and all go on only if all saw the stash, so no warp is ever
                // left waiting at a barrier of the epilogue below.
                volatile int *vote = epi_vote + 4 * (es & 1);
                if (lane == 0) vote[et >> 5] = got ? 1 : 0;
                named_barrier(1, C::kEpiThreads);
                bool all_got = true;
#pragma unroll
                for (int w = 0; w < C::kEpiThreads / 32; ++w) all_got = all_got && vote[w];
                if (!all_got) break;
                const int head0 = (ew.unit / p.n_hc) * p.group + (ew.unit % p.n_hc) * HC;
                T *out_u = static_cast<T *>(p.out) + ((size_t)ew.b * p.H_q + head0) * D;
                segment_epilogue<D, HC, T, C::kNW, C::kEpiThreads, C::kPreMax>(
                    p, et, u, c0, ns, u + blockIdx.x, out_u, s_mo, s_mm, s_ml, s_w, last_flag,
                    pre, pf_o, pf_lse);
                mbar_arrive(epi_empty);
                ew.advance(len);
            }
            // After an abort the CTA still arrives on every unit it had not
            // finished, so each unit's counter is back at zero when the
            // launch ends (those outputs are not valid; the error word says so).
            if (et == 0) {
                while (!ew.done()) {
                    const int len = ew.seg_len();
                    const long long s_u = ew.pos - ew.blk_off;
                    const int ns = cta_of(s_u + ew.nb - 1, W, P) - cta_of(s_u, W, P) + 1;
                    if (ns > 1) unit_arrive(p.ws_cnt + (long long)ew.b * units + ew.unit, ns);
                    ew.advance(len);
                }
            }
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    regs_increase<C::kConsumerRegs>();
    const int ctid = tid - 128;             // thread among the compute warps
    const int warp = ctid >> 5;             // compute warp 0 .. kNW-1
    const int grp = warp / C::kWPG;         // tile group of this warp
    const int wig = warp % C::kWPG;         // warp within its group
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

    float *sc = s_scores + warp * C::kTPW * C::kHCP;   // [TPW][HCP]
    long long seg_t0 = 0;                  // first tile of the current segment
    int n_seg = 0;

    constexpr int LP = C::kLE / 2;          // pairs per load
    constexpr int EP = C::kEPL / 2;         // pairs per lane

    while (!*abort_flag && !walk.done()) {
        const int len = walk.seg_len();
        const long long seg_t1 = seg_t0 + (long long)len * C::kSub;
        const int Tb = walk.T;
        const int lo_tok = walk.lo;
        const int sink = p.vis.sink;

        // The unit's queries, staged in shared memory by the producer.
        if (!mbar_wait(&q_full[n_seg & 1], (uint32_t)((n_seg >> 1) & 1), p.timeout_ns, p.err,
                       abort_flag))
            break;
        const T *qs = reinterpret_cast<const T *>(q_ring + (n_seg & 1) * kQSlot);
        float2 q2[HC][EP];
        // fp8 cache: half of the 2^120 the widened codes lack goes into q,
        // the other half into each row's scale.
        const float qsc = C::kFp8 ? p.scale_log2 * kE4m3Half : p.scale_log2;
        const float2 sc2 = make_float2(qsc, qsc);
#pragma unroll
        for (int g = 0; g < HC; ++g) {
#pragma unroll
            for (int c = 0; c < C::kCPL; ++c) {
                float2 f[LP];
                load_pairs<T, C::kLE>(qs + g * D + col[c], f);
#pragma unroll
                for (int j = 0; j < LP; ++j) q2[g][c * LP + j] = __fmul2_rn(f[j], sc2);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[n_seg & 1]);
        float2 o2[HC][EP];
#pragma unroll
        for (int g = 0; g < HC; ++g)
#pragma unroll
            for (int j = 0; j < EP; ++j) o2[g][j] = make_float2(0.f, 0.f);
        float m_run[C::kPasses], l_run[C::kPasses];
#pragma unroll
        for (int ps = 0; ps < C::kPasses; ++ps) { m_run[ps] = -1e30f; l_run[ps] = 0.f; }

        bool ok = true;
        // This group's first tile of the segment.
        long long n = seg_t0 + (long long)(((grp - (int)(seg_t0 % C::kNG)) % C::kNG + C::kNG) % C::kNG);
        for (; n < seg_t1; n += C::kNG) {
            const int stage = (int)(n % S);
            if (!mbar_wait(&full_bar[stage], (uint32_t)((n / S) & 1), p.timeout_ns, p.err,
                           abort_flag)) {
                ok = false;
                break;
            }
            const TK *Ks = reinterpret_cast<const TK *>(stage_base + stage * C::kStageBytes);
            const TK *Vs = Ks + C::kTileTok * D;
            // fp8 cache: row scales after the codes
            const float *ksc = reinterpret_cast<const float *>(Vs + C::kTileTok * D);
            const float *vsc = ksc + C::kTileTok;
            const int tl = (int)(n - seg_t0);
            const int blk = walk.logical(walk.blk_off + tl / C::kSub);
            const int tok0 = blk * kBlockSize + (tl % C::kSub) * C::kTileTok + wig * C::kTPW;
            const int row0 = wig * C::kTPW;
            // Global positions among this block's keys below the window
            // (bit t: key blk * 64 + t), staged by the producer.
            unsigned long long gmask = 0ull;
            if constexpr (G)
                if (blk * kBlockSize < lo_tok) gmask = s_gmask[stage];

            // ---- scores: partial dot products, reduced over the row group
#pragma unroll
            for (int ch = 0; ch < C::kChunks; ++ch) {
                float2 acc[C::kChunk * HC];
#pragma unroll
                for (int i = 0; i < C::kChunk; ++i) {
                    const int it = ch * C::kChunk + i;
                    const TK *krow = Ks + (row0 + it * C::kRPW + rg) * D;
#pragma unroll
                    for (int g = 0; g < HC; ++g) acc[i * HC + g] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < C::kCPL; ++c) {
                        float2 kp[LP];
                        load_pairs<TK, C::kLE>(krow + col[c], kp);
#pragma unroll
                        for (int g = 0; g < HC; ++g)
#pragma unroll
                            for (int j = 0; j < LP; ++j)
                                acc[i * HC + g] =
                                    __ffma2_rn(q2[g][c * LP + j], kp[j], acc[i * HC + g]);
                    }
                }
                float part[C::kChunk * HC];
#pragma unroll
                for (int i = 0; i < C::kChunk * HC; ++i) part[i] = acc[i].x + acc[i].y;
                using RR = RowReduce<C::kChunk * HC, C::kLPR>;
                const int base = RR::run(part, lane);
#pragma unroll
                for (int i = 0; i < RR::final_count(); ++i) {
                    const int v = base + i;
                    const int it = ch * C::kChunk + v / HC, g = v % HC;
                    float sv = part[i];
                    if constexpr (C::kFp8) sv *= ksc[row0 + it * C::kRPW + rg] * kE4m3Half;
                    sc[(it * C::kRPW + rg) * C::kHCP + g] = sv;
                }
            }
            __syncwarp();

            // ---- online softmax over this warp's rows (log2 domain), lazy:
            // probabilities are taken against the running max m_run, which
            // (with O and the partial sums) is raised only when a score
            // exceeds it by more than kRescaleLog2 -- every probability stays
            // below 2^kRescaleLog2.  Each lane keeps the partial sum of its
            // own (token slot, head); they are added up at the merge.
#pragma unroll
            for (int ps = 0; ps < C::kPasses; ++ps) {
                const int gs = lane / C::kTPW + C::kHPP * ps;
                const int tt = lane % C::kTPW;
                const bool active = gs < HC;
                const int pos = tok0 + tt;
                const bool valid = active && pos < Tb &&
                                   (pos >= lo_tok || pos < sink ||
                                    ((gmask >> (pos - blk * kBlockSize)) & 1ull));
                const float s = valid ? sc[tt * C::kHCP + gs] : kNegInf;
                if (__any_sync(0xffffffffu, s > m_run[ps] + kRescaleLog2)) {
                    float mx = s;
#pragma unroll
                    for (int m = 1; m < C::kTPW; m <<= 1)
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
                    const float m_new = fmaxf(m_run[ps], mx);
                    const float alpha = exp2f(m_run[ps] - m_new);
                    l_run[ps] *= alpha;
                    m_run[ps] = m_new;
#pragma unroll
                    for (int j = 0; j < C::kHPP; ++j) {
                        const int g = C::kHPP * ps + j;
                        if (g < HC) {
                            const float a = __shfl_sync(0xffffffffu, alpha, j * C::kTPW);
                            const float2 a2 = make_float2(a, a);
#pragma unroll
                            for (int e = 0; e < EP; ++e) o2[g][e] = __fmul2_rn(o2[g][e], a2);
                        }
                    }
                }
                const float pr = exp2f(s - m_run[ps]);
                l_run[ps] += pr;
                if (active) sc[tt * C::kHCP + gs] = pr;
            }
            __syncwarp();

            // ---- P V
#pragma unroll
            for (int it = 0; it < C::kIters; ++it) {
                const int rl = it * C::kRPW + rg;
                const TK *vrow = Vs + (row0 + rl) * D;
                float pg[C::kHCP];
                load_row<C::kHCP>(sc + rl * C::kHCP, pg);
                float vf = 1.f;
                if constexpr (C::kFp8) vf = vsc[row0 + rl] * kE4m3Half;
                float2 pp[HC];
#pragma unroll
                for (int g = 0; g < HC; ++g) pp[g] = make_float2(pg[g] * vf, pg[g] * vf);
#pragma unroll
                for (int c = 0; c < C::kCPL; ++c) {
                    float2 vp[LP];
                    load_pairs<TK, C::kLE>(vrow + col[c], vp);
#pragma unroll
                    for (int g = 0; g < HC; ++g)
#pragma unroll
                        for (int j = 0; j < LP; ++j)
                            o2[g][c * LP + j] = __ffma2_rn(pp[g], vp[j], o2[g][c * LP + j]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[stage]);
        }
        if (!ok) break;

        SegmentWalkerT<G> next = walk;
        next.advance(len);

        // ---- stash this warp's state for the epilogue warps
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
#pragma unroll
        for (int ps = 0; ps < C::kPasses; ++ps)
#pragma unroll
            for (int m = 1; m < C::kTPW; m <<= 1)
                l_run[ps] += __shfl_xor_sync(0xffffffffu, l_run[ps], m);
        // The epilogue of the previous segment must be done with the stash.
        if (n_seg > 0 && !mbar_wait(epi_empty, (uint32_t)((n_seg - 1) & 1), p.timeout_ns,
                                    p.err, abort_flag))
            break;
        if (rg == 0) {
#pragma unroll
            for (int g = 0; g < HC; ++g)
#pragma unroll
                for (int c = 0; c < C::kCPL; ++c)
#pragma unroll
                    for (int j = 0; j < LP; ++j)
                        *reinterpret_cast<float2 *>(&s_mo[(warp * HC + g) * D + col[c] + 2 * j]) =
                            C::kFp8 ? __fmul2_rn(o2[g][c * LP + j],
                                                 make_float2(kE4m3Half, kE4m3Half))
                                    : o2[g][c * LP + j];
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
        mbar_arrive(epi_full);
        ++n_seg;
        seg_t0 = seg_t1;
        walk = next;
    }
}

struct CombineParams {
    const int32_t *seq_lens;
    const long long *ws_prefix;
    const float *ws_o;
    const float *ws_lse;
    void *out;
    int B, H_q, H_kv, group, n_hc, max_blocks, num_ctas;
    Visibility vis;
    int D, HC;               // head dim, query heads per unit
    int copies;              // partials per (unit, CTA) slot (>= 1)
    int lanes;               // threads per float4 of output: 1, 4 or 8
    int blocks_per_unit;     // CTAs per unit: combine_blocks_per_unit(HC, D, lanes)
};

constexpr int kCombineThreads = 256;
constexpr int kCombineMaxW = 4096;       // (head, partial) weights held in shared memory

// Threads that share one float4 of output in the combine: more when a unit
// has many partials (each takes every lanes-th partial, so the chain of
// dependent loads per thread stays short and few-unit shapes still spread
// over many CTAs), one when it has few.
__host__ __device__ constexpr int combine_lanes(int expected_partials) {
    return expected_partials >= 256 ? 32
           : expected_partials >= 96 ? 16
           : expected_partials >= 32 ? 8
           : expected_partials >= 8 ? 4 : 1;
}
// CTAs of the combine kernel per unit.
__host__ __device__ constexpr int combine_blocks_per_unit(int HC, int D, int lanes) {
    return (HC * D + 4 * (kCombineThreads / lanes) - 1) / (4 * (kCombineThreads / lanes));
}

// out = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L) over the unit's split
// partials (`copies` per slot, slot-major), in CTA order (fixed,
// deterministic).  A partial with lse = -inf has weight zero.  A CTA makes
// 4 * kCombineThreads / lanes consecutive outputs of one unit: the split
// weights of the heads it spans are computed once, in shared memory (one
// warp per head), then each float4 of output is accumulated by `lanes`
// threads that take every lanes-th partial, summed with shuffles in a fixed
// order (deterministic).
template <typename T>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const CombineParams p) {
    __shared__ long long s_first;
    __shared__ int s_n, s_nb;
    __shared__ float s_w[kCombineMaxW];
    __shared__ float s_inv[kCombineThreads / 4];
    pdl_wait_primary();
    const int units = p.H_kv * p.n_hc;
    const int u = blockIdx.x / p.blocks_per_unit;
    const int part = blockIdx.x % p.blocks_per_unit;
    const int b = u / units, rem = u % units;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        int fb, sb;
        bool bad;
        const int nb = visible_blocks(p.seq_lens[b], p.vis, p.max_blocks, &fb, &sb, &bad, b);
        s_nb = nb;
        s_n = 0;
        s_first = 0;
        if (nb > 0) {
            const long long W = p.ws_prefix[p.B];
            const int P = working_ctas(W, p.num_ctas);
            const long long s_u = p.ws_prefix[b] + (long long)rem * nb;
            const int c0 = cta_of(s_u, W, P);
            const int c1 = cta_of(s_u + nb - 1, W, P);
            s_n = (c1 - c0 + 1) * p.copies;
            s_first = ((long long)u + c0) * p.copies;
        }
    }
    __syncthreads();
    const int lanes = p.lanes;
    const int outs = 4 * (kCombineThreads / lanes);      // outputs of this CTA
    const int total = p.HC * p.D;
    const int e0 = part * outs;
    const int g0 = e0 / p.D;
    const int e_last = (e0 + outs < total ? e0 + outs : total) - 1;
    const int nh = e_last / p.D - g0 + 1;                // heads spanned
    const int kvh = rem / p.n_hc, hc = rem % p.n_hc;
    T *out = static_cast<T *>(p.out) +
             ((size_t)b * p.H_q + kvh * p.group + hc * p.HC) * p.D;
    const int n = s_n;
    const long long s0 = s_first;
    const int o = tid / lanes, j = tid % lanes;
    const int e = e0 + 4 * o;                            // this thread's float4
    const bool has = e < total;
    const int g = has ? e / p.D : g0;
    if (s_nb == 0 || nh * n > kCombineMaxW || nh > kCombineThreads / 4) {
        // Empty sequence: zeros.  More weights than fit: plain two-pass loop.
        if (!has || j != 0) return;
        float r[4] = {0.f, 0.f, 0.f, 0.f};
        if (s_nb > 0) {
            float L = kNegInf;
            for (int i = 0; i < n; ++i) L = fmaxf(L, p.ws_lse[(s0 + i) * p.HC + g]);
            float den = 0.f;
            for (int i = 0; i < n; ++i) {
                const float w = exp2f(p.ws_lse[(s0 + i) * p.HC + g] - L);
                const float4 v = *reinterpret_cast<const float4 *>(
                    p.ws_o + ((s0 + i) * p.HC + g) * p.D + (e % p.D));
                r[0] = fmaf(w, v.x, r[0]);
                r[1] = fmaf(w, v.y, r[1]);
                r[2] = fmaf(w, v.z, r[2]);
                r[3] = fmaf(w, v.w, r[3]);
                den += w;
            }
            const float inv = 1.f / den;
#pragma unroll
            for (int q = 0; q < 4; ++q) r[q] *= inv;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) out[e + q] = ElemTraits<T>::from_float(r[q]);
        return;
    }
    // Split weights of heads g0 .. g0 + nh - 1 ([head][partial]), one warp
    // per head.
    for (int hh = warp; hh < nh; hh += kCombineThreads / 32) {
        const int gh = g0 + hh;
        float *w_h = s_w + hh * n;
        float L = kNegInf;
        for (int i = lane; i < n; i += 32) {
            const float v = p.ws_lse[(s0 + i) * p.HC + gh];
            w_h[i] = v;
            L = fmaxf(L, v);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, m));
        float den = 0.f;
        for (int i = lane; i < n; i += 32) {
            const float w = exp2f(w_h[i] - L);
            w_h[i] = w;
            den += w;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) den += __shfl_xor_sync(0xffffffffu, den, m);
        if (lane == 0) s_inv[hh] = 1.f / den;
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (has) {
        const float *wts = s_w + (g - g0) * n;
        const float *src = p.ws_o + (s0 * p.HC + g) * p.D + (e % p.D);
        const size_t stride = (size_t)p.HC * p.D;
#pragma unroll 4
        for (int i = j; i < n; i += lanes) {
            const float w = wts[i];
            const float4 v = *reinterpret_cast<const float4 *>(src + (size_t)i * stride);
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
    }
    for (int m = lanes / 2; m >= 1; m >>= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
    }
    if (has && j == 0) {
        const float inv = s_inv[g - g0];
        out[e] = ElemTraits<T>::from_float(acc.x * inv);
        out[e + 1] = ElemTraits<T>::from_float(acc.y * inv);
        out[e + 2] = ElemTraits<T>::from_float(acc.z * inv);
        out[e + 3] = ElemTraits<T>::from_float(acc.w * inv);
    }
}

}  // namespace attn
