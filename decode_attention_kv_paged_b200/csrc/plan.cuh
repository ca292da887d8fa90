// plan.cuh -- split-KV work partition, computed on the device from seq_lens.
//
// The flattened work list orders sequences b, then the units of b (a unit is
// one KV head, or one chunk of the query heads that share it), then the
// visible 64-token blocks of b.  Only blocks that hold at least one visible
// key are listed, so blocks wholly outside a sliding window are never read
// (attention-head article, §3: the kernel must skip masked positions).
// Only P' = min(P, W) CTAs take work, so every working CTA has a non-empty
// range: CTA i < P' takes the contiguous block range
// [floor(i*W/P'), floor((i+1)*W/P')); CTAs i >= P' have nothing to do.
// A (unit, CTA) pair that meets writes one partial result; pair slots are
// numbered unit + CTA, which is injective along the walk, so U + P slots
// always suffice.
#pragma once

#include "common.cuh"

namespace attn {

// Which cached keys a query sees, and where the block table keeps them
// (attention-head article, §3: sliding window, and window plus global
// tokens G).  Key j of a sequence with T cached tokens is visible to the
// decode query (position T - 1) when j < T and (no window, or j >= T -
// window, or j < sink, or j is in the sequence's global set G_b, or T - 1 is
// itself in G_b: a global query sees the whole history).  G_b is row b of
// gpos ([B][n_g], positions in ascending order; an entry below the previous
// one, e.g. a -1 pad, ends the row).  With ring > 0 the table row is a ring:
// the blocks holding the sink keys keep slots [0, A) (A = ceil(sink / 64));
// logical block i >= A lives in slot A + i % ring, so a window layer stores
// only the blocks its window can reach.  With ring > 0 and a global set
// (sink 0) the row starts with n_g global slots instead, slot k holding the
// block of G_b[k]: blocks before the window's first block are read through
// the global slot of their first global position, and block i from the
// window's first block on lives in slot n_g + i % ring.  A global query with
// T > window would need history the ring no longer holds and is refused.
struct Visibility {
    int window;   // > 0: sliding window of the last `window` keys
    int sink;     // > 0: the first `sink` keys stay visible (global tokens)
    int ring;     // > 0: ring of this many table slots after the sink blocks
    const int32_t *gpos = nullptr;   // n_g > 0: global positions per sequence
    int n_g = 0;
};

// Global set of sequence b: walks G_b's positions below T in ascending order.
__host__ __device__ __forceinline__ const int32_t *global_row(const Visibility &v, int b) {
    return v.gpos + (size_t)b * v.n_g;
}

// Eight entries of G_b from k0 into c (entries past the row get -1), all
// eight loads issued before any is used, so a scan of the row costs one
// memory round trip per eight entries.
__device__ __forceinline__ void global_chunk(const int32_t *g, int n_g, int k0, int32_t *c) {
#pragma unroll
    for (int j = 0; j < 8; ++j) c[j] = k0 + j < n_g ? g[k0 + j] : -1;
}

// Whether the decode query of a sequence with T keys is a global position.
__device__ __forceinline__ bool global_query(const Visibility &v, int b, int T) {
    if (v.n_g <= 0 || T <= 0) return false;
    const int32_t *g = global_row(v, b);
    int prev = -1;
    bool end = false, found = false;
    for (int k0 = 0; k0 < v.n_g && !end; k0 += 8) {
        int32_t c[8];
        global_chunk(g, v.n_g, k0, c);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            end = end || k0 + j >= v.n_g || c[j] <= prev || c[j] >= T;
            if (!end) {
                found = found || c[j] == T - 1;
                prev = c[j];
            }
        }
    }
    return found;
}

__host__ __device__ __forceinline__ int sink_blocks(const Visibility &v) {
    return v.sink > 0 ? (v.sink + kBlockSize - 1) / kBlockSize : 0;
}

// Slots ahead of the ring: the sink blocks, or one per global position.
__host__ __device__ __forceinline__ int ring_base(const Visibility &v) {
    return v.n_g > 0 ? v.n_g : sink_blocks(v);
}

// Table slot of logical block i (for a global-set ring: of a block from the
// window's first block on; earlier blocks use global_slot).
__host__ __device__ __forceinline__ int table_slot(const Visibility &v, int i) {
    if (v.ring <= 0) return i;
    const int a = ring_base(v);
    return (v.n_g <= 0 && i < a) ? i : a + i % v.ring;
}

// First visible key of the window part (0 without a window).
__host__ __device__ __forceinline__ int window_lo(const Visibility &v, int T) {
    return (v.window > 0 && T > v.window) ? T - v.window : 0;
}

// First key of the contiguous visible run of sequence b: the window's start,
// or 0 when the query itself is global.
__device__ __forceinline__ int seq_window_lo(const Visibility &v, int b, int T) {
    return global_query(v, b, T) ? 0 : window_lo(v, T);
}

// Logical block of the i-th distinct block (ascending) holding a global
// position of sequence b below block w0 (i < the count visible_blocks gave).
__device__ __forceinline__ int global_block(const Visibility &v, int b, int i) {
    const int32_t *g = global_row(v, b);
    int prev = -1, last = -1, n = 0, found = -1;
    bool end = false;
    for (int k0 = 0; k0 < v.n_g && !end; k0 += 8) {
        int32_t c[8];
        global_chunk(g, v.n_g, k0, c);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            end = end || k0 + j >= v.n_g || c[j] <= prev;
            if (!end) {
                prev = c[j];
                const int blk = c[j] / kBlockSize;
                if (blk != last) {
                    if (n == i) {
                        found = blk;
                        end = true;
                    }
                    ++n;
                    last = blk;
                }
            }
        }
    }
    return found >= 0 ? found : last;   // not reached for i < count
}

// Global-set ring layout: table slot of the i-th distinct block (ascending)
// holding a global position of sequence b, i.e. the index of the first
// position of G_b in it (0 if there is none, which callers never ask for).
__device__ __forceinline__ int global_slot(const Visibility &v, int b, int i) {
    const int32_t *g = global_row(v, b);
    int prev = -1, last = -1, n = 0, found = 0;
    bool end = false;
    for (int k0 = 0; k0 < v.n_g && !end; k0 += 8) {
        int32_t c[8];
        global_chunk(g, v.n_g, k0, c);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            end = end || k0 + j >= v.n_g || c[j] <= prev;
            if (!end) {
                prev = c[j];
                const int blk = c[j] / kBlockSize;
                if (blk != last) {
                    if (n == i) {
                        found = k0 + j;
                        end = true;
                    }
                    ++n;
                    last = blk;
                }
            }
        }
    }
    return found;
}

// Bit t set when token blk * 64 + t of sequence b is a global position.
// One warp, all 32 lanes; rows of up to 64 entries.
__device__ __forceinline__ unsigned long long global_mask(const Visibility &v, int b, int blk,
                                                       int lane) {
    const int32_t *g = global_row(v, b);
    const int k0 = lane, k1 = lane + 32;
    const int p0 = k0 < v.n_g ? g[k0] : 0, p1 = k1 < v.n_g ? g[k1] : 0;
    const int q0 = k0 == 0 ? -1 : (k0 < v.n_g ? g[k0 - 1] : 0);
    const int q1 = k1 < v.n_g ? g[k1 - 1] : 0;
    // The row ends at its first entry that does not exceed the one before.
    const unsigned e0 = __ballot_sync(0xffffffffu, k0 >= v.n_g || p0 <= q0);
    const unsigned e1 = __ballot_sync(0xffffffffu, k1 >= v.n_g || p1 <= q1);
    const int end = e0 ? __ffs(e0) - 1 : (e1 ? 32 + __ffs(e1) - 1 : 64);
    unsigned lo = 0u, hi = 0u;
    const int t0 = p0 - blk * kBlockSize, t1 = p1 - blk * kBlockSize;
    if (k0 < end && t0 >= 0 && t0 < kBlockSize) (t0 < 32 ? lo : hi) |= 1u << (t0 & 31);
    if (k1 < end && t1 >= 0 && t1 < kBlockSize) (t1 < 32 ? lo : hi) |= 1u << (t1 & 31);
    lo = __reduce_or_sync(0xffffffffu, lo);
    hi = __reduce_or_sync(0xffffffffu, hi);
    return ((unsigned long long)hi << 32) | lo;
}

// visible_blocks with a global set: the distinct blocks of global
// positions before the window, then the window run.
__device__ __forceinline__ int visible_blocks_global(int T, const Visibility &v, int b, int w1,
                                                   int *first_block, int *sink_blks) {
    const int w0 = seq_window_lo(v, b, T) / kBlockSize;
    if (w0 == 0) return w1;                               // one run [0, w1)
    const int32_t *g = global_row(v, b);
    int prev = -1, last = -1, n = 0;
    bool end = false;
    for (int k0 = 0; k0 < v.n_g && !end; k0 += 8) {
        int32_t c[8];
        global_chunk(g, v.n_g, k0, c);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            end = end || k0 + j >= v.n_g || c[j] <= prev || c[j] / kBlockSize >= w0;
            if (!end) {
                prev = c[j];
                if (c[j] / kBlockSize != last) {
                    ++n;
                    last = c[j] / kBlockSize;
                }
            }
        }
    }
    *sink_blks = n;
    *first_block = w0;
    return n + (w1 - w0);
}

// global_mask computed by one thread.
__device__ __forceinline__ unsigned long long global_mask_thread(const Visibility &v, int b,
                                                                 int blk) {
    const int32_t *g = global_row(v, b);
    unsigned long long m = 0ull;
    int prev = -1;
    for (int k0 = 0; k0 < v.n_g; k0 += 8) {
        int32_t c[8];
        global_chunk(g, v.n_g, k0, c);
        bool end = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int p = c[j];
            end = end || k0 + j >= v.n_g || p <= prev || p - blk * kBlockSize >= kBlockSize;
            if (!end) {
                prev = p;
                const int t = p - blk * kBlockSize;
                if (t >= 0) m |= 1ull << t;
            }
        }
        if (end) break;
    }
    return m;
}

// Visible blocks of sequence b with T cached tokens (current one included):
// blocks holding at least one visible key, in order.  They are *sink_blks
// blocks before the window (the sink blocks [0, A), or the distinct blocks
// of global positions) followed by a run starting at logical block
// *first_block; visible block v is logical block first_block + v -
// sink_blks for v >= sink_blks, else v (sink) or global_block(v) (set G).
// G = false compiles out the explicit-global-set code (callers that never
// see a set: it must not bloat their per-tile loops).
template <bool G = true>
__device__ __forceinline__ int visible_blocks(int T, const Visibility &v, int max_blocks,
                                              int *first_block, int *sink_blks, bool *bad,
                                              int b = 0) {
    *first_block = 0;
    *sink_blks = 0;
    if (T <= 0) {
        *bad = (T < 0);
        return 0;
    }
    if (v.ring <= 0 && T > max_blocks * kBlockSize) {
        *bad = true;
        return 0;
    }
    *bad = false;
    const int w1 = (T - 1) / kBlockSize + 1;             // one past the last block
    if (G && v.n_g > 0) {
        if (v.ring > 0 && window_lo(v, T) > 0 && global_query(v, b, T)) {
            *bad = true;                                  // history left the ring
            return 0;
        }
        return visible_blocks_global(T, v, b, w1, first_block, sink_blks);
    }
    const int w0 = window_lo(v, T) / kBlockSize;        // first window block
    const int a = sink_blocks(v) < w1 ? sink_blocks(v) : w1;
    if (a >= w0) return w1;                               // one run [0, w1)
    *sink_blks = a;
    *first_block = w0;
    return a + (w1 - w0);
}

// Number of CTAs that take work.
__device__ __forceinline__ int working_ctas(long long W, int P) {
    return W < (long long)P ? (int)W : P;
}

__device__ __forceinline__ long long cta_bound(long long i, long long W, int P) {
    return (long long)(((unsigned long long)i * (unsigned long long)W) /
                       (unsigned long long)P);
}

// The CTA whose range contains flattened block x (0 <= x < W).
__device__ __forceinline__ int cta_of(long long x, long long W, int P) {
    long long i = (long long)(((unsigned long long)x * (unsigned long long)P) /
                              (unsigned long long)W);
    while (i + 1 < P && cta_bound(i + 1, W, P) <= x) ++i;
    while (i > 0 && cta_bound(i, W, P) > x) --i;
    return (int)i;
}

struct PlanArgs {
    const int32_t *seq_lens;
    int B;
    int units_per_seq;
    Visibility vis;
    int max_blocks;
    int num_ctas;
};

struct PlanScratch {          // shared memory used by plan_locate
    long long warp_sums[32];
    long long total;
    long long base;
    int seq;
    int bad;
};

// Block-wide: total work W, and the sequence holding flattened block
// `target(W)` together with the work (blocks x units) before that sequence.
// Every thread of the block must call it (blockDim.x >= 32).  When prefix_out is non-null the
// exclusive prefix sums of work per sequence (B + 1 values) are written.
// `target_cta` selects target = cta_bound(target_cta, W, P') (none if the
// CTA has no work).
__device__ __noinline__ static void plan_locate(const PlanArgs &a, int target_cta,
                            PlanScratch *sh, long long *prefix_out,
                            unsigned *err) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = (nt + 31) >> 5;
    if (a.B <= 32) {
        // One warp: lane b holds sequence b; a warp scan gives the prefix
        // sums and W, a ballot the sequence holding the target (one round
        // trip to seq_lens and one block-wide barrier).
        if (warp == 0) {
            long long w = 0;
            bool bad = false;
            if (lane < a.B) {
                int fb, sb;
                w = (long long)visible_blocks(a.seq_lens[lane], a.vis, a.max_blocks, &fb, &sb,
                                              &bad, lane) *
                    a.units_per_seq;
            }
            long long x = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            const long long W = __shfl_sync(0xffffffffu, x, 31);
            const int P = working_ctas(W, a.num_ctas);
            const long long target =
                (W > 0 && target_cta < P) ? cta_bound(target_cta, W, P) : W;
            const long long excl = x - w;
            const unsigned hit =
                __ballot_sync(0xffffffffu, lane < a.B && w > 0 && excl <= target &&
                                               target < excl + w);
            const bool any_bad = __any_sync(0xffffffffu, bad);
            const int src = hit ? __ffs(hit) - 1 : 0;
            const long long base = __shfl_sync(0xffffffffu, excl, src);
            if (prefix_out && lane < a.B) prefix_out[lane] = excl;
            if (lane == 0) {
                sh->total = W;
                sh->seq = hit ? src : -1;
                sh->base = hit ? base : 0;
                sh->bad = any_bad ? 1 : 0;
                if (prefix_out) prefix_out[a.B] = W;
                if (any_bad && err) raise_error(err, kErrBadSeqLen);
            }
        }
        __syncthreads();
        return;
    }
    bool any_bad = false;

    // Pass 1: W.
    long long mine = 0;
    for (int b = tid; b < a.B; b += nt) {
        int fb, sb;
        bool bad;
        mine += (long long)visible_blocks(a.seq_lens[b], a.vis, a.max_blocks, &fb, &sb, &bad, b) *
                a.units_per_seq;
        any_bad |= bad;
    }
    for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
    if (lane == 0) sh->warp_sums[warp] = mine;
    if (tid == 0) { sh->seq = -1; sh->base = 0; sh->bad = 0; }
    __syncthreads();
    if (tid == 0) {
        long long t = 0;
        for (int w = 0; w < nwarps; ++w) t += sh->warp_sums[w];
        sh->total = t;
    }
    if (any_bad) sh->bad = 1;
    __syncthreads();
    const long long W = sh->total;
    const int P = working_ctas(W, a.num_ctas);
    const long long target =
        (W > 0 && target_cta < P) ? cta_bound(target_cta, W, P) : W;

    // Pass 2: exclusive scan, locate target.
    long long running = 0;
    for (int c = 0; c < a.B; c += nt) {
        const int b = c + tid;
        long long w = 0;
        if (b < a.B) {
            int fb, sb;
            bool bad;
            w = (long long)visible_blocks(a.seq_lens[b], a.vis, a.max_blocks, &fb, &sb, &bad, b) *
                a.units_per_seq;
        }
        long long x = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            long long y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        __syncthreads();
        if (lane == 31) sh->warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            long long s = (lane < nwarps) ? sh->warp_sums[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                long long y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            if (lane < nwarps) sh->warp_sums[lane] = s;
        }
        __syncthreads();
        const long long excl =
            running + (warp > 0 ? sh->warp_sums[warp - 1] : 0) + x - w;
        if (b < a.B) {
            if (prefix_out) prefix_out[b] = excl;
            if (w > 0 && excl <= target && target < excl + w) {
                sh->seq = b;
                sh->base = excl;
            }
        }
        running += sh->warp_sums[nwarps - 1];
    }
    if (tid == 0 && prefix_out) prefix_out[a.B] = running;
    if (tid == 0 && sh->bad && err) raise_error(err, kErrBadSeqLen);
    __syncthreads();
}

// Walks the segments of one CTA's block range.  A segment is the part of one
// unit's visible blocks that lies in the range.  G: the call may carry an
// explicit global set (G = false compiles that code out).
template <bool G = true>
struct SegmentWalkerT {
    // fixed
    const int32_t *seq_lens;
    Visibility vis;
    int B, units, max_blocks;
    // state
    long long pos, end;
    int b, unit, blk_off, nb, first_blk, sink_blks, T;
    int lo;   // first key of the contiguous visible run (window start, or 0)

    __device__ void load_seq() {
        bool bad;
        T = seq_lens[b];
        nb = visible_blocks<G>(T, vis, max_blocks, &first_blk, &sink_blks, &bad, b);
        lo = (G && vis.n_g > 0) ? seq_window_lo(vis, b, T) : window_lo(vis, T);
    }

    // Logical block of visible block v of the current sequence.
    __device__ int logical(int v) const {
        if (v >= sink_blks) return first_blk + (v - sink_blks);
        return (G && vis.n_g > 0) ? global_block(vis, b, v) : v;
    }

    // Table slot of visible block v of the current sequence.
    __device__ int slot(int v) const {
        if (G && v < sink_blks && vis.n_g > 0 && vis.ring > 0) return global_slot(vis, b, v);
        return table_slot(vis, logical(v));
    }

    __device__ void init(const PlanArgs &a, long long lo, long long hi,
                         int seq, long long base) {
        seq_lens = a.seq_lens; B = a.B; units = a.units_per_seq;
        vis = a.vis; max_blocks = a.max_blocks;
        pos = lo; end = hi; b = seq;
        if (pos < end) {
            load_seq();
            const long long off = lo - base;
            unit = (int)(off / nb);
            blk_off = (int)(off % nb);
        }
    }

    __device__ bool done() const { return pos >= end; }

    // Length in blocks of the current segment.
    __device__ int seg_len() const {
        long long rem = end - pos;
        int left = nb - blk_off;
        return rem < left ? (int)rem : left;
    }

    __device__ void advance(int len) {
        pos += len;
        blk_off += len;
        if (blk_off == nb) {
            blk_off = 0;
            if (++unit == units) {
                unit = 0;
                if (pos < end) {
                    do { ++b; load_seq(); } while (nb == 0 && b + 1 < B);
                }
            }
        }
    }
};
using SegmentWalker = SegmentWalkerT<true>;

}  // namespace attn
