// api.cu -- the C ABI of libattn_decode.so (declared in include/attn_decode.h):
// argument validation, per-device state (split workspace, error word), launch
// configuration, test and profiling hooks.
#include <atomic>
#include <cmath>
#include <cstring>
#include <functional>
#include <mutex>
#include <thread>

#include "attn_decode.h"
#include "gqa_launch.cuh"
#include "gqa_tc.cuh"
#include "host_state.cuh"
#include "kv_append.cuh"
#include "mla_launch.cuh"

namespace attn {

__device__ unsigned g_err_word;   // per-device error word (bits kErr*)

// Split workspace of one stream: calls on different streams may run at the
// same time, so each stream keeps its own partials and arrival counters.
struct StreamWork {
    cudaStream_t stream = nullptr;
    unsigned long long key2 = 0;  // per-thread default stream: the calling thread
    bool used = false;
    unsigned long long last_use = 0;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    unsigned *cnt = nullptr;      // split arrival counters (zero between launches)
    size_t cnt_elems = 0;
};

// Streams per device with a workspace of their own; the least recently used
// one gives up its workspace to a new stream (freed with cudaFree, which
// waits for the work still using it).
constexpr int kMaxStreams = 16;

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    unsigned *err = nullptr;      // device address of g_err_word
    unsigned long long tick = 0;
    StreamWork work[kMaxStreams];
};

// One record per device ordinal; a pointer to a record stays valid for the
// life of the process.
static std::mutex g_mu;
static DeviceState g_dev[kMaxDevices];
static thread_local int tl_num_ctas = 0;
static thread_local int tl_gqa_path = -1;
static std::atomic<int> g_force_timeout{0};
static std::atomic<long long> g_force_timeout_ns{0};
static const void *const *g_prof_start = nullptr;
static const void *const *g_prof_stop = nullptr;
static int g_prof_n = 0, g_prof_i = 0;

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA; }

// Per-device state of the current device (created on first use).
static int device_state(DeviceState **out) {
    const int dev = current_device();
    if (dev < 0) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState &st = g_dev[dev];
    if (!st.ready) {
        if (cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess)
            return ATTN_ERR_CUDA;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&st.err), g_err_word) !=
            cudaSuccess)
            return ATTN_ERR_CUDA;
        st.ready = true;
    }
    *out = &st;
    return ATTN_OK;
}

// The workspace record of `stream` on this device (taken over from the least
// recently used stream when all records are in use).  The per-thread default
// stream is one handle for many streams, so it is keyed by the calling thread
// as well.  Caller holds g_mu.
static StreamWork *stream_work_locked(DeviceState *st, cudaStream_t stream) {
    const unsigned long long key2 =
        stream == cudaStreamPerThread
            ? (unsigned long long)std::hash<std::thread::id>()(std::this_thread::get_id())
            : 0ull;
    StreamWork *victim = nullptr;
    for (StreamWork &w : st->work) {
        if (w.used && w.stream == stream && w.key2 == key2) {
            w.last_use = ++st->tick;
            return &w;
        }
        if (!victim || (!w.used && victim->used) ||
            (w.used == victim->used && w.last_use < victim->last_use))
            victim = &w;
    }
    if (victim->used) {
        // cudaFree waits for all work on the device, the old stream's included.
        if (victim->ws) cudaFree(victim->ws);
        if (victim->cnt) cudaFree(victim->cnt);
        *victim = StreamWork{};
    }
    victim->used = true;
    victim->stream = stream;
    victim->key2 = key2;
    victim->last_use = ++st->tick;
    return victim;
}

// Grow `stream`'s split workspace to at least `bytes`; returns it in *ws.
// Never during stream capture (a graph must not depend on an allocation made
// inside it).
static int ensure_workspace(DeviceState *st, size_t bytes, cudaStream_t stream, void **ws) {
    std::lock_guard<std::mutex> lk(g_mu);
    StreamWork *w = stream_work_locked(st, stream);
    if (w->ws_bytes < bytes) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return ATTN_ERR_UNSUPPORTED;
        size_t want = bytes < 2 * w->ws_bytes ? 2 * w->ws_bytes : bytes;
        want = (want + (1u << 20) - 1) & ~(size_t)((1u << 20) - 1);
        if (w->ws) {
            cudaFree(w->ws);   // implicitly waits for work that may still use it
            w->ws = nullptr;
            w->ws_bytes = 0;
        }
        if (cudaMalloc(&w->ws, want) != cudaSuccess) return ATTN_ERR_CUDA;
        w->ws_bytes = want;
    }
    *ws = w->ws;
    return ATTN_OK;
}

// Grow `stream`'s split arrival counters to at least `n` (zeroed when
// allocated; every launch leaves them at zero).  Never during capture.
static int ensure_counters(DeviceState *st, size_t n, cudaStream_t stream, unsigned **cnt) {
    std::lock_guard<std::mutex> lk(g_mu);
    StreamWork *w = stream_work_locked(st, stream);
    if (w->cnt_elems < n) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return ATTN_ERR_UNSUPPORTED;
        size_t want = n < 2 * w->cnt_elems ? 2 * w->cnt_elems : n;
        want = (want + 4095) & ~(size_t)4095;
        if (w->cnt) {
            cudaFree(w->cnt);
            w->cnt = nullptr;
            w->cnt_elems = 0;
        }
        if (cudaMalloc(&w->cnt, want * sizeof(unsigned)) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaMemset(w->cnt, 0, want * sizeof(unsigned)) != cudaSuccess) return ATTN_ERR_CUDA;
        w->cnt_elems = want;
    }
    *cnt = w->cnt;
    return ATTN_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static bool aligned16(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

static bool valid_head_dim(int d) {
    return d == 16 || d == 32 || d == 64 || d == 128 || d == 256;
}

// Whether attn_decode_gqa runs the tensor-core kernel for this problem: by
// default for groups of kTcMinGroup heads or more (there every K/V element
// feeds enough heads to make the products dense), or when forced.
static bool use_tc_path(int G, int d, int dtype) {
    const bool ok = gqa_tc_supported(d, dtype == ATTN_BF16, G);
    if (tl_gqa_path == 0) return false;
    if (tl_gqa_path >= 1) return ok;
    return ok && G >= kTcMinGroup;
}

// Which tensor-core kernel runs a unit of HC heads: the M = 128 one (Q and P
// in tensor memory) where it applies, else the M = 64 one; the testing hook
// path 2 forces the M = 64 kernel.  Measured on B200 (T = 32768, B = 8) the
// M = 128 kernel is ahead or level everywhere it applies: MQA 41.0 vs
// 49.1 us, G = 24 60.3 vs 83.9 us, G = 8 96.2 vs 98.3 us, G = 16 59.6 vs
// 58.3 us.
static bool use_tc128(int d, int HC) {
    return tl_gqa_path != 2 && gqa_tc128_supported(d, HC);
}

// Whether an fp8 call runs the M = 128 tensor-core kernel (codes widened to
// f16 on the chip) rather than the CUDA-core kernel: by default for groups of
// kTcFp8MinGroup heads or more, where the CUDA-core kernel splits the group
// into 8-head chunks and reads every tile once per chunk (measured on B200,
// T = 32768: MQA at B = 8 168 us on CUDA cores vs 68 us on tensor cores, at
// B = 1 41 vs 29 us; G = 4 at B = 8 207 vs 318 us, MHA 633 vs 1223 us);
// path 1 forces it wherever it applies, path 0 forces the CUDA cores (and
// path 2, the M = 64 kernel, has no fp8 form).
constexpr int kTcFp8MinGroup = 16;
static bool use_tc_fp8(int G, int d) {
    if (tl_gqa_path == 0 || tl_gqa_path == 2) return false;
    if (!gqa_tc128_fp8_supported(d, G)) return false;
    return tl_gqa_path == 1 || G >= kTcFp8MinGroup;
}

// Query heads per CTA for a group of G: the largest instantiated divisor.
static int heads_per_cta(int G) {
    static const int options[] = {8, 6, 4, 3, 2, 1};
    for (int hc : options)
        if (G % hc == 0) return hc;
    return 1;
}

static void take_profile_events(cudaEvent_t *start, cudaEvent_t *stop) {
    std::lock_guard<std::mutex> lk(g_mu);
    *start = nullptr;
    *stop = nullptr;
    if (g_prof_n > 0 && g_prof_i < g_prof_n) {
        *start = (cudaEvent_t)g_prof_start[g_prof_i];
        *stop = (cudaEvent_t)g_prof_stop[g_prof_i];
        ++g_prof_i;
    }
}

static void take_force_timeout(int *flag, unsigned long long *ns) {
    *flag = g_force_timeout.exchange(0);
    long long t = g_force_timeout_ns.load();
    *ns = (*flag && t > 0) ? (unsigned long long)t : kDefaultTimeoutNs;
}

// Device address of the current device's error word, for entry points
// defined in other translation units (null on failure).
unsigned *internal_error_word() {
    DeviceState *st;
    return device_state(&st) == ATTN_OK ? st->err : nullptr;
}


}  // namespace attn

using namespace attn;

extern "C" {

int attn_version(void) { return 100; }

const char *attn_status_string(int s) {
    switch (s) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_ARG: return "ATTN_ERR_ARG";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
        case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
        case ATTN_ERR_BAD_BLOCK: return "ATTN_ERR_BAD_BLOCK";
        case ATTN_ERR_BAD_SEQLEN: return "ATTN_ERR_BAD_SEQLEN";
        default: return "ATTN_UNKNOWN_STATUS";
    }
}

int attn_set_num_ctas(int n) {
    if (n < 0 || n > 65535) return ATTN_ERR_ARG;
    tl_num_ctas = n;
    return ATTN_OK;
}

int attn_set_gqa_path(int path) {
    if (path < -1 || path > 2) return ATTN_ERR_ARG;
    tl_gqa_path = path;
    return ATTN_OK;
}

int attn_set_profile_events(void *const *start_events, void *const *stop_events,
                            int n) {
    if (n < 0 || (n > 0 && (!start_events || !stop_events))) return ATTN_ERR_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_prof_start = start_events;
    g_prof_stop = stop_events;
    g_prof_n = n;
    g_prof_i = 0;
    return ATTN_OK;
}

int attn_debug_force_timeout(int enable, long long timeout_ns) {
    if (timeout_ns < 0) return ATTN_ERR_ARG;
    g_force_timeout_ns.store(timeout_ns);
    g_force_timeout.store(enable ? 1 : 0);
    return ATTN_OK;
}

int attn_decode_last_error(void *stream) {
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return ATTN_ERR_CUDA;
    unsigned word = 0, zero = 0;
    if (cudaMemcpy(&word, st->err, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (word && cudaMemcpy(st->err, &zero, sizeof zero, cudaMemcpyHostToDevice) !=
                    cudaSuccess)
        return ATTN_ERR_CUDA;
    if (word & kErrTimeout) return ATTN_ERR_TIMEOUT;
    if (word & kErrBadBlock) return ATTN_ERR_BAD_BLOCK;
    if (word & kErrBadSeqLen) return ATTN_ERR_BAD_SEQLEN;
    return ATTN_OK;
}

int attn_decode_gqa_config(int B, int H_q, int H_kv, int d, int dtype, int *num_ctas,
                           int *heads, int *path) {
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv || !valid_head_dim(d) ||
        (dtype != ATTN_F32 && dtype != ATTN_BF16 && dtype != ATTN_FP8_E4M3))
        return ATTN_ERR_ARG;
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    const int G = H_q / H_kv;
    if (num_ctas) *num_ctas = tl_num_ctas > 0 ? tl_num_ctas : st->num_sms;
    if (dtype == ATTN_FP8_E4M3) {
        const bool tc8 = use_tc_fp8(G, d);
        if (heads) *heads = tc8 ? gqa_tc128_fp8_heads_per_cta(G) : heads_per_cta(G);
        if (path) *path = tc8 ? 1 : 0;
        return ATTN_OK;
    }
    const bool tc = use_tc_path(G, d, dtype);
    const int hc = tc ? gqa_tc_heads_per_cta(G) : heads_per_cta(G);
    if (heads) *heads = hc;
    if (path) *path = tc ? (use_tc128(d, hc) ? 1 : 2) : 0;
    return ATTN_OK;
}

// Shared body of attn_decode_gqa and attn_decode_gqa_ext.
// dtype: ATTN_F32 / ATTN_BF16 for q, cache and out alike, or kFp8Cache: bf16
// q and out over an e4m3 cache with per-row scales (k_scale, v_scale).
constexpr int kFp8Cache = 100;

static int decode_gqa_impl(const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *seq_lens, const int32_t *block_table, void *out,
                           int B, int H_q, int H_kv, int d, float scale, Visibility vis,
                           void *stream, int max_blocks_per_seq, int num_blocks, int dtype,
                           const float *k_scale = nullptr, const float *v_scale = nullptr) {
    if (!q || !k_cache || !v_cache || !seq_lens || !block_table || !out) return ATTN_ERR_ARG;
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return ATTN_ERR_ARG;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0) return ATTN_ERR_ARG;
    const bool fp8 = dtype == kFp8Cache;
    if (dtype != ATTN_F32 && dtype != ATTN_BF16 && !fp8) return ATTN_ERR_ARG;
    if (fp8 && (!k_scale || !v_scale || !aligned16(k_scale) || !aligned16(v_scale)))
        return ATTN_ERR_ARG;
    if (fp8 && d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return ATTN_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return ATTN_ERR_ARG;
    if (!valid_head_dim(d)) return ATTN_ERR_UNSUPPORTED;
    if (dtype == ATTN_F32 && d > 128) return ATTN_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * kBlockSize > (1ll << 30)) return ATTN_ERR_ARG;

    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    cudaStream_t s = (cudaStream_t)stream;

    const int G = H_q / H_kv;
    const bool tc8 = fp8 && use_tc_fp8(G, d);
    const bool tc = tc8 || (!fp8 && use_tc_path(G, d, dtype));
    const int HC = tc8 ? gqa_tc128_fp8_heads_per_cta(G)
                       : (tc ? gqa_tc_heads_per_cta(G) : heads_per_cta(G));
    const int n_hc = G / HC;
    const long long units_total = (long long)B * H_kv * n_hc;
    // No more CTAs than the work could possibly fill (units x table width).
    const long long work_bound = units_total * max_blocks_per_seq;
    const int P = tl_num_ctas > 0 ? tl_num_ctas
                                  : (int)(work_bound < st->num_sms ? work_bound : st->num_sms);
    if (units_total > (1ll << 30)) return ATTN_ERR_ARG;
    const long long slots = units_total + P;

    // The tensor-core kernels write one partial per head-group copy per slot.
    const bool tc128 = tc8 || (tc && use_tc128(d, HC));
    const int copies = tc ? (tc128 ? gqa_tc128_copies(HC) : gqa_tc_copies(HC)) : 1;
    const size_t o_bytes = align256((size_t)slots * copies * HC * d * sizeof(float));
    const size_t lse_bytes = align256((size_t)slots * copies * HC * sizeof(float));
    const size_t pre_bytes = align256((size_t)(B + 1) * sizeof(long long));
    void *ws_raw = nullptr;
    rc = ensure_workspace(st, o_bytes + lse_bytes + pre_bytes, s, &ws_raw);
    if (rc) return rc;
    unsigned char *ws = static_cast<unsigned char *>(ws_raw);

    GqaLaunch L{};
    GqaParams &kp = L.kp;
    kp.q = q; kp.k_cache = k_cache; kp.v_cache = v_cache;
    kp.seq_lens = seq_lens; kp.block_table = block_table;
    kp.ws_o = reinterpret_cast<float *>(ws);
    kp.ws_lse = reinterpret_cast<float *>(ws + o_bytes);
    kp.ws_prefix = reinterpret_cast<long long *>(ws + o_bytes + lse_bytes);
    kp.err = st->err;
    kp.out = out;
    kp.k_scale = k_scale;
    kp.v_scale = v_scale;
    if (!tc) {
        rc = ensure_counters(st, (size_t)units_total, s, &kp.ws_cnt);
        if (rc) return rc;
    }
    take_force_timeout(&kp.force_timeout, &kp.timeout_ns);
    kp.scale_log2 = scale * 1.4426950408889634f;
    kp.B = B; kp.H_q = H_q; kp.H_kv = H_kv; kp.group = G; kp.n_hc = n_hc;
    kp.max_blocks = max_blocks_per_seq; kp.num_blocks = num_blocks;
    kp.vis = vis;
    kp.num_ctas = P;
    CombineParams &cp = L.cp;
    cp.seq_lens = seq_lens; cp.ws_prefix = kp.ws_prefix; cp.ws_o = kp.ws_o;
    cp.ws_lse = kp.ws_lse; cp.out = out;
    cp.B = B; cp.H_q = H_q; cp.H_kv = H_kv; cp.group = G; cp.n_hc = n_hc;
    cp.max_blocks = max_blocks_per_seq; cp.vis = vis; cp.num_ctas = P;
    cp.copies = copies;
    L.units_total = (int)units_total;
    L.stream = s;
    take_profile_events(&L.ev_start, &L.ev_stop);

    const int bf16 = dtype == ATTN_BF16;
    cudaError_t e;
    if (tc) {
        e = tc8 ? launch_gqa_tc128_fp8(L, d, HC)
                : (tc128 ? launch_gqa_tc128(L, d, HC) : launch_gqa_tc(L, d, HC));
        return cuda_status(e);
    }
    if (fp8) {
        switch (d) {
            case 64: e = launch_gqa_fp8_d64(HC, L); break;
            case 128: e = launch_gqa_fp8_d128(HC, L); break;
            default: e = launch_gqa_fp8_d256(HC, L); break;
        }
        return cuda_status(e);
    }
    switch (d) {
        case 16: e = launch_gqa_d16(HC, bf16, L); break;
        case 32: e = launch_gqa_d32(HC, bf16, L); break;
        case 64: e = launch_gqa_d64(HC, bf16, L); break;
        case 128: e = launch_gqa_d128(HC, bf16, L); break;
        default: e = launch_gqa_d256(HC, bf16, L); break;
    }
    return cuda_status(e);
}

int attn_decode_gqa(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seq_lens, const int32_t *block_table, void *out,
                    int B, int H_q, int H_kv, int d, float scale, int window,
                    void *stream, int max_blocks_per_seq, int num_blocks, int dtype) {
    return decode_gqa_impl(q, k_cache, v_cache, seq_lens, block_table, out, B, H_q, H_kv, d,
                           scale, Visibility{window > 0 ? window : 0, 0, 0}, stream,
                           max_blocks_per_seq, num_blocks, dtype);
}

// Validates a visibility record against the table width; fills `out`.
static int check_visibility(const attn_visibility *v, int max_blocks_per_seq, Visibility *out) {
    if (!v) return ATTN_ERR_ARG;
    if (v->sink_tokens < 0 || v->ring_blocks < 0 || v->n_global < 0) return ATTN_ERR_ARG;
    Visibility vis{v->window > 0 ? v->window : 0, v->sink_tokens, v->ring_blocks};
    if (v->n_global > 0) {
        // An explicit global set replaces the sink prefix; with a ring its
        // positions' blocks keep the n_global slots ahead of the ring.
        if (!v->global_pos || (reinterpret_cast<uintptr_t>(v->global_pos) & 3u) ||
            v->sink_tokens > 0)
            return ATTN_ERR_ARG;
        if (v->n_global > 64) return ATTN_ERR_UNSUPPORTED;
        vis.gpos = v->global_pos;
        vis.n_g = v->n_global;
    }
    if (vis.ring > 0) {
        // The ring must hold every block a window can reach, after the sink
        // blocks (or the global slots), inside the table row.
        if (vis.window <= 0) return ATTN_ERR_ARG;
        if ((long long)vis.ring * kBlockSize < (long long)vis.window + kBlockSize - 1)
            return ATTN_ERR_ARG;
        if ((long long)ring_base(vis) + vis.ring > max_blocks_per_seq) return ATTN_ERR_ARG;
    }
    *out = vis;
    return ATTN_OK;
}

int attn_decode_gqa_ext(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *seq_lens, const int32_t *block_table, void *out,
                        int B, int H_q, int H_kv, int d, float scale,
                        const attn_visibility *visibility, void *stream,
                        int max_blocks_per_seq, int num_blocks, int dtype) {
    Visibility vis;
    const int rc = check_visibility(visibility, max_blocks_per_seq, &vis);
    if (rc) return rc;
    return decode_gqa_impl(q, k_cache, v_cache, seq_lens, block_table, out, B, H_q, H_kv, d,
                           scale, vis, stream, max_blocks_per_seq, num_blocks, dtype);
}

int attn_decode_gqa_fp8(const void *q, const void *k_cache, const void *v_cache,
                        const float *k_scale, const float *v_scale, const int32_t *seq_lens,
                        const int32_t *block_table, void *out, int B, int H_q, int H_kv, int d,
                        float scale, const attn_visibility *visibility, void *stream,
                        int max_blocks_per_seq, int num_blocks) {
    Visibility vis{0, 0, 0};
    if (visibility) {
        const int rc = check_visibility(visibility, max_blocks_per_seq, &vis);
        if (rc) return rc;
    }
    return decode_gqa_impl(q, k_cache, v_cache, seq_lens, block_table, out, B, H_q, H_kv, d,
                           scale, vis, stream, max_blocks_per_seq, num_blocks, kFp8Cache,
                           k_scale, v_scale);
}

int kv_append_fp8(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  float *k_scale, float *v_scale, const int32_t *positions,
                  const int32_t *block_table, int B, int H_kv, int d, int max_blocks_per_seq,
                  int num_blocks, const attn_visibility *visibility, void *stream) {
    if (!k_new || !v_new || !k_cache || !v_cache || !k_scale || !v_scale || !positions ||
        !block_table)
        return ATTN_ERR_ARG;
    if (B <= 0 || H_kv <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0) return ATTN_ERR_ARG;
    if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
    Visibility vis{0, 0, 0};
    if (visibility) {
        const int rc = check_visibility(visibility, max_blocks_per_seq, &vis);
        if (rc) return rc;
    }
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    KvAppendFp8Params p{};
    p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    p.k_cache = static_cast<uint8_t *>(k_cache);
    p.v_cache = static_cast<uint8_t *>(v_cache);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.positions = positions;
    p.block_table = block_table;
    p.err = st->err;
    p.B = B; p.H_kv = H_kv; p.d = d;
    p.max_blocks = max_blocks_per_seq; p.num_blocks = num_blocks;
    p.vis = vis;
    return cuda_status(launch_kv_append_fp8(p, (cudaStream_t)stream));
}

// Shared body of attn_decode_mla (latent_scale null: bf16 cache) and
// attn_decode_mla_fp8 (E4M3 codes with per-row scales).
static int decode_mla_impl(const void *q_latent, const void *q_rope, const void *latent_cache,
                           const float *latent_scale, const int32_t *seq_lens,
                           const int32_t *block_table, void *out, int B, int H, int d_c, int d_r,
                           float scale, void *stream, int max_blocks_per_seq, int num_blocks) {
    if (!q_latent || !q_rope || !latent_cache || !seq_lens || !block_table || !out)
        return ATTN_ERR_ARG;
    if (B <= 0 || H <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0) return ATTN_ERR_ARG;
    if (!std::isfinite(scale)) return ATTN_ERR_ARG;
    if (!aligned16(q_latent) || !aligned16(q_rope) || !aligned16(latent_cache) ||
        !aligned16(out))
        return ATTN_ERR_ARG;
    if (d_c != 512 || d_r != 64) return ATTN_ERR_UNSUPPORTED;
    if (H != 128) return ATTN_ERR_UNSUPPORTED;
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    cudaEvent_t ev_start, ev_stop;
    take_profile_events(&ev_start, &ev_stop);
    return mla_decode_entry(q_latent, q_rope, latent_cache, latent_scale, seq_lens, block_table,
                            out, B, H, scale, (cudaStream_t)stream, max_blocks_per_seq,
                            num_blocks, st->num_sms, tl_num_ctas, st->err,
                            [&](size_t bytes, void **ws) {
                                return ensure_workspace(st, bytes, (cudaStream_t)stream, ws);
                            },
                            ev_start, ev_stop);
}

int attn_decode_mla(const void *q_latent, const void *q_rope, const void *latent_cache,
                    const int32_t *seq_lens, const int32_t *block_table, void *out, int B,
                    int H, int d_c, int d_r, float scale, void *stream,
                    int max_blocks_per_seq, int num_blocks) {
    return decode_mla_impl(q_latent, q_rope, latent_cache, nullptr, seq_lens, block_table, out,
                           B, H, d_c, d_r, scale, stream, max_blocks_per_seq, num_blocks);
}

int attn_decode_mla_fp8(const void *q_latent, const void *q_rope, const void *latent_codes,
                        const float *latent_scale, const int32_t *seq_lens,
                        const int32_t *block_table, void *out, int B, int H, int d_c, int d_r,
                        float scale, void *stream, int max_blocks_per_seq, int num_blocks) {
    if (!latent_scale || !aligned16(latent_scale)) return ATTN_ERR_ARG;
    return decode_mla_impl(q_latent, q_rope, latent_codes, latent_scale, seq_lens, block_table,
                           out, B, H, d_c, d_r, scale, stream, max_blocks_per_seq, num_blocks);
}

int kv_append_mla_fp8(const void *latent_new, void *latent_codes, float *latent_scale,
                      const int32_t *positions, const int32_t *block_table, int B, int d_c,
                      int d_r, int max_blocks_per_seq, int num_blocks, void *stream) {
    if (!latent_new || !latent_codes || !latent_scale || !positions || !block_table)
        return ATTN_ERR_ARG;
    if (B <= 0 || d_c <= 0 || d_r < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
        return ATTN_ERR_ARG;
    if ((d_c + d_r) % 2 || !aligned16(latent_new) || !aligned16(latent_codes))
        return ATTN_ERR_ARG;
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    KvAppendFp8Params p{};
    p.k_new = static_cast<const __nv_bfloat16 *>(latent_new);
    p.v_new = nullptr;                 // one latent row per token, no separate V
    p.k_cache = static_cast<uint8_t *>(latent_codes);
    p.v_cache = nullptr;
    p.k_scale = latent_scale;
    p.v_scale = nullptr;
    p.positions = positions;
    p.block_table = block_table;
    p.err = st->err;
    p.B = B; p.H_kv = 1; p.d = d_c + d_r;
    p.max_blocks = max_blocks_per_seq; p.num_blocks = num_blocks;
    p.vis = Visibility{0, 0, 0};
    return cuda_status(launch_kv_append_fp8(p, (cudaStream_t)stream));
}

static int kv_append_impl(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                          const int32_t *positions, const int32_t *block_table, int B,
                          int H_kv, int d, int max_blocks_per_seq, int num_blocks, int dtype,
                          Visibility vis, void *stream) {
    if (!k_new || !v_new || !k_cache || !v_cache || !positions || !block_table)
        return ATTN_ERR_ARG;
    if (B <= 0 || H_kv <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0) return ATTN_ERR_ARG;
    if (dtype != ATTN_F32 && dtype != ATTN_BF16) return ATTN_ERR_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return ATTN_ERR_ARG;
    if (!valid_head_dim(d)) return ATTN_ERR_UNSUPPORTED;
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    KvAppendParams p{};
    p.k_new = k_new; p.v_new = v_new; p.k_cache = k_cache; p.v_cache = v_cache;
    p.positions = positions; p.block_table = block_table; p.err = st->err;
    p.B = B; p.H_kv = H_kv;
    p.chunks_per_row = d * (dtype == ATTN_BF16 ? 2 : 4) / 16;
    p.max_blocks = max_blocks_per_seq; p.num_blocks = num_blocks;
    p.vis = vis;
    return cuda_status(launch_kv_append(p, (cudaStream_t)stream));
}

int kv_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
              const int32_t *positions, const int32_t *block_table, int B, int H_kv, int d,
              int max_blocks_per_seq, int num_blocks, int dtype, void *stream) {
    return kv_append_impl(k_new, v_new, k_cache, v_cache, positions, block_table, B, H_kv, d,
                          max_blocks_per_seq, num_blocks, dtype, Visibility{0, 0, 0}, stream);
}

int kv_append_ext(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  const int32_t *positions, const int32_t *block_table, int B, int H_kv, int d,
                  int max_blocks_per_seq, int num_blocks, int dtype,
                  const attn_visibility *visibility, void *stream) {
    Visibility vis;
    const int rc = check_visibility(visibility, max_blocks_per_seq, &vis);
    if (rc) return rc;
    return kv_append_impl(k_new, v_new, k_cache, v_cache, positions, block_table, B, H_kv, d,
                          max_blocks_per_seq, num_blocks, dtype, vis, stream);
}

int kv_append_mla(const void *latent_new, void *latent_cache, const int32_t *positions,
                  const int32_t *block_table, int B, int d_c, int d_r,
                  int max_blocks_per_seq, int num_blocks, void *stream) {
    if (!latent_new || !latent_cache || !positions || !block_table) return ATTN_ERR_ARG;
    if (B <= 0 || d_c <= 0 || d_r < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
        return ATTN_ERR_ARG;
    if (((d_c + d_r) * 2) % 16 != 0) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(latent_new) || !aligned16(latent_cache)) return ATTN_ERR_ARG;
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    KvAppendParams p{};
    p.k_new = latent_new; p.v_new = nullptr; p.k_cache = latent_cache; p.v_cache = nullptr;
    p.positions = positions; p.block_table = block_table; p.err = st->err;
    p.B = B; p.H_kv = 1; p.chunks_per_row = (d_c + d_r) * 2 / 16;
    p.max_blocks = max_blocks_per_seq; p.num_blocks = num_blocks;
    return cuda_status(launch_kv_append(p, (cudaStream_t)stream));
}

int attn_decode_plan(const int32_t *seq_lens, int B, int units_per_seq, int window,
                     int max_blocks_per_seq, int num_ctas, int64_t *plan_out,
                     void *stream) {
    if (!seq_lens || !plan_out || B <= 0 || units_per_seq <= 0 || num_ctas <= 0 ||
        max_blocks_per_seq <= 0)
        return ATTN_ERR_ARG;
    DeviceState *st;
    int rc = device_state(&st);
    if (rc) return rc;
    return cuda_status(launch_plan_kernel(seq_lens, B, units_per_seq,
                                          Visibility{window > 0 ? window : 0, 0, 0},
                                          max_blocks_per_seq, num_ctas,
                                          reinterpret_cast<long long *>(plan_out), st->err,
                                          (cudaStream_t)stream));
}

}  // extern "C"
