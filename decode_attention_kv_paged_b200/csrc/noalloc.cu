// noalloc.cu -- attn_decode_gqa_noalloc: GQA/MQA/MHA decode attention whose
// split scratch lives in a fixed device array inside this library, so a call
// never allocates device memory.
//
// Who needs it: callers that are not allowed to call cudaMalloc/cudaFree
// once they are running -- for example a serving process that hands all
// device memory to its own pool at start-up (so an allocation from outside
// the pool can fail or fragment it), or a latency-critical host thread that
// cannot afford the implicit device-wide synchronisation cudaFree performs
// when the regular entry point grows its workspace.
//
// The scratch is a file-scope array of ATTN_NOALLOC_SCRATCH_BYTES; every GPU
// that loads this library holds it until the process exits.  Its device
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) by the first call made on the device.
#include <mutex>

#include "attn_decode.h"
#include "gqa_launch.cuh"
#include "host_state.cuh"

namespace attn {

unsigned *internal_error_word();   // api.cu

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];
// Split arrival counters: zero when the library loads, zero after every call.
static __device__ __align__(256) unsigned g_noalloc_cnt[ATTN_NOALLOC_MAX_UNITS];

struct NoAllocDevice {
    bool ready = false;
    void *scratch = nullptr;   // device address of g_noalloc_scratch
    unsigned *cnt = nullptr;   // device address of g_noalloc_cnt
    int num_sms = 0;
};

// One record per device ordinal (fixed array: a pointer to a record stays
// valid while other threads set up other devices).
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kMaxDevices];

// First call on a device: resolve the scratch array's device address (the
// name is only a host-side stand-in) and the SM count.  No allocation.
int noalloc_setup(NoAllocDevice **out) {
    const int dev = current_device();
    if (dev < 0) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocDevice &d = g_noalloc_dev[dev];
    if (!d.ready) {
        void *ptr = nullptr, *cptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return ATTN_ERR_CUDA;
        if (cudaGetSymbolAddress(&cptr, g_noalloc_cnt) != cudaSuccess || !cptr)
            return ATTN_ERR_CUDA;
        d.cnt = static_cast<unsigned *>(cptr);
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ATTN_ERR_CUDA;
        d.scratch = ptr;
        d.num_sms = sms;
        d.ready = true;
    }
    *out = &d;
    return ATTN_OK;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

int heads_per_cta_noalloc(int G) {
    static const int options[] = {8, 6, 4, 3, 2, 1};
    for (int hc : options)
        if (G % hc == 0) return hc;
    return 1;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" int attn_decode_gqa_noalloc(const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *seq_lens,
                                       const int32_t *block_table, void *out, int B,
                                       int H_q, int H_kv, int d, float scale, int window,
                                       void *stream, int max_blocks_per_seq,
                                       int num_blocks, int dtype) {
    if (!q || !k_cache || !v_cache || !seq_lens || !block_table || !out) return ATTN_ERR_ARG;
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return ATTN_ERR_ARG;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0) return ATTN_ERR_ARG;
    if (dtype != ATTN_F32 && dtype != ATTN_BF16) return ATTN_ERR_ARG;
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return ATTN_ERR_ARG;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_cache) |
                           reinterpret_cast<uintptr_t>(v_cache) | reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis) return ATTN_ERR_ARG;
    if (d != 16 && d != 32 && d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
    if (dtype == ATTN_F32 && d > 128) return ATTN_ERR_UNSUPPORTED;
    if ((long long)max_blocks_per_seq * kBlockSize > (1ll << 30)) return ATTN_ERR_ARG;

    NoAllocDevice *dev;
    int rc = noalloc_setup(&dev);
    if (rc) return rc;
    unsigned *err = internal_error_word();
    if (!err) return ATTN_ERR_CUDA;

    const int G = H_q / H_kv;
    const int HC = heads_per_cta_noalloc(G);
    const int n_hc = G / HC;
    const int P = dev->num_sms;
    const long long units_total = (long long)B * H_kv * n_hc;
    const long long slots = units_total + P;
    const size_t o_bytes = round256((size_t)slots * HC * d * sizeof(float));
    const size_t lse_bytes = round256((size_t)slots * HC * sizeof(float));
    const size_t pre_bytes = round256((size_t)(B + 1) * sizeof(long long));
    if (units_total > ATTN_NOALLOC_MAX_UNITS ||
        o_bytes + lse_bytes + pre_bytes > (size_t)ATTN_NOALLOC_SCRATCH_BYTES)
        return ATTN_ERR_UNSUPPORTED;   // scratch would exceed the fixed array
    unsigned char *ws = static_cast<unsigned char *>(dev->scratch);

    // Nothing in the scratch has to start at zero: every partial, log-sum-exp
    // and prefix value a call reads was written earlier in the same call.
    // The arrival counters are a separate array that each call leaves at
    // zero (an aborted split still arrives).
    GqaLaunch L{};
    GqaParams &kp = L.kp;
    kp.q = q; kp.k_cache = k_cache; kp.v_cache = v_cache;
    kp.seq_lens = seq_lens; kp.block_table = block_table;
    kp.ws_o = reinterpret_cast<float *>(ws);
    kp.ws_lse = reinterpret_cast<float *>(ws + o_bytes);
    kp.ws_prefix = reinterpret_cast<long long *>(ws + o_bytes + lse_bytes);
    kp.err = err;
    kp.out = out;
    kp.ws_cnt = dev->cnt;
    kp.force_timeout = 0;
    kp.timeout_ns = kDefaultTimeoutNs;
    kp.scale_log2 = scale * 1.4426950408889634f;
    kp.B = B; kp.H_q = H_q; kp.H_kv = H_kv; kp.group = G; kp.n_hc = n_hc;
    kp.max_blocks = max_blocks_per_seq; kp.num_blocks = num_blocks;
    kp.vis = Visibility{window > 0 ? window : 0, 0, 0};
    kp.num_ctas = P;
    CombineParams &cp = L.cp;
    cp.seq_lens = seq_lens; cp.ws_prefix = kp.ws_prefix; cp.ws_o = kp.ws_o;
    cp.ws_lse = kp.ws_lse; cp.out = out;
    cp.B = B; cp.H_q = H_q; cp.H_kv = H_kv; cp.group = G; cp.n_hc = n_hc;
    cp.max_blocks = max_blocks_per_seq; cp.vis = kp.vis; cp.num_ctas = P;
    cp.copies = 1;
    L.units_total = (int)units_total;
    L.stream = (cudaStream_t)stream;
    L.ev_start = nullptr;
    L.ev_stop = nullptr;

    const int bf16 = dtype == ATTN_BF16;
    cudaError_t e;
    switch (d) {
        case 16: e = launch_gqa_d16(HC, bf16, L); break;
        case 32: e = launch_gqa_d32(HC, bf16, L); break;
        case 64: e = launch_gqa_d64(HC, bf16, L); break;
        case 128: e = launch_gqa_d128(HC, bf16, L); break;
        default: e = launch_gqa_d256(HC, bf16, L); break;
    }
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
