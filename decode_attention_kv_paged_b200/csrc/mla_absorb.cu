// mla_absorb.cu -- the two per-head products on either side of the absorbed
// MLA decode (attention-head article, §5.2 absorption):
//     q_latent[b,h] = q_c[b,h] (U^K_h)^T     (d_h -> d_c, before the decode)
//     o[b,h]        = z[b,h] U^V_h           (d_c -> d_v, after the decode)
// with U^K_h, U^V_h in R^{d_c x d_h} / R^{d_c x d_v} (k^C_j = c_j U^K_h,
// v_j = c_j U^V_h).
//
// Each is H independent products whose weight (d_c x 128 bf16, 128 KiB per
// head) is shared by all B sequences: every weight element feeds 2B flops,
// so the work is a dense contraction and runs on the tcgen05 tensor cores,
// while its time is set by streaming the weights (H x 128 KiB) from HBM
// once.  Orientation: a CTA computes out_h^T for 128 output features (the
// MMA's M, one TMEM lane per feature) and a tile of the sequences (the MMA's
// N, 32 / 64 / 128 TMEM columns), so the weight is the A operand -- K-major
// for U^K (rows of d_h), MN-major for U^V (rows of d_v) -- and is read
// exactly once; the sequences' vectors are the B operand (K-major rows,
// rows beyond B zero-filled by the TMA).  The contraction runs in 64-wide
// chunks through a ring of shared-memory stages (2-D TMA, 128-byte swizzle);
// one thread issues the MMAs, fp32 accumulation in TMEM, and four warps round
// the products to bf16 in the epilogue (one output feature per thread).
// Every wait is bounded (device error word on timeout); TMEM is always freed.
#include <mutex>

#include "attn_decode.h"
#include "common.cuh"
#include "host_state.cuh"
#include "tc_common.cuh"

namespace attn {

unsigned *internal_error_word();   // api.cu

namespace {

constexpr int kHgThreads = 128;
constexpr int kHgM = 128;          // output features per CTA (MMA M)
constexpr int kHgK = 64;           // contraction chunk per stage (one swizzle row)
constexpr int kHgMaxStages = 8;
constexpr int kHgMaxSmem = 200 * 1024;   // stages are capped to this much shared memory
constexpr int kHgABytes = kHgM * kHgK * 2;   // 16 KiB of weight per stage

struct HeadGemmParams {
    __nv_bfloat16 *out;   // [B][H][M_total]
    unsigned *err;
    unsigned long long timeout_ns;
    int B, H, M_total, K, n_tile, stages;
};

__host__ __device__ constexpr int hg_stage_bytes(int n_tile) { return kHgABytes + n_tile * kHgK * 2; }

// A_MN: the weight is stored [K][M] (U^V_h: rows of d_v), else [M][K] (U^K_h:
// rows of d_h).
template <bool A_MN>
__global__ void __launch_bounds__(kHgThreads, 1)
head_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const HeadGemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[kHgMaxStages], empty[kHgMaxStages], done;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_word;
    volatile int *abort_flag = &abort_word;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * kHgM, h = blockIdx.y, b0 = blockIdx.z * p.n_tile;
    const int nk = p.K / kHgK, S = p.stages;
    const int stage_bytes = hg_stage_bytes(p.n_tile);
    const uint32_t tcols = p.n_tile <= 32 ? 32u : (p.n_tile <= 64 ? 64u : 128u);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        abort_word = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(&tmem_base, tcols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    // Programmatic dependent launch: the set-up above overlaps the previous
    // kernel on the stream; its outputs (this call's inputs) are read only
    // after it has completed.
    pdl_wait_primary();
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            tma_prefetch_map(&tm_a);
            tma_prefetch_map(&tm_b);
            const uint64_t pol_w = l2_policy_evict_first();   // each weight is read once
            const uint64_t pol_x = l2_policy_evict_last();    // the sequences' vectors, by every feature tile
            int kc = 0;
            for (; kc < nk; ++kc) {
                const int st = kc % S;
                if (kc >= S && !mbar_wait(&empty[st], (uint32_t)(((kc / S) - 1) & 1), p.timeout_ns,
                                          p.err, abort_flag))
                    break;
                unsigned char *sa = smem + st * stage_bytes;
                unsigned char *sb = sa + kHgABytes;
                mbar_arrive_expect_tx(&full[st], stage_bytes);
                if (A_MN) {
                    // [64 K rows][64 M columns] boxes: two cover the 128 features.
                    tma_load_2d(sa, &tm_a, m0, h * p.K + kHgK * kc, &full[st], pol_w);
                    tma_load_2d(sa + kHgABytes / 2, &tm_a, m0 + 64, h * p.K + kHgK * kc, &full[st],
                                pol_w);
                } else {
                    tma_load_2d(sa, &tm_a, kHgK * kc, h * p.M_total + m0, &full[st], pol_w);
                }
                tma_load_2d(sb, &tm_b, h * p.K + kHgK * kc, b0, &full[st], pol_x);
            }
            // Every issued load lands before the CTA exits.
            for (int t = kc - S < 0 ? 0 : kc - S; t < kc; ++t)
                mbar_wait(&full[t % S], (uint32_t)((t / S) & 1), p.timeout_ns, p.err, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(kHgM, p.n_tile, A_MN ? 1 : 0, 0);
            const uint32_t base = smem_u32(smem);
            int kc = 0;
            for (; kc < nk; ++kc) {
                const int st = kc % S;
                if (!mbar_wait(&full[st], (uint32_t)((kc / S) & 1), p.timeout_ns, p.err, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t sa = base + st * stage_bytes, sb = sa + kHgABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = A_MN ? umma_desc_sw128(sa + kk * 2048, kHgABytes / 2, 1024)
                                            : umma_desc_sw128(sa + kk * 32, 16, 1024);
                    const uint64_t b = umma_desc_sw128(sb + kk * 32, 16, 1024);
                    umma_bf16(tmem, a, b, idesc, (kc | kk) != 0);
                }
                umma_commit(&empty[st]);
            }
            // `done` completes once every product issued has completed (an
            // aborted issuer still commits, so nobody waits past it).
            umma_commit(&done);
        }
        __syncwarp();
    }

    // ------------------------------------------------------------ epilogue
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&done, 0, p.timeout_ns, p.err, nullptr));
    tc_fence_after();
    if (ok && !*abort_flag) {
        const int row = 32 * warp + lane;                 // output feature m0 + row
        const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
        __nv_bfloat16 *dst = p.out + (size_t)h * p.M_total + m0 + row;
        const size_t bstride = (size_t)p.H * p.M_total;
        for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
            float v[32];
            tmem_ld32(trow + c0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int b = b0 + c0 + j;
                if (b < p.B) dst[(size_t)b * bstride] = __float2bfloat16_rn(v[j]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, tcols);
}

// ----------------------------------------------------------------- host
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

// Row-major bf16 [rows][cols], boxes of [box_rows][64] with 128-byte swizzle;
// rows past the end read as zero.
bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
              uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sequences per CTA: the smallest of 32 / 64 / 128 that holds B (more
// sequences take more CTAs).
int pick_n_tile(int B) { return B <= 32 ? 32 : (B <= 64 ? 64 : 128); }

// out[b][h][:] (M_total features) = W_h x_b for every head: the weight as
// stored [H][M_total][K] (A_MN false) or [H][K][M_total] (A_MN true), the
// inputs x as [B][H][K].
template <bool A_MN>
int launch_head_gemm(const void *w, const void *x, void *out, int B, int H, int M_total, int K,
                     cudaStream_t stream) {
    unsigned *err = internal_error_word();
    if (!err) return ATTN_ERR_CUDA;
    const int n_tile = pick_n_tile(B);
    // As many stages as the contraction has chunks (the whole weight slice
    // in flight at once), up to kHgMaxStages and kHgMaxSmem.
    int stages = K / kHgK < kHgMaxStages ? K / kHgK : kHgMaxStages;
    while (stages > 2 && stages * hg_stage_bytes(n_tile) > kHgMaxSmem) --stages;
    const int smem = stages * hg_stage_bytes(n_tile) + 1024;
    static PerDeviceFlag configured;   // the attribute is per function and device
    if (configure_once_per_device(configured, [] {
            return cudaFuncSetAttribute(head_gemm_kernel<A_MN>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kHgMaxSmem + 1024);
        }) != cudaSuccess)
        return ATTN_ERR_CUDA;
    CUtensorMap ta, tb;
    const bool ok_a = A_MN ? make_map(&ta, w, (uint64_t)M_total, (uint64_t)H * K, 64)
                           : make_map(&ta, w, (uint64_t)K, (uint64_t)H * M_total, kHgM);
    if (!ok_a || !make_map(&tb, x, (uint64_t)H * K, (uint64_t)B, (uint32_t)n_tile))
        return ATTN_ERR_CUDA;
    HeadGemmParams p{};
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.err = err;
    p.timeout_ns = kDefaultTimeoutNs;
    p.B = B;
    p.H = H;
    p.M_total = M_total;
    p.K = K;
    p.n_tile = n_tile;
    p.stages = stages;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M_total / kHgM, H, (B + n_tile - 1) / n_tile);
    cfg.blockDim = dim3(kHgThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, head_gemm_kernel<A_MN>, ta, tb, p) == cudaSuccess
               ? ATTN_OK
               : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" int attn_mla_absorb_q(const void *q_c, const void *u_k, void *q_latent, int B,
                                 int H, int d_c, int d_h, void *stream) {
    if (!q_c || !u_k || !q_latent) return ATTN_ERR_ARG;
    if (B <= 0 || H <= 0 || d_c <= 0 || d_h <= 0) return ATTN_ERR_ARG;
    if (!aligned16(q_c) || !aligned16(u_k) || !aligned16(q_latent)) return ATTN_ERR_ARG;
    if (d_c % kHgM || d_h % kHgK || H > 65535) return ATTN_ERR_UNSUPPORTED;
    // q_latent^T (d_c x B) = U^K_h (d_c x d_h, rows of d_h) x q_c^T
    return launch_head_gemm<false>(u_k, q_c, q_latent, B, H, d_c, d_h,
                                   static_cast<cudaStream_t>(stream));
}

extern "C" int attn_mla_project_out(const void *z, const void *u_v, void *o, int B, int H,
                                    int d_c, int d_v, void *stream) {
    if (!z || !u_v || !o) return ATTN_ERR_ARG;
    if (B <= 0 || H <= 0 || d_c <= 0 || d_v <= 0) return ATTN_ERR_ARG;
    if (!aligned16(z) || !aligned16(u_v) || !aligned16(o)) return ATTN_ERR_ARG;
    if (d_v % kHgM || d_c % kHgK || H > 65535) return ATTN_ERR_UNSUPPORTED;
    // o^T (d_v x B) = (U^V_h)^T (d_v x d_c; U^V_h stored [d_c][d_v]) x z^T
    return launch_head_gemm<true>(u_v, z, o, B, H, d_v, d_c, static_cast<cudaStream_t>(stream));
}
