// mla_absorb.cu -- the two per-head products on either side of the absorbed
// MLA decode (attention-head article, §5.2 absorption):
//     q_latent[b,h] = q_c[b,h] (U^K_h)^T     (d_h -> d_c, before the decode)
//     o[b,h]        = z[b,h] U^V_h           (d_c -> d_v, after the decode)
// with U^K_h, U^V_h in R^{d_c x d_h} / R^{d_c x d_v} (k^C_j = c_j U^K_h,
// v_j = c_j U^V_h).  Both are plain batched GEMMs over the heads (bf16 in and
// out, fp32 accumulation), so they run as cuBLAS strided-batched GEMMs on
// the tensor cores; the attention itself stays in mla_decode.cu.
#include <cublas_v2.h>

#include <mutex>
#include <vector>

#include "attn_decode.h"

namespace {

struct BlasState {
    bool ready = false;
    cublasHandle_t handle = nullptr;
};

std::mutex g_blas_mu;
std::vector<BlasState> g_blas;

// The calling device's cuBLAS handle (created on first use), bound to `stream`.
int blas_handle(cudaStream_t stream, cublasHandle_t *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_blas_mu);
    if ((int)g_blas.size() <= dev) g_blas.resize(dev + 1);
    BlasState &st = g_blas[dev];
    if (!st.ready) {
        if (cublasCreate(&st.handle) != CUBLAS_STATUS_SUCCESS) return ATTN_ERR_CUDA;
        cublasSetMathMode(st.handle, CUBLAS_DEFAULT_MATH);
        st.ready = true;
    }
    if (cublasSetStream(st.handle, stream) != CUBLAS_STATUS_SUCCESS) return ATTN_ERR_CUDA;
    *out = st.handle;
    return ATTN_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int attn_mla_absorb_q(const void *q_c, const void *u_k, void *q_latent, int B,
                                 int H, int d_c, int d_h, void *stream) {
    if (!q_c || !u_k || !q_latent) return ATTN_ERR_ARG;
    if (B <= 0 || H <= 0 || d_c <= 0 || d_h <= 0) return ATTN_ERR_ARG;
    if (!aligned16(q_c) || !aligned16(u_k) || !aligned16(q_latent)) return ATTN_ERR_ARG;
    if (d_c % 8 || d_h % 8) return ATTN_ERR_UNSUPPORTED;
    cublasHandle_t h;
    const int rc = blas_handle(static_cast<cudaStream_t>(stream), &h);
    if (rc) return rc;
    // Column-major view, per head h:
    //   q_latent^T [d_c x B] (ld H d_c) = (U^K_h stored as [d_h x d_c], ld d_h)^T
    //                                     x q_c^T [d_h x B] (ld H d_h)
    const float one = 1.f, zero = 0.f;
    const cublasStatus_t s = cublasGemmStridedBatchedEx(
        h, CUBLAS_OP_T, CUBLAS_OP_N, d_c, B, d_h, &one,
        u_k, CUDA_R_16BF, d_h, (long long)d_c * d_h,
        q_c, CUDA_R_16BF, H * d_h, (long long)d_h,
        &zero, q_latent, CUDA_R_16BF, H * d_c, (long long)d_c,
        H, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
    return s == CUBLAS_STATUS_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_mla_project_out(const void *z, const void *u_v, void *o, int B, int H,
                                    int d_c, int d_v, void *stream) {
    if (!z || !u_v || !o) return ATTN_ERR_ARG;
    if (B <= 0 || H <= 0 || d_c <= 0 || d_v <= 0) return ATTN_ERR_ARG;
    if (!aligned16(z) || !aligned16(u_v) || !aligned16(o)) return ATTN_ERR_ARG;
    if (d_c % 8 || d_v % 8) return ATTN_ERR_UNSUPPORTED;
    cublasHandle_t h;
    const int rc = blas_handle(static_cast<cudaStream_t>(stream), &h);
    if (rc) return rc;
    // Column-major view, per head h:
    //   o^T [d_v x B] (ld H d_v) = (U^V_h stored as [d_v x d_c], ld d_v)
    //                              x z^T [d_c x B] (ld H d_c)
    const float one = 1.f, zero = 0.f;
    const cublasStatus_t s = cublasGemmStridedBatchedEx(
        h, CUBLAS_OP_N, CUBLAS_OP_N, d_v, B, d_c, &one,
        u_v, CUDA_R_16BF, d_v, (long long)d_c * d_v,
        z, CUDA_R_16BF, H * d_c, (long long)d_c,
        &zero, o, CUDA_R_16BF, H * d_v, (long long)d_v,
        H, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
    return s == CUBLAS_STATUS_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}
