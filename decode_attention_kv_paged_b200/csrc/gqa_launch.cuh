// gqa_launch.cuh -- host-side launch of the CUDA-core split-KV kernel (which
// also combines its split partials) for one (head dim, heads-per-CTA, dtype)
// instantiation.
#pragma once

#include "gqa_decode.cuh"
#include "host_state.cuh"

namespace attn {

struct GqaLaunch {
    GqaParams kp;
    CombineParams cp;         // combine launch of the tensor-core path
    int units_total;          // B * H_kv * n_hc
    cudaStream_t stream;
    cudaEvent_t ev_start;     // optional (profiling hook), may be null
    cudaEvent_t ev_stop;
};

// Shared-memory bytes the split kernel of this instantiation needs.
template <int D, int HC, typename T, typename TK = T>
int gqa_smem_bytes() { return GqaCfg<D, HC, T, TK>::kSmemBytes; }

template <int D, int HC, typename T, typename TK = T, bool G = false>
cudaError_t launch_gqa_impl(const GqaLaunch &L) {
    using C = GqaCfg<D, HC, T, TK>;
    // The attribute is set on the function for the current device only.
    static PerDeviceFlag configured;
    cudaError_t e = configure_once_per_device(configured, [] {
        // The warpgroups' setmaxnreg shares must fit in the registers the
        // kernel is launched with, or the increase would never be granted.
        cudaFuncAttributes fa;
        cudaError_t r = cudaFuncGetAttributes(&fa, gqa_split_kernel<D, HC, T, TK, G>);
        if (r != cudaSuccess) return r;
        if (fa.numRegs * C::kThreads <
            4 * 32 * C::kProducerRegs + C::kNW * 32 * C::kConsumerRegs)
            return cudaErrorInvalidConfiguration;
        return cudaFuncSetAttribute(gqa_split_kernel<D, HC, T, TK, G>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    if (L.ev_start) cudaEventRecord(L.ev_start, L.stream);
    // The split partials are combined inside the kernel (by the last split
    // of each unit), so this is the call's only launch.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)L.kp.num_ctas);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gqa_split_kernel<D, HC, T, TK, G>, L.kp);
    if (e != cudaSuccess) return e;
    if (L.ev_stop) cudaEventRecord(L.ev_stop, L.stream);
    return cudaSuccess;
}

// Dispatch over heads-per-CTA and dtype for one head dimension D.
template <int D>
cudaError_t launch_gqa_d(int HC, int dtype_bf16, const GqaLaunch &L) {
    const bool g = L.kp.vis.n_g > 0;
#define ATTN_CASE(hc)                                                                  \
    case hc:                                                                           \
        if (dtype_bf16)                                                                \
            return g ? launch_gqa_impl<D, hc, __nv_bfloat16, __nv_bfloat16, true>(L)   \
                     : launch_gqa_impl<D, hc, __nv_bfloat16>(L);                       \
        if constexpr (D <= 128)                                                        \
            return g ? launch_gqa_impl<D, hc, float, float, true>(L)                   \
                     : launch_gqa_impl<D, hc, float>(L);                               \
        return cudaErrorNotSupported;
    switch (HC) {
        ATTN_CASE(1)
        ATTN_CASE(2)
        ATTN_CASE(3)
        ATTN_CASE(4)
        ATTN_CASE(6)
        ATTN_CASE(8)
        default: return cudaErrorInvalidValue;
    }
#undef ATTN_CASE
}

cudaError_t launch_gqa_d16(int HC, int bf16, const GqaLaunch &L);
cudaError_t launch_gqa_d32(int HC, int bf16, const GqaLaunch &L);
cudaError_t launch_gqa_d64(int HC, int bf16, const GqaLaunch &L);
cudaError_t launch_gqa_d128(int HC, int bf16, const GqaLaunch &L);
cudaError_t launch_gqa_d256(int HC, int bf16, const GqaLaunch &L);

// bf16 queries over an fp8 (e4m3 + per-row fp32 scale) cache, d in {64, 128, 256}.
template <int D>
cudaError_t launch_gqa_fp8_d(int HC, const GqaLaunch &L) {
    const bool g = L.kp.vis.n_g > 0;
#define ATTN_FP8(hc)                                                                   \
    case hc:                                                                           \
        return g ? launch_gqa_impl<D, hc, __nv_bfloat16, uint8_t, true>(L)             \
                 : launch_gqa_impl<D, hc, __nv_bfloat16, uint8_t>(L);
    switch (HC) {
        ATTN_FP8(1)
        ATTN_FP8(2)
        ATTN_FP8(3)
        ATTN_FP8(4)
        ATTN_FP8(6)
        ATTN_FP8(8)
        default: return cudaErrorInvalidValue;
    }
#undef ATTN_FP8
}
cudaError_t launch_gqa_fp8_d64(int HC, const GqaLaunch &L);
cudaError_t launch_gqa_fp8_d128(int HC, const GqaLaunch &L);
cudaError_t launch_gqa_fp8_d256(int HC, const GqaLaunch &L);

}  // namespace attn

namespace attn {
// Runs the split planner alone (one CTA per planned CTA) and writes the plan:
// out[0] = W; out[1 + 4i .. 4 + 4i] = range start, range end, first sequence,
// first unit of CTA i; then B + 1 exclusive work prefix sums.
cudaError_t launch_plan_kernel(const int32_t *seq_lens, int B, int units_per_seq,
                               Visibility vis, int max_blocks, int num_ctas,
                               long long *out, unsigned *err, cudaStream_t stream);
}  // namespace attn
