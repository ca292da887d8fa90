// gqa_fp8_d128.cu -- instantiations of the CUDA-core decode kernels for d = 128
// over an fp8 (e4m3, per-row scale) KV cache.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_fp8_d128(int HC, const GqaLaunch &L) {
    return launch_gqa_fp8_d<128>(HC, L);
}
}  // namespace attn
