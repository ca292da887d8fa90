// gqa_fp8_d64.cu -- instantiations of the CUDA-core decode kernels for d = 64
// over an fp8 (e4m3, per-row scale) KV cache.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_fp8_d64(int HC, const GqaLaunch &L) {
    return launch_gqa_fp8_d<64>(HC, L);
}
}  // namespace attn
