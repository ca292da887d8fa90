// gqa_d32.cu -- instantiations of the CUDA-core decode kernels for d = 32.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_d32(int HC, int bf16, const GqaLaunch &L) {
    return launch_gqa_d<32>(HC, bf16, L);
}
}  // namespace attn
