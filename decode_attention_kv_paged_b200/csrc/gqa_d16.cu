// gqa_d16.cu -- instantiations of the CUDA-core decode kernels for d = 16.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_d16(int HC, int bf16, const GqaLaunch &L) {
    return launch_gqa_d<16>(HC, bf16, L);
}
}  // namespace attn
