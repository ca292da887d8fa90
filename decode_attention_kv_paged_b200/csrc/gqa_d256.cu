// gqa_d256.cu -- instantiations of the CUDA-core decode kernels for d = 256.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_d256(int HC, int bf16, const GqaLaunch &L) {
    return launch_gqa_d<256>(HC, bf16, L);
}
}  // namespace attn
