// gqa_d64.cu -- instantiations of the CUDA-core decode kernels for d = 64.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_d64(int HC, int bf16, const GqaLaunch &L) {
    return launch_gqa_d<64>(HC, bf16, L);
}
}  // namespace attn
