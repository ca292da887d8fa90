// gqa_d128.cu -- instantiations of the CUDA-core decode kernels for d = 128.
#include "gqa_launch.cuh"

namespace attn {
cudaError_t launch_gqa_d128(int HC, int bf16, const GqaLaunch &L) {
    return launch_gqa_d<128>(HC, bf16, L);
}
}  // namespace attn
