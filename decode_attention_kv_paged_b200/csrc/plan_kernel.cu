// plan_kernel.cu -- the device split planner run on its own, for bit-exact
// checks against a host model of the partition.  Uses exactly the device
// functions the decode kernels use (plan.cuh).
#include "gqa_launch.cuh"

namespace attn {

__global__ void __launch_bounds__(256) plan_kernel(PlanArgs a, long long *out,
                                                  unsigned *err) {
    __shared__ PlanScratch sh;
    long long *prefix = out + 1 + 4ll * a.num_ctas;
    plan_locate(a, blockIdx.x, &sh, blockIdx.x == 0 ? prefix : nullptr, err);
    if (threadIdx.x != 0) return;
    const long long W = sh.total;
    long long *row = out + 1 + 4ll * blockIdx.x;
    if (blockIdx.x == 0) out[0] = W;
    const int P = working_ctas(W, a.num_ctas);
    const long long lo = (int)blockIdx.x < P ? cta_bound(blockIdx.x, W, P) : W;
    const long long hi = (int)blockIdx.x < P ? cta_bound(blockIdx.x + 1, W, P) : W;
    row[0] = lo;
    row[1] = hi;
    if (lo >= hi) {
        row[2] = -1;
        row[3] = -1;
        return;
    }
    SegmentWalker w;
    w.init(a, lo, hi, sh.seq, sh.base);
    row[2] = w.b;
    row[3] = w.unit;
}

cudaError_t launch_plan_kernel(const int32_t *seq_lens, int B, int units_per_seq,
                               Visibility vis, int max_blocks, int num_ctas,
                               long long *out, unsigned *err, cudaStream_t stream) {
    PlanArgs a{seq_lens, B, units_per_seq, vis, max_blocks, num_ctas};
    plan_kernel<<<num_ctas, 256, 0, stream>>>(a, out, err);
    return cudaGetLastError();
}

}  // namespace attn
