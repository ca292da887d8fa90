// mla_decode.cu -- absorbed MLA decode (placeholder until the tensor-core
// kernel lands).
#include "attn_decode.h"
#include "mla_launch.cuh"

namespace attn {
int mla_decode_entry(const void *, const void *, const void *, const int32_t *,
                     const int32_t *, void *, int, int, float, cudaStream_t, int, int,
                     int, int, unsigned *, const WorkspaceFn &) {
    return ATTN_ERR_UNSUPPORTED;
}
}  // namespace attn
