// kv_append.cuh -- parameters of the paged-cache append kernel.
#pragma once

#include "plan.cuh"

namespace attn {

struct KvAppendParams {
    const void *k_new;       // [B][H_kv][row] (row = chunks_per_row * 16 bytes)
    const void *v_new;       // same, or null (MLA latent rows: one tensor)
    void *k_cache;           // [num_blocks][H_kv][64][row]
    void *v_cache;
    const int32_t *positions;
    const int32_t *block_table;
    unsigned *err;
    int B, H_kv, chunks_per_row, max_blocks, num_blocks;
    Visibility vis;          // sink / ring: where logical block pos / 64 lives
};

cudaError_t launch_kv_append(const KvAppendParams &p, cudaStream_t stream);

}  // namespace attn
