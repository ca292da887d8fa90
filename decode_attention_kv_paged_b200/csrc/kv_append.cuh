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

struct KvAppendFp8Params {
    const __nv_bfloat16 *k_new;   // [B][H_kv][d]
    const __nv_bfloat16 *v_new;
    uint8_t *k_cache;             // [num_blocks][H_kv][64][d] e4m3 codes
    uint8_t *v_cache;
    float *k_scale;               // [num_blocks][H_kv][64] row scales
    float *v_scale;
    const int32_t *positions;
    const int32_t *block_table;
    unsigned *err;
    int B, H_kv, d, max_blocks, num_blocks;
    Visibility vis;
};

cudaError_t launch_kv_append_fp8(const KvAppendFp8Params &p, cudaStream_t stream);

}  // namespace attn
