// mla_launch.cuh -- host entry of the absorbed-MLA decode path.
#pragma once

#include <cstddef>
#include <functional>

#include "common.cuh"

namespace attn {

// Workspace provider: grows the caller's per-device workspace to `bytes` and
// returns it; returns an attn_status.
using WorkspaceFn = std::function<int(size_t bytes, void **ws)>;

// latent_scale == nullptr: bf16 latent cache; else an fp8 cache of E4M3 codes
// with one fp32 scale per cached row ([num_blocks][64]).
int mla_decode_entry(const void *q_latent, const void *q_rope, const void *latent_cache,
                     const float *latent_scale, const int32_t *seq_lens,
                     const int32_t *block_table, void *out, int B, int H, float scale,
                     cudaStream_t stream, int max_blocks, int num_blocks, int num_sms,
                     int forced_ctas, unsigned *err, const WorkspaceFn &workspace,
                     cudaEvent_t ev_start = nullptr, cudaEvent_t ev_stop = nullptr);

}  // namespace attn
