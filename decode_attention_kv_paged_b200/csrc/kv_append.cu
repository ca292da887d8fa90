// kv_append.cu -- scatter each sequence's newly produced K/V rows (or MLA
// latent row) into its paged slot.  Position pos of sequence b lands in
// logical block pos / 64, row pos % 64 (paged cache; the toolsku article's
// decode step concatenates the new K/V to the cache before attention).
#include "kv_append.cuh"

namespace attn {

// One thread per 16-byte chunk of one (sequence, head) row, for K and V.
__global__ void kv_append_kernel(const KvAppendParams p) {
    const long long total = (long long)p.B * p.H_kv * p.chunks_per_row;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i % p.chunks_per_row);
        const long long bh = i / p.chunks_per_row;
        const int h = (int)(bh % p.H_kv);
        const int b = (int)(bh / p.H_kv);
        const int pos = p.positions[b];
        const int slot = pos < 0 ? -1 : table_slot(p.vis, pos / kBlockSize);
        if (slot < 0 || slot >= p.max_blocks) {
            if (c == 0 && h == 0) raise_error(p.err, kErrBadBlock);
            continue;
        }
        const int phys = p.block_table[(size_t)b * p.max_blocks + slot];
        if (phys < 0 || phys >= p.num_blocks) {
            if (c == 0 && h == 0) raise_error(p.err, kErrBadBlock);
            continue;
        }
        const size_t dst_row =
            ((size_t)phys * p.H_kv + h) * kBlockSize + (pos % kBlockSize);
        const size_t src_row = (size_t)b * p.H_kv + h;
        const size_t rc = p.chunks_per_row;
        reinterpret_cast<uint4 *>(p.k_cache)[dst_row * rc + c] =
            reinterpret_cast<const uint4 *>(p.k_new)[src_row * rc + c];
        if (p.v_new)
            reinterpret_cast<uint4 *>(p.v_cache)[dst_row * rc + c] =
                reinterpret_cast<const uint4 *>(p.v_new)[src_row * rc + c];
    }
}

cudaError_t launch_kv_append(const KvAppendParams &p, cudaStream_t stream) {
    const long long total = (long long)p.B * p.H_kv * p.chunks_per_row;
    if (total == 0) return cudaSuccess;
    long long blocks = (total + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    kv_append_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace attn
