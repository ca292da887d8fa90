// kv_append.cu -- scatter each sequence's newly produced K/V rows (or MLA
// latent row) into its paged slot.  Position pos of sequence b lands in
// logical block pos / 64, row pos % 64 (paged cache; the toolsku article's
// decode step concatenates the new K/V to the cache before attention).
#include <cuda_fp8.h>

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

namespace attn {

// fp8 append: one warp per (sequence, KV head) row of K and one of V (K only
// for the MLA latent cache, whose row is c_j followed by kR_j).  Each
// row of d bf16 values x is stored as e4m3 codes of x * (448 / amax) (round to
// nearest even, saturating) with the fp32 row scale amax / 448, amax =
// max |x| (a zero row: scale 0, codes 0).  Divisions are IEEE round-to-nearest.
__global__ void kv_append_fp8_kernel(const KvAppendFp8Params p) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int rows = p.B * p.H_kv * (p.v_new ? 2 : 1);   // K rows, then V rows (if any)
    if (warp >= rows) return;
    const bool is_v = warp >= p.B * p.H_kv;
    const int bh = is_v ? warp - p.B * p.H_kv : warp;
    const int b = bh / p.H_kv, h = bh % p.H_kv;
    const int pos = p.positions[b];
    const int slot = pos < 0 ? -1 : table_slot(p.vis, pos / kBlockSize);
    if (slot < 0 || slot >= p.max_blocks) {
        if (lane == 0 && bh == 0 && !is_v) raise_error(p.err, kErrBadBlock);
        return;
    }
    const int phys = p.block_table[(size_t)b * p.max_blocks + slot];
    if (phys < 0 || phys >= p.num_blocks) {
        if (lane == 0 && bh == 0 && !is_v) raise_error(p.err, kErrBadBlock);
        return;
    }
    const __nv_bfloat16 *src = (is_v ? p.v_new : p.k_new) + (size_t)bh * p.d;
    const size_t row = ((size_t)phys * p.H_kv + h) * kBlockSize + pos % kBlockSize;
    uint8_t *dst = (is_v ? p.v_cache : p.k_cache) + row * p.d;
    float amax = 0.f;
    for (int i = lane; i < p.d; i += 32) amax = fmaxf(amax, fabsf(__bfloat162float(src[i])));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    for (int i = 2 * lane; i < p.d; i += 64) {
        const float2 x = make_float2(__fmul_rn(__bfloat162float(src[i]), inv),
                                     __fmul_rn(__bfloat162float(src[i + 1]), inv));
        const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
        *reinterpret_cast<__nv_fp8x2_storage_t *>(dst + i) = c;
    }
    if (lane == 0) (is_v ? p.v_scale : p.k_scale)[row] = __fdiv_rn(amax, 448.f);
}

cudaError_t launch_kv_append_fp8(const KvAppendFp8Params &p, cudaStream_t stream) {
    const int rows = p.B * p.H_kv * (p.v_new ? 2 : 1);
    const int threads = 256;
    const int blocks = (rows * 32 + threads - 1) / threads;
    kv_append_fp8_kernel<<<blocks, threads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace attn
