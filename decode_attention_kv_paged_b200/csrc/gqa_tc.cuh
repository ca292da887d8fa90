// gqa_tc.cuh -- host entry of the tensor-core (tcgen05) GQA/MQA decode path.
#pragma once

#include <cuda.h>

#include "gqa_launch.cuh"

namespace attn {

// The tensor-core kernel handles bf16, d in {64, 128, 256}, and groups of up
// to 64 query heads per pass (larger groups in multiples of 64).
bool gqa_tc_supported(int d, int dtype_bf16, int G);
int gqa_tc_heads_per_cta(int G);
// Copies of a group of HC heads in the 64 MMA rows (each takes a token
// slice); the kernel writes this many partials per (unit, CTA) slot.
int gqa_tc_copies(int HC);
// Group size from which the tensor-core path is the default.  Measured on
// B200 (B = 8, T = 32768): G = 2 CUDA cores 3% faster; G = 4 (d = 128) CUDA
// cores 3% faster at B = 8, level at B = 16 / T = 4096, 11% slower at
// B = 1 (kept on the CUDA cores); G = 6 tensor cores
// 1.3x (d = 128), 1.06x (d = 64), 1.13x (d = 256, ragged); G = 8 1.5x; from
// G = 16 1.8x-3.5x (the CUDA-core kernel splits larger groups and reads each
// K/V tile once per chunk of 8 heads).
constexpr int kTcMinGroup = 5;

cudaError_t launch_gqa_tc(const GqaLaunch &L, int d, int HC);

// The M = 128 tensor-core kernel (query and P in tensor memory): d in
// {64, 128} and units of at most 32 heads; it writes gqa_tc128_copies(HC)
// partials per (unit, CTA) slot.
bool gqa_tc128_supported(int d, int HC);
int gqa_tc128_copies(int HC);
cudaError_t launch_gqa_tc128(const GqaLaunch &L, int d, int HC);
// Its fp8 variant (E4M3 K/V codes with per-row scales, widened to f16 on the
// chip): the same shapes; HC = G, or 32 for groups that are multiples of 32.
bool gqa_tc128_fp8_supported(int d, int G);
int gqa_tc128_fp8_heads_per_cta(int G);
cudaError_t launch_gqa_tc128_fp8(const GqaLaunch &L, int d, int HC);

// 2-D tensor map over a row-major bf16 matrix [rows][cols] with 64-column,
// box_rows-row boxes and 128-byte swizzle.
bool tc_make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                 uint32_t box_rows);

}  // namespace attn
