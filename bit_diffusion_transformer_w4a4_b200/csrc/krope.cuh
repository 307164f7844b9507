// Row-blocked copy of the caller's rotary table for the fused QKV epilogue.
//
// "Nunchaku Lite ..." (axbrief.com), section "The Trade-off Between Fused
// Kernels and Generality": the rotary embedding runs inside the QKV
// projection's kernel.  There an epilogue lane owns one token row, so with the
// caller's row-major table [M][64 pairs][2] every load of a warp would touch
// 32 rows 512 bytes apart (32 cache lines per instruction, on the same L1 /
// shared-memory data path that feeds the tensor cores their operands).  This
// kernel rewrites the table once per call as
//     blk[rows_pad / 32][32 chunks][32 rows] float4,
// chunk c = (cos, sin) of pairs 2c and 2c + 1, so that a warp's load of one
// chunk for its 32 rows reads 512 contiguous bytes.  Rows M .. rows_pad - 1
// get (1, 0, 1, 0), the identity rotation (those rows are never stored).
#pragma once

#include "ptx.cuh"

namespace svdq {

// One CTA of 256 threads per 32-row block; a padded shared tile (33 float4 a
// row) keeps both the row-major writes and the column-major reads free of
// bank conflicts.  Both global sides are coalesced.
__global__ void __launch_bounds__(256) rope_block_kernel(const float4* __restrict__ rope, int M,
                                                         float4* __restrict__ blk) {
  __shared__ float4 s[32][33];
  griddep_wait();  // the table may be written by the preceding kernel
  griddep_launch_dependents();
  const int rb = blockIdx.x;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = threadIdx.x + 256 * k;
    const int r = i >> 5, c = i & 31;
    const int row = rb * 32 + r;
    s[r][c] = row < M ? __ldg(rope + static_cast<size_t>(row) * 32 + c) : make_float4(1.f, 0.f, 1.f, 0.f);
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = threadIdx.x + 256 * k;
    const int c = i >> 5, r = i & 31;
    blk[(static_cast<size_t>(rb) * 32 + c) * 32 + r] = s[r][c];
  }
}

}  // namespace svdq
