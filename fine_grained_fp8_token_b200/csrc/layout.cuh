// Output layout of the tensor-parallel column split: P ranks each compute
// Y_p = X * W_p^T for their n = N/P output columns, an all-gather stacks the
// parts as [P, M, n], and this kernel writes them as the layer's Y [M, P * n]
// (Y[m, p * n + j] = part[p, m, j]).  Pure data movement: 16-byte chunks,
// consecutive threads on consecutive chunks of a part row, so reads and
// writes are both coalesced.  Chunk indices are 32-bit (the host checks
// P * M * n / 8 < 2^32) and split by multiplicative division.
#pragma once
#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace fgfp8 {

__global__ void __launch_bounds__(256) gather_cols_kernel(const uint4* __restrict__ parts, uint32_t total,
                                                          FastDiv chunks_per_row, FastDiv rows,
                                                          uint4* __restrict__ Y) {
  const uint32_t cpr = chunks_per_row.d;                 // 16-byte chunks per part row (n / 8)
  const uint32_t M = rows.d;
  const uint32_t P_cpr = total / M;                      // chunks per output row (P * n / 8)
  const uint32_t step = gridDim.x * blockDim.x;
  // the increment never wraps past the 32-bit count (a wrapped index would restart the pass)
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i = (total - i > step) ? i + step : total) {
    const uint32_t row = chunks_per_row.div(i);          // p * M + m
    const uint32_t c = i - row * cpr;
    const uint32_t p = rows.div(row);
    const uint32_t m = row - p * M;
    FGFP8_DCHECK(m < M && c < cpr && p * cpr + c < P_cpr);
    Y[static_cast<uint64_t>(m) * P_cpr + p * cpr + c] = __ldg(parts + i);
  }
}

}  // namespace fgfp8
