// Token reordering gather/scatter ("AVQ-Attention: Adaptive Vector-Quantized
// Attention", Sec. 4.2 and Fig. 3: tokens are reordered along a space-filling
// curve so that contiguous query tiles are spatially compact).  A pure data
// move: each thread copies 16-byte pieces of one row, coalesced along the row.
#include "common.cuh"
#include "internal.h"

namespace avq {

namespace {

__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ X,
                                                      const int32_t* __restrict__ idx,
                                                      uint4* __restrict__ Y, int rows,
                                                      int vec_per_row, int inverse,
                                                      long long total, unsigned int* err) {
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int v = (int)(g % vec_per_row);
    const long long br = g / vec_per_row;  // b * rows + i
    const int i = (int)(br % rows);
    const long long b = br / rows;
    const int j = __ldg(idx + i);
    if ((unsigned)j >= (unsigned)rows) {  // an index outside the rows: refused, reported
      if (v == 0) atomicOr(err, kErrBounds);
      continue;
    }
    const long long src = inverse ? br : b * rows + j;
    const long long dst = inverse ? b * rows + j : br;
    Y[dst * vec_per_row + v] = __ldg(X + src * vec_per_row + v);
  }
}

}  // namespace

cudaError_t launch_permute(const void* X, const int32_t* idx, void* Y, int batch, int rows,
                           int row_bytes, int inverse, unsigned int* err, cudaStream_t st, LaunchLog& log) {
  const int vpr = row_bytes / 16;
  const long long total = (long long)batch * rows * vpr;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  permute_kernel<<<(unsigned)blocks, 256, 0, st>>>((const uint4*)X, idx, (uint4*)Y, rows, vpr,
                                                   inverse, total, err);
  log.add("permute");
  return cudaGetLastError();
}

}  // namespace avq
