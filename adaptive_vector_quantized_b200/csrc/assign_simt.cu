// Stage 1, assignment on CUDA cores ("AVQ-Attention: Adaptive
// Vector-Quantized Attention", Sec. 4.2, Algorithm 1: parent and child assignment).
//
// One thread per key.  The key is held in registers as fp32; the parent and
// child codewords are read with warp-uniform addresses (broadcast loads).
// Distances are in direct form sum_t (k_t - c_t)^2 in fp32.  Parent ties go
// to the lower index; a child must be strictly closer than the best child so
// far and strictly closer than the parent.
#include "common.cuh"
#include "internal.h"

namespace avq {

template <typename T, int D>
__device__ __forceinline__ float sqdist_row(const float* k, const T* c) {
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < D; t += 8) {
    float cv[8];
    load8(c + t, cv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float diff = k[t + e] - cv[e];
      acc = fmaf(diff, diff, acc);
    }
  }
  return acc;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) assign_simt_kernel(const T* __restrict__ K,
                                                          const T* __restrict__ parents,
                                                          const T* __restrict__ children,
                                                          int32_t* __restrict__ assign,
                                                          int32_t* __restrict__ counts, int H,
                                                          int N, int M0, int C) {
  const int bh = blockIdx.y;
  const int h = bh % H;
  const int j0 = blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = j0 < N;
  const int j = valid ? j0 : N - 1;  // out-of-range lanes recompute the last key, store nothing
  float k[D];
  const T* kp = K + ((size_t)bh * N + j) * D;
#pragma unroll
  for (int t = 0; t < D; t += 8) load8(kp + t, k + t);

  // nearest parent, first minimum
  const T* par = parents + (size_t)h * M0 * D;
  float best = __int_as_float(0x7f800000);
  int a = 0;
  for (int m = 0; m < M0; ++m) {
    const float dm = sqdist_row<T, D>(k, par + (size_t)m * D);
    if (dm < best) {
      best = dm;
      a = m;
    }
  }
  int code = a;
  // nearest child of a, moved only when strictly closer than a
  if (C > 0) {
    const T* ch = children + ((size_t)h * M0 + a) * C * D;
    float dchild = __int_as_float(0x7f800000);
    int cstar = 0;
    for (int c = 0; c < C; ++c) {
      const float dc = sqdist_row<T, D>(k, ch + (size_t)c * D);
      if (dc < dchild) {
        dchild = dc;
        cstar = c;
      }
    }
    if (dchild < best) code = M0 + a * C + cstar;
  }
  if (valid) assign[(size_t)bh * N + j] = code;
  count_codes(counts + (size_t)bh * M0 * (1 + C), code, valid, M0, C);
}

cudaError_t launch_assign_simt(const Shape& s, avq_dtype dt, const void* K, const void* parents,
                               const void* children, int32_t* assign, int32_t* counts,
                               cudaStream_t st, LaunchLog& log) {
  dim3 grid((s.N + 127) / 128, s.BH());
  dim3 block(128);
#define AVQ_LAUNCH(T, D)                                                                       \
  assign_simt_kernel<T, D><<<grid, block, 0, st>>>((const T*)K, (const T*)parents,            \
                                                   (const T*)children, assign, counts, s.H,   \
                                                   s.N, s.M0,                                  \
                                                   s.C)
  if (dt == AVQ_F32) {
    if (s.d == 64) AVQ_LAUNCH(float, 64); else AVQ_LAUNCH(float, 128);
  } else {
    if (s.d == 64) AVQ_LAUNCH(bf16, 64); else AVQ_LAUNCH(bf16, 128);
  }
#undef AVQ_LAUNCH
  log.add("assign_simt");
  return cudaGetLastError();
}

}  // namespace avq
