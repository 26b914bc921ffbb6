// Stage 2 on CUDA cores ("AVQ-Attention: Adaptive Vector-Quantized
// Attention", Sec. 4.3, Algorithm 2; Eqs. 6-9; Sec. D, Eq. 18).
//
// General kernel for every supported shape and both element types.  One CTA
// per (head, query block), one thread per query row.  The row's query sits
// in padded shared memory; codewords and statistics are read with
// warp-uniform addresses.  The parent pass is done in two sweeps (running max
// and denominator first, then A, x and the importance with the exact
// denominator), which is the exact two-pass denominator and equals the
// single-pass result.  Importance column sums use warp shuffles plus one
// shared atomic per warp; top-P ranks every parent in one warp (descending,
// ties to the lower index); the refinement follows Algorithm 2
// with the online max merge per selected parent.
#include "common.cuh"
#include "internal.h"

namespace avq {

namespace {

template <typename T, int D>
__device__ __forceinline__ float dot_row(const float* q, const T* c) {
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < D; t += 8) {
    float cv[8];
    load8(c + t, cv);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(q[t + e], cv[e], acc);
  }
  return acc;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) attention_simt_kernel(
    const T* __restrict__ Q, const T* __restrict__ parents, const T* __restrict__ children,
    const float* __restrict__ vsum, const int32_t* __restrict__ counts, int H, int N, int M0,
    int C, int P, int block, float scale, T* __restrict__ O, int32_t* __restrict__ sel,
    float* __restrict__ importance) {
  extern __shared__ __align__(16) float sm[];
  const int Mt = M0 * (1 + C);
  float* qs = sm;                                   // [block][D+1]
  float* nf = qs + (size_t)block * (D + 1);         // [Mt] counts as float
  float* w = nf + Mt;                               // [M0] importance
  int* ssel = reinterpret_cast<int*>(w + M0);       // [P]
  const int bh = blockIdx.y, h = bh % H, blk = blockIdx.x, nblk = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int i = blk * block + tid;
  const bool valid = tid < block && i < N;

  // query rows -> shared memory (fp32, rows padded to D+1 floats)
  for (int idx = tid; idx < block * (D / 8); idx += blockDim.x) {
    const int r = idx / (D / 8), t = (idx % (D / 8)) * 8;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (blk * block + r < N) load8(Q + ((size_t)bh * N + blk * block + r) * D + t, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) qs[r * (D + 1) + t + e] = v[e];
  }
  for (int r = tid; r < Mt; r += blockDim.x) nf[r] = (float)counts[(size_t)bh * Mt + r];
  for (int r = tid; r < M0; r += blockDim.x) w[r] = 0.f;
  __syncthreads();

  const float* qr = qs + (size_t)(tid < block ? tid : 0) * (D + 1);
  const T* par = parents + (size_t)h * M0 * D;
  const float* vs = vsum + (size_t)bh * Mt * D;

  // Sweep 1 (denominator only): running max over non-empty
  // parents (Eq. 18) and z = sum_j exp(s_j - m) n_j.
  float m = __int_as_float(0xff800000), z = 0.f;
  for (int j = 0; j < M0; ++j) {
    const float nj = nf[j];
    if (nj > 0.f) {
      const float s = scale * dot_row<T, D>(qr, par + (size_t)j * D);
      if (s > m) {
        z = z * expf(m - s) + nj;
        m = s;
      } else {
        z = fmaf(nj, expf(s - m), z);
      }
    }
  }
  // Sweep 2: A = exp(s - m) masked, x = A V-bar, importance (Eq. 7).
  float x[D];
#pragma unroll
  for (int t = 0; t < D; ++t) x[t] = 0.f;
  const float rz = 1.f / z;
  for (int j = 0; j < M0; ++j) {
    const float nj = nf[j];
    float a = 0.f;
    if (nj > 0.f) {
      const float s = scale * dot_row<T, D>(qr, par + (size_t)j * D);
      a = expf(s - m);
      const float* vj = vs + (size_t)j * D;
#pragma unroll
      for (int t = 0; t < D; t += 4) {
        const float4 v4 = __ldg(reinterpret_cast<const float4*>(vj + t));
        x[t] = fmaf(a, v4.x, x[t]);
        x[t + 1] = fmaf(a, v4.y, x[t + 1]);
        x[t + 2] = fmaf(a, v4.z, x[t + 2]);
        x[t + 3] = fmaf(a, v4.w, x[t + 3]);
      }
    }
    const float col = warp_sum(valid ? a * nj * rz : 0.f);
    if (lane == 0 && col != 0.f) atomicAdd(w + j, col);
  }
  __syncthreads();

  // Top-P (descending, ties to the lower index) in one warp.
  const int nsel = C > 0 ? P : 0;
  if (tid < 32) {
    for (int j = lane; j < M0; j += 32) {
      const float wj = w[j];
      int rank = 0;
      for (int l = 0; l < M0; ++l) {
        const float wl = w[l];
        rank += (wl > wj) || (wl == wj && l < j);
      }
      if (rank < P) ssel[rank] = j;
      if (importance) importance[((size_t)bh * nblk + blk) * M0 + j] = wj;
    }
    __syncwarp();
    if (sel)
      for (int r = lane; r < P; r += 32) sel[((size_t)bh * nblk + blk) * P + r] = ssel[r];
  }
  __syncthreads();

  // Child refinement of the selected parents.
  for (int r = 0; r < nsel; ++r) {
    const int p = ssel[r];
    const T* cc = children + ((size_t)h * M0 + p) * C * D;
    float sc[8];
    float mp = m;
    float sp = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < C) {
        sc[c] = scale * dot_row<T, D>(qr, cc + (size_t)c * D);
        sp += sc[c];
        if (nf[M0 + p * C + c] > 0.f && sc[c] > mp) mp = sc[c];  // online max
      }
    }
    sp = sp / (float)C;  // Eq. 8
    const float f = expf(m - mp);  // rescale
    z *= f;
#pragma unroll
    for (int t = 0; t < D; ++t) x[t] *= f;
    m = mp;
    const float ap = expf(sp - m);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < C) {
        const float nc = nf[M0 + p * C + c];
        if (nc > 0.f) {  // Eq. 9, dA zeroed for empty children
          const float da = expf(sc[c] - m) - ap;
          const float* vc = vs + (size_t)(M0 + p * C + c) * D;
#pragma unroll
          for (int t = 0; t < D; t += 4) {
            const float4 v4 = __ldg(reinterpret_cast<const float4*>(vc + t));
            x[t] = fmaf(da, v4.x, x[t]);
            x[t + 1] = fmaf(da, v4.y, x[t + 1]);
            x[t + 2] = fmaf(da, v4.z, x[t + 2]);
            x[t + 3] = fmaf(da, v4.w, x[t + 3]);
          }
          z = fmaf(da, nc, z);
        }
      }
    }
  }
  // Y = x / z.
  if (valid) {
    const float iz = 1.f / z;
    T* o = O + ((size_t)bh * N + i) * D;
#pragma unroll
    for (int t = 0; t < D; t += 8) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = x[t + e] * iz;
      store8(o + t, v);
    }
  }
}

}  // namespace

cudaError_t launch_attention_simt(const Shape& s, avq_dtype dt, const void* Q, const void* parents,
                                  const void* children, const float* vsum, const int32_t* counts,
                                  int P, int block, float scale, void* O, int32_t* sel,
                                  float* importance, cudaStream_t st, LaunchLog& log) {
  const int nblk = (s.N + block - 1) / block;
  dim3 grid(nblk, s.BH());
  const size_t smem = ((size_t)block * (s.d + 1) + s.Mt() + s.M0 + (P > 0 ? P : 1)) * sizeof(float);
  cudaError_t e;
#define AVQ_ATT(T, D)                                                                              \
  do {                                                                                             \
    auto kern = attention_simt_kernel<T, D>;                                                       \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);        \
    if (e != cudaSuccess) return e;                                                                \
    kern<<<grid, 128, smem, st>>>((const T*)Q, (const T*)parents, (const T*)children, vsum,        \
                                  counts, s.H, s.N, s.M0, s.C, P, block, scale, (T*)O, sel,        \
                                  importance);                                                     \
  } while (0)
  if (dt == AVQ_F32) {
    if (s.d == 64) AVQ_ATT(float, 64); else AVQ_ATT(float, 128);
  } else {
    if (s.d == 64) AVQ_ATT(bf16, 64); else AVQ_ATT(bf16, 128);
  }
#undef AVQ_ATT
  log.add("attention_simt");
  return cudaGetLastError();
}

}  // namespace avq
