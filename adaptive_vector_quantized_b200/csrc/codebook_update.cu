// Codebook update ("AVQ-Attention: Adaptive Vector-Quantized Attention",
// Sec. A "Codeword Clustering During Training", Eqs. 11-12).
//
// EMA statistics (Eq. 11) per head over every batch entry's keys:
//   S_x <- lambda S_x + (1 - lambda) sum_k k,  N_x <- lambda N_x + (1 - lambda) n_x,
// with the statistics of Eq. 3 computed on the keys (a parent counts its whole
// cluster, a child the keys that moved to it).  Parents take their means
// C_p = S_p / N_p; children the mass-weighted projection of their means M_c
// onto sum_c C_pc = C C_p (Eq. 12):
//   delta = sum_c M_c - C C_p,  sigma = sum_c 1 / N_c,  C_pc = M_c - delta / (N_c sigma).
// A code without mass keeps its position in place of a mean; massless
// children do not move and the others absorb delta (sigma over them); with no
// massive child all C children shift by delta / C.
//
// One CTA per (head, parent), one thread per dimension: the CTA reads the
// parent's and its children's counts into shared memory before anyone
// overwrites them, so the update is done in place.
#include "common.cuh"
#include "internal.h"

namespace avq {

namespace {

constexpr int kMaxChildren = 8;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

template <typename T>
__global__ void codebook_update_kernel(const float* __restrict__ ksum, const int32_t* __restrict__ counts,
                                       float* __restrict__ S, float* __restrict__ Nst, T* __restrict__ parents,
                                       T* __restrict__ children, int B, int H, int d, int M0, int C,
                                       float lambda) {
  __shared__ float sN[1 + kMaxChildren];  // updated masses of the parent and its children
  const int h = blockIdx.y, p = blockIdx.x, t = threadIdx.x;
  const int Mt = M0 * (1 + C);
  const float keep = lambda, take = 1.f - lambda;
  if (t <= C) {
    const int x = t == 0 ? p : M0 + p * C + (t - 1);
    float n = 0.f;
    for (int b = 0; b < B; ++b) n += (float)counts[((size_t)b * H + h) * Mt + x];
    sN[t] = keep * Nst[(size_t)h * Mt + x] + take * n;
  }
  __syncthreads();
  if (t <= C) Nst[(size_t)h * Mt + (t == 0 ? p : M0 + p * C + (t - 1))] = sN[t];
  if (t >= d) return;
  auto ema = [&](int x) {  // updated S_x[t]
    float sk = 0.f;
    for (int b = 0; b < B; ++b) sk += ksum[(((size_t)b * H + h) * Mt + x) * d + t];
    float* sx = S + ((size_t)h * Mt + x) * d + t;
    const float v = keep * *sx + take * sk;
    *sx = v;
    return v;
  };
  T* cp = parents + ((size_t)h * M0 + p) * d + t;
  const float sp = ema(p);
  const float par = sN[0] > 0.f ? sp / sN[0] : to_f<T>(*cp);
  *cp = from_f<T>(par);
  if (C == 0) return;
  float m[kMaxChildren];
  float sigma = 0.f, delta = -(float)C * par;
  int massive = 0;
  for (int c = 0; c < C; ++c) {
    const float sc = ema(M0 + p * C + c);
    const float nc = sN[1 + c];
    m[c] = nc > 0.f ? sc / nc : to_f<T>(children[(((size_t)h * M0 + p) * C + c) * d + t]);
    delta += m[c];
    if (nc > 0.f) {
      sigma += 1.f / nc;
      ++massive;
    }
  }
  for (int c = 0; c < C; ++c) {
    const float nc = sN[1 + c];
    const float shift = massive > 0 ? (nc > 0.f ? delta / (nc * sigma) : 0.f) : delta / (float)C;
    children[(((size_t)h * M0 + p) * C + c) * d + t] = from_f<T>(m[c] - shift);
  }
}

}  // namespace

cudaError_t launch_codebook_update(const Shape& s, avq_dtype dt, float lambda, const float* ksum,
                                   const int32_t* counts, float* S, float* Nst, void* parents,
                                   void* children, cudaStream_t st, LaunchLog& log) {
  dim3 grid(s.M0, s.H);
  const int threads = s.d > kMaxChildren + 1 ? s.d : kMaxChildren + 1;
  if (dt == AVQ_F32)
    codebook_update_kernel<float><<<grid, threads, 0, st>>>(ksum, counts, S, Nst, (float*)parents,
                                                            (float*)children, s.B, s.H, s.d, s.M0, s.C,
                                                            lambda);
  else
    codebook_update_kernel<bf16><<<grid, threads, 0, st>>>(ksum, counts, S, Nst, (bf16*)parents,
                                                           (bf16*)children, s.B, s.H, s.d, s.M0, s.C,
                                                           lambda);
  log.add("codebook_update");
  return cudaGetLastError();
}

}  // namespace avq
