// A depth-3 tree on the CUDA cores: the "deeper hierarchies" that the
// conclusion of "AVQ-Attention: Adaptive Vector-Quantized Attention" (Sec. 6)
// names as the next step, with Algorithms 1 and 2 applied one level further
// down.  Every child has C grandchildren and is their mean, as every parent
// is the mean of its children (Eq. 5).  Codes per head: parents [0, M0),
// child (m, c) at M0 + m*C + c, grandchild (m, c, g) at
// M0 + M0*C + (m*C + c)*C + g.
//
// Stage 1 (assign3_simt_kernel): one thread per key, nearest parent (first
// minimum), nearest child of it taken when strictly closer, nearest
// grandchild of that child taken when strictly closer than the child.  The
// key counts at every level it reached (Eq. 3); the value sums are formed by
// the streaming aggregation plus two upward passes.
//
// Stage 2 (attention3_simt_kernel): one CTA per (head, query block), one
// thread per query row.  The parent pass and the child refinement of the
// top-P parents follow Algorithm 2; then each of the P*C refined children
// gets an importance w_c(I) = sum_i exp(s_ic - m_i) n_c / z_i with the
// logits, maximum and denominator after the child refinement (Eq. 7, one
// level down); the top-P2 of them (descending, ties to the lower child code)
// are refined with their grandchildren: the child's logit is the mean of its
// grandchildren's (Eq. 8), dA = exp(s_g - m) - exp(s_c - m) (Eq. 9), zero for
// empty grandchildren, merged with the online maximum.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace avq {

namespace {

template <typename T, int D>
__device__ __forceinline__ float sqdist3(const float* k, const T* c) {
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
__device__ __forceinline__ float dot3(const float* q, const T* c) {
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

// Counts at every level a key reached; lanes with equal codes are merged
// before each atomic.  All 32 lanes of the warp call it.
__device__ __forceinline__ void count_level(int32_t* counts, int code, bool on) {
  const int lane = threadIdx.x & 31;
  const int key = on ? code : -1 - lane;
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  if (on && lane == __ffs(peers) - 1) atomicAdd(counts + code, __popc(peers));
}

template <typename T, int D>
__global__ void __launch_bounds__(128) assign3_simt_kernel(const T* __restrict__ K, const T* __restrict__ parents,
                                                           const T* __restrict__ children,
                                                           const T* __restrict__ grandchildren,
                                                           int32_t* __restrict__ assign,
                                                           int32_t* __restrict__ counts, int H, int N, int M0,
                                                           int C) {
  const int bh = blockIdx.y, h = bh % H;
  const int M1 = M0 * C, Mt = M0 + M1 + M1 * C;
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
    const float dm = sqdist3<T, D>(k, par + (size_t)m * D);
    if (dm < best) {
      best = dm;
      a = m;
    }
  }
  // nearest child of a, taken when strictly closer than a
  const T* ch = children + ((size_t)h * M1 + (size_t)a * C) * D;
  float dch = __int_as_float(0x7f800000);
  int cs = 0;
  for (int c = 0; c < C; ++c) {
    const float dc = sqdist3<T, D>(k, ch + (size_t)c * D);
    if (dc < dch) {
      dch = dc;
      cs = c;
    }
  }
  const bool moved = dch < best;
  const int cidx = a * C + cs;  // child index m*C + c
  // nearest grandchild of that child, taken when strictly closer than the child
  bool moved2 = false;
  int gs = 0;
  if (moved) {
    const T* gc = grandchildren + ((size_t)h * M1 * C + (size_t)cidx * C) * D;
    float dg = __int_as_float(0x7f800000);
    for (int g = 0; g < C; ++g) {
      const float dd = sqdist3<T, D>(k, gc + (size_t)g * D);
      if (dd < dg) {
        dg = dd;
        gs = g;
      }
    }
    moved2 = dg < dch;
  }
  const int code_c = M0 + cidx, code_g = M0 + M1 + cidx * C + gs;
  if (valid) assign[(size_t)bh * N + j] = moved2 ? code_g : moved ? code_c : a;
  int32_t* cnt = counts + (size_t)bh * Mt;
  count_level(cnt, a, valid);
  count_level(cnt, code_c, valid && moved);
  count_level(cnt, code_g, valid && moved2);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) attention3_simt_kernel(
    const T* __restrict__ Q, const T* __restrict__ parents, const T* __restrict__ children,
    const T* __restrict__ grandchildren, const float* __restrict__ vsum, const int32_t* __restrict__ counts,
    int H, int N, int M0, int C, int P, int P2, int block, float scale, T* __restrict__ O,
    int32_t* __restrict__ sel, int32_t* __restrict__ sel2, float* __restrict__ importance,
    float* __restrict__ importance2) {
  extern __shared__ __align__(16) float sm[];
  const int M1 = M0 * C, Mt = M0 + M1 + M1 * C, NC = P * C;
  float* qs = sm;                                   // [block][D+1]
  float* nf = qs + (size_t)block * (D + 1);         // [Mt] counts as float
  float* w = nf + Mt;                               // [M0] parents' importance
  float* w2 = w + M0;                               // [P*C] refined children's importance
  int* ssel = reinterpret_cast<int*>(w2 + (NC > 0 ? NC : 1));  // [P] parents
  int* ssel2 = ssel + (P > 0 ? P : 1);                         // [P2] child codes
  const int bh = blockIdx.y, h = bh % H, blk = blockIdx.x, nblk = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int i = blk * block + tid;
  const bool valid = tid < block && i < N;
  const float NEG_INF = __int_as_float(0xff800000);

  for (int idx = tid; idx < block * (D / 8); idx += blockDim.x) {
    const int r = idx / (D / 8), t = (idx % (D / 8)) * 8;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (blk * block + r < N) load8(Q + ((size_t)bh * N + blk * block + r) * D + t, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) qs[r * (D + 1) + t + e] = v[e];
  }
  for (int r = tid; r < Mt; r += blockDim.x) nf[r] = (float)counts[(size_t)bh * Mt + r];
  for (int r = tid; r < M0; r += blockDim.x) w[r] = 0.f;
  for (int r = tid; r < NC; r += blockDim.x) w2[r] = 0.f;
  __syncthreads();

  const float* qr = qs + (size_t)(tid < block ? tid : 0) * (D + 1);
  // bf16: the row's query as bf16 pairs in registers, multiplied with the
  // codewords by fma.rn.f32.bf16 (the bf16 products are exact in fp32); fp32:
  // the row in shared memory
  constexpr bool kBf16 = std::is_same<T, bf16>::value;
  uint32_t qv[kBf16 ? D / 2 : 1];
  if constexpr (kBf16) {
    const uint4* qp = reinterpret_cast<const uint4*>(Q + ((size_t)bh * N + (valid ? i : blk * block)) * D);
#pragma unroll
    for (int t = 0; t < D / 8; ++t) {
      const uint4 u = __ldg(qp + t);
      qv[4 * t] = u.x;
      qv[4 * t + 1] = u.y;
      qv[4 * t + 2] = u.z;
      qv[4 * t + 3] = u.w;
    }
  }
  auto qdot = [&](const T* c) -> float {
    if constexpr (kBf16) {
      // four partial sums (dims t, t+1 mod 8 in one, ...) shorten the chain of
      // dependent adds; combined in a fixed order
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t < D; t += 8) {
        const uint4 cv = __ldg(reinterpret_cast<const uint4*>(c + t));
        acc[0] = fma_bf16x2(qv[t / 2], cv.x, acc[0]);
        acc[1] = fma_bf16x2(qv[t / 2 + 1], cv.y, acc[1]);
        acc[2] = fma_bf16x2(qv[t / 2 + 2], cv.z, acc[2]);
        acc[3] = fma_bf16x2(qv[t / 2 + 3], cv.w, acc[3]);
      }
      return (acc[0] + acc[1]) + (acc[2] + acc[3]);
    } else {
      return dot3<T, D>(qr, c);
    }
  };
  const T* par = parents + (size_t)h * M0 * D;
  const T* chd = children + (size_t)h * M1 * D;
  const T* gcd = grandchildren + (size_t)h * M1 * C * D;
  const float* vs = vsum + (size_t)bh * Mt * D;
  float x[D];
#pragma unroll
  for (int t = 0; t < D; ++t) x[t] = 0.f;
  auto add_row = [&](float a, const float* v) {
#pragma unroll
    for (int t = 0; t < D; t += 4) {
      const float4 v4 = __ldg(reinterpret_cast<const float4*>(v + t));
      x[t] = fmaf(a, v4.x, x[t]);
      x[t + 1] = fmaf(a, v4.y, x[t + 1]);
      x[t + 2] = fmaf(a, v4.z, x[t + 2]);
      x[t + 3] = fmaf(a, v4.w, x[t + 3]);
    }
  };

  // parents: masked max (Eq. 18) and denominator first, then A, x and the
  // importance with the exact denominator (Eqs. 6-7)
  float m = NEG_INF, z = 0.f;
  for (int j = 0; j < M0; ++j) {
    const float nj = nf[j];
    if (nj > 0.f) {
      const float s = scale * qdot(par + (size_t)j * D);
      if (s > m) {
        z = z * expf(m - s) + nj;
        m = s;
      } else {
        z = fmaf(nj, expf(s - m), z);
      }
    }
  }
  {
    const float rz = 1.f / z;
    for (int j = 0; j < M0; ++j) {
      const float nj = nf[j];
      float a = 0.f;
      if (nj > 0.f) {
        a = expf(scale * qdot(par + (size_t)j * D) - m);
        add_row(a, vs + (size_t)j * D);
      }
      const float col = warp_sum(valid ? a * nj * rz : 0.f);
      if (lane == 0 && col != 0.f) atomicAdd(w + j, col);
    }
  }
  __syncthreads();
  // top-P parents (descending, ties to the lower index), one warp
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

  // refinement of one node with its C sub-codes: logits, online max merge,
  // the node's logit as the mean of its sub-codes' (Eq. 8), dA (Eq. 9)
  auto refine = [&](const T* sub, int code0) {
    float sc[8];
    float mp = m, sp = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < C) {
        sc[c] = scale * qdot(sub + (size_t)c * D);
        sp += sc[c];
        if (nf[code0 + c] > 0.f && sc[c] > mp) mp = sc[c];
      }
    }
    sp = sp / (float)C;
    const float f = expf(m - mp);
    z *= f;
#pragma unroll
    for (int t = 0; t < D; ++t) x[t] *= f;
    m = mp;
    const float ap = expf(sp - m);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < C) {
        const float nc = nf[code0 + c];
        if (nc > 0.f) {
          const float da = expf(sc[c] - m) - ap;
          add_row(da, vs + (size_t)(code0 + c) * D);
          z = fmaf(da, nc, z);
        }
      }
    }
  };
  for (int r = 0; r < P; ++r) {
    const int p = ssel[r];
    refine(chd + (size_t)p * C * D, M0 + p * C);
  }

  // the refined children's importance after the child refinement (also when
  // only reported)
  if (P2 > 0 || importance2 != nullptr) {
    const float rz = valid ? 1.f / z : 0.f;
    for (int u = 0; u < NC; ++u) {
      const int code = M0 + ssel[u / C] * C + (u % C);
      const float nc = nf[code];
      float a = 0.f;
      if (nc > 0.f) a = expf(scale * qdot(chd + (size_t)(code - M0) * D) - m);
      const float col = warp_sum(a * nc * rz);
      if (lane == 0 && col != 0.f) atomicAdd(w2 + u, col);
    }
    __syncthreads();
    // top-P2 children (descending, ties to the lower child code), one warp
    if (tid < 32) {
      for (int u = lane; u < NC; u += 32) {
        const float wu = w2[u];
        const int cu = ssel[u / C] * C + (u % C);
        int rank = 0;
        for (int v = 0; v < NC; ++v) {
          const float wv = w2[v];
          const int cv = ssel[v / C] * C + (v % C);
          rank += (wv > wu) || (wv == wu && cv < cu);
        }
        if (rank < P2) ssel2[rank] = M0 + cu;
        if (importance2) importance2[((size_t)bh * nblk + blk) * NC + u] = wu;
      }
      __syncwarp();
      if (sel2 && P2 > 0)
        for (int r = lane; r < P2; r += 32) sel2[((size_t)bh * nblk + blk) * P2 + r] = ssel2[r];
    }
    __syncthreads();
    for (int r = 0; r < P2; ++r) {
      const int cidx = ssel2[r] - M0;  // m*C + c
      refine(gcd + (size_t)cidx * C * D, M0 + M1 + cidx * C);
    }
  }
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

// Stage 1 of a depth-3 tree after the two-level tensor-core assignment:
// every key whose code is a child moves to that child's nearest grandchild
// when it is strictly closer (Algorithm 1, one level down; C = 8).  8 lanes
// per key, 4 keys per warp: lane s holds 16-byte chunks of the key, its child
// and the child's grandchildren (dims [s D/8, (s+1) D/8)), accumulates the 9
// partial dot products and squared norms in fp32 (bf16 x bf16 products) and
// sums them over the 8 lanes; distances |r|^2 - 2 k.r (|k|^2 is common), the
// first strict minimum among the grandchildren, moved only if strictly
// closer than the child.  Keys at a parent are left as they are.
template <int D>
__global__ void __launch_bounds__(256) assign3_grandchildren_kernel(const bf16* __restrict__ K,
                                                                    const bf16* __restrict__ children,
                                                                    const bf16* __restrict__ grandchildren,
                                                                    int32_t* __restrict__ assign, int BH,
                                                                    int H, int N, int M0) {
  constexpr int C = 8;
  constexpr int DL = D / 8;    // dims per lane
  constexpr int CHK = DL / 8;  // 16-byte chunks per lane and row
  const int M1 = M0 * C;
  const int lane = threadIdx.x & 31, sub = lane & 7, kq = lane >> 3;
  const long long total = (long long)BH * N;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long k0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4; k0 < total;
       k0 += warps * 4) {  // warp-uniform loop
    const long long key = k0 + kq;
    const int code = key < total ? assign[key] : -1;
    const bool moved = code >= M0 && code < M0 + M1;
    if (!__any_sync(0xffffffffu, moved)) continue;
    const int cl = moved ? code - M0 : 0;  // the child's index among the head's M0*C children
    const int h = (int)((moved ? key / N : 0) % H);
    const bf16* kr = K + (size_t)(moved ? key : 0) * D + sub * DL;
    const bf16* cr = children + ((size_t)h * M1 + cl) * D + sub * DL;
    const bf16* gr = grandchildren + ((size_t)h * M1 + cl) * C * D + sub * DL;
    float acc[1 + C], nrm[1 + C];
#pragma unroll
    for (int j = 0; j <= C; ++j) acc[j] = nrm[j] = 0.f;
    if (moved) {
#pragma unroll
      for (int q = 0; q < CHK; ++q) {
        const uint4 kv = __ldg(reinterpret_cast<const uint4*>(kr + q * 8));
        uint4 cv[1 + C];
        cv[0] = __ldg(reinterpret_cast<const uint4*>(cr + q * 8));
#pragma unroll
        for (int g = 0; g < C; ++g) cv[1 + g] = __ldg(reinterpret_cast<const uint4*>(gr + (size_t)g * D + q * 8));
#pragma unroll
        for (int j = 0; j <= C; ++j) {
          acc[j] = fma_bf16x2(kv.x, cv[j].x, acc[j]);
          acc[j] = fma_bf16x2(kv.y, cv[j].y, acc[j]);
          acc[j] = fma_bf16x2(kv.z, cv[j].z, acc[j]);
          acc[j] = fma_bf16x2(kv.w, cv[j].w, acc[j]);
          nrm[j] = fma_bf16x2(cv[j].x, cv[j].x, nrm[j]);
          nrm[j] = fma_bf16x2(cv[j].y, cv[j].y, nrm[j]);
          nrm[j] = fma_bf16x2(cv[j].z, cv[j].z, nrm[j]);
          nrm[j] = fma_bf16x2(cv[j].w, cv[j].w, nrm[j]);
        }
      }
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1)
#pragma unroll
      for (int j = 0; j <= C; ++j) {
        acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
        nrm[j] += __shfl_xor_sync(0xffffffffu, nrm[j], o);
      }
    if (moved && sub == 0) {
      const float dc = fmaf(-2.f, acc[0], nrm[0]);
      float dg = fmaf(-2.f, acc[1], nrm[1]);
      int gstar = 0;
#pragma unroll
      for (int g = 1; g < C; ++g) {
        const float d = fmaf(-2.f, acc[1 + g], nrm[1 + g]);
        if (d < dg) {
          dg = d;
          gstar = g;
        }
      }
      if (dg < dc) assign[key] = M0 + M1 + cl * C + gstar;
    }
  }
}

}  // namespace

cudaError_t launch_assign3_grandchildren(const Shape& s, const void* K, const void* children,
                                         const void* grandchildren, int32_t* assign, cudaStream_t st,
                                         LaunchLog& log) {
  const long long groups = ((long long)s.BH() * s.N + 3) / 4;  // 4 keys per warp
  const int blocks = (int)std::max<long long>(1, std::min<long long>((groups + 7) / 8, (long long)num_sms() * 16));
  if (s.d == 64)
    assign3_grandchildren_kernel<64><<<blocks, 256, 0, st>>>((const bf16*)K, (const bf16*)children,
                                                             (const bf16*)grandchildren, assign, s.BH(), s.H,
                                                             s.N, s.M0);
  else
    assign3_grandchildren_kernel<128><<<blocks, 256, 0, st>>>((const bf16*)K, (const bf16*)children,
                                                              (const bf16*)grandchildren, assign, s.BH(), s.H,
                                                              s.N, s.M0);
  log.add("assign3_grandchildren");
  return cudaGetLastError();
}

cudaError_t launch_assign3_simt(const Shape& s, avq_dtype dt, const void* K, const void* parents,
                                const void* children, const void* grandchildren, int32_t* assign,
                                int32_t* counts, cudaStream_t st, LaunchLog& log) {
  dim3 grid((s.N + 127) / 128, s.BH());
#define AVQ_A3(T, D)                                                                                   \
  assign3_simt_kernel<T, D><<<grid, 128, 0, st>>>((const T*)K, (const T*)parents, (const T*)children,  \
                                                  (const T*)grandchildren, assign, counts, s.H, s.N,   \
                                                  s.M0, s.C)
  if (dt == AVQ_F32) {
    if (s.d == 64) AVQ_A3(float, 64); else AVQ_A3(float, 128);
  } else {
    if (s.d == 64) AVQ_A3(bf16, 64); else AVQ_A3(bf16, 128);
  }
#undef AVQ_A3
  log.add("assign3_simt");
  return cudaGetLastError();
}

cudaError_t launch_attention3_simt(const Shape& s, avq_dtype dt, const void* Q, const void* parents,
                                   const void* children, const void* grandchildren, const float* vsum,
                                   const int32_t* counts, int P, int P2, int block, float scale, void* O,
                                   int32_t* sel, int32_t* sel2, float* importance, float* importance2,
                                   cudaStream_t st, LaunchLog& log) {
  const int nblk = (s.N + block - 1) / block;
  const int Mt = s.M0 + s.M0 * s.C + s.M0 * s.C * s.C;
  const int NC = P * s.C;
  dim3 grid(nblk, s.BH());
  const size_t smem = ((size_t)block * (s.d + 1) + Mt + s.M0 + (NC > 0 ? NC : 1) + (P > 0 ? P : 1) +
                       (P2 > 0 ? P2 : 1)) * sizeof(float);
  cudaError_t e;
#define AVQ_T3(T, D)                                                                                   \
  do {                                                                                                 \
    auto kern = attention3_simt_kernel<T, D>;                                                          \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);            \
    if (e != cudaSuccess) return e;                                                                    \
    kern<<<grid, 128, smem, st>>>((const T*)Q, (const T*)parents, (const T*)children,                  \
                                  (const T*)grandchildren, vsum, counts, s.H, s.N, s.M0, s.C, P, P2,   \
                                  block, scale, (T*)O, sel, sel2, importance, importance2);            \
  } while (0)
  if (dt == AVQ_F32) {
    if (s.d == 64) AVQ_T3(float, 64); else AVQ_T3(float, 128);
  } else {
    if (s.d == 64) AVQ_T3(bf16, 64); else AVQ_T3(bf16, 128);
  }
#undef AVQ_T3
  log.add("attention3_simt");
  return cudaGetLastError();
}

}  // namespace avq
