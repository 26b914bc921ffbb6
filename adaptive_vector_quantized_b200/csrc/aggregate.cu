// Stage 1, aggregation ("AVQ-Attention: Adaptive Vector-Quantized Attention",
// Sec. 4.2, the aggregation of Algorithm 1; Eq. 3).
//
// Given every key's final code, each key adds its value to its parent, and to
// its child when it moved to one.  Parents therefore hold their whole
// cluster, children only the keys closer to them than to the parent.  The
// key counts n of Eq. 3 come either from the assignment kernels or, for the
// warpgroup tensor-core assignment, from the same streaming pass (each run
// adds its length to its code) followed by the same upward pass as the sums.
//
// Streaming variant: runs of equal codes are summed in registers and added to
// the statistics with global vector reductions; see aggregate_stream_kernel.
//
// Deterministic variant: keys are stably sorted by (parent, child) with a
// counting sort over fixed 1024-key chunks, each segment is summed in key
// order by one warp, and parent totals are formed as stay + children in a
// fixed order.  Nothing depends on the grid or the GPU's size.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace avq {

namespace {

// Streaming variant (the default), in two steps.  First every key's value is
// added to its final code only (the child if it moved, else the parent):
// every warp owns a contiguous range of keys of one head (so runs of equal
// codes stay long), lanes cover the head dimension, a warp ballot per 32-key
// group marks where runs start, and the keys are walked in sub-batches of
// eight (one coalesced row load per key, the next sub-batch in flight while
// the current one is added) whose per-key work is a bit test and the adds,
// into two partial sums per run.  A finished run is
// added to the global value sums (L2 resident) with one vector reduction per
// lane (and, when `counts` is given, lane 0 adds the run's length to its
// code's count).  Then each parent adds its children's sums (and counts) to
// its own, which makes it the sum over its whole cluster (Eq. 3).
constexpr int kStreamThreads = 256;

// One lane's E consecutive elements of a value row, as loaded.
template <typename T, int E>
struct Frag;
template <>
struct Frag<bf16, 2> {
  using R = uint32_t;
  __device__ __forceinline__ static R load(const bf16* p) { return __ldg(reinterpret_cast<const unsigned*>(p)); }
  __device__ __forceinline__ static void unpack(R r, float* o) { o[0] = bf16_lo(r); o[1] = bf16_hi(r); }
};
template <>
struct Frag<bf16, 4> {
  using R = uint2;
  __device__ __forceinline__ static R load(const bf16* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ static void unpack(R r, float* o) {
    o[0] = bf16_lo(r.x); o[1] = bf16_hi(r.x); o[2] = bf16_lo(r.y); o[3] = bf16_hi(r.y);
  }
};
template <>
struct Frag<float, 2> {
  using R = float2;
  __device__ __forceinline__ static R load(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
  __device__ __forceinline__ static void unpack(R r, float* o) { o[0] = r.x; o[1] = r.y; }
};
template <>
struct Frag<float, 4> {
  using R = float4;
  __device__ __forceinline__ static R load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ __forceinline__ static void unpack(R r, float* o) { o[0] = r.x; o[1] = r.y; o[2] = r.z; o[3] = r.w; }
};

template <int E>
__device__ __forceinline__ void flush_sum(float* vsum, int code, const float* acc, int lane, int D) {
  float* row = vsum + (size_t)code * D + lane * E;
  if constexpr (E == 2) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(row), "f"(acc[0]), "f"(acc[1]) : "memory");
  } else {
    red_add_v4(row, acc[0], acc[1], acc[2], acc[3]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kStreamThreads) aggregate_stream_kernel(
    const T* __restrict__ V, const int32_t* __restrict__ assign, float* __restrict__ vsum,
    int32_t* __restrict__ counts, int BH, int N, int Mt, int keys_per_warp) {
  constexpr int E = D / 32;
  using F = Frag<T, E>;
  grid_dependency_wait();  // codes (and zeroed sums) of the launches before
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (kStreamThreads / 32) + (threadIdx.x >> 5);
  const int warps_per_head = (N + keys_per_warp - 1) / keys_per_warp;
  const int bh = gw / warps_per_head;
  const int j0 = (gw % warps_per_head) * keys_per_warp;
  const int j1 = min(N, j0 + keys_per_warp);
  if (bh >= BH || j0 >= j1) return;
  float* vs = vsum + (size_t)bh * Mt * D;
  const T* vb = V + (size_t)bh * N * D + lane * E;
  const int32_t* asg = assign + (size_t)bh * N;
  int32_t* cn = counts ? counts + (size_t)bh * Mt : nullptr;

  // two partial sums per run (even and odd keys of a group) halve the chain of
  // dependent adds; they are combined when the run is flushed
  float acc[2][E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[0][e] = acc[1][e] = 0.f;
  int cur = -1, run0 = j0;  // the open run's code and first key
  auto flush = [&](int end) {  // the open run ends before key `end`
    float t[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      t[e] = acc[0][e] + acc[1][e];
      acc[0][e] = acc[1][e] = 0.f;
    }
    flush_sum<E>(vs, cur, t, lane, D);
    if (cn && lane == 0) atomicAdd(cn + cur, end - run0);
  };
  int code_next = j0 + lane < j1 ? __ldg(asg + j0 + lane) : -1;
  for (int g = j0; g < j1; g += 32) {
    const int code = code_next;
    code_next = g + 32 + lane < j1 ? __ldg(asg + g + 32 + lane) : -1;
    const int prevc = __shfl_up_sync(0xffffffffu, code, 1);
    const int nlive = __popc(__ballot_sync(0xffffffffu, code >= 0));
    // run starts relative to the previous key (lane 0 compares with the open run)
    const unsigned newR = __ballot_sync(0xffffffffu, code >= 0 && (lane == 0 ? code != cur : prevc != code));
    // keys in sub-batches of 8: the next sub-batch's rows are loaded while the
    // current one is walked (16 rows in flight per warp, few registers); a
    // full group of 32 keys takes a copy of the walk without per-key bounds
    auto walk = [&](auto full_t) {
      constexpr bool kFull = decltype(full_t)::value;
      const int n = kFull ? 32 : nlive;
      const T* rows = vb + (size_t)g * D;
      typename F::R raw[8], nxt[8];
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (kFull || b < n) raw[b] = F::load(rows + (size_t)b * D);
#pragma unroll 1
      for (int b0 = 0; b0 < n; b0 += 8) {
        const bool more = b0 + 8 < n;
#pragma unroll
        for (int b = 0; b < 8; ++b)
          if (kFull ? more : b0 + 8 + b < n) nxt[b] = F::load(rows + (size_t)(b0 + 8 + b) * D);
        const unsigned starts = (newR >> b0) & 0xffu;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const int u = b0 + b;
          if (kFull || u < n) {
            float v[E];
            F::unpack(raw[b], v);
            if ((starts >> b) & 1u) {
              if (cur >= 0) flush(g + u);
              cur = __shfl_sync(0xffffffffu, code, u);
              run0 = g + u;
            }
#pragma unroll
            for (int e = 0; e < E; ++e) acc[b & 1][e] += v[e];
          }
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) raw[b] = nxt[b];
      }
    };
    if (nlive == 32)
      walk(std::true_type{});
    else
      walk(std::false_type{});
  }
  if (cur >= 0) flush(j1);
}

// Nodes hold their whole subtree: add the sums of the n nodes' children
// (keys that moved on) to each node's own (keys that stopped there), children
// in index order.  Node i of the level starting at code `lo` has its C
// children at codes lo2 + i*C .. lo2 + i*C + C - 1 (for a two-level tree:
// lo = 0, n = M0, lo2 = M0).
__global__ void __launch_bounds__(256) aggregate_parents_kernel(float* __restrict__ vsum,
                                                               int32_t* __restrict__ counts, int BH, int Mt,
                                                               int lo, int n, int lo2, int C, int D) {
  grid_dependency_wait();  // the streamed sums and counts
  const long long total = (long long)BH * n * D;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < total;
       u += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(u % D);
    const long long bp = u / D;
    const int p = (int)(bp % n);
    float* vs = vsum + (bp / n) * (long long)Mt * D;
    float s = vs[(size_t)(lo + p) * D + t];
    for (int c = 0; c < C; ++c) s += vs[(size_t)(lo2 + p * C + c) * D + t];
    vs[(size_t)(lo + p) * D + t] = s;
    if (counts && t == 0) {
      int32_t* ns = counts + (bp / n) * (long long)Mt;
      int k = ns[lo + p];
      for (int c = 0; c < C; ++c) k += ns[lo2 + p * C + c];
      ns[lo + p] = k;
    }
  }
}

// ---- deterministic variant ------------------------------------------------
constexpr int kDetChunk = 1024;  // keys per sort chunk (fixed: independent of the GPU)
constexpr int kDetWarps = 4;     // chunks per CTA

__device__ __forceinline__ int sort_bin(int code, int M0, int C) {
  // parent*(C+1) + 0 for keys that stay at the parent, + 1 + c for child c
  if (code < M0) return code * (C + 1);
  const int r = code - M0;
  const int p = r / C;
  return p * (C + 1) + 1 + (r - p * C);
}

// hist[bh][bin][chunk]: keys of `chunk` that fall in `bin`.
__global__ void __launch_bounds__(kDetWarps * 32) det_hist_kernel(const int32_t* __restrict__ assign,
                                                                  int* __restrict__ hist, int N,
                                                                  int M0, int C, int nch) {
  extern __shared__ int hs[];  // [kDetWarps][Mt]
  const int Mt = M0 * (1 + C);
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* h = hs + warp * Mt;
  for (int i = lane; i < Mt; i += 32) h[i] = 0;
  __syncwarp();
  const int ch = blockIdx.x * kDetWarps + warp;
  if (ch < nch) {
    const int j0 = ch * kDetChunk, j1 = min(N, j0 + kDetChunk);
    for (int j = j0 + lane; j < j1; j += 32) atomicAdd(h + sort_bin(assign[(size_t)bh * N + j], M0, C), 1);
    __syncwarp();
    int* out = hist + (size_t)bh * Mt * nch;
    for (int b = lane; b < Mt; b += 32) out[(size_t)b * nch + ch] = h[b];
  }
}

// In place exclusive scan of hist[bh][*] (bin-major, then chunk): one CTA per head.
__global__ void __launch_bounds__(1024) det_scan_kernel(int* __restrict__ hist, int total) {
  __shared__ int part[1024];
  int* h = hist + (size_t)blockIdx.x * total;
  const int per = (total + blockDim.x - 1) / blockDim.x;
  const int s0 = threadIdx.x * per, s1 = min(total, s0 + per);
  int sum = 0;
  for (int i = s0; i < s1; ++i) sum += h[i];
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // Hillis-Steele inclusive scan
    const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = threadIdx.x ? part[threadIdx.x - 1] : 0;
  for (int i = s0; i < s1; ++i) {
    const int c = h[i];
    h[i] = run;
    run += c;
  }
}

// Stable scatter of key indices into sorted order (one warp per chunk).
__global__ void __launch_bounds__(kDetWarps * 32) det_scatter_kernel(
    const int32_t* __restrict__ assign, const int* __restrict__ offs, int* __restrict__ order,
    int N, int M0, int C, int nch) {
  extern __shared__ int cs[];  // [kDetWarps][Mt] running positions
  const int Mt = M0 * (1 + C);
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ch = blockIdx.x * kDetWarps + warp;
  if (ch >= nch) return;
  int* pos = cs + warp * Mt;
  const int* o = offs + (size_t)bh * Mt * nch;
  for (int b = lane; b < Mt; b += 32) pos[b] = o[(size_t)b * nch + ch];
  __syncwarp();
  const int j0 = ch * kDetChunk, j1 = min(N, j0 + kDetChunk);
  int* ord = order + (size_t)bh * N;
  for (int jb = j0; jb < j1; jb += 32) {
    const int j = jb + lane;
    const bool ok = j < j1;
    const int bin = ok ? sort_bin(assign[(size_t)bh * N + j], M0, C) : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int base = ok ? pos[bin] : 0;
    __syncwarp();
    if (ok) {
      ord[base + rank] = j;
      if (rank == 0) pos[bin] = base + __popc(peers);
    }
    __syncwarp();
  }
}

// One warp per (bh, bin): sum of the segment's value rows in sorted (= key) order.
template <typename T, int D>
__global__ void __launch_bounds__(256) det_segsum_kernel(const T* __restrict__ V,
                                                         const int* __restrict__ offs,
                                                         const int* __restrict__ order,
                                                         float* __restrict__ seg, int N, int Mt,
                                                         int nch) {
  constexpr int E = D / 32;
  const int bh = blockIdx.y;
  const int bin = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bin >= Mt) return;
  const int* o = offs + (size_t)bh * Mt * nch;
  const int start = o[(size_t)bin * nch];
  const int end = bin + 1 < Mt ? o[(size_t)(bin + 1) * nch] : N;
  const int* ord = order + (size_t)bh * N;
  const T* vb = V + (size_t)bh * N * D + lane * E;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int i = start; i < end; i += 8) {
    float v[8][E];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (i + u < end) loadE<E>(vb + (size_t)__ldg(ord + i + u) * D, v[u]);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (i + u < end) {
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += v[u][e];
      }
    }
  }
  float* out = seg + ((size_t)bh * Mt + bin) * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = acc[e];
}

// vsum/counts from the segment sums: child (p,c) = segment (p, 1+c); parent p =
// stay segment + children segments in child order.
__global__ void det_combine_kernel(const float* __restrict__ seg, const int* __restrict__ offs,
                                   float* __restrict__ vsum, int32_t* __restrict__ counts, int N,
                                   int M0, int C, int D, int nch) {
  const int bh = blockIdx.y;
  const int Mt = M0 * (1 + C);
  const int p = blockIdx.x;
  const int* o = offs + (size_t)bh * Mt * nch;
  const float* sg = seg + (size_t)bh * Mt * D;
  float* vs = vsum + (size_t)bh * Mt * D;
  int32_t* ns = counts + (size_t)bh * Mt;
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    const int b0 = p * (C + 1);
    float tot = sg[(size_t)b0 * D + t];
    for (int c = 0; c < C; ++c) {
      const float v = sg[(size_t)(b0 + 1 + c) * D + t];
      tot += v;
      vs[(size_t)(M0 + p * C + c) * D + t] = v;
    }
    vs[(size_t)p * D + t] = tot;
  }
  if (threadIdx.x == 0) {
    auto seg_len = [&](int bin) {
      const int s = o[(size_t)bin * nch];
      const int e = bin + 1 < Mt ? o[(size_t)(bin + 1) * nch] : N;
      return e - s;
    };
    const int b0 = p * (C + 1);
    int tot = seg_len(b0);
    for (int c = 0; c < C; ++c) {
      const int n = seg_len(b0 + 1 + c);
      ns[M0 + p * C + c] = n;
      tot += n;
    }
    ns[p] = tot;
  }
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t aggregate_det_workspace(const Shape& s) {
  const size_t nch = (s.N + kDetChunk - 1) / kDetChunk;
  const size_t hist = align256((size_t)s.BH() * s.Mt() * nch * sizeof(int));
  const size_t order = align256((size_t)s.BH() * s.N * sizeof(int));
  const size_t seg = align256((size_t)s.BH() * s.Mt() * s.d * sizeof(float));
  return hist + order + seg;
}

cudaError_t launch_aggregate(const Shape& s, avq_dtype dt, const void* V, const int32_t* assign,
                             float* vsum, int32_t* counts, unsigned int* err, cudaStream_t st,
                             LaunchLog& log, bool vsum_zeroed, bool depth3, bool count) {
  cudaError_t e = cudaSuccess;
  const int Mt = depth3 ? s.M0 + s.M0 * s.C + s.M0 * s.C * s.C : s.Mt();
  if (!vsum_zeroed) {
    e = cudaMemsetAsync(vsum, 0, (size_t)s.BH() * Mt * s.d * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  int32_t* cnt = count ? counts : nullptr;  // counts left to this pass (zeroed by the caller)
  const int sms = num_sms();
  // grid sized for about 32 resident warps per SM, each a contiguous multiple of 32 keys
  const long long total_keys = (long long)s.BH() * s.N;
  const long long want_warps = (long long)sms * 32;
  int kpw = (int)((total_keys + want_warps - 1) / want_warps);
  kpw = ((kpw + 31) / 32) * 32;
  if (kpw < 32) kpw = 32;
  const long long warps = (long long)s.BH() * ((s.N + kpw - 1) / kpw);
  const unsigned blocks = (unsigned)((warps + (kStreamThreads / 32) - 1) / (kStreamThreads / 32));
#define AVQ_STREAM(T, D)                                                                          \
  e = launch_after(aggregate_stream_kernel<T, D>, dim3(blocks), dim3(kStreamThreads), 0, st, (const T*)V, \
                   assign, vsum, cnt, s.BH(), s.N, Mt, kpw)
  if (dt == AVQ_F32) {
    if (s.d == 64) AVQ_STREAM(float, 64); else AVQ_STREAM(float, 128);
  } else {
    if (s.d == 64) AVQ_STREAM(bf16, 64); else AVQ_STREAM(bf16, 128);
  }
#undef AVQ_STREAM
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (s.C > 0) {
    const long long work = (long long)s.BH() * s.M0 * s.d;
    const int pb = (int)std::min<long long>((work + 255) / 256, (long long)sms * 8);
    if (depth3) {  // children first take their grandchildren's sums
      const long long work3 = (long long)s.BH() * s.M0 * s.C * s.d;
      const int pb3 = (int)std::min<long long>((work3 + 255) / 256, (long long)sms * 8);
      e = launch_after(aggregate_parents_kernel, dim3(pb3), dim3(256), 0, st, vsum, cnt, s.BH(), Mt, s.M0,
                       s.M0 * s.C, s.M0 + s.M0 * s.C, s.C, s.d);
      if (e != cudaSuccess) return e;
    }
    e = launch_after(aggregate_parents_kernel, dim3(pb), dim3(256), 0, st, vsum, cnt, s.BH(), Mt, 0, s.M0, s.M0,
                     s.C, s.d);
    if (e != cudaSuccess) return e;
  }
  log.add(s.C > 0 ? "aggregate_stream aggregate_parents" : "aggregate_stream");
  (void)err;
  return cudaGetLastError();
}

cudaError_t launch_aggregate_det(const Shape& s, avq_dtype dt, const void* V,
                                 const int32_t* assign, float* vsum, int32_t* counts, void* ws,
                                 cudaStream_t st, LaunchLog& log) {
  const int nch = (s.N + kDetChunk - 1) / kDetChunk;
  const int Mt = s.Mt();
  char* w = static_cast<char*>(ws);
  int* hist = reinterpret_cast<int*>(w);
  w += align256((size_t)s.BH() * Mt * nch * sizeof(int));
  int* order = reinterpret_cast<int*>(w);
  w += align256((size_t)s.BH() * s.N * sizeof(int));
  float* seg = reinterpret_cast<float*>(w);

  const size_t hsmem = (size_t)kDetWarps * Mt * sizeof(int);
  cudaError_t e;
  if (hsmem > 48 * 1024) {
    e = cudaFuncSetAttribute(det_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(det_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem);
    if (e != cudaSuccess) return e;
  }
  dim3 g1((nch + kDetWarps - 1) / kDetWarps, s.BH());
  det_hist_kernel<<<g1, kDetWarps * 32, hsmem, st>>>(assign, hist, s.N, s.M0, s.C, nch);
  det_scan_kernel<<<s.BH(), 1024, 0, st>>>(hist, Mt * nch);
  det_scatter_kernel<<<g1, kDetWarps * 32, hsmem, st>>>(assign, hist, order, s.N, s.M0, s.C, nch);
  dim3 g4((Mt + 7) / 8, s.BH());
  if (dt == AVQ_F32) {
    if (s.d == 64) det_segsum_kernel<float, 64><<<g4, 256, 0, st>>>((const float*)V, hist, order, seg, s.N, Mt, nch);
    else det_segsum_kernel<float, 128><<<g4, 256, 0, st>>>((const float*)V, hist, order, seg, s.N, Mt, nch);
  } else {
    if (s.d == 64) det_segsum_kernel<bf16, 64><<<g4, 256, 0, st>>>((const bf16*)V, hist, order, seg, s.N, Mt, nch);
    else det_segsum_kernel<bf16, 128><<<g4, 256, 0, st>>>((const bf16*)V, hist, order, seg, s.N, Mt, nch);
  }
  det_combine_kernel<<<dim3(s.M0, s.BH()), 128, 0, st>>>(seg, hist, vsum, counts, s.N, s.M0, s.C,
                                                         s.d, nch);
  log.add("det_hist det_scan det_scatter det_segsum det_combine");
  return cudaGetLastError();
}

}  // namespace avq
