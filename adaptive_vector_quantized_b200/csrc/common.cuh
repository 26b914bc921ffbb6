// Device helpers shared by the AVQ kernels: element loads/stores for the two
// supported element types and small warp utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace avq {

typedef __nv_bfloat16 bf16;

// Error bits recorded in the per-device error word.
enum : unsigned int {
  kErrTimeout = 1u,   // a bounded wait ran out
  kErrBounds = 2u,    // a debug bounds check refused an access
  kErrInternal = 4u,  // an impossible state (e.g. a TMEM allocation failure)
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// bf16 pair x bf16 pair accumulated into fp32, the low halves first: the
// products of two bf16 values are exact in fp32, so this equals two fmaf on
// the values converted to fp32 (two roundings).
__device__ __forceinline__ float fma_bf16x2(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t.reg .f32 t;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 t, a0, b0, %3;\n\t"
      "fma.rn.f32.bf16 %0, a1, b1, t;\n\t}"
      : "=f"(d)
      : "r"(a), "r"(b), "f"(c));
  return d;
}

// 8 consecutive elements -> fp32 (p must be 16-byte aligned).
__device__ __forceinline__ void load8(const float* p, float* o) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const bf16* p, float* o) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  o[0] = bf16_lo(u.x); o[1] = bf16_hi(u.x);
  o[2] = bf16_lo(u.y); o[3] = bf16_hi(u.y);
  o[4] = bf16_lo(u.z); o[5] = bf16_hi(u.z);
  o[6] = bf16_lo(u.w); o[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;  // one paired conversion, round to nearest even; `lo` in the low half
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 8 fp32 -> 8 consecutive elements (16-byte aligned destination).
__device__ __forceinline__ void store8(float* p, const float* v) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(bf16* p, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

// E consecutive elements (E in {2, 4}) -> fp32, naturally aligned.
template <int E>
__device__ __forceinline__ void loadE(const float* p, float* o) {
  if constexpr (E == 2) {
    const float2 a = __ldg(reinterpret_cast<const float2*>(p));
    o[0] = a.x; o[1] = a.y;
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  }
}
template <int E>
__device__ __forceinline__ void loadE(const bf16* p, float* o) {
  if constexpr (E == 2) {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    o[0] = bf16_lo(u); o[1] = bf16_hi(u);
  } else {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    o[0] = bf16_lo(u.x); o[1] = bf16_hi(u.x);
    o[2] = bf16_lo(u.y); o[3] = bf16_hi(u.y);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Key counts n of Eq. 3 for one key per lane: +1 for its parent, +1 for its
// child when it moved.  Lanes with equal codes are merged before the atomic.
// Must be called by all 32 lanes of the warp.
__device__ __forceinline__ void count_codes(int32_t* counts, int code, bool valid, int M0, int C) {
  const int lane = threadIdx.x & 31;
  const int par = code < M0 ? code : (code - M0) / (C > 0 ? C : 1);
  const int pkey = valid ? par : -1 - lane;
  const unsigned peers_p = __match_any_sync(0xffffffffu, pkey);
  if (valid && lane == __ffs(peers_p) - 1) atomicAdd(counts + par, __popc(peers_p));
  const bool moved = valid && code >= M0;
  const int ckey = moved ? code : -1 - lane;
  const unsigned peers_c = __match_any_sync(0xffffffffu, ckey);
  if (moved && lane == __ffs(peers_c) - 1) atomicAdd(counts + code, __popc(peers_c));
}

// The same for a caller that already knows the key's parent `par`.
__device__ __forceinline__ void count_codes_par(int32_t* counts, int par, int code, bool valid, int M0) {
  const int lane = threadIdx.x & 31;
  const int pkey = valid ? par : -1 - lane;
  const unsigned peers_p = __match_any_sync(0xffffffffu, pkey);
  if (valid && lane == __ffs(peers_p) - 1) atomicAdd(counts + par, __popc(peers_p));
  const bool moved = valid && code >= M0;
  const int ckey = moved ? code : -1 - lane;
  const unsigned peers_c = __match_any_sync(0xffffffffu, ckey);
  if (moved && lane == __ffs(peers_c) - 1) atomicAdd(counts + code, __popc(peers_c));
}

// Vector reduction into global memory (sm_90+): four fp32 adds in one op.
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Programmatic dependent launch.  A kernel launched with launch_after may
// start while the previous kernel on its stream is still finishing; it must
// execute grid_dependency_wait() before it reads anything that kernel (or any
// earlier work on the stream) wrote, and may do independent set-up before.
// allow_dependents() lets the next such kernel be scheduled before this one
// ends (it still waits for this one's completion at its own
// grid_dependency_wait()).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace avq
