// Stage 1 assignment on the tcgen05 tensor cores ("AVQ-Attention: Adaptive
// Vector-Quantized Attention", Sec. 4.2, Algorithm 1: parent and child assignment).
//
// Persistent CTAs walk contiguous ranges of 128-key tiles.  Per tile:
//   K tile      TMA (128B swizzle) into a two-slot ring, the next tile in
//               flight while the current one is processed
//   parents     D = K P^T on tcgen05 into TMEM (M = 128 keys, N = M0);
//               thread r owns key r = TMEM lane r and takes the first
//               minimum of |p|^2 - 2 k.p over the parents (|k|^2 is the same
//               for every codeword of a key and is dropped)
//   children    the C = 8 children of every parent are in shared memory as
//               one swizzled atom each, so the children of two adjacent
//               parents form an N = 16 operand tile: one MMA per parent pair
//               that some key of the tile chose gives every key of the tile
//               its dot products with those 16 children (TMEM, in rounds of
//               16 pairs); each thread then loads the 8 columns of its own
//               parent (one TMEM load per distinct pair in its warp).  When
//               the children do not fit in shared memory they are read from
//               L2 and the dot products are bf16 x bf16 -> fp32 fused
//               multiply-adds on the CUDA cores.  Either way the key moves
//               to the first strictly smallest child only if it is strictly
//               closer than the parent
//   output      assign[key] = parent, or M0 + parent*C + child
// Codewords are first converted into the swizzled-atom image shared with
// the attention kernel (8 codes x 64 dims per 1024-byte atom) plus their
// squared norms in fp32.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace avq {

namespace {

constexpr int kKeys = 128;

struct AssignArgs {
  const bf16* cw;      // [H][Mt/8][KH][8][64] swizzled codeword atoms
  const float* norms;  // [H][Mt] squared norms
  int32_t* assign;     // [BH][N]
  int32_t* counts;     // [BH][Mt], accumulated (zeroed by the caller)
  unsigned int* err;
  int H, N, M0, C, nblk, ntiles, tiles_per_cta;
};

// bf16 pair x bf16 pair accumulated into fp32 (two exact products, two roundings).
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

template <int D, bool CH_SMEM>
struct AssignSmem {
  static constexpr int KH = D / 64;
  // parents image | children image (optional) | K ring [2] | norms | pair bits | barriers
  __host__ __device__ static size_t parents_bytes(int M0) { return (size_t)M0 * D * 2; }
  __host__ __device__ static size_t children_bytes(int M0, int C) { return CH_SMEM ? (size_t)M0 * C * D * 2 : 0; }
  __host__ __device__ static size_t ring_off(int M0, int C) { return parents_bytes(M0) + children_bytes(M0, C); }
  __host__ __device__ static size_t norms_off(int M0, int C) { return ring_off(M0, C) + 2 * kKeys * D * 2; }
  __host__ __device__ static size_t pairs_off(int M0, int C) {
    return (norms_off(M0, C) + (size_t)M0 * (1 + C) * 4 + 15) & ~(size_t)15;
  }
  __host__ __device__ static size_t bar_off(int M0, int C) { return pairs_off(M0, C) + 16; }
  __host__ __device__ static size_t total(int M0, int C) { return bar_off(M0, C) + 64; }
};

template <int D, bool CH_SMEM>
__global__ void __launch_bounds__(128) assign_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                                                        const AssignArgs a) {
  using S = AssignSmem<D, CH_SMEM>;
  constexpr int KH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int M0 = a.M0, C = a.C, Mt = M0 * (1 + C);
  uint8_t* sPar = sm;
  uint8_t* sCh = sm + S::parents_bytes(M0);
  uint8_t* sRing = sm + S::ring_off(M0, C);
  float* sNorm = reinterpret_cast<float*>(sm + S::norms_off(M0, C));
  uint32_t* sPairs = reinterpret_cast<uint32_t*>(sm + S::pairs_off(M0, C));  // 128-bit set of parent pairs
  uint64_t* bar_k = reinterpret_cast<uint64_t*>(sm + S::bar_off(M0, C));  // [2]
  uint64_t* bar_cb = bar_k + 2;
  uint64_t* bar_mma = bar_k + 3;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar_k + 4);
  int* sAbort = reinterpret_cast<int*>(bar_k + 4) + 1;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int t0 = blockIdx.x * a.tiles_per_cta;
  const int t1 = min(a.ntiles, t0 + a.tiles_per_cta);
  if (t0 >= t1) return;
  const uint32_t ncols = CH_SMEM ? 256u : (M0 <= 32 ? 32u : M0 <= 64 ? 64u : M0 <= 128 ? 128u : 256u);

  if (tid == 0) {
    tc::mbar_init(&bar_k[0], 1);
    tc::mbar_init(&bar_k[1], 1);
    tc::mbar_init(bar_cb, 1);
    tc::mbar_init(bar_mma, 1);
    tc::fence_mbar_init();
    *sAbort = 0;
    sPairs[0] = sPairs[1] = sPairs[2] = sPairs[3] = 0;
    tc::prefetch_tensormap(&kmap);
  }
  if (warp == 0) {
    tc::tmem_alloc(sTmem, ncols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  auto issue_k = [&](int t, int slot) {
    const int bh = t / a.nblk, blk = t % a.nblk;
    tc::mbar_arrive_expect_tx(&bar_k[slot], kKeys * D * 2);
#pragma unroll
    for (int kh = 0; kh < KH; ++kh)
      tc::tma_load_3d(sRing + slot * (kKeys * D * 2) + kh * (kKeys * 128), &kmap, kh * 64, blk * kKeys, bh,
                      &bar_k[slot]);
  };
  if (tid == 0) {
    issue_k(t0, 0);
    if (t0 + 1 < t1) issue_k(t0 + 1, 1);
  }

  const uint32_t idesc = tc::idesc_bf16(kKeys, M0, 0, 0);
  const uint32_t sParA = tc::smem_u32(sPar);
  uint32_t ph_cb = 0, ph_mma = 0;
  int cur_h = -1;
  const float INF = __int_as_float(0x7f800000);

  for (int t = t0; t < t1; ++t) {
    const int it = t - t0, slot = it & 1;
    const uint32_t ph_k = (it >> 1) & 1;
    const int bh = t / a.nblk, blk = t % a.nblk, h = bh % a.H;
    if (h != cur_h) {  // (re)load the head's codebook image and norms
      if (tid == 0) {
        const size_t bytes = S::parents_bytes(M0) + S::children_bytes(M0, C);
        tc::mbar_arrive_expect_tx(bar_cb, (uint32_t)bytes);
        const bf16* src = a.cw + (size_t)h * Mt * D;
        // parents and (optionally) children are contiguous in the image
        size_t off = 0;
        while (off < bytes) {
          const uint32_t part = (uint32_t)std::min<size_t>(bytes - off, 65536);
          tc::bulk_g2s(sPar + off, reinterpret_cast<const uint8_t*>(src) + off, part, bar_cb);
          off += part;
        }
      }
      for (int j = tid; j < Mt; j += 128) sNorm[j] = __ldg(a.norms + (size_t)h * Mt + j);
      if (!tc::mbar_wait(bar_cb, ph_cb)) {
        atomicOr(a.err, kErrTimeout);
        *sAbort = 1;
      }
      ph_cb ^= 1;
      cur_h = h;
      __syncthreads();
    }
    if (!tc::mbar_wait(&bar_k[slot], ph_k)) {
      atomicOr(a.err, kErrTimeout);
      *sAbort = 1;
    }
    __syncthreads();
    if (*sAbort) break;
    const uint8_t* sK = sRing + slot * (kKeys * D * 2);
    if (tid == 0) {
      tc::tc_fence_after();
      const uint32_t sKa = tc::smem_u32(sK);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t ad = tc::sdesc_sw128(sKa + (k >> 2) * (kKeys * 128) + (k & 3) * 32, 16, 1024);
        const uint64_t bd = tc::sdesc_sw128(sParA + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
        tc::mma_bf16(tmem, ad, bd, idesc, k > 0);
      }
      tc::mma_commit(bar_mma);
    }
    if (!tc::mbar_wait(bar_mma, ph_mma)) atomicOr(a.err, kErrTimeout);
    ph_mma ^= 1;
    tc::tc_fence_after();

    // nearest parent: first minimum of |p|^2 - 2 k.p; four independent running
    // minima over interleaved 16-column groups, merged in index order
    float best = INF;
    int par = 0;
    for (int g0 = 0; g0 < M0; g0 += 64) {
      uint32_t r[64];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (g0 + q * 16 < M0) tc::tmem_ld16(tmem + lane_off + g0 + q * 16, r + q * 16);
      tc::tmem_wait_ld();
      float bq[4];
      int iq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        bq[q] = INF;
        iq[q] = 0;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = g0 + q * 16 + e;
          if (m < M0) {
            const float dm = fmaf(-2.f, __uint_as_float(r[q * 16 + e]), sNorm[m]);
            if (dm < bq[q]) {
              bq[q] = dm;
              iq[q] = m;
            }
          }
        }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (bq[q] < best) {
          best = bq[q];
          par = iq[q];
        }
    }
    int code = par;
    if constexpr (CH_SMEM) {
      if (C > 0) {  // C == 8 on this path
        const int pair = par >> 1;
        atomicOr(&sPairs[pair >> 5], 1u << (pair & 31));
        tc::tc_fence_before();
        __syncthreads();  // pair set complete, parents' logits read
        uint32_t bits[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) bits[w] = sPairs[w];
        int npairs = 0, slot = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          if (w < (pair >> 5)) slot += __popc(bits[w]);
          npairs += __popc(bits[w]);
        }
        slot += __popc(bits[pair >> 5] & ((1u << (pair & 31)) - 1u));
        const uint32_t idesc16 = tc::idesc_bf16(kKeys, 16, 0, 0);
        const uint32_t sKa = tc::smem_u32(sK), sCha = tc::smem_u32(sCh);
        float vals[8];
        for (int round = 0; round * 16 < npairs; ++round) {
          if (tid == 0) {
            tc::tc_fence_after();
            int idx = 0;
            for (int w = 0; w < 4; ++w) {
              uint32_t b = bits[w];
              while (b) {
                const int q = w * 32 + __ffs(b) - 1;
                b &= b - 1;
                if (idx >= round * 16 && idx < round * 16 + 16) {
                  const uint32_t col = (uint32_t)(idx - round * 16) * 16;
#pragma unroll
                  for (int k = 0; k < D / 16; ++k) {
                    const uint64_t ad = tc::sdesc_sw128(sKa + (k >> 2) * (kKeys * 128) + (k & 3) * 32, 16, 1024);
                    const uint64_t bd = tc::sdesc_sw128(sCha + (2 * q) * (KH * 1024) + (k >> 2) * 1024 + (k & 3) * 32,
                                                        16, KH * 1024);
                    tc::mma_bf16(tmem + col, ad, bd, idesc16, k > 0);
                  }
                }
                ++idx;
              }
            }
            tc::mma_commit(bar_mma);
          }
          if (!tc::mbar_wait(bar_mma, ph_mma)) atomicOr(a.err, kErrTimeout);
          ph_mma ^= 1;
          tc::tc_fence_after();
          // one TMEM load per distinct pair slot among this warp's keys
          const int my = (slot >= round * 16 && slot < round * 16 + 16) ? slot - round * 16 : -1;
          unsigned pending = __ballot_sync(0xffffffffu, my >= 0);
          while (pending) {
            const int leader = __ffs(pending) - 1;
            const int sl = __shfl_sync(0xffffffffu, my, leader);
            uint32_t r[16];
            tc::tmem_ld16(tmem + lane_off + sl * 16, r);
            tc::tmem_wait_ld();
            if (my == sl) {
              const int half = (par & 1) * 8;
#pragma unroll
              for (int c = 0; c < 8; ++c) vals[c] = __uint_as_float(half ? r[8 + c] : r[c]);
            }
            pending &= ~__ballot_sync(0xffffffffu, my == sl);
          }
          tc::tc_fence_before();
          __syncthreads();  // TMEM columns free for the next round
        }
        float dchild = INF;
        int cstar = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float dc = fmaf(-2.f, vals[c], sNorm[M0 + par * 8 + c]);
          if (dc < dchild) {
            dchild = dc;
            cstar = c;
          }
        }
        if (dchild < best) code = M0 + par * 8 + cstar;
        if (tid < 4) sPairs[tid] = 0;  // for the next tile (read by everyone above)
      }
    } else if (C > 0) {  // C == 8; children from L2, dot products on the CUDA cores
      // key row in registers, 16-byte chunks in rotated order
      const int rot = tid & 7;
      uint4 kq[KH][8];
#pragma unroll
      for (int kh = 0; kh < KH; ++kh)
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int lc = (s + rot) & 7;
          kq[kh][s] = *reinterpret_cast<const uint4*>(sK + kh * (kKeys * 128) + tid * 128 + ((lc ^ rot) << 4));
        }
      const uint8_t* atom = reinterpret_cast<const uint8_t*>(a.cw + ((size_t)h * Mt + M0 + par * 8) * D);
      float dchild = INF;
      int cstar = 0;
      for (int c = 0; c < 8; ++c) {
        float acc = 0.f;
#pragma unroll
        for (int kh = 0; kh < KH; ++kh)
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const int lc = (s + rot) & 7;
            const uint4 cv = __ldg(reinterpret_cast<const uint4*>(atom + kh * 1024 + c * 128 + ((lc ^ c) << 4)));
            acc = fma_bf16x2(kq[kh][s].x, cv.x, acc);
            acc = fma_bf16x2(kq[kh][s].y, cv.y, acc);
            acc = fma_bf16x2(kq[kh][s].z, cv.z, acc);
            acc = fma_bf16x2(kq[kh][s].w, cv.w, acc);
          }
        const float dc = fmaf(-2.f, acc, sNorm[M0 + par * 8 + c]);
        if (dc < dchild) {
          dchild = dc;
          cstar = c;
        }
      }
      if (dchild < best) code = M0 + par * 8 + cstar;
    }
    const int row = blk * kKeys + tid;
    if (row < a.N) a.assign[(size_t)bh * a.N + row] = code;
    count_codes(a.counts + (size_t)bh * Mt, code, row < a.N, M0, C);

    tc::tc_fence_before();
    __syncthreads();  // K slot and TMEM free
    if (tid == 0 && t + 2 < t1) issue_k(t + 2, slot);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, ncols);
  }
}

// Codewords -> swizzled-atom image (code a in atom a/8, row a%8) and fp32
// squared norms.  Children of parent p are codes M0 + p*C + c.
template <int D>
__global__ void __launch_bounds__(256) codebook_prep_kernel(const bf16* __restrict__ parents,
                                                            const bf16* __restrict__ children,
                                                            bf16* __restrict__ cw,
                                                            float* __restrict__ norms, int H, int M0,
                                                            int C) {
  constexpr int KH = D / 64;
  const int Mt = M0 * (1 + C);
  const long long total = (long long)H * Mt;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < total;
       u += (long long)gridDim.x * blockDim.x) {
    const int code = (int)(u % Mt);
    const long long h = u / Mt;
    const bf16* src = code < M0 ? parents + ((size_t)h * M0 + code) * D
                                : children + ((size_t)h * M0 * C + (code - M0)) * D;
    float nrm = 0.f;
    const int r = code & 7;
#pragma unroll
    for (int chunk = 0; chunk < D / 8; ++chunk) {
      float v[8];
      load8(src + chunk * 8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) nrm = fmaf(v[e], v[e], nrm);
      const int kh = chunk >> 3, c = chunk & 7;
      store8(cw + (((size_t)h * (Mt / 8) + (code >> 3)) * KH + kh) * 512 + r * 64 + ((c ^ r) * 8), v);
    }
    norms[u] = nrm;
  }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <int D, bool CH>
cudaError_t launch_impl(const Shape& s, const CUtensorMap& kmap, AssignArgs a, cudaStream_t st) {
  using S = AssignSmem<D, CH>;
  const size_t smem = S::total(s.M0, s.C) + 1024;
  cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel<D, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int per_sm = smem <= 110 * 1024 ? 2 : 1;
  const int ctas = std::min(a.ntiles, num_sms() * per_sm);
  a.tiles_per_cta = (a.ntiles + ctas - 1) / ctas;
  const int grid = (a.ntiles + a.tiles_per_cta - 1) / a.tiles_per_cta;
  assign_tc_kernel<D, CH><<<grid, 128, smem, st>>>(kmap, a);
  return cudaGetLastError();
}

}  // namespace

bool assign_tc_supported(const Shape& s, avq_dtype dt) {
  if (dt != AVQ_BF16) return false;
  if (s.d != 64 && s.d != 128) return false;
  if (s.M0 % 16 != 0 || s.M0 > 256) return false;
  if (s.C != 0 && s.C != 8) return false;
  return true;
}

size_t assign_tc_workspace(const Shape& s) {
  return align256((size_t)s.H * s.Mt() * s.d * 2) + align256((size_t)s.H * s.Mt() * 4);
}

cudaError_t launch_assign_tc(const Shape& s, const void* K, const void* parents, const void* children,
                             int32_t* assign, int32_t* counts, void* ws, unsigned int* err, cudaStream_t st,
                             LaunchLog& log) {
  bf16* cw = static_cast<bf16*>(ws);
  float* norms = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)s.H * s.Mt() * s.d * 2));
  const long long work = (long long)s.H * s.Mt();
  const int pblocks = (int)std::max<long long>(1, std::min<long long>((work + 255) / 256, num_sms() * 4));
  if (s.d == 64)
    codebook_prep_kernel<64><<<pblocks, 256, 0, st>>>((const bf16*)parents, (const bf16*)children, cw, norms,
                                                      s.H, s.M0, s.C);
  else
    codebook_prep_kernel<128><<<pblocks, 256, 0, st>>>((const bf16*)parents, (const bf16*)children, cw, norms,
                                                       s.H, s.M0, s.C);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  log.add("codebook_prep");

  CUtensorMap kmap;
  e = make_tmap_3d_bf16(&kmap, K, s.d, s.N, s.BH(), 64, kKeys);
  if (e != cudaSuccess) return e;
  AssignArgs a;
  a.cw = cw;
  a.norms = norms;
  a.assign = assign;
  a.counts = counts;
  a.err = err;
  a.H = s.H;
  a.N = s.N;
  a.M0 = s.M0;
  a.C = s.C;
  a.nblk = (s.N + kKeys - 1) / kKeys;
  a.ntiles = a.nblk * s.BH();
  a.tiles_per_cta = 1;
  const size_t ch_bytes = (size_t)s.M0 * s.C * s.d * 2;
  const bool ch_smem = ch_bytes <= 96 * 1024;
  if (s.d == 64)
    e = ch_smem ? launch_impl<64, true>(s, kmap, a, st) : launch_impl<64, false>(s, kmap, a, st);
  else
    e = ch_smem ? launch_impl<128, true>(s, kmap, a, st) : launch_impl<128, false>(s, kmap, a, st);
  log.add(ch_smem ? "assign_tc" : "assign_tc_l2children");
  return e;
}

}  // namespace avq
