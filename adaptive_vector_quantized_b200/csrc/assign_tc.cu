// Stage 1 assignment on the tcgen05 tensor cores ("AVQ-Attention: Adaptive
// Vector-Quantized Attention", Sec. 4.2, Algorithm 1: parent and child assignment).
//
// Persistent CTAs walk contiguous ranges of 128-key tiles.  Per tile:
//   K tile      TMA (128B swizzle) into a two-slot ring, the next tile in
//               flight while the current one is processed
//   parents     T = K P^T - |p|^2 / 2 on tcgen05 into TMEM (M = 128 keys,
//               N = M0; the norm term is one more K step, ones times the
//               bf16 triple hi + mid + lo of -|p|^2 / 2); thread r owns key
//               r = TMEM lane r and takes the first maximum of T over the
//               parents, i.e. the first minimum of |p|^2 - 2 k.p (|k|^2 is
//               the same for every codeword of a key and is dropped)
//   children    the C = 8 children of every parent are in shared memory as
//               one swizzled atom each, so the children of two adjacent
//               parents form an N = 16 operand tile: one MMA per parent pair
//               that some key of the tile chose gives every key of the tile
//               its dot products with those 16 children (TMEM, in rounds of
//               16 pairs); each thread then loads the 8 columns of its own
//               parent (one TMEM load per distinct pair in its warp).  When
//               the children do not fit in shared memory, this kernel writes
//               the parents only and a second launch (assign_children_kernel)
//               refines every key on the CUDA cores: 8 lanes per key, each
//               lane a slice of the dims of the key, its parent and the 8
//               children (coalesced 16-byte loads from L2), the partial dot
//               products summed over the 8 lanes.  Either way the key moves
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
  int count;  // warpgroup kernel: 0 leaves the counts to the streaming value sums
};


// bf16 bits of x, round to nearest even.
__device__ __forceinline__ uint32_t bf16_bits(float x) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
}

template <int D, bool CH_SMEM>
struct AssignSmem {
  // parents image | children image (optional) | K ring [2] | A and B of the
  // norm step | norms | pair bits | barriers
  __host__ __device__ static size_t parents_bytes(int M0) { return (size_t)M0 * D * 2; }
  __host__ __device__ static size_t children_bytes(int M0, int C) { return CH_SMEM ? (size_t)M0 * C * D * 2 : 0; }
  __host__ __device__ static size_t ring_off(int M0, int C) { return parents_bytes(M0) + children_bytes(M0, C); }
  __host__ __device__ static size_t ones_off(int M0, int C) { return ring_off(M0, C) + 2 * kKeys * D * 2; }
  __host__ __device__ static size_t bnorm_off(int M0, int C) { return ones_off(M0, C) + kKeys * 128; }
  __host__ __device__ static size_t norms_off(int M0, int C) { return bnorm_off(M0, C) + (size_t)M0 * 128; }
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
  grid_dependency_wait();  // the codebook image, norms and zeroed statistics
  constexpr int KH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int M0 = a.M0, C = a.C, Mt = M0 * (1 + C);
  uint8_t* sPar = sm;
  uint8_t* sCh = sm + S::parents_bytes(M0);
  uint8_t* sRing = sm + S::ring_off(M0, C);
  uint8_t* sOnes = sm + S::ones_off(M0, C);
  uint8_t* sBn = sm + S::bnorm_off(M0, C);
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
  // A of the norm step: row r = (1, 1, 1, 0, ...) in logical 16-byte chunk 0
  for (int i = tid; i < kKeys * 8; i += 128) {
    const int r = i >> 3, pos = i & 7;
    reinterpret_cast<uint4*>(sOnes)[i] =
        pos == (r & 7) ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0, 0, 0, 0);
  }
  tc::fence_proxy_async_smem();
  if (warp == 0) {
    tc::tmem_alloc(sTmem, ncols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  // per barrier, the parity of the phase that thread 0's last copy or MMA on
  // it completes (bit b of `issued` once there was one): bits 0-1 the K ring
  // slots, 2 the MMAs, 3 the codebook image; drained on the way out
  uint32_t issued = 0, exp_par = 0;
  auto note = [&](int b, uint32_t ph) {
    issued |= 1u << b;
    exp_par = (exp_par & ~(1u << b)) | ((ph & 1u) << b);
  };
  auto issue_k = [&](int t, int slot) {
    const int bh = t / a.nblk, blk = t % a.nblk;
    note(slot, (uint32_t)((t - t0) >> 1));  // waited at tile t - t0 with parity ((t - t0) >> 1) & 1
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
        note(3, ph_cb);
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
      for (int i = tid; i < M0 * 8; i += 128) {  // B of the norm step: -|p|^2 / 2 as a bf16 triple
        const int m = i >> 3, pos = i & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (pos == (m & 7)) {
          const float n = -0.5f * __ldg(a.norms + (size_t)h * Mt + m);
          const uint32_t hi = bf16_bits(n);
          const float r1 = n - __uint_as_float(hi << 16);
          const uint32_t mid = bf16_bits(r1);
          const uint32_t lo = bf16_bits(r1 - __uint_as_float(mid << 16));
          v = make_uint4(hi | (mid << 16), lo, 0u, 0u);
        }
        reinterpret_cast<uint4*>(sBn)[i] = v;
      }
      tc::fence_proxy_async_smem();
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
      tc::mma_bf16(tmem, tc::sdesc_sw128(tc::smem_u32(sOnes), 16, 1024), tc::sdesc_sw128(tc::smem_u32(sBn), 16, 1024),
                   idesc, 1);
      note(2, ph_mma);
      tc::mma_commit(bar_mma);
    }
    if (!tc::mbar_wait(bar_mma, ph_mma)) atomicOr(a.err, kErrTimeout);
    ph_mma ^= 1;
    tc::tc_fence_after();

    // nearest parent: first maximum of T = k.p - |p|^2 / 2 (the MMA's norm
    // step added the second term); four independent running maxima over
    // interleaved 16-column groups, merged in index order
    float bestT = -INF;
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
        bq[q] = -INF;
        iq[q] = 0;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = g0 + q * 16 + e;
          if (m < M0) {
            const float v = __uint_as_float(r[q * 16 + e]);
            if (v > bq[q]) {
              bq[q] = v;
              iq[q] = m;
            }
          }
        }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (bq[q] > bestT) {
          bestT = bq[q];
          par = iq[q];
        }
    }
    const float best = -2.f * bestT;  // the parent's |p|^2 - 2 k.p, for the child test
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
            note(2, ph_mma);
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
    }
    const int row = blk * kKeys + tid;
    if (row < a.N) a.assign[(size_t)bh * a.N + row] = code;
    count_codes(a.counts + (size_t)bh * Mt, code, row < a.N, M0, C);

    tc::tc_fence_before();
    __syncthreads();  // K slot and TMEM free
    if (tid == 0 && t + 2 < t1) issue_k(t + 2, slot);
  }

  // nothing in flight before TMEM is freed (the waits return at once for
  // completed operations; 1 ms limit)
  if (issued) {
    uint64_t* const bars[4] = {&bar_k[0], &bar_k[1], bar_mma, bar_cb};
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if ((issued >> b) & 1u)
        if (!tc::mbar_wait(bars[b], (exp_par >> b) & 1u, 1000000ull)) atomicOr(a.err, kErrTimeout);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, ncols);
  }
}

// ---------------------------------------------------------------------------
// Warpgroup-pipelined variant for M0 <= 64 with the children in shared memory.
// One CTA per SM holds the head's codebook image once; each of its NWG
// warpgroups walks its own interleaved sequence of 128-key tiles with its own
// two-slot K ring, barriers and 128 TMEM columns, so that the tensor-core
// latency of one warpgroup's tile hides behind the other warpgroups' work.
// Children of a tile: the child atoms of the parents that some key chose are
// gathered (in index order, up to 8 per round) into a contiguous staging
// operand, so one MMA chain of N = 8 x (atoms, rounded up to even) gives every
// key its dot products with all those children.  When those parents need more
// than one round, only the parents that two or more of the tile's keys chose
// are gathered, and the keys of the others get their 8 child dot products on
// the CUDA cores (a warp per key) while the MMA runs.
// Scores: T = k.c - |c|^2 / 2 orders the codewords of a key like the squared
// distance |k|^2 - 2 T, reversed.  For the parents the -|p|^2 / 2 term is
// folded into the MMA as one more K step: A holds 1, 1, 1 in its first three
// columns, B the bf16 triple (hi, mid, lo) whose sum is -|p|^2 / 2 to within
// 2^-24 of it, so TMEM receives T directly.
constexpr int kStageAtoms = 8;
// Thread 0 of each warpgroup issues the K copies and every MMA: a tile's
// child MMA goes in ahead of the next tile's parent MMA, and one issuer per
// barrier keeps the drain on the way out exact (it waits for the phase of
// the issuer's last operation).

template <int D>
struct WgSmem {
  static constexpr int KH = D / 64;
  static constexpr size_t kTile = (size_t)kKeys * D * 2;
  static constexpr size_t kStage = (size_t)kStageAtoms * KH * 1024;
  static constexpr size_t kWg = 2 * kTile + kStage;
  static constexpr size_t kOnes = (size_t)kKeys * 128;  // A operand of the norm step
  static constexpr size_t kBnorm = 64 * 128;            // B operand of the norm step
  __host__ __device__ static size_t cb_bytes(int M0, int C) { return (size_t)M0 * (1 + C) * D * 2; }
  __host__ __device__ static size_t ones_off(int M0, int C) { return (cb_bytes(M0, C) + 1023) & ~(size_t)1023; }
  __host__ __device__ static size_t bnorm_off(int M0, int C) { return ones_off(M0, C) + kOnes; }
  __host__ __device__ static size_t wg_off(int M0, int C) { return bnorm_off(M0, C) + kBnorm; }
  __host__ __device__ static size_t norms_off(int M0, int C, int nwg) { return wg_off(M0, C) + nwg * kWg; }
  __host__ __device__ static size_t misc_off(int M0, int C, int nwg) {
    return (norms_off(M0, C, nwg) + (size_t)M0 * (1 + C) * 4 + 15) & ~(size_t)15;
  }
  // barriers: cb + 4 per warpgroup; parent masks: 8 words per warpgroup
  // ([tile parity][present lo, hi, shared lo, hi]); tmem base, abort
  __host__ __device__ static size_t total(int M0, int C, int nwg) {
    return misc_off(M0, C, nwg) + 8 * (1 + 4 * nwg) + 32 * nwg + 16;
  }
};

__device__ __forceinline__ void wg_bar(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
// Named-barrier sync of one warpgroup that also ORs a flag over its threads.
__device__ __forceinline__ bool wg_bar_or(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}
// Position of the n-th (0-based) set bit of a 32-bit word (binary search
// with population counts; the word has more than n set bits).
__device__ __forceinline__ int nth_set(uint32_t m, int n) {
  int pos = 0;
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const int c = __popc(m & ((1u << w) - 1u));
    if (n >= c) {
      n -= c;
      m >>= w;
      pos += w;
    }
  }
  return pos;
}


template <int D, int M0>
__global__ void __launch_bounds__(384, 1) assign_wg_kernel(const __grid_constant__ CUtensorMap kmap,
                                                           const AssignArgs a) {
  using S = WgSmem<D>;
  constexpr int KH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nwg = blockDim.x >> 7;
  const int C = a.C, Mt = M0 * (1 + C);
  const int tid = threadIdx.x, g = tid >> 7, wt = tid & 127, wwarp = wt >> 5, lane = tid & 31;
  uint8_t* sPar = sm;
  const uint8_t* sCh = sm + (size_t)M0 * D * 2;
  uint8_t* sRing = sm + S::wg_off(M0, C) + (size_t)g * S::kWg;
  uint8_t* sStage = sRing + 2 * S::kTile;
  uint8_t* sOnes = sm + S::ones_off(M0, C);
  uint8_t* sBn = sm + S::bnorm_off(M0, C);
  float* sNorm = reinterpret_cast<float*>(sm + S::norms_off(M0, C, nwg));  // -|c|^2 / 2
  uint64_t* bar_cb = reinterpret_cast<uint64_t*>(sm + S::misc_off(M0, C, nwg));
  uint64_t* bar_k = bar_cb + 1 + 4 * g;  // [2]
  uint64_t* bar_p = bar_k + 2;           // parent MMA done
  uint64_t* bar_c = bar_k + 3;           // child MMA done
  uint32_t* sMaskAll = reinterpret_cast<uint32_t*>(bar_cb + 1 + 4 * nwg);
  uint32_t* sMask = sMaskAll + 8 * g;  // [tile parity][present lo, hi, shared lo, hi]
  uint32_t* sTmem = sMaskAll + 8 * nwg;
  int* sAbort = reinterpret_cast<int*>(sTmem + 1);

  const int t0 = blockIdx.x * a.tiles_per_cta;
  const int t1 = min(a.ntiles, t0 + a.tiles_per_cta);
  if (t0 >= t1) return;
  const uint32_t ncols = nwg == 1 ? 128u : nwg == 2 ? 256u : 512u;

  if (tid == 0) {
    tc::mbar_init(bar_cb, 1);
    for (int w = 0; w < 4 * nwg; ++w) tc::mbar_init(bar_cb + 1 + w, 1);
    tc::fence_mbar_init();
    for (int w = 0; w < 8 * nwg; ++w) sMaskAll[w] = 0;
    *sAbort = 0;
    tc::prefetch_tensormap(&kmap);
  }
  // staging starts zeroed: padding atoms feed columns nobody reads, but stay finite
  for (int i = wt; i < (int)(S::kStage / 16); i += 128)
    reinterpret_cast<uint4*>(sStage)[i] = make_uint4(0, 0, 0, 0);
  // A of the norm step: row r = (1, 1, 1, 0, ...) in logical 16-byte chunk 0
  for (int i = tid; i < (int)(S::kOnes / 16); i += blockDim.x) {
    const int r = i >> 3, pos = i & 7;
    reinterpret_cast<uint4*>(sOnes)[i] =
        pos == (r & 7) ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0, 0, 0, 0);
  }
  tc::fence_proxy_async_smem();
  if (tid < 32) {
    tc::tmem_alloc(sTmem, ncols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_g = *sTmem + (uint32_t)g * 128u;
  const uint32_t lane_off = (uint32_t)(wwarp * 32) << 16;
  const int barid = 1 + g;
  // the set-up above may overlap the codebook preparation; its image, norms
  // and zeroed statistics are read below
  grid_dependency_wait();

  // per barrier, the parity of the phase that this thread's last copy or MMA
  // on it completes (bit b of `issued` once there was one): bits 0-1 the K
  // ring slots, 2 parent MMAs, 3 child MMAs, 4 the codebook image; drained
  // on the way out
  uint32_t issued = 0, exp_par = 0;
  auto note = [&](int b, uint32_t ph) {
    issued |= 1u << b;
    exp_par = (exp_par & ~(1u << b)) | ((ph & 1u) << b);
  };
  // K tile t for the j-th tile of this warpgroup (ring slot j & 1)
  auto issue_k = [&](int t, int j) {
    const int bh = t / a.nblk, blk = t % a.nblk, slot = j & 1;
    note(slot, (uint32_t)(j >> 1));
    tc::mbar_arrive_expect_tx(&bar_k[slot], (uint32_t)S::kTile);
#pragma unroll
    for (int kh = 0; kh < KH; ++kh)
      tc::tma_load_3d(sRing + slot * S::kTile + kh * (kKeys * 128), &kmap, kh * 64, blk * kKeys, bh,
                      &bar_k[slot]);
  };

  const uint32_t idescP = tc::idesc_bf16(kKeys, M0, 0, 0);
  const uint32_t sParA = tc::smem_u32(sPar), sStA = tc::smem_u32(sStage);
  const uint32_t sOnesA = tc::smem_u32(sOnes), sBnA = tc::smem_u32(sBn);
  uint32_t ph_cb = 0, ph_p = 0, ph_c = 0;
  int cur_h = -1, it = 0;
  bool aborted = false, kerr = false;
  // parent scores of the K tile in `kslot` into TMEM half `kslot` (norm step
  // last); the j-th tile's MMA completes the phase of parity j & 1
  auto issue_parents = [&](int kslot, int j) {
    note(2, (uint32_t)j);
    const uint32_t sKa = tc::smem_u32(sRing + kslot * S::kTile);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint64_t ad = tc::sdesc_sw128(sKa + (k >> 2) * (kKeys * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(sParA + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
      tc::mma_bf16(tmem_g + (uint32_t)kslot * 64u, ad, bd, idescP, k > 0);
    }
    tc::mma_bf16(tmem_g + (uint32_t)kslot * 64u, tc::sdesc_sw128(sOnesA, 16, 1024),
                 tc::sdesc_sw128(sBnA, 16, 1024), idescP, 1);
    tc::mma_commit(bar_p);
  };

  for (int s0 = t0; s0 < t1;) {
    const int bh = s0 / a.nblk;
    const int s1 = min(t1, (bh + 1) * a.nblk);
    const int h = bh % a.H;
    if (h != cur_h) {  // (re)load the head's codebook image and norms, CTA-wide
      if (tid == 0) {
        const size_t bytes = S::cb_bytes(M0, C);
        note(4, ph_cb);
        tc::mbar_arrive_expect_tx(bar_cb, (uint32_t)bytes);
        const uint8_t* src = reinterpret_cast<const uint8_t*>(a.cw + (size_t)h * Mt * D);
        for (size_t off = 0; off < bytes;) {
          const uint32_t part = (uint32_t)std::min<size_t>(bytes - off, 65536);
          tc::bulk_g2s(sPar + off, src + off, part, bar_cb);
          off += part;
        }
      }
      for (int j = tid; j < Mt; j += blockDim.x) sNorm[j] = -0.5f * __ldg(a.norms + (size_t)h * Mt + j);
      for (int i = tid; i < 64 * 8; i += blockDim.x) {  // B of the norm step
        const int m = i >> 3, pos = i & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M0 && pos == (m & 7)) {
          const float n = -0.5f * __ldg(a.norms + (size_t)h * Mt + m);
          const uint32_t hi = bf16_bits(n);
          const float r1 = n - __uint_as_float(hi << 16);
          const uint32_t mid = bf16_bits(r1);
          const uint32_t lo = bf16_bits(r1 - __uint_as_float(mid << 16));
          v = make_uint4(hi | (mid << 16), lo, 0u, 0u);
        }
        reinterpret_cast<uint4*>(sBn)[i] = v;
      }
      tc::fence_proxy_async_smem();
      if (!tc::mbar_wait(bar_cb, ph_cb)) {
        atomicOr(a.err, kErrTimeout);
        *sAbort = 1;
      }
      ph_cb ^= 1;
      cur_h = h;
      __syncthreads();
      if (*sAbort) break;
    }
    const int first = s0 + g;
    // prologue (thread 0): K of the first two tiles, parent MMA of the first
    if (wt == 0 && first < s1) {
      issue_k(first, it);
      if (first + nwg < s1) issue_k(first + nwg, it + 1);
    }
    if (wt == 0 && first < s1) {
      if (tc::mbar_wait(&bar_k[it & 1], (it >> 1) & 1)) {
        tc::tc_fence_after();
        issue_parents(it & 1, it);
      } else {
        kerr = true;
      }
    }
    for (int t = first; t < s1; t += nwg, ++it) {
      const int slot = it & 1;
      const uint32_t tP = tmem_g + (uint32_t)slot * 64u;  // parent, then child scores of this tile
      bool bad = false;
      if (wt == 0) bad = !tc::mbar_wait(bar_p, ph_p);
      if (wt == 0) bad = bad || kerr;
      ph_p ^= 1;
      tc::tc_fence_before();
      if (wg_bar_or(barid, bad)) {  // parent scores of tile t in TMEM
        if (wt == 0) atomicOr(a.err, kErrTimeout);
        aborted = true;
        break;
      }
      tc::tc_fence_after();
      // next tile's parent MMA into the other half (its scores there were read
      // before the barrier above), so that it overlaps this tile's epilogue
      auto next_parents = [&](int issuer) {
        if (wt == issuer && t + nwg < s1) {
          if (tc::mbar_wait(&bar_k[slot ^ 1], ((it + 1) >> 1) & 1)) {
            tc::tc_fence_after();
            issue_parents(slot ^ 1, it + 1);
          } else {
            kerr = true;
          }
        }
      };
      if (C == 0) {
        next_parents(0);
        if (wt == 0 && t + 2 * nwg < s1) issue_k(t + 2 * nwg, it + 2);  // K slot read by nothing else
      }

      // nearest parent = first maximum of T over the M0 parents: eight running
      // maxima over contiguous groups of M0/8 columns, merged in index order
      float best;
      int par;
      {
        constexpr int G = M0 / 8;
        uint32_t r[M0];
#pragma unroll
        for (int q = 0; q < M0 / 16; ++q) tc::tmem_ld16(tP + lane_off + q * 16, r + q * 16);
        tc::tmem_wait_ld();
        float bv[8];
        int bi[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          bv[q] = __uint_as_float(r[q * G]);
          bi[q] = q * G;
        }
#pragma unroll
        for (int e = 1; e < G; ++e)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float v = __uint_as_float(r[q * G + e]);
            if (v > bv[q]) {
              bv[q] = v;
              bi[q] = q * G + e;
            }
          }
#pragma unroll
        for (int w = 1; w < 8; w *= 2)
#pragma unroll
          for (int q = 0; q < 8; q += 2 * w)
            if (bv[q + w] > bv[q]) {
              bv[q] = bv[q + w];
              bi[q] = bi[q + w];
            }
        best = bv[0];
        par = bi[0];
      }
      int code = par;
      if (C > 0) {  // C == 8 on this path
        // the tile's parents: present (some key chose it) and shared (a second
        // warp of the tile, or a second key of this warp, chose it too)
        uint32_t* mk = sMask + slot * 4;
        const bool dup = __popc(__match_any_sync(0xffffffffu, par)) > 1;
        const uint32_t lo = __reduce_or_sync(0xffffffffu, par < 32 ? 1u << par : 0u);
        const uint32_t hi = __reduce_or_sync(0xffffffffu, par >= 32 ? 1u << (par - 32) : 0u);
        const uint32_t dlo = __reduce_or_sync(0xffffffffu, dup && par < 32 ? 1u << par : 0u);
        const uint32_t dhi = __reduce_or_sync(0xffffffffu, dup && par >= 32 ? 1u << (par - 32) : 0u);
        if ((wt & 31) == 0) {
          const uint32_t olo = lo ? atomicOr(mk, lo) : 0u;
          const uint32_t ohi = hi ? atomicOr(mk + 1, hi) : 0u;
          if ((lo & olo) | dlo) atomicOr(mk + 2, (lo & olo) | dlo);
          if ((hi & ohi) | dhi) atomicOr(mk + 3, (hi & ohi) | dhi);
        }
        tc::tc_fence_before();
        wg_bar(barid);  // parent sets complete, parent scores read
        if (wt == 0) {  // the other parity's sets, for the next tile
#pragma unroll
          for (int w = 0; w < 4; ++w) sMask[(slot ^ 1) * 4 + w] = 0;
        }
        // child scores on the tensor cores for every present parent when they
        // fit one round, else for the shared parents only; the keys of the
        // other parents (one key each) get theirs on the CUDA cores, while the
        // child MMA runs
        const uint32_t p_lo = mk[0], p_hi = mk[1];
        const bool one_round = __popc(p_lo) + __popc(p_hi) <= kStageAtoms;
        const uint32_t m_lo = one_round ? p_lo : mk[2], m_hi = one_round ? p_hi : mk[3];
        const int n_lo = __popc(m_lo), np = n_lo + __popc(m_hi);
        const bool in_mma = par < 32 ? ((m_lo >> par) & 1u) != 0 : ((m_hi >> (par - 32)) & 1u) != 0;
        const int myslot = !in_mma ? -1
                           : par < 32 ? __popc(m_lo & ((1u << par) - 1u))
                                      : n_lo + __popc(m_hi & ((1u << (par - 32)) - 1u));
        float vals[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) vals[c] = 0.f;
        // one key at a time, the warp's 32 lanes take its 8 children x 4
        // quarters of the dims (bf16 products, fp32 sums), read from the K tile
        // and the children's atoms in shared memory (128-byte swizzle)
        auto simt_children = [&]() {
          unsigned todo = __ballot_sync(0xffffffffu, !in_mma);
          const int c = lane >> 2, qd = lane & 3;
          const uint8_t* kt = sRing + slot * S::kTile;
          while (todo) {
            const int kl = __ffs(todo) - 1;
            todo &= todo - 1;
            const int kp = __shfl_sync(0xffffffffu, par, kl);
            const int krow = wwarp * 32 + kl;
            const uint8_t* ch = sCh + (size_t)kp * (KH * 1024);
            float dot = 0.f;
#pragma unroll
            for (int kh = 0; kh < KH; ++kh)
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const int chunk = qd * 2 + h2;
                const uint4 kv = *reinterpret_cast<const uint4*>(kt + kh * (kKeys * 128) + krow * 128 +
                                                                 ((chunk ^ (krow & 7)) << 4));
                const uint4 cv = *reinterpret_cast<const uint4*>(ch + kh * 1024 + c * 128 + ((chunk ^ c) << 4));
                dot = fma_bf16x2(kv.x, cv.x, dot);
                dot = fma_bf16x2(kv.y, cv.y, dot);
                dot = fma_bf16x2(kv.z, cv.z, dot);
                dot = fma_bf16x2(kv.w, cv.w, dot);
              }
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              const float v = __shfl_sync(0xffffffffu, dot, cc * 4);
              if (lane == kl) vals[cc] = v;
            }
          }
        };
        if (np == 0) next_parents(0);  // no child MMA for this tile
        for (int r0 = 0; r0 < np; r0 += kStageAtoms) {
          const int nr = min(kStageAtoms, np - r0);
          const int nat = (nr + 1) & ~1;
          {  // 16 threads per atom, KH * 4 chunks of 16 bytes each
            const int j = wt >> 4;
            if (j < nr) {
              const int n = r0 + j;
              const int p = n < n_lo ? nth_set(m_lo, n) : 32 + nth_set(m_hi, n - n_lo);
              const uint4* src = reinterpret_cast<const uint4*>(sCh + (size_t)p * (KH * 1024));
              uint4* dst = reinterpret_cast<uint4*>(sStage + (size_t)j * (KH * 1024));
              uint4 v[KH * 4];
#pragma unroll
              for (int u = 0; u < KH * 4; ++u) v[u] = src[(wt & 15) + 16 * u];
#pragma unroll
              for (int u = 0; u < KH * 4; ++u) dst[(wt & 15) + 16 * u] = v[u];
            }
          }
          tc::fence_proxy_async_smem();
          wg_bar(barid);  // staging written
          // this round's child MMA, then (first round) the next tile's parent
          // MMA behind it, both from thread 0, so that the child scores the
          // tile waits for are not queued behind the next tile's parents
          if (wt == 0) {
            tc::tc_fence_after();
            const uint32_t idescC = tc::idesc_bf16(kKeys, 8 * nat, 0, 0);
            const uint32_t sKa = tc::smem_u32(sRing + slot * S::kTile);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t ad = tc::sdesc_sw128(sKa + (k >> 2) * (kKeys * 128) + (k & 3) * 32, 16, 1024);
              const uint64_t bd = tc::sdesc_sw128(sStA + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
              tc::mma_bf16(tP, ad, bd, idescC, k > 0);
            }
            note(3, ph_c);
            tc::mma_commit(bar_c);
            if (r0 == 0) next_parents(0);
            if (!tc::mbar_wait(bar_c, ph_c)) atomicOr(a.err, kErrTimeout);
          }
          if (r0 == 0) simt_children();
          ph_c ^= 1;
          wg_bar(barid);  // child scores in TMEM; the CUDA-core children done
          tc::tc_fence_after();
          // the round's child columns in two 32-column loads (only the halves
          // that some key of the warp needs), each key taking its slot's 8
          const int my = (myslot >= r0 && myslot < r0 + kStageAtoms) ? myslot - r0 : -1;
#pragma unroll
          for (int hh = 0; hh < kStageAtoms / 4; ++hh) {
            if (__any_sync(0xffffffffu, my >= 4 * hh && my < 4 * hh + 4)) {
              uint32_t rr[32];
              tc::tmem_ld16(tP + lane_off + hh * 32, rr);
              tc::tmem_ld16(tP + lane_off + hh * 32 + 16, rr + 16);
              tc::tmem_wait_ld();
#pragma unroll
              for (int s4 = 0; s4 < 4; ++s4)
                if (my == 4 * hh + s4) {
#pragma unroll
                  for (int c = 0; c < 8; ++c) vals[c] = __uint_as_float(rr[8 * s4 + c]);
                }
            }
          }
          if (r0 + kStageAtoms < np) {
            tc::tc_fence_before();
            wg_bar(barid);  // staging and child columns free for the next round
          }
        }
        if (np == 0) {
          simt_children();
          wg_bar(barid);  // the K tile is read by nothing else
        }
        if (wt == 0 && t + 2 * nwg < s1) issue_k(t + 2 * nwg, it + 2);  // K slot free
        float tchild = vals[0] + sNorm[M0 + par * 8];
        int cstar = 0;
#pragma unroll
        for (int c = 1; c < 8; ++c) {
          const float tc = vals[c] + sNorm[M0 + par * 8 + c];
          if (tc > tchild) {
            tchild = tc;
            cstar = c;
          }
        }
        if (tchild > best) code = M0 + par * 8 + cstar;
      }
      const int row = (t - bh * a.nblk) * kKeys + wt;
      if (row < a.N) a.assign[(size_t)bh * a.N + row] = code;
      if (a.count) count_codes_par(a.counts + (size_t)bh * Mt, par, code, row < a.N, M0);
    }
    if (aborted) *sAbort = 1;
    tc::tc_fence_before();
    __syncthreads();  // every warpgroup done with this head's image
    if (*sAbort) break;
    s0 = s1;
  }

  // nothing in flight before TMEM is freed (the waits return at once for
  // completed operations; 1 ms limit)
  if (issued) {
    uint64_t* const bars[5] = {&bar_k[0], &bar_k[1], bar_p, bar_c, bar_cb};
#pragma unroll
    for (int b = 0; b < 5; ++b)
      if ((issued >> b) & 1u)
        if (!tc::mbar_wait(bars[b], (exp_par >> b) & 1u, 1000000ull)) atomicOr(a.err, kErrTimeout);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (tid < 32) {
    tc::tc_fence_after();
    tc::tmem_dealloc(*sTmem, ncols);
  }
}

// Parents only, for codebooks whose children do not fit in shared memory (or
// C = 0): persistent CTAs over contiguous 128-key tiles; the parents' image of
// the head and the norm step's operands stay in shared memory, K tiles come
// through a two-slot TMA ring, and TMEM holds two score slots, so the next
// tile's MMA runs while this tile's first maximum of T is taken.  Two
// warpgroups take the maximum, each over alternate 64-column groups of the
// same TMEM lanes (its own keys' rows), and the first merges the second's
// result in index order.  With children, assign_children_kernel then refines
// every key (and counts); without, this kernel counts.
template <int D>
struct ParentsSmem {
  // parents image | K ring [2] | A and B of the norm step | second warpgroup's
  // maxima [128] and their parents [128] | barriers | tmem, abort
  __host__ __device__ static size_t ring_off(int M0) { return (size_t)M0 * D * 2; }
  __host__ __device__ static size_t ones_off(int M0) { return ring_off(M0) + 2 * kKeys * D * 2; }
  __host__ __device__ static size_t bnorm_off(int M0) { return ones_off(M0) + kKeys * 128; }
  __host__ __device__ static size_t xchg_off(int M0) { return bnorm_off(M0) + (size_t)M0 * 128; }
  __host__ __device__ static size_t bar_off(int M0) { return xchg_off(M0) + 2 * kKeys * 4; }
  __host__ __device__ static size_t total(int M0) { return bar_off(M0) + 64; }
};

template <int D>
__global__ void __launch_bounds__(256) assign_parents_kernel(const __grid_constant__ CUtensorMap kmap,
                                                             const AssignArgs a) {
  using S = ParentsSmem<D>;
  grid_dependency_wait();  // the codebook image, norms and zeroed statistics
  constexpr int KH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int M0 = a.M0, C = a.C, Mt = M0 * (1 + C);
  uint8_t* sPar = sm;
  uint8_t* sRing = sm + S::ring_off(M0);
  uint8_t* sOnes = sm + S::ones_off(M0);
  uint8_t* sBn = sm + S::bnorm_off(M0);
  float* sXT = reinterpret_cast<float*>(sm + S::xchg_off(M0));  // [kKeys]
  int* sXP = reinterpret_cast<int*>(sXT + kKeys);               // [kKeys]
  uint64_t* bar_k = reinterpret_cast<uint64_t*>(sm + S::bar_off(M0));  // [2]
  uint64_t* bar_cb = bar_k + 2;
  uint64_t* bar_mma = bar_k + 3;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar_k + 4);
  int* sAbort = reinterpret_cast<int*>(bar_k + 4) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, wg = tid >> 7, wt = tid & 127;
  const int nthr = blockDim.x;
  const int t0 = blockIdx.x * a.tiles_per_cta;
  const int t1 = min(a.ntiles, t0 + a.tiles_per_cta);
  if (t0 >= t1) return;
  const uint32_t slot_cols = M0 <= 32 ? 32u : M0 <= 64 ? 64u : M0 <= 128 ? 128u : 256u;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) tc::mbar_init(bar_k + i, 1);
    tc::fence_mbar_init();
    *sAbort = 0;
    tc::prefetch_tensormap(&kmap);
  }
  // A of the norm step: row r = (1, 1, 1, 0, ...) in logical 16-byte chunk 0
  for (int i = tid; i < kKeys * 8; i += nthr) {
    const int r = i >> 3, pos = i & 7;
    reinterpret_cast<uint4*>(sOnes)[i] =
        pos == (r & 7) ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0, 0, 0, 0);
  }
  tc::fence_proxy_async_smem();
  if (warp == 0) {
    tc::tmem_alloc(sTmem, 2 * slot_cols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  // per barrier, the parity of the phase that thread 0's last copy or MMA on
  // it completes (bit b of `issued` once there was one): bits 0-1 the K ring
  // slots, 2 the parents' image, 3 the MMAs (the order of the barriers
  // bar_k[0..3]); drained on the way out
  uint32_t issued = 0, exp_par = 0;
  auto note = [&](int b, uint32_t ph) {
    issued |= 1u << b;
    exp_par = (exp_par & ~(1u << b)) | ((ph & 1u) << b);
  };
  auto issue_k = [&](int t) {  // tile t into ring slot (t - t0) & 1
    const int it = t - t0, slot = it & 1, bh = t / a.nblk, blk = t % a.nblk;
    note(slot, (uint32_t)(it >> 1));
    tc::mbar_arrive_expect_tx(&bar_k[slot], kKeys * D * 2);
#pragma unroll
    for (int kh = 0; kh < KH; ++kh)
      tc::tma_load_3d(sRing + slot * (kKeys * D * 2) + kh * (kKeys * 128), &kmap, kh * 64, blk * kKeys, bh,
                      &bar_k[slot]);
  };
  uint32_t ph_cb = 0, ph_mma = 0;
  // the head's parents' image and the norm step's B (CTA-wide)
  auto load_head = [&](int h) {
    if (tid == 0) {
      const uint32_t bytes = (uint32_t)(M0 * D * 2);
      note(2, ph_cb);
      tc::mbar_arrive_expect_tx(bar_cb, bytes);
      const uint8_t* src = reinterpret_cast<const uint8_t*>(a.cw + (size_t)h * Mt * D);
      for (uint32_t off = 0; off < bytes; off += 65536)
        tc::bulk_g2s(sPar + off, src + off, min(bytes - off, 65536u), bar_cb);
    }
    for (int i = tid; i < M0 * 8; i += nthr) {  // -|p|^2 / 2 as a bf16 triple
      const int m = i >> 3, pos = i & 7;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (pos == (m & 7)) {
        const float n = -0.5f * __ldg(a.norms + (size_t)h * Mt + m);
        const uint32_t hi = bf16_bits(n);
        const float r1 = n - __uint_as_float(hi << 16);
        const uint32_t mid = bf16_bits(r1);
        const uint32_t lo = bf16_bits(r1 - __uint_as_float(mid << 16));
        v = make_uint4(hi | (mid << 16), lo, 0u, 0u);
      }
      reinterpret_cast<uint4*>(sBn)[i] = v;
    }
    tc::fence_proxy_async_smem();
    if (!tc::mbar_wait(bar_cb, ph_cb)) {
      atomicOr(a.err, kErrTimeout);
      *sAbort = 1;
    }
    ph_cb ^= 1;
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
  };
  const uint32_t idesc = tc::idesc_bf16(kKeys, M0, 0, 0);
  // thread 0: wait for tile t's K, then T = K P^T - |p|^2 / 2 into its TMEM slot
  auto issue_mma = [&](int t) {
    const int it = t - t0, slot = it & 1;
    if (!tc::mbar_wait(&bar_k[slot], (uint32_t)(it >> 1) & 1u)) {
      atomicOr(a.err, kErrTimeout);
      *sAbort = 1;
      return;
    }
    tc::tc_fence_after();
    const uint32_t sKa = tc::smem_u32(sRing + slot * (kKeys * D * 2)), sParA = tc::smem_u32(sPar);
    const uint32_t d = tmem + (uint32_t)slot * slot_cols;
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint64_t ad = tc::sdesc_sw128(sKa + (k >> 2) * (kKeys * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(sParA + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
      tc::mma_bf16(d, ad, bd, idesc, k > 0);
    }
    tc::mma_bf16(d, tc::sdesc_sw128(tc::smem_u32(sOnes), 16, 1024), tc::sdesc_sw128(tc::smem_u32(sBn), 16, 1024),
                 idesc, 1);
    note(3, (uint32_t)it);  // the it-th commit completes phase it
    tc::mma_commit(bar_mma);
  };

  int cur_h = (t0 / a.nblk) % a.H;
  if (tid == 0) {
    issue_k(t0);
    if (t0 + 1 < t1) issue_k(t0 + 1);
  }
  load_head(cur_h);
  if (tid == 0 && !*sAbort) issue_mma(t0);
  __syncthreads();  // the abort flag is the same for every thread below
  const float NEG_INF = __int_as_float(0xff800000);
  for (int t = t0; t < t1; ++t) {
    const int it = t - t0, slot = it & 1;
    const int bh = t / a.nblk, blk = t % a.nblk;
    if (*sAbort) break;  // uniform: read after the barrier that ended the previous tile
    if (!tc::mbar_wait(bar_mma, ph_mma)) {
      atomicOr(a.err, kErrTimeout);
      *sAbort = 1;
    }
    ph_mma ^= 1;
    tc::tc_fence_after();
    if (tid == 0 && t + 2 < t1) issue_k(t + 2);  // this tile's K slot is read
    if (t + 1 < t1) {  // the next tile's MMA into the other slot, behind a head change if any
      const int hn = ((t + 1) / a.nblk) % a.H;
      if (hn != cur_h) {
        load_head(hn);
        cur_h = hn;
      }
      if (tid == 0 && !*sAbort) issue_mma(t + 1);
    }
    // first maximum of T: this warpgroup's 64-column groups (wg, wg + 2, ...),
    // four independent running maxima over interleaved 16-column groups in
    // each, merged in index order
    const uint32_t ts = tmem + (uint32_t)slot * slot_cols + lane_off;
    float bestT = NEG_INF;
    int par = wg == 0 ? 0 : M0;  // the merge keeps an in-range parent whatever the scores
    for (int g0 = wg * 64; g0 < M0; g0 += 128) {
      uint32_t r[64];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (g0 + q * 16 < M0) tc::tmem_ld16(ts + g0 + q * 16, r + q * 16);
      tc::tmem_wait_ld();
      float bq[4];
      int iq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        bq[q] = NEG_INF;
        iq[q] = 0;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = g0 + q * 16 + e;
          if (m < M0) {
            const float v = __uint_as_float(r[q * 16 + e]);
            if (v > bq[q]) {
              bq[q] = v;
              iq[q] = m;
            }
          }
        }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (bq[q] > bestT) {
          bestT = bq[q];
          par = iq[q];
        }
    }
    if (wg == 1) {
      sXT[wt] = bestT;
      sXP[wt] = par;
    }
    __syncthreads();  // the second warpgroup's maxima are in
    if (wg == 0) {  // merge: the larger T, equal T to the lower parent index
      const float ot = sXT[wt];
      const int op = sXP[wt];
      if (ot > bestT || (ot == bestT && op < par)) {
        bestT = ot;
        par = op;
      }
      const int row = blk * kKeys + wt;
      if (row < a.N) a.assign[(size_t)bh * a.N + row] = par;
      if (C == 0) count_codes(a.counts + (size_t)bh * Mt, par, row < a.N, M0, C);
    }
    tc::tc_fence_before();
    __syncthreads();  // this TMEM slot is read: the MMA two tiles on may overwrite it
  }

  // nothing in flight before TMEM is freed (the waits return at once for
  // completed operations; 1 ms limit)
  if (issued) {
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if ((issued >> b) & 1u)
        if (!tc::mbar_wait(bar_k + b, (exp_par >> b) & 1u, 1000000ull)) atomicOr(a.err, kErrTimeout);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 2 * slot_cols);
  }
}

// Child refinement for keys whose parent is already in `assign` (C = 8):
// 8 lanes per key, 4 keys per warp.  Lane s of a key holds dims
// [s D/8, (s+1) D/8) of the key, its parent and its 8 children (16-byte
// loads; the 8 lanes of a key read each 128- or 256-byte row once,
// coalesced), accumulates the 9 partial dot products in fp32 (bf16 x bf16
// products) and sums them over the 8 lanes.  Distances |c|^2 - 2 k.c with the
// fp32 squared norms; the key moves to the first strictly smallest child only
// if it is strictly closer than its parent.  Counts: the parent for every
// key, the child for keys that moved.
template <int D>
__global__ void __launch_bounds__(256) assign_children_kernel(const bf16* __restrict__ K,
                                                              const bf16* __restrict__ parents,
                                                              const bf16* __restrict__ children,
                                                              const float* __restrict__ norms,
                                                              int32_t* __restrict__ assign,
                                                              int32_t* __restrict__ counts, int BH, int H,
                                                              int N, int M0) {
  grid_dependency_wait();  // the parents of the pass before
  constexpr int C = 8;
  constexpr int DL = D / 8;      // dims per lane
  constexpr int CHK = DL / 8;    // 16-byte chunks per lane and row
  const int Mt = M0 * (1 + C);
  const int lane = threadIdx.x & 31, sub = lane & 7, kq = lane >> 3;
  const long long total = (long long)BH * N;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long k0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4; k0 < total;
       k0 += warps * 4) {  // warp-uniform loop
    const long long key = k0 + kq;
    const bool live = key < total;
    const long long bh = live ? key / N : 0;
    const int h = (int)(bh % H);
    const int p = live ? __ldg(assign + key) : 0;
    const bf16* kr = K + (size_t)(live ? key : 0) * D + sub * DL;
    const bf16* pr = parents + ((size_t)h * M0 + p) * D + sub * DL;
    const bf16* cr = children + ((size_t)h * M0 + p) * C * D + sub * DL;
    float acc[1 + C];
#pragma unroll
    for (int j = 0; j <= C; ++j) acc[j] = 0.f;
#pragma unroll
    for (int q = 0; q < CHK; ++q) {
      const uint4 kv = __ldg(reinterpret_cast<const uint4*>(kr + q * 8));
      uint4 cv[1 + C];
      cv[0] = __ldg(reinterpret_cast<const uint4*>(pr + q * 8));
#pragma unroll
      for (int c = 0; c < C; ++c) cv[1 + c] = __ldg(reinterpret_cast<const uint4*>(cr + (size_t)c * D + q * 8));
#pragma unroll
      for (int j = 0; j <= C; ++j) {
        acc[j] = fma_bf16x2(kv.x, cv[j].x, acc[j]);
        acc[j] = fma_bf16x2(kv.y, cv[j].y, acc[j]);
        acc[j] = fma_bf16x2(kv.z, cv[j].z, acc[j]);
        acc[j] = fma_bf16x2(kv.w, cv[j].w, acc[j]);
      }
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1)
#pragma unroll
      for (int j = 0; j <= C; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    if (live && sub == 0) {
      const float* nh = norms + (size_t)h * Mt;
      const float dp = fmaf(-2.f, acc[0], nh[p]);
      float dc = fmaf(-2.f, acc[1], nh[M0 + p * C]);
      int cstar = 0;
#pragma unroll
      for (int c = 1; c < C; ++c) {
        const float d = fmaf(-2.f, acc[1 + c], nh[M0 + p * C + c]);
        if (d < dc) {
          dc = d;
          cstar = c;
        }
      }
      int32_t* cnt = counts + (size_t)bh * Mt;
      atomicAdd(cnt + p, 1);
      if (dc < dp) {
        const int code = M0 + p * C + cstar;
        assign[key] = code;
        atomicAdd(cnt + code, 1);
      }
    }
  }
}

// Codewords -> swizzled-atom image (code a in atom a/8, row a%8) and fp32
// squared norms.  Children of parent p are codes M0 + p*C + c.
template <int D>
__global__ void __launch_bounds__(256) codebook_prep_kernel(const bf16* __restrict__ parents,
                                                            const bf16* __restrict__ children,
                                                            bf16* __restrict__ cw,
                                                            float* __restrict__ norms, int H, int M0,
                                                            int C, uint4* __restrict__ zero_a,
                                                            long long n_a, uint4* __restrict__ zero_b,
                                                            long long n_b) {
  constexpr int KH = D / 64;
  constexpr int CH = D / 8;  // 16-byte chunks per code: one thread each
  allow_dependents();  // the assignment's set-up may overlap this launch
  grid_dependency_wait();  // the workspace image may still be read by the launch before
  const int Mt = M0 * (1 + C);
  const long long total = (long long)H * Mt * CH;
  const long long span = (total + 31) / 32 * 32;  // whole warps, so the shuffles see every lane
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < span;
       u += (long long)gridDim.x * blockDim.x) {
    const bool live = u < total;
    const int chunk = (int)(u % CH);
    const long long hc = u / CH;  // h * Mt + code
    const int code = (int)(hc % Mt);
    const long long h = hc / Mt;
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.f;
    if (live) {
      const bf16* src = code < M0 ? parents + ((size_t)h * M0 + code) * D
                                  : children + ((size_t)h * M0 * C + (code - M0)) * D;
      load8(src + chunk * 8, v);
      const int r = code & 7, kh = chunk >> 3, c = chunk & 7;
      store8(cw + (((size_t)h * (Mt / 8) + (code >> 3)) * KH + kh) * 512 + r * 64 + ((c ^ r) * 8), v);
    }
    float nrm = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) nrm = fmaf(v[e], v[e], nrm);
#pragma unroll
    for (int o = CH / 2; o >= 1; o >>= 1) nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
    if (live && chunk == 0) norms[hc] = nrm;
  }
  // the stage's accumulators (counts, value sums) start at zero: cleared here
  // instead of by separate memsets
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_a + n_b;
       i += (long long)gridDim.x * blockDim.x) {
    if (i < n_a)
      zero_a[i] = z;
    else
      zero_b[i - n_a] = z;
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
  return launch_after(assign_tc_kernel<D, CH>, dim3(grid), dim3(128), smem, st, kmap, a);
}

constexpr size_t kMaxSmem = 227 * 1024;

template <int D>
cudaError_t launch_parents(const Shape& s, const CUtensorMap& kmap, AssignArgs a, cudaStream_t st) {
  const size_t smem = ParentsSmem<D>::total(s.M0) + 1024;
  cudaError_t e = cudaFuncSetAttribute(assign_parents_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // CTAs per SM: shared memory (228 KB per SM, 1 KB reserved per CTA) and
  // TMEM (512 columns; two score slots per CTA)
  const int slot = s.M0 <= 32 ? 32 : s.M0 <= 64 ? 64 : s.M0 <= 128 ? 128 : 256;
  const int per_sm = std::max(1, std::min((int)((228 * 1024) / (smem + 1024)), 512 / (2 * slot)));
  const int ctas = std::min(a.ntiles, num_sms() * per_sm);
  a.tiles_per_cta = (a.ntiles + ctas - 1) / ctas;
  const int grid = (a.ntiles + a.tiles_per_cta - 1) / a.tiles_per_cta;
  return launch_after(assign_parents_kernel<D>, dim3(grid), dim3(256), smem, st, kmap, a);
}

// Warpgroups per CTA for the pipelined kernel (0: the image does not fit).
template <int D>
int wg_count(const Shape& s) {
  for (int nwg = 3; nwg >= 1; --nwg)
    if (WgSmem<D>::total(s.M0, s.C, nwg) + 1024 <= kMaxSmem) return nwg;
  return 0;
}

template <int D, int M0>
cudaError_t launch_wg_m(const Shape& s, const CUtensorMap& kmap, AssignArgs a, int nwg, cudaStream_t st) {
  const size_t smem = WgSmem<D>::total(s.M0, s.C, nwg) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(assign_wg_kernel<D, M0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ctas = std::min(a.ntiles, num_sms());
  a.tiles_per_cta = (a.ntiles + ctas - 1) / ctas;
  const int grid = (a.ntiles + a.tiles_per_cta - 1) / a.tiles_per_cta;
  return launch_after(assign_wg_kernel<D, M0>, dim3(grid), dim3(128 * nwg), smem, st, kmap, a);
}

template <int D>
cudaError_t launch_wg(const Shape& s, const CUtensorMap& kmap, AssignArgs a, int nwg, cudaStream_t st) {
  switch (s.M0) {
    case 16: return launch_wg_m<D, 16>(s, kmap, a, nwg, st);
    case 32: return launch_wg_m<D, 32>(s, kmap, a, nwg, st);
    case 48: return launch_wg_m<D, 48>(s, kmap, a, nwg, st);
    default: return launch_wg_m<D, 64>(s, kmap, a, nwg, st);
  }
}

}  // namespace

bool assign_tc_supported(const Shape& s, avq_dtype dt) {
  if (dt != AVQ_BF16) return false;
  if (s.d != 64 && s.d != 128) return false;
  if (s.M0 % 16 != 0 || s.M0 > 256) return false;
  if (s.C != 0 && s.C != 8) return false;
  return true;
}

bool assign_tc_uses_warpgroups(const Shape& s) {
  return s.M0 <= 64 && (s.d == 64 ? wg_count<64>(s) : wg_count<128>(s)) > 0;
}

size_t assign_tc_workspace(const Shape& s) {
  return align256((size_t)s.H * s.Mt() * s.d * 2) + align256((size_t)s.H * s.Mt() * 4);
}

cudaError_t launch_assign_tc(const Shape& s, const void* K, const void* parents, const void* children,
                             int32_t* assign, int32_t* counts, void* ws, unsigned int* err, cudaStream_t st,
                             LaunchLog& log, float* vsum_to_zero, bool* counts_left) {
  if (counts_left) *counts_left = false;
  bf16* cw = static_cast<bf16*>(ws);
  float* norms = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)s.H * s.Mt() * s.d * 2));
  const long long work = (long long)s.H * s.Mt() * (s.d / 8);
  const int pblocks = (int)std::max<long long>(1, std::min<long long>((work + 255) / 256, num_sms() * 8));
  // counts (and the value sums when given) are zeroed by the same launch; both
  // are 16-byte aligned and a whole number of 16-byte words (M0 % 16 == 0)
  const long long n_counts = (long long)s.BH() * s.Mt() * 4 / 16;
  const long long n_vsum = vsum_to_zero ? (long long)s.BH() * s.Mt() * s.d * 4 / 16 : 0;
  uint4* zc = reinterpret_cast<uint4*>(counts);
  uint4* zv = reinterpret_cast<uint4*>(vsum_to_zero);
  cudaError_t e;
  if (s.d == 64)
    e = launch_after(codebook_prep_kernel<64>, dim3(pblocks), dim3(256), 0, st, (const bf16*)parents,
                     (const bf16*)children, cw, norms, s.H, s.M0, s.C, zc, n_counts, zv, n_vsum);
  else
    e = launch_after(codebook_prep_kernel<128>, dim3(pblocks), dim3(256), 0, st, (const bf16*)parents,
                     (const bf16*)children, cw, norms, s.H, s.M0, s.C, zc, n_counts, zv, n_vsum);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
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
  a.count = 1;
  const size_t ch_bytes = (size_t)s.M0 * s.C * s.d * 2;
  if (s.M0 <= 64) {  // warpgroup-pipelined kernel when the whole image fits
    const int nwg = s.d == 64 ? wg_count<64>(s) : wg_count<128>(s);
    if (nwg > 0) {
      // the streaming value sums count runs of equal codes far more cheaply
      // than the tile's warp-aggregated atomics on the assignment's chain
      if (counts_left) a.count = 0;
      e = s.d == 64 ? launch_wg<64>(s, kmap, a, nwg, st) : launch_wg<128>(s, kmap, a, nwg, st);
      if (e == cudaSuccess && counts_left) *counts_left = true;
      log.add("assign_tc_wg");
      return e;
    }
  }
  const bool ch_smem = s.C > 0 && ch_bytes <= 96 * 1024;
  if (ch_smem) {
    e = s.d == 64 ? launch_impl<64, true>(s, kmap, a, st) : launch_impl<128, true>(s, kmap, a, st);
    log.add("assign_tc");
    return e;
  }
  // children too large for shared memory (or none): parents on the tensor
  // cores, then the children refined by a CUDA-core launch with many warps
  e = s.d == 64 ? launch_parents<64>(s, kmap, a, st) : launch_parents<128>(s, kmap, a, st);
  if (e != cudaSuccess) return e;
  log.add("assign_tc_parents");
  if (s.C > 0) {
    const long long groups = ((long long)s.BH() * s.N + 3) / 4;  // 4 keys per warp
    const int blocks = (int)std::max<long long>(1, std::min<long long>((groups + 7) / 8, (long long)num_sms() * 16));
    if (s.d == 64)
      e = launch_after(assign_children_kernel<64>, dim3(blocks), dim3(256), 0, st, (const bf16*)K,
                       (const bf16*)parents, (const bf16*)children, (const float*)norms, assign, counts, s.BH(),
                       s.H, s.N, s.M0);
    else
      e = launch_after(assign_children_kernel<128>, dim3(blocks), dim3(256), 0, st, (const bf16*)K,
                       (const bf16*)parents, (const bf16*)children, (const float*)norms, assign, counts, s.BH(),
                       s.H, s.N, s.M0);
    if (e != cudaSuccess) return e;
    e = cudaGetLastError();
    log.add("assign_children");
  }
  return e;
}

}  // namespace avq
