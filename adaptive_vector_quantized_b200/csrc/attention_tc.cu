// Stage 2 on the tcgen05 tensor cores ("AVQ-Attention: Adaptive
// Vector-Quantized Attention", Sec. 4.3, Algorithm 2; Eqs. 6-9; Sec. D).
//
// One CTA per (head, block of 128 queries), 4 warps; thread i owns query row
// i, which is TMEM lane i of every accumulator.  Per block:
//   Q tile    TMA (128B swizzle) -> shared memory, stays for both logit MMAs
//   parents   S = Q C_p^T on tcgen05 into TMEM; each thread loads its row,
//             takes the masked max (Eq. 18), A = 2^(t - m) with t the scaled
//             log2-domain logit, z = sum A n; the importance column sums
//             (Eq. 7) are warp butterfly reduce-scatters in fp32; A goes to
//             shared memory as bf16 and x = A Vbar_p accumulates in TMEM.
//             If the parents do not fit one tile (or two_pass is set) the
//             parent tiles are swept twice: running max and z first, then A,
//             x and the importance with the exact denominator.
//   top-P     ranks of the M0 importances (descending, ties to the lower
//             index), all 128 threads.
//   children  the selected parents' children (C = 8: one swizzle atom each)
//             are bulk-copied from a prepared bf16 image; S_c = Q C_c^T on
//             tcgen05; per row the parent logit is the mean of its 8 child
//             logits (Eq. 8); dA = 2^(t_c - m) - 2^(t_p - m), zero for empty
//             children (Eq. 9); x += dA Vbar_c on tcgen05; z += dA n_c.
//             The reference max stays the parents' max unless a child logit
//             exceeds it by more than 2^24, in which case x (TMEM) and z are
//             rescaled first; the result is the same as the online merge of
//             Algorithm 2 because the max cancels in x / z.
//   output    O = x / z, bf16, staged in shared memory and stored by TMA.
// The codewords and the value sums are first converted by a small kernel
// into bf16 images of 1024-byte swizzled atoms (8 codes x 64 dims), so that
// every operand tile is one or more contiguous bulk copies.
#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"
#include "fastmath.cuh"

namespace avq {
namespace {

constexpr int kRows = 128;          // queries per block (MMA M)
constexpr int kTile = 64;           // parent codes per tile / child codes per chunk
constexpr int kChunkParents = kTile / 8;
constexpr float kRescaleLog2 = 24.f;

struct AttnArgs {
  const bf16* cw;   // [H][Mt/8][KH][8][64] swizzled codeword atoms
  const bf16* vb;   // [BH][Mt/8][NH][8][64] swizzled value-sum atoms
  const int32_t* counts;  // [BH][Mt]
  int32_t* sel;     // [BH][nblk][P] or null
  float* importance;  // [BH][nblk][M0] or null
  unsigned int* err;
  int H, N, M0, C, P, nblk, two_pass, BH;
  float scale_log2;  // scale * log2(e)
};

// shared memory plan (bytes); every operand region 1024-aligned
template <int D>
struct Smem {
  // codeword tile buffers: at d = 128 two, so that the next tile's codewords
  // arrive while this tile is processed (two CTAs per SM still fit); at d = 64
  // one (four CTAs per SM)
  static constexpr int kNB = D == 128 ? 2 : 1;
  static constexpr int kQ = 0;                              // Q tile / O staging
  static constexpr int kCW = kQ + kRows * D * 2;            // codeword tile(s) (64 codes each)
  static constexpr int kVB = kCW + kNB * kTile * D * 2;     // value-sum tile (64 codes)
  static constexpr int kPR = kVB + kTile * D * 2;           // probabilities [128][64] bf16
  static constexpr int kNF = kPR + kRows * kTile * 2;       // counts of the tile (float)
  static constexpr int kBI = kNF + kTile * 4;               // mask bias of the tile (0 / -inf)
  static constexpr int kW = kBI + kTile * 4;                // importance [256]
  static constexpr int kWP = kW + 256 * 4;                  // per-warp partial sums [4][kTile]
  static constexpr int kSEL = kWP + 4 * kTile * 4;          // selected parents [256]
  static constexpr int kRK = kSEL + 256 * 4;                // partial ranks [2][128]
  static constexpr int kCNTP = kRK + 256 * 4;               // the parents' counts (float) [256]
  static constexpr int kBAR = kCNTP + 256 * 4;              // 5 mbarriers
  static constexpr int kMISC = kBAR + 40;                   // tmem base, abort flag
  static constexpr int kTotal = kMISC + 32;
  static constexpr uint32_t kTmemCols = D == 64 ? 128 : 256;  // logits [64] + output [D]
};

__device__ __forceinline__ void fail(unsigned int* err, int* abort_flag) {
  atomicOr(err, kErrTimeout);
  *abort_flag = 1;
}

// Butterfly reduce-scatter of 32 per-lane values: lane L returns the warp sum
// of element L.
__device__ __forceinline__ float reduce_scatter32(float* v, int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const bool hi = (lane & s) != 0;
      const float send = hi ? v[i] : v[i + s];
      const float keep = hi ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

__device__ __forceinline__ void store_chunk8(uint8_t* tile, int row, int col, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(tile + (col >> 6) * (kRows * 128) + tc::sw128_offset(row, col & 63)) = u;
}

// 64 TMEM columns of this thread's row -> registers.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t* r) {
  tc::tmem_ld16(taddr, r);
  tc::tmem_ld16(taddr + 16, r + 16);
  tc::tmem_ld16(taddr + 32, r + 32);
  tc::tmem_ld16(taddr + 48, r + 48);
  tc::tmem_wait_ld();
}

template <int D>
__global__ void __launch_bounds__(128, D == 64 ? 4 : 2) attention_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                           const __grid_constant__ CUtensorMap omap,
                                                           const AttnArgs a) {
  using S = Smem<D>;
  grid_dependency_wait();  // the image preparation before
  constexpr int KH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + S::kQ;
  uint8_t* sCW = sm + S::kCW;
  uint8_t* sVB = sm + S::kVB;
  uint8_t* sPR = sm + S::kPR;
  float* sNF = reinterpret_cast<float*>(sm + S::kNF);
  float* sBI = reinterpret_cast<float*>(sm + S::kBI);
  float* sW = reinterpret_cast<float*>(sm + S::kW);
  float* sWP = reinterpret_cast<float*>(sm + S::kWP);
  int* sSEL = reinterpret_cast<int*>(sm + S::kSEL);
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(sm + S::kBAR);
  uint64_t* bar_cp = bar_q + 1;   // codeword tiles in buffer 0
  uint64_t* bar_mma = bar_q + 2;
  uint64_t* bar_vb = bar_q + 3;   // value-sum tiles (waited on only before the value MMA)
  uint64_t* bar_cp1 = bar_q + 4;  // codeword tiles in buffer 1 (d = 128)
  int* sRK = reinterpret_cast<int*>(sm + S::kRK);
  float* sCNTP = reinterpret_cast<float*>(sm + S::kCNTP);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + S::kMISC);
  int* sAbort = reinterpret_cast<int*>(sm + S::kMISC + 4);
  float* sNtot = reinterpret_cast<float*>(sm + S::kMISC + 8);  // keys of the head (extrapolation)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x, bh = blockIdx.y, h = bh % a.H;
  const int row0 = blk * kRows;
  const bool valid = row0 + tid < a.N;
  const int M0 = a.M0, Mt = M0 * (1 + a.C);
  const int groups = Mt / 8;
  const bf16* cw_h = a.cw + (size_t)h * groups * KH * 512;
  const bf16* vb_bh = a.vb + (size_t)bh * groups * KH * 512;
  const int32_t* cnt = a.counts + (size_t)bh * Mt;
  const float NEG_INF = __int_as_float(0xff800000);
  const float sl2 = a.scale_log2;

  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    tc::mbar_init(bar_cp, 1);
    tc::mbar_init(bar_mma, 1);
    tc::mbar_init(bar_vb, 1);
    tc::mbar_init(bar_cp1, 1);
    tc::fence_mbar_init();
    *sAbort = 0;
    *sNtot = 0.f;
    tc::prefetch_tensormap(&qmap);
    tc::prefetch_tensormap(&omap);
  }
  if (warp == 0) {
    tc::tmem_alloc(sTmem, S::kTmemCols);
    tc::tmem_relinquish();
  }
  for (int j = tid; j < M0; j += 128) {
    sW[j] = 0.f;
    sCNTP[j] = (float)__ldg(cnt + j);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tS = tmem;          // logits, 64 columns
  const uint32_t tX = tmem + kTile;  // output accumulator, D columns
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  uint32_t ph_cp = 0, ph_mma = 0, ph_vb = 0, ph_cp1 = 0;
  // per barrier, the parity of the phase that thread 0's last copy or MMA on
  // it completes (bit b of `issued` once there was one): drained on the way out
  uint32_t issued = 0, exp_par = 0;
  auto note = [&](int b, uint32_t ph) {
    issued |= 1u << b;
    exp_par = (exp_par & ~(1u << b)) | (ph << b);
  };
  if (tid == 0) {
    note(0, 0);
    tc::mbar_arrive_expect_tx(bar_q, kRows * D * 2);
#pragma unroll
    for (int kh = 0; kh < KH; ++kh) tc::tma_load_3d(sQ + kh * kRows * 128, &qmap, kh * 64, row0, bh, bar_q);
  }

  const uint32_t idesc_x = tc::idesc_bf16(kRows, D, 0, 1);
  const uint32_t sQa = tc::smem_u32(sQ), sCWa = tc::smem_u32(sCW), sVBa = tc::smem_u32(sVB),
                 sPRa = tc::smem_u32(sPR);
  // S = Q * CW^T over n codes (n a multiple of 16, <= 64) from codeword
  // buffer `b` -- one thread
  auto issue_logits = [&](int n, int b) {
    note(3, ph_mma);
    const uint32_t idesc = tc::idesc_bf16(kRows, n, 0, 0);
    const uint32_t cwa = sCWa + (uint32_t)(b * kTile * D * 2);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint64_t ad = tc::sdesc_sw128(sQa + (k >> 2) * (kRows * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(cwa + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
      tc::mma_bf16(tS, ad, bd, idesc, k > 0);
    }
    tc::mma_commit(bar_mma);
  };
  // x += PR * VB over n codes -- one thread
  auto issue_values = [&](int n, bool acc) {
    note(3, ph_mma);
    for (int k = 0; k < n / 16; ++k) {
      const uint64_t ad = tc::sdesc_sw128(sPRa + (k & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(sVBa + k * 2 * (KH * 1024), 1024, KH * 1024);
      tc::mma_bf16(tX, ad, bd, idesc_x, (acc || k > 0) ? 1u : 0u);
    }
    tc::mma_commit(bar_mma);
  };
  auto wait_mma = [&]() {
    if (!tc::mbar_wait(bar_mma, ph_mma)) fail(a.err, sAbort);
    ph_mma ^= 1;
    tc::tc_fence_after();
  };
  auto wait_cp = [&](int b) {
    if (b == 0) {
      if (!tc::mbar_wait(bar_cp, ph_cp)) fail(a.err, sAbort);
      ph_cp ^= 1;
    } else {
      if (!tc::mbar_wait(bar_cp1, ph_cp1)) fail(a.err, sAbort);
      ph_cp1 ^= 1;
    }
  };
  // parent tile t's codewords into buffer b (thread 0)
  auto copy_tile = [&](int t, int b) {
    const int n = min(kTile, M0 - t * kTile);
    const uint32_t cwb = (uint32_t)n * D * 2;
    uint64_t* bar = b == 0 ? bar_cp : bar_cp1;
    if (b == 0) note(1, ph_cp); else note(4, ph_cp1);
    tc::mbar_arrive_expect_tx(bar, cwb);
    tc::bulk_g2s(sCW + b * kTile * D * 2, cw_h + (size_t)(t * kTile / 8) * KH * 512, cwb, bar);
  };
  auto wait_vb = [&]() {
    if (!tc::mbar_wait(bar_vb, ph_vb)) fail(a.err, sAbort);
    ph_vb ^= 1;
  };

  float m = NEG_INF, z = 0.f;
  const int nT = (M0 + kTile - 1) / kTile;
  // two_pass == 2: one sweep over the parent tiles, the importance of each
  // tile from the count-extrapolated denominator (Sec. B, Eqs. 13-14)
  const bool extrap = a.two_pass == 2;
  const int sweeps = extrap ? 1 : (a.two_pass || nT > 1) ? 2 : 1;
  if (extrap) {  // N of Eq. 13: the keys of the head, the sum of the parents' counts
    float c = 0.f;
    for (int j = tid; j < M0; j += 128) c += (float)__ldg(cnt + j);
    c = warp_sum(c);
    if (lane == 0) atomicAdd(sNtot, c);  // read after the next CTA barrier
  }
  float nseen = 0.f;  // keys of the parents in the tiles swept so far
  bool x_started = false;
  bool q_ready = false;

  // ---- parents: one sweep (all parents in one tile) or two (running max and
  //      denominator first, then probabilities, values and importance) ----
  // The g-th tile of the sweeps uses codeword buffer g % kNB; with two
  // buffers, tile g + 1's copy is issued as soon as tile g's logit MMA is
  // (buffer (g + 1) % 2 was last read by tile g - 1's MMA, which completed).
  constexpr int kNB = S::kNB;
  if (kNB == 2 && tid == 0) copy_tile(0, 0);
  for (int sweep = 0; sweep < sweeps; ++sweep) {
    const bool last = sweep == sweeps - 1;
    for (int t = 0; t < nT; ++t) {
      const int c0 = t * kTile;
      const int n = min(kTile, M0 - c0);
      const int g = sweep * nT + t, b = g % kNB;
      uint8_t* cwbuf = sCW + b * kTile * D * 2;
      if (tid == 0) {
        if (kNB == 1) copy_tile(t, 0);
        if (last) {
          note(2, ph_vb);
          tc::mbar_arrive_expect_tx(bar_vb, (uint32_t)n * D * 2);
          tc::bulk_g2s(sVB, vb_bh + (size_t)(c0 / 8) * KH * 512, (uint32_t)n * D * 2, bar_vb);
        }
      }
      // a partial tile: zero the unused codeword rows so that the logits MMA can
      // always run over 64 columns with finite results
      for (int i = tid; i < (kTile - n) * KH * 8; i += 128) {
        const int row = n + i / (KH * 8), rest = i % (KH * 8);
        *reinterpret_cast<uint4*>(cwbuf + (row >> 3) * (KH * 1024) + (rest >> 3) * 1024 + (row & 7) * 128 +
                                  (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
      for (int j = tid; j < kTile; j += 128) {
        const float nf = j < n ? sCNTP[c0 + j] : 0.f;
        sNF[j] = nf;
        sBI[j] = nf > 0.f ? 0.f : NEG_INF;
      }
      tc::fence_proxy_async_smem();
      if (!q_ready) {
        if (!tc::mbar_wait(bar_q, 0)) fail(a.err, sAbort);
        q_ready = true;
      }
      wait_cp(b);
      __syncthreads();
      if (*sAbort) goto done;
      if (tid == 0) {
        tc::tc_fence_after();
        issue_logits(kTile, b);
        if (kNB == 2 && g + 1 < sweeps * nT) copy_tile((g + 1) % nT, b ^ 1);
      }
      wait_mma();
      {
        uint32_t r[64];
        tmem_ld64(tS + lane_off, r);
        const float4* bi4 = reinterpret_cast<const float4*>(sBI);
        const float4* nf4 = reinterpret_cast<const float4*>(sNF);
        // t = scaled log2 logit; the bias is 0 for non-empty codes, -inf for empty
        // codes and unused columns (Eq. 18: those never set the max)
        float tm[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const float4 b = bi4[e >> 2];
          const float t0 = fmaf(__uint_as_float(r[e]), sl2, b.x), t1 = fmaf(__uint_as_float(r[e + 1]), sl2, b.y);
          const float t2 = fmaf(__uint_as_float(r[e + 2]), sl2, b.z), t3 = fmaf(__uint_as_float(r[e + 3]), sl2, b.w);
          r[e] = __float_as_uint(t0); r[e + 1] = __float_as_uint(t1);
          r[e + 2] = __float_as_uint(t2); r[e + 3] = __float_as_uint(t3);
          tm[0] = fmaxf(tm[0], t0); tm[1] = fmaxf(tm[1], t1); tm[2] = fmaxf(tm[2], t2); tm[3] = fmaxf(tm[3], t3);
        }
        const float tmax = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
        if (!last || sweeps == 1) {
          const float mn = fmaxf(m, tmax);
          if (extrap) {
            // x holds the earlier tiles' A V-bar relative to the old max: rescale
            // it (TMEM) to the new one; the previous value MMA has completed
            const bool grow = x_started && mn != m;
            if (__syncthreads_or(grow)) {
              tc::tc_fence_after();
              const float f = grow ? tc::ex2(m - mn) : 1.f;
              for (int g = 0; g < D; g += 16) {
                uint32_t xr[16];
                tc::tmem_ld16(tX + lane_off + g, xr);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) xr[e] = __float_as_uint(__uint_as_float(xr[e]) * f);
                tc::tmem_st16(tX + lane_off + g, xr);
              }
              tc::tmem_wait_st();
            }
            for (int j = 0; j < 64; ++j) nseen += sNF[j];
          }
          if (mn == NEG_INF) {  // every parent seen so far is empty: A = 0
#pragma unroll
            for (int e = 0; e < 64; ++e) r[e] = 0u;
          } else {
            float zp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 64; e += 4) {
              const float4 nf = nf4[e >> 2];
              const float a0 = tc::ex2(__uint_as_float(r[e]) - mn), a1 = tc::ex2(__uint_as_float(r[e + 1]) - mn);
              const float a2 = tc::ex2(__uint_as_float(r[e + 2]) - mn), a3 = tc::ex2(__uint_as_float(r[e + 3]) - mn);
              zp[0] = fmaf(a0, nf.x, zp[0]); zp[1] = fmaf(a1, nf.y, zp[1]);
              zp[2] = fmaf(a2, nf.z, zp[2]); zp[3] = fmaf(a3, nf.w, zp[3]);
              if (sweeps == 1) {  // single sweep: keep A = 2^(t - m) in place
                r[e] = __float_as_uint(a0); r[e + 1] = __float_as_uint(a1);
                r[e + 2] = __float_as_uint(a2); r[e + 3] = __float_as_uint(a3);
              }
            }
            z = z * tc::ex2(m - mn) + ((zp[0] + zp[1]) + (zp[2] + zp[3]));
            m = mn;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) r[e] = __float_as_uint(tc::ex2(__uint_as_float(r[e]) - m));
        }
        if (last) {
          // probabilities as bf16, importance column sums of A / z in fp32
          // (A / Z~ with Z~ = z N / N_seen when extrapolating)
          const float rz = !valid || !(z > 0.f) ? 0.f : extrap ? nseen / (*sNtot * z) : 1.f / z;
#pragma unroll
          for (int q = 0; q < 8; ++q) store_chunk8(sPR, tid, q * 8, reinterpret_cast<const float*>(r) + q * 8);
          float v[32];
#pragma unroll
          for (int hgrp = 0; hgrp < 2; ++hgrp) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[hgrp * 32 + e]) * rz;
            sWP[warp * kTile + hgrp * 32 + lane] = reduce_scatter32(v, lane);
          }
        }
      }
      if (last) {
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        wait_vb();
        __syncthreads();
        for (int j = tid; j < n; j += 128)
          sW[c0 + j] += sNF[j] * ((sWP[j] + sWP[kTile + j]) + (sWP[2 * kTile + j] + sWP[3 * kTile + j]));
        if (tid == 0) {
          tc::tc_fence_after();
          issue_values(n, x_started);
        }
        x_started = true;
        wait_mma();
      }
      tc::tc_fence_before();
      __syncthreads();
      if (*sAbort) goto done;
    }
  }

  // ---- top-P over the importance (descending, ties to the lower index) ----
  // rank_j = #{l : w_l > w_j or (w_l == w_j and l < j)}; for M0 <= 64 two
  // threads share each j, each counting over half of the l range
  {
    const int P = a.P;
    if (M0 <= 64) {
      const int j = tid % M0, half = tid / M0;
      if (tid < 2 * M0) {
        const float wj = sW[j];
        const int l0 = half * (M0 >> 1), l1 = half ? M0 : (M0 >> 1);
        int rank = 0;
        for (int l = l0; l < l1; ++l) {
          const float wl = sW[l];
          rank += (wl > wj) || (wl == wj && l < j);
        }
        sRK[half * 128 + j] = rank;
      }
      __syncthreads();
      if (tid < M0) {
        const int rank = sRK[tid] + sRK[128 + tid];
        if (rank < P) sSEL[rank] = tid;
        if (a.importance) a.importance[((size_t)bh * a.nblk + blk) * M0 + tid] = sW[tid];
      }
    } else {
      for (int j = tid; j < M0; j += 128) {
        const float wj = sW[j];
        int rank = 0;
        for (int l = 0; l < M0; ++l) {
          const float wl = sW[l];
          rank += (wl > wj) || (wl == wj && l < j);
        }
        if (rank < P) sSEL[rank] = j;
        if (a.importance) a.importance[((size_t)bh * a.nblk + blk) * M0 + j] = wj;
      }
    }
    __syncthreads();
    if (a.sel)
      for (int r = tid; r < P; r += 128) a.sel[((size_t)bh * a.nblk + blk) * P + r] = sSEL[r];
  }

  // ---- child refinement in chunks of 8 selected parents ----
  if (a.C > 0 && a.P > 0) {
    float mref = m;
    const int nch = (a.P + kChunkParents - 1) / kChunkParents;
    for (int q = 0; q < nch; ++q) {
      // an odd number of parents is padded with a copy of the last one (masked
      // as empty) so that the MMA N stays a multiple of 16
      const int np = min(kChunkParents, a.P - q * kChunkParents);
      const int slots = (np + 1) & ~1;
      const int n = slots * 8;
      if (tid == 0) {
        note(1, ph_cp);
        note(2, ph_vb);
        tc::mbar_arrive_expect_tx(bar_cp, 1u * slots * KH * 1024);
        tc::mbar_arrive_expect_tx(bar_vb, 1u * slots * KH * 1024);
        for (int r = 0; r < slots; ++r) {
          const int p = sSEL[q * kChunkParents + min(r, np - 1)];
          const size_t g = (size_t)(M0 / 8 + p) * KH * 512;
          tc::bulk_g2s(sCW + r * KH * 1024, cw_h + g, KH * 1024, bar_cp);
        }
        for (int r = 0; r < slots; ++r) {
          const int p = sSEL[q * kChunkParents + min(r, np - 1)];
          const size_t g = (size_t)(M0 / 8 + p) * KH * 512;
          tc::bulk_g2s(sVB + r * KH * 1024, vb_bh + g, KH * 1024, bar_vb);
        }
      }
      for (int j = tid; j < kTile; j += 128) {
        const int r = j >> 3;
        sNF[j] = r < np ? (float)__ldg(cnt + M0 + sSEL[q * kChunkParents + r] * 8 + (j & 7)) : 0.f;
      }
      wait_cp(0);
      __syncthreads();
      if (*sAbort) goto done;
      if (tid == 0) {
        tc::tc_fence_after();
        issue_logits(n, 0);
      }
      wait_mma();
      uint32_t r[64];
      tmem_ld64(tS + lane_off, r);
      const float4* nf4 = reinterpret_cast<const float4*>(sNF);
      // row max of the raw logits over non-empty children (the scale is positive)
      float cm[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
      for (int e = 0; e < 64; e += 4) {
        const float4 nf = nf4[e >> 2];
        cm[0] = fmaxf(cm[0], nf.x > 0.f ? __uint_as_float(r[e]) : NEG_INF);
        cm[1] = fmaxf(cm[1], nf.y > 0.f ? __uint_as_float(r[e + 1]) : NEG_INF);
        cm[2] = fmaxf(cm[2], nf.z > 0.f ? __uint_as_float(r[e + 2]) : NEG_INF);
        cm[3] = fmaxf(cm[3], nf.w > 0.f ? __uint_as_float(r[e + 3]) : NEG_INF);
      }
      const float cmax = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3])) * sl2;
      // rare: a child logit far above the reference max -> rescale x and z
      const bool need = cmax > mref + kRescaleLog2;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? tc::ex2(mref - cmax) : 1.f;
        for (int g = 0; g < D; g += 16) {
          uint32_t xr[16];
          tc::tmem_ld16(tX + lane_off + g, xr);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) xr[e] = __float_as_uint(__uint_as_float(xr[e]) * f);
          tc::tmem_st16(tX + lane_off + g, xr);
        }
        tc::tmem_wait_st();
        z *= f;
        if (need) mref = cmax;
      }
      // dA = 2^(t_c - m) - 2^(t_p - m) with t = scale*log2(e)*S and the parent
      // logit t_p the mean of its children's logits (Eq. 8); zero for empty children
      const float nm = -mref, sl8 = sl2 * 0.125f;
      float zp[2] = {0.f, 0.f};
#pragma unroll
      for (int sl = 0; sl < 8; ++sl) {
        float ssum = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ssum += __uint_as_float(r[sl * 8 + e]);
        const float ap = tc::ex2(fmaf(ssum, sl8, nm));
        const float4 na = nf4[sl * 2], nb = nf4[sl * 2 + 1];
        const float nfv[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
        float da[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          da[e] = nfv[e] > 0.f ? tc::ex2(fmaf(__uint_as_float(r[sl * 8 + e]), sl2, nm)) - ap : 0.f;
          zp[e & 1] = fmaf(da[e], nfv[e], zp[e & 1]);
        }
        store_chunk8(sPR, tid, sl * 8, da);
      }
      z += zp[0] + zp[1];
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      wait_vb();
      __syncthreads();
      if (tid == 0) {
        tc::tc_fence_after();
        issue_values(n, true);
      }
      wait_mma();
      tc::tc_fence_before();
      __syncthreads();
      if (*sAbort) goto done;
    }
  }

  // ---- O = x / z -> bf16 -> shared (Q region) -> TMA store ----
  {
    const float iz = 1.f / z;
    for (int g = 0; g < D; g += 16) {
      uint32_t xr[16];
      tc::tmem_ld16(tX + lane_off + g, xr);
      tc::tmem_wait_ld();
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(xr[e]) * iz;
      store_chunk8(sQ, tid, g, v);
      store_chunk8(sQ, tid, g + 8, v + 8);
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
#pragma unroll
      for (int kh = 0; kh < KH; ++kh) tc::tma_store_3d(&omap, sQ + kh * kRows * 128, kh * 64, row0, bh);
      tc::bulk_commit_group();
      tc::bulk_wait_group_read0();
    }
  }

done:
  // nothing in flight before TMEM is freed (the waits return at once for
  // completed operations; 1 ms limit)
  if (issued) {
    uint64_t* const bars[5] = {bar_q, bar_cp, bar_vb, bar_mma, bar_cp1};
#pragma unroll
    for (int b = 0; b < 5; ++b)
      if ((issued >> b) & 1u)
        if (!tc::mbar_wait(bars[b], (exp_par >> b) & 1u, 1000000ull)) atomicOr(a.err, kErrTimeout);
  }
  if (tid == 0) tc::bulk_wait_group_read0();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, S::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Fast path for one parent tile (M0 in {16, 32, 48, 64}, single sweep).
// Same algorithm and data layout as the general kernel above; what changes is
// work skipped because it cannot change the result, and earlier copies:
//   - the parent masks (Eq. 18) are applied only when the block has an empty
//     parent (a block-uniform test);
//   - children: the rescale test uses the unmasked child maximum, so in the
//     common case every 2^(t - m) is at most 2^24 and dA of an empty child is
//     finite; its value sum and count are exactly zero, so it adds nothing to
//     x or z and needs no mask.  Only if the unmasked maximum exceeds the
//     reference by more than 2^24 are the masks applied (and x, z rescaled if
//     the masked maximum does too).  A padding slot (odd number of parents in
//     a chunk) gets a zero value atom for the same reason;
//   - the codewords of chunk q + 1 are copied as soon as the logit MMA of
//     chunk q has read its own, the value sums as soon as its value MMA has;
//   - the value MMAs are not waited for until their operands are reused;
//   - the kernel is persistent: a CTA walks a contiguous range of (head,
//     block) units and fetches the next unit's Q tile and parent codewords as
//     soon as the current unit's last logit MMA has read its own, the parents'
//     value sums as soon as its last value MMA has; the O tile is staged in
//     the PR buffer and its TMA store is waited for only before PR is
//     written again.
template <int D>
struct FastSmem {
  static constexpr int kAtomBytes = 1024 * (D / 64);       // one 8-code atom group
  static constexpr int kQ = 0;                             // Q tile
  static constexpr int kCW = kQ + kRows * D * 2;           // codewords: parents, then chunks
  static constexpr int kVB = kCW + 8 * kAtomBytes;         // value sums: parents, then chunks
  static constexpr int kPR = kVB + 8 * kAtomBytes;         // probabilities / dA [128][64] bf16; O staging
  static constexpr int kNF = kPR + kRows * D * 2;          // counts [2][64]: parents, current chunk
  static constexpr int kW = kNF + 2 * 64 * 4;              // ranking keys [64]
  static constexpr int kWP = kW + 64 * 4;                  // per-warp partial sums [4][64]
  static constexpr int kSEL = kWP + 4 * 64 * 4;            // selected parents [64]
  static constexpr int kCNT = kSEL + 64 * 4;               // counts of the unit's head [Mt <= 576]
  static constexpr int kBAR = kCNT + 576 * 4;              // 5 mbarriers
  static constexpr int kMISC = kBAR + 64;                  // tmem base, abort flag
  static constexpr int kTotal = kMISC + 32;
  static constexpr uint32_t kTmemCols = D == 64 ? 128 : 256;  // logits [64] + output [D]
};

// MMAs are issued by one elected lane of a warp (issuing takes 60-90 cycles
// per instruction): the logit MMAs by warp 0, the value MMAs by warp 3, so
// that the two overlap each other and the waits that thread 0 takes.

// Of each selected parent's 8 child exponentials, the first 2 * kPolyPairs
// are evaluated on the FMA pipe (fm::exp2_poly2), the others on the
// special-function unit, so that neither pipe alone bounds the child pass.
constexpr int kPolyPairs = 1;

template <int D, int M0>
__global__ void __launch_bounds__(128, D == 64 ? 4 : 2) attention_fast_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap, const AttnArgs a) {
  using S = FastSmem<D>;
  constexpr int KH = D / 64;
  constexpr int AB = S::kAtomBytes;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + S::kQ;
  uint8_t* sCW = sm + S::kCW;
  uint8_t* sVB = sm + S::kVB;
  uint8_t* sPR = sm + S::kPR;
  float* sNF = reinterpret_cast<float*>(sm + S::kNF);  // [0..63] parents, [64..127] current chunk
  uint32_t* sKEY = reinterpret_cast<uint32_t*>(sm + S::kW);  // importance ranking keys [64]
  float* sWP = reinterpret_cast<float*>(sm + S::kWP);
  int* sSEL = reinterpret_cast<int*>(sm + S::kSEL);
  const int32_t* sCNT = reinterpret_cast<const int32_t*>(sm + S::kCNT);
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(sm + S::kBAR);
  uint64_t* bar_cw = bar_q + 1;   // parents' codewords and the head's counts
  uint64_t* bar_vb = bar_q + 2;   // parents' value sums
  uint64_t* bar_mma = bar_q + 3;  // logit MMAs
  uint64_t* bar_x = bar_q + 4;    // value MMAs
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + S::kMISC);
  int* sAbort = reinterpret_cast<int*>(sm + S::kMISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = a.C, Mt = M0 * (1 + C), P = a.P;
  const float NEG_INF = __int_as_float(0xff800000);
  const float sl2 = a.scale_log2;
  const float2 sl2x2 = fm::f2(sl2, sl2);
  // this CTA's contiguous range of units u = bh * nblk + block
  const int total = a.BH * a.nblk;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int u0 = blockIdx.x * per, u1 = min(total, u0 + per);
  if (u0 >= u1) return;
  const int nch = (C > 0 && P > 0) ? (P + kChunkParents - 1) / kChunkParents : 0;
  auto unit_cw = [&](int u) { return a.cw + (size_t)((u / a.nblk) % a.H) * (Mt / 8) * KH * 512; };
  auto unit_vb = [&](int u) { return a.vb + (size_t)(u / a.nblk) * (Mt / 8) * KH * 512; };
  // mbarrier phases (the same in every thread), and per barrier the parity
  // of the phase that the last operation issued by this thread completes
  // (bit b of `issued` set once one was issued): on the way out the kernel
  // waits, with a limit, for those, so no copy or MMA is in flight when it
  // frees TMEM and returns, also after a timed-out wait
  constexpr int kBars = 5;
  uint32_t ph = 0;  // bit b: parity of barrier b's next phase
  uint32_t issued = 0, exp_par = 0;
  auto note = [&](int b) {
    issued |= 1u << b;
    exp_par = (exp_par & ~(1u << b)) | (ph & (1u << b));
  };
  // the next unit's Q tile and parents' codewords / value sums (thread 0)
  auto load_q = [&](int u) {
    note(0);
    tc::mbar_arrive_expect_tx(bar_q, kRows * D * 2);
#pragma unroll
    for (int kh = 0; kh < KH; ++kh)
      tc::tma_load_3d(sQ + kh * kRows * 128, &qmap, kh * 64, (u % a.nblk) * kRows, u / a.nblk, bar_q);
  };
  auto load_pcw = [&](int u) {
    note(1);
    tc::mbar_arrive_expect_tx(bar_cw, M0 * D * 2 + Mt * 4);
    tc::bulk_g2s(sCW, unit_cw(u), M0 * D * 2, bar_cw);
    tc::bulk_g2s(sm + S::kCNT, a.counts + (size_t)(u / a.nblk) * Mt, Mt * 4, bar_cw);
  };
  auto load_pvb = [&](int u) {
    note(2);
    tc::mbar_arrive_expect_tx(bar_vb, M0 * D * 2);
    tc::bulk_g2s(sVB, unit_vb(u), M0 * D * 2, bar_vb);
  };

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i) tc::mbar_init(bar_q + i, 1);
    tc::fence_mbar_init();
    *sAbort = 0;
  }
  if (warp == 0) {
    tc::tmem_alloc(sTmem, S::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();  // barriers initialised before anyone waits on them
  tc::tc_fence_after();
  if (tid == 0) {
    tc::prefetch_tensormap(&qmap);
    tc::prefetch_tensormap(&omap);
  }
  // images and counts of the preparation before; Q too, since the launch
  // that wrote it may have ended only just before that preparation began
  grid_dependency_wait();
  if (tid == 0) {
    load_q(u0);
    load_pcw(u0);
    load_pvb(u0);
  }
  {
    const uint32_t tmem = *sTmem;
    const uint32_t tS = tmem;          // logits
    const uint32_t tX = tmem + kTile;  // output accumulator, D columns
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t sQa = tc::smem_u32(sQ), sCWa = tc::smem_u32(sCW), sVBa = tc::smem_u32(sVB),
                   sPRa = tc::smem_u32(sPR);
    const uint32_t idesc_x = tc::idesc_bf16(kRows, D, 0, 1);

    auto issue_logits = [&](int n) {  // S = Q * CW^T over n codes
      note(3);
      const uint32_t idesc = tc::idesc_bf16(kRows, n, 0, 0);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint64_t ad = tc::sdesc_sw128(sQa + (k >> 2) * (kRows * 128) + (k & 3) * 32, 16, 1024);
        const uint64_t bd = tc::sdesc_sw128(sCWa + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
        tc::mma_bf16(tS, ad, bd, idesc, k > 0);
      }
      tc::mma_commit(bar_mma);
    };
    // x (+)= PR[:, 16 k0 ..] * VB over n codes (K steps k0 .. k0 + n/16)
    auto issue_values = [&](int n, int k0, bool acc, uint64_t* bar, int b) {
      note(b);
      for (int k = k0; k < k0 + n / 16; ++k) {
        const uint64_t ad = tc::sdesc_sw128(sPRa + (k & 3) * 32, 16, 1024);
        const uint64_t bd = tc::sdesc_sw128(sVBa + k * 2 * AB, 1024, KH * 1024);
        tc::mma_bf16(tX, ad, bd, idesc_x, (acc || k > k0) ? 1u : 0u);
      }
      tc::mma_commit(bar);
    };
    // Waits are taken by thread 0 alone; the others meet it at the CTA barrier
    // that follows every wait, so no warp spins on the issue slots.
    auto wait_bar = [&](int b) {
      if (tid == 0 && !tc::mbar_wait(bar_q + b, (ph >> b) & 1u)) fail(a.err, sAbort);
      ph ^= 1u << b;
    };
    // child atoms of chunk q (codewords or value sums) into the staging
    // buffer: `slots` atoms, slot i from selected parent min(i, np - 1), as
    // 16-byte cp.async pieces spread over all threads, one commit group.  An
    // odd parent count is padded with a copy of the last parent's codewords
    // (and zero value sums), so that the MMAs' N and K are multiples of 16.
    auto chunk_np = [&](int q) { return min(kChunkParents, P - q * kChunkParents); };
    auto chunk_slots = [&](int q) { return (chunk_np(q) + 1) & ~1; };
    // thread t copies the 16-byte pieces t, t + 128, ... : always the same
    // piece offset of every (128 / kPieces)-th atom
    constexpr int kPieces = AB / 16;               // 64 (d = 64) or 128 (d = 128)
    constexpr int kAtomStep = 128 / kPieces;       // atoms advanced per round of 128 pieces
    const int my_off = (tid % kPieces) * 16, my_sl0 = tid / kPieces;
    auto copy_atoms = [&](uint8_t* dst, const bf16* src_h, int q, int slots) {
      const int np = chunk_np(q);
      const int* selq = sSEL + q * kChunkParents;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(src_h) + (size_t)(M0 / 8) * AB + my_off;
      uint8_t* d0 = dst + my_off;
#pragma unroll
      for (int r = 0; r < kChunkParents / kAtomStep; ++r) {
        const int sl = my_sl0 + r * kAtomStep;
        if (sl < slots) tc::cp_async16(d0 + sl * AB, src + (size_t)selq[min(sl, np - 1)] * AB);
      }
      tc::cp_async_commit();
    };
    auto copy_cw = [&](int q, const bf16* cw_h) { copy_atoms(sCW, cw_h, q, chunk_slots(q)); };
    auto copy_vb = [&](int q, const bf16* vb_bh) { copy_atoms(sVB, vb_bh, q, chunk_np(q)); };

    for (int u = u0; u < u1; ++u) {
    const int bh = u / a.nblk, blk = u % a.nblk;
    const int row0 = blk * kRows;
    const bool valid = row0 + tid < a.N;
    const bf16* cw_h = unit_cw(u);
    const bf16* vb_bh = unit_vb(u);
    const bool has_next = u + 1 < u1;
    wait_bar(0);  // Q
    wait_bar(1);  // parents' codewords and counts
    __syncthreads();
    float nfj = 0.f;
    if (tid < M0) {
      nfj = (float)sCNT[tid];
      sNF[tid] = nfj;
    }
    tc::tc_fence_before();
    const bool any_empty = __syncthreads_or(tid < M0 && !(nfj > 0.f)) != 0;
    tc::tc_fence_after();
    if (*sAbort) goto done;

    // ---- parents: logits, masked max, A = 2^(t - m), z, importance ----
    if (warp == 0) {
      if (tc::elect_one()) {
        tc::tc_fence_after();
        issue_logits(M0);
      }
      __syncwarp();
    }
    wait_bar(3);
    if (tid == 0) {
      tc::bulk_wait_group_read0();  // the previous unit's O store has read its staging (PR)
      if (nch == 0 && has_next) {   // Q and the parents' codewords are read: next unit's
        load_q(u + 1);
        load_pcw(u + 1);
      }
    }
    __syncthreads();
    tc::tc_fence_after();
    float m, z;
    {
      // the row's logits are read from TMEM twice: all M0 at once (one wait)
      // for the maximum, then 32 at a time for A = 2^(t - m) (to PR in bf16,
      // and back over the logits in fp32 for the importance, which needs
      // 1 / z of the whole row)
      const float4* nf4 = reinterpret_cast<const float4*>(sNF);
      float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
      for (int c0 = 0; c0 < M0; c0 += 32) {  // columns c0 .. min(c0 + 32, M0) - 1
        constexpr int W = M0 < 32 ? M0 : 32;
        uint32_t r[W];
#pragma unroll
        for (int g = 0; g < W / 16; ++g)
          if (c0 + g * 16 < M0) tc::tmem_ld16(tS + lane_off + c0 + g * 16, r + g * 16);
        tc::tmem_wait_ld();
        const float* t = reinterpret_cast<const float*>(r);
        if (!any_empty) {
#pragma unroll
          for (int e = 0; e < W; e += 4) {
            if (c0 + e >= M0) break;
            mx0 = fm::max3(mx0, t[e], t[e + 1]);
            mx1 = fm::max3(mx1, t[e + 2], t[e + 3]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < W; e += 4) {
            if (c0 + e >= M0) break;
            const float4 nf = nf4[(c0 + e) >> 2];
            mx0 = fm::max3(mx0, nf.x > 0.f ? t[e] : NEG_INF, nf.y > 0.f ? t[e + 1] : NEG_INF);
            mx1 = fm::max3(mx1, nf.z > 0.f ? t[e + 2] : NEG_INF, nf.w > 0.f ? t[e + 3] : NEG_INF);
          }
        }
      }
      m = fmaxf(mx0, mx1) * sl2;
      const float2 nm2 = fm::f2(-m, -m);
      float2 zp = fm::f2(0.f, 0.f);
      auto a_pass = [&](auto masked_t) {
        constexpr bool kMasked = decltype(masked_t)::value;
#pragma unroll
        for (int g2 = 0; g2 < M0 / 16; g2 += 2) {
          uint32_t r[32];
          tc::tmem_ld16(tS + lane_off + g2 * 16, r);
          if (g2 + 1 < M0 / 16) tc::tmem_ld16(tS + lane_off + g2 * 16 + 16, r + 16);
          tc::tmem_wait_ld();
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int g = g2 + gg;
            if (g < M0 / 16) {
              uint32_t* rg = r + gg * 16;
#pragma unroll
              for (int e = 0; e < 16; e += 4) {
                const float4 nf = nf4[(g * 16 + e) >> 2];
                const float2 x01 = fm::fma2(fm::f2(__uint_as_float(rg[e]), __uint_as_float(rg[e + 1])), sl2x2, nm2);
                const float2 x23 = fm::fma2(fm::f2(__uint_as_float(rg[e + 2]), __uint_as_float(rg[e + 3])), sl2x2, nm2);
                float a0 = tc::ex2(x01.x), a1 = tc::ex2(x01.y), a2 = tc::ex2(x23.x), a3 = tc::ex2(x23.y);
                if (kMasked) {
                  a0 = nf.x > 0.f ? a0 : 0.f;
                  a1 = nf.y > 0.f ? a1 : 0.f;
                  a2 = nf.z > 0.f ? a2 : 0.f;
                  a3 = nf.w > 0.f ? a3 : 0.f;
                }
                zp = fm::fma2(fm::f2(a0, a1), fm::f2(nf.x, nf.y), zp);
                zp = fm::fma2(fm::f2(a2, a3), fm::f2(nf.z, nf.w), zp);
                rg[e] = __float_as_uint(a0);
                rg[e + 1] = __float_as_uint(a1);
                rg[e + 2] = __float_as_uint(a2);
                rg[e + 3] = __float_as_uint(a3);
              }
              store_chunk8(sPR, tid, g * 16, reinterpret_cast<const float*>(rg));
              store_chunk8(sPR, tid, g * 16 + 8, reinterpret_cast<const float*>(rg) + 8);
              tc::tmem_st16(tS + lane_off + g * 16, rg);
            }
          }
        }
      };
      if (any_empty)
        a_pass(std::true_type{});
      else
        a_pass(std::false_type{});
      tc::tmem_wait_st();
      z = zp.x + zp.y;
      // importance column sums of A / z (Eq. 7), fp32.  The A values are read
      // back in the 16x256b shape, in which each thread holds two adjacent
      // columns of four rows of its warp (rows l/4, l/4 + 8 of each 16-lane
      // half); the four rows' 1/z are scaled in, then a three-step butterfly
      // reduce-scatter over the lanes that share l % 4 leaves lane l holding
      // the warp's sums of columns 2l and 2l + 1.
      const float rz = valid ? 1.f / z : 0.f;
      const int rl = lane >> 2;
      const float z0 = __shfl_sync(0xffffffffu, rz, rl), z1 = __shfl_sync(0xffffffffu, rz, rl + 8),
                  z2 = __shfl_sync(0xffffffffu, rz, rl + 16), z3 = __shfl_sync(0xffffffffu, rz, rl + 24);
      float2 cs[8];
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        if (hc * 32 < M0) {
          uint32_t lo[16], hi[16];
          fm::tmem_ld_16x256b_x4(tS + lane_off + hc * 32, lo);                // rows l/4, l/4 + 8
          fm::tmem_ld_16x256b_x4(tS + lane_off + (16u << 16) + hc * 32, hi);  // rows 16 + l/4, 24 + l/4
          tc::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int grp = hc * 4 + k;
            float2 s = fm::mul2(fm::f2(__uint_as_float(lo[4 * k]), __uint_as_float(lo[4 * k + 1])), fm::f2(z0, z0));
            s = fm::fma2(fm::f2(__uint_as_float(lo[4 * k + 2]), __uint_as_float(lo[4 * k + 3])), fm::f2(z1, z1), s);
            s = fm::fma2(fm::f2(__uint_as_float(hi[4 * k]), __uint_as_float(hi[4 * k + 1])), fm::f2(z2, z2), s);
            s = fm::fma2(fm::f2(__uint_as_float(hi[4 * k + 2]), __uint_as_float(hi[4 * k + 3])), fm::f2(z3, z3), s);
            cs[grp] = grp * 8 < M0 ? s : fm::f2(0.f, 0.f);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) cs[hc * 4 + k] = fm::f2(0.f, 0.f);
        }
      }
      // reduce-scatter: lane bit 4 splits groups 0-3 / 4-7, bit 3 the pairs,
      // bit 2 the last two; lane l ends with group l / 4
#pragma unroll
      for (int step = 0; step < 3; ++step) {
        const int half = 4 >> step, bit = 16 >> step;
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float2 send = up ? cs[i] : cs[i + half];
          const float2 keep = up ? cs[i + half] : cs[i];
          const float rx = __shfl_xor_sync(0xffffffffu, send.x, bit);
          const float ry = __shfl_xor_sync(0xffffffffu, send.y, bit);
          cs[i] = fm::add2(keep, fm::f2(rx, ry));
        }
      }
      *reinterpret_cast<float2*>(sWP + warp * 64 + 2 * lane) = cs[0];
    }
    tc::fence_proxy_async_smem();
    wait_bar(2);  // parents' value sums
    tc::tc_fence_before();
    __syncthreads();
    if (*sAbort) goto done;
    // ranking key of parent j: its importance with the 6 lowest mantissa bits
    // replaced by 63 - j (importances are >= 0, so the unsigned order of the
    // bits is the order of the values; equal values rank the lower index
    // first).  The importance reported is the key's value part (relative
    // change below 2^-17).
    if (tid < M0) {
      const float wj = nfj * ((sWP[tid] + sWP[64 + tid]) + (sWP[128 + tid] + sWP[192 + tid]));
      sKEY[tid] = (__float_as_uint(wj) & ~63u) | (uint32_t)(63 - tid);
    }
    __syncthreads();
    // ---- top-P over the importance (descending, ties to the lower index) ----
    // thread j < M0 of the first two warps ranks parent j against all keys,
    // while the last warp issues the parents' value MMA
    if (tid < M0) {
      const uint32_t kj = sKEY[tid];
      int r0 = 0, r1 = 0;
#pragma unroll
      for (int l = 0; l < M0; l += 8) {
        const uint4 ka = *reinterpret_cast<const uint4*>(sKEY + l);
        const uint4 kb = *reinterpret_cast<const uint4*>(sKEY + l + 4);
        r0 += (ka.x > kj) + (ka.y > kj) + (ka.z > kj) + (ka.w > kj);
        r1 += (kb.x > kj) + (kb.y > kj) + (kb.z > kj) + (kb.w > kj);
      }
      const int rank = r0 + r1;
      if (rank < P) {
        sSEL[rank] = tid;
        if (a.sel) a.sel[((size_t)bh * a.nblk + blk) * P + rank] = tid;
      }
      if (a.importance) a.importance[((size_t)bh * a.nblk + blk) * M0 + tid] = __uint_as_float(kj & ~63u);
    }
    if (warp == 3) {
      if (tc::elect_one()) {
        tc::tc_fence_after();
        issue_values(M0, 0, false, bar_x, 4);
      }
      __syncwarp();
    }
    __syncthreads();

    // ---- child refinement in chunks of 8 selected parents ----
    // Chunk q: its codewords were copied during chunk q - 1 (chunk 0's right
    // after the selection), its logit MMA issued as soon as they and the
    // logit region were free; the chunk's value sums are copied, and the next
    // chunk's codewords, while its dA pass runs.
    float mref = m;
    if (nch > 0) {
      copy_cw(0, cw_h);  // the parent logit MMA has read the parents' codewords
      tc::cp_async_wait<0>();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncthreads();
      if (warp == 0) {
        if (tc::elect_one()) {
          tc::tc_fence_after();
          issue_logits(chunk_slots(0) * 8);
        }
        __syncwarp();
      }
    }
    for (int q = 0; q < nch; ++q) {
      const int np = chunk_np(q);
      const int n = chunk_slots(q) * 8;
      float* nfc = sNF + 64;
      if (tid < 64) {
        const int rr = tid >> 3;
        nfc[tid] = rr < np ? (float)sCNT[M0 + sSEL[q * kChunkParents + rr] * 8 + (tid & 7)] : 0.f;
      }
      wait_bar(3);  // this chunk's logits
      wait_bar(4);  // the previous value MMA (the parents' at q = 0) has read PR and VB
      if (tid == 0 && q + 1 == nch && has_next) {  // the last logit MMA: Q and CW are free
        load_q(u + 1);
        load_pcw(u + 1);
      }
      __syncthreads();
      tc::tc_fence_after();
      copy_vb(q, vb_bh);
      if (q + 1 < nch) copy_cw(q + 1, cw_h);  // this chunk's logits are done
      // dA = 2^(t_c - m) - 2^(t_p - m), t_p the mean of the 8 child logits
      // (Eq. 8), with m the parents' maximum; the unmasked child maximum is
      // taken on the way.  Empty children need no mask while every 2^(t - m)
      // stays below 2^24: their value sums and counts are exactly zero.  The
      // first kPolyPairs pairs of each parent's children take 2^x on the FMA
      // pipe, the others on the special-function unit.
      const float4* nf4 = reinterpret_cast<const float4*>(nfc);
      float2 zc = fm::f2(0.f, 0.f);
      float cm0 = NEG_INF, cm1 = NEG_INF;
      auto da_pass = [&](auto masked_t, float mr) {
        constexpr bool kMasked = decltype(masked_t)::value;
        const float nm = -mr, sl8 = sl2 * 0.125f;
        const float2 nm2 = fm::f2(nm, nm);
#pragma unroll
        for (int g2 = 0; g2 < 4; g2 += 2) {
          if (g2 * 16 < n) {
            uint32_t r[32];
            tc::tmem_ld16(tS + lane_off + g2 * 16, r);
            if (g2 * 16 + 16 < n) tc::tmem_ld16(tS + lane_off + g2 * 16 + 16, r + 16);
            tc::tmem_wait_ld();
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
              const int sl = 2 * g2 + s4;  // parent slot
              if (sl * 8 < n) {
                const float* tt = reinterpret_cast<const float*>(r) + s4 * 8;
                if (!kMasked) {
                  cm0 = fm::max3(cm0, tt[0], tt[1]);
                  cm1 = fm::max3(cm1, tt[2], tt[3]);
                  cm0 = fm::max3(cm0, tt[4], tt[5]);
                  cm1 = fm::max3(cm1, tt[6], tt[7]);
                }
                const float2 s01 = fm::add2(fm::f2(tt[0], tt[1]), fm::f2(tt[2], tt[3]));
                const float2 s45 = fm::add2(fm::f2(tt[4], tt[5]), fm::f2(tt[6], tt[7]));
                const float2 sm2 = fm::add2(s01, s45);
                const float ap = tc::ex2(fmaf(sm2.x + sm2.y, sl8, nm));
                const float2 nap = fm::f2(-ap, -ap);
                const float4 na = nf4[sl * 2], nb = nf4[sl * 2 + 1];
                const float nfv[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
                uint4 pk;
                uint32_t* pkw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                  const float2 x = fm::fma2(fm::f2(tt[e], tt[e + 1]), sl2x2, nm2);
                  float2 ev;
                  if (e < 2 * kPolyPairs) {
                    ev = fm::exp2_poly2(x);
                  } else {
                    ev = fm::f2(tc::ex2(x.x), tc::ex2(x.y));
                  }
                  float2 da = fm::add2(ev, nap);
                  if (kMasked) {
                    da.x = nfv[e] > 0.f ? da.x : 0.f;
                    da.y = nfv[e + 1] > 0.f ? da.y : 0.f;
                  }
                  zc = fm::fma2(da, fm::f2(nfv[e], nfv[e + 1]), zc);
                  pkw[e >> 1] = pack_bf16x2(da.x, da.y);
                }
                *reinterpret_cast<uint4*>(sPR + tc::sw128_offset(tid, sl * 8)) = pk;
              }
            }
          }
        }
      };
      da_pass(std::false_type{}, mref);
      if (np & 1)  // padding slot: zero value sums, so it adds nothing
        for (int i = tid; i < AB / 16; i += 128)
          reinterpret_cast<uint4*>(sVB + np * AB)[i] = make_uint4(0, 0, 0, 0);
      tc::cp_async_wait<0>();  // this chunk's value sums and the next chunk's codewords
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      const float cmax_any = fmaxf(cm0, cm1) * sl2;
      if (__syncthreads_or(cmax_any > mref + kRescaleLog2)) {  // block-uniform, rare
        // masked maximum over non-empty children; rescale x and z if it is far
        // above the reference, then dA again with the masks applied
        tc::tc_fence_after();
        float cmm0 = NEG_INF, cmm1 = NEG_INF;
        for (int g = 0; g < 4; ++g) {
          if (g * 16 < n) {
            uint32_t r[16];
            tc::tmem_ld16(tS + lane_off + g * 16, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              cmm0 = fmaxf(cmm0, nfc[g * 16 + e] > 0.f ? __uint_as_float(r[e]) : NEG_INF);
              cmm1 = fmaxf(cmm1, nfc[g * 16 + e + 1] > 0.f ? __uint_as_float(r[e + 1]) : NEG_INF);
            }
          }
        }
        const float cmax = fmaxf(cmm0, cmm1) * sl2;
        const bool need = cmax > mref + kRescaleLog2;
        if (__syncthreads_or(need)) {
          tc::tc_fence_after();
          const float f = need ? tc::ex2(mref - cmax) : 1.f;
          for (int g = 0; g < D; g += 16) {
            uint32_t xr[16];
            tc::tmem_ld16(tX + lane_off + g, xr);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) xr[e] = __float_as_uint(__uint_as_float(xr[e]) * f);
            tc::tmem_st16(tX + lane_off + g, xr);
          }
          tc::tmem_wait_st();
          z *= f;
          if (need) mref = cmax;
        }
        zc = fm::f2(0.f, 0.f);
        da_pass(std::true_type{}, mref);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
      }
      z += zc.x + zc.y;
      if (*sAbort) goto done;
      if (warp == 3) {  // this chunk's value MMA
        if (tc::elect_one()) {
          tc::tc_fence_after();
          issue_values(n, 0, true, bar_x, 4);
        }
        __syncwarp();
      } else if (warp == 0 && q + 1 < nch) {  // the next chunk's logits (its codewords are in)
        if (tc::elect_one()) {
          tc::tc_fence_after();
          issue_logits(chunk_slots(q + 1) * 8);
        }
        __syncwarp();
      }
    }
    wait_bar(4);  // the last value MMA (the parents' when there are no chunks)
    if (tid == 0 && has_next) load_pvb(u + 1);
    __syncthreads();
    tc::tc_fence_after();

    // ---- O = x / z -> bf16 -> shared (PR region) -> TMA store (waited for
    //      only before the staging is written again) ----
    {
      const float iz = 1.f / z;
      const float2 iz2 = fm::f2(iz, iz);
#pragma unroll
      for (int g = 0; g < D; g += 16) {
        uint32_t xr[16];
        tc::tmem_ld16(tX + lane_off + g, xr);
        tc::tmem_wait_ld();
        float v[16];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float2 o = fm::mul2(fm::f2(__uint_as_float(xr[e]), __uint_as_float(xr[e + 1])), iz2);
          v[e] = o.x;
          v[e + 1] = o.y;
        }
        store_chunk8(sPR, tid, g, v);
        store_chunk8(sPR, tid, g + 8, v + 8);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) tc::tma_store_3d(&omap, sPR + kh * kRows * 128, kh * 64, row0, bh);
        tc::bulk_commit_group();
      }
    }
    }  // units
  }
done:
  // nothing of this CTA in flight before TMEM is freed: copies and MMAs this
  // thread issued (the waits return at once for completed ones; 1 ms limit)
  if (issued) {
#pragma unroll
    for (int b = 0; b < kBars; ++b)
      if ((issued >> b) & 1u)
        if (!tc::mbar_wait(bar_q + b, (exp_par >> b) & 1u, 1000000ull)) atomicOr(a.err, kErrTimeout);
  }
  tc::cp_async_wait<0>();
  if (tid == 0) tc::bulk_wait_group_read0();  // the last O store has read the staging
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(*sTmem, S::kTmemCols);
  }
}


// Codewords and value sums -> bf16 images of swizzled atoms.  Code a of a head
// (parents first, then child c of parent p at M0 + p*C + c) lands in atom
// a/8, row a%8; for d = 128 each atom group holds two 64-column halves.
template <int D>
__global__ void __launch_bounds__(256) attention_prep_kernel(const bf16* __restrict__ parents,
                                                             const bf16* __restrict__ children,
                                                             const float* __restrict__ vsum,
                                                             bf16* __restrict__ cw, bf16* __restrict__ vb,
                                                             int H, int BH, int M0, int C) {
  constexpr int KH = D / 64;
  allow_dependents();  // the attention's set-up and first Q tile may overlap this launch
  grid_dependency_wait();  // the statistics of the launches before; the images may still be read
  const int Mt = M0 * (1 + C);
  const int chunks_per_code = D / 8;
  const long long n_cw = (long long)H * Mt * chunks_per_code;
  const long long n_vb = (long long)BH * Mt * chunks_per_code;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < n_cw + n_vb;
       g += (long long)gridDim.x * blockDim.x) {
    const bool is_cw = g < n_cw;
    const long long u = is_cw ? g : g - n_cw;
    const int chunk = (int)(u % chunks_per_code);
    const long long hc = u / chunks_per_code;
    const int code = (int)(hc % Mt);
    const long long head = hc / Mt;  // h for codewords, bh for value sums
    float v[8];
    if (is_cw) {
      const bf16* src = code < M0 ? parents + ((size_t)head * M0 + code) * D
                                  : children + ((size_t)head * M0 * C + (code - M0)) * D;
      load8(src + chunk * 8, v);
    } else {
      load8(vsum + ((size_t)head * Mt + code) * D + chunk * 8, v);
    }
    const int kh = chunk >> 3, c = chunk & 7, r = code & 7;
    bf16* dst = (is_cw ? cw : vb) + (((size_t)head * (Mt / 8) + (code >> 3)) * KH + kh) * 512 + r * 64 +
                ((c ^ r) * 8);
    store8(dst, v);
  }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <int D, int M0>
cudaError_t launch_fast_m(dim3 grid, const CUtensorMap& qmap, const CUtensorMap& omap, const AttnArgs& a,
                          cudaStream_t st) {
  const int smem = FastSmem<D>::kTotal + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(attention_fast_kernel<D, M0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // persistent: as many CTAs as fit at once (TMEM and registers allow four
  // per SM at d = 64, two at d = 128), each walking a contiguous range of
  // (head, block) units so that it can fetch the next unit's operands early
  constexpr int kCtasPerSm = D == 64 ? 4 : 2;
  const long long units = (long long)grid.x * grid.y;
  grid = dim3((unsigned)std::max<long long>(1, std::min<long long>(units, (long long)num_sms() * kCtasPerSm)));
  e = launch_after(attention_fast_kernel<D, M0>, dim3(grid), dim3(128), smem, st, qmap, omap, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_fast(int M0, dim3 grid, const CUtensorMap& qmap, const CUtensorMap& omap, const AttnArgs& a,
                        cudaStream_t st) {
  switch (M0) {
    case 16: return launch_fast_m<D, 16>(grid, qmap, omap, a, st);
    case 32: return launch_fast_m<D, 32>(grid, qmap, omap, a, st);
    case 48: return launch_fast_m<D, 48>(grid, qmap, omap, a, st);
    default: return launch_fast_m<D, 64>(grid, qmap, omap, a, st);
  }
}

}  // namespace

bool attention_tc_supported(const Shape& s, avq_dtype dt, int P, int block, int /*two_pass*/) {
  if (dt != AVQ_BF16 || block != 128) return false;
  if (s.d != 64 && s.d != 128) return false;
  if (s.M0 % 16 != 0 || s.M0 > 256) return false;
  if (s.C != 0 && s.C != 8) return false;
  (void)P;
  return true;
}

size_t attention_tc_workspace(const Shape& s, int, int, int) {
  return align256((size_t)s.H * s.Mt() * s.d * 2) + align256((size_t)s.BH() * s.Mt() * s.d * 2);
}

cudaError_t launch_attention_tc(const Shape& s, const void* Q, const void* parents,
                                const void* children, const float* vsum, const int32_t* counts,
                                int P, int block, float scale, int two_pass, void* O,
                                int32_t* sel, float* importance, void* ws, unsigned int* err,
                                cudaStream_t st, LaunchLog& log) {
  (void)block;
  bf16* cw = static_cast<bf16*>(ws);
  bf16* vb = reinterpret_cast<bf16*>(static_cast<char*>(ws) + align256((size_t)s.H * s.Mt() * s.d * 2));
  const long long work = (long long)(s.H + s.BH()) * s.Mt() * (s.d / 8);
  const int pblocks = (int)std::min<long long>((work + 255) / 256, (long long)num_sms() * 8);
  cudaError_t e;
  if (s.d == 64)
    e = launch_after(attention_prep_kernel<64>, dim3(pblocks), dim3(256), 0, st, (const bf16*)parents,
                     (const bf16*)children, vsum, cw, vb, s.H, s.BH(), s.M0, s.C);
  else
    e = launch_after(attention_prep_kernel<128>, dim3(pblocks), dim3(256), 0, st, (const bf16*)parents,
                     (const bf16*)children, vsum, cw, vb, s.H, s.BH(), s.M0, s.C);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  log.add("attention_prep");

  CUtensorMap qmap, omap;
  e = make_tmap_3d_bf16(&qmap, Q, s.d, s.N, s.BH(), 64, kRows);
  if (e != cudaSuccess) return e;
  e = make_tmap_3d_bf16(&omap, O, s.d, s.N, s.BH(), 64, kRows);
  if (e != cudaSuccess) return e;

  AttnArgs a;
  a.cw = cw;
  a.vb = vb;
  a.counts = counts;
  a.sel = sel;
  a.importance = importance;
  a.err = err;
  a.H = s.H;
  a.N = s.N;
  a.M0 = s.M0;
  a.C = s.C;
  a.P = P;
  a.nblk = (s.N + kRows - 1) / kRows;
  a.BH = s.BH();
  a.two_pass = two_pass;
  a.scale_log2 = scale * 1.4426950408889634f;
  dim3 grid(a.nblk, s.BH());
  if (!two_pass && s.M0 <= 64) {  // one parent tile: the fast kernel
    e = s.d == 64 ? launch_fast<64>(s.M0, grid, qmap, omap, a, st) : launch_fast<128>(s.M0, grid, qmap, omap, a, st);
    log.add("attention_tc_fast");
    return e;
  }
  if (s.d == 64) {
    const int smem = Smem<64>::kTotal + 1024;
    e = cudaFuncSetAttribute(attention_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_after(attention_tc_kernel<64>, grid, dim3(128), smem, st, qmap, omap, a);
    if (e != cudaSuccess) return e;
  } else {
    const int smem = Smem<128>::kTotal + 1024;
    e = cudaFuncSetAttribute(attention_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_after(attention_tc_kernel<128>, grid, dim3(128), smem, st, qmap, omap, a);
    if (e != cudaSuccess) return e;
  }
  log.add("attention_tc");
  return cudaGetLastError();
}

}  // namespace avq

