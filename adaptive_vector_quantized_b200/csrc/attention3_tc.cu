// Stage 2 over a depth-3 tree on the tcgen05 tensor cores ("AVQ-Attention:
// Adaptive Vector-Quantized Attention", Algorithm 2 of Sec. 4.3 applied a
// second time one level down, the deeper hierarchies of Sec. 6; Eqs. 6-9;
// the masked maximum of Sec. D).
//
// One CTA per (head, block of 128 queries), 4 warps; thread i owns query row
// i, TMEM lane i.  TMEM: logits (128 columns) and the output accumulator x
// (D columns).  Per block:
//   parents        S = Q P^T into TMEM; masked max (Eq. 18), A = 2^(t - m)
//                  with t the log2-domain logit, z = sum A n, the importance
//                  column sums (Eq. 7); top-P; x = A Vbar_p.
//   children       the P <= 16 selected parents' 8 children each, one MMA of
//                  N <= 128: dA = 2^(t_c - m) - 2^(t_p - m), t_p the mean of
//                  the parent's 8 child logits (Eq. 8), zero for empty
//                  children (Eq. 9); x += dA Vbar_c, z += dA n_c.
//   child ranking  w_c = n_c sum_i 2^(t_ic - m_i) / z_i with z after the
//                  child refinement, from the child logits still in TMEM;
//                  top-P2 (descending, ties to the lower child code).
//   grandchildren  the same refinement with the P2 <= 16 selected children's
//                  8 grandchildren each, the child's logit taken as the mean
//                  of its grandchildren's.
//   output         O = x / z, bf16, TMA store.
// The reference maximum stays the parents' unless a sub-code logit exceeds it
// by more than 2^24 (x and z are then rescaled first); x / z and the
// importances do not depend on that choice.  Codeword rows (bf16) are copied
// straight from the parents / children / grandchildren arrays into 128-byte
// swizzled atoms of 8 codes by cp.async; value-sum rows (fp32) are read,
// rounded to bf16 and stored in the same layout, so no image and no
// workspace is needed.
#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "fastmath.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace avq {
namespace {

constexpr int kRows = 128;           // queries per block (MMA M)
constexpr int kMaxSel = 16;          // selected parents / children per level (8 codes each)
constexpr float kRescaleLog2 = 24.f;

struct Attn3Args {
  const bf16* parents;        // [H][M0][D]
  const bf16* children;       // [H][M0*8][D]
  const bf16* grandchildren;  // [H][M0*64][D]
  const float* vsum;          // [BH][Mt3][D]
  const int32_t* counts;      // [BH][Mt3]
  int32_t* sel;               // [BH][nblk][P]
  int32_t* sel2;              // [BH][nblk][P2]
  float* importance;          // [BH][nblk][M0] or null
  float* importance2;         // [BH][nblk][P*8] or null
  unsigned int* err;
  int H, N, P, P2, nblk;
  float scale_log2;  // scale * log2(e)
};

template <int D>
struct Smem3 {
  static constexpr int kAB = 1024 * (D / 64);       // one atom group: 8 codes x D
  static constexpr int kQ = 0;                      // Q tile; O staging
  static constexpr int kCW = kQ + kRows * D * 2;    // codeword atoms (<= 16)
  static constexpr int kVB = kCW + kMaxSel * kAB;   // value-sum atoms (<= 16)
  static constexpr int kPR = kVB + kMaxSel * kAB;   // A / dA [128][128] bf16: two 64-column slabs
  static constexpr int kNP = kPR + kRows * 128 * 2;  // parents' counts [64] (float)
  static constexpr int kNS = kNP + 64 * 4;          // the level's sub-code counts [128] (float)
  static constexpr int kW = kNS + 128 * 4;          // parents' ranking keys [64] (u32)
  static constexpr int kKEY = kW + 64 * 4;          // children's ranking keys [128] (u64)
  static constexpr int kWP = kKEY + 128 * 8;        // per-warp partial column sums [4][128]
  static constexpr int kSEL = kWP + 4 * 128 * 4;    // selected parents [16], children [16]
  static constexpr int kBAR = kSEL + 2 * kMaxSel * 4;  // 3 mbarriers
  static constexpr int kMISC = kBAR + 32;           // tmem base, abort flag
  static constexpr int kTotal = kMISC + 16;
  static constexpr uint32_t kTmemCols = 256;        // logits [128] + x [D]
};

__device__ __forceinline__ void store_chunk8(uint8_t* tile, int row, int col, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(tile + (col >> 6) * (kRows * 128) + tc::sw128_offset(row, col & 63)) = u;
}

// Offset of 16-byte piece c (dims 8c .. 8c+7) of code i in an atom array.
template <int D>
__device__ __forceinline__ uint32_t atom_piece(int i, int c) {
  const int r = i & 7;
  return (uint32_t)((i >> 3) * Smem3<D>::kAB + (c >> 3) * 1024 + r * 128 + (((c & 7) ^ r) << 4));
}

// Lane l of the warp gets the sum over the warp of columns 2l, 2l+1 of the
// 8 groups of 8 columns in cs (group g: columns 8g + 2 (l % 4) + {0, 1} held
// by lane l): a three-step butterfly reduce-scatter.
__device__ __forceinline__ float2 column_sums64(float2* cs, int lane) {
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
  return cs[0];
}

template <int D, int M0>
__global__ void __launch_bounds__(128, D == 64 ? 2 : 1) attention3_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap, const Attn3Args a) {
  using S = Smem3<D>;
  constexpr int KH = D / 64;
  constexpr int AB = S::kAB;
  constexpr int CPR = D / 8;  // 16-byte pieces per codeword row
  constexpr int M1 = M0 * 8, Mt = M0 + M1 + M1 * 8;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + S::kQ;
  uint8_t* sCW = sm + S::kCW;
  uint8_t* sVB = sm + S::kVB;
  uint8_t* sPR = sm + S::kPR;
  float* sNP = reinterpret_cast<float*>(sm + S::kNP);
  float* sNS = reinterpret_cast<float*>(sm + S::kNS);
  uint32_t* sW = reinterpret_cast<uint32_t*>(sm + S::kW);
  unsigned long long* sKEY = reinterpret_cast<unsigned long long*>(sm + S::kKEY);
  float* sWP = reinterpret_cast<float*>(sm + S::kWP);
  int* sSEL = reinterpret_cast<int*>(sm + S::kSEL);
  int* sSEL2 = sSEL + kMaxSel;
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(sm + S::kBAR);
  uint64_t* bar_mma = bar_q + 1;  // logit MMAs
  uint64_t* bar_x = bar_q + 2;    // value MMAs
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + S::kMISC);
  int* sAbort = reinterpret_cast<int*>(sm + S::kMISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, blk = blockIdx.x, h = bh % a.H;
  const int row0 = blk * kRows;
  const bool valid = row0 + tid < a.N;
  const int P = a.P, P2 = a.P2;
  const size_t ublk = (size_t)bh * a.nblk + blk;
  const int32_t* cnt = a.counts + (size_t)bh * Mt;
  const float* vs = a.vsum + (size_t)bh * Mt * D;
  const bf16* par = a.parents + (size_t)h * M0 * D;
  const bf16* chd = a.children + (size_t)h * M1 * D;
  const bf16* gcd = a.grandchildren + (size_t)h * M1 * 8 * D;
  const float NEG_INF = __int_as_float(0xff800000);
  const float sl2 = a.scale_log2;
  const float2 sl2x2 = fm::f2(sl2, sl2);

  // mbarrier phases (the same in every thread) and, per barrier, the parity of
  // the phase that this thread's last issued operation completes (bit b of
  // `issued` once there was one): drained, with a limit, on the way out
  constexpr int kBars = 3;
  uint32_t ph = 0, issued = 0, exp_par = 0;
  auto note = [&](int b) {
    issued |= 1u << b;
    exp_par = (exp_par & ~(1u << b)) | (ph & (1u << b));
  };
  // waits are taken by thread 0 alone; the others meet it at the CTA barrier
  // that follows every wait
  auto wait_bar = [&](int b) {
    if (tid == 0 && !tc::mbar_wait(bar_q + b, (ph >> b) & 1u)) {
      atomicOr(a.err, kErrTimeout);
      *sAbort = 1;
    }
    ph ^= 1u << b;
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
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tS = tmem;         // logits, 128 columns
  const uint32_t tX = tmem + 128;   // output accumulator, D columns
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t sQa = tc::smem_u32(sQ), sCWa = tc::smem_u32(sCW), sVBa = tc::smem_u32(sVB),
                 sPRa = tc::smem_u32(sPR);
  const uint32_t idesc_x = tc::idesc_bf16(kRows, D, 0, 1);

  // S = Q * CW^T over n codes
  auto issue_logits = [&](int n) {
    note(1);
    const uint32_t idesc = tc::idesc_bf16(kRows, n, 0, 0);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint64_t ad = tc::sdesc_sw128(sQa + (k >> 2) * (kRows * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(sCWa + (k >> 2) * 1024 + (k & 3) * 32, 16, KH * 1024);
      tc::mma_bf16(tS, ad, bd, idesc, k > 0);
    }
    tc::mma_commit(bar_mma);
  };
  // x (+)= PR[:, :n] * VB over n codes
  auto issue_values = [&](int n, bool acc) {
    note(2);
    for (int k = 0; k < n / 16; ++k) {
      const uint64_t ad = tc::sdesc_sw128(sPRa + (k >> 2) * (kRows * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t bd = tc::sdesc_sw128(sVBa + k * 2 * AB, 1024, KH * 1024);
      tc::mma_bf16(tX, ad, bd, idesc_x, (acc || k > 0) ? 1u : 0u);
    }
    tc::mma_commit(bar_x);
  };
  // `rows` codeword rows into the codeword atoms (cp.async, one commit group)
  auto copy_cw = [&](int rows, auto src) {
    for (int p = tid; p < rows * CPR; p += 128) {
      const int i = p / CPR, c = p % CPR;
      tc::cp_async16(sCW + atom_piece<D>(i, c), src(i) + c * 8);
    }
    tc::cp_async_commit();
  };
  // `rows` value-sum rows (fp32) -> bf16 atoms; a null row is zero
  auto copy_vb = [&](int rows, auto src) {
    for (int p0 = tid; p0 < rows * CPR; p0 += 4 * 128) {
      float4 v[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int p = p0 + j * 128;
        const float* s = p < rows * CPR ? src(p / CPR) : nullptr;
        if (s != nullptr) {
          const float4* s4 = reinterpret_cast<const float4*>(s + (p % CPR) * 8);
          v[j][0] = __ldg(s4);
          v[j][1] = __ldg(s4 + 1);
        } else {
          v[j][0] = v[j][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int p = p0 + j * 128;
        if (p < rows * CPR) {
          uint4 u;
          u.x = pack_bf16x2(v[j][0].x, v[j][0].y);
          u.y = pack_bf16x2(v[j][0].z, v[j][0].w);
          u.z = pack_bf16x2(v[j][1].x, v[j][1].y);
          u.w = pack_bf16x2(v[j][1].z, v[j][1].w);
          *reinterpret_cast<uint4*>(sVB + atom_piece<D>(p / CPR, p % CPR)) = u;
        }
      }
    }
  };

  float m, z, mref;
  {
    // ---- parents: operands ----
    if (tid == 0) {
      tc::prefetch_tensormap(&qmap);
      tc::prefetch_tensormap(&omap);
      note(0);
      tc::mbar_arrive_expect_tx(bar_q, kRows * D * 2);
#pragma unroll
      for (int kh = 0; kh < KH; ++kh) tc::tma_load_3d(sQ + kh * kRows * 128, &qmap, kh * 64, row0, bh, bar_q);
    }
    copy_cw(M0, [&](int i) { return par + (size_t)i * D; });
    float nfj = 0.f;
    if (tid < M0) {
      nfj = (float)__ldg(cnt + tid);
      sNP[tid] = nfj;
    }
    copy_vb(M0, [&](int i) { return vs + (size_t)i * D; });
    tc::cp_async_wait<0>();
    tc::fence_proxy_async_smem();
    wait_bar(0);  // Q
    tc::tc_fence_before();
    const bool any_empty = __syncthreads_or(tid < M0 && !(nfj > 0.f)) != 0;
    tc::tc_fence_after();
    if (*sAbort) goto done;
    if (warp == 0) {
      if (tc::elect_one()) {
        tc::tc_fence_after();
        issue_logits(M0);
      }
      __syncwarp();
    }
    wait_bar(1);
    __syncthreads();
    tc::tc_fence_after();
    if (*sAbort) goto done;

    // ---- parents: masked max, A = 2^(t - m), z, importance ----
    const float4* nf4 = reinterpret_cast<const float4*>(sNP);
    {
      float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
      for (int c0 = 0; c0 < M0; c0 += 32) {  // columns c0 .. min(c0 + 32, M0) - 1
        uint32_t r[32];
#pragma unroll
        for (int g = 0; g < 2; ++g)
          if (c0 + g * 16 < M0) tc::tmem_ld16(tS + lane_off + c0 + g * 16, r + g * 16);
        tc::tmem_wait_ld();
        const float* t = reinterpret_cast<const float*>(r);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          if (c0 + e >= M0) break;
          const float4 nf = nf4[(c0 + e) >> 2];
          if (!any_empty) {
            mx0 = fm::max3(mx0, t[e], t[e + 1]);
            mx1 = fm::max3(mx1, t[e + 2], t[e + 3]);
          } else {
            mx0 = fm::max3(mx0, nf.x > 0.f ? t[e] : NEG_INF, nf.y > 0.f ? t[e + 1] : NEG_INF);
            mx1 = fm::max3(mx1, nf.z > 0.f ? t[e + 2] : NEG_INF, nf.w > 0.f ? t[e + 3] : NEG_INF);
          }
        }
      }
      m = fmaxf(mx0, mx1) * sl2;
    }
    {
      const float2 nm2 = fm::f2(-m, -m);
      float2 zp = fm::f2(0.f, 0.f);
#pragma unroll
      for (int g = 0; g < M0 / 16; ++g) {
        uint32_t r[16];
        tc::tmem_ld16(tS + lane_off + g * 16, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 nf = nf4[(g * 16 + e) >> 2];
          const float2 x01 = fm::fma2(fm::f2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), sl2x2, nm2);
          const float2 x23 = fm::fma2(fm::f2(__uint_as_float(r[e + 2]), __uint_as_float(r[e + 3])), sl2x2, nm2);
          float a0 = tc::ex2(x01.x), a1 = tc::ex2(x01.y), a2 = tc::ex2(x23.x), a3 = tc::ex2(x23.y);
          if (any_empty) {
            a0 = nf.x > 0.f ? a0 : 0.f;
            a1 = nf.y > 0.f ? a1 : 0.f;
            a2 = nf.z > 0.f ? a2 : 0.f;
            a3 = nf.w > 0.f ? a3 : 0.f;
          }
          zp = fm::fma2(fm::f2(a0, a1), fm::f2(nf.x, nf.y), zp);
          zp = fm::fma2(fm::f2(a2, a3), fm::f2(nf.z, nf.w), zp);
          r[e] = __float_as_uint(a0);
          r[e + 1] = __float_as_uint(a1);
          r[e + 2] = __float_as_uint(a2);
          r[e + 3] = __float_as_uint(a3);
        }
        store_chunk8(sPR, tid, g * 16, reinterpret_cast<const float*>(r));
        store_chunk8(sPR, tid, g * 16 + 8, reinterpret_cast<const float*>(r) + 8);
        tc::tmem_st16(tS + lane_off + g * 16, r);
      }
      tc::tmem_wait_st();
      z = zp.x + zp.y;
    }
    mref = m;
    {
      // importance column sums of A / z (Eq. 7) from A read back in the
      // 16x256b shape: lane l holds columns 8k + 2 (l % 4) + {0, 1} of rows
      // l/4, l/4 + 8 (first 16 lanes) and 16 + l/4, 24 + l/4 of its warp
      const float rz = valid ? 1.f / z : 0.f;
      const int rl = lane >> 2;
      const float z0 = __shfl_sync(0xffffffffu, rz, rl), z1 = __shfl_sync(0xffffffffu, rz, rl + 8),
                  z2 = __shfl_sync(0xffffffffu, rz, rl + 16), z3 = __shfl_sync(0xffffffffu, rz, rl + 24);
      float2 cs[8];
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        if (hc * 32 < M0) {
          uint32_t lo[16], hi[16];
          fm::tmem_ld_16x256b_x4(tS + lane_off + hc * 32, lo);
          fm::tmem_ld_16x256b_x4(tS + lane_off + (16u << 16) + hc * 32, hi);
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
      *reinterpret_cast<float2*>(sWP + warp * 128 + 2 * lane) = column_sums64(cs, lane);
    }
    tc::fence_proxy_async_smem();  // PR
    tc::tc_fence_before();
    __syncthreads();
    // ranking key of parent j: its importance with the 6 lowest mantissa bits
    // replaced by 63 - j (importances are >= 0: the unsigned order of the bits
    // is the order of the values; equal values rank the lower index first);
    // the importance reported is the key's value part
    if (tid < M0) {
      const float wj = nfj * ((sWP[tid] + sWP[128 + tid]) + (sWP[256 + tid] + sWP[384 + tid]));
      sW[tid] = (__float_as_uint(wj) & ~63u) | (uint32_t)(63 - tid);
    }
    __syncthreads();
    if (tid < M0) {
      const uint32_t kj = sW[tid];
      int rank = 0;
#pragma unroll
      for (int l = 0; l < M0; l += 4) {
        const uint4 k4 = *reinterpret_cast<const uint4*>(sW + l);
        rank += (k4.x > kj) + (k4.y > kj) + (k4.z > kj) + (k4.w > kj);
      }
      if (rank < P) {
        sSEL[rank] = tid;
        a.sel[ublk * P + rank] = tid;
      }
      if (a.importance) a.importance[ublk * M0 + tid] = __uint_as_float(kj & ~63u);
    }
    if (warp == 3) {  // x = A Vbar_p
      if (tc::elect_one()) {
        tc::tc_fence_after();
        issue_values(M0, false);
      }
      __syncwarp();
    }
    __syncthreads();
  }

  {
    // one refinement level: np selected nodes (slots padded to an even
    // number), their 8 sub-codes each.  Codewords and counts first, then the
    // previous value MMA is waited for before the value sums and PR are
    // overwritten; the logit MMA runs meanwhile.
    auto refine = [&](int np, auto cw_row, auto vb_row, auto count_of) {
      const int slots = (np + 1) & ~1, n = slots * 8;
      copy_cw(n, [&](int i) { return cw_row(min(i >> 3, np - 1), i & 7); });
      if (tid < n) sNS[tid] = (tid >> 3) < np ? (float)count_of(tid >> 3, tid & 7) : 0.f;
      tc::cp_async_wait<0>();
      tc::fence_proxy_async_smem();
      wait_bar(2);  // the previous value MMA has read PR and VB
      tc::tc_fence_before();
      __syncthreads();
      if (*sAbort) return false;
      if (warp == 0) {
        if (tc::elect_one()) {
          tc::tc_fence_after();
          issue_logits(n);
        }
        __syncwarp();
      }
      copy_vb(n, [&](int i) { return (i >> 3) < np ? vb_row(i >> 3, i & 7) : nullptr; });
      tc::fence_proxy_async_smem();
      wait_bar(1);
      __syncthreads();
      tc::tc_fence_after();
      if (*sAbort) return false;
      // dA = 2^(t_s - m) - 2^(t_n - m), t_n the mean of the node's 8 sub-code
      // logits (Eq. 8), with the reference maximum; the unmasked sub-code
      // maximum on the way.  Empty sub-codes need no mask while every
      // 2^(t - m) stays below 2^24: their value sums and counts are zero.
      const float4* ns4 = reinterpret_cast<const float4*>(sNS);
      float2 zc = fm::f2(0.f, 0.f);
      float cm0 = NEG_INF, cm1 = NEG_INF;
      auto da_pass = [&](auto masked_t) {
        constexpr bool kMasked = decltype(masked_t)::value;
        const float nm = -mref, sl8 = sl2 * 0.125f;
        const float2 nm2 = fm::f2(nm, nm);
#pragma unroll
        for (int g2 = 0; g2 < 8; g2 += 2) {
          if (g2 * 16 < n) {
            uint32_t r[32];
            tc::tmem_ld16(tS + lane_off + g2 * 16, r);
            if (g2 * 16 + 16 < n) tc::tmem_ld16(tS + lane_off + g2 * 16 + 16, r + 16);
            tc::tmem_wait_ld();
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
              const int sl = 2 * g2 + s4;  // node slot
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
                const float4 na = ns4[sl * 2], nb = ns4[sl * 2 + 1];
                const float nfv[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
                uint4 pk;
                uint32_t* pkw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                  const float2 x = fm::fma2(fm::f2(tt[e], tt[e + 1]), sl2x2, nm2);
                  float2 da = fm::add2(fm::f2(tc::ex2(x.x), tc::ex2(x.y)), nap);
                  if (kMasked) {
                    da.x = nfv[e] > 0.f ? da.x : 0.f;
                    da.y = nfv[e + 1] > 0.f ? da.y : 0.f;
                  }
                  zc = fm::fma2(da, fm::f2(nfv[e], nfv[e + 1]), zc);
                  pkw[e >> 1] = pack_bf16x2(da.x, da.y);
                }
                *reinterpret_cast<uint4*>(sPR + (sl >> 3) * (kRows * 128) + tc::sw128_offset(tid, (sl & 7) * 8)) = pk;
              }
            }
          }
        }
      };
      da_pass(std::false_type{});
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      const float cmax_any = fmaxf(cm0, cm1) * sl2;
      if (__syncthreads_or(cmax_any > mref + kRescaleLog2)) {  // block-uniform, rare
        // masked maximum over non-empty sub-codes; rescale x and z if it is far
        // above the reference, then dA again with the masks applied
        tc::tc_fence_after();
        float cmm0 = NEG_INF, cmm1 = NEG_INF;
        for (int g = 0; g < 8; ++g) {
          if (g * 16 < n) {
            uint32_t r[16];
            tc::tmem_ld16(tS + lane_off + g * 16, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              cmm0 = fmaxf(cmm0, sNS[g * 16 + e] > 0.f ? __uint_as_float(r[e]) : NEG_INF);
              cmm1 = fmaxf(cmm1, sNS[g * 16 + e + 1] > 0.f ? __uint_as_float(r[e + 1]) : NEG_INF);
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
        da_pass(std::true_type{});
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
      }
      z += zc.x + zc.y;
      if (warp == 3) {  // x += dA Vbar
        if (tc::elect_one()) {
          tc::tc_fence_after();
          issue_values(n, true);
        }
        __syncwarp();
      }
      return true;
    };

    // ---- children of the top-P parents ----
    if (P > 0) {
      const bool ok = refine(
          P, [&](int s, int c) { return chd + ((size_t)sSEL[s] * 8 + c) * D; },
          [&](int s, int c) { return vs + (size_t)(M0 + sSEL[s] * 8 + c) * D; },
          [&](int s, int c) { return __ldg(cnt + M0 + sSEL[s] * 8 + c); });
      if (!ok) goto done;

      // ---- the refined children's importance, after the child refinement ----
      const int NC = P * 8;
      if (P2 > 0 || a.importance2 != nullptr) {
        const int n = ((P + 1) & ~1) * 8;
        const float rz = valid ? 1.f / z : 0.f;
        const int rl = lane >> 2;
        float zr[4], mr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          zr[j] = __shfl_sync(0xffffffffu, rz, rl + 8 * j);
          mr[j] = __shfl_sync(0xffffffffu, mref, rl + 8 * j);
        }
        auto ev = [&](uint32_t t, int j) { return tc::ex2(fmaf(__uint_as_float(t), sl2, -mr[j])) * zr[j]; };
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half * 64 < n) {
            float2 cs[8];
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
              const int c0 = half * 64 + hc * 32;
              if (c0 < n) {
                uint32_t lo[16], hi[16];
                fm::tmem_ld_16x256b_x4(tS + lane_off + c0, lo);
                fm::tmem_ld_16x256b_x4(tS + lane_off + (16u << 16) + c0, hi);
                tc::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int col = c0 + 8 * k + 2 * (lane & 3);
                  const float sx = (ev(lo[4 * k], 0) + ev(lo[4 * k + 2], 1)) + (ev(hi[4 * k], 2) + ev(hi[4 * k + 2], 3));
                  const float sy =
                      (ev(lo[4 * k + 1], 0) + ev(lo[4 * k + 3], 1)) + (ev(hi[4 * k + 1], 2) + ev(hi[4 * k + 3], 3));
                  cs[hc * 4 + k] = fm::f2(sNS[col] > 0.f ? sx : 0.f, sNS[col + 1] > 0.f ? sy : 0.f);
                }
              } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) cs[hc * 4 + k] = fm::f2(0.f, 0.f);
              }
            }
            *reinterpret_cast<float2*>(sWP + warp * 128 + half * 64 + 2 * lane) = column_sums64(cs, lane);
          }
        }
        tc::tc_fence_before();
        __syncthreads();
        // ranking key of slot u (parent rank u / 8, child u % 8): the
        // importance's bits above the complement of the child code, so that
        // equal importances rank the lower child code first
        unsigned long long ku = 0;
        int cu = 0;
        if (tid < NC) {
          const float wu = sNS[tid] * ((sWP[tid] + sWP[128 + tid]) + (sWP[256 + tid] + sWP[384 + tid]));
          cu = sSEL[tid >> 3] * 8 + (tid & 7);
          ku = ((unsigned long long)__float_as_uint(wu) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)cu);
          sKEY[tid] = ku;
          if (a.importance2) a.importance2[ublk * NC + tid] = wu;
        }
        __syncthreads();
        if (tid < NC) {
          int rank = 0;
          for (int v = 0; v < NC; v += 2) {
            const ulonglong2 k2 = *reinterpret_cast<const ulonglong2*>(sKEY + v);
            rank += (k2.x > ku) + (v + 1 < NC && k2.y > ku);
          }
          if (rank < P2) {
            sSEL2[rank] = cu;
            a.sel2[ublk * P2 + rank] = M0 + cu;
          }
        }
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
      }

      // ---- grandchildren of the top-P2 children ----
      if (P2 > 0) {
        const bool ok2 = refine(
            P2, [&](int s, int g) { return gcd + ((size_t)sSEL2[s] * 8 + g) * D; },
            [&](int s, int g) { return vs + (size_t)(M0 + M1 + sSEL2[s] * 8 + g) * D; },
            [&](int s, int g) { return __ldg(cnt + M0 + M1 + sSEL2[s] * 8 + g); });
        if (!ok2) goto done;
      }
    }
  }

  // ---- O = x / z -> bf16 -> shared (Q region) -> TMA store ----
  wait_bar(2);  // the last value MMA
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (*sAbort) goto done;
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
      store_chunk8(sQ, tid, g, v);
      store_chunk8(sQ, tid, g + 8, v + 8);
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
#pragma unroll
      for (int kh = 0; kh < KH; ++kh) tc::tma_store_3d(&omap, sQ + kh * kRows * 128, kh * 64, row0, bh);
      tc::bulk_commit_group();
    }
  }

done:
  // nothing of this CTA in flight before TMEM is freed and the CTA exits
  if (issued) {
#pragma unroll
    for (int b = 0; b < kBars; ++b)
      if ((issued >> b) & 1u)
        if (!tc::mbar_wait(bar_q + b, (exp_par >> b) & 1u, 1000000ull)) atomicOr(a.err, kErrTimeout);
  }
  tc::cp_async_wait<0>();
  if (tid == 0) tc::bulk_wait_group_read0();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, S::kTmemCols);
  }
}

template <int D, int M0>
cudaError_t launch3_m(const Shape& s, const CUtensorMap& qmap, const CUtensorMap& omap, const Attn3Args& a,
                      cudaStream_t st) {
  const int smem = Smem3<D>::kTotal + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(attention3_tc_kernel<D, M0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attention3_tc_kernel<D, M0><<<dim3(a.nblk, s.BH()), 128, smem, st>>>(qmap, omap, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch3_d(const Shape& s, const CUtensorMap& qmap, const CUtensorMap& omap, const Attn3Args& a,
                      cudaStream_t st) {
  switch (s.M0) {
    case 16: return launch3_m<D, 16>(s, qmap, omap, a, st);
    case 32: return launch3_m<D, 32>(s, qmap, omap, a, st);
    case 48: return launch3_m<D, 48>(s, qmap, omap, a, st);
    default: return launch3_m<D, 64>(s, qmap, omap, a, st);
  }
}

}  // namespace

bool attention3_tc_supported(const Shape& s, avq_dtype dt, int P, int P2, int block) {
  return dt == AVQ_BF16 && block == kRows && (s.d == 64 || s.d == 128) && s.C == 8 && s.M0 % 16 == 0 &&
         s.M0 >= 16 && s.M0 <= 64 && P <= kMaxSel && P2 <= kMaxSel;
}

cudaError_t launch_attention3_tc(const Shape& s, const void* Q, const void* parents, const void* children,
                                 const void* grandchildren, const float* vsum, const int32_t* counts, int P,
                                 int P2, float scale, void* O, int32_t* sel, int32_t* sel2, float* importance,
                                 float* importance2, unsigned int* err, cudaStream_t st, LaunchLog& log) {
  CUtensorMap qmap, omap;
  cudaError_t e = make_tmap_3d_bf16(&qmap, Q, s.d, s.N, s.BH(), 64, kRows);
  if (e != cudaSuccess) return e;
  e = make_tmap_3d_bf16(&omap, O, s.d, s.N, s.BH(), 64, kRows);
  if (e != cudaSuccess) return e;
  Attn3Args a;
  a.parents = static_cast<const bf16*>(parents);
  a.children = static_cast<const bf16*>(children);
  a.grandchildren = static_cast<const bf16*>(grandchildren);
  a.vsum = vsum;
  a.counts = counts;
  a.sel = sel;
  a.sel2 = sel2;
  a.importance = importance;
  a.importance2 = importance2;
  a.err = err;
  a.H = s.H;
  a.N = s.N;
  a.P = P;
  a.P2 = P2;
  a.nblk = (s.N + kRows - 1) / kRows;
  a.scale_log2 = scale * 1.4426950408889634f;
  e = s.d == 64 ? launch3_d<64>(s, qmap, omap, a, st) : launch3_d<128>(s, qmap, omap, a, st);
  log.add("attention3_tc");
  return e;
}

}  // namespace avq
