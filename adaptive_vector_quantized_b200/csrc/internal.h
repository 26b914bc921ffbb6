// Host-side launch interface between the C ABI (avq_api.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "avq.h"

namespace avq {

struct Shape {
  int B, H, N, d, M0, C;
  int BH() const { return B * H; }
  int Mt() const { return M0 * (1 + C); }
};

// Every launcher returns cudaSuccess or the launch error, and appends the
// names of the kernels it enqueued to `names` (space separated).
struct LaunchLog {
  char text[512];
  int len;
  void add(const char* name);
};

// ---- stage 1 ------------------------------------------------------------
// Algorithm 1, assignment: writes assign[BH][N] and adds the key
// counts (Eq. 3) into counts[BH][Mt], which the caller zeroes first.
cudaError_t launch_assign_simt(const Shape& s, avq_dtype dt, const void* K, const void* parents,
                               const void* children, int32_t* assign, int32_t* counts,
                               cudaStream_t st, LaunchLog& log);
// Algorithm 1, value sums for given codes, streaming variant.
// vsum is zeroed inside unless vsum_zeroed; counts are added here only when
// `count` is set (then zeroed by the caller and left out by the assignment),
// else the assignment kernels produce them.  depth3: codes of a three-level
// tree (parents, M0*C children, M0*C*C grandchildren).
cudaError_t launch_aggregate(const Shape& s, avq_dtype dt, const void* V, const int32_t* assign,
                             float* vsum, int32_t* counts, unsigned int* err, cudaStream_t st,
                             LaunchLog& log, bool vsum_zeroed = false, bool depth3 = false,
                             bool count = false);
// Depth-3 tree (three levels, codes parents | M0*C children | M0*C*C
// grandchildren): assignment one level deeper on the CUDA cores; counts are
// added into counts[BH][Mt3], which the caller zeroes first.
// Depth-3 stage 1 after the two-level tensor-core assignment (bf16, C = 8,
// d in {64, 128}): keys at a child move to its nearest grandchild when
// strictly closer; assign[] is rewritten in place (no counts).
cudaError_t launch_assign3_grandchildren(const Shape& s, const void* K, const void* children,
                                         const void* grandchildren, int32_t* assign, cudaStream_t st,
                                         LaunchLog& log);
cudaError_t launch_assign3_simt(const Shape& s, avq_dtype dt, const void* K, const void* parents,
                                const void* children, const void* grandchildren, int32_t* assign,
                                int32_t* counts, cudaStream_t st, LaunchLog& log);
// Depth-3 attention on the CUDA cores: parents, the top-P parents' children,
// the top-P2 refined children's grandchildren.
// Depth-3 attention on the tensor cores: bf16, block 128, d 64 or 128, C 8,
// M0 in {16, 32, 48, 64}, P and P2 at most 16.
bool attention3_tc_supported(const Shape& s, avq_dtype dt, int P, int P2, int block);
cudaError_t launch_attention3_tc(const Shape& s, const void* Q, const void* parents, const void* children,
                                 const void* grandchildren, const float* vsum, const int32_t* counts, int P,
                                 int P2, float scale, void* O, int32_t* sel, int32_t* sel2, float* importance,
                                 float* importance2, unsigned int* err, cudaStream_t st, LaunchLog& log);
cudaError_t launch_attention3_simt(const Shape& s, avq_dtype dt, const void* Q, const void* parents,
                                   const void* children, const void* grandchildren, const float* vsum,
                                   const int32_t* counts, int P, int P2, int block, float scale, void* O,
                                   int32_t* sel, int32_t* sel2, float* importance, float* importance2,
                                   cudaStream_t st, LaunchLog& log);
// Deterministic aggregation (fixed-order sums, independent of the grid).
size_t aggregate_det_workspace(const Shape& s);
cudaError_t launch_aggregate_det(const Shape& s, avq_dtype dt, const void* V,
                                 const int32_t* assign, float* vsum, int32_t* counts, void* ws,
                                 cudaStream_t st, LaunchLog& log);

// tcgen05 assignment kernel (bf16, d in {64,128}, M0 a multiple of 16 up to 256,
// C in {0, 8}); needs assign_tc_workspace(s) bytes of workspace.
bool assign_tc_supported(const Shape& s, avq_dtype dt);
size_t assign_tc_workspace(const Shape& s);
// True when launch_assign_tc takes the warpgroup kernel for this shape (the
// whole two-level codebook image in shared memory).
bool assign_tc_uses_warpgroups(const Shape& s);
// Zeroes counts itself (and vsum when vsum_to_zero is given) before the
// assignment adds into them.  With counts_left given, the warpgroup kernel
// may leave the counts to the streaming value sums: *counts_left tells the
// caller whether it did.
cudaError_t launch_assign_tc(const Shape& s, const void* K, const void* parents,
                             const void* children, int32_t* assign, int32_t* counts, void* ws,
                             unsigned int* err, cudaStream_t st, LaunchLog& log,
                             float* vsum_to_zero = nullptr, bool* counts_left = nullptr);

// ---- stage 2 ------------------------------------------------------------
cudaError_t launch_attention_simt(const Shape& s, avq_dtype dt, const void* Q, const void* parents,
                                  const void* children, const float* vsum, const int32_t* counts,
                                  int P, int block, float scale, void* O, int32_t* sel,
                                  float* importance, cudaStream_t st, LaunchLog& log);

bool attention_tc_supported(const Shape& s, avq_dtype dt, int P, int block, int two_pass);
size_t attention_tc_workspace(const Shape& s, int P, int block, int two_pass);
cudaError_t launch_attention_tc(const Shape& s, const void* Q, const void* parents,
                                const void* children, const float* vsum, const int32_t* counts,
                                int P, int block, float scale, int two_pass, void* O,
                                int32_t* sel, float* importance, void* ws, unsigned int* err,
                                cudaStream_t st, LaunchLog& log);

// ---- token permutation ----------------------------------------------------
// Sec. A, Eqs. 11-12: EMA statistics S [H][Mt][d], Nst [H][Mt] updated in
// place from the keys' Eq. 3 statistics ksum [BH][Mt][d], counts [BH][Mt];
// parents [H][M0][d] and children [H][M0][C][d] rewritten in place.
cudaError_t launch_codebook_update(const Shape& s, avq_dtype dt, float lambda, const float* ksum,
                                   const int32_t* counts, float* S, float* Nst, void* parents,
                                   void* children, cudaStream_t st, LaunchLog& log);
// Indices outside [0, rows) are skipped and set kErrBounds in err.
cudaError_t launch_permute(const void* X, const int32_t* idx, void* Y, int batch, int rows,
                           int row_bytes, int inverse, unsigned int* err, cudaStream_t st, LaunchLog& log);

// 3-D tiled TMA map over a bf16 tensor [batch][rows][inner] (inner contiguous),
// box {box_inner, box_rows, 1}, 128-byte swizzle, zero fill out of bounds.
cudaError_t make_tmap_3d_bf16(CUtensorMap* map, const void* base, int inner, int rows, int batch,
                              int box_inner, int box_rows);

// Device address of the current device's error word.
unsigned int* error_word();
// One thread waits, with the given limit, on an mbarrier that nothing
// completes (self-test of the bounded waits; sets kErrTimeout in err).
cudaError_t launch_exp2_probe(const float* x, float* y, long long n, cudaStream_t st);
cudaError_t launch_wait_probe(unsigned int* err, unsigned long long timeout_ns, cudaStream_t st);

int num_sms();

}  // namespace avq
