/*
 * avq.h -- C ABI of libavq.so, a B200-native (sm_100a) forward pass of
 * AVQ-Attention ("AVQ-Attention: Adaptive Vector-Quantized Attention").
 *
 * Two stages, as in the paper's inference pipeline (Sec. 4.3 "Summary",
 * Fig. 4): avq_quantize builds the statistics of the full codebook tree
 * (Sec. 4.2, Algorithm 1); avq_attention attends over the parents with
 * count-weighted online softmax, picks the top-P parents per query block and
 * replaces their contribution with their children's (Sec. 4.3, Algorithm 2).
 *
 * Conventions shared by every call
 *   - Ownership: the caller allocates and owns every buffer, host or device.
 *     The library allocates no memory and keeps no state across calls except
 *     thread-local settings (avq_set_path) and diagnostics (avq_last_error,
 *     avq_last_kernels), one device-side error word per GPU and the static
 *     scratch array of avq_quantize_noalloc.
 *   - Execution: device calls are enqueued on `stream` (NULL = legacy default
 *     stream) and return without synchronising.  Results are valid once the
 *     stream has completed the call.
 *   - Errors: arguments are validated on the host before anything is launched;
 *     a failed check returns AVQ_ERR_INVALID_ARG, AVQ_ERR_UNSUPPORTED or
 *     AVQ_ERR_WORKSPACE, launches nothing and leaves every output untouched.
 *     AVQ_ERR_CUDA means a launch was rejected by the CUDA runtime.  Faults
 *     detected inside kernels (a bounded wait that ran out) are recorded in
 *     the device error word and reported by avq_check_device.
 *   - Fault injection for tests of a caller's error handling: if the
 *     environment variable AVQ_FAULT is "quantize", "attention",
 *     "codebook_update", "permute" or "all", the named entry points return
 *     AVQ_ERR_CUDA after their argument checks, before any launch (nothing
 *     reaches the GPU).  Unset or empty: no effect.
 *   - Layouts are dense row-major.  BH = B*H; tensor [B,H,N,d] puts head
 *     (b,h) at offset (b*H+h)*N*d.  Device pointers must be 16-byte aligned.
 *   - Codebook: one per head, shared by the batch (Algorithm 1 input
 *     C in R^{H x Mtotal x D}).  Mt = M0*(1+C).  Codeword a < M0 is parent a;
 *     codeword M0 + m*C + c is child c of parent m (Algorithm 1's first-child
 *     index).  Each parent must equal the mean of its children (Sec. 4.1,
 *     Eq. 5); the attention recovers parent logits from that (Eq. 8).
 */
#ifndef AVQ_H
#define AVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* A CUDA stream (cudaStream_t).  NULL selects the legacy default stream. */
typedef struct CUstream_st* avq_stream_t;

typedef enum {
  AVQ_OK = 0,
  AVQ_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or shape    */
  AVQ_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement  */
  AVQ_ERR_CUDA = 3,        /* the CUDA runtime rejected a launch or copy    */
  AVQ_ERR_DEVICE = 4,      /* a kernel recorded an error in the error word  */
  AVQ_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out            */
  AVQ_ERR_WORKSPACE = 6    /* workspace missing or smaller than required    */
} avq_status;

/* Element type of Q, K, V, O and of the codebook.  Arithmetic is fp32 in
 * both cases (fp32 accumulation of bf16 products on the tensor cores). */
typedef enum { AVQ_F32 = 0, AVQ_BF16 = 1 } avq_dtype;

/* Problem shape of one attention layer.  Supported: B, H >= 1; N >= 1;
 * d in {64, 128}; 1 <= M0 <= 256; 0 <= C <= 8; B*H <= 65535 (one grid row
 * per head) and B*H*N < 2^31.  Outside: AVQ_ERR_UNSUPPORTED. */
typedef struct {
  int B, H, N, d, M0, C;
} avq_dims;

/* Kernel family selection (thread-local; default AVQ_PATH_AUTO).
 * AUTO picks the tensor-core kernels where they apply, SIMT otherwise.
 * SIMT forces the general CUDA-core kernels.  TC forces the tcgen05
 * kernels and makes calls they do not cover return AVQ_ERR_UNSUPPORTED. */
typedef enum { AVQ_PATH_AUTO = 0, AVQ_PATH_SIMT = 1, AVQ_PATH_TC = 2 } avq_path;

/* Values of avq_attention's `two_pass` argument (importance denominator). */
typedef enum {
  AVQ_DENOM_AUTO = 0,
  AVQ_DENOM_TWO_PASS = 1,
  AVQ_DENOM_EXTRAPOLATED = 2
} avq_denominator;

/*
 * avq_quantize -- full-tree key quantisation and aggregation
 * (Sec. 4.2 "Vector Quantization for (A)VQ-Attention", Algorithm 1, Eq. 3).
 *
 * Every key K[b,h,j] goes to its nearest parent a (squared Euclidean
 * distance, ties to the lower index); it moves to the nearest child c* of a
 * (ties to the first child) only if that child is strictly closer than a.
 * Outputs (device, written in full; the call zeroes them first):
 *   assign [B,H,N]    int32  final code: a, or M0 + a*C + c* if moved
 *   vsum   [B,H,Mt,d] fp32   value sums V-bar (Eq. 3): a parent sums its whole
 *                            cluster, a child only the keys that moved to it
 *   counts [B,H,Mt]   int32  key counts n with the same membership
 * Inputs (device): K, V [B,H,N,d]; parents [H,M0,d]; children [H,M0,C,d]
 * (may be NULL when C == 0), all of `dtype`.
 * deterministic != 0 makes vsum the sequential fp32 sum of each code's keys
 * in key order (a parent: the keys that stayed, then its children in child
 * order), which no launch shape enters: bitwise reproducible from run to run
 * and independent of the GPU's size (needs workspace).
 * Workspace: `ws` (device, 256-byte aligned) of at least
 * avq_workspace_size(...) bytes; may be NULL when that size is 0.
 */
avq_status avq_quantize(const avq_dims* dims, avq_dtype dtype,
                        const void* K, const void* V,
                        const void* parents, const void* children,
                        int32_t* assign, float* vsum, int32_t* counts,
                        int deterministic, void* ws, size_t ws_bytes,
                        avq_stream_t stream);

/*
 * avq_quantize_noalloc -- avq_quantize without a caller workspace.  This call
 * is an engineering addition of this library; the paper has no counterpart.
 *
 * For callers that cannot hand over device memory for a workspace: a runtime
 * whose device memory is reserved up front by its own pool and that must not
 * allocate while it serves requests, or a plain C caller that wants a single
 * call with no buffer to size, allocate and keep alive.  Nothing is
 * allocated: the tensor-core codebook image lives in a fixed device array of
 * AVQ_NOALLOC_SCRATCH_BYTES inside the library, one per GPU.
 *
 * Arguments, outputs and results are those of avq_quantize with
 * deterministic = 0 (the fixed-order reduction needs scratch that grows with
 * N, so it is not offered here).  counts is zeroed by the call, as in
 * avq_quantize; the static scratch needs no clearing.
 *
 * Limit: the tensor-core path needs H*Mt*d*2 bytes (rounded up to 256) plus
 * H*Mt*4 bytes (rounded up to 256) of scratch; above AVQ_NOALLOC_SCRATCH_BYTES
 * the call returns AVQ_ERR_WORKSPACE and launches nothing.  Shapes or dtypes
 * without a tensor-core kernel (and AVQ_PATH_SIMT) use the CUDA-core
 * assignment, which needs no scratch.
 *
 * Set-up: the first call on each device, with that device current, resolves
 * the scratch array's device address; make that first call before any stream
 * capture.
 *
 * Races: every call on one device shares the one scratch array.  Calls
 * ordered on one stream are safe; two calls whose executions may overlap
 * (different streams without ordering between them, or different host threads
 * on one device) overwrite each other's codebook image and give wrong results.
 */
#define AVQ_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
avq_status avq_quantize_noalloc(const avq_dims* dims, avq_dtype dtype,
                                const void* K, const void* V,
                                const void* parents, const void* children,
                                int32_t* assign, float* vsum, int32_t* counts,
                                avq_stream_t stream);

/*
 * avq_attention -- adaptive attention with per-query-block refinement
 * (Sec. 4.3 "Computing (A)VQ-Attention with Flash Attention", Algorithm 2;
 * Eqs. 6-9; masked running max of Sec. D, Eq. 18).
 *
 * For each head and each block I of `block` consecutive queries (the last
 * block may be shorter): logits S = scale * Q C^T over the M0 parents; running
 * max over non-empty parents; A = exp(S - m), zero for empty parents;
 * x = A V-bar, z = A n (Eq. 6); importance w_j(I) = sum_i A_ij n_j / z_i
 * (Eq. 7); the P parents of largest w (descending, ties to the lower index)
 * are refined: child logits S_c, parent logit recovered as their mean (Eq. 8),
 * dA = exp(S_c) - exp(S_p) (Eq. 9), zero for empty children, added to x and z;
 * O = x / z.  With C == 0 or P == 0 no refinement happens (flat VQ attention,
 * Eq. 4).
 * Inputs (device): Q [B,H,N,d] of `dtype`; parents, children as for
 * avq_quantize; vsum, counts as produced by avq_quantize.
 * P in [0, M0]; block in {64, 128}; scale > 0 (1/sqrt(d) for standard
 * attention; the paper omits it for clarity, Sec. 3.1).
 * two_pass selects how the importance denominator is formed when the parents
 * span several tiles of 64 codes (M0 > 64):
 *   AVQ_DENOM_AUTO (0): exact; one pass when the parents fit one tile, else
 *     the two-pass form below; with P == 0 and importance == NULL (nothing
 *     then depends on the denominator) one pass over the tiles with a
 *     running maximum, whatever M0.
 *   AVQ_DENOM_TWO_PASS (1): exact two-pass denominator: a first pass over
 *     parent tiles finds the row max and z, a second recomputes the logits
 *     for x and the importance.  Results equal the single-pass ones.
 *   AVQ_DENOM_EXTRAPOLATED (2): one pass over the parent tiles in index order;
 *     the importance of the parents of tile J uses the count-extrapolated
 *     denominator Z~(J) = (N / N_seen(J)) * sum_{t <= J} Z(t) (Sec. B,
 *     Eqs. 13-14), so the selection may differ from the exact one; x, z and
 *     O are computed exactly for whatever is selected.  Needs the
 *     tensor-core kernel when M0 > 64 (else AVQ_ERR_UNSUPPORTED).
 * Any other value is AVQ_ERR_INVALID_ARG.
 * Outputs (device): O [B,H,N,d] of `dtype`; sel [B,H,nblk,P] int32, the
 * selected parents in descending importance (nblk = ceil(N/block)), may be
 * NULL when P == 0; importance [B,H,nblk,M0] fp32 or NULL.
 * Workspace as for avq_quantize.
 */
avq_status avq_attention(const avq_dims* dims, avq_dtype dtype, const void* Q,
                         const void* parents, const void* children,
                         const float* vsum, const int32_t* counts,
                         int P, int block, float scale, int two_pass,
                         void* O, int32_t* sel, float* importance,
                         void* ws, size_t ws_bytes, avq_stream_t stream);

/*
 * avq_quantize3 -- a depth-3 tree: Algorithm 1 (Sec. 4.2) one level further
 * down, the "deeper hierarchies" named as the next step in the conclusion
 * (Sec. 6).  Every child has C grandchildren and should be their mean, as
 * every parent the mean of its children (Eq. 5).
 *
 * Every key goes to its nearest parent a (ties to the lower index), then to
 * the nearest child c* of a (first strict minimum) if strictly closer than a,
 * then to the nearest grandchild g* of c* if strictly closer than c*.
 * Codes per head (Mt3 = M0 + M0*C + M0*C*C):
 *   parents [0, M0); child (m, c) at M0 + m*C + c; grandchild (m, c, g) at
 *   M0 + M0*C + (m*C + c)*C + g.
 * Outputs (device, written in full; the call zeroes them first):
 *   assign [B,H,N]      int32  final code
 *   vsum   [B,H,Mt3,d]  fp32   value sums (Eq. 3): every node holds the keys of
 *                              its subtree that reached it
 *   counts [B,H,Mt3]    int32  key counts with the same membership
 * Inputs (device): K, V [B,H,N,d]; parents [H,M0,d]; children [H,M0,C,d];
 * grandchildren [H,M0,C,C,d], all of `dtype`; 1 <= C <= 8.  No workspace.
 * Kernels: for bf16 with C == 8 and a two-level codebook image that fits one
 * CTA's shared memory (M0 <= 64), the parent and child decisions run on the
 * tensor cores as in avq_quantize, their codebook image in the static scratch
 * array of avq_quantize_noalloc (same set-up and race rules: calls whose
 * executions may overlap on one device must not share it), and a CUDA-core
 * pass refines the keys at a child with its grandchildren; otherwise (also
 * when the image does not fit that array, and under AVQ_PATH_SIMT) one
 * CUDA-core kernel takes all three decisions.
 * AVQ_PATH_TC on a shape without the tensor-core route: AVQ_ERR_UNSUPPORTED.
 */
avq_status avq_quantize3(const avq_dims* dims, avq_dtype dtype, const void* K, const void* V,
                         const void* parents, const void* children, const void* grandchildren,
                         int32_t* assign, float* vsum, int32_t* counts, avq_stream_t stream);

/*
 * avq_attention3 -- Algorithm 2 (Sec. 4.3) over a depth-3 tree.
 *
 * Per query block: the parents' pass and the child refinement of the top-P
 * parents as in avq_attention; then each of the P*C refined children gets
 * an importance in the sense of Eq. 7 with the logits, maximum and
 * denominator of the attention after that refinement,
 *   w_c(I) = sum_{i in I} exp(s_ic - m_i) n_c / z_i,
 * the top-P2 of them (descending, ties to the lower child code) are refined
 * with their grandchildren: the child's logit is the mean of its
 * grandchildren's (Eq. 8), dA = exp(s_ig) - exp(s_ic) (Eq. 9), zero for
 * empty grandchildren, merged with the online maximum.  Y = x / z.
 * Outputs (device): O [B,H,N,d] (dtype); sel [B,H,nblk,P] parents in
 * descending importance; sel2 [B,H,nblk,P2] child codes (M0 + m*C + c) in
 * descending child importance; importance [B,H,nblk,M0] (nullable);
 * importance2 [B,H,nblk,P*C] (nullable), the refined children in the order of
 * sel, C each.  0 <= P <= M0, 0 <= P2 <= P*C, block 64 or 128; vsum and
 * counts as avq_quantize3 writes them.  No workspace.
 * Kernels: for bf16, block 128, C == 8, M0 in {16, 32, 48, 64}, d 64 or 128
 * and P, P2 <= 16, one tensor-core kernel (a CTA per query block; the
 * codeword rows and the value sums, rounded to bf16, are read straight from
 * the arguments, so nothing is prepared); otherwise (and under
 * AVQ_PATH_SIMT) a CUDA-core kernel.  AVQ_PATH_TC on another shape:
 * AVQ_ERR_UNSUPPORTED.
 */
avq_status avq_attention3(const avq_dims* dims, avq_dtype dtype, const void* Q, const void* parents,
                          const void* children, const void* grandchildren, const float* vsum,
                          const int32_t* counts, int P, int P2, int block, float scale, void* O,
                          int32_t* sel, int32_t* sel2, float* importance, float* importance2,
                          avq_stream_t stream);

/*
 * avq_codebook_update -- codebook update for training (Sec. A "Codeword
 * Clustering During Training", Eqs. 11-12).
 *
 * EMA statistics, per head over every batch entry (Eq. 11):
 *   S_x <- lambda S_x + (1 - lambda) ksum_x,  N_x <- lambda N_x + (1 - lambda) counts_x,
 * where ksum, counts are the Eq. 3 statistics of the keys, i.e. the vsum and
 * counts outputs of avq_quantize called with the keys in place of the
 * values (a parent counts its whole cluster, a child the keys that moved to
 * it).  Then each parent becomes its mean S_p / N_p and its children the
 * mass-weighted projection of their means M_c onto sum_c C_pc = C C_p
 * (Eq. 12): C_pc = M_c - delta / (N_c sigma) with delta = sum_c M_c - C C_p
 * and sigma = sum_c 1 / N_c, which restores Eq. 5.  A code whose updated N is
 * 0 has no mean and keeps its current position; massless children do not
 * move (the others absorb delta), and with no massive child all C children
 * shift by delta / C.
 * Arguments (device): ksum [B,H,Mt,d] fp32 and counts [B,H,Mt] int32 (read);
 * S [H,Mt,d] fp32 and Nst [H,Mt] fp32, the EMA state (read and written);
 * parents [H,M0,d] and children [H,M0,C,d] of `dtype`, the codebook (read
 * and rewritten in place).  0 <= lambda <= 1.  dims->N is not used.
 * Arithmetic is fp32; the bf16 codebook is rounded to nearest, so Eq. 5
 * then holds to bf16 rounding.
 */
avq_status avq_codebook_update(const avq_dims* dims, avq_dtype dtype, float lambda,
                               const float* ksum, const int32_t* counts, float* S, float* Nst,
                               void* parents, void* children, avq_stream_t stream);

/*
 * avq_permute -- token reordering gather/scatter (Sec. 4.2 and Fig. 3:
 * tokens reordered along a space-filling curve so that query tiles are
 * spatially compact).
 * X, Y [batch, rows, row_bytes] (device); idx [rows] int32 (device), a
 * permutation of 0..rows-1 shared by every batch entry.
 * inverse == 0: Y[b, i] = X[b, idx[i]]  (gather into curve order)
 * inverse != 0: Y[b, idx[i]] = X[b, i]  (scatter back)
 * row_bytes must be a positive multiple of 16; X and Y must not overlap.
 * On the device, an index outside [0, rows) is refused (that row is not
 * copied) and sets the bounds bit of the device error word, which the next
 * avq_check_device reports as AVQ_ERR_DEVICE; an in-range idx that is not a
 * permutation is not detected.
 */
avq_status avq_permute(const void* X, const int32_t* idx, void* Y, int batch, int rows,
                       int row_bytes, int inverse, avq_stream_t stream);

/*
 * avq_hilbert_order -- host helper: idx[t] = raster index (y*side + x) of the
 * t-th cell of a Hilbert curve over a side x side grid, side a power of two
 * (the power-of-two case of the generalised Hilbert curve of Sec. 4.2).
 * idx is host memory of side*side int32.
 */
avq_status avq_hilbert_order(int side, int32_t* idx);

/*
 * avq_gilbert_order -- host helper: idx[t] = raster index (y*width + x) of the
 * t-th cell of a generalised Hilbert ("Gilbert") curve over a width x height
 * grid of any size (Sec. 4.2 and Fig. 3: tokens reordered so that tiles of
 * consecutive tokens are compact 2-D regions, e.g. the 28 x 28 patch grid).
 * The curve starts at cell (0, 0), moves one cell up, down, left or right at
 * every step and visits every cell once; on a 2^k x 2^k grid it is the curve
 * of avq_hilbert_order.  idx is host memory of width*height int32, the
 * permutation to pass to avq_permute.  Returns AVQ_ERR_INVALID_ARG for a
 * non-positive size, width*height > INT32_MAX or a NULL idx.
 */
avq_status avq_gilbert_order(int width, int height, int32_t* idx);

/*
 * avq_selftest_wait -- self-test of the failure path of the kernels' bounded
 * waits: launches one thread that waits on an mbarrier nothing completes.
 * The wait gives up after timeout_us microseconds (1 .. 1000000), sets the
 * timeout bit of the device error word and the kernel ends; the next
 * avq_check_device then returns AVQ_ERR_TIMEOUT and clears the word.  Every
 * mbarrier wait in the library's kernels takes this path when a copy or MMA
 * completion does not arrive in time (limit 2 s), and the kernels then finish
 * without leaving copies or MMAs in flight.  Asynchronous on `stream`;
 * AVQ_ERR_INVALID_ARG for an out-of-range timeout (before any launch).
 */
avq_status avq_selftest_wait(int timeout_us, avq_stream_t stream);

/*
 * avq_selftest_exp2 -- evaluates the FMA-pipe 2^x that the one-tile attention
 * kernel uses for a quarter of its child exponentials (Cody-Waite reduction
 * to x = j + f, |f| <= 1/2, and a fitted cubic for 2^f; relative error at
 * most 7.5e-5 for normal results), so that tests can hold it to that bound.
 * x, y: device fp32 arrays of n elements (n even, 0 <= n <= 2^30; 8-byte
 * aligned); y[i] = 2^x[i] for -127 <= x[i] < 128 (inputs below -127 are
 * clamped there).  Asynchronous on `stream`; AVQ_ERR_INVALID_ARG for a null
 * pointer, an odd or out-of-range n or a misaligned pointer (before any
 * launch).
 */
avq_status avq_selftest_exp2(const float* x, float* y, int64_t n, avq_stream_t stream);

/* Bytes of device workspace that avq_quantize and avq_attention need for
 * these arguments (the larger of the two).  0 means none. */
size_t avq_workspace_size(const avq_dims* dims, avq_dtype dtype, int deterministic,
                          int two_pass, int P, int block);

/* Synchronises `stream`, reads and clears the current device's error word.
 * Returns AVQ_OK, AVQ_ERR_TIMEOUT, AVQ_ERR_DEVICE or AVQ_ERR_CUDA. */
avq_status avq_check_device(avq_stream_t stream);

/* Thread-local kernel family selection; returns the previous setting, or -1
 * for a value outside avq_path. */
int avq_set_path(int path);

const char* avq_status_string(avq_status status);
/* Thread-local text of the last failure on this thread ("" if none). */
const char* avq_last_error(void);
/* Thread-local, space-separated names of the kernels the last successful
 * call on this thread enqueued. */
const char* avq_last_kernels(void);
/* Library version, major*10000 + minor*100 + patch. */
int avq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AVQ_H */
