// C ABI of libavq.so: host-side validation and dispatch.  Every check runs on
// the host before anything is enqueued; a failed check launches nothing.
#include <math.h>
#include <stdarg.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace avq {

// One error word per device (module-scope device memory, created with the
// module; no allocation by the library).
__device__ unsigned int g_avq_error_word;

namespace {
avq_status noalloc_scratch(void** out);  // the static scratch of this device (defined below)
thread_local char t_error[512];
thread_local char t_kernels[512];
thread_local int t_path = AVQ_PATH_AUTO;

avq_status fail(avq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_error, sizeof(t_error), fmt, ap);
  va_end(ap);
  return s;
}

// Host-side fault injection for tests of the callers' error handling: when
// the environment variable AVQ_FAULT names an entry point ("quantize",
// "attention", "codebook_update", "permute") or is "all", that call returns
// AVQ_ERR_CUDA after its argument checks and before anything reaches the GPU.
bool injected(const char* entry) {
  const char* v = getenv("AVQ_FAULT");
  if (v == nullptr || *v == 0) return false;
  return strcmp(v, "all") == 0 || strcmp(v, entry) == 0;
}
avq_status injected_fail(const char* entry) {
  return fail(AVQ_ERR_CUDA, "injected failure before launch (AVQ_FAULT=%s, %s)", getenv("AVQ_FAULT"), entry);
}

avq_status cuda_fail(cudaError_t e, const char* where) {
  return fail(AVQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  return dev;
}

avq_status check_dims(const avq_dims* d, avq_dtype dt) {
  if (d == nullptr) return fail(AVQ_ERR_INVALID_ARG, "dims is NULL");
  if (dt != AVQ_F32 && dt != AVQ_BF16) return fail(AVQ_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (d->B < 1 || d->H < 1 || d->N < 1)
    return fail(AVQ_ERR_INVALID_ARG, "B, H and N must be >= 1 (got %d, %d, %d)", d->B, d->H, d->N);
  if (d->d != 64 && d->d != 128) return fail(AVQ_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d->d);
  if (d->M0 < 1 || d->M0 > 256) return fail(AVQ_ERR_UNSUPPORTED, "M0 must be in [1, 256] (got %d)", d->M0);
  if (d->C < 0 || d->C > 8) return fail(AVQ_ERR_UNSUPPORTED, "C must be in [0, 8] (got %d)", d->C);
  const long long rows = (long long)d->B * d->H * d->N;
  if (rows > (1ll << 31) - 1)
    return fail(AVQ_ERR_UNSUPPORTED, "B*H*N = %lld exceeds the supported range", rows);
  if ((long long)d->B * d->H > 65535)  // several kernels take one grid row per (batch, head)
    return fail(AVQ_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535", (long long)d->B * d->H);
  return AVQ_OK;
}

Shape to_shape(const avq_dims* d) { return Shape{d->B, d->H, d->N, d->d, d->M0, d->C}; }

avq_status check_ws(size_t need, void* ws, size_t ws_bytes) {
  if (need == 0) return AVQ_OK;
  if (ws == nullptr || ws_bytes < need)
    return fail(AVQ_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu at %p)", need,
                ws_bytes, ws);
  if (!aligned(ws, 256)) return fail(AVQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  return AVQ_OK;
}

#define AVQ_REQUIRE_PTR(p, name)                                                        \
  do {                                                                                  \
    if ((p) == nullptr) return fail(AVQ_ERR_INVALID_ARG, "%s is NULL", name);           \
    if (!aligned((p), 16)) return fail(AVQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

}  // namespace

void LaunchLog::add(const char* name) {
  const int n = (int)strlen(name);
  if (len + n + 2 >= (int)sizeof(text)) return;
  if (len) text[len++] = ' ';
  memcpy(text + len, name, n);
  len += n;
  text[len] = 0;
}

unsigned int* error_word() {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_avq_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_err_ptr[dev];
}

int num_sms() {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sms[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    g_sms[dev] = v;
  }
  return g_sms[dev];
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}
}  // namespace

cudaError_t make_tmap_3d_bf16(CUtensorMap* map, const void* base, int inner, int rows, int batch,
                              int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)batch};
  const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * rows};
  const cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace avq

using namespace avq;

extern "C" {

const char* avq_status_string(avq_status s) {
  switch (s) {
    case AVQ_OK: return "AVQ_OK";
    case AVQ_ERR_INVALID_ARG: return "AVQ_ERR_INVALID_ARG";
    case AVQ_ERR_UNSUPPORTED: return "AVQ_ERR_UNSUPPORTED";
    case AVQ_ERR_CUDA: return "AVQ_ERR_CUDA";
    case AVQ_ERR_DEVICE: return "AVQ_ERR_DEVICE";
    case AVQ_ERR_TIMEOUT: return "AVQ_ERR_TIMEOUT";
    case AVQ_ERR_WORKSPACE: return "AVQ_ERR_WORKSPACE";
  }
  return "AVQ_ERR_UNKNOWN";
}

const char* avq_last_error(void) { return t_error; }
const char* avq_last_kernels(void) { return t_kernels; }
int avq_version(void) { return 100; }

int avq_set_path(int path) {
  if (path != AVQ_PATH_AUTO && path != AVQ_PATH_SIMT && path != AVQ_PATH_TC) return -1;
  const int old = t_path;
  t_path = path;
  return old;
}

size_t avq_workspace_size(const avq_dims* dims, avq_dtype dtype, int deterministic, int two_pass,
                          int P, int block) {
  if (dims == nullptr) return 0;
  const Shape s = to_shape(dims);
  size_t need = 0;
  if (assign_tc_supported(s, dtype)) need += (assign_tc_workspace(s) + 255) & ~(size_t)255;
  if (deterministic) need += aggregate_det_workspace(s);
  if (attention_tc_supported(s, dtype, P, block, two_pass)) {
    const size_t a = attention_tc_workspace(s, P, block, two_pass);
    if (a > need) need = a;
  }
  return need;
}

avq_status avq_quantize(const avq_dims* dims, avq_dtype dtype, const void* K, const void* V,
                        const void* parents, const void* children, int32_t* assign, float* vsum,
                        int32_t* counts, int deterministic, void* ws, size_t ws_bytes,
                        avq_stream_t stream) {
  t_error[0] = 0;
  avq_status st = check_dims(dims, dtype);
  if (st != AVQ_OK) return st;
  const Shape s = to_shape(dims);
  AVQ_REQUIRE_PTR(K, "K");
  AVQ_REQUIRE_PTR(V, "V");
  AVQ_REQUIRE_PTR(parents, "parents");
  if (s.C > 0) AVQ_REQUIRE_PTR(children, "children");
  AVQ_REQUIRE_PTR(assign, "assign");
  AVQ_REQUIRE_PTR(vsum, "vsum");
  AVQ_REQUIRE_PTR(counts, "counts");
  const bool tc_ok = assign_tc_supported(s, dtype);
  if (t_path == AVQ_PATH_TC && !tc_ok)
    return fail(AVQ_ERR_UNSUPPORTED, "no tensor-core assignment kernel for this shape/dtype");
  const bool use_tc = tc_ok && t_path != AVQ_PATH_SIMT;
  // workspace: [tensor-core codebook image | deterministic reduction scratch]
  const size_t ws_tc = use_tc ? (assign_tc_workspace(s) + 255) & ~(size_t)255 : 0;
  const size_t ws_det = deterministic ? aggregate_det_workspace(s) : 0;
  if (ws_tc + ws_det > 0) {
    st = check_ws(ws_tc + ws_det, ws, ws_bytes);
    if (st != AVQ_OK) return st;
  }
  void* ws_det_ptr = ws_det ? static_cast<char*>(ws) + ws_tc : nullptr;
  if (injected("quantize")) return injected_fail("avq_quantize");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  LaunchLog log{};
  cudaError_t e;
  unsigned int* err = error_word();
  if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
  // the tensor-core path zeroes counts (and, for the atomic-order value sums,
  // vsum) in its codebook preparation launch
  bool counts_left = false;  // counts left by the assignment to the streaming sums
  if (use_tc) {
    e = launch_assign_tc(s, K, parents, children, assign, counts, ws, err, cs, log,
                         deterministic ? nullptr : vsum, deterministic ? nullptr : &counts_left);
  } else {
    e = cudaMemsetAsync(counts, 0, (size_t)s.BH() * s.Mt() * sizeof(int32_t), cs);
    if (e != cudaSuccess) return cuda_fail(e, "zero counts");
    e = launch_assign_simt(s, dtype, K, parents, children, assign, counts, cs, log);
  }
  if (e != cudaSuccess) return cuda_fail(e, "assignment launch");
  if (deterministic)
    e = launch_aggregate_det(s, dtype, V, assign, vsum, counts, ws_det_ptr, cs, log);
  else
    e = launch_aggregate(s, dtype, V, assign, vsum, counts, err, cs, log, use_tc, false, counts_left);
  if (e != cudaSuccess) return cuda_fail(e, "aggregation launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}

avq_status avq_attention(const avq_dims* dims, avq_dtype dtype, const void* Q, const void* parents,
                         const void* children, const float* vsum, const int32_t* counts, int P,
                         int block, float scale, int two_pass, void* O, int32_t* sel,
                         float* importance, void* ws, size_t ws_bytes, avq_stream_t stream) {
  t_error[0] = 0;
  avq_status st = check_dims(dims, dtype);
  if (st != AVQ_OK) return st;
  const Shape s = to_shape(dims);
  if (P < 0 || P > s.M0) return fail(AVQ_ERR_INVALID_ARG, "P must be in [0, M0] (got %d)", P);
  if (block != 64 && block != 128)
    return fail(AVQ_ERR_UNSUPPORTED, "block must be 64 or 128 (got %d)", block);
  if (!(scale > 0.f) || !isfinite(scale))
    return fail(AVQ_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (two_pass < 0 || two_pass > 2)
    return fail(AVQ_ERR_INVALID_ARG, "two_pass must be 0, 1 or 2 (got %d)", two_pass);
  AVQ_REQUIRE_PTR(Q, "Q");
  AVQ_REQUIRE_PTR(parents, "parents");
  if (s.C > 0) AVQ_REQUIRE_PTR(children, "children");
  AVQ_REQUIRE_PTR(vsum, "vsum");
  AVQ_REQUIRE_PTR(counts, "counts");
  AVQ_REQUIRE_PTR(O, "O");
  if (P > 0) AVQ_REQUIRE_PTR(sel, "sel");
  if (importance != nullptr && !aligned(importance, 16))
    return fail(AVQ_ERR_INVALID_ARG, "importance is not 16-byte aligned");
  const bool tc_ok = attention_tc_supported(s, dtype, P, block, two_pass);
  if (t_path == AVQ_PATH_TC && !tc_ok)
    return fail(AVQ_ERR_UNSUPPORTED, "no tensor-core attention kernel for this shape/dtype");
  const bool use_tc = tc_ok && t_path != AVQ_PATH_SIMT;
  // the extrapolated denominator differs from the exact one only over several
  // parent tiles, which only the tensor-core kernel sweeps
  if (two_pass == 2 && s.M0 > 64 && !use_tc)
    return fail(AVQ_ERR_UNSUPPORTED, "the extrapolated denominator needs the tensor-core kernel");
  if (injected("attention")) return injected_fail("avq_attention");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  LaunchLog log{};
  cudaError_t e;
  if (use_tc) {
    st = check_ws(attention_tc_workspace(s, P, block, two_pass), ws, ws_bytes);
    if (st != AVQ_OK) return st;
    unsigned int* err = error_word();
    if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
    // with no selection and no importance output nothing depends on the
    // importance denominator: one sweep over several parent tiles (online
    // maximum); a single tile keeps the one-tile kernel
    const bool one_sweep = two_pass == AVQ_DENOM_AUTO && P == 0 && importance == nullptr && s.M0 > 64;
    const int sweep_mode = one_sweep ? AVQ_DENOM_EXTRAPOLATED : two_pass;
    e = launch_attention_tc(s, Q, parents, children, vsum, counts, P, block, scale, sweep_mode, O,
                            sel, importance, ws, err, cs, log);
  } else {
    e = launch_attention_simt(s, dtype, Q, parents, children, vsum, counts, P, block, scale, O,
                              sel, importance, cs, log);
  }
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}

avq_status avq_quantize3(const avq_dims* dims, avq_dtype dtype, const void* K, const void* V,
                         const void* parents, const void* children, const void* grandchildren,
                         int32_t* assign, float* vsum, int32_t* counts, avq_stream_t stream) {
  t_error[0] = 0;
  avq_status st = check_dims(dims, dtype);
  if (st != AVQ_OK) return st;
  const Shape s = to_shape(dims);
  if (s.C < 1) return fail(AVQ_ERR_INVALID_ARG, "a depth-3 tree needs C >= 1 (got %d)", s.C);
  AVQ_REQUIRE_PTR(K, "K");
  AVQ_REQUIRE_PTR(V, "V");
  AVQ_REQUIRE_PTR(parents, "parents");
  AVQ_REQUIRE_PTR(children, "children");
  AVQ_REQUIRE_PTR(grandchildren, "grandchildren");
  AVQ_REQUIRE_PTR(assign, "assign");
  AVQ_REQUIRE_PTR(vsum, "vsum");
  AVQ_REQUIRE_PTR(counts, "counts");
  // tensor-core path: the two-level warpgroup assignment (its codebook image
  // in the library's static scratch), then the grandchild refinement on the
  // CUDA cores; the counts of all three levels from the value-sum passes
  const bool tc_ok = s.C == 8 && assign_tc_supported(s, dtype) && assign_tc_uses_warpgroups(s) &&
                     assign_tc_workspace(s) <= AVQ_NOALLOC_SCRATCH_BYTES;
  if (t_path == AVQ_PATH_TC && !tc_ok)
    return fail(AVQ_ERR_UNSUPPORTED, "no tensor-core assignment for this depth-3 shape/dtype");
  const bool use_tc = tc_ok && t_path != AVQ_PATH_SIMT;
  if (injected("quantize3")) return injected_fail("avq_quantize3");
  void* scratch = nullptr;
  if (use_tc) {
    st = noalloc_scratch(&scratch);
    if (st != AVQ_OK) return st;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const size_t mt3 = (size_t)s.M0 + (size_t)s.M0 * s.C + (size_t)s.M0 * s.C * s.C;
  LaunchLog log{};
  unsigned int* err = error_word();
  if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
  cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)s.BH() * mt3 * sizeof(int32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "zero counts");
  bool count_in_sums = false;
  if (use_tc) {
    e = launch_assign_tc(s, K, parents, children, assign, counts, scratch, err, cs, log, nullptr,
                         &count_in_sums);
    if (e == cudaSuccess && !count_in_sums) e = cudaErrorInvalidValue;  // the warpgroup kernel must leave the counts
    if (e == cudaSuccess) e = launch_assign3_grandchildren(s, K, children, grandchildren, assign, cs, log);
  } else {
    e = launch_assign3_simt(s, dtype, K, parents, children, grandchildren, assign, counts, cs, log);
  }
  if (e != cudaSuccess) return cuda_fail(e, "assignment launch");
  e = launch_aggregate(s, dtype, V, assign, vsum, counts, err, cs, log, false, true, count_in_sums);
  if (e != cudaSuccess) return cuda_fail(e, "aggregation launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}

avq_status avq_attention3(const avq_dims* dims, avq_dtype dtype, const void* Q, const void* parents,
                          const void* children, const void* grandchildren, const float* vsum,
                          const int32_t* counts, int P, int P2, int block, float scale, void* O,
                          int32_t* sel, int32_t* sel2, float* importance, float* importance2,
                          avq_stream_t stream) {
  t_error[0] = 0;
  avq_status st = check_dims(dims, dtype);
  if (st != AVQ_OK) return st;
  const Shape s = to_shape(dims);
  if (s.C < 1) return fail(AVQ_ERR_INVALID_ARG, "a depth-3 tree needs C >= 1 (got %d)", s.C);
  if (P < 0 || P > s.M0) return fail(AVQ_ERR_INVALID_ARG, "P must be in [0, M0] (got %d)", P);
  if (P2 < 0 || P2 > P * s.C)
    return fail(AVQ_ERR_INVALID_ARG, "P2 must be in [0, P*C] (got %d with P*C = %d)", P2, P * s.C);
  if (block != 64 && block != 128)
    return fail(AVQ_ERR_UNSUPPORTED, "block must be 64 or 128 (got %d)", block);
  if (!(scale > 0.f) || !isfinite(scale)) return fail(AVQ_ERR_INVALID_ARG, "scale must be finite and > 0");
  AVQ_REQUIRE_PTR(Q, "Q");
  AVQ_REQUIRE_PTR(parents, "parents");
  AVQ_REQUIRE_PTR(children, "children");
  AVQ_REQUIRE_PTR(grandchildren, "grandchildren");
  AVQ_REQUIRE_PTR(vsum, "vsum");
  AVQ_REQUIRE_PTR(counts, "counts");
  AVQ_REQUIRE_PTR(O, "O");
  if (P > 0) AVQ_REQUIRE_PTR(sel, "sel");
  if (P2 > 0) AVQ_REQUIRE_PTR(sel2, "sel2");
  if (importance != nullptr && !aligned(importance, 16))
    return fail(AVQ_ERR_INVALID_ARG, "importance is not 16-byte aligned");
  if (importance2 != nullptr && !aligned(importance2, 16))
    return fail(AVQ_ERR_INVALID_ARG, "importance2 is not 16-byte aligned");
  const bool tc_ok = attention3_tc_supported(s, dtype, P, P2, block);
  if (t_path == AVQ_PATH_TC && !tc_ok)
    return fail(AVQ_ERR_UNSUPPORTED, "no tensor-core depth-3 attention for this shape/dtype/P/P2/block");
  if (injected("attention3")) return injected_fail("avq_attention3");
  LaunchLog log{};
  cudaError_t e;
  if (tc_ok && t_path != AVQ_PATH_SIMT) {
    unsigned int* err = error_word();
    if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
    e = launch_attention3_tc(s, Q, parents, children, grandchildren, vsum, counts, P, P2, scale, O, sel, sel2,
                             importance, importance2, err, reinterpret_cast<cudaStream_t>(stream), log);
  } else {
    e = launch_attention3_simt(s, dtype, Q, parents, children, grandchildren, vsum, counts, P, P2, block,
                               scale, O, sel, sel2, importance, importance2,
                               reinterpret_cast<cudaStream_t>(stream), log);
  }
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}

avq_status avq_codebook_update(const avq_dims* dims, avq_dtype dtype, float lambda, const float* ksum,
                               const int32_t* counts, float* S, float* Nst, void* parents, void* children,
                               avq_stream_t stream) {
  t_error[0] = 0;
  avq_status st = check_dims(dims, dtype);
  if (st != AVQ_OK) return st;
  const Shape s = to_shape(dims);
  if (!(lambda >= 0.f && lambda <= 1.f)) return fail(AVQ_ERR_INVALID_ARG, "lambda must be in [0, 1]");
  AVQ_REQUIRE_PTR(ksum, "ksum");
  AVQ_REQUIRE_PTR(counts, "counts");
  AVQ_REQUIRE_PTR(S, "S");
  AVQ_REQUIRE_PTR(Nst, "Nst");
  AVQ_REQUIRE_PTR(parents, "parents");
  if (s.C > 0) AVQ_REQUIRE_PTR(children, "children");
  if (injected("codebook_update")) return injected_fail("avq_codebook_update");
  LaunchLog log{};
  cudaError_t e = launch_codebook_update(s, dtype, lambda, ksum, counts, S, Nst, parents, children,
                                         reinterpret_cast<cudaStream_t>(stream), log);
  if (e != cudaSuccess) return cuda_fail(e, "codebook update launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}

avq_status avq_permute(const void* X, const int32_t* idx, void* Y, int batch, int rows,
                       int row_bytes, int inverse, avq_stream_t stream) {
  t_error[0] = 0;
  if (batch < 1 || rows < 1) return fail(AVQ_ERR_INVALID_ARG, "batch and rows must be >= 1");
  if (row_bytes < 16 || row_bytes % 16 != 0)
    return fail(AVQ_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16");
  AVQ_REQUIRE_PTR(X, "X");
  AVQ_REQUIRE_PTR(Y, "Y");
  if (idx == nullptr) return fail(AVQ_ERR_INVALID_ARG, "idx is NULL");
  if (!aligned(idx, 4)) return fail(AVQ_ERR_INVALID_ARG, "idx is not 4-byte aligned");
  const size_t bytes = (size_t)batch * rows * row_bytes;
  const char* x = static_cast<const char*>(X);
  const char* y = static_cast<const char*>(Y);
  if (x < y + bytes && y < x + bytes) return fail(AVQ_ERR_INVALID_ARG, "X and Y overlap");
  if (injected("permute")) return injected_fail("avq_permute");
  unsigned int* err = error_word();
  if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
  LaunchLog log{};
  cudaError_t e = launch_permute(X, idx, Y, batch, rows, row_bytes, inverse, err,
                                 reinterpret_cast<cudaStream_t>(stream), log);
  if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}

avq_status avq_selftest_wait(int timeout_us, avq_stream_t stream) {
  t_error[0] = 0;
  if (timeout_us < 1 || timeout_us > 1000000)
    return fail(AVQ_ERR_INVALID_ARG, "timeout_us must be in [1, 1000000] (got %d)", timeout_us);
  unsigned int* err = error_word();
  if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
  const cudaError_t e =
      launch_wait_probe(err, 1000ull * (unsigned long long)timeout_us, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", "wait_probe");
  return AVQ_OK;
}

avq_status avq_selftest_exp2(const float* x, float* y, int64_t n, avq_stream_t stream) {
  t_error[0] = 0;
  AVQ_REQUIRE_PTR(x, "x");
  AVQ_REQUIRE_PTR(y, "y");
  if (n < 0 || n > (int64_t(1) << 30) || (n & 1))
    return fail(AVQ_ERR_INVALID_ARG, "n must be even and in [0, 2^30] (got %lld)", (long long)n);
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 7u)
    return fail(AVQ_ERR_INVALID_ARG, "x and y must be 8-byte aligned");
  const cudaError_t e = launch_exp2_probe(x, y, (long long)n, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "exp2 self-test launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", "exp2_probe");
  return AVQ_OK;
}

avq_status avq_check_device(avq_stream_t stream) {
  t_error[0] = 0;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_avq_error_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (word == 0) return AVQ_OK;
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbol(g_avq_error_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  if (word & kErrTimeout) return fail(AVQ_ERR_TIMEOUT, "a bounded device wait ran out (word 0x%x)", word);
  return fail(AVQ_ERR_DEVICE, "device error word 0x%x", word);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// avq_quantize_noalloc: stage 1 for callers that cannot hand the library a
// workspace.  The tensor-core assignment needs a bf16 image of the codebook
// and its squared norms; here they live in a fixed module-scope device array
// instead of caller memory, so the call allocates nothing.
namespace avq {

__device__ __align__(256) unsigned char g_avq_noalloc_scratch[AVQ_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];

// Resolves the scratch array's address on the current device, once per
// device (the first call on a device does this set-up).
avq_status noalloc_scratch(void** out) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_avq_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(AVQ_ERR_CUDA, "cannot resolve the static scratch on device %d: %s", dev,
                  cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return AVQ_OK;
}
}  // namespace
}  // namespace avq

extern "C" avq_status avq_quantize_noalloc(const avq_dims* dims, avq_dtype dtype, const void* K,
                                           const void* V, const void* parents, const void* children,
                                           int32_t* assign, float* vsum, int32_t* counts,
                                           avq_stream_t stream) {
  t_error[0] = 0;
  avq_status st = check_dims(dims, dtype);
  if (st != AVQ_OK) return st;
  const Shape s = to_shape(dims);
  AVQ_REQUIRE_PTR(K, "K");
  AVQ_REQUIRE_PTR(V, "V");
  AVQ_REQUIRE_PTR(parents, "parents");
  if (s.C > 0) AVQ_REQUIRE_PTR(children, "children");
  AVQ_REQUIRE_PTR(assign, "assign");
  AVQ_REQUIRE_PTR(vsum, "vsum");
  AVQ_REQUIRE_PTR(counts, "counts");
  const bool tc_ok = assign_tc_supported(s, dtype);
  if (t_path == AVQ_PATH_TC && !tc_ok)
    return fail(AVQ_ERR_UNSUPPORTED, "no tensor-core assignment kernel for this shape/dtype");
  const bool use_tc = tc_ok && t_path != AVQ_PATH_SIMT;
  if (injected("quantize")) return injected_fail("avq_quantize_noalloc");
  void* scratch = nullptr;
  if (use_tc) {
    const size_t need = assign_tc_workspace(s);
    if (need > AVQ_NOALLOC_SCRATCH_BYTES)
      return fail(AVQ_ERR_WORKSPACE,
                  "the codebook image needs %zu bytes but the static scratch holds %zu; "
                  "call avq_quantize with a workspace instead",
                  need, (size_t)AVQ_NOALLOC_SCRATCH_BYTES);
    st = noalloc_scratch(&scratch);
    if (st != AVQ_OK) return st;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  LaunchLog log{};
  unsigned int* err = error_word();
  if (err == nullptr) return fail(AVQ_ERR_CUDA, "cannot resolve the device error word");
  // The assignment kernels add into counts, so counts must start at zero.
  // The scratch needs no clearing: the codebook image is rewritten in full
  // by every call before the assignment reads it.
  cudaError_t e;
  bool counts_left = false;  // counts left by the assignment to the streaming sums
  if (use_tc) {  // counts and vsum zeroed by the codebook preparation launch
    e = launch_assign_tc(s, K, parents, children, assign, counts, scratch, err, cs, log, vsum, &counts_left);
  } else {
    e = cudaMemsetAsync(counts, 0, (size_t)s.BH() * s.Mt() * sizeof(int32_t), cs);
    if (e != cudaSuccess) return cuda_fail(e, "zero counts");
    e = launch_assign_simt(s, dtype, K, parents, children, assign, counts, cs, log);
  }
  if (e != cudaSuccess) return cuda_fail(e, "assignment launch");
  e = launch_aggregate(s, dtype, V, assign, vsum, counts, err, cs, log, use_tc, false, counts_left);
  if (e != cudaSuccess) return cuda_fail(e, "aggregation launch");
  snprintf(t_kernels, sizeof(t_kernels), "%s", log.text);
  return AVQ_OK;
}
