// Host side of libckda.so: argument validation, the device status word and
// dispatch to the kernels.  Every check happens before any CUDA call, so an
// argument error launches nothing and touches no memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "ckda.h"

namespace ckda {
cudaError_t launch_decode(int dtype, int out_dtype, int dk, int dv, const void* q, const void* k,
                          const void* v, const float* alpha, const float* beta, const float* bg,
                          const float* wg, const float* theta, float* S, void* out, int BH,
                          cudaStream_t stream);
cudaError_t launch_fwd_simt(int dtype, int out_dtype, int dk, int dv, const void* q,
                            const void* k, const void* v, const float* alpha, const float* beta,
                            const float* bg, const float* wg, const float* theta,
                            const float* S0, const int32_t* cu, void* out, float* S_final,
                            int n_seqs, int T, int H, int C, int* status, cudaStream_t stream);
// Returns cudaErrorNotSupported when the shape is not covered by the
// tensor-core kernels (the caller then uses the CUDA-core kernel).
cudaError_t launch_fwd_tc(int phases, int dtype, int out_dtype, int dk, int dv, const void* q,
                          const void* k, const void* v, const float* alpha, const float* beta,
                          const float* bg, const float* wg, const float* theta, const float* S0,
                          const int32_t* cu, void* out, float* S_final, int n_seqs, int T, int H,
                          int C, void* ws, int* status, cudaStream_t stream);
bool fwd_tc_supported(int dtype, int dk, int dv, int C, int n_seqs, int T, int H, bool varlen);
size_t fwd_tc_workspace_bytes(int dtype, int dk, int dv, int C, int n_seqs, int T, int H,
                              bool varlen);
cudaError_t launch_bounded_wait_probe(int* status, unsigned long long limit_ns,
                                      cudaStream_t stream);
size_t bwd_workspace_bytes(int dk, int dv, int n_seqs, int T, int H, bool varlen);
size_t fwd_tc_scan_workspace_bytes(int dk, int dv, int n_seqs, int T, int H, int G);
cudaError_t launch_fwd_tc_scan(int out_dtype, int dv, const void* q, const void* k,
                               const void* v, const float* alpha, const float* beta,
                               const float* S0, void* out, float* S_final, int n_seqs, int T,
                               int H, int G, void* ws, int* status, cudaStream_t stream);
cudaError_t launch_bwd(int dtype, int grad_dtype, int dk_, int dv_, const void* q, const void* k,
                       const void* v, const float* alpha, const float* beta, const float* S0,
                       const int32_t* cu, const void* dO, const float* dSf, float* dq, float* dk,
                       float* dv, float* dalpha, float* dbeta, float* dS0, void* ws, int n_seqs,
                       int T, int H, int* status, cudaStream_t stream);
}  // namespace ckda

// First device-side error since the last ckda_device_status() call.
__device__ int g_ckda_status = 0;

// Scratch of ckda_fwd_chunked_static: one fixed array per device, allocated
// with the module, never by a call.  Nothing in it needs to start at zero.
static __device__ __align__(256) uint8_t g_ckda_scratch[CKDA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int*> g_status_ptr[kMaxDevices];

// Device address of the status word on the current device (looked up once
// per device; cudaGetSymbolAddress needs that device to be current).
int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int* p = g_status_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_ckda_status) != cudaSuccess) return nullptr;
    p = static_cast<int*>(addr);
    g_status_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the static scratch on the current device, looked up
// once per device (the first call on a device must not be inside a stream
// capture: the lookup is not a stream operation).
void* scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_ckda_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// Forward phases: the inputs are read by the factor phase, out is written by
// the carry phase; the one-call forward runs both.
constexpr int kFactors = 1, kCarry = 2, kBoth = 3;

int validate_fwd(const void* q, const void* k, const void* v, const float* alpha,
                 const float* beta, const float* S0, const int32_t* cu, const void* out,
                 const float* S_final, int B, int T, int H, int d_k, int d_v, int* chunk,
                 int dtype, int out_dtype, int phases = kBoth) {
  if (B < 0 || T < 0 || H <= 0) return CKDA_ERR_INVALID_ARG;
  if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
  if (out_dtype != CKDA_F32 && out_dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
  if (!supported_d(d_k) || !supported_d(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (*chunk == 0) *chunk = 64;
  if (*chunk != 16 && *chunk != 32 && *chunk != 64) return CKDA_ERR_UNSUPPORTED;
  const int64_t tokens = (cu != nullptr) ? (int64_t)T : (int64_t)B * T;
  if (tokens > 0 && (phases & kFactors) && (!q || !k || !v || !alpha || !beta))
    return CKDA_ERR_INVALID_ARG;
  if (tokens > 0 && (phases & kCarry) && (!out || !v)) return CKDA_ERR_INVALID_ARG;
  if (cu == nullptr && (int64_t)B * T * H > (int64_t)INT32_MAX) return CKDA_ERR_UNSUPPORTED;
  if (cu != nullptr && B == 0 && T != 0) return CKDA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, alpha, beta, S0, out, S_final, cu};
  for (const void* p : ptrs)
    if (p != nullptr && !aligned16(p) && p != cu) return CKDA_ERR_MISALIGNED;
  if (cu != nullptr && (reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return CKDA_ERR_MISALIGNED;
  if (out != nullptr && (out == q || out == k || out == v || out == alpha || out == beta))
    return CKDA_ERR_INVALID_ARG;
  return CKDA_OK;
}

// `bg` and `wg` non-NULL select the Gated DeltaNet-2 form: `bg` takes beta's
// place in the shared checks, `wg` is checked here.  `sfda` selects the SFDA
// form: `theta` (required when there are tokens) is checked here.
int fwd_impl(bool allow_tc, int phases, const void* q, const void* k, const void* v,
             const float* alpha, const float* beta, const float* bg, const float* wg,
             const float* S0, const int32_t* cu, void* out, float* S_final, int B, int T, int H,
             int d_k, int d_v, int chunk, int dtype, int out_dtype, void* workspace,
             size_t workspace_bytes, void* stream, bool sfda = false,
             const float* theta = nullptr) {
  const bool gdn2 = bg != nullptr || wg != nullptr;
  int rc = validate_fwd(q, k, v, alpha, gdn2 ? bg : beta, S0, cu, out, S_final, B, T, H, d_k,
                        d_v, &chunk, dtype, out_dtype, phases);
  if (rc != CKDA_OK) return rc;
  const int64_t tokens = (cu != nullptr) ? (int64_t)T : (int64_t)B * T;
  if (gdn2) {
    if (tokens > 0 && (bg == nullptr || wg == nullptr)) return CKDA_ERR_INVALID_ARG;
    if (wg != nullptr && !aligned16(wg)) return CKDA_ERR_MISALIGNED;
    if (out != nullptr && out == wg) return CKDA_ERR_INVALID_ARG;
  }
  if (sfda) {
    if (tokens > 0 && theta == nullptr) return CKDA_ERR_INVALID_ARG;
    if (theta != nullptr && !aligned16(theta)) return CKDA_ERR_MISALIGNED;
    if (out != nullptr && out == theta) return CKDA_ERR_INVALID_ARG;
  }
  const int n_seqs = B;
  const bool tc = allow_tc && n_seqs > 0 &&
                  ckda::fwd_tc_supported(dtype, d_k, d_v, chunk, n_seqs, T, H, cu != nullptr);
  // the two-phase calls exist only on the tensor-core path
  if (phases != kBoth && !tc && n_seqs > 0) return CKDA_ERR_UNSUPPORTED;
  if (n_seqs == 0) return CKDA_OK;
  if (tc) {
    const size_t need =
        ckda::fwd_tc_workspace_bytes(dtype, d_k, d_v, chunk, n_seqs, T, H, cu != nullptr);
    if (workspace == nullptr || workspace_bytes < need ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return CKDA_ERR_WORKSPACE;
    const void* ws_end = static_cast<const uint8_t*>(workspace) + need;
    const void* ptrs[] = {q, k, v, alpha, beta, bg, wg, theta, S0, out, S_final, cu};
    for (const void* p : ptrs)
      if (p != nullptr && p >= workspace && p < ws_end) return CKDA_ERR_WORKSPACE;
  }
  int* status = status_ptr();
  if (status == nullptr) return CKDA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorNotSupported;
  if (tc)
    e = ckda::launch_fwd_tc(phases, dtype, out_dtype, d_k, d_v, q, k, v, alpha, beta, bg, wg,
                            sfda ? theta : nullptr, S0, cu, out, S_final, n_seqs, T, H, chunk,
                            workspace, status, st);
  if (e == cudaErrorNotSupported)
    e = ckda::launch_fwd_simt(dtype, out_dtype, d_k, d_v, q, k, v, alpha, beta, bg, wg,
                              sfda ? theta : nullptr, S0, cu, out, S_final, n_seqs, T, H, chunk,
                              status, st);
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

// Sizes only: validate with stand-in aligned pointers that are never used.
int validate_sizes(int B, int T, int H, int d_k, int d_v, int* chunk, int dtype, int out_dtype,
                   int varlen) {
  const void* p = reinterpret_cast<const void*>(static_cast<uintptr_t>(1) << 20);
  const int32_t* cu = varlen ? reinterpret_cast<const int32_t*>(static_cast<uintptr_t>(2) << 20)
                             : nullptr;
  return validate_fwd(p, p, p, static_cast<const float*>(p), static_cast<const float*>(p),
                      nullptr, cu, reinterpret_cast<const void*>(static_cast<uintptr_t>(3) << 20),
                      nullptr, B, T, H, d_k, d_v, chunk, dtype, out_dtype);
}

// The decode steps: `bg`, `wg` non-NULL select Gated DeltaNet-2 (b takes
// beta's place in the checks), `theta` non-NULL SFDA.
int decode_impl(const void* q, const void* k, const void* v, const float* alpha,
                const float* beta, const float* bg, const float* wg, const float* theta,
                float* S_inout, void* out, int B, int H, int d_k, int d_v, int dtype,
                int out_dtype, void* stream) {
  if (B < 0 || H <= 0) return CKDA_ERR_INVALID_ARG;
  if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
  if (out_dtype != CKDA_F32 && out_dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
  if (!supported_d(d_k) || !supported_d(d_v)) return CKDA_ERR_UNSUPPORTED;
  if ((int64_t)B * H > (int64_t)INT32_MAX) return CKDA_ERR_UNSUPPORTED;
  if (B == 0) return CKDA_OK;
  const bool g2 = bg != nullptr || wg != nullptr;
  if (!q || !k || !v || !alpha || !S_inout || !out) return CKDA_ERR_INVALID_ARG;
  if (g2 ? (!bg || !wg) : !beta) return CKDA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, alpha, g2 ? bg : beta, wg, theta, S_inout, out};
  for (const void* p : ptrs)
    if (p != nullptr && !aligned16(p)) return CKDA_ERR_MISALIGNED;
  if (out == S_inout || out == q || out == k || out == v) return CKDA_ERR_INVALID_ARG;
  cudaError_t e = ckda::launch_decode(dtype, out_dtype, d_k, d_v, q, k, v, alpha, beta, bg, wg,
                                      theta, S_inout, out, B * H, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}
}  // namespace

extern "C" {

int ckda_version(void) { return 100; }

const char* ckda_status_string(int status) {
  switch (status) {
    case CKDA_OK: return "ok";
    case CKDA_ERR_INVALID_ARG: return "invalid argument (NULL pointer or bad size)";
    case CKDA_ERR_UNSUPPORTED: return "unsupported head size, chunk size or dtype";
    case CKDA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case CKDA_ERR_CUDA: return "CUDA runtime or launch error";
    case CKDA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    case CKDA_ERR_BAD_SEQLENS: return "cu_seqlens is not a valid offsets array";
    case CKDA_ERR_WORKSPACE: return "workspace missing, too small, misaligned or overlapping";
  }
  return "unknown status";
}

int ckda_fwd_chunked(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const float* S0, const int32_t* cu_seqlens, void* out,
                     float* S_final, int B, int T, int H, int d_k, int d_v, int chunk, int dtype,
                     int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_impl(true, kBoth, q, k, v, alpha, beta, nullptr, nullptr, S0, cu_seqlens, out,
                  S_final, B, T, H, d_k, d_v, chunk, dtype, out_dtype, workspace,
                  workspace_bytes, stream);
}

int ckda_fwd_chunked_static(const void* q, const void* k, const void* v, const float* alpha,
                            const float* beta, const float* S0, const int32_t* cu_seqlens,
                            void* out, float* S_final, int B, int T, int H, int d_k, int d_v,
                            int chunk, int dtype, int out_dtype, void* stream) {
  int rc = validate_fwd(q, k, v, alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, d_k, d_v,
                        &chunk, dtype, out_dtype);
  if (rc != CKDA_OK) return rc;
  const size_t need =
      B > 0 ? ckda::fwd_tc_workspace_bytes(dtype, d_k, d_v, chunk, B, T, H, cu_seqlens != nullptr)
            : 0;
  if (need > (size_t)CKDA_STATIC_SCRATCH_BYTES) return CKDA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (need > 0 && (ws = scratch_ptr()) == nullptr) return CKDA_ERR_CUDA;
  return fwd_impl(true, kBoth, q, k, v, alpha, beta, nullptr, nullptr, S0, cu_seqlens, out,
                  S_final, B, T, H, d_k, d_v, chunk, dtype, out_dtype, ws,
                  need > 0 ? (size_t)CKDA_STATIC_SCRATCH_BYTES : 0, stream);
}

int ckda_gdn2_fwd_chunked(const void* q, const void* k, const void* v, const float* alpha,
                          const float* b, const float* w, const float* S0,
                          const int32_t* cu_seqlens, void* out, float* S_final, int B, int T, int H,
                          int d_k, int d_v, int chunk, int dtype, int out_dtype, void* workspace,
                          size_t workspace_bytes, void* stream) {
  // (both gates NULL: checked as the beta form with beta NULL)
  return fwd_impl(true, kBoth, q, k, v, alpha, nullptr, b, w, S0, cu_seqlens, out, S_final, B,
                  T, H, d_k, d_v, chunk, dtype, out_dtype, workspace, workspace_bytes, stream);
}

int ckda_sfda_fwd_chunked(const void* q, const void* k, const void* v, const float* alpha,
                          const float* theta, const float* beta, const float* S0,
                          const int32_t* cu_seqlens, void* out, float* S_final, int B, int T,
                          int H, int d_k, int d_v, int chunk, int dtype, int out_dtype,
                          void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_impl(true, kBoth, q, k, v, alpha, beta, nullptr, nullptr, S0, cu_seqlens, out,
                  S_final, B, T, H, d_k, d_v, chunk, dtype, out_dtype, workspace,
                  workspace_bytes, stream, /*sfda=*/true, theta);
}

int ckda_sfda_fwd_chunked_fp32core(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* theta, const float* beta,
                                   const float* S0, const int32_t* cu_seqlens, void* out,
                                   float* S_final, int B, int T, int H, int d_k, int d_v,
                                   int chunk, int dtype, int out_dtype, void* stream) {
  return fwd_impl(false, kBoth, q, k, v, alpha, beta, nullptr, nullptr, S0, cu_seqlens, out,
                  S_final, B, T, H, d_k, d_v, chunk, dtype, out_dtype, nullptr, 0, stream,
                  /*sfda=*/true, theta);
}

int ckda_fwd_factors(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const int32_t* cu_seqlens, int B, int T, int H, int d_k,
                     int d_v, int chunk, int dtype, void* workspace, size_t workspace_bytes,
                     void* stream) {
  return fwd_impl(true, kFactors, q, k, v, alpha, beta, nullptr, nullptr, nullptr, cu_seqlens,
                  nullptr, nullptr, B, T, H, d_k, d_v, chunk, dtype, CKDA_F32, workspace,
                  workspace_bytes, stream);
}

int ckda_fwd_carry(const void* v, const float* S0, const int32_t* cu_seqlens, void* out,
                   float* S_final, int B, int T, int H, int d_k, int d_v, int chunk, int dtype,
                   int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_impl(true, kCarry, nullptr, nullptr, v, nullptr, nullptr, nullptr, nullptr, S0,
                  cu_seqlens, out, S_final, B, T, H, d_k, d_v, chunk, dtype, out_dtype,
                  workspace, workspace_bytes, stream);
}

int ckda_fwd_chunked_fp32core(const void* q, const void* k, const void* v, const float* alpha,
                              const float* beta, const float* S0, const int32_t* cu_seqlens,
                              void* out, float* S_final, int B, int T, int H, int d_k, int d_v,
                              int chunk, int dtype, int out_dtype, void* stream) {
  return fwd_impl(false, kBoth, q, k, v, alpha, beta, nullptr, nullptr, S0, cu_seqlens, out,
                  S_final, B, T, H, d_k, d_v, chunk, dtype, out_dtype, nullptr, 0, stream);
}

int ckda_fwd_chunked_path(int B, int T, int H, int d_k, int d_v, int chunk, int dtype,
                          int out_dtype, int varlen) {
  int rc = validate_sizes(B, T, H, d_k, d_v, &chunk, dtype, out_dtype, varlen);
  if (rc != CKDA_OK) return rc;
  return ckda::fwd_tc_supported(dtype, d_k, d_v, chunk, B, T, H, varlen != 0) ? 1 : 0;
}

int64_t ckda_fwd_chunked_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk,
                                         int dtype, int out_dtype, int varlen) {
  int rc = validate_sizes(B, T, H, d_k, d_v, &chunk, dtype, out_dtype, varlen);
  if (rc != CKDA_OK) return rc;
  return (int64_t)ckda::fwd_tc_workspace_bytes(dtype, d_k, d_v, chunk, B, T, H, varlen != 0);
}

int64_t ckda_fwd_chunked_scan_workspace_bytes(int B, int T, int H, int d_k, int d_v,
                                              int segments) {
  int chunk = 64;
  int rc = validate_sizes(B, T, H, d_k, d_v, &chunk, CKDA_BF16, CKDA_F32, 0);
  if (rc != CKDA_OK) return rc;
  if (segments < 1) return CKDA_ERR_INVALID_ARG;
  if (B == 0) return 0;
  if (!ckda::fwd_tc_supported(CKDA_BF16, d_k, d_v, 64, B, T, H, false)) return CKDA_ERR_UNSUPPORTED;
  return (int64_t)ckda::fwd_tc_scan_workspace_bytes(d_k, d_v, B, T, H, segments);
}

int ckda_fwd_chunked_scan(const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, const float* S0, void* out, float* S_final, int B,
                          int T, int H, int d_k, int d_v, int chunk, int dtype, int out_dtype,
                          int segments, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_fwd(q, k, v, alpha, beta, S0, nullptr, out, S_final, B, T, H, d_k, d_v,
                        &chunk, dtype, out_dtype);
  if (rc != CKDA_OK) return rc;
  if (segments < 1) return CKDA_ERR_INVALID_ARG;
  if (B == 0) return CKDA_OK;
  if (!ckda::fwd_tc_supported(dtype, d_k, d_v, chunk, B, T, H, false)) return CKDA_ERR_UNSUPPORTED;
  const size_t need = ckda::fwd_tc_scan_workspace_bytes(d_k, d_v, B, T, H, segments);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return CKDA_ERR_WORKSPACE;
  {
    const void* ws_end = static_cast<const uint8_t*>(workspace) + need;
    const void* ptrs[] = {q, k, v, alpha, beta, S0, out, S_final};
    for (const void* p : ptrs)
      if (p != nullptr && p >= workspace && p < ws_end) return CKDA_ERR_WORKSPACE;
  }
  if (S_final != nullptr && S_final == S0 && segments > 1) return CKDA_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (status == nullptr) return CKDA_ERR_CUDA;
  cudaError_t e = ckda::launch_fwd_tc_scan(out_dtype, d_v, q, k, v, alpha, beta, S0, out, S_final,
                                           B, T, H, segments, workspace, status,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

int64_t ckda_bwd_chunked_workspace_bytes(int B, int T, int H, int d_k, int d_v, int varlen) {
  if (B < 0 || T < 0 || H <= 0) return CKDA_ERR_INVALID_ARG;
  if (!supported_d(d_k) || !supported_d(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (varlen && B == 0 && T != 0) return CKDA_ERR_INVALID_ARG;
  if (!varlen && (int64_t)B * T * H > (int64_t)INT32_MAX) return CKDA_ERR_UNSUPPORTED;
  if (B == 0) return 0;
  return (int64_t)ckda::bwd_workspace_bytes(d_k, d_v, B, T, H, varlen != 0);
}

int ckda_bwd_chunked(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const float* S0, const int32_t* cu_seqlens,
                     const void* dO, const float* dS_final, float* dq, float* dk, float* dv,
                     float* dalpha, float* dbeta, float* dS0, int B, int T, int H, int d_k,
                     int d_v, int dtype, int grad_dtype, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (B < 0 || T < 0 || H <= 0) return CKDA_ERR_INVALID_ARG;
  if (dtype != CKDA_F32 && dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
  if (grad_dtype != CKDA_F32 && grad_dtype != CKDA_BF16) return CKDA_ERR_UNSUPPORTED;
  if (!supported_d(d_k) || !supported_d(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (cu_seqlens == nullptr && (int64_t)B * T * H > (int64_t)INT32_MAX) return CKDA_ERR_UNSUPPORTED;
  if (cu_seqlens != nullptr && B == 0 && T != 0) return CKDA_ERR_INVALID_ARG;
  const int64_t tokens = (cu_seqlens != nullptr) ? (int64_t)T : (int64_t)B * T;
  if (tokens > 0 && (!q || !k || !v || !alpha || !beta || !dO || !dq || !dk || !dv || !dalpha ||
                     !dbeta))
    return CKDA_ERR_INVALID_ARG;
  const void* ins[] = {q, k, v, alpha, beta, S0, dO, dS_final};
  const void* outs[] = {dq, dk, dv, dalpha, dbeta, dS0};
  for (const void* p : ins)
    if (p != nullptr && !aligned16(p)) return CKDA_ERR_MISALIGNED;
  for (const void* p : outs)
    if (p != nullptr && !aligned16(p)) return CKDA_ERR_MISALIGNED;
  if (cu_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
    return CKDA_ERR_MISALIGNED;
  for (const void* o : outs) {
    if (o == nullptr) continue;
    for (const void* p : ins)
      if (p != nullptr && o == p) return CKDA_ERR_INVALID_ARG;
  }
  if (B == 0) return CKDA_OK;
  const size_t need = ckda::bwd_workspace_bytes(d_k, d_v, B, T, H, cu_seqlens != nullptr);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return CKDA_ERR_WORKSPACE;
  {
    const void* ws_end = static_cast<const uint8_t*>(workspace) + need;
    for (const void* p : ins)
      if (p != nullptr && p >= workspace && p < ws_end) return CKDA_ERR_WORKSPACE;
    for (const void* p : outs)
      if (p != nullptr && p >= workspace && p < ws_end) return CKDA_ERR_WORKSPACE;
  }
  int* status = status_ptr();
  if (status == nullptr) return CKDA_ERR_CUDA;
  cudaError_t e = ckda::launch_bwd(dtype, grad_dtype, d_k, d_v, q, k, v, alpha, beta, S0,
                                   cu_seqlens, dO, dS_final, dq, dk, dv, dalpha, dbeta, dS0,
                                   workspace, B, T, H, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}


int ckda_decode_step(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, float* S_inout, void* out, int B, int H, int d_k, int d_v,
                     int dtype, int out_dtype, void* stream) {
  return decode_impl(q, k, v, alpha, beta, nullptr, nullptr, nullptr, S_inout, out, B, H, d_k,
                     d_v, dtype, out_dtype, stream);
}

int ckda_gdn2_decode_step(const void* q, const void* k, const void* v, const float* alpha,
                          const float* b, const float* w, float* S_inout, void* out, int B, int H,
                          int d_k, int d_v, int dtype, int out_dtype, void* stream) {
  if (B > 0 && (!b || !w)) return CKDA_ERR_INVALID_ARG;
  return decode_impl(q, k, v, alpha, nullptr, b, w, nullptr, S_inout, out, B, H, d_k, d_v, dtype,
                     out_dtype, stream);
}

int ckda_sfda_decode_step(const void* q, const void* k, const void* v, const float* alpha,
                          const float* theta, const float* beta, float* S_inout, void* out, int B,
                          int H, int d_k, int d_v, int dtype, int out_dtype, void* stream) {
  if (B > 0 && !theta) return CKDA_ERR_INVALID_ARG;
  return decode_impl(q, k, v, alpha, beta, nullptr, nullptr, theta, S_inout, out, B, H, d_k, d_v,
                     dtype, out_dtype, stream);
}

int ckda_selftest_bounded_wait(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 10000000) return CKDA_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (status == nullptr) return CKDA_ERR_CUDA;
  cudaError_t e = ckda::launch_bounded_wait_probe(
      status, 1000ull * (unsigned long long)limit_us, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

int ckda_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return CKDA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ckda_status, sizeof(int)) != cudaSuccess) return CKDA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_ckda_status, &zero, sizeof(int)) != cudaSuccess)
      return CKDA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
