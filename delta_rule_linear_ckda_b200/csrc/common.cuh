// Shared device helpers for the CKDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ckda.h"

namespace ckda {

// Record the first device-side error in the status word (first writer wins).
__device__ __forceinline__ void set_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

// ---- element conversion -------------------------------------------------

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float x) { return x; }
  static __device__ __forceinline__ float from_f32(float x) { return x; }
  // 16 bytes hold 4 values
  static constexpr int kVec = 4;
};

template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
  static constexpr int kVec = 8;
};

// Load 8 consecutive elements (16 bytes for bf16, two 16-byte words for
// fp32) and widen them to fp32.
__device__ __forceinline__ void load8_f32(const float* p, float* dst) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w;
  dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
}

__device__ __forceinline__ void load8_f32(const __nv_bfloat16* p, float* dst) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    dst[2 * i] = f.x;
    dst[2 * i + 1] = f.y;
  }
}

// Load 4 consecutive elements and widen them to fp32.
__device__ __forceinline__ float4 load4_f32(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16* p) {
  uint2 raw = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  float2 a = __bfloat1622float2(h[0]);
  float2 b = __bfloat1622float2(h[1]);
  return make_float4(a.x, a.y, b.x, b.y);
}

// Store 4 consecutive fp32 values, narrowing to the output type.
__device__ __forceinline__ void store4(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}

__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 raw;
  raw.x = *reinterpret_cast<uint32_t*>(&a);
  raw.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = raw;
}

// Packed batches whose CTAs each walk one whole sequence: the sequence the
// CTA with grid index `z` takes is the one of rank z when the sequences are
// ordered by decreasing length (ties by index), so the longest start first
// and the last CTAs the block scheduler hands out are short ones (longest
// processing time first).  The map is a bijection for any offsets array, a
// malformed one included (seq_range still flags it).  Block-wide: every
// thread of the CTA calls it once, before any other use of the barrier.
// Fixed-length batches (cu == NULL) and very large batches keep z.
constexpr int kLongestFirstMaxSeqs = 1024;
__device__ __forceinline__ int seq_longest_first(const int32_t* cu, int n_seqs, int z) {
  if (cu == nullptr || n_seqs > kLongestFirstMaxSeqs) return z;
  __shared__ int pick;
  if (threadIdx.x == 0) pick = z;
  __syncthreads();
  for (int n = threadIdx.x; n < n_seqs; n += blockDim.x) {
    const int ln = cu[n + 1] - cu[n];
    int rank = 0;
    for (int m = 0; m < n_seqs; ++m) {
      const int lm = cu[m + 1] - cu[m];
      rank += (lm > ln || (lm == ln && m < n)) ? 1 : 0;
    }
    if (rank == z) pick = n;
  }
  __syncthreads();
  return pick;
}

// Token range of sequence n: fixed-length batches use n*T .. (n+1)*T;
// packed batches read (and validate) the offsets array.
struct SeqRange {
  int64_t begin;
  int64_t end;
  bool ok;
};

__device__ __forceinline__ SeqRange seq_range(const int32_t* cu, int n, int n_seqs, int T,
                                              int* status) {
  SeqRange r;
  if (cu == nullptr) {
    r.begin = (int64_t)n * T;
    r.end = r.begin + T;
    r.ok = true;
    return r;
  }
  int a = cu[n];
  int b = cu[n + 1];
  bool ok = (a >= 0) && (a <= b) && (b <= T);
  if (n == 0 && a != 0) ok = false;
  if (n == n_seqs - 1 && b != T) ok = false;
  if (!ok) {
    set_status(status, CKDA_ERR_BAD_SEQLENS);
  }
  r.begin = a;
  r.end = b;
  r.ok = ok;
  return r;
}

}  // namespace ckda
