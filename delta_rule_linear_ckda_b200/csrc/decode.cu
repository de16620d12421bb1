// Recurrent decode step: one token for every (sequence, head), in place on
// the fp32 state.  ("Complex KDA ..." page, section "Yazilim Gelistirme
// Acisindan Pratik Cikarimlar": constant-size state at inference.)
//
// Per (b, h), with S' = Diag(alpha) S:
//   r = S'^T k,  p = S'^T q,  u = beta (v - r),  o = p + (k . q) u,
//   S <- S' + k u^T
// which is S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T and
// o_t = S_t^T q_t rearranged so that S is read once and written once.
//
// The step moves 2 * d_k * d_v * 4 bytes of state per head and does ~6
// flops per state element: it is bound by HBM bandwidth.  Each CTA owns
// one (b, h); each thread owns 4 adjacent columns (one 16-byte vector) of
// d_k * d_v / (4 * blockDim) rows, held in registers between the read and
// the write.  Column reductions over d_k combine register partials through
// shared memory.  State traffic uses streaming cache hints (each element is
// touched once per step).
#include "common.cuh"

namespace ckda {

template <int DK, int DV>
struct DecodeShape {
  static constexpr int kCpr = DV / 4;  // threads across one row (float4 each)
  static constexpr int kThreads = (DK * DV / 4 < 256) ? DK * DV / 4 : 256;
  static constexpr int kRpp = kThreads / kCpr;  // rows covered per pass
  static constexpr int kRows = DK / kRpp;       // rows per thread
  static_assert(kThreads % 32 == 0 || kThreads < 32, "block size");
  static_assert(DK % kRpp == 0, "row split");
};

template <int DK, int DV, typename Tin, typename Tout>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::kThreads, 2)
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, const float* __restrict__ alpha,
                   const float* __restrict__ beta, float* __restrict__ S,
                   Tout* __restrict__ out) {
  using Sh = DecodeShape<DK, DV>;
  constexpr int CPR = Sh::kCpr, RPP = Sh::kRpp, NR = Sh::kRows, NT = Sh::kThreads;
  __shared__ float4 red_r[RPP][CPR];
  __shared__ float4 red_p[RPP][CPR];
  __shared__ float kq_part[(NT + 31) / 32];

  const int bh = blockIdx.x;
  const int t = threadIdx.x;
  const int c = t % CPR;
  const int g = t / CPR;
  const size_t kvec = (size_t)bh * DK;
  float4* Sb = reinterpret_cast<float4*>(S + (size_t)bh * DK * DV);

  // Issue every state load first (16 bytes each, streaming).
  float4 s[NR];
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const int i = g + RPP * m;
    s[m] = __ldcs(Sb + (size_t)i * CPR + c);
  }
  float kr[NR];
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const int i = g + RPP * m;
    const float a = __ldg(alpha + kvec + i);
    const float kk = Elem<Tin>::to_f32(k[kvec + i]);
    const float qq = Elem<Tin>::to_f32(q[kvec + i]);
    kr[m] = kk;
    s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
    r.x = fmaf(s[m].x, kk, r.x); r.y = fmaf(s[m].y, kk, r.y);
    r.z = fmaf(s[m].z, kk, r.z); r.w = fmaf(s[m].w, kk, r.w);
    p.x = fmaf(s[m].x, qq, p.x); p.y = fmaf(s[m].y, qq, p.y);
    p.z = fmaf(s[m].z, qq, p.z); p.w = fmaf(s[m].w, qq, p.w);
  }
  red_r[g][c] = r;
  red_p[g][c] = p;

  // k . q over d_k: one partial per warp, summed below.
  float kq = 0.f;
  for (int i = t; i < DK; i += NT)
    kq = fmaf(Elem<Tin>::to_f32(k[kvec + i]), Elem<Tin>::to_f32(q[kvec + i]), kq);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
  if ((t & 31) == 0) kq_part[t >> 5] = kq;
  __syncthreads();

  float4 R = red_r[0][c], P = red_p[0][c];
#pragma unroll 8
  for (int gg = 1; gg < RPP; ++gg) {
    const float4 a = red_r[gg][c], b = red_p[gg][c];
    R.x += a.x; R.y += a.y; R.z += a.z; R.w += a.w;
    P.x += b.x; P.y += b.y; P.z += b.z; P.w += b.w;
  }
  float kqt = 0.f;
#pragma unroll
  for (int w = 0; w < (NT + 31) / 32; ++w) kqt += kq_part[w];

  const float bt = __ldg(beta + bh);
  const float4 vv = load4_f32(v + (size_t)bh * DV + 4 * c);
  float4 u;
  u.x = bt * (vv.x - R.x); u.y = bt * (vv.y - R.y);
  u.z = bt * (vv.z - R.z); u.w = bt * (vv.w - R.w);
  if (g == 0) {
    float4 o;
    o.x = fmaf(kqt, u.x, P.x); o.y = fmaf(kqt, u.y, P.y);
    o.z = fmaf(kqt, u.z, P.z); o.w = fmaf(kqt, u.w, P.w);
    store4(out + (size_t)bh * DV + 4 * c, o);
  }
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const int i = g + RPP * m;
    float4 o = s[m];
    o.x = fmaf(kr[m], u.x, o.x); o.y = fmaf(kr[m], u.y, o.y);
    o.z = fmaf(kr[m], u.z, o.z); o.w = fmaf(kr[m], u.w, o.w);
    __stcs(Sb + (size_t)i * CPR + c, o);
  }
}

template <int DK, int DV, typename Tin, typename Tout>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* alpha,
                                   const float* beta, float* S, void* out, int BH,
                                   cudaStream_t stream) {
  using Sh = DecodeShape<DK, DV>;
  decode_step_kernel<DK, DV, Tin, Tout><<<BH, Sh::kThreads, 0, stream>>>(
      static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v), alpha,
      beta, S, static_cast<Tout*>(out));
  return cudaGetLastError();
}

template <int DK, typename Tin, typename Tout>
static cudaError_t launch_decode_dv(int dv, const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, float* S, void* out,
                                    int BH, cudaStream_t stream) {
  switch (dv) {
    case 16: return launch_decode_t<DK, 16, Tin, Tout>(q, k, v, alpha, beta, S, out, BH, stream);
    case 32: return launch_decode_t<DK, 32, Tin, Tout>(q, k, v, alpha, beta, S, out, BH, stream);
    case 64: return launch_decode_t<DK, 64, Tin, Tout>(q, k, v, alpha, beta, S, out, BH, stream);
    case 128: return launch_decode_t<DK, 128, Tin, Tout>(q, k, v, alpha, beta, S, out, BH, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename Tin, typename Tout>
static cudaError_t launch_decode_dk(int dk, int dv, const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, float* S, void* out,
                                    int BH, cudaStream_t stream) {
  switch (dk) {
    case 16: return launch_decode_dv<16, Tin, Tout>(dv, q, k, v, alpha, beta, S, out, BH, stream);
    case 32: return launch_decode_dv<32, Tin, Tout>(dv, q, k, v, alpha, beta, S, out, BH, stream);
    case 64: return launch_decode_dv<64, Tin, Tout>(dv, q, k, v, alpha, beta, S, out, BH, stream);
    case 128: return launch_decode_dv<128, Tin, Tout>(dv, q, k, v, alpha, beta, S, out, BH, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(int dtype, int out_dtype, int dk, int dv, const void* q, const void* k,
                          const void* v, const float* alpha, const float* beta, float* S, void* out,
                          int BH, cudaStream_t stream) {
  if (dtype == CKDA_BF16) {
    if (out_dtype == CKDA_BF16)
      return launch_decode_dk<__nv_bfloat16, __nv_bfloat16>(dk, dv, q, k, v, alpha, beta, S, out,
                                                            BH, stream);
    return launch_decode_dk<__nv_bfloat16, float>(dk, dv, q, k, v, alpha, beta, S, out, BH, stream);
  }
  if (out_dtype == CKDA_BF16)
    return launch_decode_dk<float, __nv_bfloat16>(dk, dv, q, k, v, alpha, beta, S, out, BH, stream);
  return launch_decode_dk<float, float>(dk, dv, q, k, v, alpha, beta, S, out, BH, stream);
}

}  // namespace ckda
