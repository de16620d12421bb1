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
// Gated DeltaNet-2 ("Gated DeltaNet-2" page, Methodology section 1): the read
// uses e = b . k and u = w . v - r (no beta).  SFDA ("Semidirect Fourier Delta
// Attention (SFDA)" page, "Arquitectura Central"): S' = Lambda S, each pair of
// rows (2p, 2p+1) turned by alpha_p (cos theta_p, sin theta_p); a thread then
// holds whole row pairs, and each pair's (cos, sin) is computed once per row
// group and passed to the group's lanes by warp shuffles.
//
// The step moves 2 * d_k * d_v * 4 bytes of state per head and does ~6
// flops per state element: it is bound by HBM bandwidth.  Each CTA owns
// one (b, h); each thread owns 4 adjacent columns (one 16-byte vector) of
// d_k * d_v / (4 * blockDim) rows, held in registers between the read and
// the write.  Column reductions over d_k combine register partials through
// shared memory.  State traffic uses streaming cache hints (each element is
// touched once per step).  The per-row vectors (k, q, the decay or the
// erase gate: one value per state row, shared by all the threads of a row)
// are requested first, one entry per thread, and staged in shared memory;
// then the state; then v and the write-side gate.  Every global load thus
// precedes the block barriers, which the compiler does not move loads
// across: a CTA waits for one DRAM round trip, not one per barrier.
#include "common.cuh"

namespace ckda {

// Gate families of the decode step.
constexpr int kDecKda = 0, kDecGdn2 = 1, kDecSfda = 2;

template <int DK, int DV, bool SF = false>
struct DecodeShape {
  static constexpr int kCpr = DV / 4;  // threads across one row (float4 each)
  static constexpr int kThreads0 = (DK * DV / 4 < 256) ? DK * DV / 4 : 256;
  // SFDA: at least two rows per thread (a whole row pair)
  static constexpr int kThreads = (SF && DK * kCpr / kThreads0 < 2) ? kThreads0 / 2 : kThreads0;
  static constexpr int kRpp = kThreads / kCpr;  // rows covered per pass
  static constexpr int kRows = DK / kRpp;       // rows per thread
  static_assert(kThreads % 32 == 0 || kThreads < 32, "block size");
  static_assert(DK % kRpp == 0, "row split");
  static_assert(!SF || kRows % 2 == 0, "row pairs");
  // the per-row vectors take one entry per thread
  static_assert(kThreads >= DK, "vector staging");
  // SFDA: a row group's pairs are evaluated by its own lanes (one each) and
  // a group lies within one warp
  static_assert(!SF || (kRows / 2 <= kCpr && 32 % kCpr == 0 && kThreads % 32 == 0), "pair lanes");
};

// bg, wg: the Gated DeltaNet-2 gates ([BH, d_k], [BH, d_v]); theta: the SFDA
// phases ([BH, d_k / 2], alpha then holds d_k / 2 decays); unused otherwise.
template <int DK, int DV, typename Tin, typename Tout, int GK>
__global__ void __launch_bounds__(DecodeShape<DK, DV, GK == kDecSfda>::kThreads, 2)
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, const float* __restrict__ alpha,
                   const float* __restrict__ beta, const float* __restrict__ bg,
                   const float* __restrict__ wg, const float* __restrict__ theta,
                   float* __restrict__ S, Tout* __restrict__ out) {
  constexpr bool G2 = GK == kDecGdn2, SF = GK == kDecSfda;
  using Sh = DecodeShape<DK, DV, SF>;
  constexpr int CPR = Sh::kCpr, RPP = Sh::kRpp, NR = Sh::kRows, NT = Sh::kThreads;
  __shared__ float4 red_r[RPP][CPR];
  __shared__ float4 red_p[RPP][CPR];
  __shared__ float kq_part[(NT + 31) / 32];
  // the per-row vectors: k, q, the decay (not SFDA) and the erase direction
  // b . k (GDN-2)
  __shared__ float vk[DK], vq[DK], va[SF ? 1 : DK], vb[G2 ? DK : 1];

  const int bh = blockIdx.x;
  const int t = threadIdx.x;
  const int c = t % CPR;
  const int g = t / CPR;
  const size_t kvec = (size_t)bh * DK;
  float4* Sb = reinterpret_cast<float4*>(S + (size_t)bh * DK * DV);
  // the rows of this thread: g + RPP m (SFDA: 2 (g + RPP (m / 2)) + m % 2, so
  // both rows of a pair are held by the same thread)
  auto row_of = [&](int m) -> int { return SF ? 2 * (g + RPP * (m >> 1)) + (m & 1) : g + RPP * m; };

  // SFDA: the phase and decay of the pair this thread evaluates (below),
  // requested before the state so that they arrive first
  float th_in = 0.f, al_in = 0.f;
  if constexpr (SF) {
    if (c < NR / 2) {
      th_in = __ldg(theta + (size_t)bh * (DK / 2) + g + RPP * c);
      al_in = __ldg(alpha + (size_t)bh * (DK / 2) + g + RPP * c);
    }
  }
  // the per-row vectors, one entry per thread t < d_k (blockDim >= d_k)
  float lk = 0.f, lq = 0.f, la = 0.f, lb = 0.f;
  if (t < DK) {
    lk = Elem<Tin>::to_f32(k[kvec + t]);
    lq = Elem<Tin>::to_f32(q[kvec + t]);
    if constexpr (!SF) la = __ldg(alpha + kvec + t);
    if constexpr (G2) lb = __ldg(bg + kvec + t);
  }
  // Then every state load (16 bytes each, streaming).
  float4 s[NR];
#pragma unroll
  for (int m = 0; m < NR; ++m) s[m] = __ldcs(Sb + (size_t)row_of(m) * CPR + c);
  if (t < DK) {
    vk[t] = lk;
    vq[t] = lq;
    if constexpr (!SF) va[t] = la;
    if constexpr (G2) vb[t] = lk * lb;
  }
  // this thread's v columns and write-side gate (read after the reduction)
  const float4 vv = load4_f32(v + (size_t)bh * DV + 4 * c);
  float4 ww = make_float4(0.f, 0.f, 0.f, 0.f);
  float bt = 0.f;
  if constexpr (G2)
    ww = *reinterpret_cast<const float4*>(wg + (size_t)bh * DV + 4 * c);
  else
    bt = __ldg(beta + bh);
  __syncthreads();
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (SF) {
    // The pairs' rotation-decay gates: the thread at column j < NR / 2 of a
    // row group evaluates pair g + RPP j (rows 2 (g + RPP j) and the next),
    // which every thread of the group holds; a group is CPR consecutive
    // lanes of one warp, so the others read the value by a shuffle.
    float2 mine = make_float2(0.f, 0.f);
    if (c < NR / 2) {
      float sn, cs;
      sincosf(th_in, &sn, &cs);
      mine = make_float2(al_in * cs, al_in * sn);
    }
    const int lane0 = (t & 31) & ~(CPR - 1);
    // S' = Lambda S on every row pair, then the column sums
#pragma unroll
    for (int m = 0; m < NR; m += 2) {
      const float2 l = make_float2(__shfl_sync(0xffffffffu, mine.x, lane0 + (m >> 1)),
                                   __shfl_sync(0xffffffffu, mine.y, lane0 + (m >> 1)));
      const float4 e = s[m], o = s[m + 1];
      s[m] = make_float4(fmaf(-l.y, o.x, l.x * e.x), fmaf(-l.y, o.y, l.x * e.y),
                         fmaf(-l.y, o.z, l.x * e.z), fmaf(-l.y, o.w, l.x * e.w));
      s[m + 1] = make_float4(fmaf(l.y, e.x, l.x * o.x), fmaf(l.y, e.y, l.x * o.y),
                             fmaf(l.y, e.z, l.x * o.z), fmaf(l.y, e.w, l.x * o.w));
    }
  }
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const int i = row_of(m);
    const float kk = vk[i];
    const float qq = vq[i];
    if constexpr (!SF) {
      const float a = va[i];
      s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;
    }
    const float ek = G2 ? vb[i] : kk;  // the read direction
    r.x = fmaf(s[m].x, ek, r.x); r.y = fmaf(s[m].y, ek, r.y);
    r.z = fmaf(s[m].z, ek, r.z); r.w = fmaf(s[m].w, ek, r.w);
    p.x = fmaf(s[m].x, qq, p.x); p.y = fmaf(s[m].y, qq, p.y);
    p.z = fmaf(s[m].z, qq, p.z); p.w = fmaf(s[m].w, qq, p.w);
  }
  red_r[g][c] = r;
  red_p[g][c] = p;

  // k . q over d_k: one partial per warp, summed below.
  float kq = lk * lq;
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

  float4 u;
  if constexpr (G2) {
    // u = w . v - r
    u.x = fmaf(ww.x, vv.x, -R.x); u.y = fmaf(ww.y, vv.y, -R.y);
    u.z = fmaf(ww.z, vv.z, -R.z); u.w = fmaf(ww.w, vv.w, -R.w);
  } else {
    u.x = bt * (vv.x - R.x); u.y = bt * (vv.y - R.y);
    u.z = bt * (vv.z - R.z); u.w = bt * (vv.w - R.w);
  }
  if (g == 0) {
    float4 o;
    o.x = fmaf(kqt, u.x, P.x); o.y = fmaf(kqt, u.y, P.y);
    o.z = fmaf(kqt, u.z, P.z); o.w = fmaf(kqt, u.w, P.w);
    store4(out + (size_t)bh * DV + 4 * c, o);
  }
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const int i = row_of(m);
    float4 o = s[m];
    const float kk = vk[i];
    o.x = fmaf(kk, u.x, o.x); o.y = fmaf(kk, u.y, o.y);
    o.z = fmaf(kk, u.z, o.z); o.w = fmaf(kk, u.w, o.w);
    __stcs(Sb + (size_t)i * CPR + c, o);
  }
}

// Gates of a decode call: beta (CKDA), b and w (Gated DeltaNet-2), or beta
// with the phases (SFDA).
struct DecGates {
  const float* beta;
  const float* b;
  const float* w;
  const float* theta;
};

template <int DK, int DV, typename Tin, typename Tout>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const float* alpha,
                                   DecGates gt, float* S, void* out, int BH, cudaStream_t stream) {
#define CKDA_DEC(GKV)                                                                          \
  decode_step_kernel<DK, DV, Tin, Tout, GKV>                                                   \
      <<<BH, DecodeShape<DK, DV, GKV == kDecSfda>::kThreads, 0, stream>>>(                      \
          static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v),   \
          alpha, gt.beta, gt.b, gt.w, gt.theta, S, static_cast<Tout*>(out))
  if (gt.theta != nullptr)
    CKDA_DEC(kDecSfda);
  else if (gt.b != nullptr)
    CKDA_DEC(kDecGdn2);
  else
    CKDA_DEC(kDecKda);
#undef CKDA_DEC
  return cudaGetLastError();
}

template <int DK, typename Tin, typename Tout>
static cudaError_t launch_decode_dv(int dv, const void* q, const void* k, const void* v,
                                    const float* alpha, DecGates gt, float* S, void* out, int BH,
                                    cudaStream_t stream) {
  switch (dv) {
    case 16: return launch_decode_t<DK, 16, Tin, Tout>(q, k, v, alpha, gt, S, out, BH, stream);
    case 32: return launch_decode_t<DK, 32, Tin, Tout>(q, k, v, alpha, gt, S, out, BH, stream);
    case 64: return launch_decode_t<DK, 64, Tin, Tout>(q, k, v, alpha, gt, S, out, BH, stream);
    case 128: return launch_decode_t<DK, 128, Tin, Tout>(q, k, v, alpha, gt, S, out, BH, stream);
  }
  return cudaErrorInvalidValue;
}

template <typename Tin, typename Tout>
static cudaError_t launch_decode_dk(int dk, int dv, const void* q, const void* k, const void* v,
                                    const float* alpha, DecGates gt, float* S, void* out, int BH,
                                    cudaStream_t stream) {
  switch (dk) {
    case 16: return launch_decode_dv<16, Tin, Tout>(dv, q, k, v, alpha, gt, S, out, BH, stream);
    case 32: return launch_decode_dv<32, Tin, Tout>(dv, q, k, v, alpha, gt, S, out, BH, stream);
    case 64: return launch_decode_dv<64, Tin, Tout>(dv, q, k, v, alpha, gt, S, out, BH, stream);
    case 128: return launch_decode_dv<128, Tin, Tout>(dv, q, k, v, alpha, gt, S, out, BH, stream);
  }
  return cudaErrorInvalidValue;
}

// bg and wg non-NULL: the Gated DeltaNet-2 form (beta unused); theta
// non-NULL: the SFDA form (alpha holds d_k / 2 decays).
cudaError_t launch_decode(int dtype, int out_dtype, int dk, int dv, const void* q, const void* k,
                          const void* v, const float* alpha, const float* beta, const float* bg,
                          const float* wg, const float* theta, float* S, void* out, int BH,
                          cudaStream_t stream) {
  const DecGates gt{beta, bg, wg, theta};
  if (dtype == CKDA_BF16) {
    if (out_dtype == CKDA_BF16)
      return launch_decode_dk<__nv_bfloat16, __nv_bfloat16>(dk, dv, q, k, v, alpha, gt, S, out,
                                                            BH, stream);
    return launch_decode_dk<__nv_bfloat16, float>(dk, dv, q, k, v, alpha, gt, S, out, BH, stream);
  }
  if (out_dtype == CKDA_BF16)
    return launch_decode_dk<float, __nv_bfloat16>(dk, dv, q, k, v, alpha, gt, S, out, BH, stream);
  return launch_decode_dk<float, float>(dk, dv, q, k, v, alpha, gt, S, out, BH, stream);
}

}  // namespace ckda
