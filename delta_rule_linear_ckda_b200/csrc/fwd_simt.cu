// Chunkwise WY forward of CKDA on fp32 CUDA cores (every product and sum in
// fp32; inputs widened from bf16 or fp32).  This is the fp32-faithful path:
// any d_k, d_v in {16, 32, 64, 128} and chunk C in {16, 32, 64}.
//
// Chunk algebra (for one chunk of positions r = 0..C-1 with start state S0,
// P(r, s) = alpha_{s+1} * ... * alpha_r channel-wise, P(r, r) = 1):
//   Gamma_r = P(r, -1), rho_s = P(C-1, s), gamma = Gamma_{C-1}
//   T[r, s] = beta_r sum_i k_ri k_si P_i(r, s)        (s < r)
//   A[r, s] = sum_i q_ri k_si P_i(r, s)               (s <= r)
//   [W | U~] = (I + T)^-1 diag(beta) [K * Gamma | V]
//   U = U~ - W S0;   O = (Q * Gamma) S0 + A U;   S_C = Diag(gamma) S0 + (K * rho)^T U
// Sources: "Semidirect Fourier Delta Attention" page, "El Teorema de
// Chunk-WY Constructivo" and "Principales Contribuciones" item 3 (affine
// block transfer); "Gated DeltaNet-2" page, Methodology section 3 (decay
// absorbed into the WY factors, triangular solve (I + T)^-1).
//
// Every gate product is a running product of alphas: no division, no
// logarithm, so zero and negative gates are exact and underflow goes to 0.
// Positions past the end of a sequence are identity transitions
// (alpha = 1, beta = 0, q = k = v = 0) and produce no output.
//
// Gated DeltaNet-2 ("Gated DeltaNet-2" page, Methodology section 1) replaces
// beta_r by an erase gate b_r in [0, 1]^d_k on the key side and a write gate
// w_r in [0, 1]^d_v on the value side.  The same derivation then gives, with
// E = B * K and Z = W_g * V (rows e_r = b_r * k_r, z_r = w_r * v_r):
//   T[r, s] = sum_i e_ri k_si P_i(r, s),   [W | U~] = (I + T)^-1 [E * Gamma | Z]
// and everything else unchanged; the G2 instantiation computes that form.
//
// SFDA ("Semidirect Fourier Delta Attention (SFDA)" page, "Arquitectura
// Central") replaces Diag(alpha_r) by the phase-decay gate Lambda_r, block
// diagonal with 2x2 blocks lambda_rp = alpha_rp (cos theta_rp, sin theta_rp)
// read as complex scalars acting on the channel pairs (2p, 2p+1).  Gate
// products stay products of those complex scalars (still division-free), and
// with P(r, s) = Lambda_r ... Lambda_{s+1}:
//   T[r, s] = beta_r k_r^T P(r, s) k_s,   A[r, s] = q_r^T P(r, s) k_s
//   W rows beta_r Gamma_r^T k_r, Q' rows Gamma_r^T q_r  (conjugate products)
//   K-hat rows P(C-1, s) k_s,   S_C = Gamma S0 + K-hat^T U  (Gamma on row pairs)
// which the SFDA instantiation computes.  Zero phases reproduce the CKDA
// instantiation bit for bit when the decays of a pair are equal.
//
// One CTA owns one (sequence, head, d_v slice of width BV) and walks its
// chunks in order; the slice of the state stays in shared memory in fp32.
#include <cooperative_groups.h>

#include "common.cuh"

namespace ckda {
namespace simt {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kMaxC = 64;

// Gate families of the kernel.
constexpr int kKda = 0;   // beta_r, Diag(alpha_r)
constexpr int kGdn2 = 1;  // erase gate b_r, write gate w_r, Diag(alpha_r)
constexpr int kSfda = 2;  // beta_r, phase-decay blocks alpha_rp e^{i theta_rp}

template <int DK, int BV>
struct Smem {
  static constexpr int KS = DK + 4;  // row stride of [C][DK] tiles (floats)
  static constexpr int VS = BV + 4;  // row stride of [C][BV] and [DK][BV] tiles
  static constexpr int CS = kMaxC + 4;
  static constexpr int kK = 0;
  static constexpr int kQ = kK + kMaxC * KS;
  static constexpr int kA = kQ + kMaxC * KS;
  static constexpr int kW = kA + kMaxC * KS;
  static constexpr int kV = kW + kMaxC * KS;
  static constexpr int kT = kV + kMaxC * VS;
  static constexpr int kAm = kT + kMaxC * CS;
  static constexpr int kS = kAm + kMaxC * CS;
  static constexpr int kBeta = kS + DK * VS;
  static constexpr int kGam = kBeta + kMaxC;
  static constexpr int kFloats = kGam + DK;
  static constexpr size_t kBytes = sizeof(float) * kFloats;
};

// Channels held by each lane while building the score blocks.
template <int DK>
struct LaneChannels {
  static constexpr int kPer = DK >= 32 ? DK / 32 : 1;
  static __device__ __forceinline__ bool active(int lane) { return lane * kPer < DK; }
};

template <int N>
__device__ __forceinline__ void lds(const float* p, float* x) {
  if constexpr (N == 4) {
    float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else if constexpr (N == 2) {
    float2 a = *reinterpret_cast<const float2*>(p);
    x[0] = a.x; x[1] = a.y;
  } else {
    x[0] = p[0];
  }
}

// Sum an 8-vector over the 32 lanes of a warp and leave the total of
// element e in every lane whose index satisfies (lane & 7) == e, in v[0].
__device__ __forceinline__ void reduce_scatter8(float* v, int lane) {
  {
    const bool up = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = up ? v[i] : v[i + 4];
      const float keep = up ? v[i + 4] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
  }
  {
    const bool up = lane & 2;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = up ? v[i] : v[i + 2];
      const float keep = up ? v[i + 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
  }
  {
    const bool up = lane & 1;
    const float send = up ? v[0] : v[1];
    const float keep = up ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 8);
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 16);
}

// (a + ib)(x + iy), real and imaginary parts; with b = 0 the results are
// exactly a x and a y.
__device__ __forceinline__ float cmul_re(float a, float b, float x, float y) {
  return fmaf(-b, y, a * x);
}
__device__ __forceinline__ float cmul_im(float a, float b, float x, float y) {
  return fmaf(b, x, a * y);
}

template <int DK, int BV, typename Tin, typename Tout, int GK>
__global__ void __launch_bounds__(kThreads, 1)
fwd_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                const float* __restrict__ alpha, const float* __restrict__ beta,
                const float* __restrict__ bg, const float* __restrict__ wg,
                const float* __restrict__ theta, const float* S0,
                const int32_t* __restrict__ cu, Tout* __restrict__ out, float* S_final,
                int n_seqs, int T, int H, int DV, int C, int* status) {
  constexpr bool G2 = GK == kGdn2;
  constexpr bool SF = GK == kSfda;
  using L = Smem<DK, BV>;
  constexpr int KS = L::KS, VS = L::VS, CS = L::CS;
  extern __shared__ __align__(16) float smem[];
  float* Ks = smem + L::kK;   // k, then K * rho
  float* Qs = smem + L::kQ;   // q, then Q * Gamma
  float* As = smem + L::kA;   // alpha (SFDA: lambda pairs, real then imaginary part)
  float* Ws = smem + L::kW;   // beta K Gamma, then W (G2: E = b * k, then E * Gamma, then W)
  float* Vs = smem + L::kV;   // v, then beta v (G2: w * v), then U~, then U
  float* Tm = smem + L::kT;   // T (strictly lower)
  float* Am = smem + L::kAm;  // A (lower incl. diagonal)
  float* Ss = smem + L::kS;   // state slice [DK][BV]
  float* bs = smem + L::kBeta;
  float* gs = smem + L::kGam;  // gamma (SFDA: complex pairs)

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int j0 = blockIdx.x * BV;
  const int h = blockIdx.y;
  const int n = seq_longest_first(cu, n_seqs, blockIdx.z);

  const SeqRange sr = seq_range(cu, n, n_seqs, T, status);
  if (!sr.ok) return;

  // The two d_v halves of one (sequence, head) run as a cluster of two CTAs
  // when C = 64 (see the launch): the S-independent score blocks T and A are
  // then split between them, each computing half of the columns and writing
  // them into both its own tiles and its partner's (distributed shared
  // memory).  Cluster barriers replace the block barriers at the start of a
  // chunk (neither CTA still reads the tiles the other is about to write)
  // and after the score blocks (both halves present in both CTAs).
  cg::cluster_group cluster = cg::this_cluster();
  const bool pair = cluster.num_blocks() == 2;
  const int prank = pair ? (int)cluster.block_rank() : 0;
  float* Tm_peer = pair ? cluster.map_shared_rank(Tm, prank ^ 1) : Tm;
  float* Am_peer = pair ? cluster.map_shared_rank(Am, prank ^ 1) : Am;
  auto chunk_sync = [&]() {
    if (pair)
      cluster.sync();
    else
      __syncthreads();
  };

  const size_t sbase = ((size_t)n * H + h) * DK * DV + j0;
  for (int e = tid; e < DK * BV / 4; e += kThreads) {
    const int i = e / (BV / 4), c4 = e % (BV / 4);
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (S0 != nullptr) val = *reinterpret_cast<const float4*>(S0 + sbase + (size_t)i * DV + 4 * c4);
    *reinterpret_cast<float4*>(Ss + i * VS + 4 * c4) = val;
  }

  for (int64_t t0 = sr.begin; t0 < sr.end; t0 += C) {
    const int Lc = (sr.end - t0 < (int64_t)C) ? (int)(sr.end - t0) : C;
    chunk_sync();  // previous chunk finished with every buffer (in both CTAs of a pair)

    // ---- stage inputs (fp32), identity transitions past the end ---------
    for (int e = tid; e < C * DK / 4; e += kThreads) {
      const int r = e / (DK / 4), c4 = e % (DK / 4);
      float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), qq = kk;
      float4 aa = SF ? make_float4(1.f, 0.f, 1.f, 0.f) : make_float4(1.f, 1.f, 1.f, 1.f);
      float4 ee = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < Lc) {
        const size_t off = ((size_t)(t0 + r) * H + h) * DK + 4 * c4;
        kk = load4_f32(k + off);
        qq = load4_f32(q + off);
        if constexpr (SF) {
          // channels 4 c4 .. 4 c4 + 3 are the pairs 2 c4 and 2 c4 + 1
          const size_t goff = ((size_t)(t0 + r) * H + h) * (DK / 2) + 2 * c4;
          const float2 a2 = *reinterpret_cast<const float2*>(alpha + goff);
          const float2 t2 = *reinterpret_cast<const float2*>(theta + goff);
          float s0, c0, s1, c1;
          sincosf(t2.x, &s0, &c0);
          sincosf(t2.y, &s1, &c1);
          aa = make_float4(a2.x * c0, a2.x * s0, a2.y * c1, a2.y * s1);
        } else {
          aa = *reinterpret_cast<const float4*>(alpha + off);
        }
        if constexpr (G2) {
          const float4 bb = *reinterpret_cast<const float4*>(bg + off);
          ee = make_float4(bb.x * kk.x, bb.y * kk.y, bb.z * kk.z, bb.w * kk.w);
        }
      }
      if constexpr (G2) *reinterpret_cast<float4*>(Ws + r * KS + 4 * c4) = ee;
      *reinterpret_cast<float4*>(Ks + r * KS + 4 * c4) = kk;
      *reinterpret_cast<float4*>(Qs + r * KS + 4 * c4) = qq;
      *reinterpret_cast<float4*>(As + r * KS + 4 * c4) = aa;
    }
    for (int e = tid; e < C * BV / 4; e += kThreads) {
      const int r = e / (BV / 4), c4 = e % (BV / 4);
      float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < Lc) {
        const size_t voff = ((size_t)(t0 + r) * H + h) * DV + j0 + 4 * c4;
        vv = load4_f32(v + voff);
        if constexpr (G2) {
          const float4 ww = *reinterpret_cast<const float4*>(wg + voff);
          vv = make_float4(ww.x * vv.x, ww.y * vv.y, ww.z * vv.z, ww.w * vv.w);
        }
      }
      *reinterpret_cast<float4*>(Vs + r * VS + 4 * c4) = vv;
    }
    if constexpr (!G2) {
      for (int r = tid; r < C; r += kThreads)
        bs[r] = (r < Lc) ? beta[(size_t)(t0 + r) * H + h] : 0.f;
    }
    __syncthreads();

    // ---- score blocks T and A: four columns per warp ------------------
    // For column s, x = k_s * P(r, s) is carried down the rows r > s by
    // multiplying with alpha_r; the dot products with k_r (G2: e_r) and q_r
    // give T[r, s] / beta_r (G2: T[r, s]) and A[r, s].  Lanes split the
    // channels; eight rows are reduced at once.  A warp takes the columns
    // s0, s0 + 8, s0 + 16, s0 + 24 together (s0 = warp, then warp + 32): their
    // rows run in the same blocks of eight, column m joining at block m, so
    // each row's alpha, k and q are read once for up to four independent
    // chains.
    {
      using LC = LaneChannels<DK>;
      constexpr int CPL = LC::kPer;
      const bool act = LC::active(lane);
      const int cb = lane * CPL;
      // x <- gate_r x on this lane's channels (SFDA: complex pairs)
      auto step = [&](float* x, const float* a) {
        if constexpr (SF) {
          if constexpr (CPL >= 2) {
#pragma unroll
            for (int c = 0; c < CPL; c += 2) {
              const float xr = x[c], xi = x[c + 1];
              x[c] = cmul_re(a[c], a[c + 1], xr, xi);
              x[c + 1] = cmul_im(a[c], a[c + 1], xr, xi);
            }
          } else {
            // one channel per lane: the pair partner is the neighbouring lane
            const float xo = __shfl_xor_sync(0xffffffffu, x[0], 1);
            const float lo = __shfl_xor_sync(0xffffffffu, a[0], 1);
            const bool odd = lane & 1;
            const float lre = odd ? lo : a[0], lim = odd ? a[0] : lo;
            x[0] = odd ? cmul_im(lre, lim, xo, x[0]) : cmul_re(lre, lim, x[0], xo);
          }
        } else {
#pragma unroll
          for (int c = 0; c < CPL; ++c) x[c] *= a[c];
        }
      };
      // a pair splits the sixteen column quads so that each CTA's warps take
      // one quad each with the same number of rows in total: quads s0 =
      // 2w + r (warps 0..3) and 32 + 2 (w - 4) + 1 - r (warps 4..7) in CTA r
      const int s_first = pair ? ((warp < 4) ? 2 * warp + prank : 32 + 2 * (warp - 4) + 1 - prank)
                               : warp;
      const int s_step = pair ? C : 32;
      // a score-block entry into this CTA's tiles and, in a pair, the partner's
      auto put = [&](int r, int s, float t, float a) {
        Tm[r * CS + s] = t;
        Am[r * CS + s] = a;
        if (pair) {
          Tm_peer[r * CS + s] = t;
          Am_peer[r * CS + s] = a;
        }
      };
      for (int s0 = s_first; s0 < C; s0 += s_step) {
        float x[4][CPL];
        // columns of this quad: diagonal of A, zeros above the diagonal
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int s = s0 + 8 * m;
          float qs[CPL];
#pragma unroll
          for (int c = 0; c < CPL; ++c) { x[m][c] = 0.f; qs[c] = 0.f; }
          if (s < C) {
            if (act) { lds<CPL>(Ks + s * KS + cb, x[m]); lds<CPL>(Qs + s * KS + cb, qs); }
            float d = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) d = fmaf(qs[c], x[m][c], d);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            if (lane == 0) put(s, s, 0.f, d);
            for (int r = lane; r < s; r += 32) put(r, s, 0.f, 0.f);
          }
        }
        for (int blk = 0; s0 + 1 + 8 * blk < C; ++blk) {
          const int rb = s0 + 1 + 8 * blk;
          float pk[4][8], pq[4][8];
#pragma unroll
          for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) { pk[m][jj] = 0.f; pq[m][jj] = 0.f; }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int r = rb + jj;
            if (r < C) {
              float a[CPL], kr[CPL], qr[CPL];
#pragma unroll
              for (int c = 0; c < CPL; ++c) { a[c] = 1.f; kr[c] = 0.f; qr[c] = 0.f; }
              if (act) {
                lds<CPL>(As + r * KS + cb, a);
                lds<CPL>((G2 ? Ws : Ks) + r * KS + cb, kr);
                lds<CPL>(Qs + r * KS + cb, qr);
              }
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                if (m <= blk) {
                  step(x[m], a);
#pragma unroll
                  for (int c = 0; c < CPL; ++c) {
                    pk[m][jj] = fmaf(kr[c], x[m][c], pk[m][jj]);
                    pq[m][jj] = fmaf(qr[c], x[m][c], pq[m][jj]);
                  }
                }
              }
            }
          }
          const int r = rb + (lane & 7);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            if (m <= blk) {
              reduce_scatter8(pk[m], lane);
              reduce_scatter8(pq[m], lane);
              const int s = s0 + 8 * m;
              if (lane < 8 && r < C) put(r, s, G2 ? pk[m][0] : bs[r] * pk[m][0], pq[m][0]);
            }
          }
        }
      }
    }
    chunk_sync();  // (a pair: both halves of T and A in both CTAs)

    // ---- gate products: one thread per channel ------------------------
    // forward: Gamma_r (inclusive prefix); W rhs = beta K Gamma (G2: E Gamma);
    // Q <- Q Gamma
    // backward: rho_s (exclusive suffix); K <- K rho
    if constexpr (SF) {
      // one thread per channel pair p: complex running products
      if (tid < DK / 2) {
        const int e = 2 * tid, o = e + 1;
        float gr = 1.f, gi = 0.f;
        for (int r = 0; r < C; ++r) {
          const float lr = As[r * KS + e], li = As[r * KS + o];
          const float nr = cmul_re(gr, gi, lr, li), ni = cmul_im(gr, gi, lr, li);
          gr = nr;
          gi = ni;
          // beta_r Gamma_r^T k_r and Gamma_r^T q_r: multiply by conj(gamma)
          const float ke = bs[r] * Ks[r * KS + e], ko = bs[r] * Ks[r * KS + o];
          Ws[r * KS + e] = cmul_re(gr, -gi, ke, ko);
          Ws[r * KS + o] = cmul_im(gr, -gi, ke, ko);
          const float qe = Qs[r * KS + e], qo = Qs[r * KS + o];
          Qs[r * KS + e] = cmul_re(gr, -gi, qe, qo);
          Qs[r * KS + o] = cmul_im(gr, -gi, qe, qo);
        }
        gs[e] = gr;
        gs[o] = gi;
        float pr = 1.f, pi = 0.f;
        for (int s = C - 1; s >= 0; --s) {
          const float ke = Ks[s * KS + e], ko = Ks[s * KS + o];
          Ks[s * KS + e] = cmul_re(pr, pi, ke, ko);
          Ks[s * KS + o] = cmul_im(pr, pi, ke, ko);
          const float lr = As[s * KS + e], li = As[s * KS + o];
          const float nr = cmul_re(pr, pi, lr, li), ni = cmul_im(pr, pi, lr, li);
          pr = nr;
          pi = ni;
        }
      }
    } else if (tid < DK) {
      const int i = tid;
      float gmm = 1.f;
      for (int r = 0; r < C; ++r) {
        gmm *= As[r * KS + i];
        if constexpr (G2)
          Ws[r * KS + i] *= gmm;
        else
          Ws[r * KS + i] = bs[r] * Ks[r * KS + i] * gmm;
        Qs[r * KS + i] *= gmm;
      }
      gs[i] = gmm;
      float p = 1.f;
      for (int s = C - 1; s >= 0; --s) {
        Ks[s * KS + i] *= p;
        p *= As[s * KS + i];
      }
    }
    if constexpr (!G2) {
      for (int e = tid; e < C * BV; e += kThreads) {
        const int r = e / BV, c = e % BV;
        Vs[r * VS + c] *= bs[r];
      }
    }
    __syncthreads();

    // ---- WY factors: [W | U~] = (I + T)^-1 [beta K Gamma | beta V] -----
    // (G2: (I + T)^-1 [E Gamma | Z])
    // Forward substitution, one thread per column, 16 rows at a time in
    // registers: rows of earlier blocks are final when a block starts.
    if (tid < DK + BV) {
      float* X = (tid < DK) ? (Ws + tid) : (Vs + (tid - DK));
      const int xs = (tid < DK) ? KS : VS;
      for (int rb = 0; rb < C; rb += 16) {
        float acc[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) acc[m] = X[(rb + m) * xs];
        for (int s = 0; s < rb; ++s) {
          const float xv = X[s * xs];
#pragma unroll
          for (int m = 0; m < 16; ++m) acc[m] = fmaf(-Tm[(rb + m) * CS + s], xv, acc[m]);
        }
#pragma unroll
        for (int m = 1; m < 16; ++m) {
#pragma unroll
          for (int m2 = 0; m2 < m; ++m2) acc[m] = fmaf(-Tm[(rb + m) * CS + rb + m2], acc[m2], acc[m]);
        }
#pragma unroll
        for (int m = 0; m < 16; ++m) X[(rb + m) * xs] = acc[m];
      }
    }
    __syncthreads();

    // ---- state carry ----------------------------------------------------
    // (a) U = U~ - W S  (C x BV), 4x4 register tiles
    const int ntile = (C / 4) * (BV / 4);
    const int tr = tid / (BV / 4), tc = tid % (BV / 4);
    const int r0 = tr * 4, c0 = tc * 4;
    if (tid < ntile) {
      float4 acc[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = *reinterpret_cast<const float4*>(Vs + (r0 + m) * VS + c0);
#pragma unroll 4
      for (int i = 0; i < DK; ++i) {
        const float4 s4 = *reinterpret_cast<const float4*>(Ss + i * VS + c0);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float w = Ws[(r0 + m) * KS + i];
          acc[m].x = fmaf(-w, s4.x, acc[m].x); acc[m].y = fmaf(-w, s4.y, acc[m].y);
          acc[m].z = fmaf(-w, s4.z, acc[m].z); acc[m].w = fmaf(-w, s4.w, acc[m].w);
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) *reinterpret_cast<float4*>(Vs + (r0 + m) * VS + c0) = acc[m];
    }
    __syncthreads();

    // (b) O = (Q Gamma) S + A U  -> out rows of real tokens
    if (tid < ntile) {
      float4 acc[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int i = 0; i < DK; ++i) {
        const float4 s4 = *reinterpret_cast<const float4*>(Ss + i * VS + c0);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float w = Qs[(r0 + m) * KS + i];
          acc[m].x = fmaf(w, s4.x, acc[m].x); acc[m].y = fmaf(w, s4.y, acc[m].y);
          acc[m].z = fmaf(w, s4.z, acc[m].z); acc[m].w = fmaf(w, s4.w, acc[m].w);
        }
      }
      const int smax = min(C, r0 + 4);  // A is lower triangular
      for (int s = 0; s < smax; ++s) {
        const float4 u4 = *reinterpret_cast<const float4*>(Vs + s * VS + c0);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float w = Am[(r0 + m) * CS + s];
          acc[m].x = fmaf(w, u4.x, acc[m].x); acc[m].y = fmaf(w, u4.y, acc[m].y);
          acc[m].z = fmaf(w, u4.z, acc[m].z); acc[m].w = fmaf(w, u4.w, acc[m].w);
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = r0 + m;
        if (r < Lc) store4(out + ((size_t)(t0 + r) * H + h) * DV + j0 + c0, acc[m]);
      }
    }
    __syncthreads();

    // (c) S <- Diag(gamma) S + (K rho)^T U   (DK x BV)
    for (int tile = tid; tile < (DK / 4) * (BV / 4); tile += kThreads) {
      const int i0 = (tile / (BV / 4)) * 4, cc = (tile % (BV / 4)) * 4;
      float4 acc[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < C; ++s) {
        const float4 kh = *reinterpret_cast<const float4*>(Ks + s * KS + i0);
        const float4 u4 = *reinterpret_cast<const float4*>(Vs + s * VS + cc);
        const float khv[4] = {kh.x, kh.y, kh.z, kh.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          acc[m].x = fmaf(khv[m], u4.x, acc[m].x); acc[m].y = fmaf(khv[m], u4.y, acc[m].y);
          acc[m].z = fmaf(khv[m], u4.z, acc[m].z); acc[m].w = fmaf(khv[m], u4.w, acc[m].w);
        }
      }
      if constexpr (SF) {
        // rows (i0, i0 + 1) and (i0 + 2, i0 + 3) are channel pairs
#pragma unroll
        for (int m = 0; m < 4; m += 2) {
          float4* pe = reinterpret_cast<float4*>(Ss + (i0 + m) * VS + cc);
          float4* po = reinterpret_cast<float4*>(Ss + (i0 + m + 1) * VS + cc);
          const float4 se = *pe, so = *po;
          const float gr = gs[i0 + m], gi = gs[i0 + m + 1];
          const float4 ae = acc[m], ao = acc[m + 1];
          *pe = make_float4(fmaf(gr, se.x, fmaf(-gi, so.x, ae.x)), fmaf(gr, se.y, fmaf(-gi, so.y, ae.y)),
                            fmaf(gr, se.z, fmaf(-gi, so.z, ae.z)), fmaf(gr, se.w, fmaf(-gi, so.w, ae.w)));
          *po = make_float4(fmaf(gr, so.x, fmaf(gi, se.x, ao.x)), fmaf(gr, so.y, fmaf(gi, se.y, ao.y)),
                            fmaf(gr, so.z, fmaf(gi, se.z, ao.z)), fmaf(gr, so.w, fmaf(gi, se.w, ao.w)));
        }
      } else {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float4* sp = reinterpret_cast<float4*>(Ss + (i0 + m) * VS + cc);
          float4 sv = *sp;
          const float g = gs[i0 + m];
          sv.x = fmaf(g, sv.x, acc[m].x); sv.y = fmaf(g, sv.y, acc[m].y);
          sv.z = fmaf(g, sv.z, acc[m].z); sv.w = fmaf(g, sv.w, acc[m].w);
          *sp = sv;
        }
      }
    }
  }
  __syncthreads();
  if (S_final != nullptr) {
    for (int e = tid; e < DK * BV / 4; e += kThreads) {
      const int i = e / (BV / 4), c4 = e % (BV / 4);
      *reinterpret_cast<float4*>(S_final + sbase + (size_t)i * DV + 4 * c4) =
          *reinterpret_cast<const float4*>(Ss + i * VS + 4 * c4);
    }
  }
}

// Gates of a call: beta (CKDA), the erase and write gates (Gated DeltaNet-2)
// or beta with the phases (SFDA).
struct Gates {
  const float* beta;
  const float* b;
  const float* w;
  const float* theta;
};

template <int DK, int BV, typename Tin, typename Tout, int GK>
static cudaError_t launch_t(const void* q, const void* k, const void* v, const float* alpha,
                            Gates gt, const float* S0, const int32_t* cu, void* out,
                            float* S_final, int n_seqs, int T, int H, int DV, int C, int* status,
                            cudaStream_t stream) {
  using L = Smem<DK, BV>;
  auto kern = fwd_simt_kernel<DK, BV, Tin, Tout, GK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::kBytes);
  if (e != cudaSuccess) return e;
  // two d_v slices at C = 64: a cluster of the pair, which splits the score
  // blocks (see the kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(DV / BV, H, n_seqs);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (DV / BV == 2 && C == kMaxC) ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = attr[0].val.clusterDim.x > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const Tin*>(q), static_cast<const Tin*>(k),
                            static_cast<const Tin*>(v), alpha, gt.beta, gt.b, gt.w, gt.theta, S0,
                            cu, static_cast<Tout*>(out), S_final, n_seqs, T, H, DV, C, status);
}

template <int DK, typename Tin, typename Tout, int GK>
static cudaError_t launch_bv(const void* q, const void* k, const void* v, const float* alpha,
                             Gates gt, const float* S0, const int32_t* cu, void* out,
                             float* S_final, int n_seqs, int T, int H, int DV, int C, int* status,
                             cudaStream_t stream) {
  switch (DV) {
    case 16:
      return launch_t<DK, 16, Tin, Tout, GK>(q, k, v, alpha, gt, S0, cu, out, S_final, n_seqs, T, H,
                                             DV, C, status, stream);
    case 32:
      return launch_t<DK, 32, Tin, Tout, GK>(q, k, v, alpha, gt, S0, cu, out, S_final, n_seqs, T, H,
                                             DV, C, status, stream);
    default:  // 64 and 128: slices of 64 columns
      return launch_t<DK, 64, Tin, Tout, GK>(q, k, v, alpha, gt, S0, cu, out, S_final, n_seqs, T, H,
                                             DV, C, status, stream);
  }
}

}  // namespace simt

// `bg` and `wg` non-NULL select the Gated DeltaNet-2 form (beta unused);
// `theta` non-NULL selects the SFDA form (alpha then holds dk / 2 decays).
cudaError_t launch_fwd_simt(int dtype, int out_dtype, int dk, int dv, const void* q,
                            const void* k, const void* v, const float* alpha, const float* beta,
                            const float* bg, const float* wg, const float* theta,
                            const float* S0, const int32_t* cu, void* out, float* S_final,
                            int n_seqs, int T, int H, int C, int* status, cudaStream_t stream) {
  const simt::Gates gt{beta, bg, wg, theta};
  const int gk = theta != nullptr ? simt::kSfda : (bg != nullptr ? simt::kGdn2 : simt::kKda);
#define CKDA_SIMT_GK(DKV, TI, TO, GKV) \
  simt::launch_bv<DKV, TI, TO, GKV>(q, k, v, alpha, gt, S0, cu, out, S_final, n_seqs, T, H, dv, C, \
                                    status, stream)
#define CKDA_SIMT_CALL(DKV, TI, TO)                                     \
  (gk == simt::kSfda   ? CKDA_SIMT_GK(DKV, TI, TO, simt::kSfda)          \
   : gk == simt::kGdn2 ? CKDA_SIMT_GK(DKV, TI, TO, simt::kGdn2)          \
                       : CKDA_SIMT_GK(DKV, TI, TO, simt::kKda))
#define CKDA_SIMT_DK(DKV)                                                                  \
  case DKV:                                                                                \
    if (dtype == CKDA_BF16)                                                                \
      return out_dtype == CKDA_BF16 ? CKDA_SIMT_CALL(DKV, __nv_bfloat16, __nv_bfloat16)    \
                                    : CKDA_SIMT_CALL(DKV, __nv_bfloat16, float);           \
    return out_dtype == CKDA_BF16 ? CKDA_SIMT_CALL(DKV, float, __nv_bfloat16)              \
                                  : CKDA_SIMT_CALL(DKV, float, float);
  switch (dk) {
    CKDA_SIMT_DK(16)
    CKDA_SIMT_DK(32)
    CKDA_SIMT_DK(64)
    CKDA_SIMT_DK(128)
  }
#undef CKDA_SIMT_DK
#undef CKDA_SIMT_CALL
#undef CKDA_SIMT_GK
  return cudaErrorInvalidValue;
}

}  // namespace ckda
