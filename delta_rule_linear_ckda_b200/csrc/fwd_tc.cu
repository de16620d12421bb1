// Tensor-core (tcgen05) chunked WY forward of CKDA for bf16 inputs,
// d_k = 128, d_v in {64, 128}, chunk C = 64 (sm_100a).
//
// Chunk algebra (positions r, s = 0..C-1 of one chunk, start state S0,
// P(r, s) = alpha_{s+1} * ... * alpha_r channel-wise):
//   T[r, s] = beta_r sum_i k_ri k_si P_i(r, s)  (s < r),   A[r, s] = sum_i q_ri k_si P_i(r, s)  (s <= r)
//   Inv = (I + T)^-1,   W = Inv diag(beta) (K * Gamma),   U~ = Inv diag(beta) V
//   U = U~ - W S0,   O = (Q * Gamma) S0 + A U,   S_C = Diag(gamma) S0 + (K * rho)^T U
// ("Semidirect Fourier Delta Attention" page: "El Teorema de Chunk-WY
// Constructivo" and the exact affine block transfer of "Principales
// Contribuciones" item 3; "Gated DeltaNet-2" page, Methodology section 3:
// decay absorbed into the WY factors and the triangular solve (I + T)^-1.)
//
// The form used here groups the S0-independent work so that the carry is
// two dependent tensor-core products per chunk:
//   P  = A Inv diag(beta)
//   [W, U~; A W, A U~] = [Inv diag(beta); P] [K * Gamma, V]      (one M=128 MMA)
//   Q' = Q * Gamma - A W
//   X  = [W; Q'] S0                                             (carry MMA 1)
//   U  = U~ - X_top,   O = A U~ + X_bottom
//   D  = (K * rho)^T U,  S_C = Diag(gamma) S0 + D               (carry MMA 2)
//
// Division-free score blocks: every pair s < r is split at the anchor m of
// the highest bit in which r and s differ ("level" h, block size b = 2^h):
// P(r, s) = [alpha_m ... alpha_r] * [alpha_{s+1} ... alpha_{m-1}], two
// running products that restart at the anchor.  Each level is one GEMM of
// the anchored operands, so zero and negative gates are exact and underflow
// goes to zero; no logarithm or division is taken.
//
// One CTA (256 threads) owns one (sequence, head, 64-column d_v slice) and
// walks its chunks in order.  Inputs arrive by TMA; operands are fp16 tiles
// in 128-byte-swizzled shared memory; accumulators live in tensor memory;
// the state slice stays in fp32 registers (row i = tensor-memory lane i).
// Every mbarrier wait is bounded: on time-out the kernel records
// CKDA_ERR_DEVICE_TIMEOUT, waits once more (bounded) for its own copies,
// frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace ckda {
namespace tc {

using namespace sm100;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int BV = 64;
constexpr int NT = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

// ---- shared memory map (byte offsets from a 1024-aligned base) ----------
// region X: TMA tiles of q, k (bf16 [64][128]) and alpha (fp32 [64][128]);
// reused for the fp32 inverse workspace and the A / Inv / P operand tiles,
// then for the [W; Q'] operand tile.
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = 16384;
constexpr uint32_t OFF_A = 32768;
constexpr uint32_t OFF_TF = 0;       // T, fp32 [64][64]
constexpr uint32_t OFF_INV = 16384;  // (I + T)^-1, fp32 [64][64]
constexpr uint32_t OFF_AQ = 32768;   // A, fp16 K-major [64 r][64 s]
constexpr uint32_t OFF_IP = 40960;   // [Inv diag(beta); P], fp16 K-major [128][64]
constexpr uint32_t OFF_YF = 57344;   // inverse scratch, fp32 [16][48]
constexpr uint32_t OFF_WQ = 0;       // [W; Q'], fp16 K-major [128][128]
// region Y: score operands of two levels, then K * Gamma and Q * Gamma.
constexpr uint32_t OFF_LOP0 = 65536;  // [beta K L; Q L], fp16 K-major [64][128]
constexpr uint32_t OFF_LOP1 = 81920;
constexpr uint32_t OFF_ROP0 = 98304;  // K R, fp16 K-major [32][128]
constexpr uint32_t OFF_ROP1 = 106496;
constexpr uint32_t OFF_KG = 65536;   // K * Gamma, fp16 MN-major [64 s][128 i]
constexpr uint32_t OFF_QG = 81920;   // Q * Gamma, fp16 row-major [64][QG_STRIDE]
constexpr int QG_STRIDE = 136;
// dedicated tiles
constexpr uint32_t OFF_KH = 114688;  // K * rho, fp16 MN-major [64 s][128 i]
constexpr uint32_t OFF_V = 131072;   // v slice (TMA, 128B swizzle), bf16 -> fp16 [64 s][64 j]
constexpr uint32_t OFF_SB = 139264;  // state slice, fp16 MN-major [128 i][64 j]
constexpr uint32_t OFF_UB = 155648;  // U, fp16 MN-major [64 s][64 j]
constexpr uint32_t OFF_BETA = 163840;
constexpr uint32_t OFF_GAMMA = 164096;
constexpr uint32_t OFF_ADIAG = 164608;
constexpr uint32_t OFF_BAR = 164864;  // mbarriers: tma, mma, level0, level1
constexpr uint32_t OFF_TMEMPTR = 164896;
constexpr uint32_t kSmemUsed = 164912;
constexpr size_t kSmemBytes = kSmemUsed + 1024;

constexpr uint32_t kTmaBytes = 16384 + 16384 + 32768 + 8192;

// ---- tensor memory columns ------------------------------------------------
constexpr uint32_t TM_SCORE = 0;  // 6 levels x 32 columns (M = 64 layout)
constexpr uint32_t TM_P = 192;    // P (M = 64 layout)
constexpr uint32_t TM_W = 256;    // [W; A W]       (M = 128, 128 columns)
constexpr uint32_t TM_U = 384;    // [U~; A U~]     (M = 128, 64 columns)
constexpr uint32_t TM_X = 448;    // [W S; Q' S]    (M = 128, 64 columns)
constexpr uint32_t TM_D = 0;      // (K rho)^T U    (M = 128, 64 columns)

__device__ __forceinline__ float bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

#ifdef CKDA_TC_DEBUG
// Intermediate dump of the first chunk of CTA (0, 0, 0) (diagnostic builds only).
__device__ float* g_tc_dbg = nullptr;
#define TC_DBG(stmt)                                                                   \
  do {                                                                                 \
    if (g_tc_dbg != nullptr && c == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&         \
        blockIdx.z == 0) {                                                             \
      stmt;                                                                            \
    }                                                                                  \
  } while (0)
#else
#define TC_DBG(stmt) \
  do {               \
  } while (0)
#endif

// Tensor-core operands are fp16: the bf16 inputs convert to it exactly
// (apart from subnormals), and its 10-bit mantissa keeps the rounding of the
// intermediate operands (products of gates, the WY factors, the state) at
// 2^-11 relative instead of bf16's 2^-9.  The values involved are bounded
// (|k|, |q| <= 1 per element after normalisation, |gate products| <= 1), far
// inside fp16's range.
__device__ __forceinline__ void st_h(uint8_t* base, uint32_t off, float x) {
  *reinterpret_cast<__half*>(base + off) = __float2half_rn(x);
}

__device__ __forceinline__ void st_chunk8(uint8_t* base, uint32_t off, const float* v) {
  uint4 pk;
  pk.x = pack_f16x2(v[0], v[1]);
  pk.y = pack_f16x2(v[2], v[3]);
  pk.z = pack_f16x2(v[4], v[5]);
  pk.w = pack_f16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(base + off) = pk;
}

__device__ __forceinline__ uint32_t taddr(uint32_t tmem, int lane_base, uint32_t col) {
  return tmem + ((uint32_t)lane_base << 16) + col;
}

template <typename Tout>
__device__ __forceinline__ void store_row32(Tout* dst, const float* a, const float* x);

template <>
__device__ __forceinline__ void store_row32<float>(float* dst, const float* a, const float* x) {
#pragma unroll
  for (int e = 0; e < 32; e += 4)
    *reinterpret_cast<float4*>(dst + e) = make_float4(a[e] + x[e], a[e + 1] + x[e + 1],
                                                      a[e + 2] + x[e + 2], a[e + 3] + x[e + 3]);
}

template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16* dst, const float* a,
                                                           const float* x) {
#pragma unroll
  for (int e = 0; e < 32; e += 8) {
    uint4 pk;
    pk.x = pack_bf16x2(a[e] + x[e], a[e + 1] + x[e + 1]);
    pk.y = pack_bf16x2(a[e + 2] + x[e + 2], a[e + 3] + x[e + 3]);
    pk.z = pack_bf16x2(a[e + 4] + x[e + 4], a[e + 5] + x[e + 5]);
    pk.w = pack_bf16x2(a[e + 6] + x[e + 6], a[e + 7] + x[e + 7]);
    *reinterpret_cast<uint4*>(dst + e) = pk;
  }
}

template <typename Tout>
__global__ void __launch_bounds__(NT, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
              const float* __restrict__ beta, const float* S0, const int32_t* __restrict__ cu,
              Tout* __restrict__ out, float* S_final, int n_seqs, int T, int H, int DV,
              int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int j0 = blockIdx.x * BV;
  const int h = blockIdx.y;
  const int n = blockIdx.z;

  const SeqRange sr = seq_range(cu, n, n_seqs, T, status);
  if (!sr.ok) return;

  float* beta_s = reinterpret_cast<float*>(sm + OFF_BETA);
  float* gamma_s = reinterpret_cast<float*>(sm + OFF_GAMMA);
  float* adiag_s = reinterpret_cast<float*>(sm + OFF_ADIAG);
  const uint32_t bar_tma = sb + OFF_BAR;
  const uint32_t bar_mma = sb + OFF_BAR + 8;
  const uint32_t bar_lv0 = sb + OFF_BAR + 16;
  const uint32_t bar_lv1 = sb + OFF_BAR + 24;

  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_lv0, 1);
    mbar_init(bar_lv1, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_a);
  }
  if (warp == 0) {
    tmem_alloc(sb + OFF_TMEMPTR, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_TMEMPTR);

  // State slice: row i = 32 * (warp % 4) + lane, columns [32 * (warp / 4), +32).
  const int q4 = warp & 3;
  const int half = warp >> 2;
  const int srow = 32 * q4 + lane;
  const size_t s_off = (((size_t)n * H + h) * DK + srow) * DV + j0 + 32 * half;
  float S[32];
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (S0 != nullptr) v4 = *reinterpret_cast<const float4*>(S0 + s_off + e);
    S[e] = v4.x; S[e + 1] = v4.y; S[e + 2] = v4.z; S[e + 3] = v4.w;
  }
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) st_chunk8(sm + OFF_SB, sw128_chunk(srow, 32 * half + 8 * c4, 128), S + 8 * c4);

  const int64_t tok0 = sr.begin;
  const int64_t tok1 = sr.end;
  const int nchunks = (int)((tok1 - tok0 + C - 1) / C);
  uint32_t ph_tma = 0, ph_mma = 0, ph_lv0 = 0, ph_lv1 = 0;
  bool tma_pending = false;
  int ok = 1;

  auto issue_tma = [&](int64_t t0) {
    mbar_expect_tx(bar_tma, kTmaBytes);
    tma_load_2d(sb + OFF_Q, &tm_q, h * DK, (int)t0, bar_tma);
    tma_load_2d(sb + OFF_K, &tm_k, h * DK, (int)t0, bar_tma);
    tma_load_2d(sb + OFF_A, &tm_a, h * DK, (int)t0, bar_tma);
    tma_load_2d(sb + OFF_V, &tm_v, h * DV + j0, (int)t0, bar_tma);
  };
  if (nchunks > 0) {
    if (tid == 0) issue_tma(tok0);
    tma_pending = true;
  }

  const int ich = tid & 127;
  const bool upper = tid >= 128;
  const __nv_bfloat16* Qs = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_Q);
  const __nv_bfloat16* Ks = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_K);
  const float* As = reinterpret_cast<const float*>(sm + OFF_A);

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = tok0 + (int64_t)c * C;
    const int Lc = (tok1 - t0 < (int64_t)C) ? (int)(tok1 - t0) : C;
    if (tid < C) beta_s[tid] = (tid < Lc) ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
    ok = mbar_wait_bounded(bar_tma, ph_tma, kWaitNs);
    ph_tma ^= 1;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tma_pending = false;

    // ---- score blocks, one hierarchy level at a time ----------------------
    for (int lv = 0; lv < 6; ++lv) {
      const int b = 1 << lv;
      const int buf = lv & 1;
      if (lv >= 2) {
        if (buf) {
          ok = mbar_wait_bounded(bar_lv1, ph_lv1, kWaitNs);
          ph_lv1 ^= 1;
        } else {
          ok = mbar_wait_bounded(bar_lv0, ph_lv0, kWaitNs);
          ph_lv0 ^= 1;
        }
        ok = __syncthreads_and(ok);
        if (!ok) break;
      }
      uint8_t* LOP = sm + (buf ? OFF_LOP1 : OFF_LOP0);
      uint8_t* ROP = sm + (buf ? OFF_ROP1 : OFF_ROP0);
      const int nseg = C / (2 * b);
      if (upper) {
        // right halves: L_r = alpha_m ... alpha_r; rows rho of [beta K L] and [Q L]
        for (int j = 0; j < nseg; ++j) {
          const int m = 2 * b * j + b;
          float p = 1.f;
          for (int u = 0; u < b; ++u) {
            const int r = m + u;
            const bool val = r < Lc;
            p *= val ? As[r * DK + ich] : 1.f;
            const float kv = val ? bf(Ks + r * DK + ich) : 0.f;
            const float qv = val ? bf(Qs + r * DK + ich) : 0.f;
            const int rho = j * b + u;
            st_h(LOP, sw128_elem(rho, ich, 64), beta_s[r] * kv * p);
            st_h(LOP, sw128_elem(32 + rho, ich, 64), qv * p);
          }
        }
      } else {
        // left halves: R_s = alpha_{s+1} ... alpha_{m-1}; rows sigma of [K R]
        for (int j = 0; j < nseg; ++j) {
          const int m = 2 * b * j + b;
          float p = 1.f;
          for (int u = b - 1; u >= 0; --u) {
            const int s = m - b + u;
            const bool val = s < Lc;
            const float kv = val ? bf(Ks + s * DK + ich) : 0.f;
            st_h(ROP, sw128_elem(j * b + u, ich, 32), kv * p);
            p *= val ? As[s * DK + ich] : 1.f;
          }
        }
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t la = sb + (buf ? OFF_LOP1 : OFF_LOP0);
        const uint32_t ra = sb + (buf ? OFF_ROP1 : OFF_ROP0);
        constexpr uint32_t id = idesc_f16(64, 32, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = smem_desc(la + (kk >> 2) * (64 * 128) + (kk & 3) * 32, 16, 1024, kSwizzle128);
          const uint64_t bd = smem_desc(ra + (kk >> 2) * (32 * 128) + (kk & 3) * 32, 16, 1024, kSwizzle128);
          mma_f16(tmem + TM_SCORE + 32 * lv, ad, bd, id, kk > 0 ? 1u : 0u);
        }
        mma_commit(buf ? bar_lv1 : bar_lv0);
      }
    }
    if (!ok) break;
    ok = mbar_wait_bounded(bar_lv0, ph_lv0, kWaitNs);
    ph_lv0 ^= 1;
    ok = mbar_wait_bounded(bar_lv1, ph_lv1, kWaitNs) && ok;
    ph_lv1 ^= 1;
    ok = __syncthreads_and(ok);
    if (!ok) break;

    // ---- Gamma (prefix), rho (suffix), gamma, diag(A), identity padding ----
    {
      uint8_t* KG = sm + OFF_KG;
      __half* QG = reinterpret_cast<__half*>(sm + OFF_QG);
      uint8_t* KH = sm + OFF_KH;
      if (!upper) {
        float g = 1.f;
        for (int r = 0; r < C; ++r) {
          const bool val = r < Lc;
          g *= val ? As[r * DK + ich] : 1.f;
          const float kv = val ? bf(Ks + r * DK + ich) : 0.f;
          const float qv = val ? bf(Qs + r * DK + ich) : 0.f;
          st_h(KG, sw128_elem(r, ich, 64), kv * g);
          QG[r * QG_STRIDE + ich] = __float2half_rn(qv * g);
        }
        gamma_s[ich] = g;
      } else {
        float p = 1.f;
        for (int s = C - 1; s >= 0; --s) {
          const bool val = s < Lc;
          const float kv = val ? bf(Ks + s * DK + ich) : 0.f;
          st_h(KH, sw128_elem(s, ich, 64), kv * p);
          p *= val ? As[s * DK + ich] : 1.f;
        }
      }
      for (int rr = 0; rr < 8; ++rr) {
        const int r = 8 * warp + rr;
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc = fmaf(bf(Qs + r * DK + 4 * lane + e), bf(Ks + r * DK + 4 * lane + e), acc);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) adiag_s[r] = (r < Lc) ? acc : 0.f;
      }
      // v tile: bf16 (as loaded) -> fp16 in place; rows past the end -> 0.
      // Each 16-byte chunk stays within its 128-byte row under the swizzle.
      {
        uint4* vt = reinterpret_cast<uint4*>(sm + OFF_V);
        for (int e = tid; e < C * 8; e += NT) {
          uint4 raw = vt[e];
          if ((e >> 3) < Lc) {
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
            float f[8];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 x2 = __bfloat1622float2(p2[t]);
              f[2 * t] = x2.x;
              f[2 * t + 1] = x2.y;
            }
            raw.x = pack_f16x2(f[0], f[1]);
            raw.y = pack_f16x2(f[2], f[3]);
            raw.z = pack_f16x2(f[4], f[5]);
            raw.w = pack_f16x2(f[6], f[7]);
          } else {
            raw = make_uint4(0u, 0u, 0u, 0u);
          }
          vt[e] = raw;
        }
      }
    }
    __syncthreads();

    // ---- gather T (fp32) and A (fp16) from the level accumulators ---------
    {
      uint4* z = reinterpret_cast<uint4*>(sm + OFF_TF);
      for (int e = tid; e < (int)(40960 / 16); e += NT) z[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    tc_fence_after();
    {
      float* Tf = reinterpret_cast<float*>(sm + OFF_TF);
      uint8_t* AQ = sm + OFF_AQ;
      if (warp < 4) {
        const int rho = 16 * warp + lane;
        const int rr = rho & 31;
        for (int lv = 0; lv < 6; ++lv) {
          float v[32];
          tmem_ld32(taddr(tmem, 32 * warp, TM_SCORE + 32 * lv), v);
          tmem_ld_wait();
          if (lane < 16) {
            const int b = 1 << lv;
            const int j = rr >> lv;
            const int r = 2 * b * j + b + (rr & (b - 1));
#pragma unroll
            for (int sg = 0; sg < 32; ++sg) {
              if ((sg >> lv) == j) {
                const int s = 2 * b * j + (sg & (b - 1));
                if (rho < 32)
                  Tf[r * 64 + s] = v[sg];
                else
                  st_h(AQ, sw128_elem(r, s, 64), v[sg]);
              }
            }
          }
        }
      }
      if (tid < C) st_h(AQ, sw128_elem(tid, tid, 64), adiag_s[tid]);
    }
    tc_fence_before();
    __syncthreads();
    TC_DBG(for (int e = tid; e < 4096; e += NT) {
      g_tc_dbg[e] = reinterpret_cast<const float*>(sm + OFF_TF)[e];
      g_tc_dbg[4096 + e] = __half2float(*reinterpret_cast<const __half*>(sm + OFF_AQ + sw128_elem(e >> 6, e & 63, 64)));
    });

    // ---- (I + T)^-1 in fp32, 16 x 16 blocks ---------------------------------
    {
      const float* Tf = reinterpret_cast<const float*>(sm + OFF_TF);
      float* Inv = reinterpret_cast<float*>(sm + OFF_INV);
      float* Yf = reinterpret_cast<float*>(sm + OFF_YF);
      if (tid < 64) {
        const int base = 16 * (tid >> 4);
        const int cc = tid & 15;
        float x[16];
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2) {
          float acc = (r2 == cc) ? 1.f : 0.f;
#pragma unroll
          for (int s2 = 0; s2 < r2; ++s2) acc = fmaf(-Tf[(base + r2) * 64 + base + s2], x[s2], acc);
          x[r2] = (r2 < cc) ? 0.f : acc;
        }
#pragma unroll
        for (int r2 = 0; r2 < 16; ++r2) Inv[(base + r2) * 64 + base + cc] = x[r2];
      }
      __syncthreads();
      for (int I = 1; I < 4; ++I) {
        for (int e = tid; e < 256 * I; e += NT) {
          const int J = e >> 8, r2 = (e >> 4) & 15, cc = e & 15;
          float acc = 0.f;
          for (int K = J; K < I; ++K) {
#pragma unroll
            for (int kk = 0; kk < 16; ++kk)
              acc = fmaf(Tf[(16 * I + r2) * 64 + 16 * K + kk], Inv[(16 * K + kk) * 64 + 16 * J + cc], acc);
          }
          Yf[r2 * 48 + 16 * J + cc] = acc;
        }
        __syncthreads();
        for (int e = tid; e < 256 * I; e += NT) {
          const int J = e >> 8, r2 = (e >> 4) & 15, cc = e & 15;
          float acc = 0.f;
#pragma unroll
          for (int kk = 0; kk < 16; ++kk)
            acc = fmaf(Inv[(16 * I + r2) * 64 + 16 * I + kk], Yf[kk * 48 + 16 * J + cc], acc);
          Inv[(16 * I + r2) * 64 + 16 * J + cc] = -acc;
        }
        __syncthreads();
      }
      TC_DBG(for (int e = tid; e < 4096; e += NT) g_tc_dbg[8192 + e] = Inv[e]);
      // Inv diag(beta) -> rows 0..63 of the stacked operand
      uint8_t* IP = sm + OFF_IP;
      for (int e = tid; e < 64 * 8; e += NT) {
        const int r = e >> 3, cg = e & 7;
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = Inv[r * 64 + 8 * cg + t] * beta_s[8 * cg + t];
        st_chunk8(IP, sw128_chunk(r, 8 * cg, 128), v);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- P = A Inv diag(beta) ---------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(64, 64, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc(sb + OFF_AQ + kk * 32, 16, 1024, kSwizzle128);
        const uint64_t bd = smem_desc(sb + OFF_IP + kk * 2048, 8192, 1024, kSwizzle128);
        mma_f16(tmem + TM_P, ad, bd, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
    ph_mma ^= 1;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    {
      float v[32];
      tmem_ld32(taddr(tmem, 32 * q4, TM_P + 32 * half), v);
      tmem_ld_wait();
      if (lane < 16) {
        const int rho = 16 * q4 + lane;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          st_chunk8(sm + OFF_IP, sw128_chunk(64 + rho, 32 * half + 8 * c4, 128), v + 8 * c4);
        TC_DBG(for (int e = 0; e < 32; ++e) g_tc_dbg[12288 + rho * 64 + 32 * half + e] = v[e]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- [W, U~; A W, A U~] = [Inv diag(beta); P] [K Gamma, V] ----------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id1 = idesc_f16(128, 128, 0, 1);
      constexpr uint32_t id2 = idesc_f16(128, 64, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc(sb + OFF_IP + kk * 32, 16, 1024, kSwizzle128);
        const uint64_t bd = smem_desc(sb + OFF_KG + kk * 2048, 8192, 1024, kSwizzle128);
        mma_f16(tmem + TM_W, ad, bd, id1, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc(sb + OFF_IP + kk * 32, 16, 1024, kSwizzle128);
        const uint64_t bd = smem_desc(sb + OFF_V + kk * 2048, 8192, 1024, kSwizzle128);
        mma_f16(tmem + TM_U, ad, bd, id2, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
    ph_mma ^= 1;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();

    // ---- [W; Q' = Q Gamma - A W] -> carry operand -------------------------------
    {
      const int L = 32 * q4 + lane;
      float v[64];
      tmem_ld32(taddr(tmem, 32 * q4, TM_W + 64 * half), v);
      tmem_ld32(taddr(tmem, 32 * q4, TM_W + 64 * half + 32), v + 32);
      tmem_ld_wait();
      TC_DBG(for (int e = 0; e < 64; ++e) g_tc_dbg[16384 + L * 128 + 64 * half + e] = v[e]);
      if (L >= 64) {
        const __half* qg = reinterpret_cast<const __half*>(sm + OFF_QG) + (L - 64) * QG_STRIDE + 64 * half;
#pragma unroll
        for (int e = 0; e < 64; e += 8) {
          uint4 raw = *reinterpret_cast<const uint4*>(qg + e);
          const __half2* p2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 f = __half22float2(p2[t]);
            v[e + 2 * t] = f.x - v[e + 2 * t];
            v[e + 2 * t + 1] = f.y - v[e + 2 * t + 1];
          }
        }
      }
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        st_chunk8(sm + OFF_WQ, sw128_chunk(L, 64 * half + 8 * c8, 128), v + 8 * c8);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- carry 1: X = [W; Q'] S ---------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad =
            smem_desc(sb + OFF_WQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSwizzle128);
        const uint64_t bd = smem_desc(sb + OFF_SB + kk * 2048, 8192, 1024, kSwizzle128);
        mma_f16(tmem + TM_X, ad, bd, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
    ph_mma ^= 1;
    fence_proxy_async_smem();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    // the input tiles are free: fetch the next chunk under the rest of the carry
    if (c + 1 < nchunks) {
      if (tid == 0) issue_tma(t0 + C);
      tma_pending = true;
    }

    // ---- U = U~ - X_top -> operand;  O = A U~ + X_bottom -> out ------------------
    {
      float a[32], x[32];
      tmem_ld32(taddr(tmem, 32 * q4, TM_U + 32 * half), a);
      tmem_ld32(taddr(tmem, 32 * q4, TM_X + 32 * half), x);
      tmem_ld_wait();
      TC_DBG(for (int e = 0; e < 32; ++e) {
        g_tc_dbg[32768 + (32 * q4 + lane) * 64 + 32 * half + e] = a[e];
        g_tc_dbg[40960 + (32 * q4 + lane) * 64 + 32 * half + e] = x[e];
      });
      if (q4 < 2) {
        const int r = 32 * q4 + lane;
        float u[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) u[e] = a[e] - x[e];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          st_chunk8(sm + OFF_UB, sw128_chunk(r, 32 * half + 8 * c4, 64), u + 8 * c4);
      } else {
        const int r = 32 * (q4 - 2) + lane;
        if (r < Lc) store_row32<Tout>(out + ((size_t)(t0 + r) * H + h) * DV + j0 + 32 * half, a, x);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- carry 2: D = (K rho)^T U;  S <- Diag(gamma) S + D ----------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, 1, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc(sb + OFF_KH + kk * 2048, 8192, 1024, kSwizzle128);
        const uint64_t bd = smem_desc(sb + OFF_UB + kk * 2048, 8192, 1024, kSwizzle128);
        mma_f16(tmem + TM_D, ad, bd, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
    ph_mma ^= 1;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    {
      float d[32];
      tmem_ld32(taddr(tmem, 32 * q4, TM_D + 32 * half), d);
      tmem_ld_wait();
      const float g = gamma_s[srow];
#pragma unroll
      for (int e = 0; e < 32; ++e) S[e] = fmaf(g, S[e], d[e]);
      TC_DBG(for (int e = 0; e < 32; ++e) {
        g_tc_dbg[49152 + srow * 64 + 32 * half + e] = d[e];
        g_tc_dbg[57344 + srow * 64 + 32 * half + e] = S[e];
      });
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        st_chunk8(sm + OFF_SB, sw128_chunk(srow, 32 * half + 8 * c4, 128), S + 8 * c4);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (ok) {
    if (S_final != nullptr) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(S_final + s_off + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
  } else {
    if (tid == 0) {
      set_status(status, CKDA_ERR_DEVICE_TIMEOUT);
      // wait (bounded) for copies and tensor-core work this CTA still has in flight
      if (tma_pending) mbar_wait_bounded(bar_tma, ph_tma, kWaitNs);
      mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---- host side ------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, size_t esize,
              uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
              CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename Tout>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const float* S0, const int32_t* cu, void* out,
                     float* S_final, int n_seqs, int T, int H, int DV, int* status,
                     cudaStream_t stream) {
  const uint64_t rows = cu ? (uint64_t)T : (uint64_t)n_seqs * (uint64_t)T;
  CUtensorMap mq, mk, mv, ma;
  const bool ok = make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)H * DK, rows,
                           DK, C, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)H * DK, rows,
                           DK, C, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)H * DV, rows,
                           BV, C, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  make_map(&ma, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)H * DK,
                           rows, DK, C, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = fwd_tc_kernel<Tout>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(DV / BV, H, n_seqs);
  kern<<<grid, NT, kSmemBytes, stream>>>(mq, mk, mv, ma, beta, S0, cu, static_cast<Tout*>(out),
                                         S_final, n_seqs, T, H, DV, status);
  return cudaGetLastError();
}

}  // namespace tc

// Shapes covered by the tensor-core kernel; everything else returns
// cudaErrorNotSupported so the caller can use the CUDA-core kernel.
cudaError_t launch_fwd_tc(int dtype, int out_dtype, int dk, int dv, const void* q, const void* k,
                          const void* v, const float* alpha, const float* beta, const float* S0,
                          const int32_t* cu, void* out, float* S_final, int n_seqs, int T, int H,
                          int C, int* status, cudaStream_t stream) {
  if (dtype != CKDA_BF16 || dk != tc::DK || (dv != 64 && dv != 128) || C != tc::C)
    return cudaErrorNotSupported;
  const uint64_t rows = cu ? (uint64_t)T : (uint64_t)n_seqs * (uint64_t)T;
  if (rows == 0 || rows > 0x7fffffffull) return cudaErrorNotSupported;
  if (out_dtype == CKDA_BF16)
    return tc::launch_t<__nv_bfloat16>(q, k, v, alpha, beta, S0, cu, out, S_final, n_seqs, T, H,
                                       dv, status, stream);
  return tc::launch_t<float>(q, k, v, alpha, beta, S0, cu, out, S_final, n_seqs, T, H, dv, status,
                             stream);
}

}  // namespace ckda
