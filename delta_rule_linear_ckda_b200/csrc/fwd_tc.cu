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
// Everything except the last two lines is independent of S0, so the forward
// runs as two kernels:
//
//  1. factor2_kernel -- one work unit per (chunk, head), all units in
//     parallel (a persistent grid of two CTAs per SM walks them).  It forms
//       P  = A Inv diag(beta)
//       [W; A W] = [Inv diag(beta); P] (K * Gamma)     (one M=128 MMA)
//       Q' = Q * Gamma - A W
//     and writes [-W; Q'], K * rho, [Inv diag(beta); P] (fp16) and gamma
//     (fp32) of the unit to a workspace.
//  2. carry_kernel -- one CTA per (sequence, head, 64- or 32-column d_v
//     slice) walks its chunks in order with two dependent tensor-core
//     products each:
//       [U; O] = [Inv diag(beta); P] V + [-W; Q'] S0    (carry MMA 1)
//       D  = (K * rho)^T U,  S_C = Diag(gamma) S0 + D   (carry MMA 2)
//     since U = U~ - W S0 and O = A U~ + Q' S0 with [U~; A U~] =
//     [Inv diag(beta); P] V.  Its warps have fixed roles (state and
//     read-outs, MMA issue, TMA copies) and pass each chunk on through
//     mbarriers, while TMA streams the next chunk's factors (and its bf16 V
//     tile) in.
//
// Division-free score blocks: every pair s < r is split at the anchor m of
// the highest bit in which r and s differ ("level" h, block size b = 2^h):
// P(r, s) = [alpha_m ... alpha_r] * [alpha_{s+1} ... alpha_{m-1}], two
// running products that restart at the anchor.  Levels 2..5 (blocks of 4 to
// 32) are one GEMM each on the anchored operands; levels 0..1 (pairs inside
// aligned blocks of 4) are direct fp32 dot products.  Zero and negative
// gates are exact and underflow goes to zero; no logarithm or division.
//
// All gate products of a chunk come from one pass over aligned 4-position
// groups: every thread owns 4 channels of one group, forms the running
// products of its positions, and combines them with the products of whole
// groups and of aligned runs of them (exchanged through shared memory) into
// the level operands and into K * Gamma, Q * Gamma and K * rho.  The pass
// runs once per 32-channel quarter of d_k, so the level GEMMs are split
// along K and the next quarter's inputs stream in by TMA while the rest of
// the quarter runs.
//
// SFDA ("Semidirect Fourier Delta Attention (SFDA)" page, "Arquitectura
// Central"): the gate of channel pair (2p, 2p+1) is the complex scalar
// lambda_p = alpha_p e^{i theta_p}, i.e. a 2x2 rotation-decay block.  Those
// blocks commute, so every product above stays a running product, now of
// complex scalars; the left (row) side of T and A and the factors K * Gamma
// and Q * Gamma take the conjugate products (Gamma_r^T k_r, Gamma_r^T q_r),
// the right side and K * rho the plain ones, and the carry applies Gamma_C
// to the state's row pairs.  A conversion step turns the (alpha, theta)
// tiles of each quarter into interleaved (re, im) gates before its gate pass.
//
// Operands are fp16 tiles in 128-byte-swizzled shared memory; accumulators
// live in tensor memory; the carry kernel keeps its state slice in fp32
// registers (row i = tensor-memory lane i).  Every mbarrier wait is
// bounded: on time-out the kernel records CKDA_ERR_DEVICE_TIMEOUT, waits
// once more (bounded) for its own copies, frees its tensor memory and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace ckda {
namespace tc {

using namespace sm100;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int BV = 64;  // d_v columns of one carry CTA
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

// Level operands of the factor kernel: levels are paired (2, 3) and (4, 5),
// one M = 128 x N = 64 GEMM per pair, of which the two diagonal 64 x 32
// blocks are used.  Per pair: the left operand [levels a; b] (128 rows) and
// the right operand (64 rows), rows of one 64-channel half of d_k.
constexpr uint32_t kPairBytes = 24576;
constexpr uint32_t PAIR_ROP = 16384;

// Gate families of the factor kernel.
constexpr int kKda = 0;   // beta_r, Diag(alpha_r)
constexpr int kGdn2 = 1;  // erase gate b_r, write gate w_r, Diag(alpha_r)
constexpr int kSfda = 2;  // beta_r, phase-decay blocks alpha_p e^{i theta_p}

// ---- workspace: per unit (one chunk of one head), four arrays -------------
constexpr size_t kWsWQ = (size_t)2 * C * DK * 2;  // [-W; Q'] fp16 [128][128]
constexpr size_t kWsKH = (size_t)C * DK * 2;      // K * rho fp16 [64][128]
constexpr size_t kWsIP = (size_t)2 * C * C * 2;   // [Inv diag(beta); P] fp16 [128][64]
constexpr size_t kWsG = (size_t)DK * 4;           // gamma fp32 [128]

// ---- carry kernel: shared memory map ---------------------------------------
// Two stages of one chunk's factors, each filled by one TMA transaction.
constexpr uint32_t CS_WQ = 0;      // [-W; Q'] fp16 K-major [128][128] (two 64-column atoms)
constexpr uint32_t CS_KH = 32768;  // K * rho fp16 MN-major [64 s][128 i]
constexpr uint32_t CS_IP = 49152;  // [Inv diag(beta); P] fp16 K-major [128 r][64 s]
constexpr uint32_t CS_V = 65536;   // V slice fp16 MN-major [64 s][64 j]
constexpr uint32_t kStageBytes = 73728;
constexpr uint32_t OFF2_SB = 2 * kStageBytes;  // state slice, fp16 MN-major [128 i][64 j]
constexpr uint32_t OFF2_UB = OFF2_SB + 16384;  // U, fp16 MN-major [64 s][64 j]
constexpr uint32_t OFF2_OB = OFF2_UB + 8192;  // O staging for its TMA store: fp32 [64][32] x 2 or bf16 [64][64]
constexpr uint32_t OFF2_BAR = OFF2_OB + 16384;  // mbarriers (below)
constexpr uint32_t OFF2_TMEMPTR = OFF2_BAR + 128;
// carry mbarriers, byte offsets from OFF2_BAR
constexpr uint32_t CB_FULLA = 0;  // stage s: [-W; Q'], [Inv diag(beta); P], V loaded, + 8 s
constexpr uint32_t CB_FULLB = 16; // stage s: K * rho loaded, + 8 s
constexpr uint32_t CB_VRDY = 32;  // stage s's V converted to fp16 (conversion threads), + 8 s
constexpr uint32_t CB_SRDY = 48;  // the state's fp16 operand written (compute threads)
constexpr uint32_t CB_X = 56;     // carry 1 ([U; O]) complete (tensor-core commit)
constexpr uint32_t CB_U = 64;     // U in its operand tile (the compute threads of rows 0..63)
constexpr uint32_t CB_D = 72;     // carry 2 (D) complete (tensor-core commit)
constexpr uint32_t CB_OB = 80;    // the output staging free again (copy thread)
constexpr uint32_t CB_O = 88;     // O read out, staged or stored (the threads of rows 64..127)
constexpr uint32_t kStageBytesA = 73728 - 16384;  // a stage less K * rho
constexpr int kCarryCompute = 256;  // state / epilogue threads (8 warps)
constexpr int kCarryConvert = 128;  // V conversion threads (4 warps)
constexpr int kCarryThreads = kCarryCompute + 64 + kCarryConvert;  // + MMA warp, copy warp
constexpr uint32_t kSmem2Used = OFF2_TMEMPTR + 16;
constexpr size_t kSmem2Bytes = kSmem2Used + 1024;

// carry kernel tensor-memory columns
constexpr uint32_t kTmem2Cols = 128;
constexpr uint32_t TM2_X = 0;    // [U; O] = [U~ - W S; A U~ + Q' S]  (M = 128, 64 columns)
constexpr uint32_t TM2_D = 64;   // (K rho)^T U    (M = 128, 64 columns)

// Tensor-core operands are fp16: the bf16 inputs convert to it exactly
// (apart from subnormals), and its 10-bit mantissa keeps the rounding of the
// intermediate operands (products of gates, the WY factors, the state) at
// 2^-11 relative instead of bf16's 2^-9.  The values involved are bounded
// (|k|, |q| <= 1 per element after normalisation, |gate products| <= 1), far
// inside fp16's range.
__device__ __forceinline__ void st_h4(uint8_t* base, uint32_t off, float4 v) {
  uint2 pk;
  pk.x = pack_f16x2(v.x, v.y);
  pk.y = pack_f16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(base + off) = pk;
}

__device__ __forceinline__ void st_chunk8(uint8_t* base, uint32_t off, const float* v) {
  uint4 pk;
  pk.x = pack_f16x2(v[0], v[1]);
  pk.y = pack_f16x2(v[2], v[3]);
  pk.z = pack_f16x2(v[4], v[5]);
  pk.w = pack_f16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(base + off) = pk;
}

__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
  return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}

// Two complex products at once: (a.x + i a.y)(b.x + i b.y) and
// (a.z + i a.w)(b.z + i b.w).
__device__ __forceinline__ float4 cmul4(float4 a, float4 b) {
  return make_float4(fmaf(-a.y, b.y, a.x * b.x), fmaf(a.y, b.x, a.x * b.y),
                     fmaf(-a.w, b.w, a.z * b.z), fmaf(a.w, b.z, a.z * b.w));
}

__device__ __forceinline__ float4 conj4(float4 a) { return make_float4(a.x, -a.y, a.z, -a.w); }

__device__ __forceinline__ float4 scale4(float s, float4 a) {
  return make_float4(s * a.x, s * a.y, s * a.z, s * a.w);
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

__device__ __forceinline__ float4 ld_bf4(const uint8_t* p) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ uint32_t taddr(uint32_t tmem, int lane_base, uint32_t col) {
  return tmem + ((uint32_t)lane_base << 16) + col;
}

// Sum a 16-vector over the 16 lanes of a half-warp; afterwards lane L of the
// half holds the total of element (L & 15) in w[0].
__device__ __forceinline__ void reduce_scatter16(float* w, int lane) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? w[i] : w[i + o];
      const float keep = up ? w[i + o] : w[i];
      w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

// N consecutive output values of one row, fp32 or rounded once to bf16.
template <int N>
__device__ __forceinline__ void store_row(float* dst, const float* o) {
#pragma unroll
  for (int e = 0; e < N; e += 4)
    *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
}

template <int N>
__device__ __forceinline__ void store_row(__nv_bfloat16* dst, const float* o) {
#pragma unroll
  for (int e = 0; e < N; e += 8) {
    uint4 pk;
    pk.x = pack_bf16x2(o[e], o[e + 1]);
    pk.y = pack_bf16x2(o[e + 2], o[e + 3]);
    pk.z = pack_bf16x2(o[e + 4], o[e + 5]);
    pk.w = pack_bf16x2(o[e + 6], o[e + 7]);
    *reinterpret_cast<uint4*>(dst + e) = pk;
  }
}

// Row r (0..63) of the output tile, N columns from column c0 of the CTA's
// slice, into the 128B-swizzled staging of the TMA store: fp32 as [64][32]
// atoms (one per 32 columns), bf16 as one [64][64] atom.
template <int N>
__device__ __forceinline__ void stage_row(uint32_t ob, int r, int c0, const float* o, float) {
#pragma unroll
  for (int e = 0; e < N; e += 4) {
    const int col = c0 + e;
    const uint32_t row = ob + 8192 * (col >> 5) + 128 * r;
    sts_f4(row + (((((col & 31) >> 2)) ^ (r & 7)) << 4),
           make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]));
  }
}

template <int N>
__device__ __forceinline__ void stage_row(uint32_t ob, int r, int c0, const float* o,
                                          __nv_bfloat16) {
  const uint32_t row = ob + 128 * r;
#pragma unroll
  for (int e = 0; e < N; e += 8) {
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) w[t] = pack_bf16x2(o[e + 2 * t], o[e + 2 * t + 1]);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((((c0 + e) >> 3) ^ (r & 7)) << 4)),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                 : "memory");
  }
}

// Word offset of element (r, c) in a 64 x 64 fp32 tile whose 16-byte groups
// are XOR-swizzled by the row: a float4 column block read or written by
// threads of different rows, or a row block by threads of different column
// blocks, spreads over the banks.
__device__ __forceinline__ int fsw(int r, int c) {
  return r * 64 + ((((c >> 2) ^ r) & 15) << 2) + (c & 3);
}

// Row of position p among the 32 operand rows of level lv: the positions
// whose bit lv is set (right halves) or clear (left halves), in order.
__device__ __forceinline__ int level_row(int lv, int p) {
  return ((p >> (lv + 1)) << lv) | (p & ((1 << lv) - 1));
}

// ---- work units ----------------------------------------------------------------
//
// A unit is one chunk of one head.  Units are numbered slot * H + head, and a
// sequence's chunks occupy consecutive slots:
//   fixed-length batch:  slot = n * nch + c                   (nch = ceil(T / C))
//   packed batch:        slot = floor(cu[n] / C) + n + c
// For a packed batch the slots of sequence n end before those of n + 1
// (floor(cu[n] / C) + ceil(len_n / C) <= floor(cu[n+1] / C) + 1), so every
// slot is owned by at most one sequence and all lie below floor(T / C) + N.

struct Unit {
  int64_t idx;  // unit number; -1 = none left
  int64_t t0;   // first token row of the chunk
  int Lc;       // tokens in the chunk (1..C)
  int h;        // head
};

__device__ __forceinline__ int64_t slot_base(const int32_t* cu, int n, int nch) {
  return cu ? (int64_t)(cu[n] / C) + n : (int64_t)n * nch;
}

// The first unit at or after `ui` (stepping by `stride`) that holds tokens.
// Unit and slot numbers fit in 32 bits (the host caps units at 2^31 / 128).
__device__ Unit find_unit(int ui, int stride, int n_units, const int32_t* cu, int n_seqs, int T,
                          int H, int nch) {
  for (; ui < n_units; ui += stride) {
    const int slot = ui / H;
    const int h = ui - slot * H;
    int64_t b, e, c;
    if (cu == nullptr) {
      if (nch <= 0) break;
      const int n = slot / nch;
      c = slot - n * nch;
      b = (int64_t)n * T;
      e = b + T;
    } else {
      // last sequence n with floor(cu[n] / C) + n <= slot
      int lo = 0, hi = n_seqs - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] / C + mid <= slot)
          lo = mid;
        else
          hi = mid - 1;
      }
      b = cu[lo];
      e = cu[lo + 1];
      c = slot - (b / C + lo);
      if (b < 0 || e < b || e > T || c < 0) continue;
    }
    const int64_t t0 = b + c * C;
    if (t0 >= e) continue;
    Unit u;
    u.idx = ui;
    u.t0 = t0;
    u.Lc = (e - t0 < (int64_t)C) ? (int)(e - t0) : C;
    u.h = h;
    return u;
  }
  Unit none;
  none.idx = -1;
  none.t0 = 0;
  none.Lc = 0;
  none.h = 0;
  return none;
}

// ---- kernel 1, two CTAs per SM: per-unit WY factors (real gates) ------------------
//
// The algebra of factor_kernel for the real per-channel gates, laid out so
// that two CTAs share each SM: the barrier and shared-memory stalls of one
// CTA's phases (gate passes, inverse merges, tensor-core waits) overlap the
// other CTA's work.  256 threads and at most 105 KB of shared memory per
// CTA:
//  * the gate pass runs over 32-channel quarters of d_k (four per unit); the
//    level GEMMs of a quarter are issued as soon as its operands are written
//    (K = 32 per quarter, accumulated in tensor memory);
//  * K * rho and gamma go from registers straight to the workspace;
//  * V is not touched: the carry kernel loads the bf16 input tile itself;
//  * once the level GEMMs have read their operands, that region holds T, the
//    inverse, A (fp16), then [Inv diag(beta); P] and the -W staging.
constexpr int NT3 = 256;
constexpr int HQ = 32;  // channels of one gate sub-pass
constexpr uint32_t F2_LV = 0;        // level operands, 2 pairs x kPairBytes
constexpr uint32_t F2_TF = 0;        //   T fp32 [64][64] (fsw layout)
constexpr uint32_t F2_INV = 16384;   //   (I + T)^-1 fp32 [64][64] (fsw layout)
constexpr uint32_t F2_AQ = 32768;    //   A fp16 K-major [64 r][64 s], 128B swizzle
constexpr uint32_t F2_YF = 40960;    //   doubling scratch fp32 (<= 1024 values)
constexpr uint32_t F2_IP = 0;        //   [Inv diag(beta); P] fp16 K-major [128][64] (over T)
constexpr uint32_t F2_WS = 16384;    //   -W staging fp16 [64][128] (over the inverse)
constexpr uint32_t F2_KG = 49152;    // K * Gamma fp16 MN-major [64 s][128 i]
constexpr uint32_t F2_QG = 65536;    // Q * Gamma, then Q' (same layout)
constexpr uint32_t F2_GT = 81920;    // products of whole 4-position groups, fp32 [16][32]
constexpr uint32_t F2_T2 = 83968;    // products of aligned pairs of groups, fp32 [8][32]
constexpr uint32_t F2_PR = 84992;    // direct pairs and diag(A), fp32 [16 groups][16]
constexpr uint32_t F2_BETA = 86016;  // beta of the unit, fp32 [64]
constexpr uint32_t F2_IN = 87040;    // one sub-pass of inputs, filled by TMA:
constexpr uint32_t F2_INQ = 0, F2_INK = 4096, F2_INA = 8192, kF2InBytes = 16384;
//                                      q, k bf16 [64][32]; alpha fp32 [64][32]
constexpr uint32_t F2_BAR = F2_IN + kF2InBytes;  // mbarriers: in, lv0, lv1, mma
constexpr uint32_t F2_TMEMPTR = F2_BAR + 32;
constexpr uint32_t kF2SmemUsed = F2_TMEMPTR + 16;
constexpr size_t kF2SmemBytes = kF2SmemUsed + 1024;
static_assert(2 * (kF2SmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");
static_assert(F2_YF + 4096 <= F2_LV + 2 * kPairBytes, "inverse tiles inside the level region");
constexpr uint32_t kF2TmemCols = 256;
constexpr uint32_t TM3_LV = 0;    // level pairs (M = 128), 64 columns each; then P (M = 64)
constexpr uint32_t TM3_P = 0;
constexpr uint32_t TM3_W = 128;   // [W; A W] (M = 128, 128 columns)

// Four products as two packed fp32x2 multiplies (sm_100a); each lane rounds
// like a scalar fp32 multiply, so the results equal mul4's and scale4's.
__device__ __forceinline__ float4 mul4x(float4 a, float4 b) {
  const float2 lo = __fmul2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
  const float2 hi = __fmul2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

__device__ __forceinline__ float4 scale4x(float s, float4 a) {
  return mul4x(make_float4(s, s, s, s), a);
}

// Sum 16 values over the 8 lanes of an aligned lane octet; afterwards lane L
// of the octet holds the totals of elements 2 (L % 8) and 2 (L % 8) + 1 in
// w[0], w[1].
__device__ __forceinline__ void reduce_scatter8x2(float* w, int lane) {
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < 2 * o; ++i) {
      const float send = up ? w[i] : w[i + 2 * o];
      const float keep = up ? w[i + 2 * o] : w[i];
      w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

// Where the next sub-pass's inputs come from: unit `u` (idx < 0: none),
// quarter `j` of d_k.  SFDA fetches alpha and theta per channel pair (16 of
// each per quarter) in place of alpha per channel.
struct NextIn {
  const CUtensorMap* tq;
  const CUtensorMap* tk;
  const CUtensorMap* ta;
  const CUtensorMap* tth;  // SFDA phases (NULL otherwise)
  uint32_t dst;
  uint32_t bar;
  int x;      // first column (channel) of the quarter in the row of all heads
  int xa;     // first column of the gate tiles (the channel pair for SFDA)
  int y;      // first token row
  int valid;  // 0: nothing to fetch
};

// sin and cos of a phase for the fp16 operands of the SFDA factor kernel.
// Cody-Waite reduction to r = theta - n 2 pi, n = rint(theta / 2 pi), |r| <=
// pi: 2 pi is split into 6.28125 (eight significant bits, so n * 6.28125 is
// exact for |n| < 2^16) and the remainder, each subtracted with an fma; then
// the hardware sine and cosine, whose absolute error on [-pi, pi] is a few
// units of 2^-22, far below the fp16 rounding (2^-11) the values go through
// next.  Phases beyond 1e5 take the accurate library path instead.
__device__ __forceinline__ void phase_sincos(float th, float* s, float* c) {
  if (fabsf(th) > 1e5f) {
    sincosf(th, s, c);
    return;
  }
  constexpr float kTwoPiHi = 6.28125f;
  constexpr float kTwoPiLo = (float)(6.283185307179586 - 6.28125);
  constexpr float kInvTwoPi = (float)(1.0 / 6.283185307179586);
  const float n = rintf(th * kInvTwoPi);
  float r = fmaf(-n, kTwoPiHi, th);
  r = fmaf(-n, kTwoPiLo, r);
  __sincosf(r, s, c);
}

// SFDA: turn the (alpha, theta) tiles of one quarter (alpha at F2_INA,
// theta at F2_INA + 4096, fp32 [64 pos][16 pairs] each) into the gate tile
// the gate pass reads, fp32 [64 pos][32] with (re, im) = alpha (cos theta,
// sin theta) per pair, in place.  Every thread converts 4 pairs of one
// position; the values are read before the barrier and written after it.
__device__ __forceinline__ void phase_to_gates_q(uint32_t in, int tid) {
  const int p = tid >> 2, j = tid & 3;
  const float4 a = lds_f4(in + F2_INA + p * 64 + 16 * j);
  const float4 th = lds_f4(in + F2_INA + 4096 + p * 64 + 16 * j);
  float s0, c0, s1, c1, s2, c2, s3, c3;
  phase_sincos(th.x, &s0, &c0);
  phase_sincos(th.y, &s1, &c1);
  phase_sincos(th.z, &s2, &c2);
  phase_sincos(th.w, &s3, &c3);
  __syncthreads();
  sts_f4(in + F2_INA + p * 128 + 32 * j, make_float4(a.x * c0, a.x * s0, a.y * c1, a.y * s1));
  sts_f4(in + F2_INA + p * 128 + 32 * j + 16, make_float4(a.z * c2, a.z * s2, a.w * c3, a.w * s3));
  __syncthreads();
}

// One gate pass over quarter `jq` (channels 32 jq .. 32 jq + 31 of d_k) with
// 256 threads.  Thread (role, g, c4): warp w = 4 role + kk, g = 4 kk + lane / 8
// (positions 4g .. 4g + 3, one aligned block of 4), c4 = lane % 8 (channels
// 4 c4 .. 4 c4 + 3 of the quarter).  Each scheduler (warps kk and kk + 4)
// gets both roles of the same four groups, whose level work adds up to the
// same amount on every scheduler.  Role 0 walks forward (Gamma, K * Gamma,
// Q * Gamma, the right halves of levels 2..5, gamma to the workspace); role 1
// walks backward (K * rho straight to the workspace, the left halves) and
// adds its channels' share of the direct pairs of levels 0..1 and of diag(A)
// to the pair buffer.  The inputs are read into registers first; after the
// barrier that follows, thread 0 requests the next sub-pass's inputs into the
// same buffer (`nx`).  Operand tiles have 128-byte rows of one 64-channel
// half; this quarter fills logical 16-byte chunks 4 (jq % 2) .. 4 (jq % 2) + 3.
//
// kGdn2: the erase side uses e = b * k (b read from global memory at `bgp` +
// position * `bstride`, the quarter's channels) in place of beta * k, in the
// T rows of the level operands, the direct T pairs and E * Gamma (stored
// where K * Gamma goes).  kSfda: the gate tile holds (re, im) pairs, every
// gate product is a complex product and the row-side operands (K * Gamma,
// Q * Gamma, the left level operands) take the conjugate of their product.
template <int GK>
__device__ __noinline__ void gate_pass_q(uint32_t sb, int jq, int Lc, int tid,
                                         __half* __restrict__ kh_row0,
                                         float* __restrict__ g_dst, NextIn nx,
                                         const float* __restrict__ bgp, int bstride) {
  constexpr bool G2 = GK == kGdn2;
  constexpr bool SF = GK == kSfda;
  auto gm = [](float4 a, float4 b) -> float4 {
    if constexpr (SF)
      return cmul4(a, b);
    else
      return mul4x(a, b);
  };
  auto gc = [](float4 a) -> float4 {
    if constexpr (SF)
      return conj4(a);
    else
      return a;
  };
  const int w = tid >> 5;
  const int lane = tid & 31;
  const int role = w >> 2;
  const int kk = w & 3;
  const int g = 4 * kk + (lane >> 3);
  const int c4 = lane & 7;
  const int cl = 4 * c4;               // channel within the quarter
  const int hh = jq >> 1;              // half of d_k
  const int cq = 32 * (jq & 1) + cl;   // channel within the half
  const int ig = 64 * hh + cq;         // channel within d_k
  const float4 one = SF ? make_float4(1.f, 0.f, 1.f, 0.f) : make_float4(1.f, 1.f, 1.f, 1.f);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  const uint32_t in = sb + F2_IN;
  auto bf4 = [](uint2 raw) -> float4 {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    return make_float4(a.x, a.y, b.x, b.y);
  };
  auto h4 = [](float4 v) -> uint2 {
    uint2 pk;
    pk.x = pack_f16x2(v.x, v.y);
    pk.y = pack_f16x2(v.z, v.w);
    return pk;
  };

  float4 aa[4], ka[4], qa[4], eg[4];
  float bb[4];
  if constexpr (G2) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = 4 * g + u;
      eg[u] = (p < Lc) ? __ldg(reinterpret_cast<const float4*>(bgp + (size_t)p * bstride + cl))
                       : zero;
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int p = 4 * g + u;
    const bool val = p < Lc;
    aa[u] = val ? lds_f4(in + F2_INA + p * 128 + cl * 4) : one;
    ka[u] = val ? bf4(lds_u2(in + F2_INK + p * 64 + cl * 2)) : zero;
    qa[u] = val ? bf4(lds_u2(in + F2_INQ + p * 64 + cl * 2)) : zero;
    if constexpr (!G2) bb[u] = lds_f(sb + F2_BETA + p * 4);
  }
  // products of whole groups, and (one shuffle across neighbouring groups,
  // 8 lanes apart) of aligned pairs of groups
  const uint32_t gt = sb + F2_GT + cl * 4;
  if (role == 0) {
    const float4 t = gm(gm(aa[0], aa[1]), gm(aa[2], aa[3]));
    sts_f4(gt + g * 128, t);
    float4 o;
    o.x = __shfl_xor_sync(0xffffffffu, t.x, 8);
    o.y = __shfl_xor_sync(0xffffffffu, t.y, 8);
    o.z = __shfl_xor_sync(0xffffffffu, t.z, 8);
    o.w = __shfl_xor_sync(0xffffffffu, t.w, 8);
    if (!(g & 1)) sts_f4(sb + F2_T2 + (g >> 1) * 128 + cl * 4, gm(t, o));
  }
  __syncthreads();
  // every input of this sub-pass is in registers: the buffer takes the next one
  if (tid == 0 && nx.valid) {
    fence_proxy_async_smem();
    mbar_expect_tx(nx.bar, kF2InBytes);
    tma_load_2d(nx.dst + F2_INQ, nx.tq, nx.x, nx.y, nx.bar);
    tma_load_2d(nx.dst + F2_INK, nx.tk, nx.x, nx.y, nx.bar);
    tma_load_2d(nx.dst + F2_INA, nx.ta, nx.xa, nx.y, nx.bar);
    if constexpr (SF) tma_load_2d(nx.dst + F2_INA + 4096, nx.tth, nx.xa, nx.y, nx.bar);
  }
  if constexpr (G2) {
#pragma unroll
    for (int u = 0; u < 4; ++u) eg[u] = mul4x(eg[u], ka[u]);  // e = b * k
  }
  auto gtot = [&](int gg) -> float4 { return lds_f4(gt + gg * 128); };
  auto run2 = [&](int s2) -> float4 { return lds_f4(sb + F2_T2 + s2 * 128 + cl * 4); };
  auto run4 = [&](int s4) -> float4 { return gm(run2(2 * s4), run2(2 * s4 + 1)); };
  auto run8 = [&](int s8) -> float4 {
    return gm(gm(run2(4 * s8), run2(4 * s8 + 1)), gm(run2(4 * s8 + 2), run2(4 * s8 + 3)));
  };
  const uint32_t LV = sb + F2_LV;
  // Store addresses in the 128B-swizzled operand tiles: this thread's 4
  // channels are logical chunk 4 (jq % 2) + c4 / 2, half c4 % 2 of it; the
  // chunk is XOR-ed with the row's low three bits, which for position rows
  // and levels 3..5 are 4 (g & 1) + u and for level 2 4 ((g >> 1) & 1) + u.
  const int lchunk = 4 * (jq & 1) + (c4 >> 1);
  uint32_t xo[4], xo2[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    xo[u] = (uint32_t)(((lchunk ^ (4 * (g & 1) + u)) << 4) | ((c4 & 1) << 3));
    xo2[u] = (uint32_t)(((lchunk ^ (4 * ((g >> 1) & 1) + u)) << 4) | ((c4 & 1) << 3));
  }
  const uint32_t rowg = (uint32_t)(4 * g) * 128 + (uint32_t)hh * 8192;
  auto lrow = [&](int lv) -> uint32_t { return (uint32_t)level_row(lv, 4 * g) * 128; };
  auto pair_base = [&](int lv) -> uint32_t { return LV + ((lv - 2) >> 1) * kPairBytes; };

  if (role == 0) {
    const int g4 = g & ~3;
    float4 off4 = one;
    if (g - g4 >= 1) off4 = gtot(g4);
    if (g - g4 >= 2) off4 = gm(off4, gtot(g4 + 1));
    if (g - g4 >= 3) off4 = gm(off4, gtot(g4 + 2));
    const float4 off3 = (g & 1) ? gtot(g - 1) : one;
    const float4 off5 = (g & 4) ? gm(run4((g >> 2) & ~1), off4) : off4;
    float4 pg = (g & 8) ? gm(run8(0), off5) : off5;  // Gamma offset: every earlier group
    // the row side takes the conjugate offsets (the same values unless SF)
    const float4 off3c = gc(off3), off4c = gc(off4), off5c = gc(off5);
    const uint32_t kg_b = sb + F2_KG + rowg;
    const uint32_t qg_b = sb + F2_QG + rowg;
    const uint32_t l2b = pair_base(2) + lrow(2);
    const uint32_t l3b = pair_base(3) + 64 * 128 + lrow(3);
    const uint32_t l4b = pair_base(4) + lrow(4);
    const uint32_t l5b = pair_base(5) + 64 * 128 + lrow(5);
    float4 lp = one;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 a = aa[u];
      pg = gm(pg, a);
      lp = (u == 0) ? a : gm(lp, a);
      const uint32_t ro = 128 * u + xo[u];
      // data times the row-side gate: gc(gate) * data (conjugate for SF)
      sts_u2(kg_b + ro, h4(gm(gc(pg), G2 ? eg[u] : ka[u])));
      sts_u2(qg_b + ro, h4(gm(gc(pg), qa[u])));
      if (g & 15) {
        const float4 lpc = gc(lp);
        const float4 qlp = gm(lpc, qa[u]);
        const float4 blp = G2 ? mul4x(eg[u], lp) : scale4x(bb[u], gm(lpc, ka[u]));
        if (g & 1) {  // level 2: right half
          const uint32_t o2 = l2b + 128 * u + xo2[u];
          sts_u2(o2, h4(blp));
          sts_u2(o2 + 32 * 128, h4(qlp));
        }
        if (g & 2) {  // level 3: right half
          sts_u2(l3b + ro, h4(gm(blp, off3c)));
          sts_u2(l3b + 32 * 128 + ro, h4(gm(qlp, off3c)));
        }
        if (g & 4) {  // level 4: right half
          sts_u2(l4b + ro, h4(gm(blp, off4c)));
          sts_u2(l4b + 32 * 128 + ro, h4(gm(qlp, off4c)));
        }
        if (g & 8) {  // level 5: right half
          sts_u2(l5b + ro, h4(gm(blp, off5c)));
          sts_u2(l5b + 32 * 128 + ro, h4(gm(qlp, off5c)));
        }
      }
    }
    if (g == 15) *reinterpret_cast<float4*>(g_dst + ig) = pg;
  } else {
    float4 offr4 = one;
    if ((g | 3) - g >= 1) offr4 = gtot(g + 1);
    if ((g | 3) - g >= 2) offr4 = gm(offr4, gtot(g + 2));
    if ((g | 3) - g >= 3) offr4 = gm(offr4, gtot(g + 3));
    const float4 offr3 = (g & 1) ? one : gtot(g + 1);
    const float4 offr5 = (g & 4) ? offr4 : gm(offr4, run4((g >> 2) + 1));
    const float4 offr = (g & 8) ? offr5 : gm(offr5, run8(1));  // rho offset: every later group
    const uint32_t r2b = pair_base(2) + PAIR_ROP + lrow(2);
    const uint32_t r3b = pair_base(3) + PAIR_ROP + 32 * 128 + lrow(3);
    const uint32_t r4b = pair_base(4) + PAIR_ROP + lrow(4);
    const uint32_t r5b = pair_base(5) + PAIR_ROP + 32 * 128 + lrow(5);
    float4 ls = one;
#pragma unroll
    for (int u = 3; u >= 0; --u) {
      const float4 kls = gm(ka[u], ls);
      const uint32_t ro = 128 * u + xo[u];
      // K * rho, fp16, straight to the workspace row of position 4g + u
      *reinterpret_cast<uint2*>(kh_row0 + (size_t)(4 * g + u) * DK + ig) = h4(gm(kls, offr));
      if (!(g & 1)) sts_u2(r2b + 128 * u + xo2[u], h4(kls));
      if (!(g & 2)) sts_u2(r3b + ro, h4(gm(kls, offr3)));
      if (!(g & 4)) sts_u2(r4b + ro, h4(gm(kls, offr4)));
      if (!(g & 8)) sts_u2(r5b + ro, h4(gm(kls, offr5)));
      ls = gm(ls, aa[u]);
    }
    // direct pairs inside this aligned block of 4 (levels 0 and 1) and diag(A)
    float acc[16];
    {
      const float4 k0 = ka[0], k1 = ka[1], k2 = ka[2], k3 = ka[3];
      const float4 q1 = qa[1], q2 = qa[2], q3 = qa[3];
      // row side of the T pairs: k_r (scaled by beta_r in the gather) or e_r
      const float4 t1 = G2 ? eg[1] : k1, t2 = G2 ? eg[2] : k2, t3 = G2 ? eg[3] : k3;
      const float4 e10 = gm(aa[1], k0);
      const float4 e20 = gm(aa[2], e10);
      const float4 e21 = gm(aa[2], k1);
      const float4 e30 = gm(aa[3], e20);
      const float4 e31 = gm(aa[3], e21);
      const float4 e32 = gm(aa[3], k2);
      acc[0] = dot4(t1, e10);  acc[1] = dot4(q1, e10);
      acc[2] = dot4(t2, e20);  acc[3] = dot4(q2, e20);
      acc[4] = dot4(t2, e21);  acc[5] = dot4(q2, e21);
      acc[6] = dot4(t3, e30);  acc[7] = dot4(q3, e30);
      acc[8] = dot4(t3, e31);  acc[9] = dot4(q3, e31);
      acc[10] = dot4(t3, e32); acc[11] = dot4(q3, e32);
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[12 + u] = dot4(qa[u], ka[u]);
    }
    // sum over the 8 threads (channels) of the group
    reduce_scatter8x2(acc, lane);
    const uint32_t p0 = sb + F2_PR + 64 * g + 8 * (lane & 7);
    if (jq == 0) {
      sts_u2(p0, make_uint2(__float_as_uint(acc[0]), __float_as_uint(acc[1])));
    } else {
      const uint2 o = lds_u2(p0);
      sts_u2(p0, make_uint2(__float_as_uint(__uint_as_float(o.x) + acc[0]),
                            __float_as_uint(__uint_as_float(o.y) + acc[1])));
    }
  }
}

// One step of the recursive-doubling inverse of the unit lower-triangular
// (I + T) with NTH threads: merge diagonal blocks of size M into blocks of
// size 2M,
//   [[A, 0], [B, D]]^-1 = [[A^-1, 0], [-D^-1 B A^-1, D^-1]],  B = T block.
// Inv holds the inverses of the M-blocks and zeros above the block diagonal
// (fsw layout, as T).  A^-1 and D^-1 are lower triangular, so the first
// product only runs over rows t >= c of A^-1 and the second over t <= a of
// D^-1.
template <int M, int NTH>
__device__ __forceinline__ void inv_merge_n(const float* Tf, float* Inv, float* Yf, int tid) {
  constexpr int NMERGE = 64 / (2 * M);
  constexpr int W4 = M / 4;
  constexpr int NOUT = NMERGE * M * W4;
  for (int e = tid; e < NOUT; e += NTH) {
    const int qb = e / (M * W4), a = (e / W4) % M, c4 = e % W4;
    const int r0 = 2 * M * qb;
    const int tr = r0 + M + a;
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
    for (int t4 = c4; t4 < M / 4; ++t4) {
      const float4 tv = *reinterpret_cast<const float4*>(Tf + fsw(tr, r0 + 4 * t4));
      const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float4 iv =
            *reinterpret_cast<const float4*>(Inv + fsw(r0 + 4 * t4 + w, r0 + 4 * c4));
        y.x = fmaf(tt[w], iv.x, y.x); y.y = fmaf(tt[w], iv.y, y.y);
        y.z = fmaf(tt[w], iv.z, y.z); y.w = fmaf(tt[w], iv.w, y.w);
      }
    }
    *reinterpret_cast<float4*>(Yf + qb * M * M + a * M + 4 * c4) = y;
  }
  __syncthreads();
  for (int e = tid; e < NOUT; e += NTH) {
    const int qb = e / (M * W4), a = (e / W4) % M, c4 = e % W4;
    const int r0 = 2 * M * qb;
    const int ir = r0 + M + a;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
    for (int t4 = 0; t4 <= (a >> 2); ++t4) {
      const float4 dv = *reinterpret_cast<const float4*>(Inv + fsw(ir, r0 + M + 4 * t4));
      const float dd[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float4 yv =
            *reinterpret_cast<const float4*>(Yf + qb * M * M + (4 * t4 + w) * M + 4 * c4);
        x.x = fmaf(dd[w], yv.x, x.x); x.y = fmaf(dd[w], yv.y, x.y);
        x.z = fmaf(dd[w], yv.z, x.z); x.w = fmaf(dd[w], yv.w, x.w);
      }
    }
    *reinterpret_cast<float4*>(Inv + fsw(ir, r0 + 4 * c4)) =
        make_float4(-x.x, -x.y, -x.z, -x.w);
  }
  __syncthreads();
}

// ws_kh: K * rho fp16 [units * C][DK] (row-major), ws_g: gamma fp32 [units][DK].
// kGdn2: erase gate bg (shaped like k) in place of beta on the key side; the
// factors are [-W; Q'] with W = Inv (E * Gamma) and [Inv; A Inv] (the write
// gate is applied to V by the carry kernel).  kSfda: alpha and theta fp32
// [rows, H * DK / 2] (tm_a, tm_th); gamma is stored as (re, im) pairs.
template <int GK>
__global__ void __launch_bounds__(NT3, 2)
factor2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_th,
               const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_ip,
               const float* __restrict__ beta, const float* __restrict__ bg,
               const __nv_bfloat16* __restrict__ qg, const __nv_bfloat16* __restrict__ kg,
               const float* __restrict__ ag, const float* __restrict__ thg,
               const int32_t* __restrict__ cu, int n_seqs, int T, int H, int nch,
               int64_t n_units, __half* __restrict__ ws_kh, float* __restrict__ ws_g,
               int* status) {
  constexpr bool G2 = GK == kGdn2;
  constexpr bool SF = GK == kSfda;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int q4 = warp & 3;        // tensor-memory lane quarter of this warp
  const int quarter = warp >> 2;  // which half of a tile's columns this warp takes

  float* beta_s = reinterpret_cast<float*>(sm + F2_BETA);
  const uint32_t bar_in = sb + F2_BAR;
  const uint32_t bar_lv0 = sb + F2_BAR + 8;
  const uint32_t bar_mma = sb + F2_BAR + 24;
  if (tid == 0) {
    mbar_init(bar_in, 1);
    mbar_init(bar_lv0, 1);
    mbar_init(bar_lv0 + 8, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_a);
    if (SF) prefetch_tmap(&tm_th);
    prefetch_tmap(&tm_wq);
    prefetch_tmap(&tm_ip);
  }
  if (warp == 0) {
    tmem_alloc(sb + F2_TMEMPTR, kF2TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + F2_TMEMPTR);

  uint32_t ph_in = 0, ph_lv[2] = {0, 0}, ph_mma = 0;
  int pend_in = 0, pend_lv[2] = {0, 0}, pend_mma = 0;
  int ok = 1;
  auto wait = [&](uint32_t bar, uint32_t& ph, int& pend) -> bool {
    const bool r = mbar_wait_bounded(bar, ph, kWaitNs);
    if (r) {
      ph ^= 1;
      pend = 0;
    }
    return r;
  };
  auto next_in = [&](const Unit& uu, int jq) -> NextIn {
    NextIn n;
    n.tq = &tm_q;
    n.tk = &tm_k;
    n.ta = &tm_a;
    n.tth = SF ? &tm_th : nullptr;
    n.dst = sb + F2_IN;
    n.bar = bar_in;
    n.x = uu.h * DK + HQ * jq;
    n.xa = SF ? uu.h * (DK / 2) + (HQ / 2) * jq : n.x;
    n.y = (int)uu.t0;
    n.valid = uu.idx >= 0;
    return n;
  };
  // Shared-memory descriptors: each tile's base; a K step adds its byte
  // offset / 16 to the low field.
  const uint64_t d_lv = smem_desc(sb + F2_LV, 16, 1024, kSwizzle128);
  const uint64_t d_aq = smem_desc(sb + F2_AQ, 16, 1024, kSwizzle128);
  const uint64_t d_ipk = smem_desc(sb + F2_IP, 16, 1024, kSwizzle128);     // K-major (A)
  const uint64_t d_ipm = smem_desc(sb + F2_IP, 8192, 1024, kSwizzle128);   // MN-major (B)
  const uint64_t d_kg = smem_desc(sb + F2_KG, 8192, 1024, kSwizzle128);
  auto level_mmas = [&](int jq) {
    constexpr uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int kk = 2 * (jq & 1) + k2;
        const uint64_t ad = d_lv + (pr * kPairBytes + kk * 32) / 16;
        const uint64_t bd = d_lv + (pr * kPairBytes + PAIR_ROP + kk * 32) / 16;
        mma_f16(tmem + TM3_LV + 64 * pr, ad, bd, id, (jq > 0 || k2 > 0) ? 1u : 0u);
      }
    }
    mma_commit(bar_lv0 + 8 * (jq & 1));
  };
  auto load_beta = [&](const Unit& uu) -> float {
    if constexpr (G2) return 0.f;  // unused
    return (uu.idx >= 0 && tid < uu.Lc) ? beta[(size_t)(uu.t0 + tid) * H + uu.h] : 0.f;
  };
  // Pull a unit's input rows into L2, one 128-byte line per thread and step:
  // per token q, k (2 lines each), the gates (alpha: 4 lines; SFDA alpha and
  // theta: 2 each), and for Gated DeltaNet-2 the erase gate (4 lines), read
  // with plain loads.
  auto prefetch_unit = [&](const Unit& uu) {
    constexpr int NL = G2 ? 12 : 8;
    if (uu.idx < 0) return;
    for (int e = tid; e < C * NL; e += NT3) {
      const int r = e / NL, li = e % NL;
      if (r >= uu.Lc) break;
      const size_t row = (size_t)(uu.t0 + r) * H + uu.h;
      const void* a;
      if (li < 2) {
        a = qg + row * DK + 64 * li;
      } else if (li < 4) {
        a = kg + row * DK + 64 * (li - 2);
      } else if (li < 8) {
        if constexpr (SF) {
          const float* base = (li < 6) ? ag : thg;
          a = base + row * (DK / 2) + 32 * ((li - 4) & 1);
        } else {
          a = ag + row * DK + 32 * (li - 4);
        }
      } else {
        a = bg + row * DK + 32 * (li - 8);
      }
      prefetch_l2(a);
    }
  };

  Unit cur = find_unit(blockIdx.x, gridDim.x, (int)n_units, cu, n_seqs, T, H, nch);
  float beta_next = 0.f;
  if (cur.idx >= 0) {
    if (tid == 0) {
      const NextIn n0 = next_in(cur, 0);
      mbar_expect_tx(bar_in, kF2InBytes);
      tma_load_2d(n0.dst + F2_INQ, &tm_q, n0.x, n0.y, bar_in);
      tma_load_2d(n0.dst + F2_INK, &tm_k, n0.x, n0.y, bar_in);
      tma_load_2d(n0.dst + F2_INA, &tm_a, n0.xa, n0.y, bar_in);
      if (SF) tma_load_2d(n0.dst + F2_INA + 4096, &tm_th, n0.xa, n0.y, bar_in);
    }
    pend_in = 1;
    beta_next = load_beta(cur);
  }

  for (; cur.idx >= 0;) {
    const Unit nxt =
        find_unit((int)cur.idx + gridDim.x, gridDim.x, (int)n_units, cu, n_seqs, T, H, nch);
    const int Lc = cur.Lc;
    const size_t u = (size_t)cur.idx;
    prefetch_unit(nxt);
    // the previous unit's workspace stores read the level region and Q'
    if (tid == 0) bulk_wait_read_all();
    if (tid < C) beta_s[tid] = beta_next;
    __half* kh_row0 = ws_kh + u * C * DK;
    float* g_dst = ws_g + u * DK;

    // ---- four gate sub-passes; the level GEMMs of each follow it -------------
    for (int jq = 0; jq < 4; ++jq) {
      ok = wait(bar_in, ph_in, pend_in);
      // sub-pass jq overwrites the operand chunks the GEMMs of jq - 2 read
      if (jq >= 2) ok = wait(bar_lv0 + 8 * (jq & 1), ph_lv[jq & 1], pend_lv[jq & 1]) && ok;
      ok = __syncthreads_and(ok);
      if (!ok) break;
      const NextIn nx = (jq < 3) ? next_in(cur, jq + 1) : next_in(nxt, 0);
      if constexpr (SF) phase_to_gates_q(sb + F2_IN, tid);
      gate_pass_q<GK>(sb, jq, Lc, tid, kh_row0, g_dst, nx,
                      G2 ? bg + ((size_t)cur.t0 * H + cur.h) * DK + HQ * jq : nullptr, H * DK);
      if (nx.valid) pend_in = 1;
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        level_mmas(jq);
      }
      pend_lv[jq & 1] = 1;
    }
    if (!ok) break;
    if (tid < C) beta_next = load_beta(nxt);

    // ---- T (fp32) and A (fp16 operand) from levels 2..5, direct pairs, diag(A)
    ok = wait(bar_lv0, ph_lv[0], pend_lv[0]);
    ok = wait(bar_lv0 + 8, ph_lv[1], pend_lv[1]) && ok;
    // A's operand tile lies over level operands the GEMMs have now read: zero
    // it (entries above the diagonal stay zero)
    {
      uint4* aq = reinterpret_cast<uint4*>(sm + F2_AQ);
      aq[tid] = make_uint4(0u, 0u, 0u, 0u);
      aq[tid + NT3] = make_uint4(0u, 0u, 0u, 0u);
    }
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    {
      float* Tf = reinterpret_cast<float*>(sm + F2_TF);
      // warp (lane quarter q4, pair warp / 4): one 32-column block of a pair
      {
        const int pr = warp >> 2;
        const int L = 32 * q4 + lane;
        const int rho = L & 63;
        const int rr = rho & 31;
        const int lv = 2 + 2 * pr + (L >> 6);
        float v[32];
        tmem_ld32(taddr(tmem, 32 * q4, TM3_LV + 64 * pr + 32 * (q4 >> 1)), v);
        tmem_ld_wait();
        const int b = 1 << lv;
        const int j = rr >> lv;
        const int r = 2 * b * j + b + (rr & (b - 1));
#pragma unroll
        for (int m4 = 0; m4 < 8; ++m4) {
          if (((4 * m4) >> lv) == j) {
            const int s = b * j + 4 * m4;
            if (rho < 32) {
              *reinterpret_cast<float4*>(Tf + fsw(r, s)) =
                  make_float4(v[4 * m4], v[4 * m4 + 1], v[4 * m4 + 2], v[4 * m4 + 3]);
            } else {
              uint2 pk;
              pk.x = pack_f16x2(v[4 * m4], v[4 * m4 + 1]);
              pk.y = pack_f16x2(v[4 * m4 + 2], v[4 * m4 + 3]);
              *reinterpret_cast<uint2*>(sm + F2_AQ + sw128_elem(r, s, 64)) = pk;
            }
          }
        }
      }
      // direct pairs (r, s) inside aligned blocks of 4, and the diagonal of A
      {
        const float* prb = reinterpret_cast<const float*>(sm + F2_PR);
        const int g = tid >> 4, w = tid & 15;
        const float val = prb[tid];
        int r, s;
        if (w < 12) {
          const int jj = w >> 1;
          // pair order inside the block: (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
          r = 4 * g + ((jj == 0) ? 1 : (jj < 3 ? 2 : 3));
          s = 4 * g + ((jj == 0 || jj == 1 || jj == 3) ? 0 : (jj == 2 || jj == 4 ? 1 : 2));
        } else {
          r = s = 4 * g + (w - 12);
        }
        if (w < 12 && !(w & 1))
          Tf[fsw(r, s)] = G2 ? val : beta_s[r] * val;
        else
          *reinterpret_cast<__half*>(sm + F2_AQ + sw128_elem(r, s, 64)) = __float2half_rn(val);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- (I + T)^-1 by recursive doubling -------------------------------------------
    {
      const float* Tf = reinterpret_cast<const float*>(sm + F2_TF);
      float* Inv = reinterpret_cast<float*>(sm + F2_INV);
      float* Yf = reinterpret_cast<float*>(sm + F2_YF);
      for (int e = tid; e < 64 * 16; e += NT3) {
        const int r = e >> 4, c4 = e & 15;
        if (c4 >= 2 * (r >> 3) + 2)
          *reinterpret_cast<float4*>(Inv + fsw(r, 4 * c4)) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (tid < 64) {
        const int base = 8 * (tid >> 3), cc = tid & 7;
        float tb[8][8];
#pragma unroll
        for (int r2 = 1; r2 < 8; ++r2) {
          const float4 lo = *reinterpret_cast<const float4*>(Tf + fsw(base + r2, base));
          const float4 hi = *reinterpret_cast<const float4*>(Tf + fsw(base + r2, base + 4));
          tb[r2][0] = lo.x; tb[r2][1] = lo.y; tb[r2][2] = lo.z; tb[r2][3] = lo.w;
          tb[r2][4] = hi.x; tb[r2][5] = hi.y; tb[r2][6] = hi.z; tb[r2][7] = hi.w;
        }
        float x[8];
#pragma unroll
        for (int r2 = 0; r2 < 8; ++r2) {
          float acc = (r2 == cc) ? 1.f : 0.f;
#pragma unroll
          for (int s2 = 0; s2 < r2; ++s2) acc = fmaf(-tb[r2][s2], x[s2], acc);
          x[r2] = (r2 < cc) ? 0.f : acc;
        }
#pragma unroll
        for (int r2 = 0; r2 < 8; ++r2) Inv[fsw(base + r2, base + cc)] = x[r2];
      }
      __syncthreads();
      inv_merge_n<8, NT3>(Tf, Inv, Yf, tid);
      inv_merge_n<16, NT3>(Tf, Inv, Yf, tid);
      inv_merge_n<32, NT3>(Tf, Inv, Yf, tid);
      // Inv diag(beta) -> rows 0..63 of the stacked operand (over T, now unused)
#pragma unroll
      for (int rep = 0; rep < 2; ++rep) {
        const int r = 32 * rep + (tid >> 3), cg = tid & 7;
        const float4 lo = *reinterpret_cast<const float4*>(Inv + fsw(r, 8 * cg));
        const float4 hi = *reinterpret_cast<const float4*>(Inv + fsw(r, 8 * cg + 4));
        const float i8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = G2 ? i8[t] : i8[t] * beta_s[8 * cg + t];
        st_chunk8(sm + F2_IP, sw128_chunk(r, 8 * cg, 128), v);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- P = A Inv diag(beta) ---------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(64, 64, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM3_P, d_aq + 2 * kk, d_ipm + 128 * kk, id, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    pend_mma = 1;
    ok = wait(bar_mma, ph_mma, pend_mma);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    {
      // M = 64 accumulator: row 16 * q4 + l sits in lane l (< 16) of quarter q4
      float v[32];
      tmem_ld32(taddr(tmem, 32 * q4, TM3_P + 32 * quarter), v);
      tmem_ld_wait();
      if (lane < 16) {
        const int rho = 16 * q4 + lane;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          st_chunk8(sm + F2_IP, sw128_chunk(64 + rho, 32 * quarter + 8 * c8, 128), v + 8 * c8);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- [W; A W] = [Inv diag(beta); P] (K Gamma) ----------------------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id1 = idesc_f16(128, 128, 0, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = d_ipk + 2 * kk;
        const uint64_t bd = d_kg + 128 * kk;
        mma_f16(tmem + TM3_W, ad, bd, id1, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
      tma_store_2d(&tm_ip, sb + F2_IP, 0, (int)(u * 2 * C));
      bulk_commit();
    }
    pend_mma = 1;
    ok = wait(bar_mma, ph_mma, pend_mma);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();

    // ---- [-W; Q' = Q Gamma - A W] -> workspace -------------------------------------------
    {
      const int L = 32 * q4 + lane;
      const int r = L & 63;
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        const int col0 = 64 * quarter + 32 * cb;
        float v[32];
        tmem_ld32(taddr(tmem, 32 * q4, TM3_W + col0), v);
        tmem_ld_wait();
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float w8[8];
          if (L >= 64) {
            const uint32_t off = F2_QG + sw128_chunk(r, col0 + 8 * c8, 64);
            const uint4 raw = *reinterpret_cast<const uint4*>(sm + off);
            const __half2* p2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 f = __half22float2(p2[t]);
              w8[2 * t] = f.x - v[8 * c8 + 2 * t];
              w8[2 * t + 1] = f.y - v[8 * c8 + 2 * t + 1];
            }
            st_chunk8(sm, off, w8);
          } else {
#pragma unroll
            for (int t = 0; t < 8; ++t) w8[t] = -v[8 * c8 + t];
            st_chunk8(sm, F2_WS + sw128_chunk(r, col0 + 8 * c8, 64), w8);
          }
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      const int y = (int)(u * 2 * C);
      tma_store_2d(&tm_wq, sb + F2_WS, 0, y);
      tma_store_2d(&tm_wq, sb + F2_WS + 8192, 64, y);
      tma_store_2d(&tm_wq, sb + F2_QG, 0, y + C);
      tma_store_2d(&tm_wq, sb + F2_QG + 8192, 64, y + C);
      bulk_commit();
    }
    cur = nxt;
  }
  if (tid == 0) bulk_wait_all();
  if (!ok) {
    if (tid == 0) {
      set_status(status, CKDA_ERR_DEVICE_TIMEOUT);
      if (pend_in) mbar_wait_bounded(bar_in, ph_in, kWaitNs);
      if (pend_lv[0]) mbar_wait_bounded(bar_lv0, ph_lv[0], kWaitNs);
      if (pend_lv[1]) mbar_wait_bounded(bar_lv0 + 8, ph_lv[1], kWaitNs);
      if (pend_mma) mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kF2TmemCols);
}

// ---- kernel 2: the chunk-to-chunk carry ---------------------------------------------

// SF: gamma holds (re, im) pairs and multiplies the state's row pairs
// (2p, 2p+1) as a complex scalar; the partner row is the neighbouring lane.
//
// Segments (the chunk-parallel scan): a sequence's chunks split into
// `seg_n` contiguous segments, chunks [g nck / seg_n, (g + 1) nck / seg_n);
// this launch runs `seg_launch` of them (blockIdx.z = n seg_launch + g).
// With summ == NULL (outputs): segment 0 starts from S0, segment g > 0 from
// seg_start[n, g] ([N, seg_n, H, DK, DV] fp32), and the last segment stores
// S_final.  With summ != NULL (the affine summary of a segment, "Principales
// Contribuciones" item 3): the launch's columns are [M | B], DK + DV of them;
// the M columns start from the identity and take no V term (the segment's
// transfer matrix), the B columns start from zero (the zero-start state);
// nothing is output and the end state goes to summ[n, g] ([N, seg_launch, H,
// DK, DK + DV] fp32).  seg_n = seg_launch = 1 is the plain forward.
//
// V comes from the bf16 input itself (tm_v16 maps the input v, [rows,
// H * d_v]) and is converted to fp16 in the stage, rows past the chunk's
// end set to zero.  WG (Gated DeltaNet-2): the conversion multiplies V by
// the write gate wg ([rows, H * d_v] fp32), giving Z = w * V.
//
// NBV: the d_v columns of one CTA, 64 or 32 (narrower slices put more CTAs
// on the GPU when there are few (sequence, head) pairs, as in one long
// sequence); each thread holds NBV / 2 columns of one state row.
template <typename Tout, bool SF, bool WG, int NBV>
__global__ void __launch_bounds__(kCarryThreads, 1)
carry_kernel(const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_kh,
             const __grid_constant__ CUtensorMap tm_ip, const __grid_constant__ CUtensorMap tm_v16,
             const __grid_constant__ CUtensorMap tm_out,
             const float* __restrict__ ws_g, const float* __restrict__ wg,
             const float* S0, const int32_t* __restrict__ cu, Tout* __restrict__ out,
             float* S_final, int n_seqs, int T, int H, int DV, int nch, int* status,
             int seg_n, int seg_launch, const float* __restrict__ seg_start,
             float* __restrict__ summ) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  constexpr int CPT = NBV / 2;  // state columns per compute thread
  const int j0 = blockIdx.x * NBV;
  const int h = blockIdx.y;
  // (a plain packed forward walks its sequences longest first)
  const int n = (seg_n == 1 && summ == nullptr) ? seq_longest_first(cu, n_seqs, blockIdx.z)
                                                : blockIdx.z / seg_launch;
  const int seg = blockIdx.z % seg_launch;
  const bool summary = summ != nullptr;
  const bool mcols = summary && j0 < DK;  // transfer-matrix columns
  const int jv = summary ? j0 - DK : j0;  // V and output column of this CTA
  const bool has_v = !mcols;              // the chunk's V term enters carry 1

  const SeqRange sr = seq_range(cu, n, n_seqs, T, status);
  if (!sr.ok) return;

  const uint32_t bar = sb + OFF2_BAR;
  if (tid == 0) {
    mbar_init(bar + CB_FULLA, 1);
    mbar_init(bar + CB_FULLA + 8, 1);
    mbar_init(bar + CB_FULLB, 1);
    mbar_init(bar + CB_FULLB + 8, 1);
    mbar_init(bar + CB_VRDY, kCarryConvert);
    mbar_init(bar + CB_VRDY + 8, kCarryConvert);
    mbar_init(bar + CB_SRDY, kCarryCompute);
    mbar_init(bar + CB_X, 1);
    mbar_init(bar + CB_U, kCarryCompute / 2);
    mbar_init(bar + CB_D, 1);
    mbar_init(bar + CB_OB, 1);
    mbar_init(bar + CB_O, kCarryCompute / 2);
    fence_mbar_init();
    prefetch_tmap(&tm_wq);
    prefetch_tmap(&tm_kh);
    prefetch_tmap(&tm_ip);
    prefetch_tmap(&tm_v16);
    prefetch_tmap(&tm_out);
  }
  if (warp == 0) {
    tmem_alloc(sb + OFF2_TMEMPTR, kTmem2Cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF2_TMEMPTR);

  const int64_t tok0 = sr.begin;
  const int64_t tok1 = sr.end;
  const int nck_all = (int)((tok1 - tok0 + C - 1) / C);
  // this segment's chunks [cbeg, cbeg + nchunks)
  const int cbeg = (int)((int64_t)seg * nck_all / seg_n);
  const int nchunks = (int)((int64_t)(seg + 1) * nck_all / seg_n) - cbeg;
  const int64_t slot0 = slot_base(cu, n, nch);
  auto unit_of = [&](int c) -> int64_t { return (slot0 + cbeg + c) * H + h; };
  auto chunk_len = [&](int c) -> int {
    const int64_t t0c = tok0 + (int64_t)(cbeg + c) * C;
    return (tok1 - t0c < (int64_t)C) ? (int)(tok1 - t0c) : C;
  };
  // whole chunks go out by TMA (the bf16 output map's box is 64 columns
  // wide, so a 32-column bf16 slice stores its rows itself)
  auto tma_out = [&](int c) -> bool {
    return !summary && ((cu == nullptr) || chunk_len(c) == C) &&
           (NBV == 64 || sizeof(Tout) == 4);
  };
  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    return mbar_wait_bounded(b, parity, kWaitNs);
  };
  int ok = 1;

  // Four roles hand each chunk to one another through mbarriers, so that
  // no block-wide barrier stands between the steps of the chunk-to-chunk
  // chain (S -> carry 1 -> U -> carry 2 -> S):
  //  * warps 0..7 (compute): the state slice in registers, the read-outs of
  //    both tensor-memory products, U into its operand tile, O staged or
  //    stored;
  //  * warp 8 (one thread): every tcgen05 MMA;
  //  * warp 9 (one thread): the stage loads and the output stores by TMA.
  //    A stage is loaded in two parts: what carry 1 reads ([-W; Q'],
  //    [Inv diag(beta); P], V) is fetched again as soon as carry 1 is done
  //    with it, K * rho once carry 2 is;
  //  * warps 10..13 (conversion): each chunk's V to fp16 as soon as it lands.
  // Each barrier completes once per chunk (the stage barriers once per two),
  // so the parity waited for follows from the chunk index.
  float S[CPT];
  int mma_pend = 0;            // MMA thread: a commit not yet seen complete
  uint32_t mma_bar = 0, mma_par = 0;
  uint32_t ld_pend = 0;        // copy thread: bit 2 s + part, a load not yet seen complete
  uint32_t ld_par = 0;         //   the same bit, the parity of that load's phase

  if (warp < 8) {
    // ---- compute warps ----------------------------------------------------------------
    // State slice: row i = 32 * (warp % 4) + lane, columns [CPT * (warp / 4), +CPT).
    const int q4 = warp & 3;
    const int half = warp >> 2;
    const int srow = 32 * q4 + lane;
    const size_t s_off = (((size_t)n * H + h) * DK + srow) * DV + j0 + CPT * half;
    const float* s_row = nullptr;
    if (seg == 0) {
      if (S0 != nullptr) s_row = S0 + s_off;
    } else {
      s_row = seg_start + ((((size_t)n * seg_n + seg) * H + h) * DK + srow) * DV + j0 +
              CPT * half;
    }
#pragma unroll
    for (int e = 0; e < CPT; e += 4) {
      float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (summary) {
        if (mcols) {
          const int c = j0 + CPT * half + e - srow;  // identity: 1 where column == row
          v4 = make_float4(c == 0 ? 1.f : 0.f, c == -1 ? 1.f : 0.f, c == -2 ? 1.f : 0.f,
                           c == -3 ? 1.f : 0.f);
        }
      } else if (s_row != nullptr) {
        v4 = *reinterpret_cast<const float4*>(s_row + e);
      }
      S[e] = v4.x; S[e + 1] = v4.y; S[e + 2] = v4.z; S[e + 3] = v4.w;
    }
#pragma unroll
    for (int c4 = 0; c4 < CPT / 8; ++c4)
      st_chunk8(sm + OFF2_SB, sw128_chunk(srow, CPT * half + 8 * c4, 128), S + 8 * c4);
    fence_proxy_async_smem();
    mbar_arrive(bar + CB_SRDY);

    // gamma of this row (SF: of its row pair, real and imaginary part)
    const int grow = SF ? (srow & ~1) : srow;
    auto load_gamma = [&](int c) -> float2 {
      if (c >= nchunks) return make_float2(1.f, 0.f);
      const float* gp = ws_g + unit_of(c) * DK + grow;
      return SF ? *reinterpret_cast<const float2*>(gp) : make_float2(*gp, 0.f);
    };
    float2 gm = load_gamma(0);
    for (int c = 0; ok && c < nchunks; ++c) {
      const uint32_t par = (uint32_t)c & 1u;
      const int64_t t0 = tok0 + (int64_t)(cbeg + c) * C;
      const int Lc = chunk_len(c);
      const bool to = tma_out(c);
      const float2 gm_next = load_gamma(c + 1);

      // ---- carry 1 done: U -> operand tile, O -> out ----------------------------
      if (!wait(bar + CB_X, par)) { ok = 0; break; }
      tc_fence_after();
      {
        float x[CPT];
        if constexpr (CPT == 32)
          tmem_ld32(taddr(tmem, 32 * q4, TM2_X + CPT * half), x);
        else
          tmem_ld16(taddr(tmem, 32 * q4, TM2_X + CPT * half), x);
        tmem_ld_wait();
        if (q4 < 2) {
#pragma unroll
          for (int c4 = 0; c4 < CPT / 8; ++c4)
            st_chunk8(sm + OFF2_UB, sw128_chunk(srow, CPT * half + 8 * c4, 64), x + 8 * c4);
        } else if (!summary) {
          const int r = srow - 64;
          if (to) {
            // the previous chunk's output store must have read its staging
            if (c > 0 && !wait(bar + CB_OB, par ^ 1u)) { ok = 0; break; }
            stage_row<CPT>(sb + OFF2_OB, r, CPT * half, x, Tout());
          } else if (r < Lc) {
            store_row<CPT>(out + ((size_t)(t0 + r) * H + h) * DV + j0 + CPT * half, x);
          }
        }
      }
      // (rows 0..63 release carry 2, rows 64..127 the output store and the
      // accumulator)
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar + (q4 < 2 ? CB_U : CB_O));

      // ---- carry 2 done: S <- Diag(gamma) S + D, its fp16 copy for the next chunk --
      if (!wait(bar + CB_D, par)) { ok = 0; break; }
      tc_fence_after();
      {
        float d[CPT];
        if constexpr (CPT == 32)
          tmem_ld32(taddr(tmem, 32 * q4, TM2_D + CPT * half), d);
        else
          tmem_ld16(taddr(tmem, 32 * q4, TM2_D + CPT * half), d);
        tmem_ld_wait();
        if constexpr (SF) {
          // even row: gr S_e - gi S_o + d;  odd row: gr S_o + gi S_e + d
          const float gi = (lane & 1) ? gm.y : -gm.y;
#pragma unroll
          for (int e = 0; e < CPT; ++e) {
            const float po = __shfl_xor_sync(0xffffffffu, S[e], 1);
            S[e] = fmaf(gm.x, S[e], fmaf(gi, po, d[e]));
          }
        } else {
#pragma unroll
          for (int e = 0; e < CPT; ++e) S[e] = fmaf(gm.x, S[e], d[e]);
        }
#pragma unroll
        for (int c4 = 0; c4 < CPT / 8; ++c4)
          st_chunk8(sm + OFF2_SB, sw128_chunk(srow, CPT * half + 8 * c4, 128), S + 8 * c4);
      }
      gm = gm_next;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar + CB_SRDY);
    }
  } else if (warp == 8) {
    // ---- MMA thread ---------------------------------------------------------------------
    if (lane == 0) {
      // Shared-memory descriptors of the carry's operands: the base of each
      // tile; a K step adds its byte offset / 16 to the low field (a stage's
      // descriptors are stage 0's plus kStageBytes / 16).
      const uint64_t d_ip0 = smem_desc(sb + CS_IP, 16, 1024, kSwizzle128);
      const uint64_t d_v0 = smem_desc(sb + CS_V, 8192, 1024, kSwizzle128);
      const uint64_t d_wq0 = smem_desc(sb + CS_WQ, 16, 1024, kSwizzle128);
      const uint64_t d_kh0 = smem_desc(sb + CS_KH, 8192, 1024, kSwizzle128);
      const uint64_t d_sb = smem_desc(sb + OFF2_SB, 8192, 1024, kSwizzle128);
      const uint64_t d_ub = smem_desc(sb + OFF2_UB, 8192, 1024, kSwizzle128);
      constexpr uint32_t id_c1 = idesc_f16(128, NBV, 0, 1);
      constexpr uint32_t id_c2 = idesc_f16(128, NBV, 1, 1);
      for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const uint32_t par = (uint32_t)c & 1u;
        const uint32_t spar = (uint32_t)(c >> 1) & 1u;
        const uint64_t so = st ? (uint64_t)(kStageBytes >> 4) : 0ull;
        // the previous chunk's O rows of the accumulator have been read out
        if (c > 0 && !wait(bar + CB_O, par ^ 1u)) { ok = 0; break; }
        if (has_v) {
          // carry 1's V term, [Inv diag(beta); P] V: independent of S, in as
          // soon as V is fp16 (the U rows of the accumulator were read out
          // before carry 2 of the previous chunk was issued)
          // (V converted implies the stage's first part has landed)
          if (!wait(bar + CB_VRDY + 8 * st, spar)) { ok = 0; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + TM2_X, d_ip0 + so + 2 * kk, d_v0 + so + 128 * kk, id_c1,
                    kk > 0 ? 1u : 0u);
        } else if (!wait(bar + CB_FULLA + 8 * st, spar)) {
          ok = 0;
          break;
        }
        // carry 1's S term, [-W; Q'] S
        if (!wait(bar + CB_SRDY, par)) { ok = 0; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16(tmem + TM2_X, d_wq0 + so + 1024 * (kk >> 2) + 2 * (kk & 3), d_sb + 128 * kk,
                  id_c1, (kk > 0 || has_v) ? 1u : 0u);
        mma_commit(bar + CB_X);
        mma_pend = 1; mma_bar = bar + CB_X; mma_par = par;
        // carry 2, D = (K rho)^T U, once U is in its tile and K rho has landed
        if (!wait(bar + CB_U, par) || !wait(bar + CB_FULLB + 8 * st, spar)) { ok = 0; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem + TM2_D, d_kh0 + so + 128 * kk, d_ub + 128 * kk, id_c2, kk > 0 ? 1u : 0u);
        mma_commit(bar + CB_D);
        mma_bar = bar + CB_D;
      }
    }
  } else if (warp == 9) {
    // ---- copy thread: stage loads and output stores by TMA ----------------------------
    if (lane == 0) {
      // part 0 of chunk c into stage st: [-W; Q'], [Inv diag(beta); P], V;
      // part 1: K * rho
      auto issue = [&](int c, int st, int part) {
        const uint32_t b = bar + (part ? CB_FULLB : CB_FULLA) + 8 * st;
        const uint32_t base = sb + st * kStageBytes;
        const int64_t uidx = unit_of(c);
        if (part == 0) {
          mbar_expect_tx(b, kStageBytesA);
          tma_load_2d(base + CS_WQ, &tm_wq, 0, (int)(uidx * 2 * C), b);
          tma_load_2d(base + CS_WQ + 16384, &tm_wq, 64, (int)(uidx * 2 * C), b);
          tma_load_2d(base + CS_IP, &tm_ip, 0, (int)(uidx * 2 * C), b);
          tma_load_2d(base + CS_V, &tm_v16, h * DV + (mcols ? 0 : jv),
                      (int)(tok0 + (int64_t)(cbeg + c) * C), b);
        } else {
          mbar_expect_tx(b, kStageBytes - kStageBytesA);
          tma_load_2d(base + CS_KH, &tm_kh, 0, (int)(uidx * C), b);
          tma_load_2d(base + CS_KH + 8192, &tm_kh, 64, (int)(uidx * C), b);
        }
        const int bit = 2 * st + part;
        ld_pend |= 1u << bit;
        ld_par = (ld_par & ~(1u << bit)) | (((uint32_t)(c >> 1) & 1u) << bit);
      };
      for (int c = 0; c < 2 && c < nchunks; ++c) {
        issue(c, c, 0);
        issue(c, c, 1);
      }
      for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const uint32_t par = (uint32_t)c & 1u;
        const bool to = tma_out(c);
        // carry 1 is done with the stage's first part: fetch chunk c + 2's
        if (!wait(bar + CB_X, par)) { ok = 0; break; }
        ld_pend &= ~(1u << (2 * st));
        if (c + 2 < nchunks) issue(c + 2, st, 0);
        // O of the chunk staged: store it
        if (!wait(bar + CB_O, par)) { ok = 0; break; }
        if (to) {
          // fixed-length batch: [T, H * d_v] per sequence, rows past T are
          // clipped; packed batch: only whole chunks come here
          const int x0 = h * DV + j0;
          if (cu == nullptr) {
            const int y0 = (cbeg + c) * C;
            tma_store_3d(&tm_out, sb + OFF2_OB, x0, y0, n);
            if (sizeof(Tout) == 4 && NBV == 64)
              tma_store_3d(&tm_out, sb + OFF2_OB + 8192, x0 + 32, y0, n);
          } else {
            const int t0 = (int)(tok0 + (int64_t)(cbeg + c) * C);
            tma_store_2d(&tm_out, sb + OFF2_OB, x0, t0);
            if (sizeof(Tout) == 4 && NBV == 64)
              tma_store_2d(&tm_out, sb + OFF2_OB + 8192, x0 + 32, t0);
          }
          bulk_commit();
        }
        // carry 2 is done with K * rho: fetch chunk c + 2's
        if (!wait(bar + CB_D, par)) { ok = 0; break; }
        ld_pend &= ~(1u << (2 * st + 1));
        if (c + 2 < nchunks) issue(c + 2, st, 1);
        if (to) bulk_wait_read_all();
        mbar_arrive(bar + CB_OB);
      }
      bulk_wait_all();
    }
  } else if (has_v) {
    // ---- conversion warps ---------------------------------------------------------------
    const int ct = tid - (kCarryCompute + 64);  // 0 .. kCarryConvert - 1
    // bf16 V (as loaded) -> fp16 in place in stage `s` (WG: times the write
    // gate), rows past the chunk's `len` tokens -> 0.  Each 16-byte chunk
    // stays within its 128-byte row under the swizzle.
    auto convert_v = [&](int s, int c) {
      const int len = chunk_len(c);
      const int64_t t0c = tok0 + (int64_t)(cbeg + c) * C;
      uint4* vt = reinterpret_cast<uint4*>(sm + s * kStageBytes + CS_V);
      constexpr int kPer = C * 8 / kCarryConvert;  // 16-byte chunks of V per thread
      static_assert(C * 8 == kPer * kCarryConvert, "V chunks per thread");
      // every load of the thread first (V from shared memory; WG: the write
      // gate from global memory), then the arithmetic
      uint4 raws[kPer];
      float4 wa[WG ? kPer : 1], wb[WG ? kPer : 1];
#pragma unroll
      for (int it = 0; it < kPer; ++it) {
        const int e = ct + it * kCarryConvert;
        raws[it] = vt[e];
        if constexpr (WG) {
          // logical columns of this 16-byte chunk: 8 * (chunk ^ (row % 8));
          // only the slice's own NBV columns are used (and read)
          const int row = e >> 3;
          const int col = 8 * ((e & 7) ^ (row & 7));
          wa[it] = wb[it] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (row < len && col < NBV) {
            const float* wp = wg + ((size_t)(t0c + row) * H + h) * DV + jv + col;
            wa[it] = __ldg(reinterpret_cast<const float4*>(wp));
            wb[it] = __ldg(reinterpret_cast<const float4*>(wp + 4));
          }
        }
      }
#pragma unroll
      for (int it = 0; it < kPer; ++it) {
        const int e = ct + it * kCarryConvert;
        const int row = e >> 3;
        uint4 raw = raws[it];
        if (row < len) {
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
          float f[8];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 x2 = __bfloat1622float2(p2[t]);
            f[2 * t] = x2.x;
            f[2 * t + 1] = x2.y;
          }
          if constexpr (WG) {
            f[0] *= wa[it].x; f[1] *= wa[it].y; f[2] *= wa[it].z; f[3] *= wa[it].w;
            f[4] *= wb[it].x; f[5] *= wb[it].y; f[6] *= wb[it].z; f[7] *= wb[it].w;
          }
          raw = make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]),
                           pack_f16x2(f[4], f[5]), pack_f16x2(f[6], f[7]));
        } else {
          raw = make_uint4(0u, 0u, 0u, 0u);
        }
        vt[e] = raw;
      }
    };
    // WG: the write-gate rows of chunk c pulled into L2 (128-byte lines
    // spread over the conversion threads) a chunk before its conversion
    // reads them
    auto prefetch_w = [&](int c) {
      if constexpr (WG) {
        constexpr int LPR = NBV / 32;  // 128-byte lines per row
        for (int e = ct; e < C * LPR; e += kCarryConvert) {
          const int r = e / LPR;
          if (c < nchunks && r < chunk_len(c))
            prefetch_l2(wg + ((size_t)(tok0 + (int64_t)(cbeg + c) * C + r) * H + h) * DV + jv +
                        32 * (e % LPR));
        }
      }
    };
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1;
      prefetch_w(c + 1);
      if (!wait(bar + CB_FULLA + 8 * st, (uint32_t)(c >> 1) & 1u)) { ok = 0; break; }
      convert_v(st, c);
      fence_proxy_async_smem();
      mbar_arrive(bar + CB_VRDY + 8 * st);
    }
  }

  ok = __syncthreads_and(ok);
  if (ok) {
    if (warp < 8) {
      const int q4 = warp & 3;
      const int half = warp >> 2;
      const int srow = 32 * q4 + lane;
      if (summary) {
        float* dst = summ + (((size_t)n * seg_launch + seg) * H + h) * DK * (DK + DV) +
                     (size_t)srow * (DK + DV) + j0 + CPT * half;
#pragma unroll
        for (int e = 0; e < CPT; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
      } else if (S_final != nullptr && seg == seg_n - 1) {
        float* dst = S_final + (((size_t)n * H + h) * DK + srow) * DV + j0 + CPT * half;
#pragma unroll
        for (int e = 0; e < CPT; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
      }
    }
  } else {
    if (tid == 0) set_status(status, CKDA_ERR_DEVICE_TIMEOUT);
    // every copy and MMA this CTA issued completes before its memory goes
    if (warp == 8 && lane == 0 && mma_pend) mbar_wait_bounded(mma_bar, mma_par, kWaitNs);
    if (warp == 9 && lane == 0) {
      for (int b2 = 0; b2 < 4; ++b2)
        if ((ld_pend >> b2) & 1u)
          mbar_wait_bounded(bar + ((b2 & 1) ? CB_FULLB : CB_FULLA) + 8 * (b2 >> 1),
                            (ld_par >> b2) & 1u, kWaitNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmem2Cols);
}

// ---- the scan over segment summaries ----------------------------------------------
//
// For one (sequence, head): S_start(0) = S0 (or 0) and
//   S_start(g + 1) = M_g S_start(g) + B_g,   g = 0 .. seg_n - 2,
// the exact affine transfer of a block of chunks ("Semidirect Fourier Delta
// Attention" page, "Principales Contribuciones" item 3), with [M_g | B_g]
// from the summary carry.  fp32 on CUDA cores: 256 threads, each an 8 x 8
// block of the DK x DV product (DV = 128; DV = 64 uses half of them).
constexpr int kScanThreads = 256;
constexpr size_t kScanSmem = (size_t)(DK * DK + DK * 128) * 4;

__global__ void __launch_bounds__(kScanThreads, 1)
scan_kernel(const float* __restrict__ summ, const float* __restrict__ S0, float* __restrict__ seg_start,
            int H, int DV, int seg_n) {
  extern __shared__ __align__(16) float sm_scan[];
  float* Ms = sm_scan;            // M_g [DK][DK]
  float* Ss = sm_scan + DK * DK;  // S_start(g) [DK][DV]
  const int tid = threadIdx.x;
  const int h = blockIdx.x, n = blockIdx.y;
  const int W = DK + DV;
  for (int e = tid; e < DK * DV; e += kScanThreads)
    Ss[e] = (S0 != nullptr) ? S0[(((size_t)n * H + h) * DK) * DV + e] : 0.f;
  const int i0 = 8 * (tid / 16), jb = 8 * (tid % 16);
  const bool act = jb < DV;
  for (int g = 0; g + 1 < seg_n; ++g) {
    const float* sg = summ + (((size_t)n * (seg_n - 1) + g) * H + h) * DK * W;
    __syncthreads();  // Ss holds S_start(g); Ms is free
    for (int e = tid; e < DK * DK; e += kScanThreads) Ms[e] = sg[(size_t)(e / DK) * W + e % DK];
    __syncthreads();
    float acc[8][8];
    if (act) {
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = sg[(size_t)(i0 + a) * W + DK + jb + b];
      for (int kx = 0; kx < DK; ++kx) {
        float m[8], x[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) m[a] = Ms[(i0 + a) * DK + kx];
#pragma unroll
        for (int b = 0; b < 8; ++b) x[b] = Ss[kx * DV + jb + b];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(m[a], x[b], acc[a][b]);
      }
    }
    __syncthreads();  // every thread is done reading Ss
    if (act) {
      float* dst = seg_start + ((((size_t)n * seg_n + g + 1) * H + h) * DK) * DV;
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          Ss[(i0 + a) * DV + jb + b] = acc[a][b];
          dst[(size_t)(i0 + a) * DV + jb + b] = acc[a][b];
        }
    }
  }
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

bool make_map3(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, size_t esize,
               uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1,
               CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Work units of a call (at least one, so the workspace maps are never empty).
int64_t n_units(bool varlen, int n_seqs, int T, int H) {
  const int64_t nch = ((int64_t)T + C - 1) / C;
  const int64_t slots = varlen ? (int64_t)T / C + n_seqs : (int64_t)n_seqs * nch;
  const int64_t u = slots * H;
  return u > 0 ? u : 1;
}

// (the same for every d_v: V is read from the input by the carry kernel)
size_t unit_bytes(int) { return kWsWQ + kWsKH + kWsIP + kWsG; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// phases: kFactors runs kernel 1 (inputs -> workspace), kCarry kernel 2
// (workspace, S0 -> out, S_final); a full forward runs both, in order, on
// `stream`.
constexpr int kFactors = 1, kCarry = 2;

// Segments of the carry phase (the chunk-parallel scan); the default is the
// plain forward (one segment).
struct Segs {
  int n = 1;                      // segments per sequence
  int launch = 1;                 // segments this carry launch runs
  const float* start = nullptr;   // start states of the segments
  float* summ = nullptr;          // non-NULL: summary launch ([M | B] per segment)
};

template <int DV, typename Tout, int GK>
cudaError_t launch_t(int phases, const void* q, const void* k, const void* v, const float* alpha,
                     const float* beta, const float* bg, const float* wg, const float* theta,
                     const float* S0, const int32_t* cu, void* out, float* S_final, int n_seqs,
                     int T, int H, void* ws, int* status, cudaStream_t stream,
                     Segs segs = Segs()) {
  constexpr bool SF = GK == kSfda;
  const uint64_t rows = cu ? (uint64_t)T : (uint64_t)n_seqs * (uint64_t)T;
  const int nch = (int)(((int64_t)T + C - 1) / C);
  const int64_t nu = n_units(cu != nullptr, n_seqs, T, H);
  // workspace arrays, in this order: [-W; Q'], K rho, [Inv diag(beta); P],
  // gamma -- every one a multiple of 512 bytes per unit
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  __half* ws_wq = reinterpret_cast<__half*>(w8);
  __half* ws_kh = reinterpret_cast<__half*>(w8 + nu * kWsWQ);
  __half* ws_ip = reinterpret_cast<__half*>(w8 + nu * (kWsWQ + kWsKH));
  float* ws_g = reinterpret_cast<float*>(w8 + nu * (kWsWQ + kWsKH + kWsIP));

  CUtensorMap mkh, mip;
  if (!make_map(&mkh, ws_kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, DK, (uint64_t)nu * C, 64, C,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mip, ws_ip, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, C, (uint64_t)nu * 2 * C, 64,
                2 * C, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  // V never enters the workspace: the carry kernel reads the bf16 input
  // itself (and applies Gated DeltaNet-2's write gate there).
  constexpr bool G2 = GK == kGdn2;
  if (phases & kFactors) {
    CUtensorMap mq, mk, ma, mth, mwq64;
    // SF: alpha and theta hold one value per channel pair (DK / 2 per head)
    const uint64_t a_cols = SF ? (uint64_t)H * (DK / 2) : (uint64_t)H * DK;
    const uint32_t a_box = SF ? HQ / 2 : HQ;
    const bool ok =
        make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)H * DK, rows, HQ, C,
                 CU_TENSOR_MAP_SWIZZLE_NONE) &&
        make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)H * DK, rows, HQ, C,
                 CU_TENSOR_MAP_SWIZZLE_NONE) &&
        make_map(&ma, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a_cols, rows, a_box, C,
                 CU_TENSOR_MAP_SWIZZLE_NONE) &&
        make_map(&mth, SF ? theta : alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a_cols, rows,
                 a_box, C, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        make_map(&mwq64, ws_wq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, DK, (uint64_t)nu * 2 * C, 64,
                 C, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    // Two CTAs per SM (the largest shared-memory carveout); the persistent
    // grid has two CTAs for every SM.  Measured on B200: the same grid of one
    // CTA per SM takes 43 % longer.
    auto k1 = factor2_kernel<GK>;
    static bool attr1 = false;
    if (!attr1) {
      cudaError_t e = set_smem(k1, kF2SmemBytes);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k1, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      attr1 = true;
    }
    const int64_t cap = 2 * (int64_t)sm_count();
    const int64_t g1 = nu < cap ? nu : cap;
    k1<<<(unsigned)g1, NT3, kF2SmemBytes, stream>>>(
        mq, mk, ma, mth, mwq64, mip, beta, bg, static_cast<const __nv_bfloat16*>(q),
        static_cast<const __nv_bfloat16*>(k), alpha, theta, cu, n_seqs, T, H, nch, nu, ws_kh,
        ws_g, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (phases & kCarry) {
    constexpr bool kF32 = sizeof(Tout) == 4;
    const CUtensorMapDataType tout =
        kF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t ob_cols = kF32 ? 32 : 64;
    CUtensorMap mwq, mout, mvin;
    if (!make_map(&mvin, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)H * DV, rows, 64, C,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const bool ok =
        make_map(&mwq, ws_wq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, DK, (uint64_t)nu * 2 * C, 64,
                 2 * C, CU_TENSOR_MAP_SWIZZLE_128B) &&
        (cu ? make_map(&mout, out, tout, sizeof(Tout), (uint64_t)H * DV, rows, ob_cols, C,
                       CU_TENSOR_MAP_SWIZZLE_128B)
            : make_map3(&mout, out, tout, sizeof(Tout), (uint64_t)H * DV, (uint64_t)T,
                        (uint64_t)n_seqs, ob_cols, C, CU_TENSOR_MAP_SWIZZLE_128B));
    if (!ok) return cudaErrorInvalidValue;
    // 32-column slices when 64-column ones would leave more than half of the
    // SMs without a carry CTA (few (sequence, head) pairs: a long sequence)
    const int cols = segs.summ != nullptr ? DK + DV : DV;
    const int64_t ctas64 = (int64_t)(cols / BV) * H * n_seqs * segs.launch;
    const bool narrow = 2 * ctas64 <= (int64_t)sm_count();
    auto k2 = narrow ? carry_kernel<Tout, SF, G2, 32> : carry_kernel<Tout, SF, G2, 64>;
    static bool attr2[2] = {false, false};
    if (!attr2[narrow]) {
      cudaError_t e = set_smem(k2, kSmem2Bytes);
      if (e != cudaSuccess) return e;
      attr2[narrow] = true;
    }
    dim3 grid(cols / (narrow ? 32 : BV), H, n_seqs * segs.launch);
    k2<<<grid, kCarryThreads, kSmem2Bytes, stream>>>(mwq, mkh, mip, mvin, mout, ws_g, wg, S0, cu,
                                          static_cast<Tout*>(out), S_final, n_seqs, T, H, DV,
                                          nch, status, segs.n, segs.launch, segs.start,
                                          segs.summ);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace tc

// Shapes covered by the tensor-core kernels: bf16 inputs, d_k = 128,
// d_v in {64, 128}, chunk 64, and every TMA row coordinate (token rows and
// workspace rows, 2 C per unit) within int32.
bool fwd_tc_supported(int dtype, int dk, int dv, int C, int n_seqs, int T, int H, bool varlen) {
  const uint64_t rows = varlen ? (uint64_t)T : (uint64_t)n_seqs * (uint64_t)T;
  if (dtype != CKDA_BF16 || dk != tc::DK || (dv != 64 && dv != 128) || C != tc::C) return false;
  if (n_seqs <= 0 || H <= 0 || rows == 0 || rows > 0x7fffffffull) return false;
  return (uint64_t)tc::n_units(varlen, n_seqs, T, H) * 2 * tc::C <= 0x7fffffffull;
}

// Workspace bytes the tensor-core path needs (0 when it does not apply).
size_t fwd_tc_workspace_bytes(int dtype, int dk, int dv, int C, int n_seqs, int T, int H,
                              bool varlen) {
  if (!fwd_tc_supported(dtype, dk, dv, C, n_seqs, T, H, varlen)) return 0;
  const int64_t nu = tc::n_units(varlen, n_seqs, T, H);
  return (size_t)nu * tc::unit_bytes(dv);
}

// ---- the chunk-parallel scan forward ------------------------------------------
// Workspace: the factor workspace, then the segment summaries [N, G - 1, H,
// DK, DK + DV] and the segment start states [N, G, H, DK, DV] (fp32).
size_t fwd_tc_scan_workspace_bytes(int dk, int dv, int n_seqs, int T, int H, int G) {
  if (!fwd_tc_supported(CKDA_BF16, dk, dv, tc::C, n_seqs, T, H, false) || G < 1) return 0;
  const size_t fw = (size_t)tc::n_units(false, n_seqs, T, H) * tc::unit_bytes(dv);
  const size_t sm = (size_t)n_seqs * (G - 1) * H * dk * (dk + dv) * 4;
  const size_t ss = (size_t)n_seqs * G * H * dk * dv * 4;
  return fw + sm + ss;
}

// The forward as G segments per sequence: factors of every chunk; the affine
// summary [M_g | B_g] of segments 0 .. G - 2 (all in parallel); the scan of
// the segments' start states; the carry of every segment from its start
// state (all in parallel).  Same result as the plain forward up to rounding.
cudaError_t launch_fwd_tc_scan(int out_dtype, int dv, const void* q, const void* k,
                               const void* v, const float* alpha, const float* beta,
                               const float* S0, void* out, float* S_final, int n_seqs, int T,
                               int H, int G, void* ws, int* status, cudaStream_t stream) {
  const size_t fw = (size_t)tc::n_units(false, n_seqs, T, H) * tc::unit_bytes(dv);
  float* summ = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + fw);
  float* starts = summ + (size_t)n_seqs * (G - 1) * H * tc::DK * (tc::DK + dv);
  const bool bf = out_dtype == CKDA_BF16;
  auto run = [&](int phases, tc::Segs sg, float* sfin) -> cudaError_t {
#define CKDA_TC_SCAN(DVV, TO)                                                                  \
  tc::launch_t<DVV, TO, tc::kKda>(phases, q, k, v, alpha, beta, nullptr, nullptr, nullptr, S0, \
                                  nullptr, out, sfin, n_seqs, T, H, ws, status, stream, sg)
    if (dv == 128) return bf ? CKDA_TC_SCAN(128, __nv_bfloat16) : CKDA_TC_SCAN(128, float);
    return bf ? CKDA_TC_SCAN(64, __nv_bfloat16) : CKDA_TC_SCAN(64, float);
#undef CKDA_TC_SCAN
  };
  cudaError_t e = run(tc::kFactors, tc::Segs(), S_final);
  if (e != cudaSuccess || G == 1) {
    if (e != cudaSuccess) return e;
    return run(tc::kCarry, tc::Segs(), S_final);
  }
  tc::Segs sum;
  sum.n = G;
  sum.launch = G - 1;
  sum.summ = summ;
  if ((e = run(tc::kCarry, sum, nullptr)) != cudaSuccess) return e;
  static bool attr = false;
  if (!attr) {
    if ((e = cudaFuncSetAttribute(tc::scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)tc::kScanSmem)) != cudaSuccess)
      return e;
    attr = true;
  }
  tc::scan_kernel<<<dim3(H, n_seqs), tc::kScanThreads, tc::kScanSmem, stream>>>(summ, S0, starts, H,
                                                                                 dv, G);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  tc::Segs fin;
  fin.n = G;
  fin.launch = G;
  fin.start = starts;
  return run(tc::kCarry, fin, S_final);
}

// Everything the tensor-core kernels do not cover returns
// cudaErrorNotSupported so the caller can use the CUDA-core kernel.
// `phases`: 1 = factors only, 2 = carry only, 3 = the whole forward.
// `bg`, `wg` non-NULL select the Gated DeltaNet-2 form (beta unused);
// `theta` non-NULL the SFDA form (alpha then holds d_k / 2 decays).
cudaError_t launch_fwd_tc(int phases, int dtype, int out_dtype, int dk, int dv, const void* q,
                          const void* k, const void* v, const float* alpha, const float* beta,
                          const float* bg, const float* wg, const float* theta, const float* S0,
                          const int32_t* cu, void* out, float* S_final, int n_seqs, int T, int H,
                          int C, void* ws, int* status, cudaStream_t stream) {
  if (!fwd_tc_supported(dtype, dk, dv, C, n_seqs, T, H, cu != nullptr))
    return cudaErrorNotSupported;
  const bool bf = out_dtype == CKDA_BF16;
  const int gk = theta != nullptr ? tc::kSfda : (bg != nullptr ? tc::kGdn2 : tc::kKda);
#define CKDA_TC_CALL(DVV, TO, G)                                                               \
  tc::launch_t<DVV, TO, G>(phases, q, k, v, alpha, beta, bg, wg, theta, S0, cu, out, S_final,   \
                           n_seqs, T, H, ws, status, stream)
#define CKDA_TC_GK(DVV, TO)                                                                    \
  (gk == tc::kSfda ? CKDA_TC_CALL(DVV, TO, tc::kSfda)                                           \
                   : (gk == tc::kGdn2 ? CKDA_TC_CALL(DVV, TO, tc::kGdn2)                        \
                                      : CKDA_TC_CALL(DVV, TO, tc::kKda)))
  if (dv == 128) return bf ? CKDA_TC_GK(128, __nv_bfloat16) : CKDA_TC_GK(128, float);
  return bf ? CKDA_TC_GK(64, __nv_bfloat16) : CKDA_TC_GK(64, float);
#undef CKDA_TC_GK
#undef CKDA_TC_CALL
}

}  // namespace ckda
