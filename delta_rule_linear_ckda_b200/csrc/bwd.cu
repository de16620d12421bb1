// Backward of the CKDA forward on fp32 CUDA cores (sm_100a): the gradient of
// a scalar loss with respect to q, k, v, alpha, beta and S0, given dL/do_t
// and dL/dS_final.
//
// The "Gated DeltaNet-2" page, Methodology section 3 (gate-aware backward),
// asks that the per-channel gates enter the gradient directly; here the gate
// gradient is dalpha = rowsum(dS' . S_prev) per token.  Per token the
// forward is (the CKDA recurrence, "Complex KDA ..." page, section "Complex
// KDA (CKDA) Mimarisi ve Parametre Genislemesi"; "Gated DeltaNet-2" page,
// Methodology section 1 with b = w = beta):
//   S' = Diag(a) S_prev,  r = S'^T k,  u = b (v - r),  S = S' + k u^T,  o = S^T q
// and its adjoint, walked in reverse with dS = dL/dS (after the token):
//   dq = S do;  dS += q do^T;  du = dS^T k;  dk = dS u + S' dr;
//   dbeta = du . (v - r);  dv = b du;  dr = -b du;  dS' = dS + k dr^T;
//   dalpha = rowsum(dS' . S_prev);  dS <- Diag(a) dS'
// with dS0 the final dS.  Every step needs the state before the token, so
// the states are recomputed: a first forward pass stores the state at every
// 16th token (workspace), and the reverse pass re-runs each 16-token segment
// from its checkpoint, storing its 17 states (workspace, L2-resident), before
// walking it backwards.  No division: zero and negative gates are exact.
//
// One CTA owns one (sequence, head, d_v slice of BV <= 32 columns) and each
// of its warps 4 columns of the slice over all d_k rows (lane l holds rows
// l * RPL .. + RPL): the recurrence never mixes columns, so every token step
// is warp-local (shuffles, no block barrier).  Only dq, dk, dalpha and dbeta
// sum over all d_v: per token the warps' partial sums meet in shared memory
// (one barrier), and the slices of one (sequence, head) form a thread-block
// cluster whose CTAs add up a segment's partial sums across the cluster
// (distributed shared memory) after a cluster barrier and store the totals.
// Recomputed states live in the workspace (L2-resident), each thread's part
// contiguous.
#include <cooperative_groups.h>

#include "common.cuh"

namespace ckda {
namespace bwd {

namespace cg = cooperative_groups;

constexpr int kC = 16;  // checkpoint interval of the first pass = segment (tokens)
constexpr int kG = 4;   // tokens per staged input block
constexpr int kNB = kC / kG;

template <int DK, int BV>
struct Cfg {
  static constexpr int NW = BV / 4;                 // warps: 4 columns each
  static constexpr int NT = 32 * NW;
  static constexpr int RPL = DK >= 32 ? DK / 32 : 1;  // state rows per lane
  static constexpr int E = RPL * 4;                 // state elements per thread
  static constexpr int TS = NT * E;                 // floats of one stored state (d_k = 16: twice d_k x BV)
  static constexpr int PW = 3 * DK + 1;             // partial sums per token: dq, dk, dalpha, dbeta
  // shared memory, in floats
  static constexpr int kWp = 0;                     // [2][NW][PW] the warps' partial sums of a token
  static constexpr int kPbuf = kWp + 2 * NW * PW;   // [2][kC][PW] the CTA's partial sums of a segment
  static constexpr int kR = kPbuf + 2 * kC * PW;    // [kC][BV] r of each token of the segment
  static constexpr int kU = kR + kC * BV;           // [kC][BV] u of each token of the segment
  static constexpr int kFloats = kU + kC * BV;
};

// Inputs of one block of kG tokens, staged in shared memory by cp.async
// (two buffers: the next block streams in while this one is used).  Byte
// offsets within one buffer; every array starts on a 16-byte boundary.
template <int DK, int BV, typename Tin, typename Tg>
struct Stage {
  static constexpr int K = 0;                                   // k   [kG][DK]  Tin
  static constexpr int A = K + kG * DK * (int)sizeof(Tin);      // alpha [kG][DK] fp32
  static constexpr int Q = A + kG * DK * 4;                     // q   [kG][DK]  Tin
  static constexpr int V = Q + kG * DK * (int)sizeof(Tin);      // v   [kG][BV]  Tin
  static constexpr int D = V + kG * BV * (int)sizeof(Tin);      // dO  [kG][BV]  Tg
  static constexpr int B = D + kG * BV * (int)sizeof(Tg);       // beta [kG]     fp32
  static constexpr int kBytes = B + 16 * ((kG * 4 + 15) / 16);
  // total dynamic shared memory of the kernel
  static constexpr size_t kSmem = sizeof(float) * Cfg<DK, BV>::kFloats + 2 * kBytes;
  static_assert((sizeof(float) * Cfg<DK, BV>::kFloats) % 16 == 0, "stage alignment");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The order in which the kernel consumes blocks of (up to) kG tokens:
//   kind 0  first pass, segment c (< nck - 1), block g of kNB (forward)
//   kind 1  second pass, segment c, block g ascending (recompute the states)
//   kind 2  second pass, segment c, block g descending (backward)
// Segments of the second pass run from nck - 1 down to 0.
struct Blk {
  int kind;  // -1: none left
  int c;
  int g;
};

struct Sched {
  int Ls, nck;
  __device__ int lc(int c) const { return min(kC, Ls - c * kC); }
  __device__ int nb(int c) const { return (lc(c) + kG - 1) / kG; }
  __device__ Blk pass2(int c) const { return c < 0 ? Blk{-1, 0, 0} : Blk{1, c, 0}; }
  __device__ Blk first() const { return nck >= 2 ? Blk{0, 0, 0} : pass2(nck - 1); }
  __device__ Blk next(Blk b) const {
    if (b.kind == 0) {
      if (b.g + 1 < kNB) return Blk{0, b.c, b.g + 1};
      if (b.c + 1 < nck - 1) return Blk{0, b.c + 1, 0};
      return pass2(nck - 1);
    }
    if (b.kind == 1) {
      if (b.g + 1 < nb(b.c)) return Blk{1, b.c, b.g + 1};
      return Blk{2, b.c, nb(b.c) - 1};
    }
    if (b.g > 0) return Blk{2, b.c, b.g - 1};
    return pass2(b.c - 1);
  }
  // tokens of a block (relative to the sequence start)
  __device__ int t0(Blk b) const { return b.c * kC + b.g * kG; }
  __device__ int nt(Blk b) const { return b.kind == 0 ? kG : min(kG, lc(b.c) - b.g * kG); }
};

// Column sums of a warp's 4 columns over all rows: p[c] holds this lane's
// share of column c; afterwards every lane holds the 4 totals in x[0..3]
// (a reduce-scatter over the lanes, then a broadcast).
__device__ __forceinline__ void col4_sums(const float* p, float* x, int lane) {
  float a[2];
  {
    const bool up = (lane & 16) != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = up ? p[i] : p[i + 2];
      const float keep = up ? p[i + 2] : p[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
  }
  float t;
  {
    const bool up = (lane & 8) != 0;
    const float send = up ? a[0] : a[1];
    const float keep = up ? a[1] : a[0];
    t = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  t += __shfl_xor_sync(0xffffffffu, t, 4);
  t += __shfl_xor_sync(0xffffffffu, t, 2);
  t += __shfl_xor_sync(0xffffffffu, t, 1);
  // lane holds column 2 * bit4 + bit3; fetch each column from a lane holding it
#pragma unroll
  for (int c = 0; c < 4; ++c) x[c] = __shfl_sync(0xffffffffu, t, ((c >> 1) << 4) | ((c & 1) << 3));
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p) {
  return Elem<T>::to_f32(*p);
}

// RPL consecutive values of type T from shared memory, widened to fp32
// (one vector load when RPL is 2 or 4; p is aligned to RPL elements).
template <int RPL, typename T>
__device__ __forceinline__ void lds_rows(const T* p, float* x) {
  if constexpr (RPL == 4 && sizeof(T) == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else if constexpr (RPL == 4 && sizeof(T) == 2) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else if constexpr (RPL == 2 && sizeof(T) == 4) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    x[0] = a.x; x[1] = a.y;
  } else if constexpr (RPL == 2 && sizeof(T) == 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    x[0] = a.x; x[1] = a.y;
  } else {
#pragma unroll
    for (int r = 0; r < RPL; ++r) x[r] = Elem<T>::to_f32(p[r]);
  }
}

template <int DK, int BV, typename Tin, typename Tg>
__global__ void __launch_bounds__(BV * 8, 2)
bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
           const float* __restrict__ alpha, const float* __restrict__ beta, const float* S0,
           const int32_t* __restrict__ cu, const Tg* __restrict__ dO,
           const float* __restrict__ dSf, float* __restrict__ dq, float* __restrict__ dk,
           float* __restrict__ dv, float* __restrict__ dalpha, float* __restrict__ dbeta,
           float* dS0, float* __restrict__ ws_ck, float* __restrict__ ws_sub, int n_seqs, int T,
           int H, int DV, int nch_fixed, int* status) {
  using L = Cfg<DK, BV>;
  using SG = Stage<DK, BV, Tin, Tg>;
  constexpr int RPL = L::RPL, E = L::E, PW = L::PW, NT = L::NT;
  extern __shared__ __align__(16) float smem[];
  float* wp = smem + L::kWp;
  float* pbuf = smem + L::kPbuf;
  float* rr = smem + L::kR;
  float* uu = smem + L::kU;
  uint8_t* stage0 = reinterpret_cast<uint8_t*>(smem + L::kFloats);

  cg::cluster_group cluster = cg::this_cluster();
  const int nsl = (int)cluster.num_blocks();
  const int srank = (int)cluster.block_rank();

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int r0 = lane * RPL;              // first state row of this lane
  const bool act = r0 < DK;               // (d_k = 16: lanes 16..31 hold no row)
  const int c0 = 4 * warp;                // first column of this warp within the slice
  const int j0 = blockIdx.x * BV;
  const int h = blockIdx.y;
  const int n = blockIdx.z;

  // the same for every CTA of the cluster (same sequence): all of them leave
  // here together or none does
  const SeqRange sr = seq_range(cu, n, n_seqs, T, status);
  if (!sr.ok) return;
  const int64_t L0 = sr.begin;
  const Sched sch{(int)(sr.end - sr.begin), (int)((sr.end - sr.begin + kC - 1) / kC)};
  const int nck = sch.nck;

  // workspace: every stored state keeps each thread's E values contiguous.
  // Checkpoints are indexed by 16-token segment slot (numbered as the
  // forward numbers its chunks: a packed sequence n starts at slot
  // floor(cu[n] / kC) + n); the kC + 1 states of the segment being walked sit
  // in a per-(sequence, head, slice) area.
  const int64_t slot0 = (cu != nullptr) ? (int64_t)(sr.begin / kC) + n : (int64_t)n * nch_fixed;
  const size_t tile = (size_t)L::TS;
  auto ck_ptr = [&](int c) -> float* {
    return ws_ck + (((size_t)(slot0 + c) * H + h) * nsl + srank) * tile + (size_t)tid * E;
  };
  float* area = ws_sub + (((size_t)n * H + h) * nsl + srank) * (kC + 1) * tile;
  auto st_ptr = [&](int m) -> float* { return area + (size_t)m * tile + (size_t)tid * E; };

  auto ld_st = [](const float* p, float* x) {
#pragma unroll
    for (int c = 0; c < E; c += 4) {
      const float4 a = *reinterpret_cast<const float4*>(p + c);
      x[c] = a.x; x[c + 1] = a.y; x[c + 2] = a.z; x[c + 3] = a.w;
    }
  };
  auto st_st = [](float* p, const float* x) {
#pragma unroll
    for (int c = 0; c < E; c += 4)
      *reinterpret_cast<float4*>(p + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
  };
  // this thread's part of a [DK, DV] fp32 state tensor: rows r0.., columns j0 + c0..
  auto ld_glob = [&](const float* base, float* x) {
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      if (act) a = *reinterpret_cast<const float4*>(base + (size_t)(r0 + r) * DV + j0 + c0);
      x[4 * r] = a.x; x[4 * r + 1] = a.y; x[4 * r + 2] = a.z; x[4 * r + 3] = a.w;
    }
  };

  // Stage the inputs of block b into buffer `sbuf` (k, alpha, v, beta; plus
  // q and dO for the backward segments), as one cp.async group.
  auto issue = [&](Blk b, int sbuf) {
    if (b.kind < 0) return;
    uint8_t* sg = stage0 + sbuf * SG::kBytes;
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(sg);
    const int64_t t0 = L0 + sch.t0(b);
    const int nt = sch.nt(b);
    const bool full = b.kind == 2;
    constexpr int KC = DK * (int)sizeof(Tin) / 16;  // 16-byte chunks per k / q row
    constexpr int AC = DK * 4 / 16;
    constexpr int VC = BV * (int)sizeof(Tin) / 16;
    constexpr int DC = BV * (int)sizeof(Tg) / 16;
    for (int e = tid; e < nt * KC; e += NT) {
      const int m = e / KC, x = e % KC;
      const size_t ti = (size_t)(t0 + m) * H + h;
      cp_async16(base + SG::K + (m * KC + x) * 16, reinterpret_cast<const uint8_t*>(k + ti * DK) + 16 * x);
      if (full)
        cp_async16(base + SG::Q + (m * KC + x) * 16, reinterpret_cast<const uint8_t*>(q + ti * DK) + 16 * x);
    }
    for (int e = tid; e < nt * AC; e += NT) {
      const int m = e / AC, x = e % AC;
      const size_t ti = (size_t)(t0 + m) * H + h;
      cp_async16(base + SG::A + (m * AC + x) * 16, reinterpret_cast<const uint8_t*>(alpha + ti * DK) + 16 * x);
    }
    for (int e = tid; e < nt * VC; e += NT) {
      const int m = e / VC, x = e % VC;
      const size_t ti = (size_t)(t0 + m) * H + h;
      cp_async16(base + SG::V + (m * VC + x) * 16, reinterpret_cast<const uint8_t*>(v + ti * DV + j0) + 16 * x);
    }
    if (full) {
      for (int e = tid; e < nt * DC; e += NT) {
        const int m = e / DC, x = e % DC;
        const size_t ti = (size_t)(t0 + m) * H + h;
        cp_async16(base + SG::D + (m * DC + x) * 16, reinterpret_cast<const uint8_t*>(dO + ti * DV + j0) + 16 * x);
      }
    }
    if (tid < nt) cp_async4(base + SG::B + 4 * tid, beta + ((size_t)(t0 + tid) * H + h));
    cp_async_commit();
  };

  // the 4 values of this warp's columns of token m, widened to fp32
  auto cols4 = [&](const uint8_t* sg, int off, bool grad, int m, float* x) {
    if (grad)
      lds_rows<4>(reinterpret_cast<const Tg*>(sg + off) + m * BV + c0, x);
    else
      lds_rows<4>(reinterpret_cast<const Tin*>(sg + off) + m * BV + c0, x);
  };
  auto rows = [&](const uint8_t* sg, int off, int m, float* x, bool f32) {
    if (!act) {
#pragma unroll
      for (int r = 0; r < RPL; ++r) x[r] = 0.f;
    } else if (f32) {
      lds_rows<RPL>(reinterpret_cast<const float*>(sg + off) + m * DK + r0, x);
    } else {
      lds_rows<RPL>(reinterpret_cast<const Tin*>(sg + off) + m * DK + r0, x);
    }
  };

  // One forward token step on this thread's block S (RPL rows x 4 columns),
  // token m of the staged block `sg`; r and u of the token go to slot
  // `slot` of the segment arrays when slot >= 0.
  auto fwd_step = [&](float* S, const uint8_t* sg, int m, int slot) {
    float a[RPL], kk[RPL];
    rows(sg, SG::A, m, a, true);
    rows(sg, SG::K, m, kk, false);
    float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        S[4 * r + c] *= a[r];
        p[c] = fmaf(S[4 * r + c], kk[r], p[c]);
      }
    float rv[4], vv[4], u[4];
    col4_sums(p, rv, lane);
    cols4(sg, SG::V, false, m, vv);
    const float bt = reinterpret_cast<const float*>(sg + SG::B)[m];
#pragma unroll
    for (int c = 0; c < 4; ++c) u[c] = bt * (vv[c] - rv[c]);
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) S[4 * r + c] = fmaf(kk[r], u[c], S[4 * r + c]);
    if (slot >= 0 && lane == 0) {
      *reinterpret_cast<float4*>(rr + slot * BV + c0) = make_float4(rv[0], rv[1], rv[2], rv[3]);
      *reinterpret_cast<float4*>(uu + slot * BV + c0) = make_float4(u[0], u[1], u[2], u[3]);
    }
  };

  float S[E];
  float dS[E];
  float Sc[E];  // the state after the token the backward walk is at
  if (S0 != nullptr) {
    ld_glob(S0 + ((size_t)n * H + h) * DK * DV, S);
  } else {
#pragma unroll
    for (int c = 0; c < E; ++c) S[c] = 0.f;
  }
  if (dSf != nullptr) {
    ld_glob(dSf + ((size_t)n * H + h) * DK * DV, dS);
  } else {
#pragma unroll
    for (int c = 0; c < E; ++c) dS[c] = 0.f;
  }

  int buf = 0, sbuf = 0, wbuf = 0;
  Blk b = sch.first();
  issue(b, 0);
  for (; b.kind >= 0;) {
    const Blk nx = sch.next(b);
    cp_async_wait_all();
    __syncthreads();      // block b is staged; every thread is done with the other buffer
    issue(nx, sbuf ^ 1);  // the next block streams in meanwhile
    const uint8_t* sg = stage0 + sbuf * SG::kBytes;
    if (b.kind == 0) {
      // ---- first pass: the state at the start of every segment ------------------
      if (b.g == 0) st_st(ck_ptr(b.c), S);
      for (int m = 0; m < kG; ++m) fwd_step(S, sg, m, -1);
    } else if (b.kind == 1) {
      // ---- second pass, segment b.c: recompute its states (the last segment's
      // start state is S already)
      if (b.g == 0) {
        if (b.c != nck - 1) ld_st(ck_ptr(b.c), S);
        st_st(st_ptr(0), S);
      }
      const int nt = sch.nt(b);
      for (int m = 0; m < nt; ++m) {
        const int j = b.g * kG + m;
        fwd_step(S, sg, m, j);
        st_st(st_ptr(j + 1), S);
      }
      if (b.g == sch.nb(b.c) - 1) {
        __syncwarp();
#pragma unroll
        for (int c = 0; c < E; ++c) Sc[c] = S[c];  // the state after the segment's last token
      }
    } else {
      // ---- second pass, segment b.c: walk block b.g backwards -------------------
      const int64_t ts = L0 + sch.t0(b);
      const int Lg = sch.nt(b);
      float* pb = pbuf + buf * kC * PW;
      for (int m = Lg - 1; m >= 0; --m) {
        const int j = b.g * kG + m;  // token index within the segment
        const size_t ti = (size_t)(ts + m) * H + h;
        float qv[RPL], kv[RPL], av[RPL], go[4], vv[4];
        rows(sg, SG::Q, m, qv, false);
        rows(sg, SG::K, m, kv, false);
        rows(sg, SG::A, m, av, true);
        cols4(sg, SG::D, true, m, go);
        cols4(sg, SG::V, false, m, vv);
        const float bt = reinterpret_cast<const float*>(sg + SG::B)[m];
        const float4 r4 = *reinterpret_cast<const float4*>(rr + j * BV + c0);
        const float4 u4 = *reinterpret_cast<const float4*>(uu + j * BV + c0);
        const float rv[4] = {r4.x, r4.y, r4.z, r4.w};
        const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
        float Sp[E];
        ld_st(st_ptr(j), Sp);
        // o = S^T q: dq (this warp's columns) and dS += q dO^T
        float dqp[RPL], p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
          dqp[r] = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            dqp[r] = fmaf(Sc[4 * r + c], go[c], dqp[r]);
            dS[4 * r + c] = fmaf(qv[r], go[c], dS[4 * r + c]);
            p[c] = fmaf(dS[4 * r + c], kv[r], p[c]);
          }
        }
        // S = S' + k u^T: du = dS^T k
        float du[4];
        col4_sums(p, du, lane);
        float dbp = 0.f, dr[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          dbp = fmaf(du[c], vv[c] - rv[c], dbp);
          dr[c] = -bt * du[c];
        }
        if (lane < 4) {
          const float d1 = (lane & 1) ? du[1] : du[0], d3 = (lane & 1) ? du[3] : du[2];
          dv[ti * DV + j0 + c0 + lane] = bt * ((lane & 2) ? d3 : d1);
        }
        float dkp[RPL], dap[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
          float x = 0.f, y = 0.f, z = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            x = fmaf(dS[4 * r + c], uv[c], x);
            y = fmaf(Sp[4 * r + c], dr[c], y);
            const float dsp = fmaf(kv[r], dr[c], dS[4 * r + c]);  // dS' = dS + k dr^T
            z = fmaf(dsp, Sp[4 * r + c], z);
            dS[4 * r + c] = av[r] * dsp;
          }
          dkp[r] = fmaf(av[r], y, x);  // dS u + S' dr, S' = Diag(a) S_prev
          dap[r] = z;
        }
        // the warps' partial sums meet in shared memory
        float* w = wp + wbuf * L::NW * PW + warp * PW;
        if (act) {
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
            w[r0 + r] = dqp[r];
            w[DK + r0 + r] = dkp[r];
            w[2 * DK + r0 + r] = dap[r];
          }
        }
        if (lane == 0) w[3 * DK] = dbp;
        __syncthreads();
        for (int e = tid; e < PW; e += NT) {
          float sum = 0.f;
#pragma unroll
          for (int ww = 0; ww < L::NW; ++ww) sum += wp[wbuf * L::NW * PW + ww * PW + e];
          pb[j * PW + e] = sum;
        }
        wbuf ^= 1;
#pragma unroll
        for (int c = 0; c < E; ++c) Sc[c] = Sp[c];
      }
      if (b.g == 0) {
        // the slices' partial sums of this segment: add across the cluster
        const int64_t tseg = L0 + (int64_t)b.c * kC;
        const int Lc = sch.lc(b.c);
        cluster.sync();
        const int EE = Lc * PW;
        const int e0 = (int)((int64_t)EE * srank / nsl), e1 = (int)((int64_t)EE * (srank + 1) / nsl);
        for (int e = e0 + tid; e < e1; e += NT) {
          float sum = 0.f;
          for (int r = 0; r < nsl; ++r) sum += cluster.map_shared_rank(pb, r)[e];
          const int m = e / PW, w = e % PW;
          const size_t ti = (size_t)(tseg + m) * H + h;
          if (w < DK)
            dq[ti * DK + w] = sum;
          else if (w < 2 * DK)
            dk[ti * DK + (w - DK)] = sum;
          else if (w < 3 * DK)
            dalpha[ti * DK + (w - 2 * DK)] = sum;
          else
            dbeta[ti] = sum;
        }
        buf ^= 1;
      }
    }
    b = nx;
    sbuf ^= 1;
  }
  if (dS0 != nullptr && act) {
    float* base = dS0 + ((size_t)n * H + h) * DK * DV;
#pragma unroll
    for (int r = 0; r < RPL; ++r)
      *reinterpret_cast<float4*>(base + (size_t)(r0 + r) * DV + j0 + c0) =
          make_float4(dS[4 * r], dS[4 * r + 1], dS[4 * r + 2], dS[4 * r + 3]);
  }
  // no CTA leaves while another may still read its partial sums
  cluster.sync();
}

template <int DK, int BV, typename Tin, typename Tg>
static cudaError_t launch_t(const void* q, const void* k, const void* v, const float* alpha,
                            const float* beta, const float* S0, const int32_t* cu, const void* dO,
                            const float* dSf, float* dq, float* dk, float* dv, float* dalpha,
                            float* dbeta, float* dS0, float* ws_ck, float* ws_sub, int n_seqs,
                            int T, int H, int DV, int* status, cudaStream_t stream) {
  using L = Cfg<DK, BV>;
  using SG = Stage<DK, BV, Tin, Tg>;
  auto kern = bwd_kernel<DK, BV, Tin, Tg>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SG::kSmem);
  if (e != cudaSuccess) return e;
  const int nsl = DV / BV;
  const int nch_fixed = (T + kC - 1) / kC;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsl, H, n_seqs);
  cfg.blockDim = dim3(L::NT, 1, 1);
  static_assert(L::NT == BV * 8, "launch bounds");
  cfg.dynamicSmemBytes = SG::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nsl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const Tin*>(q), static_cast<const Tin*>(k),
                            static_cast<const Tin*>(v), alpha, beta, S0, cu,
                            static_cast<const Tg*>(dO), dSf, dq, dk, dv, dalpha, dbeta, dS0,
                            ws_ck, ws_sub, n_seqs, T, H, DV, nch_fixed, status);
}

template <int DK, typename Tin, typename Tg>
static cudaError_t launch_dk(int dv_, const void* q, const void* k, const void* v,
                             const float* alpha, const float* beta, const float* S0,
                             const int32_t* cu, const void* dO, const float* dSf, float* dq,
                             float* dk, float* dv, float* dalpha, float* dbeta, float* dS0,
                             float* ws_ck, float* ws_sub, int n_seqs, int T, int H, int* status,
                             cudaStream_t stream) {
  if (dv_ == 16)
    return launch_t<DK, 16, Tin, Tg>(q, k, v, alpha, beta, S0, cu, dO, dSf, dq, dk, dv, dalpha,
                                     dbeta, dS0, ws_ck, ws_sub, n_seqs, T, H, dv_, status, stream);
  return launch_t<DK, 32, Tin, Tg>(q, k, v, alpha, beta, S0, cu, dO, dSf, dq, dk, dv, dalpha,
                                   dbeta, dS0, ws_ck, ws_sub, n_seqs, T, H, dv_, status, stream);
}

}  // namespace bwd

// Workspace of the backward: the checkpoints (one d_k x d_v fp32 state per
// 16-token segment slot and head) and, per sequence and head, the kC + 1
// states of a segment.
size_t bwd_workspace_bytes(int dk, int dv, int n_seqs, int T, int H, bool varlen) {
  const int64_t nch = ((int64_t)T + bwd::kC - 1) / bwd::kC;
  const int64_t slots = varlen ? (int64_t)T / bwd::kC + n_seqs : (int64_t)n_seqs * nch;
  // a stored state keeps each thread's values contiguous: max(d_k, 32) x d_v floats
  const size_t tile = (size_t)(dk > 32 ? dk : 32) * dv * sizeof(float);
  return (size_t)slots * H * tile + (size_t)n_seqs * H * (bwd::kC + 1) * tile;
}

cudaError_t launch_bwd(int dtype, int grad_dtype, int dk_, int dv_, const void* q, const void* k,
                       const void* v, const float* alpha, const float* beta, const float* S0,
                       const int32_t* cu, const void* dO, const float* dSf, float* dq, float* dk,
                       float* dv, float* dalpha, float* dbeta, float* dS0, void* ws, int n_seqs,
                       int T, int H, int* status, cudaStream_t stream) {
  const int64_t nch = ((int64_t)T + bwd::kC - 1) / bwd::kC;
  const int64_t slots = cu ? (int64_t)T / bwd::kC + n_seqs : (int64_t)n_seqs * nch;
  float* ws_ck = static_cast<float*>(ws);
  float* ws_sub = ws_ck + (size_t)slots * H * (dk_ > 32 ? dk_ : 32) * dv_;
#define CKDA_BWD_CALL(DKV, TI, TG)                                                             \
  bwd::launch_dk<DKV, TI, TG>(dv_, q, k, v, alpha, beta, S0, cu, dO, dSf, dq, dk, dv, dalpha, \
                              dbeta, dS0, ws_ck, ws_sub, n_seqs, T, H, status, stream)
#define CKDA_BWD_DK(DKV)                                                               \
  case DKV:                                                                            \
    if (dtype == CKDA_BF16)                                                            \
      return grad_dtype == CKDA_BF16 ? CKDA_BWD_CALL(DKV, __nv_bfloat16, __nv_bfloat16) \
                                     : CKDA_BWD_CALL(DKV, __nv_bfloat16, float);       \
    return grad_dtype == CKDA_BF16 ? CKDA_BWD_CALL(DKV, float, __nv_bfloat16)          \
                                   : CKDA_BWD_CALL(DKV, float, float);
  switch (dk_) {
    CKDA_BWD_DK(16)
    CKDA_BWD_DK(32)
    CKDA_BWD_DK(64)
    CKDA_BWD_DK(128)
  }
#undef CKDA_BWD_DK
#undef CKDA_BWD_CALL
  return cudaErrorInvalidValue;
}

}  // namespace ckda
