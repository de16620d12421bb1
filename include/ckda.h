/*
 * ckda.h -- C ABI of libckda.so: the Complex Kimi Delta Attention (CKDA)
 * recurrence on one NVIDIA B200 (sm_100a).
 *
 * The operation ("Complex KDA: Kimi Delta Attention Mimarisinin Ifade Gucunu
 * Anlamak ve Gelistirmek", section "Complex KDA (CKDA) Mimarisi ve Parametre
 * Genislemesi"; "Gated DeltaNet-2", Methodology section 1 with the erase and
 * write gates tied to beta_t; "Semidirect Fourier Delta Attention",
 * "Arquitectura Central" with zero phase):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with a per-channel gate alpha_t in [-1, 1]^{d_k}, a scalar delta
 * coefficient beta_t in [0, 2] per (token, head), and a d_k x d_v fp32 state
 * per (sequence, head).  The read-out uses the state after the update and no
 * query scale.  The library does not normalise q or k.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers (cudaMalloc / torch CUDA
 *    memory) on the current CUDA device, row-major and contiguous, 16-byte
 *    aligned.  The caller owns every buffer, scratch workspace included;
 *    the library allocates nothing and keeps no state between calls except
 *    one device status word.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream and returns as soon
 *    as the work is enqueued.
 *  - dtype selects the element type of q, k and v, out_dtype the element
 *    type of out: each CKDA_F32 or CKDA_BF16.  alpha, beta, S0, S_final and
 *    S_inout are always fp32.  Every output element is computed in fp32 and
 *    stored as fp32, or rounded once to bf16 (round-to-nearest-even) when
 *    out_dtype is CKDA_BF16, so a bf16 output is exactly the bf16 rounding
 *    of the fp32 output of the same call.  The state stays fp32.
 *  - Return value: CKDA_OK (0) or a negative CKDA_ERR_* code.  On an
 *    argument error nothing is launched and no memory is touched.  Errors
 *    found on the device (a bad cu_seqlens array, a bounded wait that timed
 *    out) are recorded in the device status word and reported by
 *    ckda_device_status().
 */
#ifndef CKDA_H
#define CKDA_H

#include <stddef.h>
#include <stdint.h>

/* Symbols of the C ABI are exported even when the library is compiled with
   hidden default visibility. */
#if defined(__GNUC__)
#define CKDA_API __attribute__((visibility("default")))
#else
#define CKDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  CKDA_F32 = 0,
  CKDA_BF16 = 1
};

enum {
  CKDA_OK = 0,
  CKDA_ERR_INVALID_ARG = -1,   /* NULL required pointer, negative or
                                  inconsistent sizes */
  CKDA_ERR_UNSUPPORTED = -2,   /* d_k or d_v not in {16,32,64,128}, chunk
                                  not in {0,16,32,64}, unknown dtype or
                                  out_dtype */
  CKDA_ERR_MISALIGNED = -3,    /* a pointer is not 16-byte aligned */
  CKDA_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed */
  CKDA_ERR_DEVICE_TIMEOUT = -5,/* a bounded device-side wait gave up */
  CKDA_ERR_BAD_SEQLENS = -6,   /* cu_seqlens not 0 = cu[0] <= ... <= cu[N] = T */
  CKDA_ERR_WORKSPACE = -7      /* workspace NULL, smaller than
                                  ckda_fwd_chunked_workspace_bytes(), not
                                  256-byte aligned, or overlapping a tensor */
};

/*
 * ckda_fwd_chunked -- chunkwise-parallel WY forward (prefill).
 *
 * Source of the chunk form: "Semidirect Fourier Delta Attention", sections
 * "El Teorema de Chunk-WY Constructivo" (block products as a diagonal
 * product minus a correction of rank <= chunk) and "Principales
 * Contribuciones" item 3 (exact affine block transfer between chunks);
 * "Gated DeltaNet-2", Methodology section 3 (decay absorbed into the WY
 * factors, lower-triangular solve (I + T)^-1).  The result equals the
 * token-by-token recurrence above up to rounding; the chunk size does not
 * change it.
 *
 * Fixed-length batch (cu_seqlens == NULL):
 *   q, k   [B, T, H, d_k]   (dtype)     v, out [B, T, H, d_v] (dtype)
 *   alpha  [B, T, H, d_k]   fp32        beta   [B, T, H]       fp32
 *   S0, S_final [B, H, d_k, d_v] fp32
 * Packed variable-length batch (cu_seqlens != NULL):
 *   B is the number of sequences N and T the total number of packed tokens;
 *   q, k, alpha are [T, H, d_k], v and out [T, H, d_v], beta [T, H];
 *   cu_seqlens is a DEVICE int32 array [N + 1] with cu[0] = 0,
 *   cu[n] <= cu[n+1], cu[N] = T; sequence n owns tokens [cu[n], cu[n+1]).
 *   S0 and S_final are [N, H, d_k, d_v].  The state restarts at every
 *   sequence start.  The array is validated on the device: a violation sets
 *   CKDA_ERR_BAD_SEQLENS in the status word and the affected sequences
 *   produce no output.
 *
 *   S0       may be NULL (zero initial state).
 *   S_final  may be NULL (final state not stored) and may equal S0 (each
 *            unit reads its own S0 slice before it writes the same slice).
 *   out      must not alias any input.
 *   chunk    0 (default 64), 16, 32 or 64.
 *   d_k, d_v each in {16, 32, 64, 128}.
 *   workspace, workspace_bytes
 *            device scratch owned by the caller, at least
 *            ckda_fwd_chunked_workspace_bytes() bytes for these sizes,
 *            256-byte aligned, overlapping no tensor argument; its contents
 *            on entry do not matter and on return are unspecified.  Only
 *            the tensor-core path uses it (per chunk and head: [-W; Q'],
 *            K * rho and [Inv diag(beta); P] in fp16, gamma in fp32,
 *            66,048 bytes for either d_v); when the size query returns 0
 *            both may be NULL / 0.  Calls that run concurrently (other
 *            streams) need separate workspaces; calls ordered on one stream
 *            may share one.  A workspace that is missing or too small
 *            returns CKDA_ERR_WORKSPACE and launches nothing.
 * A zero-length sequence stores S_final = S0 and writes no output rows.
 */
CKDA_API int ckda_fwd_chunked(const void* q, const void* k, const void* v,
                     const float* alpha, const float* beta, const float* S0,
                     const int32_t* cu_seqlens, void* out, float* S_final,
                     int B, int T, int H, int d_k, int d_v, int chunk,
                     int dtype, int out_dtype, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * ckda_fwd_chunked_static -- ckda_fwd_chunked without a caller workspace:
 * the tensor-core path uses a fixed scratch array that the library holds in
 * device memory (CKDA_STATIC_SCRATCH_BYTES per device, reserved when the
 * library's module is loaded).  No call allocates or frees memory.  This
 * entry point is an interface convenience of this library; the pages
 * describe no counterpart of it.
 *
 *  - Arguments, layouts and results are those of ckda_fwd_chunked; the
 *    output is bit-identical to ckda_fwd_chunked with any valid workspace.
 *  - Sizes whose workspace (ckda_fwd_chunked_workspace_bytes) exceeds
 *    CKDA_STATIC_SCRATCH_BYTES return CKDA_ERR_UNSUPPORTED and launch
 *    nothing: that is more than 1016 units of ceil(T / 64) * B * H
 *    (fixed-length) or (floor(T / 64) + N) * H (packed), e.g. B = 1,
 *    T = 2048, H = 16 fits (512 units).  Sizes on the
 *    fp32 CUDA-core path need no scratch and are always accepted.
 *  - Nothing in the scratch has to start at zero: every byte the carry
 *    kernel reads is written by the factor kernel of the same call.
 *  - The scratch is shared by every call on a device: two calls that may
 *    run at the same time (different streams, or threads without stream
 *    order) race on it and give wrong results.  Calls ordered on one stream
 *    are safe.
 *  - The first call on each device looks the scratch address up with
 *    cudaGetSymbolAddress and caches it; make that first call outside any
 *    stream capture.
 */
#define CKDA_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

CKDA_API int ckda_fwd_chunked_static(const void* q, const void* k, const void* v,
                                     const float* alpha, const float* beta,
                                     const float* S0, const int32_t* cu_seqlens,
                                     void* out, float* S_final, int B, int T, int H,
                                     int d_k, int d_v, int chunk, int dtype,
                                     int out_dtype, void* stream);

/*
 * ckda_fwd_factors, ckda_fwd_carry -- ckda_fwd_chunked in its two phases,
 * for the tensor-core path only (sizes for which ckda_fwd_chunked_path
 * returns 1; otherwise CKDA_ERR_UNSUPPORTED).
 *
 * ckda_fwd_factors reads q, k, alpha and beta (layouts as in
 * ckda_fwd_chunked; v is accepted and not read) and writes, for every chunk
 * of every head, the S0-independent WY factors into `workspace`: [-W; Q'],
 * K * rho, [Inv diag(beta); P] (fp16) and gamma (fp32).  ckda_fwd_carry
 * reads v itself and forms [U~; A U~] = [Inv diag(beta); P] V
 * ("Gated DeltaNet-2", Methodology section 3:
 * the decay absorbed into the WY factors; "Semidirect Fourier Delta
 * Attention", "Principales Contribuciones" item 3: each chunk is an affine
 * map of the state, S_end = (Diag(gamma) - (K*rho)^T W) S + (K*rho)^T U~).
 * ckda_fwd_carry applies those maps chunk after chunk from S0 and writes
 * out and S_final; it reads v (the same tensor as the factor call's, layout
 * as in ckda_fwd_chunked) and needs it non-NULL whenever there are tokens.
 *
 * Because the factors do not depend on S0, one factor call can serve
 * several carry calls with different initial states.  ckda_fwd_carry must
 * see the workspace of a completed ckda_fwd_factors call with the same B,
 * T, H, d_k, d_v, chunk, dtype and cu_seqlens (stream order or an event
 * makes it complete); the library cannot check this.  Running the two on
 * one stream equals one ckda_fwd_chunked call, bit for bit.  Arguments,
 * ownership and errors are those of ckda_fwd_chunked; out_dtype is only
 * meaningful to the carry.
 */
CKDA_API int ckda_fwd_factors(const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta,
                              const int32_t* cu_seqlens, int B, int T, int H,
                              int d_k, int d_v, int chunk, int dtype,
                              void* workspace, size_t workspace_bytes, void* stream);

CKDA_API int ckda_fwd_carry(const void* v, const float* S0, const int32_t* cu_seqlens, void* out,
                            float* S_final, int B, int T, int H, int d_k, int d_v,
                            int chunk, int dtype, int out_dtype, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * ckda_gdn2_fwd_chunked -- chunkwise forward of the Gated DeltaNet-2
 * recurrence ("Gated DeltaNet-2" technical summary, Methodology section 1):
 *
 *     S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,
 *     o_t = S_t^T q_t,
 *
 * i.e. CKDA with the scalar beta_t replaced by an erase gate b_t (per key
 * channel) and a write gate w_t (per value channel); b_t = w_t = beta_t
 * gives back ckda_fwd_chunked's recurrence.  In the chunk form T[r, s] uses
 * b_r . k_r on its row side and the WY right-hand sides are
 * [(B . K) * Gamma | W . V] (Methodology section 3).
 *
 *   b   fp32, shaped like k:  [B, T, H, d_k] (packed: [T, H, d_k])
 *   w   fp32, shaped like v:  [B, T, H, d_v] (packed: [T, H, d_v])
 * The gates are applied as given (the pages take them in [0, 1]).  Every
 * other argument, layout, ownership and error rule is that of
 * ckda_fwd_chunked, workspace included (b takes beta's place in the checks;
 * w must be non-NULL when there are tokens, 16-byte aligned and not aliased
 * by out).  The kernels are those of ckda_fwd_chunked for the same sizes
 * (ckda_fwd_chunked_path, ckda_fwd_chunked_workspace_bytes): the tcgen05
 * pair for bf16 inputs with d_k = 128, d_v in {64, 128}, chunk 64, the fp32
 * CUDA-core kernel otherwise.
 */
CKDA_API int ckda_gdn2_fwd_chunked(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* b, const float* w,
                                   const float* S0, const int32_t* cu_seqlens, void* out,
                                   float* S_final, int B, int T, int H, int d_k, int d_v,
                                   int chunk, int dtype, int out_dtype, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * ckda_sfda_fwd_chunked -- chunkwise forward of the SFDA (phase-controlled)
 * recurrence ("Semidirect Fourier Delta Attention (SFDA)" technical summary,
 * "Arquitectura Central"), in real coordinates:
 *
 *     S_t = (I - beta_t k_t k_t^T) Lambda_t S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,
 *
 * with Lambda_t block diagonal: block p (p = 0 .. d_k/2 - 1) acts on the
 * state rows (2p, 2p+1) as
 *     alpha_p * [[cos theta_p, -sin theta_p], [sin theta_p, cos theta_p]],
 * the real form of the complex gate alpha_p e^{i theta_p} on a channel whose
 * real part is row 2p and imaginary part row 2p+1.  Zero phases give back
 * ckda_fwd_chunked's recurrence with each decay on both rows of its pair; a
 * phase of pi is a negative real gate.  The chunk form is the same WY
 * factorisation with the channel-wise gate products replaced by products of
 * these complex scalars ("El Teorema de Chunk-WY Constructivo").
 *
 *   alpha  fp32 [B, T, H, d_k / 2]  (packed: [T, H, d_k / 2]) decays
 *   theta  fp32 [B, T, H, d_k / 2]  (packed: [T, H, d_k / 2]) phases, radians
 * Both are applied as given (|alpha| <= 1 keeps the transitions
 * non-expansive); cos and sin of each phase are evaluated once per token in
 * fp32.  Every other argument, layout, ownership and error rule is that of
 * ckda_fwd_chunked, workspace included: the kernels are those of
 * ckda_fwd_chunked for the same sizes (ckda_fwd_chunked_path,
 * ckda_fwd_chunked_workspace_bytes) -- the tcgen05 pair for bf16 inputs
 * with d_k = 128, d_v in {64, 128}, chunk 64, the fp32 CUDA-core kernel
 * otherwise.  theta must be non-NULL when there are tokens, 16-byte aligned
 * and not aliased by out.  The two-phase calls (ckda_fwd_factors /
 * ckda_fwd_carry) carry the real-gate form only.
 */
CKDA_API int ckda_sfda_fwd_chunked(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* theta, const float* beta,
                                   const float* S0, const int32_t* cu_seqlens, void* out,
                                   float* S_final, int B, int T, int H, int d_k, int d_v,
                                   int chunk, int dtype, int out_dtype, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * ckda_sfda_fwd_chunked_fp32core -- the same operation as
 * ckda_sfda_fwd_chunked, forced onto the fp32 CUDA-core kernel (takes no
 * workspace), as ckda_fwd_chunked_fp32core is for ckda_fwd_chunked.
 */
CKDA_API int ckda_sfda_fwd_chunked_fp32core(const void* q, const void* k, const void* v,
                                            const float* alpha, const float* theta,
                                            const float* beta, const float* S0,
                                            const int32_t* cu_seqlens, void* out,
                                            float* S_final, int B, int T, int H, int d_k,
                                            int d_v, int chunk, int dtype, int out_dtype,
                                            void* stream);

/*
 * ckda_fwd_chunked_scan -- ckda_fwd_chunked (fixed-length batches) as a
 * chunk-parallel scan over `segments` contiguous segments of each sequence's
 * chunks ("Semidirect Fourier Delta Attention", "Principales Contribuciones"
 * item 3: a block of chunks acts on its start state as the exact affine map
 * S_end = M S_start + B, with B the block's zero-start state):
 *   1. the per-chunk factors of every chunk (as ckda_fwd_chunked);
 *   2. for segments 0 .. segments - 2, all in parallel, the summary
 *      [M_g | B_g]: the carry from [I | 0] with the V term on the B columns
 *      only;
 *   3. the scan S_start(g + 1) = M_g S_start(g) + B_g (fp32, S_start(0) = S0);
 *   4. the carry of every segment from its start state, all in parallel,
 *      writing out (and S_final from the last segment).
 * The result equals ckda_fwd_chunked's up to rounding (the summaries go
 * through the same fp16 tensor-core operands as the state).  segments = 1 is
 * the plain forward.  Shapes: the tensor-core ones only (bf16 inputs,
 * d_k = 128, d_v in {64, 128}, chunk 64), cu_seqlens not supported; other
 * shapes return CKDA_ERR_UNSUPPORTED.  S_final may not alias S0 when
 * segments > 1 (segments run concurrently).  Every other argument and rule
 * is that of ckda_fwd_chunked; the workspace is
 * ckda_fwd_chunked_scan_workspace_bytes().  On B200 this does not beat the
 * plain forward at the sizes measured (the carry is latency-bound per chunk
 * and the scan triples its work); it is the single-GPU form of splitting one
 * sequence across GPUs.
 */
CKDA_API int ckda_fwd_chunked_scan(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta, const float* S0,
                                   void* out, float* S_final, int B, int T, int H, int d_k,
                                   int d_v, int chunk, int dtype, int out_dtype, int segments,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * ckda_fwd_chunked_scan_workspace_bytes -- scratch bytes of
 * ckda_fwd_chunked_scan: ckda_fwd_chunked's workspace plus
 * 4 N (segments - 1) H d_k (d_k + d_v) bytes of summaries and
 * 4 N segments H d_k d_v bytes of segment start states; or the negative
 * status a call with these sizes would return.  Pure host function.
 */
CKDA_API int64_t ckda_fwd_chunked_scan_workspace_bytes(int B, int T, int H, int d_k, int d_v,
                                                       int segments);

/*
 * ckda_fwd_chunked_workspace_bytes -- scratch bytes ckda_fwd_chunked needs
 * for these sizes (same meaning of B, T and `varlen` as in
 * ckda_fwd_chunked_path), 0 when the call runs the fp32 CUDA-core kernel,
 * or the negative status an actual call with these sizes would return.
 * Pure host function: needs no GPU.  The tensor-core path takes
 * (B * ceil(T / 64)) * H work units for a fixed-length batch and
 * (floor(T / 64) + N) * H for a packed one, each 2*64*128*2 + 64*128*2 +
 * 2*64*64*2 + 128*4 + 64*d_v*2 bytes.
 */
CKDA_API int64_t ckda_fwd_chunked_workspace_bytes(int B, int T, int H, int d_k, int d_v,
                                                  int chunk, int dtype, int out_dtype,
                                                  int varlen);

/*
 * ckda_fwd_chunked_fp32core -- the same operation and arguments as
 * ckda_fwd_chunked, forced onto the fp32 CUDA-core kernel (every product
 * and sum in fp32 FFMA, no tensor-core rounding of intermediate operands).
 * ckda_fwd_chunked itself routes here for fp32 inputs and for shapes the
 * tensor-core kernel does not cover; this entry point exists so callers (and
 * tests) can request the fp32-faithful path for bf16 inputs too.
 */
CKDA_API int ckda_fwd_chunked_fp32core(const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta,
                              const float* S0, const int32_t* cu_seqlens,
                              void* out, float* S_final, int B, int T, int H,
                              int d_k, int d_v, int chunk, int dtype,
                              int out_dtype, void* stream);

/*
 * ckda_fwd_chunked_path -- which kernel ckda_fwd_chunked runs for these
 * parameters, without launching anything: 1 = the tcgen05 tensor-core
 * kernels (bf16 inputs, d_k = 128, d_v in {64, 128}, chunk 64; fp16 operands
 * with fp32 accumulation; a per-chunk factor kernel over all chunks in
 * parallel, then a carry kernel per sequence, head and 64 (or 32) columns
 * of d_v),
 * 0 = the fp32 CUDA-core kernel, or the negative
 * status an actual call with these sizes would return.  `varlen` is nonzero
 * for a packed batch (cu_seqlens given); B and T have the same meaning as in
 * ckda_fwd_chunked.  Pure host function: needs no GPU.
 */
CKDA_API int ckda_fwd_chunked_path(int B, int T, int H, int d_k, int d_v, int chunk, int dtype,
                                   int out_dtype, int varlen);

/*
 * ckda_bwd_chunked -- backward of ckda_fwd_chunked: the gradient of a
 * scalar loss L with respect to q, k, v, alpha, beta and S0, given
 * dO = dL/dout and dS_final = dL/dS_final.  It is the adjoint of the
 * recurrence token by token, in reverse (the chain rule through
 *   S' = Diag(alpha_t) S_{t-1},  r = S'^T k_t,  u = beta_t (v_t - r),
 *   S_t = S' + k_t u^T,  o_t = S_t^T q_t;
 * "Complex KDA ...", section "Complex KDA (CKDA) Mimarisi ve Parametre
 * Genislemesi"; "Gated DeltaNet-2", Methodology section 1 with b = w =
 * beta; the gate-aware backward of "Gated DeltaNet-2", Methodology section
 * 3, names the per-channel gates entering the gradient directly but prints
 * no formula).  This is the exact gradient of the forward above, computed
 * token by token in fp32 on CUDA cores with the states recomputed from a
 * checkpoint at every 16th token -- no division, so zero and negative gates
 * are exact.
 *
 *   q, k, v, alpha, beta, S0, cu_seqlens, B, T, H, d_k, d_v, dtype:
 *            the forward's inputs, layouts and rules (ckda_fwd_chunked).
 *   dO       shaped like out, element type grad_dtype (CKDA_F32 or
 *            CKDA_BF16); required when there are tokens.
 *   dS_final [N, H, d_k, d_v] fp32, may be NULL (zero).
 *   dq, dk, dalpha [.., H, d_k] fp32;  dv [.., H, d_v] fp32;
 *   dbeta [.., H] fp32 -- shaped like q, k, alpha, v, beta; every element
 *            written; required when there are tokens.
 *   dS0      [N, H, d_k, d_v] fp32, may be NULL (not stored).  A
 *            zero-length sequence gets dS0 = dS_final.
 *   workspace, workspace_bytes
 *            device scratch of at least ckda_bwd_chunked_workspace_bytes()
 *            bytes, 256-byte aligned, overlapping no tensor argument; its
 *            contents on entry do not matter.
 * Gradients are overwritten, not accumulated.  No output may alias an
 * input; every pointer must be 16-byte aligned.  Errors as for
 * ckda_fwd_chunked (CKDA_ERR_WORKSPACE for a missing or small workspace).
 * Each (sequence, head) runs as one thread-block cluster of d_v / 32 CTAs
 * (d_v = 16: one CTA); within a CTA each warp owns 4 state columns.
 */
CKDA_API int ckda_bwd_chunked(const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta, const float* S0,
                              const int32_t* cu_seqlens, const void* dO,
                              const float* dS_final, float* dq, float* dk, float* dv,
                              float* dalpha, float* dbeta, float* dS0, int B, int T, int H,
                              int d_k, int d_v, int dtype, int grad_dtype, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * ckda_bwd_chunked_workspace_bytes -- scratch bytes ckda_bwd_chunked needs
 * (B, T and `varlen` as in ckda_fwd_chunked_path), or the negative status
 * an actual call with these sizes would return.  Pure host function: one
 * stored state of 4 max(d_k, 32) d_v bytes per 16-token segment slot and
 * head (B ceil(T / 16) slots for a fixed-length batch, floor(T / 16) + N
 * packed) plus 17 such states per sequence and head (the states of one
 * segment).
 */
CKDA_API int64_t ckda_bwd_chunked_workspace_bytes(int B, int T, int H, int d_k, int d_v,
                                                  int varlen);

/*
 * ckda_decode_step -- one recurrent token for B independent sequences,
 * in place on the state ("Complex KDA ...", section "Yazilim Gelistirme
 * Acisindan Pratik Cikarimlar": O(1) inference state).
 *   q, k, alpha [B, H, d_k]    v, out [B, H, d_v]    beta [B, H]
 *   S_inout     [B, H, d_k, d_v] fp32, read once and overwritten once.
 * No pointer may alias another, except that nothing else aliases S_inout.
 */
CKDA_API int ckda_decode_step(const void* q, const void* k, const void* v,
                     const float* alpha, const float* beta, float* S_inout,
                     void* out, int B, int H, int d_k, int d_v, int dtype,
                     int out_dtype, void* stream);

/*
 * ckda_gdn2_decode_step -- one recurrent token of the Gated DeltaNet-2
 * recurrence ("Gated DeltaNet-2", Methodology section 1), in place on the
 * state: S' = Diag(alpha) S, u = w . v - S'^T (b . k), S = S' + k u^T,
 * o = S^T q.  b [B, H, d_k] and w [B, H, d_v] fp32 take beta's place; every
 * other argument and rule is that of ckda_decode_step.
 */
CKDA_API int ckda_gdn2_decode_step(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* b, const float* w,
                                   float* S_inout, void* out, int B, int H, int d_k, int d_v,
                                   int dtype, int out_dtype, void* stream);

/*
 * ckda_sfda_decode_step -- one recurrent token of the SFDA recurrence
 * ("Semidirect Fourier Delta Attention (SFDA)", "Arquitectura Central"), in
 * place on the state: the gate of ckda_sfda_fwd_chunked (row pairs
 * (2p, 2p+1) turned by alpha_p (cos theta_p, sin theta_p)), then the delta
 * update with beta.  alpha and theta are fp32 [B, H, d_k / 2]; every other
 * argument and rule is that of ckda_decode_step.
 */
CKDA_API int ckda_sfda_decode_step(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* theta, const float* beta,
                                   float* S_inout, void* out, int B, int H, int d_k, int d_v,
                                   int dtype, int out_dtype, void* stream);

/* Human-readable text for a CKDA_* status code (static storage). */
CKDA_API const char* ckda_status_string(int status);

/*
 * ckda_device_status -- synchronise `stream`, then read and clear the
 * status word of the current device.  Returns CKDA_OK, the first device
 * error recorded since the last call (CKDA_ERR_BAD_SEQLENS,
 * CKDA_ERR_DEVICE_TIMEOUT), or CKDA_ERR_CUDA if the synchronisation itself
 * failed.
 */
CKDA_API int ckda_device_status(void* stream);

/*
 * ckda_selftest_bounded_wait -- exercise the device-side time-out path.
 * Launches one thread that waits, with the bounded wait every tensor-core
 * kernel uses, on an mbarrier nothing completes; after about `limit_us`
 * microseconds (1 .. 10,000,000) the wait gives up and records
 * CKDA_ERR_DEVICE_TIMEOUT in the status word, which ckda_device_status()
 * then returns.  Faults nothing and leaves the context usable.  Returns
 * CKDA_OK once launched, CKDA_ERR_INVALID_ARG for a limit out of range.
 */
CKDA_API int ckda_selftest_bounded_wait(int limit_us, void* stream);

/* Library ABI version (major * 100 + minor). */
CKDA_API int ckda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CKDA_H */
