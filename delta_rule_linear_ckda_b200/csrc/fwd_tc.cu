// Tensor-core (tcgen05) chunked forward for bf16 inputs.
#include "common.cuh"

namespace ckda {

cudaError_t launch_fwd_tc(int dtype, int out_dtype, int dk, int dv, const void* q, const void* k, const void* v,
                          const float* alpha, const float* beta, const float* S0,
                          const int32_t* cu, void* out, float* S_final, int n_seqs, int T, int H,
                          int C, int* status, cudaStream_t stream) {
  (void)dtype; (void)out_dtype; (void)dk; (void)dv; (void)q; (void)k; (void)v; (void)alpha; (void)beta; (void)S0;
  (void)cu; (void)out; (void)S_final; (void)n_seqs; (void)T; (void)H; (void)C; (void)status;
  (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace ckda
