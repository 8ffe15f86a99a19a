// Tensor-core quantiser without RoPE: the kernels of tq_quantize_tc.cuh for
// rows given as they are.
#include "tq_quantize_tc.cuh"

cudaError_t tq_launch_quantize_tc(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                  const tq_compressed& out, cudaStream_t st) {
  return launch_quantize_tc<false>(p, x, dt, n, ld, out, st);
}
