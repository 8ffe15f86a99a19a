// Tensor-core quantiser with a fused rotate-half RoPE (TurboESM page, "Resumo
// tecnico" section 2: RoPE is applied before the orthogonal rotation, which
// keeps attention scores exactly because Pi^T Pi = I).  Each row x at
// position pos becomes
//   x'_i       = x_i cos(pos theta_i) - x_{i+d/2} sin(pos theta_i)
//   x'_{i+d/2} = x_i sin(pos theta_i) + x_{i+d/2} cos(pos theta_i),
//   theta_i = theta^(-2i/d),  i < d/2,
// evaluated in fp32 from a caller-provided cos/sin cache, and x' is then
// encoded exactly as tq_quantize encodes an fp32 row.  The same kernels also
// serve tq_append (single-token append at a fixed position, scattered rows).
#include "tq_quantize_tc.cuh"

cudaError_t tq_launch_quantize_tc_rope(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                       const tq_compressed& out, cudaStream_t st) {
  return launch_quantize_tc<true>(p, x, dt, n, ld, out, st);
}

namespace {
// cos/sin cache: entry (pos, i) of [max_pos][d] holds cos(pos theta_i) for
// i < d/2 and sin(pos theta_{i - d/2}) for i >= d/2, computed in fp64 and
// rounded to fp32.
__global__ void tq_rope_cache_kernel(const double theta, const int d, const int max_pos, float* __restrict__ cs) {
  const int64_t total = (int64_t)max_pos * (d / 2);
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int pos = (int)(idx / (d / 2)), i = (int)(idx % (d / 2));
    const double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
    double sn, cn;
    sincos(ang, &sn, &cn);
    cs[(size_t)pos * d + i] = (float)cn;
    cs[(size_t)pos * d + d / 2 + i] = (float)sn;
  }
}
}  // namespace

cudaError_t tq_launch_rope_cache(double theta, int d, int max_pos, float* cs, cudaStream_t st) {
  const int64_t total = (int64_t)max_pos * (d / 2);
  const int grid = (int)std::min<int64_t>((total + 255) / 256, 4096);
  if (total == 0) return cudaSuccess;
  tq_rope_cache_kernel<<<grid, 256, 0, st>>>(theta, d, max_pos, cs);
  return cudaGetLastError();
}
