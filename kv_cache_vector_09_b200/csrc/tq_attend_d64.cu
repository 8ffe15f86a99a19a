// Fused decode attention, head dimension 64 (kernel in tq_attend.cuh).
#include "tq_attend.cuh"

cudaError_t tq_attend_fused_d64(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                                int64_t T, float scale, const tq_compressed& K, const tq_compressed& V,
                                float* partials, int nchunk, cudaStream_t st) {
  return tqatt::launch_attend_d<64>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
}
