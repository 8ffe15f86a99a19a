// Fused decode attention, head dimension 128 (kernel in tq_attend.cuh), and
// the dispatch over head dimensions.
#include "tq_attend.cuh"

cudaError_t tq_attend_fused_d64(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                                int64_t T, float scale, const tq_compressed& K, const tq_compressed& V,
                                float* partials, int nchunk, cudaStream_t st);

cudaError_t tq_launch_attend_fused(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq,
                                   int Hkv, int64_t T, float scale, const tq_compressed& K, const tq_compressed& V,
                                   float* partials, int nchunk, cudaStream_t st) {
  if (kp.d != vp.d || kp.m % 32 != 0 || kp.m > 256) return cudaErrorNotSupported;
  if (kp.vq_bits || vp.vq_bits) return cudaErrorNotSupported;  // FibQuant codes: CUDA-core kernel
  // row starts of 16-byte vector loads
  if ((uintptr_t)K.codes % 16 != 0 || (kp.MS > 0 && (uintptr_t)K.signs % 16 != 0)) return cudaErrorNotSupported;
  switch (kp.d) {
    case 64: return tq_attend_fused_d64(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
    case 128:
      return tqatt::launch_attend_d<128>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
    default: return cudaErrorNotSupported;
  }
}
