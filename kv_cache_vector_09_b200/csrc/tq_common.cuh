// Device helpers shared by the libtq kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_internal.h"

#define TQ_FULL_MASK 0xffffffffu

__device__ __forceinline__ float tq_to_f32(float v) { return v; }
__device__ __forceinline__ float tq_to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float tq_to_f32(__half v) { return __half2float(v); }

template <typename F>
__device__ __forceinline__ F tq_warp_sum(F v) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) v += __shfl_xor_sync(TQ_FULL_MASK, v, s);
  return v;
}

template <typename F>
__device__ __forceinline__ F tq_warp_max(F v) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) v = max(v, __shfl_xor_sync(TQ_FULL_MASK, v, s));
  return v;
}

// Unnormalised Walsh-Hadamard transform (Sylvester order) of a vector spread
// over a warp: lane `lane` holds coordinates j = lane + 32 k, k < VPL.  Bits 0-4
// of j are the lane (shuffle butterflies), higher bits are k (in-register
// butterflies).  With VPL > 16 the in-register stages stop at 16, i.e. the
// transform is block-diagonal with blocks of 512 coordinates.
template <int VPL, typename F>
__device__ __forceinline__ void tq_fwht_warp(F (&v)[VPL], int lane) {
  constexpr int KB = VPL < 16 ? VPL : 16;
#pragma unroll
  for (int h = 1; h < KB; h <<= 1) {
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      if ((k & h) == 0) {
        const F a = v[k], b = v[k + h];
        v[k] = a + b;
        v[k + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const F o = __shfl_xor_sync(TQ_FULL_MASK, v[k], s);
      v[k] = (lane & s) ? (o - v[k]) : (v[k] + o);
    }
  }
}

// D_j = -1 for coordinate j = lane + 32 k  <=>  bit `lane` of dbits[k]
__device__ __forceinline__ bool tq_dneg(const uint32_t* dbits, int k, int lane) {
  return (__ldg(dbits + k) >> lane) & 1u;
}

// Dense rotation of a vector spread over a warp (lane holds coordinates
// j = lane + 32 k, k < VPL, d = 32 VPL): v_j <- sum_i Pi_ji v_i with piT
// [d][d] holding Pi_ji at (i, j), so the lanes' loads at fixed i are
// coalesced.  buf: d elements of this warp's scratch (shared memory).
// Each output is four FMA chains over i = c mod 4 (d/4 terms each) added
// pairwise, (c0 + c1) + (c2 + c3): every product meets at most d/4 + 2
// roundings, so |error| <= (d/4 + 2) u sum_i |Pi_ji v_i| to first order.
// Defined for d <= 256 (VPL <= 8), the dense rotations the codecs allow; the
// longer instantiations are empty and never reached.
template <int VPL, typename F>
__device__ __forceinline__ void tq_dense_rotate_warp(F (&v)[VPL], int lane, const float* __restrict__ piT, F* buf) {
  if constexpr (VPL > 8) return;
  constexpr int d = 32 * VPL;
#pragma unroll
  for (int k = 0; k < VPL; ++k) buf[lane + 32 * k] = v[k];
  __syncwarp();
  F acc[4][VPL];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int k = 0; k < VPL; ++k) acc[c][k] = F(0);
  for (int i = 0; i < d; i += 4) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const F bi = buf[i + c];
#pragma unroll
      for (int k = 0; k < VPL; ++k) acc[c][k] = fma((F)__ldg(piT + (size_t)(i + c) * d + lane + 32 * k), bi, acc[c][k]);
    }
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < VPL; ++k) v[k] = (acc[0][k] + acc[1][k]) + (acc[2][k] + acc[3][k]);
}
