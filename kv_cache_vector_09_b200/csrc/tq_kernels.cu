// libtq kernels: quantise (encoder + QJL sketch), query preparation, scoring
// and split-context decode attention over the compressed cache.
#include <math.h>

#include <algorithm>

#include "tq_common.cuh"

namespace {

constexpr int kQuantWarps = 8;
constexpr float kUlp = 5.9604644775390625e-08f;  // 2^-24, unit roundoff of fp32

// Copies of the per-segment codebooks in shared memory (indexed per lane).
struct SmemBook {
  float cen[2][TQ_MAX_LEVELS];
  float bnd[2][TQ_MAX_LEVELS];
};

__device__ __forceinline__ void load_book(const tq_params& p, SmemBook& sb) {
  for (int i = threadIdx.x; i < 2 * TQ_MAX_LEVELS; i += blockDim.x) {
    sb.cen[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS] = p.cen[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS];
    sb.bnd[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS] = p.bnd[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS];
  }
}

// The FibQuant codewords live at the end of a kernel's dynamic shared memory
// (2^vq_bits float2, sized by the launcher only for codecs with block codes),
// so that scalar codecs keep their shared-memory budget.
__host__ __device__ inline size_t vq_table_bytes(const tq_params& p) {
  return p.vq_bits ? sizeof(float2) * ((size_t)1 << p.vq_bits) : 0;
}

__device__ __forceinline__ void load_vq(const tq_params& p, float2* vq) {
  if (p.vq_bits)
    for (int i = threadIdx.x; i < (1 << p.vq_bits); i += blockDim.x)
      vq[i] = make_float2(__ldg(p.vq_cb + 2 * i), __ldg(p.vq_cb + 2 * i + 1));
}

// FibQuant block codes.  Block j = (z_2j, z_2j+1) sits in lanes 2t and 2t+1
// at register k (j = 16 k + t).  vq_nearest scans codewords [n0, n1) and
// returns the nearest (ties: the lower index) with the squared distances to
// the nearest and second-nearest ones; vq_pair_nearest gives each lane of a
// pair one half of the codebook and merges the halves, so both lanes end with
// the whole codebook's answer.
template <typename F>
__device__ __forceinline__ int vq_nearest(const float2* vq, int n0, int n1, F za, F zb, F& e1, F& e2) {
  int best = n0;
  e1 = F(INFINITY);
  e2 = F(INFINITY);
  for (int n = n0; n < n1; ++n) {
    const F dx = za - (F)vq[n].x, dy = zb - (F)vq[n].y;
    const F e = dx * dx + dy * dy;
    if (e < e1) {
      e2 = e1;
      e1 = e;
      best = n;
    } else if (e < e2) {
      e2 = e;
    }
  }
  return best;
}

template <typename F>
__device__ __forceinline__ int vq_pair_nearest(const float2* vq, int N, int lane, F za, F zb, F& e1, F& e2) {
  const int odd = lane & 1;
  F a1, a2;
  const int ia = vq_nearest<F>(vq, odd ? N / 2 : 0, odd ? N : N / 2, za, zb, a1, a2);
  const F b1 = __shfl_xor_sync(TQ_FULL_MASK, a1, 1), b2 = __shfl_xor_sync(TQ_FULL_MASK, a2, 1);
  const int ib = __shfl_xor_sync(TQ_FULL_MASK, ia, 1);
  // (lo1, lo2, ilo): the lower half's results, (hi1, hi2, ihi): the upper's
  const F lo1 = odd ? b1 : a1, lo2 = odd ? b2 : a2, hi1 = odd ? a1 : b1, hi2 = odd ? a2 : b2;
  const int ilo = odd ? ib : ia, ihi = odd ? ia : ib;
  if (lo1 <= hi1) {  // equal distances: the lower index wins
    e1 = lo1;
    e2 = lo2 < hi1 ? lo2 : hi1;
    return ilo;
  }
  e1 = hi1;
  e2 = hi2 < lo1 ? hi2 : lo1;
  return ihi;
}

// bits 0, 2, .., 30 of v moved to bits 0..15 (the even lanes of a ballot)
__device__ __forceinline__ uint32_t even_bits(uint32_t v) {
  v &= 0x55555555u;
  v = (v | (v >> 1)) & 0x33333333u;
  v = (v | (v >> 2)) & 0x0f0f0f0fu;
  v = (v | (v >> 4)) & 0x00ff00ffu;
  return (v | (v >> 8)) & 0x0000ffffu;
}

// =============================================================== quantise
// One warp per row.  Lane `lane` holds coordinates j = lane + 32k (k < VPL).
//
// Every code and sign bit must equal that of an exact evaluation of the
// definitions.  The row is first evaluated in fp32 together with a rigorous
// bound on the fp32 error of every decision quantity:
//   z_i : |dz_i| <= u ((L + 2) ||u||_1 zs + 2 |z_i|)          (L = log2 p stages,
//         u = 2^-24; the FWHT sums every input once per stage, each stage's
//         nodes partition the inputs, so the rounding of one stage is at most
//         u ||u||_1; the scaling x / nu and the factor zs = sqrt(d/p) add 2u|z|)
//   r_i : |dr_i| <= u ((L + 2) ||u||_1 zs + 4 zmax + 2 cmax) / sqrt(d)
//   t_j : |dt_j| <= ||S_j||_1 max|dr| + (d + 2) u ||S_j||_2 ||r||_2
//         (the last term bounds a d-step FMA chain, Cauchy-Schwarz).
// A code whose z lies within its bound of a boundary, or a sign whose t lies
// within its bound of zero, flags the row; flagged rows are recomputed in fp64
// (norm, rotation, codes, residual, sketch), where the remaining error (~1e-16
// relative) can only matter for exact ties.
template <int VPL, typename TIn>
__global__ void __launch_bounds__(kQuantWarps * 32)
    tq_quantize_kernel(const tq_params p, const TIn* __restrict__ x, const int64_t n, const int64_t ld,
                       const tq_compressed out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ SmemBook sb;
  float2* vqs = reinterpret_cast<float2*>(smem_raw + sizeof(double) * (size_t)kQuantWarps * p.d);
  load_book(p, sb);
  load_vq(p, vqs);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d = p.d;
  double* rbuf = reinterpret_cast<double*>(smem_raw) + (size_t)warp * d;
  float* rbuf_f = reinterpret_cast<float*>(rbuf);
  constexpr int SLOTS = (VPL * 4 + 31) / 32;
  const int Q = p.MS;

  for (int64_t row = (int64_t)blockIdx.x * kQuantWarps + warp; row < n; row += (int64_t)gridDim.x * kQuantWarps) {
    const TIn* xr = x + row * ld;
    float xv[VPL];
#pragma unroll
    for (int k = 0; k < VPL; ++k) xv[k] = tq_to_f32(xr[lane + 32 * k]);
    double ss = 0.0;
    float l1 = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      ss = fma((double)xv[k], (double)xv[k], ss);
      l1 += fabsf(xv[k]);
    }
    ss = tq_warp_sum(ss);
    l1 = tq_warp_sum(l1);
    const double nu64 = sqrt(ss);
    const float inv = nu64 > 0.0 ? (float)(1.0 / nu64) : 0.0f;

    // ---------------- fp32 evaluation with decision bounds
    float z[VPL];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const float v = xv[k] * inv;
      z[k] = tq_dneg(p.dbits, k, lane) ? -v : v;
    }
    const float l1u = l1 * inv * 1.001f;  // >= ||u||_1 despite fp32 rounding of the sum
    // rotation error bound of z in units of u = 2^-24: the FWHT sums every
    // input once per stage, so each stage adds at most ||u||_1 (L stages);
    // the dense Haar product takes at most d/4 + 2 roundings per product
    // (four chains added pairwise), plus 2 for the scaling by 1/nu, so at
    // most (d/4 + 4) u sum_i |Pi_ji u_i| <= (d/4 + 4) u ||u||_2, times
    // sqrt(d) for z
    float rot_term;
    if (p.haar) {
      tq_dense_rotate_warp<VPL>(z, lane, p.piT, rbuf_f);
      const float sd = sqrtf((float)d);
#pragma unroll
      for (int k = 0; k < VPL; ++k) z[k] *= sd;
      rot_term = (float)(d / 4 + 4) * sd * 1.001f;
    } else {
      tq_fwht_warp<VPL>(z, lane);
      if (p.zscale != 1.0f) {
#pragma unroll
        for (int k = 0; k < VPL; ++k) z[k] *= p.zscale;
      }
      rot_term = (float)(p.log2_hblock + 2) * l1u * p.zscale;
    }
    const float ez0 = kUlp * rot_term;
    int code[VPL];
    float cval[VPL];  // centroid value of each coordinate (z units)
    bool flag = false;
    float zmax = 0.f;
    if (p.vq_bits) {
      // nearest codeword per block; the code is certified when the distances
      // from the fp32 block to its nearest and second-nearest codewords differ
      // by more than twice the block's error radius delta (every distance moves
      // by at most delta between the fp32 and the exact block) plus the fp32
      // evaluation error of the two distances (below 4.5 u (D1 + D2))
      const int N = 1 << p.vq_bits;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const float za = __shfl_sync(TQ_FULL_MASK, z[k], lane & ~1);
        const float zb = __shfl_sync(TQ_FULL_MASK, z[k], lane | 1);
        float e1, e2;
        const int c = vq_pair_nearest<float>(vqs, N, lane, za, zb, e1, e2);
        code[k] = c;
        cval[k] = (lane & 1) ? vqs[c].y : vqs[c].x;
        const float ea = ez0 + 2.f * kUlp * fabsf(za), eb = ez0 + 2.f * kUlp * fabsf(zb);
        const float delta = 1.01f * sqrtf(ea * ea + eb * eb);
        const float D1 = sqrtf(e1), D2 = sqrtf(e2);
        flag |= (D2 - D1) <= 2.f * delta + 8.f * kUlp * (D1 + D2);
        zmax = fmaxf(zmax, fabsf(z[k]));
      }
    }
#pragma unroll
    for (int k = 0; k < (p.vq_bits ? 0 : VPL); ++k) {
      const int s = (p.nseg == 2 && k >= VPL / 2) ? 1 : 0;
      const int nb = (1 << p.bits[s]) - 1;
      int c = 0;
      float mg = INFINITY;
      for (int b = 0; b < nb; ++b) {
        const float bv = sb.bnd[s][b];
        c += (z[k] >= bv) ? 1 : 0;
        mg = fminf(mg, fabsf(z[k] - bv));
      }
      code[k] = c;
      cval[k] = sb.cen[s][c];
      flag |= mg <= 1.01f * (ez0 + 2.f * kUlp * fabsf(z[k]));
      zmax = fmaxf(zmax, fabsf(z[k]));
    }
    float r[VPL];
    float g2 = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      r[k] = (z[k] - cval[k]) * p.inv_sqrt_d;
      g2 = fmaf(r[k], r[k], g2);
    }
    g2 = tq_warp_sum(g2);
    zmax = tq_warp_max(zmax);
    float gamma = sqrtf(g2);
    uint32_t signword = 0;
    if (Q > 0) {
#pragma unroll
      for (int k = 0; k < VPL; ++k) rbuf_f[lane + 32 * k] = r[k];
      __syncwarp();
      const float er = 1.01f * kUlp * (rot_term + 4.f * zmax + 2.f * p.cmax) * p.inv_sqrt_d;
      // sketch rows lane * Q + q: up to eight chains side by side (each one
      // the same sequential FMA chain over i as alone), then one at a time
      constexpr int QB = 8;
      for (int q0 = 0; q0 < Q; q0 += QB) {
        float t[QB];
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) t[qq] = 0.f;
        const float* sc = p.St + lane * Q + q0;
        if ((Q & 3) == 0) {
          // this lane's columns are 16-byte aligned runs (Q, q0 and m are
          // multiples of 4): one 128-bit load per four chains
          for (int i = 0; i < d; ++i) {
            const float ri = rbuf_f[i];
            const float4* s4 = reinterpret_cast<const float4*>(sc + (size_t)i * p.m);
#pragma unroll
            for (int qv = 0; qv < QB / 4; ++qv) {
              if (q0 + 4 * qv < Q) {
                const float4 a = __ldg(s4 + qv);
                t[4 * qv] = fmaf(a.x, ri, t[4 * qv]);
                t[4 * qv + 1] = fmaf(a.y, ri, t[4 * qv + 1]);
                t[4 * qv + 2] = fmaf(a.z, ri, t[4 * qv + 2]);
                t[4 * qv + 3] = fmaf(a.w, ri, t[4 * qv + 3]);
              }
            }
          }
        } else {
          for (int i = 0; i < d; ++i) {
            const float ri = rbuf_f[i];
#pragma unroll
            for (int qq = 0; qq < QB; ++qq)
              if (q0 + qq < Q) t[qq] = fmaf(__ldg(sc + (size_t)i * p.m + qq), ri, t[qq]);
          }
        }
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) {
          const int q = q0 + qq;
          if (q < Q) {
            const int col = lane * Q + q;
            const float et =
                1.01f * (__ldg(p.s_l1 + col) * er + (float)(d + 2) * kUlp * __ldg(p.s_l2 + col) * gamma * 1.01f);
            flag |= fabsf(t[qq]) <= et;
            const uint32_t wv = __ballot_sync(TQ_FULL_MASK, t[qq] >= 0.f);
            if (lane == q) signword = wv;
          }
        }
      }
      __syncwarp();
    }

    // ---------------- fp64 re-evaluation of flagged rows
    if (__any_sync(TQ_FULL_MASK, flag)) {
      double zd[VPL];
      const double invd = nu64 > 0.0 ? 1.0 / nu64 : 0.0;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const double v = (double)xv[k] * invd;
        zd[k] = tq_dneg(p.dbits, k, lane) ? -v : v;
      }
      if (p.haar) {
        tq_dense_rotate_warp<VPL>(zd, lane, p.piT, rbuf);
        const double sd = sqrt((double)d);
#pragma unroll
        for (int k = 0; k < VPL; ++k) zd[k] *= sd;
      } else {
        tq_fwht_warp<VPL>(zd, lane);
        if (p.hblock != d) {
          const double zs = sqrt((double)d / (double)p.hblock);
#pragma unroll
          for (int k = 0; k < VPL; ++k) zd[k] *= zs;
        }
      }
      const double isd = 1.0 / sqrt((double)d);
      double g2d = 0.0;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        double cv;
        if (p.vq_bits) {
          const double za = __shfl_sync(TQ_FULL_MASK, zd[k], lane & ~1);
          const double zb = __shfl_sync(TQ_FULL_MASK, zd[k], lane | 1);
          double e1, e2;
          const int c = vq_pair_nearest<double>(vqs, 1 << p.vq_bits, lane, za, zb, e1, e2);
          code[k] = c;
          cv = (lane & 1) ? (double)vqs[c].y : (double)vqs[c].x;
        } else {
          const int s = (p.nseg == 2 && k >= VPL / 2) ? 1 : 0;
          const int nb = (1 << p.bits[s]) - 1;
          int c = 0;
          for (int b = 0; b < nb; ++b) c += (zd[k] >= (double)sb.bnd[s][b]) ? 1 : 0;
          code[k] = c;
          cv = (double)sb.cen[s][c];
        }
        const double rv = (zd[k] - cv) * isd;
        rbuf[lane + 32 * k] = rv;
        g2d = fma(rv, rv, g2d);
      }
      g2d = tq_warp_sum(g2d);
      gamma = (float)sqrt(g2d);
      __syncwarp();
      for (int q = 0; q < Q; ++q) {
        const float* sc = p.St + lane * Q + q;
        double t = 0.0;
        for (int i = 0; i < d; ++i) t = fma((double)__ldg(sc + (size_t)i * p.m), rbuf[i], t);
        const uint32_t wv = __ballot_sync(TQ_FULL_MASK, t >= 0.0);
        if (lane == q) signword = wv;
      }
      __syncwarp();
    }

    // ---------------- pack and store
    uint32_t cw[SLOTS];
#pragma unroll
    for (int sl = 0; sl < SLOTS; ++sl) cw[sl] = 0;
    if (p.vq_bits) {
      // plane pl, word k / 2: blocks 16 k + t (t < 16) at bits 16 (k % 2) + t
#pragma unroll
      for (int k = 0; k < VPL; ++k)
        for (int pl = 0; pl < p.vq_bits; ++pl) {
          const uint32_t half = even_bits(__ballot_sync(TQ_FULL_MASK, (code[k] >> pl) & 1));
          const int widx = pl * p.vq_pw + (k >> 1);
#pragma unroll
          for (int sl = 0; sl < SLOTS; ++sl)
            if (sl == (widx >> 5) && lane == (widx & 31)) cw[sl] |= half << (16 * (k & 1));
        }
    }
#pragma unroll
    for (int k = 0; k < (p.vq_bits ? 0 : VPL); ++k) {
      const int s = (p.nseg == 2 && k >= VPL / 2) ? 1 : 0;
      const int kk = s ? k - VPL / 2 : k;
      for (int pl = 0; pl < p.bits[s]; ++pl) {
        const uint32_t wv = __ballot_sync(TQ_FULL_MASK, (code[k] >> pl) & 1);
        const int widx = p.segbase[s] + pl * p.pw + kk;
#pragma unroll
        for (int sl = 0; sl < SLOTS; ++sl)
          if (sl == (widx >> 5) && lane == (widx & 31)) cw[sl] = wv;
      }
    }
    const int64_t dst = row * p.out_stride + p.out_offset;  // compressed row written
    uint32_t* orow = out.codes + dst * p.W;
#pragma unroll
    for (int sl = 0; sl < SLOTS; ++sl)
      if (sl * 32 + lane < p.W) orow[sl * 32 + lane] = cw[sl];
    if (Q > 0) {
      if (lane < Q) out.signs[dst * Q + lane] = signword;
      if (lane == 0) out.rnorms[dst] = p.rnorm_is_const ? p.rnorm_const : gamma;
    }
    if (lane == 0) out.norms[dst] = (float)nu64;
  }
}

// ====================================================== query preparation
// q' = Pi q (no normalisation) and w = S q', written as [nq][d + m] floats.
template <int VPL, typename TIn>
__global__ void __launch_bounds__(256)
    tq_qprep_kernel(const tq_params p, const TIn* __restrict__ q, const int nq, float* __restrict__ qprep) {
  // one query per block: warp 0 rotates it (q' = Pi q), then every thread
  // takes sketch rows j = tid, tid + blockDim.x, .. of w = S q', reading the
  // rows of S (row-major [m][d]) with 16-byte loads
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d = p.d, m = p.m;
  float* buf = reinterpret_cast<float*>(smem_raw);
  const int row = blockIdx.x;
  if (row >= nq) return;
  float* o = qprep + (size_t)row * (d + m);
  if (warp == 0) {
    float v[VPL];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const float a = tq_to_f32(q[(size_t)row * d + lane + 32 * k]);
      v[k] = tq_dneg(p.dbits, k, lane) ? -a : a;
    }
    if (p.haar) {
      tq_dense_rotate_warp<VPL>(v, lane, p.piT, buf);
    } else {
      tq_fwht_warp<VPL>(v, lane);
#pragma unroll
      for (int k = 0; k < VPL; ++k) v[k] *= p.inv_sqrt_p;
    }
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      o[lane + 32 * k] = v[k];
      buf[lane + 32 * k] = v[k];
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < m; j += blockDim.x) {
    const float4* sr = reinterpret_cast<const float4*>(p.S + (size_t)j * d);
    float t0 = 0.f, t1 = 0.f;
    for (int i = 0; i < d / 4; i += 2) {
      const float4 a = __ldg(sr + i);
      const float4 b = __ldg(sr + i + 1);
      t0 = fmaf(a.x, buf[4 * i], t0);
      t0 = fmaf(a.y, buf[4 * i + 1], t0);
      t0 = fmaf(a.z, buf[4 * i + 2], t0);
      t0 = fmaf(a.w, buf[4 * i + 3], t0);
      t1 = fmaf(b.x, buf[4 * i + 4], t1);
      t1 = fmaf(b.y, buf[4 * i + 5], t1);
      t1 = fmaf(b.z, buf[4 * i + 6], t1);
      t1 = fmaf(b.w, buf[4 * i + 7], t1);
    }
    o[d + j] = t0 + t1;
  }
}

// ================================================================= scores
// <q', cen[code]> over all coordinates of one row, for NG queries at once;
// qp is [d][NG] in shared memory.
template <int NG>
__device__ __forceinline__ void mse_dot(const tq_params& p, const uint32_t* __restrict__ cw, const float* qp,
                                        const SmemBook& sb, const float2* vq, float (&acc)[NG]) {
  if (p.vq_bits) {
    // FibQuant: block 32w + t's codeword times (q'_2j, q'_2j+1), j = 32w + t
    for (int w = 0; w < p.vq_pw; ++w) {
      uint32_t pl[TQ_MAX_VQ_BITS];
#pragma unroll
      for (int b = 0; b < TQ_MAX_VQ_BITS; ++b) pl[b] = b < p.vq_bits ? __ldg(cw + b * p.vq_pw + w) : 0u;
      const float* qrow = qp + (size_t)(64 * w) * NG;
#pragma unroll 4
      for (int t = 0; t < 32; ++t) {
        int c = 0;
#pragma unroll
        for (int b = 0; b < TQ_MAX_VQ_BITS; ++b) c |= ((pl[b] >> t) & 1) << b;
        const float2 v = vq[c];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          acc[g] = fmaf(v.x, qrow[(2 * t) * NG + g], acc[g]);
          acc[g] = fmaf(v.y, qrow[(2 * t + 1) * NG + g], acc[g]);
        }
      }
    }
    return;
  }
  for (int s = 0; s < p.nseg; ++s) {
    const int bits = p.bits[s];
    for (int w = 0; w < p.pw; ++w) {
      uint32_t pl[4] = {0u, 0u, 0u, 0u};
      for (int b = 0; b < bits; ++b) pl[b] = __ldg(cw + p.segbase[s] + b * p.pw + w);
      const float* qrow = qp + (size_t)(s * p.seg_len + 32 * w) * NG;
#pragma unroll 8
      for (int t = 0; t < 32; ++t) {
        const int c = ((pl[0] >> t) & 1) | (((pl[1] >> t) & 1) << 1) | (((pl[2] >> t) & 1) << 2) |
                      (((pl[3] >> t) & 1) << 3);
        const float v = sb.cen[s][c];
#pragma unroll
        for (int g = 0; g < NG; ++g) acc[g] = fmaf(v, qrow[t * NG + g], acc[g]);
      }
    }
  }
}

// <w, 2 bit - 1> for NG queries; wq is [m][NG] in shared memory.
template <int NG>
__device__ __forceinline__ void qjl_dot(const tq_params& p, const uint32_t* __restrict__ sw, const float* wq,
                                        float (&acc)[NG]) {
  for (int qw = 0; qw < p.MS; ++qw) {
    const uint32_t word = __ldg(sw + qw);
    const float* wrow = wq + (size_t)32 * qw * NG;
#pragma unroll 8
    for (int t = 0; t < 32; ++t) {
      const uint32_t neg = ((~word >> t) & 1u) << 31;
#pragma unroll
      for (int g = 0; g < NG; ++g) acc[g] += __uint_as_float(__float_as_uint(wrow[t * NG + g]) ^ neg);
    }
  }
}

// Loads the prepared queries of one (b, KV head) into shared memory as
// qp [d][NG] and wq [m][NG]; query heads g >= G are zero.
template <int NG>
__device__ __forceinline__ void load_queries(const tq_params& p, const float* __restrict__ qprep, int b, int Hq,
                                             int hk, int G, float* qp, float* wq) {
  const int d = p.d, m = p.m;
  for (int idx = threadIdx.x; idx < NG * (d + m); idx += blockDim.x) {
    const int g = idx / (d + m), i = idx % (d + m);
    const float v = g < G ? qprep[(size_t)(b * Hq + hk * G + g) * (d + m) + i] : 0.f;
    if (i < d)
      qp[i * NG + g] = v;
    else
      wq[(i - d) * NG + g] = v;
  }
}

constexpr int kScoreThreads = 256;
constexpr int kScoreTile = 2048;

template <int NG>
__global__ void __launch_bounds__(kScoreThreads)
    tq_scores_kernel(const tq_params p, const float* __restrict__ qprep, const int Hq, const int Hkv, const int64_t T,
                     const tq_compressed K, float* __restrict__ logits) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ SmemBook sb;
  float* qp = reinterpret_cast<float*>(smem_raw);
  float* wq = qp + (size_t)NG * p.d;
  float2* vqs = reinterpret_cast<float2*>(wq + (size_t)NG * p.m);
  const int b = blockIdx.z, hk = blockIdx.y, G = Hq / Hkv;
  load_book(p, sb);
  load_vq(p, vqs);
  load_queries<NG>(p, qprep, b, Hq, hk, G, qp, wq);
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * kScoreTile;
  const int64_t t1 = min(T, t0 + kScoreTile);
  for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const int64_t row = ((int64_t)b * Hkv + hk) * T + t;
    float acc[NG], acc2[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) acc[g] = acc2[g] = 0.f;
    mse_dot<NG>(p, K.codes + row * p.W, qp, sb, vqs, acc);
    float gam = 0.f;
    if (p.m > 0) {
      qjl_dot<NG>(p, K.signs + row * p.MS, wq, acc2);
      gam = __ldg(K.rnorms + row);
    }
    const float nu = __ldg(K.norms + row);
    const float cq = gam * p.qjl_coef;
#pragma unroll
    for (int g = 0; g < NG; ++g)
      if (g < G)
        logits[((int64_t)b * Hq + hk * G + g) * T + t] = nu * fmaf(acc[g], p.inv_sqrt_d, cq * acc2[g]);
  }
}

// ============================================================== attention
constexpr int kAttThreads = 256;

// Split-context decode attention: block (chunk, KV head, batch) scores its
// chunk of keys for the G query heads, takes the chunk maximum and the
// exponentials (base 2, logits pre-multiplied by scale * log2(e)), and
// accumulates sum_t p_t nu_v,t cen_v[code] / sqrt(d) in the rotated space.
// Partials [B*Hq][nchunk][d + 2] hold (acc[d], max, sum).
template <int NG>
__global__ void __launch_bounds__(kAttThreads)
    tq_attend_kernel(const tq_params kp, const tq_params vp, const float* __restrict__ qprep, const int Hq,
                     const int Hkv, const int64_t T, const float scale_log2e, const tq_compressed K,
                     const tq_compressed V, float* __restrict__ partials, const int nchunk, const int chunk_len) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ SmemBook sbk, sbv;
  __shared__ float red[kAttThreads / 32][NG];
  __shared__ float gmax[NG], gsum[NG];
  const int d = kp.d;
  float* qp = reinterpret_cast<float*>(smem_raw);
  float* wq = qp + (size_t)NG * d;
  float* L = wq + (size_t)NG * kp.m;                  // [chunk_len][NG]
  float* accbuf = L + (size_t)chunk_len * NG;         // [groups][d][NG]
  // FibQuant codewords of the keys, then of the values, 8-byte aligned
  const size_t vq_off = ((size_t)(accbuf - qp) + (size_t)(kAttThreads / d) * d * NG + 1) & ~(size_t)1;
  float2* vqk = reinterpret_cast<float2*>(qp + vq_off);
  float2* vqv = vqk + (kp.vq_bits ? (1 << kp.vq_bits) : 0);
  const int b = blockIdx.z, hk = blockIdx.y, G = Hq / Hkv, chunk = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  load_book(kp, sbk);
  load_book(vp, sbv);
  load_vq(kp, vqk);
  load_vq(vp, vqv);
  load_queries<NG>(kp, qprep, b, Hq, hk, G, qp, wq);
  __syncthreads();
  const int64_t t0 = (int64_t)chunk * chunk_len;
  const int64_t t1 = min(T, t0 + chunk_len);
  const int64_t rowbase = ((int64_t)b * Hkv + hk) * T;

  // phase 1: logits
  float lmax[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) lmax[g] = -INFINITY;
  for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const int64_t row = rowbase + t;
    float acc[NG], acc2[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) acc[g] = acc2[g] = 0.f;
    mse_dot<NG>(kp, K.codes + row * kp.W, qp, sbk, vqk, acc);
    float gam = 0.f;
    if (kp.m > 0) {
      qjl_dot<NG>(kp, K.signs + row * kp.MS, wq, acc2);
      gam = __ldg(K.rnorms + row);
    }
    const float nu = __ldg(K.norms + row);
    const float cq = gam * kp.qjl_coef;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float l = nu * fmaf(acc[g], kp.inv_sqrt_d, cq * acc2[g]) * scale_log2e;
      L[(t - t0) * NG + g] = l;
      lmax[g] = fmaxf(lmax[g], l);
    }
  }
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const float v = tq_warp_max(lmax[g]);
    if (lane == 0) red[warp][g] = v;
  }
  __syncthreads();
  if (threadIdx.x < NG) {
    float v = -INFINITY;
    for (int w = 0; w < kAttThreads / 32; ++w) v = fmaxf(v, red[w][threadIdx.x]);
    gmax[threadIdx.x] = v;
  }
  __syncthreads();

  // phase 2: exponentials, times the value norm
  float lsum[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) lsum[g] = 0.f;
  for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const float nv = __ldg(V.norms + rowbase + t);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float e = exp2f(L[(t - t0) * NG + g] - gmax[g]);
      lsum[g] += e;
      L[(t - t0) * NG + g] = e * nv;
    }
  }
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const float v = tq_warp_sum(lsum[g]);
    if (lane == 0) red[warp][g] = v;
  }
  __syncthreads();
  if (threadIdx.x < NG) {
    float v = 0.f;
    for (int w = 0; w < kAttThreads / 32; ++w) v += red[w][threadIdx.x];
    gsum[threadIdx.x] = v;
  }

  // phase 3: weighted sum of dequantised values (rotated space)
  const int groups = kAttThreads / d;  // d <= 256
  const int i = threadIdx.x % d, grp = threadIdx.x / d;
  float acc[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) acc[g] = 0.f;
  if (grp < groups) {
    // scalar codes: coordinate i's own code; FibQuant: block i / 2's code,
    // component i % 2 of its codeword
    const bool vq = vp.vq_bits != 0;
    const int s = (!vq && vp.nseg == 2 && i >= vp.seg_len) ? 1 : 0;
    const int il = vq ? (i >> 1) : i - s * vp.seg_len;
    const int w = il >> 5, bit = il & 31;
    const int bits = vq ? vp.vq_bits : vp.bits[s];
    const int pstride = vq ? vp.vq_pw : vp.pw;
    const int wbase = (vq ? 0 : vp.segbase[s]) + w;
    for (int64_t t = t0 + grp; t < t1; t += groups) {
      const uint32_t* cw = V.codes + (rowbase + t) * vp.W + wbase;
      int c = 0;
      for (int pb = 0; pb < bits; ++pb) c |= ((__ldg(cw + pb * pstride) >> bit) & 1) << pb;
      const float v = vq ? ((i & 1) ? vqv[c].y : vqv[c].x) : sbv.cen[s][c];
      const float* lr = L + (t - t0) * NG;
#pragma unroll
      for (int g = 0; g < NG; ++g) acc[g] = fmaf(lr[g], v, acc[g]);
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) accbuf[((size_t)grp * d + i) * NG + g] = acc[g];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
    const int g = idx / d, ii = idx % d;
    float v = 0.f;
    for (int gr = 0; gr < groups; ++gr) v += accbuf[((size_t)gr * d + ii) * NG + g];
    float* pr = partials + ((size_t)(b * Hq + hk * G + g) * nchunk + chunk) * (d + 2);
    pr[ii] = v * vp.inv_sqrt_d;
    if (ii == 0) {
      pr[d] = gmax[g];
      pr[d + 1] = gsum[g];
    }
  }
}

// Merge the chunks of one (b, h) and rotate back: out = D * (H acc) / sqrt(p).
// Merges the chunks' (acc[d], max, sum[, a[m]]) by log-sum-exp weights, adds
// the values' QJL correction sqrt(pi/2)/m S^T a when vm > 0 (a = sum_t p_t
// nu_t gamma_t s_t, m = vm <= 128), and rotates back: out = Pi^T acc.
template <int VPL>
__global__ void __launch_bounds__(256)
    tq_attend_combine_kernel(const tq_params vp, const float* __restrict__ partials, const int nchunk, const int nbh,
                             const int vm, float* __restrict__ out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bh = blockIdx.x * (blockDim.x >> 5) + warp;
  if (bh >= nbh) return;
  const int d = vp.d, ps = d + 2 + vm;
  const float* pr = partials + (size_t)bh * nchunk * ps;
  float M = -INFINITY;
  for (int c = lane; c < nchunk; c += 32) M = fmaxf(M, pr[(size_t)c * ps + d]);
  M = tq_warp_max(M);
  float acc[VPL], as[4];
#pragma unroll
  for (int k = 0; k < VPL; ++k) acc[k] = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) as[u] = 0.f;
  float den = 0.f;
  for (int c = 0; c < nchunk; ++c) {
    const float* pc = pr + (size_t)c * ps;
    const float wgt = exp2f(pc[d] - M);
    den = fmaf(pc[d + 1], wgt, den);
#pragma unroll
    for (int k = 0; k < VPL; ++k) acc[k] = fmaf(pc[lane + 32 * k], wgt, acc[k]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (32 * u < vm) as[u] = fmaf(pc[d + 2 + lane + 32 * u], wgt, as[u]);
  }
  const float inv = 1.0f / den;
#pragma unroll
  for (int k = 0; k < VPL; ++k) acc[k] *= inv;
  if (vm > 0) {
    // acc_i += sqrt(pi/2)/m sum_j S_ji a_j / den, rows of S read coalesced
    for (int j = 0; j < vm; ++j) {
      float aj = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (u == (j >> 5)) aj = __shfl_sync(TQ_FULL_MASK, as[u], j & 31);
      aj *= inv * vp.qjl_coef;
      const float* Sj = vp.S + (size_t)j * d;
#pragma unroll
      for (int k = 0; k < VPL; ++k) acc[k] = fmaf(__ldg(Sj + lane + 32 * k), aj, acc[k]);
    }
  }
  if (vp.haar) {
    // out_i = sum_j Pi_ji acc_j, acc_j broadcast from its lane
    float o[VPL];
#pragma unroll
    for (int k = 0; k < VPL; ++k) o[k] = 0.f;
    for (int j = 0; j < d; ++j) {
      float aj = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k)
        if (k == (j >> 5)) aj = __shfl_sync(TQ_FULL_MASK, acc[k], j & 31);
#pragma unroll
      for (int k = 0; k < VPL; ++k) o[k] = fmaf(__ldg(vp.piT + (size_t)(lane + 32 * k) * d + j), aj, o[k]);
    }
#pragma unroll
    for (int k = 0; k < VPL; ++k) out[(size_t)bh * d + lane + 32 * k] = o[k];
    return;
  }
  tq_fwht_warp<VPL>(acc, lane);
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const float v = acc[k] * vp.inv_sqrt_p;
    out[(size_t)bh * d + lane + 32 * k] = tq_dneg(vp.dbits, k, lane) ? -v : v;
  }
}

int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_num_sms = v;
  }
  return g_num_sms;
}

template <typename Fn>
cudaError_t set_smem(Fn* fn, size_t bytes) {
  if (bytes > 48 * 1024) return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  return cudaSuccess;
}

template <int VPL, typename TIn>
cudaError_t launch_quantize_t(const tq_params& p, const void* x, int64_t n, int64_t ld, const tq_compressed& out,
                              cudaStream_t st) {
  const size_t smem = sizeof(double) * (size_t)kQuantWarps * p.d + vq_table_bytes(p);
  auto fn = tq_quantize_kernel<VPL, TIn>;
  cudaError_t e = set_smem(fn, smem);
  if (e != cudaSuccess) return e;
  const int64_t need = (n + kQuantWarps - 1) / kQuantWarps;
  const int grid = (int)std::min<int64_t>(need, (int64_t)num_sms() * 16);
  fn<<<grid, kQuantWarps * 32, smem, st>>>(p, (const TIn*)x, n, ld, out);
  return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_quantize_v(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                              const tq_compressed& out, cudaStream_t st) {
  switch (dt) {
    case TQ_F32: return launch_quantize_t<VPL, float>(p, x, n, ld, out, st);
    case TQ_BF16: return launch_quantize_t<VPL, __nv_bfloat16>(p, x, n, ld, out, st);
    default: return launch_quantize_t<VPL, __half>(p, x, n, ld, out, st);
  }
}

template <int VPL, typename TIn>
cudaError_t launch_qprep_t(const tq_params& p, const void* q, int nq, float* qprep, cudaStream_t st) {
  const size_t smem = sizeof(float) * (size_t)p.d;
  const int threads = p.m > 128 ? 256 : 128;
  auto fn = tq_qprep_kernel<VPL, TIn>;
  cudaError_t e = set_smem(fn, smem);
  if (e != cudaSuccess) return e;
  if (nq == 0) return cudaSuccess;
  fn<<<nq, threads, smem, st>>>(p, (const TIn*)q, nq, qprep);
  return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_qprep_v(const tq_params& p, const void* q, tq_dtype dt, int nq, float* qprep, cudaStream_t st) {
  switch (dt) {
    case TQ_F32: return launch_qprep_t<VPL, float>(p, q, nq, qprep, st);
    case TQ_BF16: return launch_qprep_t<VPL, __nv_bfloat16>(p, q, nq, qprep, st);
    default: return launch_qprep_t<VPL, __half>(p, q, nq, qprep, st);
  }
}

int padded_groups(int G) {
  int ng = 1;
  while (ng < G) ng <<= 1;
  return ng;
}

template <int NG>
cudaError_t launch_scores_g(const tq_params& p, const float* qprep, int B, int Hq, int Hkv, int64_t T,
                            const tq_compressed& K, float* logits, cudaStream_t st) {
  const size_t smem = sizeof(float) * (size_t)NG * (p.d + p.m) + vq_table_bytes(p);
  auto fn = tq_scores_kernel<NG>;
  cudaError_t e = set_smem(fn, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((T + kScoreTile - 1) / kScoreTile), (unsigned)Hkv, (unsigned)B);
  fn<<<grid, kScoreThreads, smem, st>>>(p, qprep, Hq, Hkv, T, K, logits);
  return cudaGetLastError();
}

int attend_chunk_len(int B, int Hkv, int64_t T, int nchunk) { return (int)((T + nchunk - 1) / nchunk); }

template <int NG>
cudaError_t launch_attend_g(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                            int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                            int nchunk, cudaStream_t st) {
  const int chunk_len = attend_chunk_len(B, Hkv, T, nchunk);
  const int groups = kAttThreads / kp.d;
  const size_t floats = (size_t)NG * (kp.d + kp.m) + (size_t)chunk_len * NG + (size_t)groups * kp.d * NG;
  const size_t smem = sizeof(float) * ((floats + 1) & ~(size_t)1) + vq_table_bytes(kp) + vq_table_bytes(vp);
  auto fn = tq_attend_kernel<NG>;
  cudaError_t e = set_smem(fn, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)nchunk, (unsigned)Hkv, (unsigned)B);
  fn<<<grid, kAttThreads, smem, st>>>(kp, vp, qprep, Hq, Hkv, T, scale * 1.4426950408889634f, K, V, partials, nchunk,
                                      chunk_len);
  return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_combine_v(const tq_params& vp, const float* partials, int nchunk, int nbh, float* out,
                             cudaStream_t st) {
  tq_attend_combine_kernel<VPL><<<(nbh + 7) / 8, 256, 0, st>>>(vp, partials, nchunk, nbh, vp.m, out);
  return cudaGetLastError();
}

}  // namespace

// ====================================================================== launchers
#define TQ_DISPATCH_VPL(d, CALL)              \
  switch (d) {                                \
    case 64: { constexpr int V = 2; return CALL; }    \
    case 128: { constexpr int V = 4; return CALL; }   \
    case 256: { constexpr int V = 8; return CALL; }   \
    case 512: { constexpr int V = 16; return CALL; }  \
    case 1024: { constexpr int V = 32; return CALL; } \
    case 1536: { constexpr int V = 48; return CALL; } \
    default: return cudaErrorInvalidValue;    \
  }

#define TQ_DISPATCH_NG(G, CALL)                      \
  switch (padded_groups(G)) {                        \
    case 1: { constexpr int NG = 1; return CALL; }   \
    case 2: { constexpr int NG = 2; return CALL; }   \
    case 4: { constexpr int NG = 4; return CALL; }   \
    case 8: { constexpr int NG = 8; return CALL; }   \
    case 16: { constexpr int NG = 16; return CALL; } \
    case 32: { constexpr int NG = 32; return CALL; } \
    default: return cudaErrorInvalidValue;           \
  }

cudaError_t tq_launch_quantize(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                               const tq_compressed& out, cudaStream_t st) {
  TQ_DISPATCH_VPL(p.d, (launch_quantize_v<V>(p, x, dt, n, ld, out, st)));
}

cudaError_t tq_launch_qprep(const tq_params& p, const void* q, tq_dtype dt, int nq, float* qprep, cudaStream_t st) {
  TQ_DISPATCH_VPL(p.d, (launch_qprep_v<V>(p, q, dt, nq, qprep, st)));
}

cudaError_t tq_launch_scores(const tq_params& p, const float* qprep, int B, int Hq, int Hkv, int64_t T,
                             const tq_compressed& K, float* logits, cudaStream_t st) {
  TQ_DISPATCH_NG(Hq / Hkv, (launch_scores_g<NG>(p, qprep, B, Hq, Hkv, T, K, logits, st)));
}

int tq_attend_chunks(int B, int Hq, int Hkv, int64_t T, int sms) {
  // at least two blocks per SM, chunks of at least 64 keys, and at most
  // 8192 / NG keys so that a block's logit buffer stays at 32 KB
  const int64_t units = (int64_t)B * Hkv;
  const int64_t max_len = std::min<int64_t>(2048, 8192 / padded_groups(Hkv > 0 ? Hq / Hkv : 1));
  int64_t want = units > 0 ? (2 * (int64_t)sms + units - 1) / units : 1;
  want = std::max<int64_t>(want, (T + max_len - 1) / max_len);
  want = std::min<int64_t>(want, std::max<int64_t>(1, (T + 63) / 64));
  want = std::min<int64_t>(want, std::max<int64_t>(1, T));
  return (int)std::max<int64_t>(1, want);
}

cudaError_t tq_launch_attend(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                             int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                             int nchunk, float* out, cudaStream_t st) {
  cudaError_t e = tq_launch_attend_fused(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  // the CUDA-core fallback has no QJL-corrected values
  if (e == cudaErrorNotSupported && vp.m == 0) {
    auto run = [&]() -> cudaError_t {
      TQ_DISPATCH_NG(Hq / Hkv, (launch_attend_g<NG>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st)));
    };
    e = run();
  }
  if (e != cudaSuccess) return e;
  TQ_DISPATCH_VPL(vp.d, (launch_combine_v<V>(vp, partials, nchunk, B * Hq, out, st)));
}
