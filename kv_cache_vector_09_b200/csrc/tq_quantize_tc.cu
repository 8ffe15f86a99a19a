// Tensor-core quantiser: one thread per row, 128 rows per tile (= TMEM lanes).
//
// Per row (thread): load x, apply the D signs, in-register Walsh-Hadamard
// transform of the unnormalised vector w = H (D x), quantise every coordinate
// against the boundaries scaled by the fp32 norm (z_i >= bnd_k  <=>  w_i >= nu
// bnd_k), pack the bit planes, and form the residual r = w - nu cen[code].
// The QJL sketch t = S r of the whole tile is one tensor-core product: r is
// written to TMEM as fp16 hi + lo (r = hi + lo to 2^-22), S comes from shared
// memory as fp16 hi + lo, and three passes (hi*hi, lo*hi, hi*lo) accumulate
// t in fp32 TMEM.
//
// Every code and sign decision carries a rigorous bound on its fp32 error:
//   w_i   : |dw| <= L u ||x||_1 <= L u sqrt(d) nu   (L = log2 d butterfly stages,
//           each stage's nodes partition the inputs; u = 2^-24)
//   nu    : relative error <= e_nu = (d/16 + 3) u    (8 partial sums + sqrt)
//   code  : certain when |w_i - nu bnd_k| > A + B |w_i| for every boundary,
//           A = 1.1 L u sqrt(d) nu, B = 1.1 (e_nu + 2u)
//   t_j   : certain when |t_j| > 1.1 (||S_j||_1 E_r + 2^-17.8 ||S_j||_2 ||r|| + ...)
//           with E_r the per-coordinate residual bound (see below).
// Rows with any uncertain decision (and rows whose squared norm leaves
// [1e-30, 1e30]) are recomputed in fp64 by a warp, after the tile.
#include <math.h>

#include <algorithm>

#include "tq_common.cuh"
#include "tq_tc.cuh"

namespace {

constexpr int kTile = 128;
constexpr float kU = 5.9604644775390625e-08f;  // 2^-24

struct QBook {  // codebook copy in shared memory
  float cen[2][TQ_MAX_LEVELS];
  float bnd[2][TQ_MAX_LEVELS];
};

// ---------------------------------------------------------------- helpers
template <int BITS>
struct Mag {
  static constexpr int H = 1 << (BITS - 1);  // centroids per sign
};

// Magnitude search for one coordinate: a = |w|, mt[k] = nu * (k-th positive
// boundary), k = 1..H-1.  Returns the magnitude cell m and the distance to the
// nearest compared boundary (the zero boundary included): the compared
// boundaries include both ends of the final cell.
template <int BITS>
__device__ __forceinline__ void mag_search(float a, const float* mt, int& m, float& margin) {
  if constexpr (BITS == 1) {
    m = 0;
    margin = a;
  } else if constexpr (BITS == 2) {
    const bool c = a >= mt[1];
    m = c;
    margin = fminf(a, fabsf(a - mt[1]));
  } else if constexpr (BITS == 3) {
    const bool m1 = a >= mt[2];
    const float t = m1 ? mt[3] : mt[1];
    const bool m0 = a >= t;
    m = (m1 << 1) | m0;
    margin = fminf(a, fminf(fabsf(a - mt[2]), fabsf(a - t)));
  } else {
    const bool m2 = a >= mt[4];
    const float t1 = m2 ? mt[6] : mt[2];
    const bool m1 = a >= t1;
    const float t0 = m2 ? (m1 ? mt[7] : mt[5]) : (m1 ? mt[3] : mt[1]);
    const bool m0 = a >= t0;
    m = (m2 << 2) | (m1 << 1) | m0;
    margin = fminf(fminf(a, fabsf(a - mt[4])), fminf(fabsf(a - t1), fabsf(a - t0)));
  }
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  const __half2 h = *reinterpret_cast<const __half2*>(&v);
  return __half22float2(h);
}

template <typename TIn>
__device__ __forceinline__ void load_row(const TIn* __restrict__ xr, float* v, int D, const uint32_t* dm);

// --------------------------------------------------------- exact fp64 row
// Warp-cooperative fp64 evaluation of one row (all decisions exact up to
// ties at ~1e-16), writing every output of the row.
template <int D, typename TIn>
__device__ void exact_row_fp64(const tq_params& p, const QBook& qb, const TIn* __restrict__ xr, int64_t row,
                               const tq_compressed& out, double* scratch) {
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  double v[VPL];
  double ss = 0.0;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    v[k] = (double)tq_to_f32(xr[lane + 32 * k]);
    ss = fma(v[k], v[k], ss);
  }
  ss = tq_warp_sum(ss);
  const double nu = sqrt(ss);
  const double inv = nu > 0.0 ? 1.0 / nu : 0.0;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const double u = v[k] * inv;
    v[k] = tq_dneg(p.dbits, k, lane) ? -u : u;
  }
  tq_fwht_warp<VPL>(v, lane);  // v = z = H (D u) (p = d here)
  const double isd = 1.0 / sqrt((double)D);
  int code[VPL];
  double g2 = 0.0;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int s = (p.nseg == 2 && k >= VPL / 2) ? 1 : 0;
    const int nb = (1 << p.bits[s]) - 1;
    int c = 0;
    for (int b = 0; b < nb; ++b) c += (v[k] >= (double)qb.bnd[s][b]) ? 1 : 0;
    code[k] = c;
    const double r = (v[k] - (double)qb.cen[s][c]) * isd;
    scratch[lane + 32 * k] = r;
    g2 = fma(r, r, g2);
  }
  g2 = tq_warp_sum(g2);
  __syncwarp();
  const int Q = p.MS;
  uint32_t signword = 0;
  for (int q = 0; q < Q; ++q) {
    const float* sc = p.St + lane * Q + q;
    double t = 0.0;
    for (int i = 0; i < D; ++i) t = fma((double)__ldg(sc + (size_t)i * p.m), scratch[i], t);
    const uint32_t wv = __ballot_sync(TQ_FULL_MASK, t >= 0.0);
    if (lane == q) signword = wv;
  }
  __syncwarp();
  // pack: coordinate j = lane + 32k is bit `lane` of word k of its plane
  constexpr int SLOTS = (VPL * 4 + 31) / 32;
  uint32_t cw[SLOTS];
#pragma unroll
  for (int sl = 0; sl < SLOTS; ++sl) cw[sl] = 0;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
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
  uint32_t* orow = out.codes + row * p.W;
#pragma unroll
  for (int sl = 0; sl < SLOTS; ++sl)
    if (sl * 32 + lane < p.W) orow[sl * 32 + lane] = cw[sl];
  if (Q > 0) {
    if (lane < Q) out.signs[row * Q + lane] = signword;
    if (lane == 0) out.rnorms[row] = (float)sqrt(g2);
  }
  if (lane == 0) out.norms[row] = (float)nu;
}

// ---------------------------------------------------------------- kernel
template <int D, int B0, int B1, typename TIn>
__global__ void __launch_bounds__(kTile, 2)
    tq_quantize_tc_kernel(const tq_params p, const TIn* __restrict__ x, const int64_t n, const int64_t ld,
                          const tq_compressed out, const int64_t ntiles, const uint32_t tmem_cols) {
  constexpr int NSEG = B1 > 0 ? 2 : 1;
  constexpr int SEGLEN = D / NSEG;
  constexpr int PW = SEGLEN / 32;
  constexpr int W = (B0 + B1) * PW;
  constexpr int L = (D == 64) ? 6 : 7;
  constexpr int H0 = 1 << (B0 - 1);
  constexpr int H1 = B1 > 0 ? (1 << (B1 - 1)) : 1;

  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ QBook qb;
  __shared__ uint32_t s_dmask[D];
  __shared__ int s_list[kTile];
  __shared__ int s_count;
  __shared__ int s_abort;
  __shared__ uint64_t s_bar;
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int m = p.m;
  const bool sketch = m > 0;
  // shared layout: B image (2 m D halves) | sl1 [m] | sl2 [m] | fp64 scratch [4][D]
  uint16_t* s_bimg = reinterpret_cast<uint16_t*>(smem);
  float* s_sl1 = reinterpret_cast<float*>(smem + (size_t)4 * m * D);
  float* s_sl2 = s_sl1 + m;
  double* s_scr = reinterpret_cast<double*>(smem + (size_t)4 * m * D + (size_t)8 * m) + (size_t)warp * D;

  for (int i = tid; i < 2 * TQ_MAX_LEVELS; i += kTile) {
    qb.cen[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS] = p.cen[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS];
    qb.bnd[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS] = p.bnd[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS];
  }
  for (int i = tid; i < D; i += kTile) s_dmask[i] = __ldg(p.dmask + i);
  if (tid == 0) {
    s_count = 0;
    s_abort = 0;
  }
  if (sketch) {
    const uint4* src = reinterpret_cast<const uint4*>(p.bimg);
    uint4* dst = reinterpret_cast<uint4*>(s_bimg);
    for (int i = tid; i < m * D * 4 / 16; i += kTile) dst[i] = __ldg(src + i);
    for (int i = tid; i < m; i += kTile) {
      s_sl1[i] = __ldg(p.sl1n + i);
      s_sl2[i] = __ldg(p.sl2n + i);
    }
    if (tid == 0) {
      tqtc::mbar_init(&s_bar, 1);
      tqtc::fence_mbar_init();
    }
    if (warp == 0) tqtc::tmem_alloc(&s_tmem, tmem_cols);
    tqtc::fence_proxy_async_smem();
  }
  tqtc::tc_fence_before();
  __syncthreads();
  tqtc::tc_fence_after();
  const uint32_t tbase = sketch ? s_tmem : 0u;
  const uint32_t lane_base = (uint32_t)(warp * 32);
  const uint32_t col_lo = D / 2, col_d = D;
  uint32_t phase = 0;

  // positive boundaries qb.bnd[s][H + k - 1] (k >= 1) and positive centroids
  // qb.cen[s][H + m] are read from shared memory
  const float e_nu = (float)(D / 16 + 3) * kU;
  const float Bc = 1.1f * (e_nu + 2.f * kU);
  const float sqrtD = sqrtf((float)D);
  const float cmax = p.cmax;

  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t row = tile * kTile + tid;
    const bool valid = row < n;
    // ---------------------------------------------------------- load
    float v[D];
    if (valid) {
      const TIn* xr = x + row * ld;
      if constexpr (sizeof(TIn) == 2) {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 q = __ldg(reinterpret_cast<const uint4*>(xr) + c);
          const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int i = 8 * c + 2 * h;
            float lo, hi;
            if constexpr (std::is_same<TIn, __nv_bfloat16>::value) {
              lo = __uint_as_float((w4[h] << 16) ^ s_dmask[i]);
              hi = __uint_as_float((w4[h] & 0xFFFF0000u) ^ s_dmask[i + 1]);
            } else {
              const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[h]));
              lo = __uint_as_float(__float_as_uint(f.x) ^ s_dmask[i]);
              hi = __uint_as_float(__float_as_uint(f.y) ^ s_dmask[i + 1]);
            }
            v[i] = lo;
            v[i + 1] = hi;
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < D / 4; ++c) {
          const float4 q = __ldg(reinterpret_cast<const float4*>(xr) + c);
          v[4 * c + 0] = __uint_as_float(__float_as_uint(q.x) ^ s_dmask[4 * c + 0]);
          v[4 * c + 1] = __uint_as_float(__float_as_uint(q.y) ^ s_dmask[4 * c + 1]);
          v[4 * c + 2] = __uint_as_float(__float_as_uint(q.z) ^ s_dmask[4 * c + 2]);
          v[4 * c + 3] = __uint_as_float(__float_as_uint(q.w) ^ s_dmask[4 * c + 3]);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < D; ++i) v[i] = 0.f;
    }
    // ---------------------------------------------------------- norm
    float acc8[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) acc8[a] = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) acc8[i & 7] = fmaf(v[i], v[i], acc8[i & 7]);
    const float ss = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
    bool flag = !(ss >= 1e-30f && ss <= 1e30f);
    const float nu = sqrtf(ss);
    // ---------------------------------------------------------- FWHT (in registers)
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
      for (int i = 0; i < D; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
      }
    }
    // ---------------------------------------------------------- codes, residual
    float mt0[H0], mt1[H1];
    mt0[0] = mt1[0] = 0.f;
#pragma unroll
    for (int k = 1; k < H0; ++k) mt0[k] = nu * qb.bnd[0][H0 + k - 1];
#pragma unroll
    for (int k = 1; k < H1; ++k) mt1[k] = B1 > 0 ? nu * qb.bnd[1][H1 + k - 1] : 0.f;
    const float A = 1.1f * kU * (float)L * sqrtD * nu;
    float runmin = INFINITY;
    float g2 = 0.f;
    uint32_t cw[W];
#pragma unroll
    for (int k = 0; k < W; ++k) cw[k] = 0u;
    // fp16 scale of the residual: 2^-e with nu in [2^(e-1), 2^e)
    int e2;
    frexpf(nu > 0.f ? nu : 1.f, &e2);
    e2 = max(-125, min(125, e2));
    const float rscale = ldexpf(1.f, -e2);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t hi8[8], lo8[8];
#pragma unroll
      for (int ii = 0; ii < 16; ii += 2) {
        float r2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = c0 + ii + e;
          const bool seg1 = NSEG == 2 && i >= SEGLEN;
          const float w = v[i];
          const float a = fabsf(w);
          const bool pos = w >= 0.f;
          int mcell;
          float margin;
          if (seg1) {
            mag_search<(B1 > 0 ? B1 : 1)>(a, mt1, mcell, margin);
          } else {
            mag_search<B0>(a, mt0, mcell, margin);
          }
          const float cv = nu * (seg1 ? qb.cen[1][H1 + mcell] : qb.cen[0][H0 + mcell]);
          runmin = fminf(runmin, fmaf(-Bc, a, margin));
          const int bits = seg1 ? B1 : B0;
          const int il = seg1 ? i - SEGLEN : i;
          const int wbase = (seg1 ? B0 * PW : 0) + il / 32;
          const uint32_t bit = 1u << (il & 31);
          // plane bits: top plane = sign, lower planes = magnitude bits xor !sign
#pragma unroll
          for (int pl = 0; pl < 4; ++pl) {
            if (pl < bits) {
              bool b;
              if (pl == bits - 1)
                b = pos;
              else
                b = (((mcell >> pl) & 1) != 0) != !pos;
              if (b) cw[wbase + pl * PW] |= bit;
            }
          }
          const float r = w - copysignf(cv, w);
          g2 = fmaf(r, r, g2);
          r2[e] = r * rscale;
        }
        const uint32_t h = pack_half2(r2[0], r2[1]);
        const float2 hf = unpack_half2(h);
        hi8[ii / 2] = h;
        lo8[ii / 2] = pack_half2(r2[0] - hf.x, r2[1] - hf.y);
      }
      if (sketch) {
        tqtc::tmem_st8(tqtc::tmem_addr(tbase, lane_base, c0 / 2), hi8);
        tqtc::tmem_st8(tqtc::tmem_addr(tbase, lane_base, col_lo + c0 / 2), lo8);
      }
    }
    flag |= runmin <= A;
    // ---------------------------------------------------------- sketch
    uint32_t sw[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) sw[k] = 0u;
    if (sketch) {
      tqtc::tmem_wait_st();
      tqtc::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tqtc::tc_fence_after();
        const uint32_t idesc = tqtc::instr_desc(1, 0, 0, kTile, (uint32_t)m);
        const uint32_t lbo = 16u * (uint32_t)m, sbo = 128u;
        const uint32_t bhi = tqtc::smem_u32(s_bimg), blo = bhi + 2u * (uint32_t)m * D;
        const uint32_t dcol = tbase + col_d;
        bool accum = false;
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t acol = pass == 1 ? col_lo : 0u;
          const uint32_t bb = pass == 2 ? blo : bhi;
#pragma unroll
          for (int s = 0; s < D / 16; ++s) {
            tqtc::mma_f16_ts(dcol, tbase + acol + 8u * s, tqtc::smem_desc(bb + 2u * s * lbo, lbo, sbo), idesc, accum);
            accum = true;
          }
        }
        tqtc::mma_commit(&s_bar);
      }
      const bool ok = tqtc::mbar_wait(&s_bar, phase);
      phase ^= 1u;
      if (!ok) {
        atomicExch(p.err, (uint32_t)tqtc::kErrMmaWait);
        s_abort = 1;
      }
      tqtc::tc_fence_after();
      // bound of the residual error per coordinate, in scaled units
      const float Er = rscale * 1.1f * (kU * (float)L * sqrtD * nu + (e_nu + kU) * nu * cmax +
                                        kU * (sqrtD + cmax) * nu) +
                       4.8e-7f * (sqrtD + cmax) + 2.98e-8f;
      const float R2 = rscale * sqrtf(g2) * 1.00001f;
      const float beta = 1.1f * (4.3e-6f * R2);
      const float gam0 = 1.1f * 2.98e-8f * sqrtD * R2;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c >= m / 32) break;
        uint32_t t16[2][16];
        tqtc::tmem_ld16(tqtc::tmem_addr(tbase, lane_base, col_d + 32 * c), t16[0]);
        tqtc::tmem_ld16(tqtc::tmem_addr(tbase, lane_base, col_d + 32 * c + 16), t16[1]);
        tqtc::tmem_wait_ld();
        uint32_t word = 0;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const float t = __uint_as_float(t16[jj >> 4][jj & 15]);
          const int j = 32 * c + jj;
          const float tau = 1.1f * s_sl1[j] * Er + beta * s_sl2[j] + gam0;
          flag |= !(fabsf(t) > tau);
          word |= (t >= 0.f ? 1u : 0u) << jj;
        }
        sw[c] = word;
      }
    }
    // ---------------------------------------------------------- store / defer
    if (valid) {
      if (!flag) {
        uint32_t* orow = out.codes + row * W;
        if constexpr (W % 4 == 0) {
#pragma unroll
          for (int k = 0; k < W; k += 4) *reinterpret_cast<uint4*>(orow + k) = make_uint4(cw[k], cw[k + 1], cw[k + 2], cw[k + 3]);
        } else if constexpr (W % 2 == 0) {
#pragma unroll
          for (int k = 0; k < W; k += 2) *reinterpret_cast<uint2*>(orow + k) = make_uint2(cw[k], cw[k + 1]);
        } else {
#pragma unroll
          for (int k = 0; k < W; ++k) orow[k] = cw[k];
        }
        out.norms[row] = nu;
        if (sketch) {
          const int MS = m / 32;
          uint32_t* srow = out.signs + row * MS;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (k < MS) srow[k] = sw[k];
          out.rnorms[row] = sqrtf(g2) / (nu * sqrtD);
        }
      } else {
        s_list[atomicAdd(&s_count, 1)] = tid;
      }
    }
    tqtc::tc_fence_before();
    __syncthreads();
    if (s_abort) break;
    // ---------------------------------------------------------- fp64 re-evaluation
    const int cnt = s_count;
    if (tid == 0 && cnt > 0) atomicAdd(p.exact_rows, (unsigned long long)cnt);
    for (int e = warp; e < cnt; e += kTile / 32) {
      const int64_t r = tile * kTile + s_list[e];
      exact_row_fp64<D, TIn>(p, qb, x + r * ld, r, out, s_scr);
    }
    __syncthreads();
    if (tid == 0) s_count = 0;
    __syncthreads();
    tqtc::tc_fence_after();
  }
  tqtc::tc_fence_before();
  __syncthreads();
  if (sketch && warp == 0) tqtc::tmem_dealloc(tbase, tmem_cols);
}

template <typename Fn>
cudaError_t set_smem_attr(Fn* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

int g_sms = 0;
int sm_count() {
  if (!g_sms) {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_sms = v;
  }
  return g_sms;
}

template <int D, int B0, int B1, typename TIn>
cudaError_t launch_tc(const tq_params& p, const void* x, int64_t n, int64_t ld, const tq_compressed& out,
                      cudaStream_t st) {
  const int m = p.m;
  const size_t smem = (size_t)4 * m * D + (size_t)8 * m + (size_t)4 * D * sizeof(double);
  auto fn = tq_quantize_tc_kernel<D, B0, B1, TIn>;
  cudaError_t e = set_smem_attr(fn, smem);
  if (e != cudaSuccess) return e;
  uint32_t cols = 32;
  while (cols < (uint32_t)(D + m)) cols <<= 1;
  const int64_t ntiles = (n + kTile - 1) / kTile;
  // at most two resident blocks per SM (TMEM: 2 x cols <= 512)
  const int per_sm = (m > 0 && cols > 256) ? 1 : 2;
  const int grid = (int)std::min<int64_t>(ntiles, (int64_t)sm_count() * per_sm);
  fn<<<grid, kTile, smem, st>>>(p, (const TIn*)x, n, ld, out, ntiles, cols);
  return cudaGetLastError();
}

template <int D, typename TIn>
cudaError_t dispatch_bits(const tq_params& p, const void* x, int64_t n, int64_t ld, const tq_compressed& out,
                          cudaStream_t st) {
  if (p.nseg == 1) {
    switch (p.bits[0]) {
      case 1: return launch_tc<D, 1, 0, TIn>(p, x, n, ld, out, st);
      case 2: return launch_tc<D, 2, 0, TIn>(p, x, n, ld, out, st);
      case 3: return launch_tc<D, 3, 0, TIn>(p, x, n, ld, out, st);
      case 4: return launch_tc<D, 4, 0, TIn>(p, x, n, ld, out, st);
    }
  } else if (p.bits[0] == 2 && p.bits[1] == 3) {
    return launch_tc<D, 2, 3, TIn>(p, x, n, ld, out, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t tq_launch_quantize_tc(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                  const tq_compressed& out, cudaStream_t st) {
  if (p.m > 256 || (p.m > 0 && p.m % 32 != 0)) return cudaErrorNotSupported;
  if (dt != TQ_BF16 && dt != TQ_F32) return cudaErrorNotSupported;
  if (p.d == 128) {
    return dt == TQ_BF16 ? dispatch_bits<128, __nv_bfloat16>(p, x, n, ld, out, st)
                         : dispatch_bits<128, float>(p, x, n, ld, out, st);
  }
  if (p.d == 64) {
    return dt == TQ_BF16 ? dispatch_bits<64, __nv_bfloat16>(p, x, n, ld, out, st)
                         : dispatch_bits<64, float>(p, x, n, ld, out, st);
  }
  return cudaErrorNotSupported;
}
