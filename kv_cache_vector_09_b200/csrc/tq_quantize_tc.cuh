// Tensor-core quantiser for d in {64, 128}.
//
// A block owns tiles of 128 rows; TPR = d/32 threads share a row (4 for
// d = 128), each holding 32 coordinates: chunks c = q + TPR k (k < 4) of 8
// consecutive coordinates, q = thread index within the row.  Per row:
//   load x (16-byte loads, a quad covers 64 contiguous bytes), apply the D
//   signs, Walsh-Hadamard transform of the unnormalised w = H (D x) (five
//   in-register butterfly stages over the chunk/element bits, log2 TPR
//   shuffle stages over the thread bits), quantise every coordinate against the
//   boundaries scaled by the fp32 norm (z >= bnd <=> w >= nu bnd) with a
//   magnitude binary search, pack the bit planes into a shared-memory staging
//   row, and (keys) form the residual r = w - nu cen[code] as fp16 hi + lo in
//   the tensor-core operand layout.
// The QJL sketch t = S r of the tile is one kind::f16 tcgen05.mma product
// (A = residual tile, B = fp16 hi + lo image of S, both in shared memory;
// passes hi*hi + lo*hi + hi*lo) with an fp32 accumulator in TMEM, read back by
// the warps one 32-column sign word at a time.
//
// Certified decisions (u = 2^-24, L = log2 d, nu the fp32 norm):
//   code  : |w_i - nu bnd| > A + B |w_i| with A = 1.1 L u sqrt(d) nu (fp32 FWHT
//           rounding: each stage's nodes partition the inputs, and
//           ||x||_1 <= sqrt(d) nu), B = 1.1 (e_nu + 2u), e_nu = 10u
//   sign  : |t_j| > ||S_j||_2 E + G, where E bounds ||dr||_2 of the scaled
//           residual (FWHT: ||dw||_2 <= L u sqrt(d) nu, since every stage's
//           rounding vector has norm <= u ||v_stage|| and the remaining
//           butterflies scale norms by exactly sqrt(2) each; norm error
//           (e_nu + u) ||cv||_2; subtraction u ||r||_2; fp16 split 2^-22 ||r||
//           + 2^-25 sqrt(d)) plus the tensor-core terms (S split 2^-22, omitted
//           lo*lo 2^-22, fp32 accumulation <= 2^-18 of sum |S r|) times ||r||.
// A row with an uncertain code is recomputed entirely in fp64; a row with only
// uncertain signs gets those sketch rows recomputed in fp64 (exact residual).
#pragma once

#include <math.h>

#include <algorithm>
#include <type_traits>

#include "tq_common.cuh"
#include "tq_tc.cuh"

namespace {

constexpr int kRows = 128;                     // rows per tile (= MMA M)
constexpr float kU = 5.9604644775390625e-08f;  // 2^-24

struct QBook {
  float cen[2][TQ_MAX_LEVELS];
  float bnd[2][TQ_MAX_LEVELS];
};

// Magnitude search: a = |w|, mt[k] = nu * (k-th positive boundary), k >= 1,
// one binary-search step per magnitude bit.  Returns the distance to the
// nearest compared boundary (the zero boundary included; the compared
// boundaries include both ends of the final cell) and, for each magnitude bit
// p, the difference dd[p] = a - (boundary compared for bit p) and the bit
// itself, mb[p] = (dd[p] >= 0), i.e. a >= that boundary.  For finite a the
// sign bit of dd[p] is the complement of mb[p]: a - t rounds to zero only when
// a == t, and then to +0.
template <int BITS>
__device__ __forceinline__ void mag_diff(float a, const float* mt, float* dd, bool* mb, float& margin) {
  if constexpr (BITS == 1) {
    margin = a;
  } else if constexpr (BITS == 2) {
    dd[0] = a - mt[1];
    mb[0] = dd[0] >= 0.f;
    margin = fminf(a, fabsf(dd[0]));
  } else if constexpr (BITS == 3) {
    dd[1] = a - mt[2];
    mb[1] = dd[1] >= 0.f;
    dd[0] = a - (mb[1] ? mt[3] : mt[1]);
    mb[0] = dd[0] >= 0.f;
    margin = fminf(a, fminf(fabsf(dd[1]), fabsf(dd[0])));
  } else {
    dd[2] = a - mt[4];
    mb[2] = dd[2] >= 0.f;
    dd[1] = a - (mb[2] ? mt[6] : mt[2]);
    mb[1] = dd[1] >= 0.f;
    dd[0] = a - (mb[2] ? (mb[1] ? mt[7] : mt[5]) : (mb[1] ? mt[3] : mt[1]));
    mb[0] = dd[0] >= 0.f;
    margin = fminf(fminf(a, fabsf(dd[2])), fminf(fabsf(dd[1]), fabsf(dd[0])));
  }
}

// Magnitude of the centroid of cell (mb) from ct[k] = nu * (k-th positive
// centroid), by selects (BITS <= 3).
template <int BITS>
__device__ __forceinline__ float sel_cen(const bool* mb, const float* ct) {
  if constexpr (BITS == 1) {
    return ct[0];
  } else if constexpr (BITS == 2) {
    return mb[0] ? ct[1] : ct[0];
  } else {
    const float hi = mb[0] ? ct[3] : ct[2];
    const float lo = mb[0] ? ct[1] : ct[0];
    return mb[1] ? hi : lo;
  }
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// packed f32x2 arithmetic (two fp32 lanes in one 64-bit register)
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  return (uint64_t)__float_as_uint(a) | ((uint64_t)__float_as_uint(b) << 32);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// acc += a * b
__device__ __forceinline__ void fma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
// a * b + c
__device__ __forceinline__ uint64_t fma2r(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// Shared-memory layout of one block (all offsets 16-byte aligned).
struct QLayout {
  uint32_t a_hi, a_lo, bimg, sl2n, codes, signs, nu, gam, err, flag, fmask, scratch, total;
  __host__ __device__ QLayout(int D, int m, int W, int nwarps) {
    uint32_t o = 0;
    const uint32_t atile = m > 0 ? (uint32_t)kRows * D * 2 : 0;
    a_hi = o; o += atile;
    a_lo = o; o += atile;
    bimg = o; o += (uint32_t)m * D * 4;
    sl2n = o; o += (uint32_t)((m * 4 + 15) / 16 * 16);
    codes = o; o += (uint32_t)kRows * W * 4;
    signs = o; o += (uint32_t)kRows * 8 * 4;
    nu = o; o += kRows * 4;
    gam = o; o += kRows * 4;
    err = o; o += kRows * 8;       // per row: E, G of the sign bound
    flag = o; o += kRows * 4;      // per row: 1 = uncertain sign(s), 2 = uncertain code / range
    fmask = o; o += kRows * 8 * 4; // per row: uncertain sign bits
    scratch = o; o += (uint32_t)nwarps * D * 8;
    total = (o + 127) & ~127u;
  }
};

// ------------------------------------------------------------ exact fp64
// Warp-cooperative fp64 evaluation of one row, written straight to the
// outputs.  full: every code, sign, nu and gamma is rewritten; otherwise the
// codes are certified and only the sign bits in fmask (plus nu and gamma) are.
// Position of input row `row` for the fused RoPE (0, and an error code in the
// device error word, when it lies outside the cos/sin cache).
__device__ __forceinline__ int rope_position(const tq_params& p, int64_t row, bool valid) {
  int pos = p.rope_pos ? (valid ? __ldg(p.rope_pos + row) : 0) : p.rope_pos_fixed;
  if (pos < 0 || pos >= p.rope_max_pos) {
    if (valid) atomicExch(p.err, tqtc::kErrRopePosition);
    pos = 0;
  }
  return pos;
}

// Rotate-half RoPE of the pair (a, b) = (x_i, x_{i+d/2}) with c = cos, s = sin
// of the position angle, in fp32 with a fixed operation order: the fast path
// and the fp64 re-evaluation of a row both start from these same values.
__device__ __forceinline__ void rope_pair(float& a, float& b, float c, float s) {
  const float x = a, y = b;
  a = __fmaf_rn(x, c, -__fmul_rn(y, s));
  b = __fmaf_rn(x, s, __fmul_rn(y, c));
}

template <int D, typename TIn, bool SK, bool ROPE>
__device__ void exact_row(const tq_params& p, const QBook& qb, const TIn* __restrict__ xr, int64_t row, bool full,
                          const uint32_t* fmask, const tq_compressed& out, double* scratch) {
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t orow = row * p.out_stride + p.out_offset;  // compressed row written
  float xf[VPL];
#pragma unroll
  for (int k = 0; k < VPL; ++k) xf[k] = tq_to_f32(xr[lane + 32 * k]);
  if constexpr (ROPE) {
    // coordinate lane + 32k pairs with lane + 32k + D/2, i.e. k + VPL/2
    const float* cs = p.rope_cs + (size_t)rope_position(p, row, true) * D;
#pragma unroll
    for (int k = 0; k < VPL / 2; ++k)
      rope_pair(xf[k], xf[k + VPL / 2], __ldg(cs + lane + 32 * k), __ldg(cs + D / 2 + lane + 32 * k));
  }
  double v[VPL];
  double ss = 0.0;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    v[k] = (double)xf[k];
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
  tq_fwht_warp<VPL>(v, lane);  // z = H (D u)
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
  const int MS = SK ? p.MS : 0;
  if (SK && full) {
    // every sketch row: lane owns rows lane + 32 q, reading S^T (columns
    // permuted so that lane l's q-th column is row l + 32 q) coalesced
    double t[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) t[q] = 0.0;
    for (int i = 0; i < D; ++i) {
      const double ri = scratch[i];
      const float* sti = p.St + (size_t)i * p.m + lane * MS;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < MS) t[q] = fma((double)__ldg(sti + q), ri, t[q]);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < MS) {
        const uint32_t word = __ballot_sync(TQ_FULL_MASK, t[q] >= 0.0);
        if (lane == 0) out.signs[orow * MS + q] = word;
      }
    }
  }
  // flagged sketch rows only: t_j = sum_i S_ji r_i, lanes split i, warp reduction
  for (int w = 0; SK && w < MS && !full; ++w) {
    uint32_t todo = full ? 0xffffffffu : fmask[w];
    if (!todo) continue;
    uint32_t word = full ? 0u : out.signs[orow * MS + w];
    while (todo) {
      const int jj = __ffs(todo) - 1;
      todo &= todo - 1;
      const float* Sj = p.S + (size_t)(32 * w + jj) * D;
      double t = 0.0;
#pragma unroll
      for (int k = 0; k < VPL; ++k) t = fma((double)__ldg(Sj + lane + 32 * k), scratch[lane + 32 * k], t);
      t = tq_warp_sum(t);
      word = (word & ~(1u << jj)) | ((t >= 0.0 ? 1u : 0u) << jj);
    }
    if (lane == 0) out.signs[orow * MS + w] = word;
  }
  if (full) {
    // coordinate j = lane + 32k is bit `lane` of word k of its plane
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int s = (p.nseg == 2 && k >= VPL / 2) ? 1 : 0;
      const int kk = s ? k - VPL / 2 : k;
      for (int pl = 0; pl < p.bits[s]; ++pl) {
        const uint32_t wv = __ballot_sync(TQ_FULL_MASK, (code[k] >> pl) & 1);
        if (lane == 0) out.codes[orow * p.W + p.segbase[s] + pl * p.pw + kk] = wv;
      }
    }
  }
  if (lane == 0) {
    out.norms[orow] = (float)nu;
    if (MS > 0) out.rnorms[orow] = p.rnorm_is_const ? p.rnorm_const : (float)sqrt(g2);
  }
  __syncwarp();
}

struct FixEntry {
  int64_t row;
  int full;
  uint32_t fmask[8];
};
constexpr int kFixCap = 256;

// ---------------------------------------------------------------- kernel
template <int D, int B0, int B1, bool SK, typename TIn, bool ROPE>
__global__ void __launch_bounds__(kRows * (D / 32), SK ? 1 : 2)
    tq_quantize_quad_kernel(const tq_params p, const TIn* __restrict__ x, const int64_t n, const int64_t ld,
                            const tq_compressed out, const int64_t ntiles, const uint32_t tmem_cols) {
  constexpr int TPR = D / 32;
  constexpr int NT = kRows * TPR;
  constexpr int NW = NT / 32;
  constexpr int NSEG = B1 > 0 ? 2 : 1;
  constexpr int NCH = D / 8;
  constexpr int CHSEG = NCH / NSEG;
  constexpr int PW = (D / NSEG) / 32;
  constexpr int W = (B0 + B1) * PW;
  constexpr int L = (D == 64) ? 6 : 7;
  constexpr int H0 = 1 << (B0 - 1);
  constexpr int H1 = B1 > 0 ? (1 << (B1 - 1)) : 1;
  constexpr int LBO_A = (kRows / 8) * 128;

  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ QBook qb;
  __shared__ __align__(16) uint32_t s_dmask[D];
  __shared__ FixEntry s_fix[kFixCap];
  __shared__ int s_nfix;
  __shared__ int s_abort;
  __shared__ uint64_t s_bar;
  __shared__ uint32_t s_tmem;

  const int m = SK ? p.m : 0;
  const QLayout ly(D, m, W, NW);
  uint32_t* st_codes = reinterpret_cast<uint32_t*>(smem + ly.codes);
  uint32_t* st_signs = reinterpret_cast<uint32_t*>(smem + ly.signs);
  float* st_nu = reinterpret_cast<float*>(smem + ly.nu);
  float* st_gam = reinterpret_cast<float*>(smem + ly.gam);
  float2* st_err = reinterpret_cast<float2*>(smem + ly.err);
  int* st_flag = reinterpret_cast<int*>(smem + ly.flag);
  uint32_t* st_fmask = reinterpret_cast<uint32_t*>(smem + ly.fmask);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = tid / TPR, q = tid % TPR;

  for (int i = tid; i < 2 * TQ_MAX_LEVELS; i += NT) {
    qb.cen[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS] = p.cen[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS];
    qb.bnd[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS] = p.bnd[i / TQ_MAX_LEVELS][i % TQ_MAX_LEVELS];
  }
  for (int i = tid; i < D; i += NT) s_dmask[i] = __ldg(p.dmask + i);
  for (int i = tid; i < kRows; i += NT) st_flag[i] = 0;
  if (tid == 0) {
    s_nfix = 0;
    s_abort = 0;
  }
  if constexpr (SK) {
    const uint4* src = reinterpret_cast<const uint4*>(p.bimg);
    uint4* dst = reinterpret_cast<uint4*>(smem + ly.bimg);
    if (m <= 128) {
      // one B operand of N = 2m rows, [S_hi; S_lo]: 16-byte chunk `rest` of
      // K chunk i8 of half h goes to i8 * 2m + h * m + rest
      for (int i = tid; i < m * D * 4 / 16; i += NT) {
        const int h = i / (m * D / 8), c = i % (m * D / 8);
        dst[(c / m) * 2 * m + h * m + c % m] = __ldg(src + i);
      }
    } else {
      for (int i = tid; i < m * D * 4 / 16; i += NT) dst[i] = __ldg(src + i);
    }
    for (int i = tid; i < m; i += NT) reinterpret_cast<float*>(smem + ly.sl2n)[i] = __ldg(p.sl2n + i);
    if (tid == 0) {
      tqtc::mbar_init(&s_bar, 1);
      tqtc::fence_mbar_init();
    }
    if (warp == 0) tqtc::tmem_alloc(&s_tmem, tmem_cols);
  }
  tqtc::tc_fence_before();
  __syncthreads();
  tqtc::tc_fence_after();
  const uint32_t tbase = SK ? s_tmem : 0u;
  uint32_t phase = 0;
  const float e_nu = 10.f * kU;
  const float Bc = 1.1f * (e_nu + 2.f * kU);
  const float sqrtD = sqrtf((float)D);
  const float sgn1 = (q & 1) ? -1.f : 1.f;
  const float sgn2 = (q & 2) ? -1.f : 1.f;
  double* scr = reinterpret_cast<double*>(smem + ly.scratch) + (size_t)warp * D;
  // fp64 re-evaluation of the queued rows, all warps at once (after the fast
  // path of those rows has been written and made visible by a barrier)
  auto drain = [&]() {
    const int cnt = min(s_nfix, kFixCap);
    if (tid == 0 && cnt > 0) atomicAdd(p.exact_rows, (unsigned long long)cnt);
    for (int e = warp; e < cnt; e += NW) {
      const FixEntry& f = s_fix[e];
      exact_row<D, TIn, SK, ROPE>(p, qb, x + f.row * ld, f.row, f.full != 0, f.fmask, out, scr);
    }
    __syncthreads();
    if (tid == 0) s_nfix = 0;
    __syncthreads();
  };

  // prefetch of the first tile's rows
  using Raw = typename std::conditional<sizeof(TIn) == 2, uint4, float4>::type;
  constexpr int NRAW = sizeof(TIn) == 2 ? 4 : 8;
  Raw raw[NRAW];
  auto fetch = [&](int64_t t) {
    const int64_t rw = t * kRows + r;
    if (t < ntiles && rw < n) {
      const TIn* xr = x + rw * ld;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = q + TPR * k;
        if constexpr (sizeof(TIn) == 2) {
          raw[k] = __ldg(reinterpret_cast<const uint4*>(xr + 8 * c));
        } else {
          raw[2 * k] = __ldg(reinterpret_cast<const float4*>(xr + 8 * c));
          raw[2 * k + 1] = __ldg(reinterpret_cast<const float4*>(xr + 8 * c + 4));
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < NRAW; ++k) raw[k] = Raw{0, 0, 0, 0};
    }
  };
  fetch(blockIdx.x);

  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t row0 = tile * kRows;
    const int64_t row = row0 + r;
    const bool valid = row < n;
    // ---------------------------------------------------------------- load
    float v[32];
    {
      Raw cur[NRAW];
#pragma unroll
      for (int k = 0; k < NRAW; ++k) cur[k] = raw[k];
      fetch(tile + gridDim.x);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = q + TPR * k;
        const uint4 dm0 = *reinterpret_cast<const uint4*>(s_dmask + 8 * c);
        const uint4 dm1 = *reinterpret_cast<const uint4*>(s_dmask + 8 * c + 4);
        // with the fused RoPE the D signs come after the rotation (below)
        const uint32_t dm[8] = {ROPE ? 0u : dm0.x, ROPE ? 0u : dm0.y, ROPE ? 0u : dm0.z, ROPE ? 0u : dm0.w,
                                ROPE ? 0u : dm1.x, ROPE ? 0u : dm1.y, ROPE ? 0u : dm1.z, ROPE ? 0u : dm1.w};
        if constexpr (sizeof(TIn) == 2) {
          const uint4 qd = *reinterpret_cast<const uint4*>(&cur[k]);
          const uint32_t w4[4] = {qd.x, qd.y, qd.z, qd.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[8 * k + 2 * h] = __uint_as_float((w4[h] << 16) ^ dm[2 * h]);
            v[8 * k + 2 * h + 1] = __uint_as_float((w4[h] & 0xFFFF0000u) ^ dm[2 * h + 1]);
          }
        } else {
          const float4 a = *reinterpret_cast<const float4*>(&cur[2 * k]);
          const float4 b = *reinterpret_cast<const float4*>(&cur[2 * k + 1]);
          const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) v[8 * k + e] = __uint_as_float(__float_as_uint(f[e]) ^ dm[e]);
        }
      }
    }
    if constexpr (ROPE) {
      // rotate-half RoPE, pairs (i, i + D/2): chunk c = q + TPR k (k < 2) holds
      // coordinates 8c.. of the first half and chunk c + D/16 = q + TPR (k + 2)
      // their partners, so every pair lies in this thread's registers
      const float* cs = p.rope_cs + (size_t)rope_position(p, row, valid) * D;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int c = q + TPR * k;
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(cs + 8 * c));
        const float4 c1 = __ldg(reinterpret_cast<const float4*>(cs + 8 * c + 4));
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(cs + D / 2 + 8 * c));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(cs + D / 2 + 8 * c + 4));
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) rope_pair(v[8 * k + e], v[8 * (k + 2) + e], cv[e], sv[e]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = q + TPR * k;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * k + e] = __uint_as_float(__float_as_uint(v[8 * k + e]) ^ s_dmask[8 * c + e]);
      }
    }
    // ---------------------------------------------------------------- norm, FWHT
    // Two spellings of the same arithmetic: packed f32x2 pairs (fewer
    // instructions) for the kernels without a sketch, scalar for the sketch
    // kernels, whose register budget the pairs would overrun.
    float nu;
    bool codeflag;
    if constexpr (!SK) {
      // values in packed pairs (v[2k], v[2k+1]) for f32x2 arithmetic; every
      // lane of a packed op rounds like the scalar op, so results are the same
      uint64_t P[16];
  #pragma unroll
      for (int k = 0; k < 16; ++k) P[k] = pk2(v[2 * k], v[2 * k + 1]);
      uint64_t s01 = 0ull, s23 = 0ull;  // partial sums of v_i^2 over i mod 4
  #pragma unroll
      for (int k = 0; k < 16; k += 2) {
        fma2(s01, P[k], P[k]);
        fma2(s23, P[k + 1], P[k + 1]);
      }
      float ss = (lo2(s01) + hi2(s01)) + (lo2(s23) + hi2(s23));
      ss += __shfl_xor_sync(TQ_FULL_MASK, ss, 1);
      if constexpr (TPR == 4) ss += __shfl_xor_sync(TQ_FULL_MASK, ss, 2);
      codeflag = !(ss >= 1e-30f && ss <= 1e30f);
      nu = sqrtf(ss);
      // ---------------------------------------------------------------- FWHT
      // stage h = 1 inside each pair, stages h = 2..16 between pairs, then the
      // thread-bit stages across the row's threads
  #pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float a = lo2(P[k]), b = hi2(P[k]);
        P[k] = pk2(a + b, a - b);
      }
  #pragma unroll
      for (int hp = 1; hp < 16; hp <<= 1) {
  #pragma unroll
        for (int k = 0; k < 16; ++k) {
          if ((k & hp) == 0) {
            const uint64_t a = P[k], b = P[k + hp];
            P[k] = add2(a, b);
            P[k + hp] = sub2(a, b);
          }
        }
      }
      {
        const uint64_t g1 = pk2(sgn1, sgn1);
  #pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint64_t o = pk2(__shfl_xor_sync(TQ_FULL_MASK, lo2(P[k]), 1), __shfl_xor_sync(TQ_FULL_MASK, hi2(P[k]), 1));
          P[k] = fma2r(g1, P[k], o);
        }
        if constexpr (TPR == 4) {
          const uint64_t g2 = pk2(sgn2, sgn2);
  #pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint64_t o =
                pk2(__shfl_xor_sync(TQ_FULL_MASK, lo2(P[k]), 2), __shfl_xor_sync(TQ_FULL_MASK, hi2(P[k]), 2));
            P[k] = fma2r(g2, P[k], o);
          }
        }
      }
  #pragma unroll
      for (int k = 0; k < 16; ++k) {
        v[2 * k] = lo2(P[k]);
        v[2 * k + 1] = hi2(P[k]);
      }
    } else {
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
  #pragma unroll
      for (int i = 0; i < 32; ++i) a4[i & 3] = fmaf(v[i], v[i], a4[i & 3]);
      float ss = (a4[0] + a4[1]) + (a4[2] + a4[3]);
      ss += __shfl_xor_sync(TQ_FULL_MASK, ss, 1);
      if constexpr (TPR == 4) ss += __shfl_xor_sync(TQ_FULL_MASK, ss, 2);
      codeflag = !(ss >= 1e-30f && ss <= 1e30f);
      nu = sqrtf(ss);
      // ---------------------------------------------------------------- FWHT
  #pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
  #pragma unroll
        for (int i = 0; i < 32; ++i) {
          if ((i & h) == 0) {
            const float a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
          }
        }
      }
  #pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = fmaf(sgn1, v[i], __shfl_xor_sync(TQ_FULL_MASK, v[i], 1));
      if constexpr (TPR == 4) {
  #pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = fmaf(sgn2, v[i], __shfl_xor_sync(TQ_FULL_MASK, v[i], 2));
      }
    }
    // ---------------------------------------------------------------- codes
    float mt0[H0], mt1[H1];
    mt0[0] = mt1[0] = 0.f;
#pragma unroll
    for (int k = 1; k < H0; ++k) mt0[k] = nu * qb.bnd[0][H0 + k - 1];
#pragma unroll
    for (int k = 1; k < H1; ++k) mt1[k] = nu * qb.bnd[1][H1 + k - 1];
    const float A = 1.1f * kU * (float)L * sqrtD * nu;
    int frexp_e;
    frexpf(nu > 0.f ? nu : 1.f, &frexp_e);
    frexp_e = max(-125, min(125, frexp_e));
    const float rscale = ldexpf(1.f, -frexp_e);
    float runmin = INFINITY, g2 = 0.f, cv2 = 0.f;
    // centroid magnitudes nu * cen for the sketch's residual, picked by
    // selects where the codebook has at most 4 positive cells
    constexpr bool kSel0 = B0 <= 3, kSel1 = B1 <= 3;
    float ct0[SK && kSel0 ? H0 : 1], ct1[SK && kSel1 ? H1 : 1];
    if constexpr (SK && kSel0) {
#pragma unroll
      for (int k = 0; k < H0; ++k) ct0[k] = nu * qb.cen[0][H0 + k];
    }
    if constexpr (SK && kSel1 && B1 > 0) {
#pragma unroll
      for (int k = 0; k < H1; ++k) ct1[k] = nu * qb.cen[1][H1 + k];
    }
    unsigned char* crow = reinterpret_cast<unsigned char*>(st_codes + r * W);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = q + TPR * k;
      const bool seg1 = NSEG == 2 && c >= CHSEG;
      const int cs = seg1 ? c - CHSEG : c;
      // Plane bits are gathered most recent first with funnel shifts of sign
      // bits (value e ends at bit 7 - e, reversed below): plane p below the
      // top is (mag bit p) xor (w < 0), the sign bit of dd[p] ^ w inverted;
      // the top plane is w >= 0, the sign bit of w inverted.  A coordinate
      // with w == -0 has a == 0, so its row fails the margin test and is
      // recomputed exactly; the sign bit stands for w < 0 everywhere else.
      uint32_t pb[4] = {0u, 0u, 0u, 0u};
      float rr[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float w = v[8 * k + e];
        const float a = fabsf(w);
        const uint32_t wu = __float_as_uint(w);
        float dd[3];
        bool mb[3];
        float margin;
        if (seg1) {
          mag_diff<(B1 > 0 ? B1 : 1)>(a, mt1, dd, mb, margin);
        } else {
          mag_diff<B0>(a, mt0, dd, mb, margin);
        }
        runmin = fminf(runmin, fmaf(-Bc, a, margin));
        const int bits = seg1 ? B1 : B0;
#pragma unroll
        for (int pl = 0; pl < 4; ++pl) {
          if (pl < bits - 1) pb[pl] = __funnelshift_l(__float_as_uint(dd[pl]) ^ wu, pb[pl], 1);
          if (pl == bits - 1) pb[pl] = __funnelshift_l(wu, pb[pl], 1);
        }
        if constexpr (SK) {
          float cvv;
          if (seg1) {
            if constexpr (kSel1) {
              cvv = sel_cen<(B1 > 0 ? B1 : 1)>(mb, ct1);
            } else {
              int mc = 0;
#pragma unroll
              for (int b = 0; b < (B1 > 0 ? B1 : 1) - 1; ++b) mc |= (mb[b] ? 1 : 0) << b;
              cvv = nu * qb.cen[1][H1 + mc];
            }
          } else {
            if constexpr (kSel0) {
              cvv = sel_cen<B0>(mb, ct0);
            } else {
              int mc = 0;
#pragma unroll
              for (int b = 0; b < B0 - 1; ++b) mc |= (mb[b] ? 1 : 0) << b;
              cvv = nu * qb.cen[0][H0 + mc];
            }
          }
          const float rv = w - copysignf(cvv, w);
          g2 = fmaf(rv, rv, g2);
          cv2 = fmaf(cvv, cvv, cv2);
          rr[e] = rv * rscale;
        }
      }
#pragma unroll
      for (int pl = 0; pl < 4; ++pl) pb[pl] = (__brev(pb[pl]) >> 24) ^ 0xFFu;
      const int bits = seg1 ? B1 : B0;
      const int wbase = seg1 ? B0 * PW : 0;
#pragma unroll
      for (int pl = 0; pl < 4; ++pl)
        if (pl < bits) crow[(wbase + pl * PW) * 4 + cs] = (unsigned char)pb[pl];
      if constexpr (SK) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const uint32_t h = pack_half2(rr[e], rr[e + 1]);
          const float2 hf = unpack_half2(h);
          hi[e / 2] = h;
          lo[e / 2] = pack_half2(rr[e] - hf.x, rr[e + 1] - hf.y);
        }
        const uint32_t off = (uint32_t)c * LBO_A + (uint32_t)(r / 8) * 128 + (uint32_t)(r % 8) * 16;
        *reinterpret_cast<uint4*>(smem + ly.a_hi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(smem + ly.a_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    codeflag |= runmin <= A;
    if (codeflag && valid) atomicOr(&st_flag[r], 2);
    if constexpr (SK) {
      g2 += __shfl_xor_sync(TQ_FULL_MASK, g2, 1);
      cv2 += __shfl_xor_sync(TQ_FULL_MASK, cv2, 1);
      if constexpr (TPR == 4) {
        g2 += __shfl_xor_sync(TQ_FULL_MASK, g2, 2);
        cv2 += __shfl_xor_sync(TQ_FULL_MASK, cv2, 2);
      }
    }
    if (q == 0) {
      st_nu[r] = nu;
      if constexpr (SK) {
        st_gam[r] = p.rnorm_is_const ? p.rnorm_const : sqrtf(g2) / (nu * sqrtD);
        const float R2 = rscale * sqrtf(g2) * 1.00001f;
        const float E = 1.1f * (rscale * 1.1f * (kU * (float)L * sqrtD * nu + (e_nu + kU) * sqrtf(cv2) +
                                                 kU * sqrtf(g2)) +
                                2.4e-7f * R2 + 3.0e-8f * sqrtD) +
                        1.1f * 4.3e-6f * R2;
        st_err[r] = make_float2(E, 1.1f * 3.0e-8f * sqrtD * R2);
      }
    }
    // ---------------------------------------------------------------- sketch
    if constexpr (SK) {
      tqtc::fence_proxy_async_smem();
      tqtc::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tqtc::tc_fence_after();
        const uint32_t ahi = tqtc::smem_u32(smem + ly.a_hi), alo = tqtc::smem_u32(smem + ly.a_lo);
        if (m <= 128) {
          // two products: A_hi [S_hi; S_lo] (N = 2m: columns [0, m) hi*hi,
          // [m, 2m) hi*lo) and A_lo S_hi accumulated onto columns [0, m)
          const uint32_t b2 = tqtc::smem_u32(smem + ly.bimg), lbo2 = 32u * (uint32_t)m;
          const uint32_t id2 = tqtc::instr_desc(1, 0, 0, kRows, 2u * (uint32_t)m);
          const uint32_t id1 = tqtc::instr_desc(1, 0, 0, kRows, (uint32_t)m);
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            tqtc::mma_f16_ss(tbase, tqtc::smem_desc(ahi + 2u * s * LBO_A, LBO_A, 128),
                             tqtc::smem_desc(b2 + 2u * s * lbo2, lbo2, 128), id2, s > 0);
#pragma unroll
          for (int s = 0; s < D / 16; ++s)
            tqtc::mma_f16_ss(tbase, tqtc::smem_desc(alo + 2u * s * LBO_A, LBO_A, 128),
                             tqtc::smem_desc(b2 + 2u * s * lbo2, lbo2, 128), id1, true);
        } else {
          const uint32_t idesc = tqtc::instr_desc(1, 0, 0, kRows, (uint32_t)m);
          const uint32_t lbo_b = 16u * (uint32_t)m;
          const uint32_t bhi = tqtc::smem_u32(smem + ly.bimg), blo = bhi + 2u * (uint32_t)m * D;
          bool accum = false;
#pragma unroll
          for (int pass = 0; pass < 3; ++pass) {
            const uint32_t aa = pass == 1 ? alo : ahi;
            const uint32_t bb = pass == 2 ? blo : bhi;
#pragma unroll
            for (int s = 0; s < D / 16; ++s) {
              tqtc::mma_f16_ss(tbase, tqtc::smem_desc(aa + 2u * s * LBO_A, LBO_A, 128),
                               tqtc::smem_desc(bb + 2u * s * lbo_b, lbo_b, 128), idesc, accum);
              accum = true;
            }
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
      // epilogue: warp (lane quarter lq, word c) -> sign word c of rows 32 lq + lane
      const int lq = warp & 3;
      const int rr = 32 * lq + lane;
      const float2 eg = st_err[rr];
      for (int c = warp >> 2; c < m / 32; c += NW / 4) {
        uint32_t t16[2][16], u16[2][16];
        tqtc::tmem_ld16(tqtc::tmem_addr(tbase, 32u * lq, 32u * c), t16[0]);
        tqtc::tmem_ld16(tqtc::tmem_addr(tbase, 32u * lq, 32u * c + 16u), t16[1]);
        if (m <= 128) {
          tqtc::tmem_ld16(tqtc::tmem_addr(tbase, 32u * lq, (uint32_t)m + 32u * c), u16[0]);
          tqtc::tmem_ld16(tqtc::tmem_addr(tbase, 32u * lq, (uint32_t)m + 32u * c + 16u), u16[1]);
        }
        tqtc::tmem_wait_ld();
        // sign bits gathered most recent first (bit jj ends at 31 - jj):
        // neg: t < 0; sure: |t| > tau, i.e. tau - |t| < 0.  A bit with
        // |t| <= tau (t == -0 among them) is marked uncertain and recomputed
        // exactly, so the sign bit of t stands for t < 0 on every bit kept.
        uint32_t neg = 0, sure = 0;
        const float4* sl4 = reinterpret_cast<const float4*>(smem + ly.sl2n) + 8 * c;
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 s4 = sl4[j4];
          const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int jj = 4 * j4 + i;
            float t = __uint_as_float(t16[jj >> 4][jj & 15]);
            if (m <= 128) t += __uint_as_float(u16[jj >> 4][jj & 15]);
            const float tau = fmaf(sv[i], eg.x, eg.y);
            neg = __funnelshift_l(__float_as_uint(t), neg, 1);
            sure = __funnelshift_l(__float_as_uint(tau - fabsf(t)), sure, 1);
          }
        }
        const uint32_t word = ~__brev(neg), unsure = ~__brev(sure);
        st_signs[rr * 8 + c] = word;
        st_fmask[rr * 8 + c] = unsure;
        if (unsure && row0 + rr < n) atomicOr(&st_flag[rr], 1);
      }
    }
    tqtc::tc_fence_before();
    __syncthreads();
    if (s_abort) break;
    // ---------------------------------------------------------------- write out (fast path)
    const int nrow = (int)((n - row0) < (int64_t)kRows ? (n - row0) : (int64_t)kRows);
    if (p.out_stride == 1) {
      const int64_t o0 = row0 + p.out_offset;  // contiguous output rows
      uint32_t* gcodes = out.codes + o0 * W;
      if constexpr (W % 4 == 0) {
        for (int i = tid; i < nrow * W / 4; i += NT)
          reinterpret_cast<uint4*>(gcodes)[i] = reinterpret_cast<const uint4*>(st_codes)[i];
      } else {
        for (int i = tid; i < nrow * W; i += NT) gcodes[i] = st_codes[i];
      }
      for (int i = tid; i < nrow; i += NT) out.norms[o0 + i] = st_nu[i];
      if constexpr (SK) {
        const int MS = m / 32;
        for (int i = tid; i < nrow * MS; i += NT) out.signs[o0 * MS + i] = st_signs[(i / MS) * 8 + (i % MS)];
        for (int i = tid; i < nrow; i += NT) out.rnorms[o0 + i] = st_gam[i];
      }
    } else {
      // scattered output rows (tq_append): row r goes to r * out_stride + out_offset
      for (int i = tid; i < nrow * W; i += NT)
        out.codes[((row0 + i / W) * p.out_stride + p.out_offset) * W + i % W] = st_codes[i];
      for (int i = tid; i < nrow; i += NT) out.norms[(row0 + i) * p.out_stride + p.out_offset] = st_nu[i];
      if constexpr (SK) {
        const int MS = m / 32;
        for (int i = tid; i < nrow * MS; i += NT)
          out.signs[((row0 + i / MS) * p.out_stride + p.out_offset) * MS + i % MS] = st_signs[(i / MS) * 8 + (i % MS)];
        for (int i = tid; i < nrow; i += NT) out.rnorms[(row0 + i) * p.out_stride + p.out_offset] = st_gam[i];
      }
    }
    // ---------------------------------------------------------------- queue uncertain rows
    if (tid < kRows && st_flag[tid] != 0) {
      const int e = atomicAdd(&s_nfix, 1);
      FixEntry& f = s_fix[e];
      f.row = row0 + tid;
      f.full = (st_flag[tid] & 2) != 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) f.fmask[w] = st_fmask[tid * 8 + w];
    }
    __syncthreads();
    if (s_nfix > kFixCap - kRows) drain();
    for (int i = tid; i < kRows; i += NT) st_flag[i] = 0;
    __syncthreads();
    tqtc::tc_fence_after();
  }
  tqtc::tc_fence_before();
  __syncthreads();
  if (!s_abort) drain();
  if constexpr (SK) {
    if (warp == 0) tqtc::tmem_dealloc(tbase, tmem_cols);
  }
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

template <int D, int B0, int B1, bool SK, typename TIn, bool ROPE>
cudaError_t launch_quad(const tq_params& p, const void* x, int64_t n, int64_t ld, const tq_compressed& out,
                        cudaStream_t st) {
  constexpr int TPR = D / 32;
  constexpr int NT = kRows * TPR;
  constexpr int PW = (D / (B1 > 0 ? 2 : 1)) / 32;
  constexpr int W = (B0 + B1) * PW;
  const int m = SK ? p.m : 0;
  const QLayout ly(D, m, W, NT / 32);
  auto fn = tq_quantize_quad_kernel<D, B0, B1, SK, TIn, ROPE>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ly.total);
  if (e != cudaSuccess) return e;
  uint32_t cols = 32;  // accumulator: 2m columns when the sketch uses the merged N = 2m product
  if constexpr (SK) {
    while (cols < (uint32_t)(m <= 128 ? 2 * m : m)) cols <<= 1;
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, NT, ly.total);
  if (e != cudaSuccess) return e;
  if (SK) per_sm = std::min(per_sm, (int)(512 / cols));
  per_sm = std::max(per_sm, 1);
  const int64_t ntiles = (n + kRows - 1) / kRows;
  const int grid = (int)std::min<int64_t>(ntiles, (int64_t)sm_count() * per_sm);
  fn<<<grid, NT, ly.total, st>>>(p, (const TIn*)x, n, ld, out, ntiles, cols);
  return cudaGetLastError();
}

template <int D, int B0, int B1, typename TIn, bool ROPE>
cudaError_t launch_sk(const tq_params& p, const void* x, int64_t n, int64_t ld, const tq_compressed& out,
                      cudaStream_t st) {
  return p.m > 0 ? launch_quad<D, B0, B1, true, TIn, ROPE>(p, x, n, ld, out, st)
                 : launch_quad<D, B0, B1, false, TIn, ROPE>(p, x, n, ld, out, st);
}

template <int D, typename TIn, bool ROPE>
cudaError_t dispatch_bits(const tq_params& p, const void* x, int64_t n, int64_t ld, const tq_compressed& out,
                          cudaStream_t st) {
  if (p.nseg == 1) {
    switch (p.bits[0]) {
      case 1: return launch_sk<D, 1, 0, TIn, ROPE>(p, x, n, ld, out, st);
      case 2: return launch_sk<D, 2, 0, TIn, ROPE>(p, x, n, ld, out, st);
      case 3: return launch_sk<D, 3, 0, TIn, ROPE>(p, x, n, ld, out, st);
      case 4: return launch_sk<D, 4, 0, TIn, ROPE>(p, x, n, ld, out, st);
    }
  } else if (p.bits[0] == 2 && p.bits[1] == 3) {
    return launch_sk<D, 2, 3, TIn, ROPE>(p, x, n, ld, out, st);
  }
  return cudaErrorNotSupported;
}

template <bool ROPE>
cudaError_t launch_quantize_tc(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                               const tq_compressed& out, cudaStream_t st) {
  if (p.m > 256 || (p.m > 0 && p.m % 32 != 0)) return cudaErrorNotSupported;
  if (dt != TQ_BF16 && dt != TQ_F32) return cudaErrorNotSupported;
  if (p.haar) return cudaErrorNotSupported;  // the dense Haar rotation runs on the CUDA-core encoder
  if (p.vq_bits) return cudaErrorNotSupported;  // FibQuant block codes: CUDA-core encoder
  if (p.d == 128) {
    return dt == TQ_BF16 ? dispatch_bits<128, __nv_bfloat16, ROPE>(p, x, n, ld, out, st)
                         : dispatch_bits<128, float, ROPE>(p, x, n, ld, out, st);
  }
  if (p.d == 64) {
    return dt == TQ_BF16 ? dispatch_bits<64, __nv_bfloat16, ROPE>(p, x, n, ld, out, st)
                         : dispatch_bits<64, float, ROPE>(p, x, n, ld, out, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace
