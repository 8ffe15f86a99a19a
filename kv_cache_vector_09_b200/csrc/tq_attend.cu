// Fused split-context decode attention over compressed keys and values.
//
// A block takes one chunk of one (batch, KV head)'s context and up to eight of
// that head's query heads.  It
//   1. scores every key of the chunk (estimator of the inner product: the
//      codebook term plus the QJL residual term, both scaled by the key norm),
//   2. takes the chunk's softmax statistics (maximum, sum of exponentials),
//   3. accumulates sum_t p_t nu_t cen[code_t] in the rotated space,
// and writes (acc[d], max, sum) per query; a second kernel merges the chunks
// and applies the inverse rotation.
//
// Scoring costs one shared-memory table load per coordinate and per QJL sign
// nibble.  Per block and query g the tables hold
//   lut[i][c][g] = q'_{g,i} cen_{s(i)}[c] / sqrt(d)                (code c at coordinate i)
//   nib[n][e][g] = sum_{r<4} (bit r of e ? +1 : -1) w_{g,4n+r}        (sign nibble n)
// where q' = Pi q and w = S Pi q.  Keys are staged in shared memory by
// cp.async in double-buffered tiles (one key per thread).  Values are decoded
// per lane (consecutive coordinates, codes gathered from the bit planes by a
// multiply-and-mask spread) and accumulated with packed f32x2 FMAs over query
// pairs.
#include <math.h>

#include <algorithm>

#include "tq_common.cuh"
#include "tq_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kKeyTile = kThreads;  // keys scored per tile, one per thread
constexpr int kValTile = 64;        // keys per value tile

typedef unsigned long long u64;

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fadd2(u64& acc, u64 x) { asm("add.rn.f32x2 %0, %0, %1;" : "+l"(acc) : "l"(x)); }
__device__ __forceinline__ void ffma2(u64& acc, u64 a, u64 b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float lo_f(u64 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f(u64 v) { return __uint_as_float((uint32_t)(v >> 32)); }

// bit r (r < 4) of x -> byte r; x < 16
__device__ __forceinline__ uint32_t spread4(uint32_t x) { return (x * 0x00204081u) & 0x01010101u; }

// NG query accumulators; pairs packed for f32x2 when NG >= 2
template <int NG>
struct QAcc {
  static constexpr int NP = NG / 2;
  u64 v[NP];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int k = 0; k < NP; ++k) v[k] = 0ull;
  }
  // acc += e[0..NG)   (e 16-byte aligned in shared memory)
  __device__ __forceinline__ void add(const float* e) {
    if constexpr (NG % 4 == 0) {
#pragma unroll
      for (int k = 0; k < NP; k += 2) {
        const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(e + 2 * k);
        fadd2(v[k], t.x);
        fadd2(v[k + 1], t.y);
      }
    } else {
      fadd2(v[0], *reinterpret_cast<const u64*>(e));
    }
  }
  // acc += p[0..NG) * c     (c = (cen, cen))
  __device__ __forceinline__ void fma(const u64 (&p)[NP], u64 c) {
#pragma unroll
    for (int k = 0; k < NP; ++k) ffma2(v[k], p[k], c);
  }
  __device__ __forceinline__ float get(int g) const { return (g & 1) ? hi_f(v[g >> 1]) : lo_f(v[g >> 1]); }
};

template <>
struct QAcc<1> {
  static constexpr int NP = 1;
  float v;
  __device__ __forceinline__ void zero() { v = 0.f; }
  __device__ __forceinline__ void add(const float* e) { v += *e; }
  __device__ __forceinline__ void fma(const u64 (&p)[1], u64 c) { v = fmaf(lo_f(p[0]), lo_f(c), v); }
  __device__ __forceinline__ float get(int) const { return v; }
};

// Codebook term of one segment: planes at row[k * PW + w], table rows of
// `ck` codes of NG floats per coordinate.
template <int PW, int P, int NG>
__device__ __forceinline__ void score_segment(const uint32_t* __restrict__ row, const float* __restrict__ lut,
                                              const int ck, QAcc<NG>& acc) {
  const int cstride = ck * NG;
#pragma unroll
  for (int w = 0; w < PW; ++w) {
    uint32_t pl[P];
#pragma unroll
    for (int k = 0; k < P; ++k) pl[k] = row[k * PW + w];
    const float* lw = lut + (32 * w) * cstride;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      uint32_t x = 0u;
#pragma unroll
      for (int k = 0; k < P; ++k) x |= spread4((pl[k] >> (4 * h)) & 0xFu) << k;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t c = (x >> (8 * r)) & 0xFFu;
        acc.add(lw + (4 * h + r) * cstride + (int)c * NG);
      }
    }
  }
}

template <int PW, int NG>
__device__ __forceinline__ void score_segment_bits(const uint32_t* row, const float* lut, int ck, int bits,
                                                   QAcc<NG>& acc) {
  switch (bits) {
    case 1: score_segment<PW, 1, NG>(row, lut, ck, acc); break;
    case 2: score_segment<PW, 2, NG>(row, lut, ck, acc); break;
    case 3: score_segment<PW, 3, NG>(row, lut, ck, acc); break;
    default: score_segment<PW, 4, NG>(row, lut, ck, acc); break;
  }
}

// shared-memory layout (floats), identical on host and device
struct AttLayout {
  int ck, lut, nib, L, stage, total;
  __host__ __device__ AttLayout(const tq_params& kp, const tq_params& vp, int D, int NG, int chunk_len) {
    const int kb = kp.nseg == 2 ? (kp.bits[0] > kp.bits[1] ? kp.bits[0] : kp.bits[1]) : kp.bits[0];
    ck = 1 << kb;
    lut = 0;
    nib = lut + D * ck * NG;
    L = nib + (kp.m / 4) * 16 * NG;
    stage = L + ((chunk_len * NG + 3) / 4) * 4;
    const int rs = (kp.W + kp.MS) | 1;
    const int kstage = 2 * kKeyTile * rs;
    const int vstage = 2 * kValTile * vp.W;
    const int accb = kWarps * D * NG;
    int st = kstage > vstage ? kstage : vstage;
    st = st > accb ? st : accb;
    total = stage + ((st + 3) / 4) * 4;
  }
};

template <int D, int NG>
__global__ void __launch_bounds__(kThreads, 2)
    tq_attend_fused_kernel(const tq_params kp, const tq_params vp, const float* __restrict__ qprep, const int Hq,
                           const int Hkv, const int nsub, const int64_t T, const float scale_log2e,
                           const tq_compressed K, const tq_compressed V, float* __restrict__ partials,
                           const int nchunk, const int chunk_len) {
  constexpr int NP = QAcc<NG>::NP;
  constexpr int CPL = D / 32;  // value coordinates per lane
  extern __shared__ __align__(16) float smem[];
  __shared__ __align__(16) u64 s_cenv[2][16];
  __shared__ float s_red[kWarps][NG];
  __shared__ float s_max[NG], s_sum[NG];

  const AttLayout lay(kp, vp, D, NG, chunk_len);
  float* lut = smem + lay.lut;
  float* nib = smem + lay.nib;
  float* L = smem + lay.L;
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem + lay.stage);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv;
  const int b = blockIdx.z, hk = blockIdx.y / nsub, sub = blockIdx.y % nsub, chunk = blockIdx.x;
  const int g0 = sub * NG;
  const int m = kp.m, ck = lay.ck;
  const size_t qstride = (size_t)(D + m);
  const float* qbase = qprep + (size_t)(b * Hq + hk * G + g0) * qstride;

  // ---- tables
  for (int idx = tid; idx < D * ck * NG; idx += kThreads) {
    const int g = idx % NG, c = (idx / NG) % ck, i = idx / (NG * ck);
    const int s = (kp.nseg == 2 && i >= kp.seg_len) ? 1 : 0;
    float v = 0.f;
    if (g0 + g < G && c < (1 << kp.bits[s])) v = qbase[g * qstride + i] * kp.cen[s][c] * kp.inv_sqrt_d;
    lut[idx] = v;
  }
  for (int idx = tid; idx < (m / 4) * 16 * NG; idx += kThreads) {
    const int g = idx % NG, e = (idx / NG) % 16, n = idx / (NG * 16);
    float v = 0.f;
    if (g0 + g < G) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float wv = qbase[g * qstride + D + 4 * n + r];
        v += ((e >> r) & 1) ? wv : -wv;
      }
    }
    nib[idx] = v;
  }
  if (tid < 32) {
    const int s = tid >> 4, c = tid & 15;
    const float cv = (s < vp.nseg && c < (1 << vp.bits[s])) ? vp.cen[s][c] : 0.f;
    s_cenv[s][c] = (u64)__float_as_uint(cv) | ((u64)__float_as_uint(cv) << 32);
  }

  const int64_t t0 = (int64_t)chunk * chunk_len;
  const int64_t t1 = t0 + chunk_len < T ? t0 + chunk_len : T;
  const int64_t rowbase = ((int64_t)b * Hkv + hk) * T;

  // ---- phase 1: logits (log2 units) into L
  const int Wk = kp.W, MSk = kp.MS, RS = (Wk + MSk) | 1;
  const float invW = 1.0f / (float)Wk, invMS = MSk > 0 ? 1.0f / (float)MSk : 0.f;
  auto issue_keys = [&](int buf, int64_t start) {
    const int n = (int)(t1 - start < kKeyTile ? t1 - start : kKeyTile);
    uint32_t* st = stage + buf * kKeyTile * RS;
    const uint32_t* gc = K.codes + (rowbase + start) * Wk;
    for (int idx = tid; idx < n * Wk; idx += kThreads) {
      const int r = (int)(((float)idx + 0.5f) * invW), c = idx - r * Wk;
      cp_async4(st + r * RS + c, gc + idx);
    }
    if (MSk > 0) {
      const uint32_t* gs = K.signs + (rowbase + start) * MSk;
      for (int idx = tid; idx < n * MSk; idx += kThreads) {
        const int r = (int)(((float)idx + 0.5f) * invMS), c = idx - r * MSk;
        cp_async4(st + r * RS + Wk + c, gs + idx);
      }
    }
  };
  float lmax[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) lmax[g] = -INFINITY;
  if (t0 < t1) issue_keys(0, t0);
  cp_async_commit();
  __syncthreads();  // tables
  int it = 0;
  for (int64_t tile = t0; tile < t1; tile += kKeyTile, ++it) {
    if (tile + kKeyTile < t1) issue_keys((it + 1) & 1, tile + kKeyTile);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int n = (int)(t1 - tile < kKeyTile ? t1 - tile : kKeyTile);
    if (tid < n) {
      const uint32_t* row = stage + (it & 1) * kKeyTile * RS + tid * RS;
      QAcc<NG> am, aq;
      am.zero();
      aq.zero();
      if (kp.nseg == 1) {
        score_segment_bits<D / 32, NG>(row, lut, ck, kp.bits[0], am);
      } else {
        score_segment_bits<D / 64, NG>(row + kp.segbase[0], lut, ck, kp.bits[0], am);
        score_segment_bits<D / 64, NG>(row + kp.segbase[1], lut + (D / 2) * ck * NG, ck, kp.bits[1], am);
      }
      for (int u = 0; u < MSk; ++u) {
        const uint32_t word = row[Wk + u];
#pragma unroll
        for (int h = 0; h < 8; ++h) aq.add(nib + ((8 * u + h) * 16 + (int)((word >> (4 * h)) & 0xFu)) * NG);
      }
      const int64_t rr = rowbase + tile + tid;
      const float nu = __ldg(K.norms + rr) * scale_log2e;
      const float cq = MSk > 0 ? __ldg(K.rnorms + rr) * kp.qjl_coef : 0.f;
      float* lr = L + (tile + tid - t0) * NG;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float l = nu * fmaf(cq, aq.get(g), am.get(g));
        lr[g] = l;
        lmax[g] = fmaxf(lmax[g], l);
      }
    }
    __syncthreads();
  }

  // ---- phase 2: chunk maximum, exponentials times the value norm
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const float v = tq_warp_max(lmax[g]);
    if (lane == 0) s_red[warp][g] = v;
  }
  __syncthreads();
  if (tid < NG) {
    float v = -INFINITY;
    for (int w = 0; w < kWarps; ++w) v = fmaxf(v, s_red[w][tid]);
    s_max[tid] = v;
  }
  __syncthreads();
  float lsum[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) lsum[g] = 0.f;
  for (int64_t t = t0 + tid; t < t1; t += kThreads) {
    const float nv = __ldg(V.norms + rowbase + t);
    float* lr = L + (t - t0) * NG;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float e = exp2f(lr[g] - s_max[g]);
      lsum[g] += e;
      lr[g] = e * nv;
    }
  }
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const float v = tq_warp_sum(lsum[g]);
    if (lane == 0) s_red[warp][g] = v;
  }
  __syncthreads();
  if (tid < NG) {
    float v = 0.f;
    for (int w = 0; w < kWarps; ++w) v += s_red[w][tid];
    s_sum[tid] = v;
  }

  // ---- phase 3: sum_t p_t nu_t cen[code_t] (rotated space)
  const int Wv = vp.W;
  const int i0 = lane * CPL;
  const int vs = (vp.nseg == 2 && i0 >= vp.seg_len) ? 1 : 0;
  const int il = i0 - vs * vp.seg_len;
  const int vbits = vp.bits[vs];
  const int woff = vp.segbase[vs] + (il >> 5);
  const int boff = il & 31;
  const int vpw = vp.pw;
  auto issue_vals = [&](int buf, int64_t start) {
    const int n = (int)(t1 - start < kValTile ? t1 - start : kValTile);
    uint32_t* st = stage + buf * kValTile * Wv;
    const uint32_t* gv = V.codes + (rowbase + start) * Wv;
    for (int idx = tid; idx < n * Wv; idx += kThreads) cp_async4(st + idx, gv + idx);
  };
  QAcc<NG> acc[CPL];
#pragma unroll
  for (int r = 0; r < CPL; ++r) acc[r].zero();
  __syncthreads();  // key stage no longer read
  if (t0 < t1) issue_vals(0, t0);
  cp_async_commit();
  it = 0;
  for (int64_t tile = t0; tile < t1; tile += kValTile, ++it) {
    if (tile + kValTile < t1) issue_vals((it + 1) & 1, tile + kValTile);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int n = (int)(t1 - tile < kValTile ? t1 - tile : kValTile);
    const uint32_t* st = stage + (it & 1) * kValTile * Wv;
    for (int kk = warp; kk < n; kk += kWarps) {
      const uint32_t* row = st + kk * Wv + woff;
      u64 p[NP];
      const float* lr = L + (tile + kk - t0) * NG;
      if constexpr (NG == 1) {
        p[0] = (u64)__float_as_uint(lr[0]);
      } else if constexpr (NG % 4 == 0) {
#pragma unroll
        for (int k = 0; k < NP; k += 2) {
          const ulonglong2 t2 = *reinterpret_cast<const ulonglong2*>(lr + 2 * k);
          p[k] = t2.x;
          p[k + 1] = t2.y;
        }
      } else {
        p[0] = *reinterpret_cast<const u64*>(lr);
      }
      // codes of this lane's CPL coordinates, one per byte (two words for CPL = 8)
      uint32_t x[(CPL + 3) / 4];
#pragma unroll
      for (int q = 0; q < (CPL + 3) / 4; ++q) x[q] = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k < vbits) {
          const uint32_t word = row[k * vpw] >> boff;
#pragma unroll
          for (int q = 0; q < (CPL + 3) / 4; ++q)
            x[q] |= spread4((word >> (4 * q)) & (CPL >= 4 ? 0xFu : 0x3u)) << k;
        }
      }
#pragma unroll
      for (int r = 0; r < CPL; ++r) {
        const uint32_t c = (x[r >> 2] >> (8 * (r & 3))) & 0xFFu;
        acc[r].fma(p, s_cenv[vs][c]);
      }
    }
    __syncthreads();
  }

  // ---- reduce the warps' partial sums and write (acc[d], max, sum)
  float* accb = reinterpret_cast<float*>(stage);  // [kWarps][D][NG]
#pragma unroll
  for (int r = 0; r < CPL; ++r)
#pragma unroll
    for (int g = 0; g < NG; ++g) accb[((size_t)warp * D + i0 + r) * NG + g] = acc[r].get(g);
  __syncthreads();
  for (int idx = tid; idx < NG * D; idx += kThreads) {
    const int g = idx / D, i = idx % D;
    if (g0 + g >= G) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += accb[((size_t)w * D + i) * NG + g];
    float* pr = partials + ((size_t)(b * Hq + hk * G + g0 + g) * nchunk + chunk) * (D + 2);
    pr[i] = v * vp.inv_sqrt_d;
    if (i == 0) {
      pr[D] = s_max[g];
      pr[D + 1] = s_sum[g];
    }
  }
}

template <int D, int NG>
cudaError_t launch_fused(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                         int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                         int nchunk, cudaStream_t st) {
  const int chunk_len = (int)((T + nchunk - 1) / nchunk);
  const AttLayout lay(kp, vp, D, NG, chunk_len);
  const size_t smem = sizeof(float) * (size_t)lay.total;
  if (smem > 200 * 1024) return cudaErrorNotSupported;
  auto fn = tq_attend_fused_kernel<D, NG>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int G = Hq / Hkv, nsub = (G + NG - 1) / NG;
  dim3 grid((unsigned)nchunk, (unsigned)(Hkv * nsub), (unsigned)B);
  fn<<<grid, kThreads, smem, st>>>(kp, vp, qprep, Hq, Hkv, nsub, T, scale * 1.4426950408889634f, K, V, partials,
                                   nchunk, chunk_len);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_fused_d(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                           int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                           int nchunk, cudaStream_t st) {
  const int G = Hq / Hkv;
  if (G == 1) return launch_fused<D, 1>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  if (G == 2) return launch_fused<D, 2>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  if (G <= 4) return launch_fused<D, 4>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  return launch_fused<D, 8>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
}

}  // namespace

cudaError_t tq_launch_attend_fused(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq,
                                   int Hkv, int64_t T, float scale, const tq_compressed& K, const tq_compressed& V,
                                   float* partials, int nchunk, cudaStream_t st) {
  if (kp.d != vp.d || kp.m % 32 != 0 || kp.m > 256) return cudaErrorNotSupported;
  switch (kp.d) {
    case 64: return launch_fused_d<64>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
    case 128: return launch_fused_d<128>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
    default: return cudaErrorNotSupported;
  }
}
