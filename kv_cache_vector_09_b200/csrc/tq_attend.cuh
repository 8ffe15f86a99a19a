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
// Scoring (phase 1): a thread takes two keys at a time, read straight from
// global memory into registers.  The rotated query values q'_i of the block's
// queries are read from shared memory with warp-uniform addresses (one load
// serves the 64 keys of a warp), the centroid of each key's code with a 4-byte
// lane-indexed load, and both keys accumulate with packed f32x2 FMAs over
// query pairs.  The QJL term uses a per-block table
//   nib[n][e][g] = sum_{r<4} (bit r of e ? +1 : -1) w_{g,4n+r},   w = S Pi q,
// one load per sign nibble.  Codes of four coordinates are gathered from the
// bit planes at once by a multiply-and-mask spread (bit r of a nibble -> byte r).
//
// Values (phase 3): lanes own consecutive coordinates and warps take keys in
// turn from double-buffered cp.async tiles; the probability weights are
// warp-uniform loads and the centroids 4-byte lane-indexed loads.
//
// QJL-corrected values (value codec with m > 0; TurboQuant pages: the 1-bit
// QJL stage removes the first stage's bias): the value estimate is
//   v~_t = nu_t (c_hat_t / sqrt(d) + gamma_t sqrt(pi/2)/m S^T s_t),
// and attention is linear in the values, so a block also accumulates the
// m-vector a = sum_t p_t nu_t gamma_t s_t (lane l owns entries l + 32u); the
// combine kernel applies sqrt(pi/2)/m S^T a once per (b, h) before the
// inverse rotation.
#pragma once

#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.h"

namespace tqatt {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kValTile = 64;  // keys per value tile

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
__device__ __forceinline__ u64 dup2(float x) {
  const u64 u = __float_as_uint(x);
  return u | (u << 32);
}
__device__ __forceinline__ float lo_f(u64 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f(u64 v) { return __uint_as_float((uint32_t)(v >> 32)); }

// bit r (r < 4) of x -> byte r; x < 16
__device__ __forceinline__ uint32_t spread4(uint32_t x) { return (x * 0x00204081u) & 0x01010101u; }

// float at a byte offset
__device__ __forceinline__ float ld_at(const float* base, uint32_t byte_off) {
  return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(base) + byte_off);
}

// NG query values or accumulators, packed in pairs for f32x2 when NG >= 2
template <int NG>
struct QVec {
  static constexpr int NP = NG / 2;
  u64 v[NP];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int k = 0; k < NP; ++k) v[k] = 0ull;
  }
  __device__ __forceinline__ void load(const float* e) {  // e: 8-byte aligned (16 when NG % 4 == 0)
    if constexpr (NG % 4 == 0) {
#pragma unroll
      for (int k = 0; k < NP; k += 2) {
        const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(e + 2 * k);
        v[k] = t.x;
        v[k + 1] = t.y;
      }
    } else {
      v[0] = *reinterpret_cast<const u64*>(e);
    }
  }
  __device__ __forceinline__ void add(const QVec& o) {
#pragma unroll
    for (int k = 0; k < NP; ++k) fadd2(v[k], o.v[k]);
  }
  __device__ __forceinline__ void fma(const QVec& a, float c) {  // this += a * c
    const u64 cc = dup2(c);
#pragma unroll
    for (int k = 0; k < NP; ++k) ffma2(v[k], a.v[k], cc);
  }
  __device__ __forceinline__ float get(int g) const { return (g & 1) ? hi_f(v[g >> 1]) : lo_f(v[g >> 1]); }
};

template <>
struct QVec<1> {
  static constexpr int NP = 1;
  float v;
  __device__ __forceinline__ void zero() { v = 0.f; }
  __device__ __forceinline__ void load(const float* e) { v = *e; }
  __device__ __forceinline__ void add(const QVec& o) { v += o.v; }
  __device__ __forceinline__ void fma(const QVec& a, float c) { v = fmaf(a.v, c, v); }
  __device__ __forceinline__ float get(int) const { return v; }
};

// W consecutive words of a row into registers (zeros when !valid)
template <int W>
__device__ __forceinline__ void load_row(uint32_t (&r)[W], const uint32_t* __restrict__ p, bool valid) {
  if constexpr (W % 4 == 0) {
#pragma unroll
    for (int k = 0; k < W; k += 4) {
      const uint4 v = valid ? __ldg(reinterpret_cast<const uint4*>(p + k)) : make_uint4(0u, 0u, 0u, 0u);
      r[k] = v.x; r[k + 1] = v.y; r[k + 2] = v.z; r[k + 3] = v.w;
    }
  } else if constexpr (W % 2 == 0) {
#pragma unroll
    for (int k = 0; k < W; k += 2) {
      const uint2 v = valid ? __ldg(reinterpret_cast<const uint2*>(p + k)) : make_uint2(0u, 0u);
      r[k] = v.x; r[k + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int k = 0; k < W; ++k) r[k] = valid ? __ldg(p + k) : 0u;
  }
}

// MS (runtime, 0..8) sign words of a row into s[8]
__device__ __forceinline__ void load_signs(uint32_t (&s)[8], const uint32_t* __restrict__ p, int MS, bool valid) {
#pragma unroll
  for (int k = 0; k < 8; ++k) s[k] = 0u;
  if (!valid) return;
  if (MS >= 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    s[0] = v.x; s[1] = v.y; s[2] = v.z; s[3] = v.w;
    if (MS == 8) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(p) + 1);
      s[4] = w.x; s[5] = w.y; s[6] = w.z; s[7] = w.w;
    }
  } else if (MS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    s[0] = v.x; s[1] = v.y;
  } else if (MS == 1) {
    s[0] = __ldg(p);
  }
}

// Codebook term of one segment for two keys.  Planes k < P of word w sit at
// row[base + k * PW + w]; q rows of NG floats per coordinate; cen: the
// segment's centroid table (floats).
template <int PW, int P, int NG, int W>
__device__ __forceinline__ void score_seg2(const uint32_t (&ra)[W], const uint32_t (&rb)[W], const int base,
                                           const float* __restrict__ q, const float* __restrict__ cen,
                                           QVec<NG>& A, QVec<NG>& B) {
#pragma unroll
  for (int w = 0; w < PW; ++w) {
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      uint32_t xa = 0u, xb = 0u;  // byte r = 4 * code of coordinate 32w + 4h + r
#pragma unroll
      for (int k = 0; k < P; ++k) {
        xa |= spread4((ra[base + k * PW + w] >> (4 * h)) & 0xFu) << (k + 2);
        xb |= spread4((rb[base + k * PW + w] >> (4 * h)) & 0xFu) << (k + 2);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        QVec<NG> qv;
        qv.load(q + (32 * w + 4 * h + r) * NG);
        A.fma(qv, ld_at(cen, (xa >> (8 * r)) & 0xFFu));
        B.fma(qv, ld_at(cen, (xb >> (8 * r)) & 0xFFu));
      }
    }
  }
}

// QJL term of one key: sum over sign nibbles of the nib table
template <int NG>
__device__ __forceinline__ void qjl_nib(const uint32_t (&s)[8], const int MS, const float* __restrict__ nib,
                                        QVec<NG>& A) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if (u < MS) {
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        QVec<NG> e;
        e.load(nib + ((8 * u + h) * 16 + (int)((s[u] >> (4 * h)) & 0xFu)) * NG);
        A.add(e);
      }
    }
  }
}

// shared-memory layout (floats), identical on host and device; vq: QJL-
// corrected values (value sign words staged with the codes, gamma per token)
struct AttLayout {
  int q, nib, L, gm, stage, total;
  __host__ __device__ AttLayout(const tq_params& kp, const tq_params& vp, int D, int NG, int chunk_len, bool vq) {
    const int vms = vq ? vp.MS : 0;
    q = 0;                              // [D][NG]  q' / sqrt(d)
    nib = q + D * NG;                   // [m/4][16][NG]
    L = nib + (kp.m / 4) * 16 * NG;     // [chunk_len][NG]
    gm = L + ((chunk_len * NG + 3) / 4) * 4;  // [chunk_len] value gamma (vq only)
    stage = gm + (vq ? ((chunk_len + 3) / 4) * 4 : 0);
    const int vstage = 2 * kValTile * (vp.W + vms);
    const int accb = kWarps * (D + 32 * vms) * NG;
    const int st = vstage > accb ? vstage : accb;
    total = stage + ((st + 3) / 4) * 4;
  }
};

// floats per (b, hq, chunk) partial: acc[d], max, sum, then a[m] when vq
__host__ __device__ inline int att_partial_stride(int d, int vm, bool vq) { return d + 2 + (vq ? vm : 0); }

template <int D, int NG, int KB0, int KB1, bool VQ>
__global__ void __launch_bounds__(kThreads, 2)
    attend_kernel(const tq_params kp, const tq_params vp, const float* __restrict__ qprep, const int Hq,
                  const int Hkv, const int nsub, const int64_t T, const float scale_log2e, const tq_compressed K,
                  const tq_compressed V, float* __restrict__ partials, const int nchunk, const int chunk_len) {
  constexpr int NSEG = KB1 > 0 ? 2 : 1;
  constexpr int KPW = D / NSEG / 32;
  constexpr int KW = (KB0 + KB1) * KPW;
  constexpr int CPL = D / 32;  // value coordinates per lane
  extern __shared__ __align__(16) float smem[];
  __shared__ float s_cenk[2][16], s_cenv[2][16];
  __shared__ float s_red[kWarps][NG];
  __shared__ float s_max[NG], s_sum[NG];

  const AttLayout lay(kp, vp, D, NG, chunk_len, VQ);
  float* sq = smem + lay.q;
  float* nib = smem + lay.nib;
  float* L = smem + lay.L;
  float* gm = smem + lay.gm;
  const int VMS = VQ ? vp.MS : 0;  // value sign words (<= 4)
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem + lay.stage);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv;
  const int b = blockIdx.z, hk = blockIdx.y / nsub, sub = blockIdx.y % nsub, chunk = blockIdx.x;
  const int g0 = sub * NG;
  const int m = kp.m, MSk = kp.MS;
  const size_t qstride = (size_t)(D + m);
  const float* qbase = qprep + (size_t)(b * Hq + hk * G + g0) * qstride;

  // ---- per-block tables
  for (int idx = tid; idx < D * NG; idx += kThreads) {
    const int g = idx % NG, i = idx / NG;
    sq[idx] = (g0 + g < G) ? qbase[g * qstride + i] * kp.inv_sqrt_d : 0.f;
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
    s_cenk[s][c] = (s < kp.nseg && c < (1 << kp.bits[s])) ? kp.cen[s][c] : 0.f;
    s_cenv[s][c] = (s < vp.nseg && c < (1 << vp.bits[s])) ? vp.cen[s][c] : 0.f;
  }
  __syncthreads();

  const int64_t t0 = (int64_t)chunk * chunk_len;
  const int64_t t1 = t0 + chunk_len < T ? t0 + chunk_len : T;
  const int64_t rowbase = ((int64_t)b * Hkv + hk) * T;

  // ---- phase 1: logits (log2 units) into L, two keys per thread
  float lmax[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) lmax[g] = -INFINITY;
  for (int64_t ta = t0 + tid; ta < t1; ta += 2 * kThreads) {
    const int64_t tb = ta + kThreads;
    const bool vb = tb < t1;
    uint32_t ra[KW], rb[KW], sa[8], sb[8];
    load_row<KW>(ra, K.codes + (rowbase + ta) * KW, true);
    load_row<KW>(rb, K.codes + (rowbase + tb) * KW, vb);
    load_signs(sa, K.signs + (rowbase + ta) * MSk, MSk, MSk > 0);
    load_signs(sb, K.signs + (rowbase + tb) * MSk, MSk, MSk > 0 && vb);
    QVec<NG> A, B, QA, QB;
    A.zero();
    B.zero();
    QA.zero();
    QB.zero();
    score_seg2<KPW, KB0, NG, KW>(ra, rb, 0, sq, s_cenk[0], A, B);
    if constexpr (NSEG == 2) score_seg2<KPW, KB1, NG, KW>(ra, rb, KB0 * KPW, sq + (D / 2) * NG, s_cenk[1], A, B);
    qjl_nib<NG>(sa, MSk, nib, QA);
    qjl_nib<NG>(sb, MSk, nib, QB);
    {
      const float nu = __ldg(K.norms + rowbase + ta) * scale_log2e;
      const float cq = MSk > 0 ? __ldg(K.rnorms + rowbase + ta) * kp.qjl_coef : 0.f;
      float* lr = L + (ta - t0) * NG;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float l = nu * fmaf(cq, QA.get(g), A.get(g));
        lr[g] = l;
        lmax[g] = fmaxf(lmax[g], l);
      }
    }
    if (vb) {
      const float nu = __ldg(K.norms + rowbase + tb) * scale_log2e;
      const float cq = MSk > 0 ? __ldg(K.rnorms + rowbase + tb) * kp.qjl_coef : 0.f;
      float* lr = L + (tb - t0) * NG;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float l = nu * fmaf(cq, QB.get(g), B.get(g));
        lr[g] = l;
        lmax[g] = fmaxf(lmax[g], l);
      }
    }
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
    if constexpr (VQ) gm[t - t0] = __ldg(V.rnorms + rowbase + t);
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
  const float* cenv = s_cenv[vs];
  const int Ws = Wv + VMS;  // staged words per token: codes, then sign words
  auto issue_vals = [&](int buf, int64_t start) {
    const int n = (int)(t1 - start < kValTile ? t1 - start : kValTile);
    uint32_t* st = stage + buf * kValTile * Ws;
    const uint32_t* gv = V.codes + (rowbase + start) * Wv;
    for (int idx = tid; idx < n * Wv; idx += kThreads) cp_async4(st + idx, gv + idx);
    if constexpr (VQ) {
      uint32_t* ss = st + kValTile * Wv;
      const uint32_t* gs = V.signs + (rowbase + start) * VMS;
      for (int idx = tid; idx < n * VMS; idx += kThreads) cp_async4(ss + idx, gs + idx);
    }
  };
  QVec<NG> acc[CPL];
#pragma unroll
  for (int r = 0; r < CPL; ++r) acc[r].zero();
  QVec<NG> accs[VQ ? 4 : 1];  // a[lane + 32u]
#pragma unroll
  for (int u = 0; u < (VQ ? 4 : 1); ++u) accs[u].zero();
  __syncthreads();  // L complete
  if (t0 < t1) issue_vals(0, t0);
  cp_async_commit();
  int it = 0;
  for (int64_t tile = t0; tile < t1; tile += kValTile, ++it) {
    if (tile + kValTile < t1) issue_vals((it + 1) & 1, tile + kValTile);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int n = (int)(t1 - tile < kValTile ? t1 - tile : kValTile);
    const uint32_t* st = stage + (it & 1) * kValTile * Ws;
    for (int kk = warp; kk < n; kk += kWarps) {
      const uint32_t* row = st + kk * Wv + woff;
      QVec<NG> p;
      p.load(L + (tile + kk - t0) * NG);
      // 4 * code of this lane's CPL coordinates, one per byte (two words for CPL = 8)
      uint32_t x[(CPL + 3) / 4];
#pragma unroll
      for (int q = 0; q < (CPL + 3) / 4; ++q) x[q] = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k < vbits) {
          const uint32_t word = row[k * vpw] >> boff;
#pragma unroll
          for (int q = 0; q < (CPL + 3) / 4; ++q)
            x[q] |= spread4((word >> (4 * q)) & (CPL >= 4 ? 0xFu : 0x3u)) << (k + 2);
        }
      }
#pragma unroll
      for (int r = 0; r < CPL; ++r) acc[r].fma(p, ld_at(cenv, (x[r >> 2] >> (8 * (r & 3))) & 0xFFu));
      if constexpr (VQ) {
        const uint32_t* sw = st + kValTile * Wv + kk * VMS;
        const float g = gm[tile + kk - t0];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (u < VMS) accs[u].fma(p, ((sw[u] >> lane) & 1u) ? g : -g);
      }
    }
    __syncthreads();
  }

  // ---- reduce the warps' partial sums and write (acc[d], max, sum[, a[m]])
  const int DA = D + 32 * VMS;                    // accumulated entries: d values, then m sketch entries
  const int PS = att_partial_stride(D, vp.m, VQ);
  float* accb = reinterpret_cast<float*>(stage);  // [kWarps][DA][NG]
#pragma unroll
  for (int r = 0; r < CPL; ++r)
#pragma unroll
    for (int g = 0; g < NG; ++g) accb[((size_t)warp * DA + i0 + r) * NG + g] = acc[r].get(g);
  if constexpr (VQ) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (u < VMS)
#pragma unroll
        for (int g = 0; g < NG; ++g) accb[((size_t)warp * DA + D + lane + 32 * u) * NG + g] = accs[u].get(g);
  }
  __syncthreads();
  for (int idx = tid; idx < NG * DA; idx += kThreads) {
    const int g = idx / DA, i = idx % DA;
    if (g0 + g >= G) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += accb[((size_t)w * DA + i) * NG + g];
    float* pr = partials + ((size_t)(b * Hq + hk * G + g0 + g) * nchunk + chunk) * PS;
    if (i < D) {
      pr[i] = v * vp.inv_sqrt_d;
    } else {
      pr[D + 2 + (i - D)] = v;  // a_j, j = i - D
    }
    if (i == 0) {
      pr[D] = s_max[g];
      pr[D + 1] = s_sum[g];
    }
  }
}

template <int D, int NG, int KB0, int KB1, bool VQ>
cudaError_t launch_attend_q(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                            int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                            int nchunk, cudaStream_t st) {
  const int chunk_len = (int)((T + nchunk - 1) / nchunk);
  const AttLayout lay(kp, vp, D, NG, chunk_len, VQ);
  const size_t smem = sizeof(float) * (size_t)lay.total;
  if (smem > 200 * 1024) return cudaErrorNotSupported;
  auto fn = attend_kernel<D, NG, KB0, KB1, VQ>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int G = Hq / Hkv, nsub = (G + NG - 1) / NG;
  dim3 grid((unsigned)nchunk, (unsigned)(Hkv * nsub), (unsigned)B);
  fn<<<grid, kThreads, smem, st>>>(kp, vp, qprep, Hq, Hkv, nsub, T, scale * 1.4426950408889634f, K, V, partials,
                                   nchunk, chunk_len);
  return cudaGetLastError();
}

// values with a sketch of 32, 64 or 128 rows take the QJL-corrected kernel
template <int D, int NG, int KB0, int KB1>
cudaError_t launch_attend(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                          int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                          int nchunk, cudaStream_t st) {
  if (vp.m == 0)
    return launch_attend_q<D, NG, KB0, KB1, false>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  if (vp.m > 128) return cudaErrorNotSupported;
  return launch_attend_q<D, NG, KB0, KB1, true>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
}

template <int D, int KB0, int KB1>
cudaError_t launch_attend_ng(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                             int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                             int nchunk, cudaStream_t st) {
  const int G = Hq / Hkv;
  if (G == 1) return launch_attend<D, 1, KB0, KB1>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  if (G == 2) return launch_attend<D, 2, KB0, KB1>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  if (G <= 4) return launch_attend<D, 4, KB0, KB1>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  return launch_attend<D, 8, KB0, KB1>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
}

// key bit layouts with a fused kernel: one segment of 1..4 bits, or 2 + 3 bits
template <int D>
cudaError_t launch_attend_d(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq, int Hkv,
                            int64_t T, float scale, const tq_compressed& K, const tq_compressed& V, float* partials,
                            int nchunk, cudaStream_t st) {
  if (kp.nseg == 1) {
    switch (kp.bits[0]) {
      case 1: return launch_attend_ng<D, 1, 0>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
      case 2: return launch_attend_ng<D, 2, 0>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
      case 3: return launch_attend_ng<D, 3, 0>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
      case 4: return launch_attend_ng<D, 4, 0>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
    }
  } else if (kp.bits[0] == 2 && kp.bits[1] == 3) {
    return launch_attend_ng<D, 2, 3>(kp, vp, qprep, B, Hq, Hkv, T, scale, K, V, partials, nchunk, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace tqatt
