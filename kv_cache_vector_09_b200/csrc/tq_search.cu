// Top-k search over a compressed index on the tensor cores (kind::f16
// tcgen05.mma, fp32 accumulation in TMEM).
//
// The score of query i and index row t is the estimator of tq_scores,
//   s = nu_t / sqrt(d) * ( sum_c q'_c cen[code_c] + g_t sum_j w_j sgn_j ),
//   g_t = gamma_t sqrt(pi/2) / m * sqrt(d),   w = S q',   sgn = 2 bit - 1,
// a dense contraction of the dequantised row against the query.  Both sides
// are split into fp16 hi + lo parts and three products per element are
// accumulated (hi*hi + lo*hi + hi*lo; the omitted lo*lo is below 2^-22 of
// the term), in K groups of 16 elements:
//   group of 16 coordinates:  A = [cen_hi | cen_lo],  B = [q_hi | q_lo]
//   group of 16 sketch rows:  A = [g_hi s | g_lo s],  B = [w_hi | w_lo]
// and the three MMAs of a group pair (A_hi, B_hi), (A_lo, B_hi), (A_hi, B_lo)
// with B scaled per query by 2^e (w by 2^(e-6), g by 2^6) to keep the fp16
// parts normal.  A is built per 128-row tile by CUDA-core warps straight
// into a shared-memory ring (codes -> centroid hi/lo pairs), B is a
// per-query image built once per call and streamed from L2 by bulk copies;
// the fp32 accumulator is double-buffered in TMEM so that the epilogue of one
// tile overlaps the MMAs of the next.  One block per SM:
//   warps 0-3   A builders (warp w builds rows 32 w ..)
//   warp 4      B producer (bulk copies into a ring of 4..8 stages)
//   warp 5      MMA issue: 3 MMAs (M = 128, N = 256, K = 16) per group
//   warps 6-13  epilogue: scores of the tile -> per-query top-k lists in
//               shared memory (each query's list updated by one warp)
// A final kernel merges the blocks' lists.  Every mbarrier wait is bounded.
#include <math.h>

#include <algorithm>

#include "tq_common.cuh"
#include "tq_internal.h"
#include "tq_tc.cuh"

namespace {

constexpr int kRowsT = 128;                // index rows per tile (MMA M)
constexpr int kQT = 256;                   // queries per tile (MMA N)
constexpr int kStepBytes = kQT * 16 * 2;   // one K = 16 step of B: 8 KB
constexpr int kGroupBytes = 2 * kStepBytes;  // [hi | lo]
constexpr int kBStagesMax = 8;               // B ring depth: as many as shared memory allows
constexpr int kCandCap = 2048;             // candidate buffer of the epilogue (entries)
constexpr int kASlots = 8;                 // A ring in shared memory, [hi | lo] per slot
constexpr int kABatch = 4;                 // groups signalled together; at most kASlots / 2, so that a
                                           // batch never waits on a slot of its own
constexpr int kASlotBytes = 2 * kRowsT * 16 * 2;  // two K = 16 steps of 128 rows: 8 KB
constexpr int kThreads = 448;
constexpr float kQjlGain = 64.f;           // 2^6 on the A side of the sketch groups

__device__ __forceinline__ uint32_t spread4(uint32_t x) { return (x * 0x00204081u) & 0x01010101u; }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t half_bits(float v) { return (uint32_t)__half_as_ushort(__float2half_rn(v)); }

__device__ __forceinline__ bool better(float s, int r, float ts, int tr) { return s > ts || (s == ts && r < tr); }

// ---------------------------------------------------------------- query side
// Per-query exponent e: max(|q'|, |w| 2^-6) 2^e < 2^14.
__global__ void __launch_bounds__(256) search_qexp_kernel(const float* __restrict__ qprep, int nq, int d, int m,
                                                          int* __restrict__ qexp, float* __restrict__ qscale) {
  const int lane = threadIdx.x & 31;
  const int qi = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (qi >= nq) return;
  const float* row = qprep + (size_t)qi * (d + m);
  float mx = 0.f;
  for (int i = lane; i < d; i += 32) mx = fmaxf(mx, fabsf(row[i]));
  for (int j = lane; j < m; j += 32) mx = fmaxf(mx, fabsf(row[d + j]) * (1.f / kQjlGain));
  mx = tq_warp_max(mx);
  if (lane == 0) {
    int ex = 0;
    frexpf(mx > 0.f ? mx : 1.f, &ex);
    const int e = 14 - ex;
    qexp[qi] = e;
    qscale[qi] = ldexpf(1.f, -e);
  }
}

// B image: [query tile][group][hi, lo][8 KB], one thread per (query, group).
// Within a step: element (n, kk) at (kk / 8) * 4096 + (n / 8) * 128 + (n % 8) * 16 + (kk % 8) * 2.
__global__ void __launch_bounds__(256) search_bimg_kernel(const float* __restrict__ qprep, const int* __restrict__ qexp,
                                                          int nq, int nqt, int d, int m, uint8_t* __restrict__ img) {
  const int ngroups = d / 16 + m / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)nqt * kQT * ngroups) return;
  const int n_all = (int)(idx % (nqt * kQT));
  const int g = (int)(idx / (nqt * kQT));
  const int qt = n_all / kQT, n = n_all % kQT;
  uint32_t hi[8], lo[8];
  if (n_all < nq) {
    const float* row = qprep + (size_t)n_all * (d + m);
    const int e = qexp[n_all];
    const bool sk = g >= d / 16;
    const float* src = sk ? row + d + 16 * (g - d / 16) : row + 16 * g;
    const int es = sk ? e - 6 : e;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      uint32_t h2 = 0u, l2 = 0u;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float v = ldexpf(src[2 * p + t], es);
        const __half h = __float2half_rn(v);
        const float r = v - __half2float(h);
        h2 |= (uint32_t)__half_as_ushort(h) << (16 * t);
        l2 |= half_bits(r) << (16 * t);
      }
      hi[p] = h2;
      lo[p] = l2;
    }
  } else {
#pragma unroll
    for (int p = 0; p < 8; ++p) hi[p] = lo[p] = 0u;
  }
  uint8_t* gbase = img + ((size_t)qt * ngroups + g) * kGroupBytes;
  const uint32_t off = (uint32_t)(n / 8) * 128u + (uint32_t)(n % 8) * 16u;
  const uint32_t* parts[2] = {hi, lo};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const uint32_t* v = parts[s];
    *reinterpret_cast<uint4*>(gbase + s * kStepBytes + off) = make_uint4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<uint4*>(gbase + s * kStepBytes + 4096 + off) = make_uint4(v[4], v[5], v[6], v[7]);
  }
}

// ---------------------------------------------------------------- search
struct SearchArgs {
  const uint32_t* codes;
  const uint32_t* signs;
  const float* norms;
  const float* rnorms;
  int64_t n;
  int nq;          // queries in this batch
  int nqt;         // query tiles
  int k;
  const uint8_t* img;
  const float* qscale;
  int bstages;     // B ring depth (<= kBStagesMax)
  float* part_s;   // [grid][nq][k]
  int* part_i;
};

__device__ __forceinline__ int64_t unit_begin(int64_t units, int b, int g) { return units * b / g; }

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    search_kernel(const tq_params p, const SearchArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t a_full[kASlots], a_empty[kASlots], b_full[kBStagesMax], b_empty[kBStagesMax];
  __shared__ uint64_t d_full[2], d_empty[2], drained, epi_bar;
  __shared__ int s_ncand[2];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ uint32_t s_cen[16];  // fp16 cen hi | lo << 16, by code

  const int d = p.d, m = p.m, W = p.W, MS = p.MS, PW = p.pw;
  const int gc = d / 16, ngroups = gc + m / 16;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nq = a.nq, k = a.k;

  const int kBStages = a.bstages;
  unsigned char* bring = smem;                                        // [kBStages][kGroupBytes]
  unsigned char* aring = smem + kBStages * kGroupBytes;               // [kASlots][kASlotBytes]
  float* stg = reinterpret_cast<float*>(aring + kASlots * kASlotBytes);  // [2][32][kRowsT] score staging
  // the candidate buffer shares the staging tile's memory: a tile uses one
  // or the other
  int* cand_q = reinterpret_cast<int*>(stg);                              // [kCandCap] candidates: query,
  int* cand_r = cand_q + kCandCap;                                        //   row,
  float* cand_s = reinterpret_cast<float*>(cand_r + kCandCap);            //   score
  float* s_qscale = stg + 2 * 32 * kRowsT;                                // [nq]
  float* tops = s_qscale + nq;                                            // [nq][k]
  int* tidx = reinterpret_cast<int*>(tops + (size_t)nq * k);              // [nq][k]

  const int64_t nkt = (a.n + kRowsT - 1) / kRowsT;
  const int64_t units = nkt * a.nqt;
  const int64_t u0 = unit_begin(units, blockIdx.x, gridDim.x), u1 = unit_begin(units, blockIdx.x + 1, gridDim.x);
  const int64_t nul = u1 - u0;

  for (int i = tid; i < nq * k; i += kThreads) {
    tops[i] = -INFINITY;
    tidx[i] = 0x7FFFFFFF;
  }
  for (int i = tid; i < nq; i += kThreads) s_qscale[i] = __ldg(a.qscale + i);
  if (tid < 16) {
    const float c = tid < (1 << BITS) ? p.cen[0][tid] : 0.f;
    const __half h = __float2half_rn(c);
    s_cen[tid] = (uint32_t)__half_as_ushort(h) | (half_bits(c - __half2float(h)) << 16);
  }
  if (tid == 0) {
    for (int i = 0; i < kASlots; ++i) {
      tqtc::mbar_init(&a_full[i], 128);
      tqtc::mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < kBStages; ++i) {
      tqtc::mbar_init(&b_full[i], 1);
      tqtc::mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tqtc::mbar_init(&d_full[i], 1);
      tqtc::mbar_init(&d_empty[i], 256);
    }
    tqtc::mbar_init(&drained, 1);
    tqtc::mbar_init(&epi_bar, 256);
    tqtc::fence_mbar_init();
    s_abort = 0;
    s_ncand[0] = s_ncand[1] = 0;
  }
  if (warp == 0) tqtc::tmem_alloc(&s_tmem, 512);
  tqtc::tc_fence_before();
  __syncthreads();
  tqtc::tc_fence_after();
  const uint32_t tbase = s_tmem;  // accumulators: columns [0, 256) and [256, 512)
  auto fail = [&](uint32_t code) {
    atomicExch(p.err, code);
    s_abort = 1;
  };

  if (warp < 4) {
    // ---------------------------------------------------------- A builders
    const int rloc = 32 * warp + lane;
    const float gk = p.qjl_coef * sqrtf((float)d) * kQjlGain;
    // put one group into its ring slot (after the slot's previous MMAs are
    // done); groups are signalled in batches of kABatch: one proxy fence,
    // then an arrival per slot
    auto put = [&](int64_t x, const uint32_t (&hi)[8], const uint32_t (&lo)[8]) -> bool {
      const int slot = (int)(x % kASlots);
      if (x >= kASlots &&
          !tqtc::mbar_wait_sleep_or_abort(&a_empty[slot], (uint32_t)((x / kASlots - 1) & 1), &s_abort, 128)) {
        fail(tqtc::kErrMmaWait);
        return false;
      }
      // K-major core matrices: (row, k) at (k / 8) * 2048 + (row / 8) * 128 + (row % 8) * 16 + (k % 8) * 2
      unsigned char* sl = aring + (size_t)slot * kASlotBytes + (rloc / 8) * 128 + (rloc % 8) * 16;
      *reinterpret_cast<uint4*>(sl) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(sl + 2048) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
      *reinterpret_cast<uint4*>(sl + 4096) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(sl + 6144) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
      return true;
    };
    // signal groups x0 .. x0 + cnt - 1
    auto signal = [&](int64_t x0, int cnt) {
      tqtc::fence_proxy_async_smem();  // the MMAs read these stores through the async proxy
      for (int i = 0; i < cnt; ++i) tqtc::mbar_arrive(&a_full[(int)((x0 + i) % kASlots)]);
    };
    // 16 codes (one 16-bit half of each plane word) -> centroid hi / lo pairs
    auto decode16 = [&](const uint32_t (&pl)[BITS], uint32_t (&hi)[8], uint32_t (&lo)[8]) {
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint32_t y = 0u;  // byte r = 4 * code of coordinate 4 t + r
#pragma unroll
        for (int b = 0; b < BITS; ++b) y |= spread4((pl[b] >> (4 * t)) & 0xFu) << (b + 2);
        uint32_t hl[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
          hl[r] = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(s_cen) + ((y >> (8 * r)) & 0xFFu));
        hi[2 * t] = prmt(hl[0], hl[1], 0x5410);
        lo[2 * t] = prmt(hl[0], hl[1], 0x7632);
        hi[2 * t + 1] = prmt(hl[2], hl[3], 0x5410);
        lo[2 * t + 1] = prmt(hl[2], hl[3], 0x7632);
      }
    };
    bool alive = true;
    for (int64_t ul = 0; ul < nul && alive && !s_abort; ++ul) {
      const int64_t kt = (u0 + ul) / a.nqt;
      const int64_t row = kt * kRowsT + rloc;
      const bool valid = row < a.n;
      const uint32_t* crow = a.codes + (valid ? row : 0) * W;
      const uint32_t* srow = a.signs + (valid ? row : 0) * MS;
      const int64_t x0 = ul * ngroups;
      if (PW % 4 == 0) {
        // coordinate groups in blocks of four words per plane (one 16-byte
        // load each, eight groups), the next block loaded while this one is
        // built
        uint4 cur[BITS], nxt[BITS];
#pragma unroll
        for (int b = 0; b < BITS; ++b)
          cur[b] = valid ? __ldg(reinterpret_cast<const uint4*>(crow + b * PW)) : make_uint4(0u, 0u, 0u, 0u);
        for (int blk = 0; blk < PW / 4 && alive; ++blk) {
          if (blk + 1 < PW / 4) {
#pragma unroll
            for (int b = 0; b < BITS; ++b)
              nxt[b] = valid ? __ldg(reinterpret_cast<const uint4*>(crow + b * PW + 4 * blk + 4))
                             : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int ww = 0; ww < 4; ++ww) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t pl[BITS];
#pragma unroll
              for (int b = 0; b < BITS; ++b) {
                const uint32_t v = ww == 0 ? cur[b].x : ww == 1 ? cur[b].y : ww == 2 ? cur[b].z : cur[b].w;
                pl[b] = v >> (16 * hh);
              }
              uint32_t hi[8], lo[8];
              decode16(pl, hi, lo);
              if (alive && !put(x0 + 2 * (4 * blk + ww) + hh, hi, lo)) alive = false;
            }
            if (alive && (ww & 1)) signal(x0 + 8 * blk + 2 * (ww - 1), kABatch);
          }
          if (!alive) break;
#pragma unroll
          for (int b = 0; b < BITS; ++b) cur[b] = nxt[b];
        }
      } else {
        for (int g = 0; g < gc && alive; ++g) {
          uint32_t pl[BITS];
#pragma unroll
          for (int b = 0; b < BITS; ++b) pl[b] = valid ? (__ldg(crow + b * PW + (g >> 1)) >> (16 * (g & 1))) : 0u;
          uint32_t hi[8], lo[8];
          decode16(pl, hi, lo);
          if ((alive = put(x0 + g, hi, lo))) signal(x0 + g, 1);
        }
      }
      if (m > 0 && alive) {
        const float gv = valid ? __ldg(a.rnorms + row) * gk : 0.f;
        const __half h = __float2half_rn(gv);
        const uint32_t hb = __half_as_ushort(h), lb = half_bits(gv - __half2float(h));
        const uint32_t ghi2 = hb | (hb << 16), glo2 = lb | (lb << 16);
        // sketch groups: the two halves of every sign word
        int pending = 0;
        for (int g = 0; g < 2 * MS && alive; ++g) {
          const uint32_t bits = valid ? (__ldg(srow + (g >> 1)) >> (16 * (g & 1))) : 0xFFFFu;
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int pp = 0; pp < 8; ++pp) {
            // sign bit 0 -> negative: flip the fp16 sign bits
            const uint32_t nb = ~bits >> (2 * pp);
            const uint32_t mask = ((nb & 1u) << 15) | ((nb & 2u) << 30);
            hi[pp] = ghi2 ^ mask;
            lo[pp] = glo2 ^ mask;
          }
          alive = put(x0 + gc + g, hi, lo);
          if (alive && (++pending == kABatch || g == 2 * MS - 1)) {
            signal(x0 + gc + g + 1 - pending, pending);
            pending = 0;
          }
        }
      }
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------- B producer
    if (lane == 0) {
      int64_t issued = 0;
      int st = 0, wrap = 0;  // ring stage and completed passes over the ring
      for (int64_t ul = 0; ul < nul && !s_abort; ++ul) {
        const int64_t qt = (u0 + ul) % a.nqt;
        const uint8_t* src = a.img + (size_t)qt * ngroups * kGroupBytes;
        for (int g = 0; g < ngroups; ++g) {
          if (wrap > 0 && !tqtc::mbar_wait_sleep_or_abort(&b_empty[st], (uint32_t)((wrap - 1) & 1), &s_abort, 64)) {
            fail(tqtc::kErrCopyWait);
            break;
          }
          tqtc::mbar_arrive_expect_tx(&b_full[st], (uint32_t)kGroupBytes);
          tqtc::bulk_g2s(bring + (size_t)st * kGroupBytes, src + (size_t)g * kGroupBytes, (uint32_t)kGroupBytes,
                         &b_full[st]);
          ++issued;
          if (++st == kBStages) {
            st = 0;
            ++wrap;
          }
        }
      }
      // let every copy still in flight land before the block exits (bounded)
      for (int64_t x = issued > kBStages ? issued - kBStages : 0; x < issued; ++x)
        if (!tqtc::mbar_wait_or_abort(&b_full[x % kBStages], (uint32_t)((x / kBStages) & 1), nullptr))
          atomicExch(p.err, tqtc::kErrCopyWait);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc = tqtc::instr_desc(1, 0, 0, kRowsT, kQT);
      // descriptors of slot 0 / stage 0; other slots and stages, and the lo
      // halves, are offsets of the 16-byte-unit address field
      const uint64_t adesc0 = tqtc::smem_desc(tqtc::smem_u32(aring), 2048u, 128u);
      const uint64_t bdesc0 = tqtc::smem_desc(tqtc::smem_u32(bring), 4096u, 128u);
      // fast path: the barrier is usually complete already
      auto wait_full = [&](uint64_t* bar, uint32_t parity) -> bool {
        return tqtc::mbar_try_wait(bar, parity) || tqtc::mbar_wait_or_abort(bar, parity, &s_abort);
      };
      int st = 0, wrap = 0;  // B ring stage and completed passes over the ring
      for (int64_t ul = 0; ul < nul && !s_abort; ++ul) {
        const int db = (int)(ul & 1);
        if (ul >= 2 && !tqtc::mbar_wait_or_abort(&d_empty[db], (uint32_t)((ul / 2 - 1) & 1), &s_abort)) {
          fail(tqtc::kErrMmaWait);
          break;
        }
        bool ok = true;
        const uint32_t dcol = tbase + 256u * (uint32_t)db;
        // two K groups per iteration (ngroups is even): both groups' operands
        // are checked, then their six MMAs go out back to back
        for (int g = 0; g < ngroups; g += 2) {
          const int64_t x = ul * ngroups + g;
          const int slot = (int)(x % kASlots);  // x even: slot + 1 < kASlots
          const uint32_t apar = (uint32_t)((x / kASlots) & 1);
          const int st2 = st + 1 == kBStages ? 0 : st + 1;
          const uint32_t bpar2 = (uint32_t)((st2 == 0 ? wrap + 1 : wrap) & 1);
          if (!wait_full(&a_full[slot], apar) || !wait_full(&a_full[slot + 1], apar) ||
              !wait_full(&b_full[st], (uint32_t)(wrap & 1)) || !wait_full(&b_full[st2], bpar2)) {
            fail(tqtc::kErrMmaWait);
            ok = false;
            break;
          }
          tqtc::tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int sl = slot + h, sb = h ? st2 : st;
            const uint64_t ahi = adesc0 + (uint64_t)(sl * (kASlotBytes >> 4)), alo = ahi + (4096u >> 4);
            const uint64_t bhi = bdesc0 + (uint64_t)(sb * (kGroupBytes >> 4)), blo = bhi + (uint64_t)(kStepBytes >> 4);
            tqtc::mma_f16_ss(dcol, ahi, bhi, idesc, g > 0 || h > 0);  // A_hi B_hi
            tqtc::mma_f16_ss(dcol, alo, bhi, idesc, true);            // A_lo B_hi
            tqtc::mma_f16_ss(dcol, ahi, blo, idesc, true);            // A_hi B_lo
          }
          tqtc::mma_commit(&a_empty[slot]);
          tqtc::mma_commit(&a_empty[slot + 1]);
          tqtc::mma_commit(&b_empty[st]);
          tqtc::mma_commit(&b_empty[st2]);
          if (st2 == 0) ++wrap;
          st = st2 + 1 == kBStages ? 0 : st2 + 1;
          if (st == 0 && st2 != 0) ++wrap;
        }
        if (!ok) break;
        tqtc::mma_commit(&d_full[db]);
      }
      tqtc::mma_commit(&drained);
      if (!tqtc::mbar_wait_or_abort(&drained, 0, nullptr)) atomicExch(p.err, tqtc::kErrMmaWait);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // Eight warps: warp e reads TMEM lanes 32 (warp % 4) .. of accumulator
    // columns [128 h, 128 h + 128), h = e / 4.  Per tile, a filter pass reads
    // the warp's four 32-column chunks, compares every score with its
    // query's current k-th best and appends the rare candidates to a shared
    // buffer; the accumulator is released as soon as every chunk is read.
    // The owner warp of each query (column j of a chunk -> warp j / 4) then
    // inserts that query's candidates.  A tile with more candidates than the
    // buffer holds (the first tile of every query tile, whose lists are
    // still empty) takes the staging path: scores staged in shared memory a
    // chunk per half at a time, owner warps (column j -> warp 4 h + j / 8)
    // updating their queries (few candidates in order, many by k rounds of a
    // warp argmax), the accumulator released after the last chunk.
    const uint32_t quarter = (uint32_t)(warp & 3);
    const int e8 = warp - 6;  // 0..7
    const int half = e8 >> 2;
    const int rloc = 32 * (int)quarter + lane;
    const float inv_sqrt_d = p.inv_sqrt_d;
    // bounded barrier of the eight epilogue warps (an mbarrier phase each)
    uint32_t ephase = 0u;
    auto epi_sync = [&]() -> bool {
      tqtc::mbar_arrive(&epi_bar);
      const bool ok = tqtc::mbar_wait_or_abort(&epi_bar, ephase, &s_abort);
      ephase ^= 1u;
      if (!ok) fail(tqtc::kErrMmaWait);
      return ok;
    };
    // insert (s, r) into query qi's list (one lane; the caller owns qi)
    auto insert1 = [&](int qi, float sv, int rv) {
      float* tq = tops + (size_t)qi * k;
      int* ti = tidx + (size_t)qi * k;
      if (!better(sv, rv, tq[k - 1], ti[k - 1])) return;
      int pos = k - 1;
      while (pos > 0 && better(sv, rv, tq[pos - 1], ti[pos - 1])) {
        tq[pos] = tq[pos - 1];
        ti[pos] = ti[pos - 1];
        --pos;
      }
      tq[pos] = sv;
      ti[pos] = rv;
    };
    int db = 0;          // accumulator buffer of the current tile
    uint32_t dcol = 0u;  // its first TMEM column
    auto load_chunk = [&](int c, uint32_t (&dv)[32]) {
      tqtc::tmem_ld16(tqtc::tmem_addr(tbase, 32u * quarter, dcol + 32u * c), *reinterpret_cast<uint32_t(*)[16]>(dv));
      tqtc::tmem_ld16(tqtc::tmem_addr(tbase, 32u * quarter, dcol + 32u * c + 16u),
                      *reinterpret_cast<uint32_t(*)[16]>(dv + 16));
      tqtc::tmem_wait_ld();
    };
    auto release_d = [&]() {
      tqtc::tc_fence_before();
      tqtc::mbar_arrive(&d_empty[db]);
    };
    bool alive = true;
    for (int64_t ul = 0; ul < nul && alive; ++ul) {
      const int64_t kt = (u0 + ul) / a.nqt, qt = (u0 + ul) % a.nqt;
      const int64_t row = kt * kRowsT + rloc;
      const bool valid = row < a.n;
      const float rs = valid ? __ldg(a.norms + row) * inv_sqrt_d : 0.f;
      int* ncand = &s_ncand[ul & 1];
      db = (int)(ul & 1);
      dcol = 256u * (uint32_t)db;
      if (!tqtc::mbar_wait_or_abort(&d_full[db], (uint32_t)((ul / 2) & 1), &s_abort)) {
        fail(tqtc::kErrMmaWait);
        break;
      }
      tqtc::tc_fence_after();
      // ---- filter pass over this warp's four chunks
      for (int cc = 0; cc < 4; ++cc) {
        const int c = 4 * half + cc;
        uint32_t dv[32];
        load_chunk(c, dv);
        const int qbase = (int)qt * kQT + 32 * c;
        // candidate mask first (loads only), then the rare writes
        uint32_t cmask = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int qi = qbase + j;
          if (qi < nq) {
            const float sv = __uint_as_float(dv[j]) * rs * s_qscale[qi];
            dv[j] = __float_as_uint(sv);
            const bool cnd = better(sv, (int)row, tops[(size_t)qi * k + k - 1], tidx[(size_t)qi * k + k - 1]);
            cmask |= (cnd ? 1u : 0u) << j;
          }
        }
        if (valid && cmask) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if ((cmask >> j) & 1u) {
              const int pos = atomicAdd(ncand, 1);
              if (pos < kCandCap) {
                cand_q[pos] = qbase + j;
                cand_r[pos] = (int)row;
                cand_s[pos] = __uint_as_float(dv[j]);
              }
            }
          }
        }
      }
      if (!(alive = epi_sync())) break;
      const int n_c = *reinterpret_cast<volatile int*>(ncand);
      if (e8 == 0 && lane == 0) s_ncand[(ul + 1) & 1] = 0;  // next tile's counter
      if (n_c <= kCandCap) {
        release_d();
        for (int base = 0; base < n_c; base += 32) {
          const int e = base + lane;
          const int qi = e < n_c ? cand_q[e] : -1;
          const bool mine = qi >= 0 && (((qi - (int)qt * kQT) & 31) >> 2) == e8;
          unsigned mask = __ballot_sync(0xFFFFFFFFu, mine);
          while (mask) {
            const int leader = __ffs(mask) - 1;
            if (lane == leader) insert1(qi, cand_s[e], cand_r[e]);
            mask &= mask - 1;
            __syncwarp();
          }
        }
      } else {
        // ---- staging path: chunk 4 h + cc of each half per round
        float* sbuf = stg + half * 32 * kRowsT;
        for (int cc = 0; cc < 4 && alive; ++cc) {
          const int c = 4 * half + cc;
          uint32_t dv[32];
          load_chunk(c, dv);
          if (cc == 3) release_d();
          const int qbase = (int)qt * kQT + 32 * c;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int qi = qbase + j;
            const float sc = qi < nq ? s_qscale[qi] : 0.f;
            sbuf[j * kRowsT + rloc] = valid ? __uint_as_float(dv[j]) * rs * sc : -INFINITY;
          }
          if (!(alive = epi_sync())) break;
          for (int jj = 0; jj < 8; ++jj) {
            const int j = (e8 & 3) * 8 + jj, qi = qbase + j;
            if (qi >= nq) continue;
            float* tq = tops + (size_t)qi * k;
            int* ti = tidx + (size_t)qi * k;
            const float ths = tq[k - 1];
            const int thr = ti[k - 1];
            float v[4];
            int r[4];
            unsigned cm = 0u;  // candidate bits of this lane
            int cnt = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v[i] = sbuf[j * kRowsT + lane + 32 * i];
              r[i] = (int)(kt * kRowsT) + lane + 32 * i;
              const bool cand = r[i] < a.n && better(v[i], r[i], ths, thr);
              cm |= (cand ? 1u : 0u) << i;
              cnt += __popc(__ballot_sync(0xFFFFFFFFu, cand));
            }
            if (cnt == 0) continue;
            if (cnt <= 4) {
              for (int i = 0; i < 4; ++i) {
                unsigned mask = __ballot_sync(0xFFFFFFFFu, (cm >> i) & 1u);
                while (mask) {
                  const int leader = __ffs(mask) - 1;
                  if (lane == leader) insert1(qi, v[i], r[i]);
                  mask &= mask - 1;
                  __syncwarp();
                }
              }
            } else {
              // merge: lanes < k hold the current list; k rounds of a warp argmax
              float ls = lane < k ? tq[lane] : -INFINITY;
              int lr = lane < k ? ti[lane] : 0x7FFFFFFF;
              bool lused = lane >= k;
              float outs = -INFINITY;
              int outr = 0x7FFFFFFF;
              for (int rnd = 0; rnd < k; ++rnd) {
                float bs = -INFINITY;
                int br = 0x7FFFFFFF;
                if (!lused && better(ls, lr, bs, br)) {
                  bs = ls;
                  br = lr;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  if (((cm >> i) & 1u) && better(v[i], r[i], bs, br)) {
                    bs = v[i];
                    br = r[i];
                  }
                float ws = bs;
                int wr = br;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                  const float os = __shfl_xor_sync(0xFFFFFFFFu, ws, o);
                  const int orr = __shfl_xor_sync(0xFFFFFFFFu, wr, o);
                  if (better(os, orr, ws, wr)) {
                    ws = os;
                    wr = orr;
                  }
                }
                if (lane == rnd) {
                  outs = ws;
                  outr = wr;
                }
                // the owner retires the winner (rows are distinct)
                if (!lused && lr == wr) lused = true;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  if (((cm >> i) & 1u) && r[i] == wr) cm &= ~(1u << i);
              }
              __syncwarp();
              if (lane < k) {
                tq[lane] = outs;
                ti[lane] = outr;
              }
              __syncwarp();
            }
          }
          // this pass's staging tile is read before the next pass writes it
          if (!(alive = epi_sync())) break;
        }
      }
      // every list update of this tile is done before the next filter pass
      if (alive) alive = epi_sync();
    }
  }
  tqtc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tqtc::tmem_dealloc(tbase, 512);
  // this block's lists
  float* ps = a.part_s + (size_t)blockIdx.x * nq * k;
  int* pi = a.part_i + (size_t)blockIdx.x * nq * k;
  for (int i = tid; i < nq * k; i += kThreads) {
    ps[i] = tops[i];
    pi[i] = tidx[i];
  }
}

// Merge the blocks' lists: one warp per query, k rounds of a warp argmax
// over the candidates ranked below the previous pick.
__global__ void __launch_bounds__(256) search_merge_kernel(const float* __restrict__ part_s,
                                                           const int* __restrict__ part_i, int nblk, int nq, int k,
                                                           int q0, int32_t* __restrict__ idx, float* __restrict__ score) {
  const int lane = threadIdx.x & 31;
  const int qi = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (qi >= nq) return;
  float ps = INFINITY;
  int pr = -1;
  for (int r = 0; r < k; ++r) {
    float bs = -INFINITY;
    int br = 0x7FFFFFFF;
    for (int c = lane; c < nblk * k; c += 32) {
      const int blk = c / k, j = c % k;
      const float s = part_s[((size_t)blk * nq + qi) * k + j];
      const int rr = part_i[((size_t)blk * nq + qi) * k + j];
      if (rr == 0x7FFFFFFF) continue;
      if (better(ps, pr, s, rr) && better(s, rr, bs, br)) {
        bs = s;
        br = rr;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xFFFFFFFFu, bs, o);
      const int orr = __shfl_xor_sync(0xFFFFFFFFu, br, o);
      if (better(os, orr, bs, br)) {
        bs = os;
        br = orr;
      }
    }
    if (lane == 0) {
      idx[(size_t)(q0 + qi) * k + r] = br;
      score[(size_t)(q0 + qi) * k + r] = bs;
    }
    ps = bs;
    pr = br;
  }
}

int g_sms_search = 0;
int sms() {
  if (!g_sms_search) {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_sms_search = v;
  }
  return g_sms_search;
}

}  // namespace

// query batch: the largest multiple of 256 (or nq) whose lists fit 64 KB (512
// queries at k = 10; each batch re-reads the index, so batches stay large)
int tq_search_batch(int nq, int k) {
  const int per = 8 * k + 4;
  int nb = (64 * 1024 / per) / kQT * kQT;
  if (nb < kQT) nb = kQT;
  return nq < nb ? nq : nb;
}

size_t tq_search_bytes(const tq_params& p, int nq, int k, int nsm) {
  const int nb = tq_search_batch(nq, k);
  const int nqt = (nb + kQT - 1) / kQT;
  const int ngroups = p.d / 16 + p.m / 16;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return al(sizeof(float) * (size_t)nb * (p.d + p.m)) + al(sizeof(int) * nb) + al(sizeof(float) * nb) +
         al((size_t)nqt * ngroups * kGroupBytes) + 2 * al(sizeof(float) * (size_t)nsm * nb * k);
}

int tq_search_sms() { return sms(); }

cudaError_t tq_launch_search(const tq_params& p, const float* qprep, int nq, int q0, const tq_compressed& X,
                             int64_t n, int k, int32_t* idx, float* score, void* ws, cudaStream_t st) {
  const int nb = nq;  // this batch (<= tq_search_batch)
  const int nqt = (nb + kQT - 1) / kQT;
  const int ngroups = p.d / 16 + p.m / 16;
  const int nsm = sms();
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  // qprep sits at the start of the workspace (written by the caller)
  w += al(sizeof(float) * (size_t)tq_search_batch(nb, k) * (p.d + p.m));
  int* qexp = reinterpret_cast<int*>(w);
  w += al(sizeof(int) * tq_search_batch(nb, k));
  float* qscale = reinterpret_cast<float*>(w);
  w += al(sizeof(float) * tq_search_batch(nb, k));
  uint8_t* img = w;
  w += al((size_t)nqt * ngroups * kGroupBytes);
  const int64_t nkt = (n + kRowsT - 1) / kRowsT;
  const int grid = (int)std::min<int64_t>((int64_t)nsm, nkt * nqt);
  float* part_s = reinterpret_cast<float*>(w);
  w += al(sizeof(float) * (size_t)nsm * tq_search_batch(nb, k) * k);
  int* part_i = reinterpret_cast<int*>(w);

  search_qexp_kernel<<<(nb + 7) / 8, 256, 0, st>>>(qprep, nb, p.d, p.m, qexp, qscale);
  const int64_t nth = (int64_t)nqt * kQT * ngroups;
  search_bimg_kernel<<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(qprep, qexp, nb, nqt, p.d, p.m, img);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  SearchArgs a;
  a.codes = X.codes;
  a.signs = X.signs;
  a.norms = X.norms;
  a.rnorms = X.rnorms;
  a.n = n;
  a.nq = nb;
  a.nqt = nqt;
  a.k = k;
  a.img = img;
  a.qscale = qscale;
  a.part_s = part_s;
  a.part_i = part_i;
  // the B ring takes what shared memory the rest leaves (227 KB per block,
  // 2 KB kept for the static part)
  const size_t fixed = (size_t)kASlots * kASlotBytes + 2 * 32 * kRowsT * 4 + (size_t)nb * 4 + (size_t)nb * k * 8;
  a.bstages = (int)std::min<size_t>(kBStagesMax, (227 * 1024 - 2048 - fixed) / kGroupBytes);
  if (a.bstages < 2) return cudaErrorNotSupported;
  size_t smem = (size_t)a.bstages * kGroupBytes + fixed;
  // the block takes all 512 TMEM columns: ask for more than half of the SM's
  // shared memory so that a second block never waits on the allocation
  {
    int dev = 0, per_sm = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess || per_sm <= 0)
      per_sm = 228 * 1024;
    smem = std::max(smem, (size_t)(per_sm / 2 + 1024));
  }
  switch (p.bits[0]) {
#define TQ_SEARCH_CASE(B)                                                                                  \
  case B: {                                                                                                \
    auto fn = search_kernel<B>;                                                                            \
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                  \
    if (e != cudaSuccess) return e;                                                                        \
    fn<<<grid, kThreads, smem, st>>>(p, a);                                                                \
    break;                                                                                                 \
  }
    TQ_SEARCH_CASE(1)
    TQ_SEARCH_CASE(2)
    TQ_SEARCH_CASE(3)
    TQ_SEARCH_CASE(4)
#undef TQ_SEARCH_CASE
    default: return cudaErrorNotSupported;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  search_merge_kernel<<<(nb + 7) / 8, 256, 0, st>>>(part_s, part_i, grid, nb, k, q0, idx, score);
  return cudaGetLastError();
}
