// Tensor-core scoring of compressed keys (kind::i8 tcgen05.mma).
//
// The estimator's two dot products per (key, query) are sums of query values
// selected by key bits:
//   <q', cen[code]> = sum_{segment s, odd plane subset t} alpha_st <q'_s, sigma_t>
//   <w, sign>       = sum_j w_j sigma_j,       sigma = 2 bit - 1
// (the plane identity: a symmetric codebook's centroid is an odd multilinear
// function of the code's bit signs, and the product of an odd set of bit signs
// is 2 * xor(bits) - 1).  With sigma = 2b - 1 both become
//   sum_k b_k v_k - corr,   v_k = 2 alpha q'_i  (or 2 w_j),
// a 0/1-by-real contraction over K = 32 * (source words) per key.
//
// A (keys, M = 128 per tile) goes to TMEM as u8 bytes: source word u (a plane
// word, an xor of plane words, or a sign word) becomes eight 32-bit columns
// word & (0x01010101 << r), r < 8, so K index k = 32u + 4r + j holds
// 2^r * bit(r + 8j).  B (queries) holds round(v_k 2^(e - r)) split into four
// balanced base-256 s8 limbs, in shared memory.  The s32 accumulation is
// exact; the epilogue rebuilds I = sum_l 256^l D_l, scales by 2^-e and
// subtracts corr.
//
// Centroid-limb form (one segment of 3-bit codes): the plane identity needs
// four odd plane subsets (16 source words at d = 128), one byte of K per key
// bit.  Instead each coordinate's centroid, as the 16-bit fixed point
// C = rint(cen * 2^f) = C_0 + 256 C_1 in two balanced s8 limbs, takes two bytes
// of K: 8 source words for the first term, 12 MMAs per tile in place of 20.
// The query image of limb-1 words holds the query limbs one slot up, so both
// limbs accumulate into the same columns.  Two approximations, both far inside
// the logit tolerance of 1e-3 of nu ||q|| / sqrt(d):
//   |cen - C 2^-f| <= 2^-(f+1), f = 13 for the 3-bit codebooks (max |cen| < 4):
//     the first term moves by at most 2^-14 ||q'||_1 / sqrt(d) <= 2^-14 ||q||;
//   q' is rounded to 22 bits of its largest element (three limbs, so that the
//     shifted limb-1 image still fits four): the first term moves by at most
//     2^-22 ||q|| sqrt(d), i.e. d 2^-22 of the tolerance floor.
//
// The limb bytes come from byte permutes, not table gathers: a 3-bit code is
// a prmt selector into the eight limb bytes of the codebook held in two
// registers, so one prmt yields the limbs of four coordinates.  The selector
// word of group g < 4 of a 32-coordinate word holds the code of coordinate
// g + 4k in nibble k (masked shifts of the three plane words); its low half
// feeds TMEM column 2g and its high half column 2g + 1, so byte j of column
// 2g + h is coordinate g + 4j + 16h, and the query image uses the same order.
#include <math.h>

#include <algorithm>

#include "tq_common.cuh"
#include "tq_tc.cuh"

namespace {

constexpr int kKeys = 128;

__host__ __device__ constexpr int term_mask(int bits, int t) {
  return bits == 1 ? 1
         : bits == 2 ? (t == 0 ? 1 : 2)
         : bits == 3 ? (t < 3 ? (1 << t) : 7)
                     : (t < 4 ? (1 << t) : (t == 4 ? 7 : t == 5 ? 11 : t == 6 ? 13 : 14));
}

// the centroid-limb form applies to one segment of 3-bit codes
__host__ __device__ inline bool use_cl(const tq_params& p) { return p.nseg == 1 && p.bits[0] == 3; }

// fixed-point exponent f of the centroid limbs: the largest f with
// max |cen| * 2^f <= 32512, so that both balanced s8 limbs stay in range
__host__ __device__ inline int cl_shift(const tq_params& p) {
  int ex = 0;
  frexpf(p.cmax > 0.f ? p.cmax : 1.f, &ex);  // cmax < 2^ex
  int f = 15 - ex;
  if (ldexpf(p.cmax, f) > 32512.f) --f;
  return f;
}

// Source words of a tile, in K order: the MSE words [0, U_mse) (plane form:
// odd plane subsets; centroid-limb form: limb-0 words then limb-1 words), then
// the MS sign words.  One accumulator per tile, N columns: the MSE columns
// [0, 4G) and the QJL columns [QO, QO + 4G), four query limbs per query; the
// query image holds zeros in the QJL columns of MSE words and in the MSE
// columns of sign words, so every word of a tile accumulates into the same
// TMEM region and the epilogue reads 2 * round16(4G) columns.
struct Geom {
  int U_mse, U, Kt, G, QO, N, lbo, bbytes, gstride;
  bool cl;
  __host__ __device__ Geom(const tq_params& p, int G_) {
    cl = use_cl(p);
    U_mse = 0;
    for (int s = 0; s < p.nseg; ++s) U_mse += p.nterms[s] * p.pw;
    if (cl) U_mse = 2 * p.pw;
    U = U_mse + p.MS;
    Kt = 32 * U;
    G = G_;
    QO = ((4 * G_ + 15) / 16) * 16;
    N = 2 * QO;
    lbo = (N / 8) * 128;
    bbytes = Kt * N;
    gstride = ((bbytes + 16 * G_ + 127) / 128) * 128;  // B image + 4 floats per query
  }
  // TMEM columns of one tile slot: A (8 per source word) and D (N)
  __host__ __device__ uint32_t acols() const { return 8u * (uint32_t)U; }
  __host__ __device__ uint32_t slot_cols() const { return acols() + (uint32_t)N; }
};

// K byte k of a centroid-limb word holds coordinate cl_coord(k) of the word's
// 32 (see the expansion: byte j of TMEM column 2g + h is g + 4j + 16h)
__host__ __device__ inline int cl_coord(int k) { return (k >> 3) + 4 * (k & 3) + 16 * ((k >> 2) & 1); }

// ------------------------------------------------------------ B operand
// Query image.  Blocks (group, part): every block of a (batch, KV head) group
// copies the group's G prepared query rows [q' (d) | w = S q' (m)] into shared
// memory and computes the per-query exponents, then writes part `blockIdx.y`
// of the group's image (part 0 also the per-query constants).
//   MSE columns, plane words: limb l of round(2 alpha q'_i 2^(e - r)), |.| < 2^30
//   MSE columns, centroid-limb words: the three limbs of round(q'_i 2^e),
//       |.| < 2^22, in slots 0..2 for limb-0 words and 1..3 (times 256) for
//       limb-1 words, so that slot l sums 256^l-weighted centroid limbs
//   QJL columns, sign words: limb l of round(2 w_j 2^(e - r)), |.| < 2^30
// The scoring kernel is launched as its programmatic dependent: it starts
// streaming keys while this kernel runs and waits for its results only where
// it reads them.
__global__ void __launch_bounds__(256) tq_scores_bbuild_kernel(const tq_params p, const float* __restrict__ qprep,
                                                               const int Hq, const int Hkv, uint8_t* __restrict__ ws) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) float qw[];  // [G][d + m]: q' then w
  const Geom g(p, Hq / Hkv);
  const int grp = blockIdx.x, b = grp / Hkv, hk = grp % Hkv;
  const int d = p.d, m = p.m, L = p.seg_len, ld = d + m;
  __shared__ int s_xmse[32], s_xqjl[32];    // exponents e
  uint8_t* out = ws + (size_t)grp * g.gstride;
  float* consts = reinterpret_cast<float*>(out + g.bbytes);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x / 32;
  for (int i = threadIdx.x; i < g.G * ld; i += blockDim.x)
    qw[i] = qprep[(size_t)(b * Hq + hk * g.G) * ld + i];
  __syncthreads();
  for (int gq = warp; gq < g.G; gq += nw) {
    const float* qv = qw + gq * ld;
    float mx = 0.f, corr = 0.f;
    for (int s = 0; s < p.nseg; ++s) {
      float amax = 0.f, qmax = 0.f, qsum = 0.f;
      for (int t = 0; t < p.nterms[s]; ++t) amax = fmaxf(amax, fabsf(p.alpha[s][t]));
      float asum = 0.f;
      for (int t = 0; t < p.nterms[s]; ++t) asum += p.alpha[s][t];
      for (int i = lane; i < L; i += 32) {
        const float v = qv[s * L + i];
        qmax = fmaxf(qmax, fabsf(v));
        qsum += v;
      }
      qmax = tq_warp_max(qmax);
      qsum = tq_warp_sum(qsum);
      if (g.cl) {
        mx = qmax;  // centroid limbs: the image holds q' itself, no correction
      } else {
        mx = fmaxf(mx, 2.f * amax * qmax);
        corr += asum * qsum;
      }
    }
    float wmax = 0.f, wsum = 0.f;
    for (int j = lane; j < m; j += 32) {
      const float v = qv[d + j];
      wmax = fmaxf(wmax, fabsf(v));
      wsum += v;
    }
    wmax = tq_warp_max(wmax);
    wsum = tq_warp_sum(wsum);
    if (lane == 0) {
      int ex;
      frexpf(mx > 0.f ? mx : 1.f, &ex);
      const int em = (g.cl ? 22 : 30) - ex;  // |v| 2^em < 2^22 (three limbs) or 2^30 (four)
      frexpf(wmax > 0.f ? 2.f * wmax : 1.f, &ex);
      const int eq = 30 - ex;
      s_xmse[gq] = em;
      s_xqjl[gq] = eq;
      if (blockIdx.y == 0) {
        consts[4 * gq + 0] = ldexpf(1.f, -em);
        consts[4 * gq + 1] = corr;
        consts[4 * gq + 2] = ldexpf(1.f, -eq);
        consts[4 * gq + 3] = wsum;
      }
    }
  }
  __syncthreads();
  const int u0 = p.nterms[0] * p.pw;
  const int total = g.Kt * g.N, per = (total + gridDim.y - 1) / gridDim.y;
  const int i0 = blockIdx.y * per, i1 = min(total, i0 + per);
  for (int idx = i0 + threadIdx.x; idx < i1; idx += blockDim.x) {
    const int n = idx / g.Kt, k = idx % g.Kt;
    const bool qjl_col = n >= g.QO;
    const int gq = (qjl_col ? n - g.QO : n) / 4, l = n % 4;
    const int u = k / 32, r = (k % 32) / 4, j = k % 4, bp = r + 8 * j;
    const bool sign_word = u >= g.U_mse;
    int8_t limb = 0;
    if (gq < g.G && qjl_col == sign_word) {
      const float* qv = qw + gq * ld;
      float v;
      int e, sh = r, slot = l;
      if (!sign_word && g.cl) {
        // limb h = u / pw of the centroids of word u % pw, coordinates in the
        // expansion's order; limb-1 words see the query limbs one slot up
        v = qv[32 * (u % p.pw) + cl_coord(k % 32)];
        e = s_xmse[gq];
        sh = 0;
        slot = l - u / p.pw;
      } else if (!sign_word) {
        const int s = (p.nseg == 2 && u >= u0) ? 1 : 0;
        const int uu = s ? u - u0 : u;
        const int t = uu / p.pw, w = uu % p.pw;
        v = 2.f * p.alpha[s][t] * qv[s * L + 32 * w + bp];
        e = s_xmse[gq];
      } else {
        v = 2.f * qv[d + 32 * (u - g.U_mse) + bp];
        e = s_xqjl[gq];
      }
      int x = __float2int_rn(ldexpf(v, e - sh));
      // balanced base-256 digits
      int lv = 0;
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        const int dq = (int)(int8_t)(x & 0xFF);
        if (qd == slot) lv = dq;
        x = (x - dq) >> 8;
      }
      limb = (int8_t)lv;
    }
    const int off = (k / 16) * g.lbo + (n / 8) * 128 + (n % 8) * 16 + (k % 16);
    out[off] = (uint8_t)limb;
  }
}

// ------------------------------------------------------------ scoring
// Warp-specialised, one block per SM, tiles of 128 keys of one (batch, KV
// head) group; a block owns a contiguous range of tiles.  Tile i of the block
// uses slot i % NI: A buffer and accumulator in TMEM, MMA issuer warp.
//   warps 0-7   expansion, two groups of four: group i % 2 reads tile i's
//               codes/signs from the ring and builds its A operand (u8 planes
//               or s8 centroid limbs); warp w owns TMEM lanes 32(w%4)..+31
//   warps 8-15  epilogue, two groups of four: group i % 2 reads tile i's
//               accumulator, rebuilds the two sums and writes the logits
//   warps 16-17 producers: warp 16 + x makes the bulk copies of the tiles of
//               parity x (codes, signs, norms) into the ring; warp 16 also
//               copies each group's query operand into one of two buffers.  A
//               ring stage is free once the tile's expansion group (codes,
//               signs) and epilogue group (norms) have both read it
//   warps 18-21 MMA issue: warp 18 + j issues every MMA of the tiles in slot j
// A tcgen05.mma stream from one thread costs about a hundred cycles per
// instruction at these shapes, while streams from different warps into
// different accumulators overlap on the tensor core: hence one issuer per slot.
// mbarriers: ring_full/ring_empty (producer <-> expansion), a_full[j]
// (expansion -> issuer j), a_free[j] (issuer j's commit -> expansion),
// d_full[j] (issuer j's commit -> epilogue), d_empty[j] (epilogue -> issuer
// j), b_full/b_empty (producer <-> issuers, query operand).  NI is even and
// the expansion and epilogue groups split tiles by parity, so each barrier's
// phases are waited for in order by one consumer: a wait on a phase parity
// then never meets its barrier a phase behind (which would pass at once) or
// two phases ahead (which would never pass).
constexpr int kStages = 12;  // even: stage st only ever holds tiles of parity st % 2
constexpr int kMaxSlots = 4;
constexpr int kExpWarps = 8, kEpiWarps = 8;
constexpr int kEpiWarp0 = kExpWarps, kProdWarp = kExpWarps + kEpiWarps, kIssWarp0 = kProdWarp + 2;
constexpr int kThreads = 32 * (kIssWarp0 + kMaxSlots);

// one ring stage: codes [128][W], signs [128][MS], norms [128], rnorms [128]
__host__ __device__ inline int ring_stage_bytes(int W, int MS) { return kKeys * (W + MS + 2) * 4; }

// Position of a block's tile in (group, first key): one division at the start,
// then a running count (a 64-bit division per tile costs hundreds of cycles in
// a single-thread loop).
struct TileCursor {
  int64_t grp, t0;
  __device__ TileCursor(int64_t tile, int64_t tpg) {
    grp = tile / tpg;
    t0 = (tile - grp * tpg) * kKeys;
  }
  // moves `step` tiles on; groups hold tpg tiles, i.e. tpg * kKeys keys
  __device__ void advance(int step, int64_t tpg_keys) {
    t0 += (int64_t)step * kKeys;
    while (t0 >= tpg_keys) {
      t0 -= tpg_keys;
      ++grp;
    }
  }
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

template <int D, int B0, int B1, bool RING, int NI>
__global__ void __launch_bounds__(kThreads, 1)
    tq_scores_tc_kernel(const tq_params p, const tq_compressed K, float* __restrict__ logits,
                        const uint8_t* __restrict__ ws, const int Hq, const int Hkv, const int64_t T,
                        const int64_t tiles_per_group, const int64_t ntiles) {
  constexpr int NSEG = B1 > 0 ? 2 : 1;
  constexpr int PW = (D / NSEG) / 32;
  constexpr int W = (B0 + B1) * PW;
  constexpr int NT0 = B0 == 1 ? 1 : B0 == 2 ? 2 : B0 == 3 ? 4 : 8;
  constexpr int NT1 = B1 == 0 ? 0 : B1 == 1 ? 1 : B1 == 2 ? 2 : B1 == 3 ? 4 : 8;
  constexpr bool CL = B0 == 3 && B1 == 0;  // centroid-limb form (use_cl)
  constexpr int U_MSE = CL ? 2 * PW : (NT0 + NT1) * PW;
  static_assert(NI % 2 == 0 && NI <= kMaxSlots, "tile slots must split evenly between the two tile parities");

  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t ring_full[kStages], ring_empty[kStages];
  __shared__ uint64_t a_full[NI], a_free[NI], d_full[NI], d_empty[NI], b_full[2], b_empty[2], drained[NI];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const Geom g(p, Hq / Hkv);
  const int MS = p.MS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bstride = ((g.bbytes + 16 * g.G + 127) / 128) * 128;  // one query-operand buffer
  unsigned char* bbuf = smem;                                     // [2][bstride]
  unsigned char* ring = smem + 2 * bstride;                       // [kStages][ring_stage_bytes]
  const int sbytes = ring_stage_bytes(W, MS);
  const uint32_t scols = g.slot_cols(), acols = g.acols();        // slot j: A at j * scols, D after it

  const int64_t t_begin = (int64_t)blockIdx.x * ntiles / gridDim.x;
  const int64_t t_end = (int64_t)(blockIdx.x + 1) * ntiles / gridDim.x;
  const int64_t ntl = t_end - t_begin;
  const int64_t tpg_keys = tiles_per_group * kKeys;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      tqtc::mbar_init(&ring_full[i], 1);
      tqtc::mbar_init(&ring_empty[i], RING ? 256 : 128);
    }
    for (int i = 0; i < NI; ++i) {
      tqtc::mbar_init(&a_full[i], 128);
      tqtc::mbar_init(&a_free[i], 1);
      tqtc::mbar_init(&d_full[i], 1);
      tqtc::mbar_init(&d_empty[i], 128);
      tqtc::mbar_init(&drained[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tqtc::mbar_init(&b_full[i], 1);
      tqtc::mbar_init(&b_empty[i], (uint32_t)NI);
    }
    tqtc::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0) tqtc::tmem_alloc(&s_tmem, 512);
  tqtc::tc_fence_before();
  __syncthreads();
  tqtc::tc_fence_after();
  const uint32_t tbase = s_tmem;
  auto fail = [&](uint32_t code) {
    atomicExch(p.err, code);
    s_abort = 1;
  };

  if (warp == kProdWarp || warp == kProdWarp + 1) {
    // ---------------------------------------------------------- producers
    const int px = warp - kProdWarp;  // tile parity of this producer
    if (lane == 0) {
      int64_t cur = -1, issued = 0;
      int gi = -1;
      TileCursor tc(t_begin, tiles_per_group);
      bool dep_done = false;
      for (int64_t i = 0; i < ntl && !s_abort; ++i, tc.advance(1, tpg_keys)) {
        const int64_t grp = tc.grp;
        if (RING && (int)(i & 1) == px) {
          const int st = (int)(i % kStages);
          if (i >= kStages &&
              !tqtc::mbar_wait_or_abort(&ring_empty[st], (uint32_t)((i / kStages - 1) & 1), &s_abort)) {
            fail(tqtc::kErrCopyWait);
            break;
          }
          const int64_t t0 = tc.t0;
          const int64_t rows = (T - t0) < kKeys ? (T - t0) : kKeys;
          const int64_t row0 = grp * T + t0;
          unsigned char* dst = ring + (size_t)st * sbytes;
          const uint32_t bc = (uint32_t)(rows * W * 4), bs = (uint32_t)(rows * MS * 4), bn = (uint32_t)(rows * 4);
          tqtc::mbar_arrive_expect_tx(&ring_full[st], bc + bs + (MS > 0 ? 2u : 1u) * bn);
          tqtc::bulk_g2s(dst, K.codes + row0 * W, bc, &ring_full[st]);
          if (MS > 0) tqtc::bulk_g2s(dst + kKeys * W * 4, K.signs + row0 * MS, bs, &ring_full[st]);
          unsigned char* dn = dst + kKeys * (W + MS) * 4;
          tqtc::bulk_g2s(dn, K.norms + row0, bn, &ring_full[st]);
          if (MS > 0) tqtc::bulk_g2s(dn + kKeys * 4, K.rnorms + row0, bn, &ring_full[st]);
          issued = i + 1;
        }
        if (px == 0 && grp != cur) {
          if (!dep_done) {  // the query image comes from the preceding prep kernel
            asm volatile("griddepcontrol.wait;" ::: "memory");
            dep_done = true;
          }
          cur = grp;
          ++gi;
          const int gb = gi & 1;
          if (gi >= 2 && !tqtc::mbar_wait_or_abort(&b_empty[gb], (uint32_t)((gi / 2 - 1) & 1), &s_abort)) {
            fail(tqtc::kErrCopyWait);
            break;
          }
          tqtc::mbar_arrive_expect_tx(&b_full[gb], (uint32_t)bstride);
          tqtc::bulk_g2s(bbuf + gb * bstride, ws + (size_t)grp * g.gstride, (uint32_t)bstride, &b_full[gb]);
        }
      }
      // let every copy still in flight land before the block exits (bounded)
      for (int64_t i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
        if ((int)(i & 1) == px &&
            !tqtc::mbar_wait_or_abort(&ring_full[i % kStages], (uint32_t)((i / kStages) & 1), nullptr))
          atomicExch(p.err, tqtc::kErrCopyWait);
      for (int j = gi > 0 ? gi - 1 : 0; j <= gi; ++j)
        if (!tqtc::mbar_wait_or_abort(&b_full[j & 1], (uint32_t)((j / 2) & 1), nullptr))
          atomicExch(p.err, tqtc::kErrCopyWait);
    }
  } else if (warp >= kIssWarp0) {
    // ---------------------------------------------------------- MMA issue
    const int js = warp - kIssWarp0;  // tile slot of this issuer
    if (lane == 0 && js < NI) {
      // centroid limbs are signed; masked plane and sign bytes reach 128
      const uint32_t idesc_u8 = tqtc::instr_desc(2, 0, 1, kKeys, (uint32_t)g.N);  // A u8, B s8
      const uint32_t idesc_s8 = tqtc::instr_desc(2, 1, 1, kKeys, (uint32_t)g.N);  // A s8, B s8
      const uint32_t a0 = tbase + (uint32_t)js * scols, dst = a0 + acols;
      const uint64_t step = (uint64_t)((2u * (uint32_t)g.lbo) >> 4);
      int64_t cur = -1;
      int gi = -1;
      TileCursor tc(t_begin, tiles_per_group);
      for (int64_t i = 0; i < ntl && !s_abort; ++i, tc.advance(1, tpg_keys)) {
        const int64_t grp = tc.grp;
        // every issuer follows the group changes (b_full, b_empty), whatever
        // the slots of the tiles that carry them
        if (grp != cur) {
          if (gi >= 0) tqtc::mma_commit(&b_empty[gi & 1]);  // previous group's operand is free once done
          cur = grp;
          ++gi;
          if (!tqtc::mbar_wait_or_abort(&b_full[gi & 1], (uint32_t)((gi / 2) & 1), &s_abort)) {
            fail(tqtc::kErrCopyWait);
            break;
          }
        }
        if ((int)(i % NI) != js) continue;
        const uint32_t ph = (uint32_t)((i / NI) & 1);
        if (!tqtc::mbar_wait_or_abort(&a_full[js], ph, &s_abort)) {
          fail(tqtc::kErrMmaWait);
          break;
        }
        if (i >= NI && !tqtc::mbar_wait_or_abort(&d_empty[js], ph ^ 1u, &s_abort)) {
          fail(tqtc::kErrMmaWait);
          break;
        }
        tqtc::tc_fence_after();
        uint64_t desc = tqtc::smem_desc(tqtc::smem_u32(bbuf + (gi & 1) * bstride), (uint32_t)g.lbo, 128);
        // unrolled: the issuing thread shares its SMSP with busy warps, so
        // every instruction between two MMAs costs several cycles
#pragma unroll
        for (int u = 0; u < U_MSE + 8; ++u) {
          if (u < U_MSE + MS) {
            tqtc::mma_i8_ts(dst, a0 + 8u * (uint32_t)u, desc, (CL && u < U_MSE) ? idesc_s8 : idesc_u8, u != 0);
            desc += step;
          }
        }
        tqtc::mma_commit(&a_free[js]);
        tqtc::mma_commit(&d_full[js]);
      }
      // every MMA issued has completed before TMEM is released (bounded)
      tqtc::mma_commit(&drained[js]);
      if (!tqtc::mbar_wait_or_abort(&drained[js], 0, nullptr)) atomicExch(p.err, tqtc::kErrMmaWait);
    }
  } else if (warp < kExpWarps) {
    // ---------------------------------------------------------- expansion
    const uint32_t lane_base = 32u * (uint32_t)(warp & 3);
    const int xg = warp >> 2, kt = tid & 127;  // tile parity of this group, key of this thread
    // centroid limbs as prmt tables: byte c of (tl, th) is limb h of code c
    uint32_t tl0 = 0u, th0 = 0u, tl1 = 0u, th1 = 0u;
    if constexpr (CL) {
      const float sc = ldexpf(1.f, cl_shift(p));
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int v = __float2int_rn(p.cen[0][c] * sc);
        const int h0 = (int)(int8_t)(v & 0xFF), h1 = (v - h0) >> 8;
        const uint32_t b0 = (uint32_t)(h0 & 0xFF), b1 = (uint32_t)(h1 & 0xFF);
        if (c < 4) {
          tl0 |= b0 << (8 * c);
          tl1 |= b1 << (8 * c);
        } else {
          th0 |= b0 << (8 * (c - 4));
          th1 |= b1 << (8 * (c - 4));
        }
      }
    }
    TileCursor tc(t_begin + xg, tiles_per_group);
    for (int64_t i = xg; i < ntl; i += 2, tc.advance(2, tpg_keys)) {
      const int64_t grp = tc.grp;
      const int64_t t0 = tc.t0;
      const int js = (int)(i % NI);
      const bool valid = t0 + kt < T;
      uint32_t kcw[W], ksw[8];
#pragma unroll
      for (int k = 0; k < W; ++k) kcw[k] = 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k) ksw[k] = 0u;
      if constexpr (RING) {
        const int st = (int)(i % kStages);
        if (!tqtc::mbar_wait_or_abort(&ring_full[st], (uint32_t)((i / kStages) & 1), &s_abort)) {
          fail(tqtc::kErrCopyWait);
          break;
        }
        if (valid) {
          const unsigned char* src = ring + (size_t)st * sbytes;
          const uint32_t* c32 = reinterpret_cast<const uint32_t*>(src) + kt * W;
          if constexpr (W % 4 == 0) {
#pragma unroll
            for (int k = 0; k < W; k += 4) {
              const uint4 q4 = *reinterpret_cast<const uint4*>(c32 + k);
              kcw[k] = q4.x; kcw[k + 1] = q4.y; kcw[k + 2] = q4.z; kcw[k + 3] = q4.w;
            }
          } else if constexpr (W % 2 == 0) {
#pragma unroll
            for (int k = 0; k < W; k += 2) {
              const uint2 q2 = *reinterpret_cast<const uint2*>(c32 + k);
              kcw[k] = q2.x; kcw[k + 1] = q2.y;
            }
          } else {
#pragma unroll
            for (int k = 0; k < W; ++k) kcw[k] = c32[k];
          }
          const uint32_t* s32 = reinterpret_cast<const uint32_t*>(src + kKeys * W * 4) + kt * MS;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (k < MS) ksw[k] = s32[k];
        }
        tqtc::mbar_arrive(&ring_empty[st]);
      } else if (valid) {
        const int64_t row = grp * T + t0 + kt;
#pragma unroll
        for (int k = 0; k < W; ++k) kcw[k] = __ldg(K.codes + row * W + k);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k < MS) ksw[k] = __ldg(K.signs + row * MS + k);
      }
      // slot js's A is free once the MMAs of tile i - NI are done
      if (i >= NI && !tqtc::mbar_wait_or_abort(&a_free[js], (uint32_t)((i / NI - 1) & 1), &s_abort)) {
        fail(tqtc::kErrMmaWait);
        break;
      }
      tqtc::tc_fence_after();
      const uint32_t a0 = (uint32_t)js * scols;
      auto emit = [&](int u, uint32_t word) {
        uint32_t regs[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) regs[r] = word & (0x01010101u << r);
        tqtc::tmem_st8(tqtc::tmem_addr(tbase, lane_base, a0 + 8u * (uint32_t)u), regs);
      };
      if constexpr (CL) {
#pragma unroll
        for (int w = 0; w < PW; ++w) {
          const uint32_t p0 = kcw[w], p1 = kcw[PW + w], p2 = kcw[2 * PW + w];
          uint32_t r0[8], r1[8];
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            // nibble k: code of coordinate gg + 4k (bit 4k + j from plane j)
            const uint32_t x1 = gg >= 1 ? p1 >> (gg - 1) : p1 << 1;
            const uint32_t x2 = gg >= 2 ? p2 >> (gg - 2) : p2 << (2 - gg);
            const uint32_t sel = ((p0 >> gg) & 0x11111111u) | (x1 & 0x22222222u) | (x2 & 0x44444444u);
            const uint32_t shi = sel >> 16;
            r0[2 * gg] = prmt(tl0, th0, sel);
            r1[2 * gg] = prmt(tl1, th1, sel);
            r0[2 * gg + 1] = prmt(tl0, th0, shi);
            r1[2 * gg + 1] = prmt(tl1, th1, shi);
          }
          tqtc::tmem_st8(tqtc::tmem_addr(tbase, lane_base, a0 + 8u * (uint32_t)w), r0);
          tqtc::tmem_st8(tqtc::tmem_addr(tbase, lane_base, a0 + 8u * (uint32_t)(PW + w)), r1);
        }
      } else {
#pragma unroll
        for (int s = 0; s < NSEG; ++s) {
          const int bits = s ? B1 : B0;
          const int base = s ? B0 * PW : 0;
          const int nt = s ? NT1 : NT0;
          const int ubase = s ? NT0 * PW : 0;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (t < nt) {
              const int mask = term_mask(bits, t);
#pragma unroll
              for (int w = 0; w < PW; ++w) {
                uint32_t word = 0u;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  if ((mask >> k) & 1) word ^= kcw[base + k * PW + w];
                emit(ubase + t * PW + w, word);
              }
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (k < MS) emit(U_MSE + k, ksw[k]);
      tqtc::tmem_wait_st();
      tqtc::tc_fence_before();
      tqtc::mbar_arrive(&a_full[js]);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int eg = (warp - kEpiWarp0) >> 2, et = (tid - 32 * kEpiWarp0) & 127;  // tile parity, key
    const uint32_t lane_base = 32u * (uint32_t)(warp & 3);
    const float kcl = CL ? ldexpf(p.inv_sqrt_d, -cl_shift(p)) : 0.f;  // 2^-f / sqrt(d)
    TileCursor tc(t_begin + eg, tiles_per_group);
    int64_t cur = -1;
    int bq = 0, hk = 0;
    // the key norms: from the tile's ring stage, or (no ring) loaded from
    // global memory one tile ahead
    auto load_norms = [&](const TileCursor& c, float& nu, float& gam) {
      const bool ok = c.t0 + et < T;
      const int64_t r = c.grp * T + c.t0 + et;
      nu = ok ? __ldg(K.norms + r) : 0.f;
      gam = (ok && MS > 0) ? __ldg(K.rnorms + r) : 0.f;
    };
    float nxt_nu = 0.f, nxt_gam = 0.f;
    if (!RING && eg < ntl) load_norms(tc, nxt_nu, nxt_gam);
    asm volatile("griddepcontrol.wait;" ::: "memory");  // per-query constants of the prep kernel
    for (int64_t i = eg; i < ntl; i += 2, tc.advance(2, tpg_keys)) {
      const int64_t grp = tc.grp;
      const int64_t t0 = tc.t0;
      const int js = (int)(i % NI);
      if (grp != cur) {  // (batch, KV head) of the group, once per group
        cur = grp;
        bq = (int)(grp / Hkv);
        hk = (int)(grp - (int64_t)bq * Hkv);
      }
      const int64_t t = t0 + et;
      const bool valid = t < T;
      float knu, kgam;
      if constexpr (RING) {
        const int st = (int)(i % kStages);
        if (!tqtc::mbar_wait_or_abort(&ring_full[st], (uint32_t)((i / kStages) & 1), &s_abort)) {
          fail(tqtc::kErrCopyWait);
          break;
        }
        const float* nr = reinterpret_cast<const float*>(ring + (size_t)st * sbytes + kKeys * (W + MS) * 4);
        knu = valid ? nr[et] : 0.f;
        kgam = (valid && MS > 0) ? nr[kKeys + et] : 0.f;
        tqtc::mbar_arrive(&ring_empty[st]);
      } else {
        knu = nxt_nu;
        kgam = nxt_gam;
        if (i + 2 < ntl) {
          TileCursor nc = tc;
          nc.advance(2, tpg_keys);
          load_norms(nc, nxt_nu, nxt_gam);
        }
      }
      const float* cs_all = reinterpret_cast<const float*>(ws + (size_t)grp * g.gstride + g.bbytes);
      if (!tqtc::mbar_wait_or_abort(&d_full[js], (uint32_t)((i / NI) & 1), &s_abort)) {
        fail(tqtc::kErrMmaWait);
        break;
      }
      tqtc::tc_fence_after();
      const uint32_t dset = (uint32_t)js * scols + acols;
      const float cq = kgam * p.qjl_coef;
      for (int qc = 0; qc < g.QO / 16; ++qc) {
        // per-query constants of the group (2^-e scales, correction sums),
        // requested before the accumulator loads so that both latencies overlap
        float4 cs[4];
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4)
          cs[g4] = (4 * qc + g4 < g.G) ? __ldg(reinterpret_cast<const float4*>(cs_all) + 4 * qc + g4)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t dm[16], dq[16];
        tqtc::tmem_ld16(tqtc::tmem_addr(tbase, lane_base, dset + 16u * qc), dm);
        if (MS > 0) tqtc::tmem_ld16(tqtc::tmem_addr(tbase, lane_base, dset + (uint32_t)g.QO + 16u * qc), dq);
        tqtc::tmem_wait_ld();
        if (qc == g.QO / 16 - 1) {
          tqtc::tc_fence_before();
          tqtc::mbar_arrive(&d_empty[js]);
        }
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          const int gq = 4 * qc + g4;
          if (gq < g.G && valid) {
            // I = sum_l 256^l D_l over the query's four limb columns (exact s32 sums)
            float im = (float)(int)dm[4 * g4 + 3];
            im = fmaf(im, 256.f, (float)(int)dm[4 * g4 + 2]);
            im = fmaf(im, 256.f, (float)(int)dm[4 * g4 + 1]);
            im = fmaf(im, 256.f, (float)(int)dm[4 * g4 + 0]);
            float val;
            if constexpr (CL)
              val = (im * cs[g4].x) * kcl;
            else
              val = fmaf(im, cs[g4].x, -cs[g4].y) * p.inv_sqrt_d;
            if (MS > 0) {
              float iq = (float)(int)dq[4 * g4 + 3];
              iq = fmaf(iq, 256.f, (float)(int)dq[4 * g4 + 2]);
              iq = fmaf(iq, 256.f, (float)(int)dq[4 * g4 + 1]);
              iq = fmaf(iq, 256.f, (float)(int)dq[4 * g4 + 0]);
              val = fmaf(cq, fmaf(iq, cs[g4].z, -cs[g4].w), val);
            }
            logits[((int64_t)bq * Hq + hk * g.G + gq) * T + t] = knu * val;
          }
        }
      }
    }
  }
  tqtc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tqtc::tmem_dealloc(tbase, 512);
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

int smem_per_sm() {
  static int v = 0;
  if (!v) {
    int dev = 0, x = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&x, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess || x <= 0)
      x = 228 * 1024;
    v = x;
  }
  return v;
}

bool supported(const tq_params& p, int G, uint32_t* cols_out) {
  if (!p.plane_ok || (p.d != 64 && p.d != 128)) return false;
  if (p.m > 256) return false;
  if (!(p.nseg == 1 || (p.bits[0] == 2 && p.bits[1] == 3))) return false;
  const Geom g(p, G);
  if (g.bbytes > 64 * 1024 || g.N > 256) return false;
  if (2u * g.slot_cols() > 512) return false;  // two tile slots at least
  // query-operand buffers and key ring in the shared memory of one block
  int W = 0;
  for (int s = 0; s < p.nseg; ++s) W += p.bits[s] * p.pw;
  const size_t bstride = (size_t)((g.bbytes + 16 * G + 127) / 128) * 128;
  if (2 * bstride + (size_t)kStages * ring_stage_bytes(W, p.MS) > 224u * 1024u) return false;
  if (cols_out) *cols_out = 512;
  return true;
}

template <int D, int B0, int B1, bool RING, int NI>
cudaError_t launch_scores_t(const tq_params& p, const tq_compressed& K, float* logits, const uint8_t* ws, int B,
                            int Hq, int Hkv, int64_t T, cudaStream_t st) {
  constexpr int W = (B0 + B1) * ((D / (B1 > 0 ? 2 : 1)) / 32);
  const Geom g(p, Hq / Hkv);
  const size_t bstride = (size_t)((g.bbytes + 16 * g.G + 127) / 128) * 128;
  size_t smem = 2 * bstride + (RING ? (size_t)kStages * ring_stage_bytes(W, p.MS) : 0);
  // the block takes all 512 TMEM columns: ask for more than half of the SM's
  // shared memory so that a second block never waits on the allocation
  smem = std::max(smem, (size_t)(smem_per_sm() / 2 + 1024));
  auto fn = tq_scores_tc_kernel<D, B0, B1, RING, NI>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t tpg = (T + kKeys - 1) / kKeys;
  const int64_t ntiles = (int64_t)B * Hkv * tpg;
  const int grid = (int)std::min<int64_t>(ntiles, (int64_t)sm_count());
  // programmatic dependent launch: the block's set-up and key stream overlap
  // the tail of the prep kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fn, p, K, logits, ws, Hq, Hkv, T, tpg, ntiles);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int B0, int B1>
cudaError_t launch_scores(const tq_params& p, const tq_compressed& K, float* logits, const uint8_t* ws, int B,
                          int Hq, int Hkv, int64_t T, uint32_t cols, cudaStream_t st) {
  (void)cols;
  // bulk copies need 16-byte aligned tile starts and sizes: T a multiple of 4
  const bool ring = (T % 4) == 0 && (uintptr_t)K.codes % 16 == 0 && (p.MS == 0 || (uintptr_t)K.signs % 16 == 0);
  // four tile slots where TMEM holds them, else two (always an even count)
  const Geom g(p, Hq / Hkv);
  if ((uint32_t)kMaxSlots * g.slot_cols() <= 512u)
    return ring ? launch_scores_t<D, B0, B1, true, kMaxSlots>(p, K, logits, ws, B, Hq, Hkv, T, st)
                : launch_scores_t<D, B0, B1, false, kMaxSlots>(p, K, logits, ws, B, Hq, Hkv, T, st);
  return ring ? launch_scores_t<D, B0, B1, true, 2>(p, K, logits, ws, B, Hq, Hkv, T, st)
              : launch_scores_t<D, B0, B1, false, 2>(p, K, logits, ws, B, Hq, Hkv, T, st);
}

}  // namespace

size_t tq_scores_tc_bytes(const tq_params& p, int B, int Hq, int Hkv) {
  if (Hkv <= 0 || Hq % Hkv) return 0;
  if (!supported(p, Hq / Hkv, nullptr)) return 0;
  const Geom g(p, Hq / Hkv);
  return (size_t)B * Hkv * g.gstride;
}

bool tq_scores_tc_supported(const tq_params& p, int Hq, int Hkv) {
  return Hkv > 0 && Hq % Hkv == 0 && !p.vq_bits && supported(p, Hq / Hkv, nullptr);
}

cudaError_t tq_launch_scores_tc(const tq_params& p, const float* qprep, int B, int Hq, int Hkv, int64_t T,
                                const tq_compressed& K, float* logits, void* ws_tc, cudaStream_t st) {
  uint32_t cols = 0;
  if (!supported(p, Hq / Hkv, &cols)) return cudaErrorNotSupported;
  uint8_t* ws = reinterpret_cast<uint8_t*>(ws_tc);
  const size_t smem = sizeof(float) * (size_t)(Hq / Hkv) * (p.d + p.m);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(tq_scores_bbuild_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
  }
  tq_scores_bbuild_kernel<<<dim3((unsigned)(B * Hkv), 8), 256, smem, st>>>(p, qprep, Hq, Hkv, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  switch (p.d * 100 + p.bits[0] * 10 + (p.nseg == 2 ? p.bits[1] : 0)) {
    case 12810: return launch_scores<128, 1, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 12820: return launch_scores<128, 2, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 12830: return launch_scores<128, 3, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 12840: return launch_scores<128, 4, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 12823: return launch_scores<128, 2, 3>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 6410: return launch_scores<64, 1, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 6420: return launch_scores<64, 2, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 6430: return launch_scores<64, 3, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 6440: return launch_scores<64, 4, 0>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
    case 6423: return launch_scores<64, 2, 3>(p, K, logits, ws, B, Hq, Hkv, T, cols, st);
  }
  return cudaErrorNotSupported;
}
