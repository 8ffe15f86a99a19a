// Internal definitions shared by the host code and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/tq.h"

#define TQ_MAX_LEVELS 16
#define TQ_MAX_VQ_BITS 8  // FibQuant k = 2: at most 256 codewords
#define TQ_MAX_M 1024
#define TQ_HBLOCK_MAX 512  // longest Hadamard block; longer vectors use blocks

// Everything a kernel needs about a codec, passed by value as a kernel argument.
struct tq_params {
  int d;          // head dimension
  int nseg;       // 1 or 2 segments (coordinate halves)
  int seg_len;    // d / nseg
  int pw;         // words per bit plane = seg_len / 32
  int m;          // QJL rows (0: none)
  int W;          // code words per row
  int MS;         // sign words per row = m / 32
  int hblock;     // Hadamard block length p
  int log2_hblock;
  int bits[2];    // bits per segment
  int segbase[2]; // first code word of each segment in a row
  float zscale;   // sqrt(d / p): z = H(D u) * zscale
  float inv_sqrt_d;
  float inv_sqrt_p;
  float qjl_coef; // sqrt(pi/2) / m
  float cmax;     // max |centroid| over segments
  float cen[2][TQ_MAX_LEVELS];
  float bnd[2][TQ_MAX_LEVELS];  // 2^bits - 1 used, rest +inf
  const float* S;       // [m][d] row-major
  const float* St;      // [d][m] transposed, columns permuted: column lane*Q + q = row lane + 32q
  const float* s_l1;    // [m] sum_i |S_ji| (permuted like St's columns)
  const float* s_l2;    // [m] ||S_j||_2    (permuted like St's columns)
  const uint32_t* dbits;  // [ceil(d/32)] bit t of word w set <=> D_{32w+t} = -1
  // tables of the tensor-core quantiser (m <= 256, d <= 128)
  const uint16_t* bimg;   // fp16 S_hi then S_lo, each [m][d] in the K-major no-swizzle
                          // core-matrix layout: (j, i) at (i/8)*16m + (j/8)*128 + (j%8)*16 + (i%8)*2 bytes
  const uint32_t* dmask;  // [d] 0x80000000 where D_i = -1, else 0
  const float* sl1n;      // [m] sum_i |S_ji| (natural row order)
  const float* sl2n;      // [m] ||S_j||_2
  // fused rotate-half RoPE of tq_quantize_rope and tq_append (rope_cs null:
  // none): cos/sin cache [rope_max_pos][d] with cos(pos theta_i) at i < d/2 and
  // sin(pos theta_i) at d/2 + i; row r takes position rope_pos[r], or
  // rope_pos_fixed when rope_pos is null
  const float* rope_cs;
  const int32_t* rope_pos;
  int rope_max_pos;
  int rope_pos_fixed;
  // dense Haar rotation (TQ_ROTATION_HAAR): Pi^T [d][d] fp32, element (i, j)
  // = Pi_ji, so that lanes reading consecutive j at fixed i are coalesced; the
  // codec's D signs are all +1
  int haar;
  const float* piT;
  // FibQuant k = 2 block codes (vq_bits > 0; bits/nseg/cen/bnd unused):
  // vq_pw words per plane (d / 64), vq_cb [2^vq_bits][2] fp32 in z units
  int vq_bits;
  int vq_pw;
  const float* vq_cb;
  // per-element residual sign (TQ_RESIDUAL_SIGN): rnorms hold this constant
  // instead of ||r|| (0 with the QJL sketch)
  float rnorm_const;
  int rnorm_is_const;
  // output rows: input row r is written to compressed row r * out_stride + out_offset
  int64_t out_stride;
  int64_t out_offset;
  uint32_t* err;          // device error word (bounded waits that gave up), zero when healthy
  unsigned long long* exact_rows;  // rows re-evaluated in fp64 since the last reset
  // plane identity of the symmetric codebooks: with s_k = 2 bit_k - 1,
  //   cen[code] = sum_t alpha[seg][t] * prod_{k in term t} s_k,
  // over the odd subsets of planes (term masks tq_term_mask[bits][t]); the
  // product of an odd subset equals 2 * xor(bits) - 1.
  int nterms[2];
  float alpha[2][8];
  int plane_ok;   // 1 if the identity reproduces every centroid (always, for
                  // exactly symmetric codebooks)
};

// odd subsets of the bit planes, as bit masks, per bit width (1..4)
static const int tq_term_mask[5][8] = {{0}, {1}, {1, 2}, {1, 2, 4, 7}, {1, 2, 4, 8, 7, 11, 13, 14}};
static const int tq_term_count[5] = {0, 1, 2, 4, 8};

struct tq_codec {
  tq_spec spec;
  int device;  // -1: host-only
  tq_params p;
  std::vector<float> S_host;        // [m][d]
  std::vector<uint32_t> dbits_host; // [ceil(d/32)]
  std::vector<float> cen_host[2];
  std::vector<float> bnd_host[2];
  double mu = 0.0;  // TQ_RESIDUAL_SIGN: mean residual magnitude (z units)
  std::vector<double> haar;  // TQ_ROTATION_HAAR: Pi [d][d] row-major, fp64
  std::vector<float> vq_host;  // FibQuant codebook [2^vq_bits][2] (z units)
  // device allocations (one block)
  void* dev_block = nullptr;
};

// thread-local error detail
void tq_set_error(const char* fmt, ...);
tq_status tq_fail(tq_status st, const char* fmt, ...);

// launchers implemented in the .cu files; arguments already validated
cudaError_t tq_launch_quantize(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                               const tq_compressed& out, cudaStream_t st);
// tensor-core quantiser; returns cudaErrorNotSupported when the codec or dtype
// has no tensor-core variant (the caller then uses the generic kernel)
cudaError_t tq_launch_quantize_tc(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                  const tq_compressed& out, cudaStream_t st);
// the same with the fused RoPE of p.rope_cs (tq_quantize_rope.cu)
cudaError_t tq_launch_quantize_tc_rope(const tq_params& p, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                       const tq_compressed& out, cudaStream_t st);
// fills a RoPE cos/sin cache [max_pos][d] in fp64, rounded to fp32
cudaError_t tq_launch_rope_cache(double theta, int d, int max_pos, float* cs, cudaStream_t st);
// tensor-core scorer: whether it takes the shape, the workspace bytes it
// needs after the query-prep block (0 if the configuration has no
// tensor-core variant), and the launch (query image, then the scoring
// kernel) on prepared queries
bool tq_scores_tc_supported(const tq_params& p, int Hq, int Hkv);
size_t tq_scores_tc_bytes(const tq_params& p, int B, int Hq, int Hkv);
cudaError_t tq_launch_scores_tc(const tq_params& p, const float* qprep, int B, int Hq, int Hkv, int64_t T,
                                const tq_compressed& K, float* logits, void* ws_tc, cudaStream_t st);
cudaError_t tq_launch_qprep(const tq_params& p, const void* q, tq_dtype dt, int nq, float* qprep,
                            cudaStream_t st);
cudaError_t tq_launch_scores(const tq_params& p, const float* qprep, int B, int Hq, int Hkv, int64_t T,
                             const tq_compressed& K, float* logits, cudaStream_t st);
int tq_attend_chunks(int B, int Hq, int Hkv, int64_t T, int num_sms);
// top-k search (tq_search.cu): queries per batch, workspace bytes, and one
// batch of nq queries (qprep at the start of ws, written by the caller)
int tq_search_batch(int nq, int k);
size_t tq_search_bytes(const tq_params& p, int nq, int k, int nsm);
cudaError_t tq_launch_search(const tq_params& p, const float* qprep, int nq, int q0, const tq_compressed& X,
                             int64_t n, int k, int32_t* idx, float* score, void* ws, cudaStream_t st);
// fused attention (tq_attend.cu): d in {64, 128}, m <= 256; cudaErrorNotSupported otherwise
cudaError_t tq_launch_attend_fused(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq,
                                   int Hkv, int64_t T, float scale, const tq_compressed& K, const tq_compressed& V,
                                   float* partials, int nchunk, cudaStream_t st);
cudaError_t tq_launch_attend(const tq_params& kp, const tq_params& vp, const float* qprep, int B, int Hq,
                             int Hkv, int64_t T, float scale, const tq_compressed& K, const tq_compressed& V,
                             float* partials, int nchunk, float* out, cudaStream_t st);
