/*
 * tq.h -- C ABI of libtq: TurboQuant-style KV-cache compression and scoring
 * over the compressed keys and values, for NVIDIA B200 (sm_100a).
 *
 * The method (as the source pages describe it):
 *   "FibQuant: Quantizacao Vetorial Universal para Compressao de KV-Cache de
 *   Acesso Aleatorio", section 1: a random-access codec stores the vector norm,
 *   applies a shared random orthogonal rotation and quantises every rotated
 *   coordinate with a scalar Lloyd-Max table; section 2.3: the decoder reads
 *   the codes, undoes the rotation and scales by the norm; every token's record
 *   has a fixed size and a fixed address.
 *   "TurboQuant: Compressao Avancada da Google para Cache KV ...", section
 *   "TurboQuant: Uma Nova Abordagem": the rotation is a randomized Hadamard
 *   transform and a 1-bit quantized Johnson-Lindenstrauss (QJL) stage on the
 *   residual makes inner-product estimates unbiased.
 *   "Compressao KV eficaz com TurboQuant", section "Por dentro do processo":
 *   the JL transform of the residual is reduced to one sign bit per projected
 *   coordinate.
 *   "TurboESM ...", "Resumo tecnico" section 2: one fused decode kernel
 *   dequantises and runs an online softmax with no dequantised copy.
 *
 * Definitions used by every call (d = head dimension, m = QJL rows):
 *   nu = ||x||_2,  u = x / nu (u = 0 if nu = 0)
 *   y  = Pi u,  Pi = blockdiag(H_p, ..., H_p) diag(D) / sqrt(p),
 *        H_p the Sylvester-Hadamard matrix H[i][j] = (-1)^popcount(i & j),
 *        p = d if d is a power of two, else p = 512 (d a multiple of 512);
 *        D = +-1 signs drawn from the codec seed
 *   z  = sqrt(d) y                         (unit-variance rotated coordinate)
 *   code_i = #{k : bnd_k <= z_i}           (Lloyd-Max cells, ties go up)
 *   r  = y - cen[code] / sqrt(d),  gamma = ||r||_2
 *   bit_j = ((S r)_j >= 0),  S an m x d matrix of iid N(0,1) fp32 entries
 *   estimate of <q, x>:
 *        nu * ( <Pi q, cen[code]> / sqrt(d)
 *               + gamma * sqrt(pi/2) / m * <S Pi q, 2 bit - 1> )
 *
 * Conventions.
 *   - Every pointer passed to a compute call is a device pointer on the codec's
 *     device, 16-byte aligned, owned by the caller.  The library owns only the
 *     tq_codec.  Compute calls allocate no memory: tq_scores and tq_attend take
 *     a caller workspace sized by their *_workspace_size call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream.  The calling thread's current
 *     device must be the codec's device.
 *   - Arguments are validated on the host before anything is launched; on any
 *     error nothing is written and the status says why
 *     (tq_last_error_string() has the detail, per thread).  Errors of earlier
 *     asynchronous work surface as TQ_ERR_CUDA on a later call or at sync.
 *   - A codec is immutable after creation; concurrent calls on distinct
 *     streams are safe.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* bad size, pointer, alignment, device or enum */
  TQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d = 96)       */
  TQ_ERR_NO_MEMORY = 3,     /* codec creation could not allocate             */
  TQ_ERR_CUDA = 4,          /* a CUDA runtime call failed                    */
  TQ_ERR_DEVICE_ASSERT = 5, /* a kernel reported a failed internal check     */
  TQ_ERR_NOT_CONVERGED = 6  /* Lloyd-Max iteration limit reached             */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* Codec parameters.
 *   d        : 64, 128, 256, 512, 1024 or 1536 (1024 and 1536 rotate in
 *              512-coordinate Hadamard blocks)
 *   nseg     : 1, or 2 = the two coordinate halves [0, d/2) and [d/2, d) use
 *              seg_bits[0] and seg_bits[1] bits (e.g. 2 + 3 = 2.5 bits/coord)
 *   seg_bits : 1..4 bits per coordinate for each segment
 *   m        : QJL rows, 0 (MSE-only codes, no signs, no residual norm) or a
 *              multiple of 32, at most 1024
 *   seed     : draws D (splitmix64 from `seed`, top bit 1 -> -1) and S
 *              (splitmix64 from seed ^ 0x5851F42D4C957F2D, Box-Muller cosine
 *              branch on output pairs, double, rounded to fp32, row-major m x d)
 *   residual : TQ_RESIDUAL_QJL (0) or TQ_RESIDUAL_SIGN (1), see tq_residual
 *   rotation : TQ_ROTATION_RHT (0) or TQ_ROTATION_HAAR (1), see tq_rotation
 *   vq_bits  : 0 = scalar Lloyd-Max codes (seg_bits); 1..8 = FibQuant k = 2
 *              vector codes (FibQuant page, sections 2.2-2.3): the rotated
 *              coordinates are cut into d/2 blocks (z_2j, z_2j+1), each block
 *              stores the index of its nearest codeword among N = 2^vq_bits,
 *              i.e. vq_bits / 2 bits per coordinate (0.5 .. 4, half steps);
 *              needs nseg = 1 (seg_bits is then ignored) and TQ_RESIDUAL_QJL.
 *              The codebook (in z units, fp32, see tq_codec_vq_codebook) is a
 *              planar Fibonacci spiral, point n at angle n * 2 pi (1 - 1/phi)
 *              and radius r_n = sqrt(d (1 - (1 - (n + 1/2)/N)^(4/d))) (the
 *              Bennett-Gersho density f^(1/2) of the block law), refined by
 *              40 Lloyd iterations over the 16384 quasi-Monte-Carlo points
 *              i = 0.. of that law (radius sqrt(d (1 - (1 - (i + 1/2)/16384)
 *              ^(2/(d-2)))), angle i * 2 pi (1 - 1/phi)); three restarts turn
 *              the spiral by r/3 of the golden angle, the least-distortion one
 *              is kept.  Code = the nearest codeword (ties: lower index).    */
typedef struct {
  int32_t d;
  int32_t nseg;
  int32_t seg_bits[2];
  int32_t m;
  uint64_t seed;
  int32_t residual;   /* tq_residual: form of the 1-bit residual stage */
  int32_t rotation;   /* tq_rotation: the shared random rotation Pi */
  int32_t vq_bits;    /* 0: scalar codes; 1..8: FibQuant k = 2 block codes */
} tq_spec;

/* Rotation (tq_spec.rotation).
 *   TQ_ROTATION_RHT  : Pi = blockdiag(H_p) diag(D) / sqrt(p), the randomized
 *                      Hadamard transform (TurboQuant news page).
 *   TQ_ROTATION_HAAR : a dense Haar-distributed orthogonal Pi (FibQuant page,
 *                      section 1, step 2, "rotacao ortogonal aleatoria
 *                      compartilhada (Haar)"): the Q of the QR factorisation,
 *                      R with a positive diagonal, of a d x d matrix of iid
 *                      N(0, 1) drawn like S from splitmix64(seed ^
 *                      0x2545F4914F6CDD1D); D = I.  d <= 256; it is applied
 *                      as dense products (encoder, query preparation, inverse
 *                      rotation of the attention output).                    */
typedef enum { TQ_ROTATION_RHT = 0, TQ_ROTATION_HAAR = 1 } tq_rotation;

/* Residual stage (tq_spec.residual).
 *   TQ_RESIDUAL_QJL  : sign(S r) with the seeded Gaussian S (m rows) and
 *                      gamma = ||r|| stored per row (the TurboQuant pages).
 *   TQ_RESIDUAL_SIGN : one sign bit per coordinate, sign(r_i), with a constant
 *                      magnitude mu (TurboESM page, "Resumo tecnico" section 2,
 *                      "Correcao de Residuo QJL de 1 Bit": the sign of the
 *                      quantisation residual per element plus a first-order
 *                      correction by the residual's mean magnitude).  mu is
 *                      E|z - cen[code(z)]| under the rotated-coordinate law
 *                      f_d, computed from the codebook (no data calibration).
 *                      Requires nseg = 1 and m = d; the codec then uses S = I,
 *                      and the stored per-row "rnorms" hold the constant
 *                      mu sqrt(2d/pi), so that every estimator term reads
 *                        nu (<Pi q, cen[code]> + mu <Pi q, 2 bit - 1>) / sqrt(d). */
typedef enum { TQ_RESIDUAL_QJL = 0, TQ_RESIDUAL_SIGN = 1 } tq_residual;

/* One compressed row per vector, structure-of-arrays, all caller-owned device
 * memory with n rows:
 *   codes  [n][W] uint32, W = sum_s seg_bits[s] * (d / nseg) / 32.
 *          Planar layout: segments in order; inside segment s, bit planes
 *          p = 0..seg_bits[s]-1; inside a plane, word w holds bit p of the codes
 *          of the segment's coordinates 32w..32w+31, coordinate 32w+t at bit t.
 *          FibQuant codes (vq_bits > 0): W = vq_bits * d / 64, planes
 *          p = 0..vq_bits-1 of d/64 words; word w of plane p holds bit p of
 *          the codeword indices of blocks 32w..32w+31, block 32w+t at bit t.
 *   signs  [n][m/32] uint32, bit j%32 of word j/32 = bit_j; NULL iff m == 0
 *   norms  [n] fp32, nu
 *   rnorms [n] fp32, gamma; NULL iff m == 0                                   */
typedef struct {
  uint32_t *codes;
  uint32_t *signs;
  float *norms;
  float *rnorms;
} tq_compressed;

typedef struct tq_codec tq_codec; /* opaque: codebooks, D, S, device tables */

/* Lloyd-Max codebook for the rotated-coordinate law (host only, pure).
 * Solves the 2^bits-level MSE-optimal scalar quantiser of
 *   f_d(z) = C_d (1 - z^2/d)^((d-3)/2),  |z| < sqrt(d),
 * the exact marginal of sqrt(d) * u_1 for u uniform on the unit sphere (the
 * "Beta" coordinate law the explainer page attributes to the random rotation;
 * the FibQuant page's k = 1 spherical-Beta source), alternating the midpoint
 * and centroid conditions until the centroids move by less than `tol`.
 *   bits in 1..4; d >= 4; tol <= 0 selects 1e-12; max_iter <= 0 selects 20000.
 *   centroids  [2^bits]     out, ascending, symmetric, fp32 of the double solution
 *   boundaries [2^bits - 1] out, fp32 of the double midpoints
 * Returns TQ_ERR_NOT_CONVERGED (outputs untouched) if max_iter is reached.   */
TQ_API tq_status tq_make_codebook(int bits, int d, double tol, int max_iter,
                           float *centroids, float *boundaries);

/* Create a codec for `spec` on CUDA device `device` (uploads D, S, codebooks
 * and derived tables; this call allocates device memory).  device = -1 makes a
 * host-only codec usable with tq_codec_export and tq_codec_layout only.
 * *out is set only on TQ_OK.                                                 */
TQ_API tq_status tq_codec_create(const tq_spec *spec, int device, tq_codec **out);

/* Free a codec (NULL is a no-op).  The caller must ensure no work using it is
 * still in flight.                                                           */
TQ_API tq_status tq_codec_destroy(tq_codec *codec);

/* Host copies of the codec's random draws and codebooks, for checking.
 * Any pointer may be NULL to skip it.
 *   S      [m][d] fp32
 *   dsigns [ceil(d/32)] words, bit t of word w set  <=>  D_{32w+t} = -1
 *   cen    [sum_s 2^seg_bits[s]]      per-segment centroids, concatenated
 *   bnd    [sum_s 2^seg_bits[s] - 1]  per-segment boundaries, concatenated    */
TQ_API tq_status tq_codec_export(const tq_codec *codec, float *S, uint32_t *dsigns,
                          float *cen, float *bnd);

/* FibQuant codebook of a codec with vq_bits > 0: cb [2^vq_bits][2] fp32, in
 * z units (codeword n = (cb[n][0], cb[n][1]) reconstructs the block
 * (z_2j, z_2j+1)).  TQ_ERR_INVALID_ARG for a scalar codec.                  */
TQ_API tq_status tq_codec_vq_codebook(const tq_codec *codec, float *cb);

/* The codec's rotation as a dense matrix: Pi [d][d] fp32 row-major, y = Pi u
 * (host copy, for checking; the Hadamard rotation is expanded).            */
TQ_API tq_status tq_codec_rotation(const tq_codec *codec, float *Pi);

/* Row sizes of the compressed format in 32-bit words (either pointer may be
 * NULL): code_words = W, sign_words = m / 32.                               */
TQ_API tq_status tq_codec_layout(const tq_codec *codec, int *code_words,
                          int *sign_words);

/* Compress n rows (encoder of the FibQuant page, section 2.3, plus the QJL
 * residual sketch of the TurboQuant pages).
 *   x     [n][ld] elements of `dtype` (TQ_F32, TQ_BF16 or TQ_F16); row i
 *         starts at element i*ld; ld >= d and ld * sizeof(dtype) % 16 == 0
 *   out   device arrays with n rows (see tq_compressed)
 * Codes and sign bits equal those of an exact (real-arithmetic) evaluation of
 * the definitions above: a fast fp32 evaluation decides every code and sign
 * whose margin exceeds a proven fp32 error bound, and the few rows with a
 * closer decision are recomputed in fp64.  n = 0 is a no-op.                */
TQ_API tq_status tq_quantize(const tq_codec *codec, const void *x, tq_dtype dtype,
                      int64_t n, int64_t ld, const tq_compressed *out,
                      void *stream);

/* Rotary position embedding fused into the encoder (TurboESM page, "Resumo
 * tecnico" section 2, "Pipeline de Transformacao Ortogonal Invariante ao
 * RoPE": RoPE is applied first and the orthogonal rotation after it, so the
 * attention scores of the rotated vectors equal those of the RoPE'd ones).
 * Rotate-half convention, pairs (i, i + d/2), theta_i = theta^(-2i/d):
 *   x'_i       = x_i cos(pos theta_i) - x_{i+d/2} sin(pos theta_i)
 *   x'_{i+d/2} = x_i sin(pos theta_i) + x_{i+d/2} cos(pos theta_i),  i < d/2.
 *   cos_sin    device [max_pos][d] fp32, 16-byte aligned: entry (pos, i) is
 *              cos(pos theta_i) for i < d/2 and sin(pos theta_{i-d/2}) for
 *              i >= d/2 (tq_rope_cache fills it)
 *   positions  device [n] int32, the position of each row (tq_quantize_rope);
 *              tq_append ignores it (every appended row is at position t).
 * x' is evaluated in fp32 with a fixed operation order and then encoded
 * exactly as tq_quantize encodes an fp32 row; it differs from real-arithmetic
 * RoPE by a few fp32 rounding errors, so only coordinates whose rotated value
 * lies within about 1e-6 of a decision boundary can take the other code.     */
typedef struct {
  const float *cos_sin;
  int32_t max_pos;
  const int32_t *positions;
} tq_rope;

/* Fill a cos/sin cache [max_pos][d] for tq_rope on the current device (fp64
 * arithmetic, rounded to fp32).  theta > 1 (10000 for the ESM-2 and Llama
 * models), d even.                                                          */
TQ_API tq_status tq_rope_cache(double theta, int d, int max_pos, float *cos_sin,
                               void *stream);

/* tq_quantize of the RoPE'd rows: row i is rotated by RoPE at position
 * rope->positions[i] before normalisation.  A position outside [0, max_pos)
 * is replaced by 0 and recorded as code 3 in the codec's device error word
 * (tq_codec_device_error).  Requires d = 64 or 128, TQ_BF16 or TQ_F32 rows,
 * m <= 256, scalar codes and the Hadamard rotation (else TQ_ERR_UNSUPPORTED). */
TQ_API tq_status tq_quantize_rope(const tq_codec *codec, const void *x, tq_dtype dtype,
                                  int64_t n, int64_t ld, const tq_rope *rope,
                                  const tq_compressed *out, void *stream);

/* Single-token decode append: compress one new row per (batch, KV head) into
 * its fixed slot of the cache (FibQuant page, section 1: every token's record
 * has a fixed size and address, so any token is written and decoded on its
 * own).
 *   x      [rows][ld] new key or value rows, row r = b * Hkv + h_kv
 *   cache  compressed arrays of rows * T rows; row r goes to cache row
 *          r * T + t, the layout tq_scores and tq_attend read
 *   t      position of the new token, 0 <= t < T
 *   rope   NULL, or the RoPE of the new rows at position t (t < max_pos;
 *          positions is ignored)
 * Other rows of the cache are not touched.  With RoPE the same shape limits
 * as tq_quantize_rope apply.                                                  */
TQ_API tq_status tq_append(const tq_codec *codec, const void *x, tq_dtype dtype,
                           int64_t rows, int64_t ld, const tq_rope *rope, int64_t t,
                           int64_t T, const tq_compressed *cache, void *stream);

/* Workspace bytes for tq_scores with B batches of Hq query heads over Hkv KV
 * heads (the query side is prepared per (batch, KV head) group).            */
TQ_API tq_status tq_scores_workspace_size(const tq_codec *kc, int B, int Hq,
                                          int Hkv, size_t *bytes);

/* Attention logits over compressed keys (unscaled estimator above).
 *   q       [B][Hq][d] of `dtype`, contiguous
 *   K       compressed keys, B*Hkv*T rows; key (b, h_kv, t) is row
 *           (b*Hkv + h_kv)*T + t
 *   logits  [B][Hq][T] fp32 out; query head h uses KV head h / (Hq / Hkv)
 *   workspace, ws_bytes  >= tq_scores_workspace_size(kc, B, Hq, Hkv)
 * Hq must be a multiple of Hkv, Hq / Hkv <= 32.  T = 0 is a no-op.  With
 * FibQuant codes the first term reads <q'_2j, q'_2j+1> . cb[code_j] per block. */
TQ_API tq_status tq_scores(const tq_codec *kc, const void *q, tq_dtype dtype, int B,
                    int Hq, int Hkv, int64_t T, const tq_compressed *K,
                    float *logits, void *workspace, size_t ws_bytes,
                    void *stream);

/* tq_scores for callers that cannot allocate device memory (no counterpart on
 * the source pages; it exists for callers such as code under a fixed,
 * pre-allocated memory budget, plug-ins whose host framework owns every
 * allocation, or bindings without access to CUDA's allocator).  Same
 * arguments and result as tq_scores, minus the workspace: the scratch is a
 * 2 MiB array inside libtq (held on every GPU that loads the library until
 * the process exits).
 *   - Calls needing more scratch than that (tq_scores_workspace_size(kc, B, Hq,
 *     Hkv) above 2 MiB) return TQ_ERR_UNSUPPORTED and write nothing.
 *   - The first call on a device looks up the array's device address; make it
 *     before any stream capture.  The address is cached for the life of the
 *     process and does not survive a device reset (cudaDeviceReset): no
 *     tq_scores_noalloc call may follow one in the same process.
 *   - Every call shares the one array: calls whose kernels may overlap on the
 *     GPU (other streams, other host threads) race and must be serialised.
 *   - It calls no allocator (no cudaMalloc, cudaFree or allocating library). */
TQ_API tq_status tq_scores_noalloc(const tq_codec *kc, const void *q,
                                   tq_dtype dtype, int B, int Hq, int Hkv,
                                   int64_t T, const tq_compressed *K,
                                   float *logits, void *stream);

/* Workspace bytes for tq_attend (depends on the current device's SM count). */
TQ_API tq_status tq_attend_workspace_size(const tq_codec *kc, const tq_codec *vc,
                                   int B, int Hq, int Hkv, int64_t T,
                                   size_t *bytes);

/* Decode attention over compressed keys and values (fused decode of the
 * TurboESM page, "Resumo tecnico" section 2): for each (b, h):
 *   p   = softmax over t of scale * logit(b, h, t)   (scale 0 -> 1/sqrt(d))
 *   out = Pi_v^T  sum_t p_t v~_t,  v~_t = nu_v,t cen_v[code_v,t] / sqrt(d)
 *         + nu_v,t gamma_v,t sqrt(pi/2)/m_v S_v^T (2 bit_v,t - 1)
 * i.e. the values are dequantised with their own codec `vc` and never
 * written out.  When vc has a sketch (m_v > 0, at most 128) the second term,
 * the QJL residual estimate, makes every v~_t unbiased for its value (the
 * TurboQuant pages' unbiasing stage applied to values); with m_v = 0 it is
 * absent.  Shapes as tq_scores; out [B][Hq][d] fp32.  kc and vc must have the
 * same d.  T >= 1.  FibQuant codes (vq_bits > 0) on either side run on the
 * CUDA-core kernel, which needs m_v = 0 (else TQ_ERR_UNSUPPORTED).          */
TQ_API tq_status tq_attend(const tq_codec *kc, const tq_codec *vc, const void *q,
                    tq_dtype dtype, int B, int Hq, int Hkv, int64_t T,
                    float scale, const tq_compressed *K,
                    const tq_compressed *V, void *workspace, size_t ws_bytes,
                    float *out, void *stream);

/* Workspace bytes for tq_search_topk with nq queries and top-k (k >= 1). */
TQ_API tq_status tq_search_workspace_size(const tq_codec *codec, int nq, int k,
                                          size_t *bytes);

/* Nearest-neighbour search over a compressed index (the vector-search use
 * the "Google acelera LLMs em 8 vezes" page names: an index of quantised
 * embeddings searched by inner product, with no indexing beyond quantising).
 * For every query i < nq (q: [nq][d], dtype as tq_scores) and every index row
 * t < n (index: n rows written by tq_quantize with the same codec), the score
 * is the tq_scores estimate
 *   s(i, t) = nu_t (<q'_i, cen[c_t]> / sqrt(d) + gamma_t sqrt(pi/2)/m <S q'_i, 2 b_t - 1>)
 * and idx[i][0..k) / score[i][0..k) (device, int32 / fp32, row-major) receive
 * the k best rows in descending score, ties to the lower row index.  The
 * scores are never stored in full: tensor-core tiles of 128 rows x 256
 * queries feed per-query top-k lists.  Requires scalar codes of one segment,
 * d a multiple of 32 with 64 <= d <= 2048, m <= 512, k <= 32, 1 <= k <= n,
 * n < 2^31.  The workspace (device, 256-byte aligned) is sized by
 * tq_search_workspace_size.                                                 */
TQ_API tq_status tq_search_topk(const tq_codec *codec, const void *q, tq_dtype dtype,
                                int nq, const tq_compressed *index, int64_t n, int k,
                                int32_t *idx, float *score, void *workspace,
                                size_t ws_bytes, void *stream);

/* Device-side health of a codec.  Kernels that wait on tensor-core or copy
 * completion give up after a bounded time (about two seconds), record a
 * nonzero code in the codec's device error word and return early.  This call
 * synchronises `stream`, reads the word into *code (0 = healthy, 1 = an MMA
 * completion wait timed out, 2 = a copy wait timed out), clears it, and
 * returns TQ_ERR_DEVICE_ASSERT if it was set.                                */
TQ_API tq_status tq_codec_device_error(const tq_codec *codec, void *stream,
                                       uint32_t *code);

/* Number of rows tq_quantize has re-evaluated in fp64 with this codec (rows
 * whose fp32 evaluation left some code or sign decision within its error
 * bound) since creation or the last reset.  Synchronises `stream`; reset != 0
 * zeroes the counter after reading it.                                      */
TQ_API tq_status tq_codec_exact_rows(const tq_codec *codec, void *stream,
                                     int reset, uint64_t *rows);

/* Human-readable status and the calling thread's last error detail.        */
TQ_API const char *tq_status_string(tq_status status);
TQ_API const char *tq_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
