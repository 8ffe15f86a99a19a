"""Plain, slow, double-precision CPU oracle of the TurboQuant-style path.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What it computes, and where that is stated (page titles as they appear in the
source pages):

* "FibQuant: Quantizacao Vetorial Universal ...", section 1 (the three-step
  interface of TURBOQUANT: store the norm, apply a shared random orthogonal
  rotation, quantise every rotated coordinate with a scalar Lloyd-Max table)
  and section 2.3 (encoder: nu = ||x||, rotate x / nu; decoder: codes ->
  inverse rotation -> scale by the norm).
* "TurboQuant: Compressao Avancada da Google ...", section "TurboQuant: Uma
  Nova Abordagem": the rotation is a randomized Hadamard transform that keeps
  Euclidean geometry, and a quantized Johnson-Lindenstrauss (QJL) stage removes
  the inner-product bias of the first stage.
* "Compressao KV eficaz com TurboQuant", section "Por dentro do processo": the
  random rotation makes each coordinate Beta-distributed and nearly
  independent, so a scalar quantiser per coordinate is used; the MSE-optimal
  stage biases inner products; QJL projects the residual with a JL transform
  and keeps one sign bit per projected coordinate, giving an unbiased
  estimator.
* "TurboESM ...", "Resumo tecnico" section 2 (RoPE first, then the orthogonal
  rotation, so attention scores are preserved exactly; a fused decode that
  dequantises and runs an online softmax without an intermediate copy).
  ``rope_rotate_half`` is that RoPE (rotate-half pairs (i, i + d/2), angle
  pos * theta^(-2i/d)); the encoder of RoPE'd keys is ``quantize`` of its
  output.
* "FibQuant ...", section 2.2 (codebook) and 2.3 (encoder): with k = 2 the
  rotated unit vector is cut into d/2 blocks of two consecutive coordinates and
  every block takes the nearest of N = 2^vq_bits shared codewords (vq_bits / 2
  bits per coordinate).  The codebook (``fibquant_codebook``) starts from a
  planar Fibonacci spiral with Bennett-Gersho radii and is refined by Lloyd's
  algorithm with several restarts.  Readings: codewords live in z units (the
  page's unit-ball source scaled by sqrt(d)); the expectation Lloyd needs is
  taken over a deterministic quasi-Monte-Carlo point set of the block law
  (``fibquant_source_points``); 40 iterations, 3 restarts turned by a fraction
  of the golden angle, the least-distortion restart kept; codewords in fp32.
* The estimator of <q, x> that the library evaluates is
  nu * ( <Pi q, c_hat> / sqrt(d) + ||r|| * sqrt(pi/2) / m * <S Pi q, sign(S r)> ).

Readings where the pages are silent:

* rotation Pi = H_d diag(D) / sqrt(d), H_d the Sylvester-Hadamard matrix
  H[i][j] = (-1)^popcount(i & j), D iid +-1; d = 1536 uses three 512-blocks;
* the codebook is Lloyd-Max for the exact marginal of sqrt(d) * u_1, u uniform
  on the sphere S^{d-1}: f_d(z) = C_d (1 - z^2/d)^((d-3)/2) on |z| < sqrt(d)
  (the "Beta" coordinate law of the rotated unit vector); boundaries are the
  midpoints of adjacent centroids; the library publishes both in fp32;
* code_i = #{k : bnd_k <= z_i}  (z == boundary goes to the upper cell);
* residual r = y - c_hat / sqrt(d) in the rotated unit-vector space; the
  sketch matrix S (m x d, iid N(0,1), fp32) multiplies r; bit = (S r >= 0);
* nu and ||r|| are stored in fp32;
* random draws: splitmix64 (S. Vigna's public-domain generator) seeded with
  ``seed`` for D (bit 63 of each output: 0 -> +1, 1 -> -1) and with
  ``seed ^ 0x5851F42D4C957F2D`` for S (Box-Muller cosine branch on two outputs,
  evaluated in double, rounded to fp32).

Parity pins live in ``tests/test_oracle_pins.py``.  Parity unpinned: none of the
functions below (every one has at least one independent pin); the pages' own
quality figures (cosine similarities, perplexities, recall) are not reproduced
here because they need model weights and datasets.
"""
from __future__ import annotations

import dataclasses
import functools
import math
from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np
from scipy import integrate, special

__all__ = [
    "splitmix64", "rademacher_signs", "gaussian_sketch", "S_SEED_XOR",
    "sylvester_hadamard", "rotation_matrix", "Codec", "make_codec",
    "fd_density", "fd_normaliser", "gaussian_density", "lloyd_max", "published_codebook",
    "Compressed", "quantize", "quantize_with", "pack_codes", "unpack_codes", "pack_bits", "unpack_bits",
    "estimate_scores", "attend", "dequantize", "search_topk", "exact_topk", "topk_rows", "hadamard_block",
    "rope_rotate_half", "residual_mean_magnitude", "haar_rotation", "HAAR_SEED_XOR",
    "fibquant_init", "fibquant_source_points", "fibquant_codebook", "fibquant_distortion",
]

MASK64 = (1 << 64) - 1
S_SEED_XOR = 0x5851F42D4C957F2D
HAAR_SEED_XOR = 0x2545F4914F6CDD1D
HADAMARD_BLOCK = 512          # largest Hadamard block; longer vectors use blocks


# --------------------------------------------------------------------------- PRNG
def splitmix64(seed: int, n: int) -> List[int]:
    """First n outputs of splitmix64 started at state ``seed`` (Vigna's
    definition: state += 0x9E3779B97F4A7C15, then the two xor-shift-multiply
    rounds and a final xor-shift)."""
    s = seed & MASK64
    out = []
    for _ in range(n):
        s = (s + 0x9E3779B97F4A7C15) & MASK64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out.append(z ^ (z >> 31))
    return out


def rademacher_signs(seed: int, d: int) -> np.ndarray:
    """D_i = +1 if the top bit of the i-th output is 0, else -1."""
    return np.array([1.0 if (o >> 63) == 0 else -1.0 for o in splitmix64(seed, d)])


def gaussian_sketch(seed: int, m: int, d: int) -> np.ndarray:
    """S (m x d, row-major), one Box-Muller normal per pair of outputs, rounded
    to fp32.  U1 = ((o1 >> 11) + 1) / 2^53 in (0, 1], U2 = (o2 >> 11) / 2^53."""
    outs = splitmix64(seed ^ S_SEED_XOR, 2 * m * d)
    vals = np.empty(m * d, dtype=np.float32)
    for k in range(m * d):
        u1 = ((outs[2 * k] >> 11) + 1) * 2.0 ** -53
        u2 = (outs[2 * k + 1] >> 11) * 2.0 ** -53
        vals[k] = np.float32(math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2))
    return vals.reshape(m, d)


# ----------------------------------------------------------------------- rotation
def sylvester_hadamard(n: int) -> np.ndarray:
    """H[i][j] = (-1)^popcount(i & j), n a power of two."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    par = np.vectorize(lambda v: bin(int(v)).count("1") & 1)(i & j)
    return np.where(par == 1, -1.0, 1.0)


@functools.lru_cache(maxsize=None)
def _hadamard_cached(n: int) -> np.ndarray:
    return sylvester_hadamard(n)


def hadamard_block(d: int) -> int:
    """Block length of the randomized Hadamard rotation for head dimension d."""
    if d & (d - 1) == 0:
        return d
    if d % HADAMARD_BLOCK == 0:
        return HADAMARD_BLOCK
    raise ValueError(f"unsupported dimension {d}")


def haar_rotation(seed: int, d: int) -> np.ndarray:
    """Dense Haar-distributed orthogonal Pi (FibQuant page, section 1: a shared
    random orthogonal rotation, Haar): G is d x d iid N(0, 1), drawn like S
    (Box-Muller cosine branch on output pairs of splitmix64 from
    seed ^ HAAR_SEED_XOR, row-major, in double), and Pi is the Q of G = QR with
    the signs fixed so that diag(R) > 0 (the unique such Q, Haar-distributed
    when G is Gaussian)."""
    outs = splitmix64(seed ^ HAAR_SEED_XOR, 2 * d * d)
    g = np.empty(d * d)
    for k in range(d * d):
        u1 = ((outs[2 * k] >> 11) + 1) * 2.0 ** -53
        u2 = (outs[2 * k + 1] >> 11) * 2.0 ** -53
        g[k] = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
    Q, R = np.linalg.qr(g.reshape(d, d))
    return Q * np.sign(np.diag(R))[None, :]


def rotation_matrix(D: np.ndarray) -> np.ndarray:
    """Pi = blockdiag(H_p, ..., H_p) diag(D) / sqrt(p), p = block length."""
    d = D.shape[0]
    p = hadamard_block(d)
    Hp = _hadamard_cached(p)
    Pi = np.zeros((d, d))
    for s in range(0, d, p):
        Pi[s:s + p, s:s + p] = Hp * D[None, s:s + p] / math.sqrt(p)
    return Pi


# --------------------------------------------------------------------------- RoPE
def rope_rotate_half(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding in the rotate-half convention, in double:
    for i < d/2 the pair (x_i, x_{i+d/2}) of a row at position pos is rotated
    by the angle pos * theta^(-2i/d):
        x'_i       = x_i cos(a) - x_{i+d/2} sin(a)
        x'_{i+d/2} = x_i sin(a) + x_{i+d/2} cos(a)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    pos = np.asarray(positions, dtype=np.float64).reshape(-1, 1)
    ang = pos * np.power(float(theta), -2.0 * np.arange(h, dtype=np.float64) / d)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[:, :h] = x[:, :h] * c - x[:, h:] * s
    out[:, h:] = x[:, :h] * s + x[:, h:] * c
    return out


# ----------------------------------------------------------------------- codebook
def fd_normaliser(d: int) -> float:
    """C_d with int f_d = 1: Gamma(d/2) / (sqrt(pi d) Gamma((d-1)/2))."""
    return math.exp(math.lgamma(d / 2) - math.lgamma((d - 1) / 2)) / math.sqrt(math.pi * d)


def fd_density(d: int) -> Tuple[Callable[[float], float], float]:
    """Density of z = sqrt(d) * u_1, u uniform on S^{d-1}, and its support edge."""
    c = fd_normaliser(d)
    a = (d - 3) / 2.0

    def f(z: float) -> float:
        t = 1.0 - z * z / d
        return c * math.exp(a * math.log1p(-z * z / d)) if t > 0 else 0.0
    return f, math.sqrt(d)


def gaussian_density() -> Tuple[Callable[[float], float], float]:
    """N(0, 1), the d -> infinity limit of f_d (used only to pin the solver)."""
    return (lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)), math.inf


def _cell_moments(f: Callable[[float], float], lo: float, hi: float) -> Tuple[float, float]:
    p = integrate.quad(f, lo, hi, epsabs=0.0, epsrel=2e-14, limit=400)[0]
    m1 = integrate.quad(lambda z: z * f(z), lo, hi, epsabs=0.0, epsrel=2e-14, limit=400)[0]
    return p, m1


def lloyd_max(bits: int, density: Tuple[Callable[[float], float], float],
              tol: float = 1e-12, max_iter: int = 20000) -> Tuple[np.ndarray, np.ndarray, int]:
    """Lloyd-Max scalar quantiser with 2^bits levels for a symmetric density.

    Alternates the two optimality conditions until the centroids move by less
    than ``tol``: boundaries at midpoints of adjacent centroids, and each
    centroid the conditional mean of its cell.  Symmetry (c_k = -c_{L-1-k}) is
    imposed by solving the positive half only.  Returns (centroids, boundaries,
    iterations) in double precision, ascending.
    """
    f, edge = density
    L = 1 << bits
    h = L // 2
    # start from Gaussian quantiles of equal-probability half cells
    c = np.array([special.ndtri(0.5 + 0.5 * (j + 0.5) / h) for j in range(h)])
    c = np.minimum(c, 0.999 * edge) if math.isfinite(edge) else c
    it = 0
    for it in range(1, max_iter + 1):
        b = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [edge]])
        new = np.empty(h)
        for j in range(h):
            p, m1 = _cell_moments(f, b[j], b[j + 1])
            new[j] = m1 / p
        delta = np.max(np.abs(new - c))
        c = new
        if delta < tol:
            break
    else:
        raise RuntimeError("Lloyd-Max did not converge")
    cen = np.concatenate([-c[::-1], c])
    bnd = 0.5 * (cen[:-1] + cen[1:])
    return cen, bnd, it


@functools.lru_cache(maxsize=None)
def published_codebook(bits: int, d: int) -> Tuple[np.ndarray, np.ndarray]:
    """fp32 centroids and fp32 boundaries (midpoint computed in double, then
    rounded) of the Lloyd-Max quantiser for f_d."""
    cen, _, _ = lloyd_max(bits, fd_density(d))
    bnd = np.array([np.float32(0.5 * (cen[k] + cen[k + 1])) for k in range(len(cen) - 1)], dtype=np.float32)
    return cen.astype(np.float32), bnd


# ------------------------------------------------------------ FibQuant, k = 2
GOLDEN_ANGLE = math.pi * (3.0 - math.sqrt(5.0))   # 2 pi (1 - 1/phi)


def fibquant_init(N: int, d: int, offset: float = 0.0) -> np.ndarray:
    """Initial k = 2 codebook of the FibQuant page (section 2.2), in z units
    (z = sqrt(d) times the rotated unit vector): N points on a planar Fibonacci
    spiral, point n at angle n * golden_angle + offset and at the radius whose
    Bennett-Gersho point density (proportional to f^(k/(k+2)) = f^(1/2) of the
    source density f_{d,2}(z) ~ (1 - |z|^2/d)^((d-4)/2)) leaves a fraction
    (n + 1/2)/N of the points inside: Lambda(r) = 1 - (1 - r^2/d)^(d/4), so
        r_n^2 = d (1 - (1 - (n + 1/2)/N)^(4/d))."""
    n = np.arange(N, dtype=np.float64)
    r = np.sqrt(d * (1.0 - np.power(1.0 - (n + 0.5) / N, 4.0 / d)))
    a = n * GOLDEN_ANGLE + offset
    return np.stack([r * np.cos(a), r * np.sin(a)], axis=1)


def fibquant_source_points(d: int, M: int) -> np.ndarray:
    """A deterministic quasi-Monte-Carlo stand-in for the source f_{d,2}: M
    equally weighted points, point i at the radius whose radial CDF is
    (i + 1/2)/M (for u uniform on S^{d-1}, u_1^2 + u_2^2 ~ Beta(1, (d-2)/2),
    CDF 1 - (1 - t)^((d-2)/2), so |z|^2 = d (1 - (1 - (i + 1/2)/M)^(2/(d-2))))
    and at angle i * golden_angle."""
    i = np.arange(M, dtype=np.float64)
    r = np.sqrt(d * (1.0 - np.power(1.0 - (i + 0.5) / M, 2.0 / (d - 2))))
    a = i * GOLDEN_ANGLE
    return np.stack([r * np.cos(a), r * np.sin(a)], axis=1)


def _nearest(points: np.ndarray, cb: np.ndarray) -> np.ndarray:
    d2 = ((points[:, None, :] - cb[None, :, :]) ** 2).sum(axis=2)
    return np.argmin(d2, axis=1)                     # ties -> lower index


def fibquant_distortion(points: np.ndarray, cb: np.ndarray) -> float:
    """Mean squared error per 2-block of the nearest-codeword quantiser."""
    idx = _nearest(points, cb)
    return float(np.mean(((points - cb[idx]) ** 2).sum(axis=1)))


@functools.lru_cache(maxsize=None)
def fibquant_codebook(vq_bits: int, d: int, M: int = 16384, iters: int = 40, restarts: int = 3) -> np.ndarray:
    """FibQuant k = 2 codebook (page section 2.2): the Fibonacci-spiral
    initialisation refined by Lloyd's algorithm (nearest-codeword cells, then
    every codeword moved to the mean of its cell) on the quasi-Monte-Carlo
    source points, from `restarts` initial spirals turned by r * golden_angle /
    restarts; the restart with the least distortion is kept (ties: the
    first).  Returned in fp32, [N][2], z units."""
    pts = fibquant_source_points(d, M)
    N = 1 << vq_bits
    best, best_d = None, math.inf
    for rs in range(restarts):
        cb = fibquant_init(N, d, rs * GOLDEN_ANGLE / restarts)
        for _ in range(iters):
            idx = _nearest(pts, cb)
            cnt = np.bincount(idx, minlength=N)
            sx = np.bincount(idx, weights=pts[:, 0], minlength=N)
            sy = np.bincount(idx, weights=pts[:, 1], minlength=N)
            keep = cnt > 0
            cb = cb.copy()
            cb[keep, 0] = sx[keep] / cnt[keep]
            cb[keep, 1] = sy[keep] / cnt[keep]
        dist = fibquant_distortion(pts, cb)
        if dist < best_d:
            best, best_d = cb, dist
    return best.astype(np.float32)


# -------------------------------------------------------------------------- codec
def residual_mean_magnitude(cen: np.ndarray, bnd: np.ndarray, d: int) -> float:
    """mu = E|z - cen[code(z)]| for z with density f_d and the published
    codebook (the constant of the per-element residual sign): the integral of
    |z - c_k| f_d(z) over every cell, by adaptive quadrature."""
    f, edge = fd_density(d)
    e = np.concatenate([[-edge], np.asarray(bnd, np.float64), [edge]])
    mu = 0.0
    for k, c in enumerate(np.asarray(cen, np.float64)):
        for lo, hi in ((e[k], min(c, e[k + 1])), (max(c, e[k]), e[k + 1])):
            if hi > lo:
                mu += integrate.quad(lambda z: abs(z - c) * f(z), lo, hi, epsabs=0.0, epsrel=1e-13, limit=400)[0]
    return mu


@dataclasses.dataclass
class Codec:
    d: int
    seg_bits: Tuple[int, ...]
    m: int
    seed: int
    D: np.ndarray                     # (d,) +-1
    S: np.ndarray                     # (m, d) fp32
    cen: List[np.ndarray]             # per segment, fp32, ascending
    bnd: List[np.ndarray]             # per segment, fp32, ascending
    # residual stage: "qjl" (sign(S r) and ||r||) or "sign" (TurboESM: sign(r_i)
    # per coordinate and the constant mean magnitude mu; then S = I, m = d)
    residual: str = "qjl"
    mu: float = 0.0
    # rotation: "rht" (randomized Hadamard from D) or "haar" (dense, D = 1)
    rotation: str = "rht"
    haar: Optional[np.ndarray] = None
    # FibQuant k = 2 (vq_bits > 0): blocks (z_2j, z_2j+1) take the nearest of
    # the 2^vq_bits codewords of vq_cb [N][2] (fp32, z units); seg_bits unused
    vq_bits: int = 0
    vq_cb: Optional[np.ndarray] = None

    @property
    def nseg(self) -> int:
        return len(self.seg_bits)

    @property
    def seg_len(self) -> int:
        return self.d // self.nseg

    @property
    def plane_words(self) -> int:
        """Words per bit plane: ceil(segment length / 32)."""
        return (self.seg_len + 31) // 32

    @property
    def words(self) -> int:
        if self.vq_bits:
            return self.vq_bits * ((self.d // 2 + 31) // 32)
        return sum(b * self.plane_words for b in self.seg_bits)

    @functools.cached_property
    def Pi(self) -> np.ndarray:
        return self.haar if self.rotation == "haar" else rotation_matrix(self.D)

    def coord_cen(self, codes: np.ndarray) -> np.ndarray:
        """Centroid (z units) of every coordinate's code; codes (..., d).  With
        FibQuant the code of coordinate i is its block's codeword index and the
        centroid is that codeword's component i % 2."""
        if self.vq_bits:
            cb = self.vq_cb.astype(np.float64)
            return cb[codes, np.arange(self.d) % 2]
        out = np.empty(codes.shape)
        L = self.seg_len
        for s in range(self.nseg):
            out[..., s * L:(s + 1) * L] = self.cen[s].astype(np.float64)[codes[..., s * L:(s + 1) * L]]
        return out


def make_codec(d: int, seg_bits: Sequence[int], m: int, seed: int,
               D: Optional[np.ndarray] = None, S: Optional[np.ndarray] = None, residual: str = "qjl",
               rotation: str = "rht", vq_bits: int = 0) -> Codec:
    """Codec from the seed (or from explicit D and S, for Monte-Carlo tests).
    residual="sign" is TurboESM's per-element residual sign: one segment,
    m = d, S = I, and mu from the codebook.  rotation="haar" takes the dense
    Haar rotation of the seed (D = 1)."""
    seg_bits = tuple(int(b) for b in seg_bits)
    haar = None
    if rotation == "haar":
        D = np.ones(d)
        haar = haar_rotation(seed, d)
    elif D is None:
        D = rademacher_signs(seed, d)
    cen, bnd = [], []
    for b in seg_bits:
        c, bb = published_codebook(b, d)
        cen.append(c)
        bnd.append(bb)
    mu = 0.0
    if residual == "sign":
        if len(seg_bits) != 1 or m != d:
            raise ValueError("the per-element residual sign needs one segment and m = d")
        S = np.eye(d, dtype=np.float32)
        mu = residual_mean_magnitude(cen[0], bnd[0], d)
    elif S is None:
        S = gaussian_sketch(seed, m, d) if m > 0 else np.zeros((0, d), dtype=np.float32)
    vq_cb = fibquant_codebook(vq_bits, d) if vq_bits else None
    return Codec(d, seg_bits, m, seed, np.asarray(D, dtype=np.float64), np.asarray(S), cen, bnd, residual, mu,
                 rotation, haar, vq_bits, vq_cb)


# ---------------------------------------------------------------------- bit packing
def _pack_vq(codes: np.ndarray, codec: Codec) -> np.ndarray:
    """FibQuant codes: plane p (p = 0..vq_bits-1), word w holds bit p of the
    codes of blocks 32w..32w+31, block 32w+t at bit t; codes holds each
    block's index on both of its coordinates."""
    n, nb = codes.shape[0], codec.d // 2
    pw = (nb + 31) // 32
    blk = codes[:, 0::2].astype(np.uint64)
    out = np.zeros((n, codec.vq_bits * pw), dtype=np.uint64)
    for p in range(codec.vq_bits):
        for w in range(pw):
            for t in range(min(32, nb - 32 * w)):
                out[:, p * pw + w] |= ((blk[:, 32 * w + t] >> np.uint64(p)) & np.uint64(1)) << np.uint64(t)
    return out.astype(np.uint32)


def _unpack_vq(words: np.ndarray, codec: Codec) -> np.ndarray:
    n, nb = words.shape[0], codec.d // 2
    pw = (nb + 31) // 32
    w64 = words.astype(np.uint64)
    blk = np.zeros((n, nb), dtype=np.int64)
    for p in range(codec.vq_bits):
        for w in range(pw):
            for t in range(min(32, nb - 32 * w)):
                blk[:, 32 * w + t] |= ((w64[:, p * pw + w] >> np.uint64(t)) & np.uint64(1)).astype(np.int64) << p
    return np.repeat(blk, 2, axis=1)


def pack_codes(codes: np.ndarray, codec: Codec) -> np.ndarray:
    """Planar packing: segments in order; inside a segment of b bits, plane p
    (p = 0..b-1) holds bit p of each code; word w of a plane holds the codes of
    coordinates 32w..32w+31 of the segment, coordinate 32w+t at bit t (bits
    past the end of a segment shorter than a whole word are zero)."""
    if codec.vq_bits:
        return _pack_vq(codes, codec)
    n = codes.shape[0]
    L = codec.seg_len
    out = np.zeros((n, codec.words), dtype=np.uint64)
    col = 0
    for s, b in enumerate(codec.seg_bits):
        seg = codes[:, s * L:(s + 1) * L].astype(np.uint64)
        for p in range(b):
            for w in range(codec.plane_words):
                acc = np.zeros(n, dtype=np.uint64)
                for t in range(min(32, L - 32 * w)):
                    acc |= ((seg[:, 32 * w + t] >> np.uint64(p)) & np.uint64(1)) << np.uint64(t)
                out[:, col] = acc
                col += 1
    return out.astype(np.uint32)


def unpack_codes(words: np.ndarray, codec: Codec) -> np.ndarray:
    if codec.vq_bits:
        return _unpack_vq(words, codec)
    n = words.shape[0]
    L = codec.seg_len
    w64 = words.astype(np.uint64)
    codes = np.zeros((n, codec.d), dtype=np.int64)
    col = 0
    for s, b in enumerate(codec.seg_bits):
        for p in range(b):
            for w in range(codec.plane_words):
                for t in range(min(32, L - 32 * w)):
                    bit = (w64[:, col] >> np.uint64(t)) & np.uint64(1)
                    codes[:, s * L + 32 * w + t] |= bit.astype(np.int64) << p
                col += 1
    return codes


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """bits (n, m) of 0/1 -> (n, m/32) words, bit j of the row at bit j%32 of word j//32."""
    n, m = bits.shape
    out = np.zeros((n, m // 32), dtype=np.uint64)
    for j in range(m):
        out[:, j // 32] |= bits[:, j].astype(np.uint64) << np.uint64(j % 32)
    return out.astype(np.uint32)


def unpack_bits(words: np.ndarray, m: int) -> np.ndarray:
    w64 = words.astype(np.uint64)
    return np.stack([((w64[:, j // 32] >> np.uint64(j % 32)) & np.uint64(1)).astype(np.int64)
                     for j in range(m)], axis=1) if m else np.zeros((words.shape[0], 0), np.int64)


# ------------------------------------------------------------------------ encoder
@dataclasses.dataclass
class Compressed:
    codes: np.ndarray        # (n, W) uint32, planar
    signs: np.ndarray        # (n, m/32) uint32
    norms: np.ndarray        # (n,) fp32, nu
    rnorms: np.ndarray       # (n,) fp32, ||r||
    # diagnostics, not part of the stored format
    code_idx: np.ndarray = None      # (n, d) codes
    z: np.ndarray = None             # (n, d) sqrt(d) * rotated unit vector
    code_margin: np.ndarray = None   # (n, d) min_k |z - bnd_k|
    t: np.ndarray = None             # (n, m) S r
    nu64: np.ndarray = None
    gamma64: np.ndarray = None


def quantize(x: np.ndarray, codec: Codec) -> Compressed:
    """Encode rows of x (n x d, any float dtype; evaluated in double)."""
    x = np.asarray(x, dtype=np.float64)
    d = codec.d
    nu = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(nu > 0, nu, 1.0)
    u = np.where(nu[:, None] > 0, x / safe[:, None], 0.0)
    y = u @ codec.Pi.T
    z = math.sqrt(d) * y
    return quantize_with(z, y, nu, codec)


def quantize_with(z: np.ndarray, y: np.ndarray, nu: np.ndarray, codec: Codec) -> Compressed:
    d = codec.d
    L = codec.seg_len
    codes = np.empty(z.shape, dtype=np.int64)
    margin = np.empty(z.shape)
    if codec.vq_bits:
        # FibQuant section 2.3: each block (z_2j, z_2j+1) takes its nearest
        # codeword (ties: the lower index); the margin is the block's distance
        # to its Voronoi cell's boundary, the least over the other codewords c_j
        # of the distance to the bisector of c_i1 and c_j,
        # (|z - c_j|^2 - |z - c_i1|^2) / (2 |c_j - c_i1|)
        cb = codec.vq_cb.astype(np.float64)
        blocks = z.reshape(z.shape[0], d // 2, 2)
        d2 = ((blocks[:, :, None, :] - cb[None, None, :, :]) ** 2).sum(axis=3)
        i1 = np.argmin(d2, axis=2)
        d1 = np.take_along_axis(d2, i1[:, :, None], 2)
        sep = np.sqrt(((cb[:, None, :] - cb[None, :, :]) ** 2).sum(axis=2))[i1]
        with np.errstate(divide="ignore", invalid="ignore"):
            bis = np.where(sep > 0, (d2 - d1) / (2.0 * sep), np.inf)
        bis[np.arange(bis.shape[2])[None, None, :] == i1[:, :, None]] = np.inf
        codes[:] = np.repeat(i1, 2, axis=1)
        margin[:] = np.repeat(np.min(bis, axis=2), 2, axis=1)
    for s in range(codec.nseg if not codec.vq_bits else 0):
        zs = z[:, s * L:(s + 1) * L]
        bnd = codec.bnd[s].astype(np.float64)
        codes[:, s * L:(s + 1) * L] = np.sum(zs[:, :, None] >= bnd[None, None, :], axis=2)
        margin[:, s * L:(s + 1) * L] = np.min(np.abs(zs[:, :, None] - bnd[None, None, :]), axis=2)
    r = y - codec.coord_cen(codes) / math.sqrt(d)
    gamma = np.sqrt(np.sum(r * r, axis=1))
    if codec.m > 0:
        t = r @ codec.S.astype(np.float64).T
        signs = pack_bits((t >= 0).astype(np.int64))
    else:
        t = np.zeros((z.shape[0], 0))
        signs = np.zeros((z.shape[0], 0), dtype=np.uint32)
    if codec.residual == "sign":
        # the stored residual scale is the constant mu sqrt(2d/pi) of the
        # format (every estimator then reads mu / sqrt(d) per sign)
        rn = np.full(z.shape[0], np.float32(codec.mu * math.sqrt(2.0 * d / math.pi)), dtype=np.float32)
    else:
        rn = gamma.astype(np.float32) if codec.m > 0 else np.zeros(0, np.float32)
    return Compressed(pack_codes(codes, codec), signs, nu.astype(np.float32), rn, codes, z, margin, t, nu, gamma)


def dequantize(comp: Compressed, codec: Codec, rotated: bool = False, qjl: bool = False) -> np.ndarray:
    """Decoder: codes -> centroids -> inverse rotation -> times the norm.
    ``rotated=True`` stops before the inverse rotation.  ``qjl=True`` adds the
    QJL residual estimate, x~ = nu (c_hat / sqrt(d) + ||r|| sqrt(pi/2) / m S^T s)
    in the rotated space with s = 2 bit - 1: since E[sign(S_j r) S_j] =
    sqrt(2/pi) r / ||r|| for a Gaussian row S_j, it is unbiased for x over S
    (the same correction the score estimator applies to <q, x>)."""
    codes = unpack_codes(comp.codes, codec)
    yhat = codec.coord_cen(codes) / math.sqrt(codec.d)
    if qjl and codec.residual == "sign":
        # TurboESM: the first-order correction mu sign(r_i) per coordinate
        s = 2.0 * unpack_bits(comp.signs, codec.d) - 1.0
        yhat = yhat + codec.mu * s / math.sqrt(codec.d)
    elif qjl and codec.m > 0:
        s = 2.0 * unpack_bits(comp.signs, codec.m) - 1.0
        corr = s @ codec.S.astype(np.float64)
        yhat = yhat + comp.rnorms.astype(np.float64)[:, None] * (math.sqrt(math.pi / 2) / codec.m) * corr
    yhat = yhat * comp.norms.astype(np.float64)[:, None]
    return yhat if rotated else yhat @ codec.Pi


# ---------------------------------------------------------------------- estimator
def estimate_scores(q: np.ndarray, comp: Compressed, codec: Codec,
                    B: int, Hq: int, Hkv: int, T: int) -> np.ndarray:
    """Unscaled logits [B, Hq, T]: for key row (b*Hkv + h_kv)*T + t with
    h_kv = h_q // (Hq/Hkv),
        l = nu * ( <q', c_hat>/sqrt(d) + ||r|| sqrt(pi/2)/m <S q', s> ),
    q' = Pi q, c_hat the centroids (z units), s = 2*bit - 1 (no QJL term if m = 0)."""
    d, m = codec.d, codec.m
    G = Hq // Hkv
    q = np.asarray(q, dtype=np.float64).reshape(B, Hq, d)
    qr = q @ codec.Pi.T
    chat = codec.coord_cen(unpack_codes(comp.codes, codec))
    nu = comp.norms.astype(np.float64)
    if m > 0:
        w = qr @ codec.S.astype(np.float64).T
        s = 2.0 * unpack_bits(comp.signs, m) - 1.0
        gam = comp.rnorms.astype(np.float64)
    out = np.empty((B, Hq, T))
    for b in range(B):
        for h in range(Hq):
            rows = (b * Hkv + h // G) * T + np.arange(T)
            val = chat[rows] @ qr[b, h] / math.sqrt(d)
            if codec.residual == "sign":
                # TurboESM: nu (<q', c_hat> + mu <q', sign(r)>) / sqrt(d)
                val = val + codec.mu / math.sqrt(d) * (s[rows] @ qr[b, h])
            elif m > 0:
                val = val + gam[rows] * math.sqrt(math.pi / 2) / m * (s[rows] @ w[b, h])
            out[b, h] = nu[rows] * val
    return out


def attend(q: np.ndarray, K: Compressed, V: Compressed, kc: Codec, vc: Codec,
           B: int, Hq: int, Hkv: int, T: int, scale: Optional[float] = None) -> np.ndarray:
    """Decode attention [B, Hq, d]: p = softmax(scale * l) over the T keys of
    the query's KV head (scale defaults to 1/sqrt(d)), then
    out = Pi^T sum_t p_t v~_t with the values' own codec, v~ the QJL-corrected
    rotated value when the value codec has a sketch (m > 0) and
    nu c_hat / sqrt(d) otherwise."""
    d = kc.d
    G = Hq // Hkv
    if scale is None or scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    logits = estimate_scores(q, K, kc, B, Hq, Hkv, T) * scale
    vrot = dequantize(V, vc, rotated=True, qjl=True)
    out = np.empty((B, Hq, d))
    for b in range(B):
        for h in range(Hq):
            l = logits[b, h]
            p = np.exp(l - np.max(l))
            p = p / np.sum(p)
            rows = (b * Hkv + h // G) * T + np.arange(T)
            out[b, h] = (p @ vrot[rows]) @ vc.Pi
    return out


# ------------------------------------------------------------------------- search
def search_topk(q: np.ndarray, comp: Compressed, codec: Codec, k: int,
                row_offset: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Top-k rows of the compressed index for each query by the estimator,
    descending, ties to the lower row index.  Returns (idx, score)."""
    q = np.asarray(q, dtype=np.float64)
    nq = q.shape[0]
    n = comp.norms.shape[0]
    qr = q @ codec.Pi.T
    chat = codec.coord_cen(unpack_codes(comp.codes, codec))
    val = qr @ chat.T / math.sqrt(codec.d)
    if codec.m > 0:
        w = qr @ codec.S.astype(np.float64).T
        s = 2.0 * unpack_bits(comp.signs, codec.m) - 1.0
        val = val + (w @ s.T) * (comp.rnorms.astype(np.float64)[None, :] * math.sqrt(math.pi / 2) / codec.m)
    sc = val * comp.norms.astype(np.float64)[None, :]
    return topk_rows(sc, k, row_offset)


def exact_topk(q: np.ndarray, x: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Top-k of the exact inner products <q, x_row> (for recall)."""
    sc = np.asarray(q, np.float64) @ np.asarray(x, np.float64).T
    return topk_rows(sc, k, 0)


def topk_rows(sc: np.ndarray, k: int, row_offset: int) -> Tuple[np.ndarray, np.ndarray]:
    nq, n = sc.shape
    idx = np.empty((nq, k), dtype=np.int64)
    val = np.empty((nq, k))
    ar = np.arange(n)
    for i in range(nq):
        order = np.lexsort((ar, -sc[i]))[:k]
        idx[i] = order + row_offset
        val[i] = sc[i, order]
    return idx, val
