"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a published
test vector or table, an independent construction, a closed form, an
invariant, brute force on tiny inputs, or a Monte-Carlo expectation.  They are
chosen so that a plausible slip in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong scale) fails at least one of them.
"""
import math

import mpmath
import numpy as np
import pytest
from scipy import stats

import oracle as O
import synth
from conftest import golden_path


# ------------------------------------------------------------------ random draws
def test_splitmix64_reference_outputs():
    want = [int(l, 16) for l in open(golden_path("splitmix64_state0.txt")) if l.startswith("0x")]
    assert O.splitmix64(0, 3) == want


def test_rademacher_signs_follow_top_bit():
    outs = O.splitmix64(7, 256)
    D = O.rademacher_signs(7, 256)
    assert set(np.unique(D)) == {-1.0, 1.0}
    # top bit set <=> the integer is at least 2^63
    assert all((D[i] < 0) == (outs[i] >= 2 ** 63) for i in range(256))
    assert abs(np.mean(D)) < 0.2


def test_gaussian_sketch_is_standard_normal():
    S = O.gaussian_sketch(3, 64, 512).astype(np.float64).ravel()
    assert S.dtype == np.float64 and S.size == 64 * 512
    ks = stats.kstest(S, "norm")
    assert ks.pvalue > 1e-3, ks
    assert abs(S.mean()) < 0.02 and abs(S.var() - 1) < 0.02
    # the D stream and the S stream are different streams of the same seed
    assert not np.allclose(O.gaussian_sketch(3, 1, 8), O.gaussian_sketch(4, 1, 8))


def test_sketch_is_row_major_m_by_d():
    # entry (j, i) comes from the output pair 2*(j*d + i), 2*(j*d + i) + 1
    m, d = 3, 8
    S = O.gaussian_sketch(5, m, d)
    outs = O.splitmix64(5 ^ O.S_SEED_XOR, 2 * m * d)
    j, i = 2, 5
    k = j * d + i
    u1 = ((outs[2 * k] >> 11) + 1) / 2.0 ** 53
    u2 = (outs[2 * k + 1] >> 11) / 2.0 ** 53
    # a Box-Muller normal from (u1, u2) has |g| <= sqrt(-2 ln u1)
    assert abs(S[j, i]) <= math.sqrt(-2 * math.log(u1)) * (1 + 1e-6)
    assert np.sign(S[j, i]) == np.sign(math.cos(2 * math.pi * u2))


# --------------------------------------------------------------------- rotation
def _kron_hadamard(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


@pytest.mark.parametrize("n", [2, 8, 64, 128, 512])
def test_hadamard_matches_sylvester_recursion(n):
    assert np.array_equal(O.sylvester_hadamard(n), _kron_hadamard(n))


def test_hadamard_8_literal():
    H8 = O.sylvester_hadamard(8)
    # rows of H_8 in Sylvester order, written out
    lit = ["++++++++", "+-+-+-+-", "++--++--", "+--++--+",
           "++++----", "+-+--+-+", "++----++", "+--+-++-"]
    want = np.array([[1.0 if c == "+" else -1.0 for c in r] for r in lit])
    assert np.array_equal(H8, want)
    assert np.array_equal(H8 @ H8, 8 * np.eye(8))


@pytest.mark.parametrize("d", [8, 64, 128, 1536])
def test_rotation_is_orthogonal(d):
    D = O.rademacher_signs(11, d)
    Pi = O.rotation_matrix(D)
    assert np.abs(Pi @ Pi.T - np.eye(d)).max() < 1e-12
    rng = np.random.default_rng(0)
    x, y = rng.standard_normal((2, d)) * 3
    assert abs(np.linalg.norm(Pi @ x) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)
    assert abs((Pi @ x) @ (Pi @ y) - x @ y) < 1e-12 * np.linalg.norm(x) * np.linalg.norm(y)


def test_rotation_spreads_an_outlier():
    # a single-channel spike is spread evenly over all rotated coordinates
    d = 128
    Pi = O.rotation_matrix(O.rademacher_signs(0, d))
    e = np.zeros(d)
    e[17] = 100.0
    y = Pi @ e
    assert np.allclose(np.abs(y), 100.0 / math.sqrt(d), atol=1e-12)


def test_rope_before_rotation_keeps_scores():
    # TurboESM, "Resumo tecnico" section 2: RoPE first, then Pi; Pi^T Pi = I
    d = 64
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((2, 5, d))
    pos = np.array([0, 1, 17, 400, 4095])
    qr = synth.rope_rotate_half(q, pos, 10000.0)
    kr = synth.rope_rotate_half(k, pos, 10000.0)
    Pi = O.rotation_matrix(O.rademacher_signs(1, d))
    lhs = np.einsum("td,td->t", qr @ Pi.T, kr @ Pi.T)
    rhs = np.einsum("td,td->t", qr, kr)
    assert np.abs(lhs - rhs).max() < 1e-11


def test_rope_rotates_a_plane_by_position_times_frequency():
    # d = 2: one pair rotated by pos * theta^0 = pos radians
    out = O.rope_rotate_half(np.array([[1.0, 0.0], [0.0, 1.0]]), np.array([1, 1]), 10000.0)
    assert np.allclose(out, [[math.cos(1), math.sin(1)], [-math.sin(1), math.cos(1)]], atol=1e-15)
    # d = 4, theta = 100: pairs (0, 2) and (1, 3); frequencies 100^0 = 1 and
    # 100^(-2/4) = 0.1; at position 3 the angles are 3 and 0.3 rad
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    a0, a1 = 3.0, 0.3
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            1 * math.sin(a0) + 3 * math.cos(a0), 2 * math.sin(a1) + 4 * math.cos(a1)]
    assert np.allclose(O.rope_rotate_half(x, np.array([3]), 100.0)[0], want, atol=1e-14)
    # position 0 is the identity
    y = np.random.default_rng(0).standard_normal((3, 64))
    assert np.array_equal(O.rope_rotate_half(y, np.zeros(3), 10000.0), y)


def test_rope_scores_depend_only_on_relative_position():
    # <RoPE(q, a), RoPE(k, b)> depends on a - b only (and norms are kept)
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal((2, 1, 64))
    def dot(a, b):
        return float(O.rope_rotate_half(q, [a], 10000.0)[0] @ O.rope_rotate_half(k, [b], 10000.0)[0])
    assert abs(dot(5, 3) - dot(4002, 4000)) < 1e-10
    assert abs(dot(0, 0) - float(q[0] @ k[0])) < 1e-12
    assert abs(np.linalg.norm(O.rope_rotate_half(q, [777], 10000.0)) - np.linalg.norm(q)) < 1e-12


def test_oracle_rope_agrees_with_the_generator_and_commutes_with_pi():
    # two independent implementations of the same definition agree, and the
    # rotation Pi after RoPE keeps every score (TurboESM, "Resumo tecnico" 2)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((6, 128))
    pos = np.array([0, 1, 2, 100, 4095, 31])
    assert np.abs(O.rope_rotate_half(x, pos, 10000.0) - synth.rope_rotate_half(x, pos, 10000.0)).max() < 1e-12
    Pi = O.rotation_matrix(O.rademacher_signs(2, 128))
    r = O.rope_rotate_half(x, pos, 10000.0)
    assert np.abs((r @ Pi.T) @ (r @ Pi.T).T - r @ r.T).max() < 1e-10


# --------------------------------------------------------------------- codebook
def _golden_max():
    rows = {}
    for line in open(golden_path("max1960_gaussian_lloyd_max.txt")):
        if line.startswith("#") or not line.strip():
            continue
        b, lv, mse = line.split()
        # tolerance: one unit in the last printed digit of each entry (the 1960
        # table's last digit is not always correctly rounded)
        rows[int(b)] = ([(float(v), 10.0 ** -len(v.split(".")[1])) for v in lv.split(",")],
                        float(mse))
    return rows


def _mse(cen, bnd, f, edge):
    from scipy import integrate
    e = np.concatenate([[-edge], bnd, [edge]])
    return sum(integrate.quad(lambda z: (z - cen[k]) ** 2 * f(z), e[k], e[k + 1], epsrel=1e-12)[0]
               for k in range(len(cen)))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_gaussian_limit_matches_max_1960(bits):
    levels, mse = _golden_max()[bits]
    cen, bnd, _ = O.lloyd_max(bits, O.gaussian_density())
    pos = cen[len(cen) // 2:]
    for got, (want, tol) in zip(pos, levels):
        assert abs(got - want) <= tol * 1.0001, (pos, levels)
    f, edge = O.gaussian_density()
    assert abs(_mse(cen, bnd, f, edge) - mse) < 1e-3 * mse


@pytest.mark.parametrize("d", [8, 64, 128, 1536])
def test_lloyd_max_one_bit_closed_form(d):
    # c_1 = E[z | z > 0] = sqrt(d) Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    want = math.sqrt(d) * math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    cen, bnd, _ = O.lloyd_max(1, O.fd_density(d))
    assert abs(cen[1] - want) < 1e-11 and cen[0] == -cen[1] and bnd[0] == 0.0
    pub_c, pub_b = O.published_codebook(1, d)
    assert pub_c[1] == np.float32(want)


@pytest.mark.parametrize("d", [8, 64, 1536])
def test_fd_density_is_the_sphere_marginal(d):
    # sqrt(d) * (first coordinate of a uniform unit vector) has density f_d
    f, edge = O.fd_density(d)
    total = mpmath.quad(lambda z: f(float(z)), [-edge, 0, edge])
    assert abs(total - 1) < 1e-10
    rng = np.random.default_rng(d)
    g = rng.standard_normal((40000, d))
    z = math.sqrt(d) * g[:, 0] / np.linalg.norm(g, axis=1)
    from scipy import integrate
    cdf = np.vectorize(lambda t: integrate.quad(f, -edge, t)[0])
    ks = stats.kstest(z[:4000], cdf)
    assert ks.pvalue > 1e-3, ks
    # the variance of the marginal is exactly 1
    var = mpmath.quad(lambda z: float(z) ** 2 * f(float(z)), [-edge, 0, edge])
    assert abs(var - 1) < 1e-9


@pytest.mark.parametrize("bits,d", [(2, 128), (3, 128), (4, 128), (2, 64), (3, 1536), (3, 8)])
def test_lloyd_max_centroid_and_midpoint_conditions(bits, d):
    cen, bnd, _ = O.lloyd_max(bits, O.fd_density(d))
    f, edge = O.fd_density(d)
    mpmath.mp.dps = 30
    e = [-edge] + list(bnd) + [edge]
    for k in range(len(cen)):
        lo, hi = mpmath.mpf(e[k]), mpmath.mpf(e[k + 1])
        p = mpmath.quad(lambda z: f(float(z)), [lo, hi])
        m1 = mpmath.quad(lambda z: z * f(float(z)), [lo, hi])
        assert abs(cen[k] - float(m1 / p)) < 1e-10, (k, cen[k], float(m1 / p))
    assert np.allclose(bnd, 0.5 * (cen[:-1] + cen[1:]), rtol=0, atol=0)
    assert np.array_equal(cen, -cen[::-1])
    pub_c, pub_b = O.published_codebook(bits, d)
    assert np.array_equal(pub_c, cen.astype(np.float32))
    assert np.array_equal(pub_b, bnd.astype(np.float32))


def test_lloyd_max_is_a_local_minimum():
    bits, d = 3, 64
    cen, bnd, _ = O.lloyd_max(bits, O.fd_density(d))
    f, edge = O.fd_density(d)
    base = _mse(cen, bnd, f, edge)
    for k in range(len(cen)):
        for eps in (1e-3, -1e-3):
            c2 = cen.copy()
            c2[k] += eps
            assert _mse(c2, bnd, f, edge) > base
    for k in range(len(bnd)):
        for eps in (1e-3, -1e-3):
            b2 = bnd.copy()
            b2[k] += eps
            assert _mse(cen, b2, f, edge) > base
    # distortion falls by roughly 4x per bit (6 dB per bit rule) at these rates
    m2 = _mse(*O.lloyd_max(2, O.fd_density(d))[:2], f, edge)
    assert 3.0 < m2 / base < 4.5


# -------------------------------------------------------------------- quantiser
def _codec(d, bits, m, seed=0):
    return O.make_codec(d, bits, m, seed)


@pytest.mark.parametrize("bits", [1, 2])
def test_quantizer_is_nearest_product_codeword_d8(bits):
    d = 8
    c = _codec(d, (bits,), 32)
    rng = np.random.default_rng(bits)
    x = rng.standard_t(3, size=(40, d))
    comp = O.quantize(x, c)
    cen = c.cen[0].astype(np.float64)
    L = len(cen)
    grid = np.array(np.meshgrid(*[np.arange(L)] * d, indexing="ij")).reshape(d, -1).T  # L^d codewords
    words = cen[grid]
    for n in range(x.shape[0]):
        dist = np.sum((words - comp.z[n][None, :]) ** 2, axis=1)
        best = grid[np.argmin(dist)]
        if np.min(comp.code_margin[n]) > 1e-9:
            assert np.array_equal(best, comp.code_idx[n])


def test_quantizer_three_bits_nearest_centroid_per_coordinate():
    d = 8
    c = _codec(d, (3,), 32)
    x = np.random.default_rng(9).standard_normal((200, d))
    comp = O.quantize(x, c)
    cen = c.cen[0].astype(np.float64)
    near = np.argmin(np.abs(comp.z[:, :, None] - cen[None, None, :]), axis=2)
    ok = comp.code_margin > 1e-9
    assert np.array_equal(near[ok], comp.code_idx[ok])


def test_code_rule_boundary_goes_to_upper_cell():
    d = 8
    c = _codec(d, (2,), 32)
    bnd = c.bnd[0].astype(np.float64)
    z = np.array([[bnd[0], bnd[1], bnd[2], np.nextafter(bnd[2], -np.inf), -10.0, 10.0, 0.0, bnd[0] - 1e-300]])
    comp = O.quantize_with(z, z / math.sqrt(d), np.ones(1), c)
    assert list(comp.code_idx[0]) == [1, 2, 3, 2, 0, 3, 2, 0 if bnd[0] - 1e-300 < bnd[0] else 1]


def test_planar_packing_positions():
    # segment s, plane p, word w, bit t  <->  bit p of the code of coordinate s*L + 32w + t
    c = O.make_codec(128, (2, 3), 64, 0)   # W = 2*2 + 3*2 = 10 words
    assert c.words == 10
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 64 + 32 + 5] = 0b100     # segment 1, word 1, bit 5, plane 2
    codes[0, 3] = 0b10                # segment 0, word 0, bit 3, plane 1
    w = O.pack_codes(codes, c)[0]
    want = np.zeros(10, dtype=np.uint32)
    want[1 * 2 + 0] = 1 << 3                  # seg 0: planes 0,1 x words 0,1 -> plane 1 word 0 = index 2
    want[4 + 2 * 2 + 1] = 1 << 5              # seg 1 starts at 4; plane 2 word 1 -> 4 + 4 + 1
    assert np.array_equal(w, want)
    rnd = np.random.default_rng(0).integers(0, 4, size=(7, 128))
    rnd[:, 64:] = np.random.default_rng(1).integers(0, 8, size=(7, 64))
    assert np.array_equal(O.unpack_codes(O.pack_codes(rnd, c), c), rnd)
    bits = np.random.default_rng(2).integers(0, 2, size=(5, 64))
    assert np.array_equal(O.unpack_bits(O.pack_bits(bits), 64), bits)
    one = np.zeros((1, 64), dtype=np.int64)
    one[0, 37] = 1
    assert list(O.pack_bits(one)[0]) == [0, 1 << 5]


def test_sketch_index_convention():
    # t_j = sum_i S[j, i] r_i : an S with one non-zero picks one residual coordinate
    d, m = 8, 32
    S = np.zeros((m, d), dtype=np.float32)
    S[4, 6] = 1.0
    S[9, 2] = -1.0
    c = O.make_codec(d, (1,), m, 0, S=S)
    x = np.random.default_rng(4).standard_normal((3, d))
    comp = O.quantize(x, c)
    r = comp.z / math.sqrt(d) - c.coord_cen(comp.code_idx) / math.sqrt(d)
    assert np.allclose(comp.t[:, 4], r[:, 6], atol=1e-15)
    assert np.allclose(comp.t[:, 9], -r[:, 2], atol=1e-15)
    assert np.allclose(comp.t[:, 0], 0)


def test_zero_vector_and_zero_residual():
    d, m = 64, 64
    c = _codec(d, (3,), m, seed=2)
    # a rotated point exactly on the reconstruction grid has zero residual, so
    # the estimate is nu <Pi q, y_hat> = <q, nu Pi^T y_hat> exactly
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 8, size=(4, d))
    z = c.coord_cen(codes)
    nu = np.array([2.5, 1.0, 0.125, 3.0])
    comp = O.quantize_with(z, z / math.sqrt(d), nu, c)
    assert np.array_equal(comp.code_idx, codes)
    assert comp.gamma64.max() == 0.0 and np.all(comp.t == 0)
    assert np.all(O.unpack_bits(comp.signs, m) == 1)          # sign(0) = +1
    x = nu[:, None] * (z / math.sqrt(d)) @ c.Pi
    q = rng.standard_normal((1, 4, d))
    l = O.estimate_scores(q, comp, c, 1, 4, 4, 1)
    exact = np.einsum("hd,hd->h", q[0], x)
    assert np.allclose(l[0, :, 0], exact, rtol=1e-12, atol=1e-12)
    # nu = 0: all logits are zero, codes are those of z = 0
    zc = O.quantize(np.zeros((1, d)), c)
    assert zc.norms[0] == 0 and np.all(zc.code_idx == np.sum(c.bnd[0] <= 0))
    assert np.all(O.estimate_scores(q[:, :1], zc, c, 1, 1, 1, 1) == 0)


def test_decoder_error_matches_codebook_distortion():
    # E ||x - x_hat||^2 / ||x||^2 equals the per-coordinate Lloyd-Max MSE
    d, bits = 128, 3
    c = _codec(d, (bits,), 0)
    x = np.random.default_rng(8).standard_t(3, size=(3000, d))
    comp = O.quantize(x, c)
    xh = O.dequantize(comp, c)
    rel = np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1)
    f, edge = O.fd_density(d)
    cen, bnd, _ = O.lloyd_max(bits, O.fd_density(d))
    want = _mse(cen, bnd, f, edge)
    assert abs(rel.mean() - want) < 0.05 * want, (rel.mean(), want)


# -------------------------------------------------------------------- estimator
def test_qjl_estimator_is_unbiased_monte_carlo():
    # QJL (TurboQuant news page; explainer page section "Por dentro"): over the
    # Gaussian sketch, E[l] = <q, x> given the codes
    d, m, N = 16, 32, 20000
    rng = np.random.default_rng(21)
    x = rng.standard_t(3, size=(1, d))
    q = rng.standard_normal((1, 1, d))
    c0 = O.make_codec(d, (2,), m, 0, S=np.zeros((m, d)))
    comp0 = O.quantize(x, c0)
    exact = float(q[0, 0] @ x[0])
    est = np.empty(N)
    qr = (q[0, 0] @ c0.Pi.T)
    r = comp0.z[0] / math.sqrt(d) - c0.coord_cen(comp0.code_idx)[0] / math.sqrt(d)
    mse_part = qr @ c0.coord_cen(comp0.code_idx)[0] / math.sqrt(d)
    for k in range(N):
        S = rng.standard_normal((m, d))
        c = O.make_codec(d, (2,), m, 0, D=c0.D, S=S)
        comp = O.quantize(x, c)
        est[k] = O.estimate_scores(q, comp, c, 1, 1, 1, 1)[0, 0, 0]
    se = est.std() / math.sqrt(N)
    assert abs(est.mean() - exact) < 4 * se + 1e-6 * abs(exact), (est.mean(), exact, se)
    # the single-draw spread is bounded by nu * ||r|| * ||q|| * sqrt(pi / (2 m))
    nu = np.linalg.norm(x)
    assert est.std() <= nu * np.linalg.norm(r) * np.linalg.norm(q) * math.sqrt(math.pi / (2 * m)) * 1.05
    # the MSE-only part alone misses the residual term
    assert abs(nu * mse_part - exact) > 10 * se


def test_mse_only_estimator_is_biased_and_qjl_is_not():
    # one-bit codes, averaged over rotations: E<q', y_hat> / <q, u> -> c_1 sqrt(2/pi) ~ 2/pi
    d, N = 64, 3000
    rng = np.random.default_rng(33)
    x = rng.standard_normal((1, d))
    q = (x + 0.5 * rng.standard_normal((1, d)))[None]
    exact = float(q[0, 0] @ x[0])
    mse_only, full = np.empty(N), np.empty(N)
    for k in range(N):
        D = rng.choice([-1.0, 1.0], size=d)
        c = O.make_codec(d, (1,), 64, 0, D=D, S=rng.standard_normal((64, d)))
        comp = O.quantize(x, c)
        full[k] = O.estimate_scores(q, comp, c, 1, 1, 1, 1)[0, 0, 0]
        cm = O.make_codec(d, (1,), 0, 0, D=D)
        mse_only[k] = O.estimate_scores(q, O.quantize(x, cm), cm, 1, 1, 1, 1)[0, 0, 0]
    ratio = mse_only.mean() / exact
    c1 = O.published_codebook(1, d)[0][1]
    assert abs(ratio - c1 * math.sqrt(2 / math.pi)) < 0.03, ratio
    assert abs(full.mean() - exact) < 4 * full.std() / math.sqrt(N)


def test_gqa_rows_and_accuracy_at_four_bits():
    # with 4-bit codes and m = 128 each logit is close to its own key's inner product
    B, Hq, Hkv, T, d = 2, 4, 2, 16, 128
    c = _codec(d, (4,), 128, seed=3)
    x = synth.heavy_rows(5, B * Hkv * T, d).to(dtype=__import__("torch").float64).numpy()
    q = np.random.default_rng(6).standard_normal((B, Hq, d))
    comp = O.quantize(x, c)
    l = O.estimate_scores(q, comp, c, B, Hq, Hkv, T)
    for b in range(B):
        for h in range(Hq):
            rows = (b * Hkv + h // (Hq // Hkv)) * T + np.arange(T)
            exact = x[rows] @ q[b, h]
            scale = np.linalg.norm(x[rows], axis=1) * np.linalg.norm(q[b, h])
            assert np.all(np.abs(l[b, h] - exact) < 0.08 * scale)


# -------------------------------------------------------------------- attention
def test_attend_special_cases():
    d = 64
    kc = _codec(d, (2,), 64, seed=1)
    vc = _codec(d, (4,), 0, seed=1)
    rng = np.random.default_rng(2)
    # T = 1: the output is the single dequantised value
    k1, v1 = rng.standard_normal((2, 1, d))
    q = rng.standard_normal((1, 2, d))
    K, V = O.quantize(k1, kc), O.quantize(v1, vc)
    out = O.attend(q, K, V, kc, vc, 1, 2, 1, 1)
    vhat = O.dequantize(V, vc)[0]
    assert np.allclose(out[0, 0], vhat, atol=1e-12) and np.allclose(out[0, 1], vhat, atol=1e-12)
    # all logits equal (q = 0): the output is the mean of the dequantised values
    T = 9
    k, v = rng.standard_normal((2, T, d))
    K, V = O.quantize(k, kc), O.quantize(v, vc)
    out = O.attend(np.zeros((1, 1, d)), K, V, kc, vc, 1, 1, 1, T)
    assert np.allclose(out[0, 0], O.dequantize(V, vc).mean(axis=0), atol=1e-12)
    # a dominant logit selects its value
    q = 50 * k[3:4][None] / np.linalg.norm(k[3])
    out = O.attend(q, K, V, kc, vc, 1, 1, 1, T, scale=1.0)
    assert np.allclose(out[0, 0], O.dequantize(V, vc)[3], atol=1e-6)




def _test_rotation(codec):
    """Pi built here from a Sylvester matrix and the codec's D."""
    d = codec.d
    return _kron_hadamard(d) * codec.D[None, :] / math.sqrt(d)


def test_attend_softmax_weights_worked_by_hand():
    # Every vector is x = nu Pi^T c_hat / ||c_hat|| for chosen codes (c_hat
    # their centroids), so its norm is nu and its codes are the chosen ones
    # (checked).  With m = 0 the key estimate is nu <Pi q, c_hat> / sqrt(d)
    # and the rotated dequantised value nu c_hat / sqrt(d): both follow from
    # the chosen codes by plain dot products.  q is chosen so that the logits
    # are (0, sqrt(d) ln 2, 0): softmax weights (1/4, 1/2, 1/4) at the default
    # temperature 1/sqrt(d), and (1/6, 4/6, 1/6) at an explicit scale 2/sqrt(d).
    d = 64
    kc = _codec(d, (2,), 0, seed=3)
    vc = _codec(d, (3,), 0, seed=5)
    Pk, Pv = _test_rotation(kc), _test_rotation(vc)
    rng = np.random.default_rng(8)
    # codes of Gaussian draws, so that ||c_hat||^2 / d is near 1 and the
    # normalised centroids stay inside their cells
    kcodes = [np.searchsorted(kc.bnd[0], rng.standard_normal(d), side="right") for _ in range(2)]
    vcodes = [np.searchsorted(vc.bnd[0], rng.standard_normal(d), side="right") for _ in range(3)]
    knu, vnu = (1.75, 0.625), (0.875, 2.0, 1.25)      # exact in fp32
    kchat = [kc.cen[0].astype(np.float64)[c] for c in kcodes]
    vchat = [vc.cen[0].astype(np.float64)[c] for c in vcodes]
    keys = np.stack([knu[t] * (kchat[t] / np.linalg.norm(kchat[t])) @ Pk for t in (0, 1, 0)])
    vals = np.stack([vnu[t] * (vchat[t] / np.linalg.norm(vchat[t])) @ Pv for t in range(3)])
    K, V = O.quantize(keys, kc), O.quantize(vals, vc)
    assert np.array_equal(K.code_idx, np.stack([kcodes[0], kcodes[1], kcodes[0]]))
    assert np.array_equal(V.code_idx, np.stack(vcodes))
    assert list(K.norms) == [1.75, 0.625, 1.75] and list(V.norms) == [0.875, 2.0, 1.25]
    # rotated query q' in the span of the two key centroid vectors
    a0, a1 = (knu[t] * kchat[t] / math.sqrt(d) for t in (0, 1))
    G = np.array([[a0 @ a0, a0 @ a1], [a1 @ a0, a1 @ a1]])
    c0, c1 = np.linalg.solve(G, [0.0, math.sqrt(d) * math.log(2.0)])
    qrot = c0 * a0 + c1 * a1
    q = (qrot @ Pk)[None, None]                        # q = Pi^T q'
    vrot = [vnu[t] * vchat[t] / math.sqrt(d) for t in range(3)]
    for scale, w in ((None, (0.25, 0.5, 0.25)), (2.0 / math.sqrt(d), (1 / 6, 4 / 6, 1 / 6))):
        out = O.attend(q, K, V, kc, vc, 1, 1, 1, 3, scale=scale)[0, 0]
        want = (w[0] * vrot[0] + w[1] * vrot[1] + w[2] * vrot[2]) @ Pv
        assert np.abs(out - want).max() < 1e-12 * np.abs(want).max(), (scale, np.abs(out - want).max())
    # a wrong temperature (1 instead of 1/sqrt(d)) moves the output far away
    out1 = O.attend(q, K, V, kc, vc, 1, 1, 1, 3, scale=1.0)[0, 0]
    want = (0.25 * vrot[0] + 0.5 * vrot[1] + 0.25 * vrot[2]) @ Pv
    assert np.abs(out1 - want).max() > 0.1 * np.abs(want).max()

def test_qjl_corrected_values_are_unbiased_monte_carlo():
    # Given the codes (fixed D), x~ = nu (c_hat/sqrt(d) + gamma sqrt(pi/2)/m
    # S^T s) averages to x over independent Gaussian S; the MSE-only
    # reconstruction does not.  Each S draw is a fresh seed of the generator.
    d, m, N = 64, 32, 3000
    rng = np.random.default_rng(12)
    x = rng.standard_normal((1, d)) * 2.0
    D = O.rademacher_signs(3, d)
    draws = []
    for k in range(N):
        c = O.make_codec(d, (2,), m, seed=1000 + k, D=D)
        draws.append(O.dequantize(O.quantize(x, c), c, qjl=True)[0])
    draws = np.array(draws)
    c0 = O.make_codec(d, (2,), m, seed=0, D=D)
    mse_only = O.dequantize(O.quantize(x, c0), c0)[0]
    sem = draws.std(axis=0) / math.sqrt(N)
    assert np.all(np.abs(draws.mean(axis=0) - x[0]) < 4.5 * sem + 1e-12)
    # the MSE-only reconstruction is off by far more than the Monte-Carlo error
    assert np.linalg.norm(mse_only - x[0]) > 20 * np.linalg.norm(sem)


def test_qjl_corrected_values_special_cases():
    d = 64
    rng = np.random.default_rng(13)
    c = _codec(d, (3,), 64, seed=2)
    x = rng.standard_normal((5, d))
    comp = O.quantize(x, c)
    # without a sketch the correction is absent
    c0 = _codec(d, (3,), 0, seed=2)
    comp0 = O.quantize(x, c0)
    assert np.array_equal(O.dequantize(comp0, c0, qjl=True), O.dequantize(comp0, c0))
    # a residual of norm zero adds nothing (gamma = 0)
    comp.rnorms[:] = 0.0
    assert np.allclose(O.dequantize(comp, c, qjl=True), O.dequantize(comp, c), atol=1e-15)
    # T = 1 attention returns the corrected value itself
    comp = O.quantize(x[:1], c)
    kc = _codec(d, (2,), 64, seed=4)
    K = O.quantize(rng.standard_normal((1, d)), kc)
    out = O.attend(rng.standard_normal((1, 1, d)), K, comp, kc, c, 1, 1, 1, 1)
    assert np.allclose(out[0, 0], O.dequantize(comp, c, qjl=True)[0], atol=1e-12)


def _sphere_marginal_samples(d, n, seed):
    """z = sqrt(d) u_1 for u uniform on the sphere S^{d-1} (u = g / ||g||)."""
    rng = np.random.default_rng(seed)
    out = np.empty(n)
    for i in range(0, n, 4096):
        g = rng.standard_normal((min(4096, n - i), d))
        out[i:i + g.shape[0]] = math.sqrt(d) * g[:, 0] / np.linalg.norm(g, axis=1)
    return out


@pytest.mark.parametrize("bits,d", [(2, 64), (3, 128)])
def test_residual_mean_magnitude_monte_carlo(bits, d):
    # mu = E|z - Q(z)| under the sphere marginal, and the first-order
    # correction by mu sign(r) lowers the squared error by exactly mu^2:
    # E (r - mu sign r)^2 = E r^2 - 2 mu E|r| + mu^2 = D - mu^2
    c = O.make_codec(d, (bits,), d, 0, residual="sign")
    z = _sphere_marginal_samples(d, 200_000, bits + d)
    cen, bnd = c.cen[0].astype(np.float64), c.bnd[0].astype(np.float64)
    r = z - cen[np.searchsorted(bnd, z, side="right")]
    a = np.abs(r)
    assert abs(a.mean() - c.mu) < 4 * a.std() / math.sqrt(z.size), (a.mean(), c.mu)
    e = (r - c.mu * np.sign(r)) ** 2
    want = np.mean(r * r) - c.mu ** 2
    assert abs(e.mean() - want) < 4 * e.std() / math.sqrt(z.size) + 1e-3 * want


def test_residual_mean_magnitude_gaussian_limit():
    # for large d the sphere marginal tends to N(0, 1) and the codebook to
    # Max's table (fixture), so mu tends to E|Z - Q_Max(Z)|
    rows = _golden_max()
    levels = [v for v, _ in rows[3][0]]
    cen = np.array(sorted([-v for v in levels] + levels))
    bnd = 0.5 * (cen[:-1] + cen[1:])
    phi = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    from scipy import integrate
    e = np.concatenate([[-np.inf], bnd, [np.inf]])
    mu_g = 0.0
    for k, ck in enumerate(cen):
        mu_g += integrate.quad(lambda z: abs(z - ck) * phi(z), e[k], ck)[0]
        mu_g += integrate.quad(lambda z: abs(z - ck) * phi(z), ck, e[k + 1])[0]
    c = O.make_codec(1536, (3,), 1536, 0, residual="sign")
    assert abs(c.mu - mu_g) < 3e-3, (c.mu, mu_g)


def test_sign_residual_estimator_and_format():
    # the estimator reads nu (<q', c_hat> + mu <q', sign(r)>) / sqrt(d): its
    # error is smaller than the MSE-only one on average, and the stored scale
    # is the constant mu sqrt(2d/pi)
    d = 128
    c = O.make_codec(d, (3,), d, 1, residual="sign")
    c0 = O.make_codec(d, (3,), 0, 1)
    rng = np.random.default_rng(21)
    x = rng.standard_normal((400, d))
    q = rng.standard_normal((1, 1, d))
    comp, comp0 = O.quantize(x, c), O.quantize(x, c0)
    assert np.all(comp.rnorms == np.float32(c.mu * math.sqrt(2 * d / math.pi)))
    exact = x @ q[0, 0]
    est = O.estimate_scores(q, comp, c, 1, 1, 1, 400)[0, 0]
    est0 = O.estimate_scores(q, comp0, c0, 1, 1, 1, 400)[0, 0]
    assert np.mean((est - exact) ** 2) < 0.8 * np.mean((est0 - exact) ** 2)
    # and the corrected reconstruction is closer to x than the MSE-only one
    err = np.linalg.norm(O.dequantize(comp, c, qjl=True) - x, axis=1)
    err0 = np.linalg.norm(O.dequantize(comp0, c0) - x, axis=1)
    assert np.mean(err ** 2) < np.mean(err0 ** 2)


def test_haar_rotation_is_orthogonal_and_haar():
    # orthogonal to rounding; and Haar: for Pi uniform on O(d) the first column
    # is uniform on the sphere, so sqrt(d) Pi_00 follows f_d (KS over seeds),
    # and distinct entries are uncorrelated
    d = 16
    Pi = O.haar_rotation(3, 64)
    assert np.abs(Pi @ Pi.T - np.eye(64)).max() < 1e-12
    vals, prods = [], []
    for sd in range(300):
        P = O.haar_rotation(sd, d)
        vals.append(math.sqrt(d) * P[0, 0])
        prods.append(P[0, 0] * P[1, 1])
    f, edge = O.fd_density(d)
    from scipy import integrate
    cdf = lambda z: integrate.quad(f, -edge, z)[0]
    ks = stats.kstest(vals, np.vectorize(cdf))
    assert ks.pvalue > 1e-3, ks
    assert abs(np.mean(prods)) < 4 * np.std(prods) / math.sqrt(len(prods))
    # the QR convention: the codec's Pi maps G to an upper-triangular R with
    # a positive diagonal, i.e. Pi^T G = R
    outs = O.splitmix64(3 ^ O.HAAR_SEED_XOR, 2 * 64 * 64)
    G = np.array([math.sqrt(-2 * math.log(((outs[2 * k] >> 11) + 1) * 2.0 ** -53))
                  * math.cos(2 * math.pi * (outs[2 * k + 1] >> 11) * 2.0 ** -53) for k in range(64 * 64)]).reshape(64, 64)
    R = Pi.T @ G
    assert np.abs(np.tril(R, -1)).max() < 1e-10 and np.all(np.diag(R) > 0)


def test_haar_codec_quantizes_in_its_rotation():
    # with a Haar codec, the codes are those of z = sqrt(d) Pi x / ||x|| and
    # the estimator keeps inner products (QJL Monte Carlo at one S draw is in
    # the generic tests; here: exact reconstruction of an on-grid vector)
    d = 64
    c = O.make_codec(d, (3,), 0, 5, rotation="haar")
    rng = np.random.default_rng(2)
    codes = np.searchsorted(c.bnd[0], rng.standard_normal(d), side="right")
    chat = c.cen[0].astype(np.float64)[codes]
    x = 1.5 * (chat / np.linalg.norm(chat)) @ c.haar          # Pi^T y as a row
    comp = O.quantize(x[None], c)
    assert np.array_equal(comp.code_idx[0], codes)
    assert np.allclose(O.dequantize(comp, c)[0], 1.5 * (chat / math.sqrt(d)) @ c.haar, atol=1e-12)


# ----------------------------------------------------------------------- top-k
def test_topk_order_and_ties():
    sc = np.array([[0.5, 2.0, 2.0, -1.0, 2.0, 0.7]])
    idx, val = O.topk_rows(sc, 4, 100)
    assert list(idx[0]) == [101, 102, 104, 105] and list(val[0]) == [2.0, 2.0, 2.0, 0.7]
    rng = np.random.default_rng(1)
    sc = rng.integers(0, 20, size=(3, 200)).astype(float)
    idx, _ = O.topk_rows(sc, 10, 0)
    for i in range(3):
        want = sorted(range(200), key=lambda j: (-sc[i, j], j))[:10]
        assert list(idx[i]) == want


@pytest.mark.parametrize("bits,d", [(1, 128), (2, 128), (3, 128), (4, 128), (2, 64), (3, 1536)])
def test_plane_identity_of_symmetric_codebooks(bits, d):
    # With s_k = 2 bit_k - 1, every function of the code is a multilinear
    # polynomial in the s_k (Walsh expansion); a codebook with
    # cen[c] = -cen[2^b - 1 - c] has only odd-degree terms, and the product of
    # an odd set of s_k equals 2 * xor(bits) - 1.  Checked exhaustively.
    cen = O.published_codebook(bits, d)[0].astype(np.float64)
    L = 1 << bits
    sgn = np.array([[1.0 if (c >> k) & 1 else -1.0 for k in range(bits)] for c in range(L)])
    coef = {}
    for S in range(1, L):
        prod = np.prod(np.where([(S >> k) & 1 for k in range(bits)], sgn, 1.0), axis=1)
        coef[S] = float(cen @ prod) / L
    assert abs(float(cen.sum()) / L) == 0.0
    for S, a in coef.items():
        if bin(S).count("1") % 2 == 0:
            assert a == 0.0, (S, a)
    for c in range(L):
        rec = 0.0
        for S, a in coef.items():
            if bin(S).count("1") % 2 == 1:
                par = bin(c & S).count("1") & 1
                rec += a * (2.0 * par - 1.0 if bin(S).count("1") % 2 else 1.0)
        assert abs(rec - cen[c]) < 1e-12 * (1 + abs(cen[c]))



@pytest.mark.parametrize("m", [64, 0])
def test_search_scores_are_the_estimator(m):
    # The search ranks the index rows by the same estimator as tq_scores: each
    # query against all n rows is one decode head (B = Hq = Hkv = 1, T = n).
    # With k = n the search returns every row, so its scores can be compared
    # row by row with estimate_scores, and its order with a plain sort.
    d, n, nq = 64, 257, 4
    codec = _codec(d, (3,), m, seed=4)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((n, d)) * rng.uniform(0.1, 3.0, (n, 1))
    x[200] = x[17]                          # two rows with equal scores
    q = rng.standard_normal((nq, d))
    comp = O.quantize(x, codec)
    idx, score = O.search_topk(q, comp, codec, n, row_offset=5)
    for i in range(nq):
        full = O.estimate_scores(q[i][None, None], comp, codec, 1, 1, 1, n)[0, 0]
        rows = idx[i] - 5
        assert sorted(rows.tolist()) == list(range(n))
        assert np.all(np.abs(score[i] - full[rows]) <= 1e-12 * np.abs(full).max())
        want = sorted(range(n), key=lambda r: (-full[r], r))
        assert rows.tolist() == want
        assert rows.tolist().index(17) < rows.tolist().index(200)
    # a smaller k is the prefix of the full order
    idx3, score3 = O.search_topk(q, comp, codec, 3)
    assert np.array_equal(idx3, idx[:, :3] - 5) and np.array_equal(score3, score[:, :3])


# ------------------------------------------------------------- FibQuant, k = 2
def _block_radius_cdf(d):
    """CDF of |(z_1, z_2)|^2 for z = sqrt(d) u, u uniform on S^{d-1}, by
    quadrature of the 2-D marginal (1 - rho^2/d)^((d-4)/2) times the ring
    length 2 pi rho (normalised numerically, not by a closed form)."""
    from scipy import integrate
    g = lambda rho: rho * (1.0 - rho * rho / d) ** ((d - 4) / 2.0)
    tot = integrate.quad(g, 0.0, math.sqrt(d), epsrel=1e-12)[0]
    return lambda s: integrate.quad(g, 0.0, math.sqrt(min(max(s, 0.0), d)), epsrel=1e-12)[0] / tot


@pytest.mark.parametrize("d", [16, 128])
def test_fibquant_source_points_follow_the_block_law(d):
    # the quasi-Monte-Carlo stand-in for the block source: its squared radii
    # match sampled blocks of uniform unit vectors (two-sample KS) and the
    # quadrature CDF of the 2-D marginal, and its moments are E|z|^2 = 2 and
    # E|z|^4 = 8d / (d + 2) (z_1^2 + z_2^2 = d Beta(1, (d-2)/2))
    pts = O.fibquant_source_points(d, 16384)
    r2 = (pts ** 2).sum(axis=1)
    assert abs(r2.mean() - 2.0) < 1e-3
    assert abs((r2 ** 2).mean() - 8.0 * d / (d + 2)) < 2e-3 * 8
    rng = np.random.default_rng(d)
    g = rng.standard_normal((20000, d))
    u = g / np.linalg.norm(g, axis=1, keepdims=True)
    mc = d * (u[:, 0] ** 2 + u[:, 1] ** 2)
    assert stats.ks_2samp(r2, mc).pvalue > 1e-3
    cdf = _block_radius_cdf(d)
    for qv in (0.1, 0.5, 0.9, 0.99):
        s = float(np.quantile(r2, qv))
        assert abs(cdf(s) - qv) < 2e-4, (qv, cdf(s))
    # the angles advance by the golden angle 2 pi (1 - 1/phi)
    ang = np.arctan2(pts[:, 1], pts[:, 0])
    step = np.mod(np.diff(ang), 2 * math.pi)
    phi = (1 + math.sqrt(5)) / 2
    assert np.allclose(step, 2 * math.pi * (1 - 1 / phi), atol=1e-9)


@pytest.mark.parametrize("d,N", [(64, 16), (128, 32)])
def test_fibquant_spiral_radii_are_bennett_gersho(d, N):
    # section 2.2: the point density of the initial spiral follows f^(k/(k+2))
    # = f^(1/2) of the block law; the fraction of the N points inside radius
    # r_n must be the quadrature of that density, (n + 1/2) / N
    from scipy import integrate
    lam = lambda rho: rho * (1.0 - rho * rho / d) ** ((d - 4) / 4.0)
    tot = integrate.quad(lam, 0.0, math.sqrt(d), epsrel=1e-12)[0]
    cb = O.fibquant_init(N, d)
    r = np.linalg.norm(cb, axis=1)
    assert np.all(np.diff(r) > 0)
    for n in range(N):
        frac = integrate.quad(lam, 0.0, r[n], epsrel=1e-12)[0] / tot
        assert abs(frac - (n + 0.5) / N) < 1e-9, (n, frac)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_fibquant_two_codewords_are_antipodal_scalar_centroids(d):
    # N = 2 on a rotationally symmetric source: the optimum splits the plane by
    # a line through 0 and puts each codeword at its half-plane's mean, i.e.
    # at distance E[z_1 | z_1 > 0] = the 1-bit Lloyd-Max centroid (closed form)
    cb = O.fibquant_codebook(1, d).astype(np.float64)
    want = math.sqrt(d) * math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    assert np.allclose(np.linalg.norm(cb, axis=1), want, rtol=3e-3), (np.linalg.norm(cb, axis=1), want)
    assert np.linalg.norm(cb[0] + cb[1]) < 3e-3


def test_fibquant_lloyd_descends_to_a_fixed_point():
    # Lloyd never increases the distortion, and the result is (nearly) the
    # mean of its own cells over the source points
    d, vb = 64, 4
    pts = O.fibquant_source_points(d, 16384)
    seq = [O.fibquant_distortion(pts, O.fibquant_codebook.__wrapped__(vb, d, iters=it, restarts=1).astype(np.float64))
           for it in (0, 1, 2, 5, 10, 40)]
    assert all(b <= a * (1 + 1e-6) for a, b in zip(seq, seq[1:])), seq
    assert seq[-1] < 0.97 * seq[0]
    cb = O.fibquant_codebook(vb, d).astype(np.float64)
    d2 = ((pts[:, None, :] - cb[None, :, :]) ** 2).sum(axis=2)
    own = d2.argmin(axis=1)
    for n in range(len(cb)):
        cell = pts[own == n]
        assert len(cell) > 0
        assert np.linalg.norm(cell.mean(axis=0) - cb[n]) < 0.02, n


@pytest.mark.parametrize("b", [2, 3])
def test_fibquant_beats_scalar_lloyd_max_at_integer_rates(b):
    # section 3.2 / 4: at matched rate the k = 2 code has strictly lower MSE
    # than the scalar Lloyd-Max table (integrated exactly under f_d)
    d = 128
    f, edge = O.fd_density(d)
    cen, bnd, _ = O.lloyd_max(b, O.fd_density(d))
    scalar = _mse(cen, bnd, f, edge)
    pts = O.fibquant_source_points(d, 16384)
    vq = O.fibquant_distortion(pts, O.fibquant_codebook(2 * b, d).astype(np.float64)) / 2
    assert vq < 0.97 * scalar, (vq, scalar)
    # and the fractional rate b + 1/2 lies between the neighbouring integer rates
    half = O.fibquant_distortion(pts, O.fibquant_codebook(2 * b + 1, d).astype(np.float64)) / 2
    assert vq * 0.4 < half < vq * 0.75


def test_fibquant_packing_positions():
    # block 32w + t's code bit p sits at bit t of word p * pw + w
    d = 64
    c = O.make_codec(d, (1,), 0, 0, vq_bits=3)
    blk = np.arange(32) % 8
    codes = np.repeat(blk, 2)[None]
    w = O.pack_codes(codes, c)
    assert w.shape == (1, 3) and c.words == 3
    assert [int(v) for v in w[0]] == [0xAAAAAAAA, 0xCCCCCCCC, 0xF0F0F0F0]
    assert np.array_equal(O.unpack_codes(w, c), codes)


def test_fibquant_encoder_is_the_nearest_codeword():
    # brute force on small rows: every block's code is its nearest codeword;
    # moving the block by 0.999 of its margin in any direction keeps the code,
    # moving it just past the margin towards the nearest bisector changes it
    d = 16
    c = O.make_codec(d, (1,), 0, 0, vq_bits=4)
    cb = c.vq_cb.astype(np.float64)
    x = np.random.default_rng(3).standard_t(3, size=(20, d))
    comp = O.quantize(x, c)
    rng = np.random.default_rng(4)
    for i in range(x.shape[0]):
        for j in range(d // 2):
            zb = comp.z[i, 2 * j:2 * j + 2]
            dist = [float(np.sum((zb - cw) ** 2)) for cw in cb]
            n = comp.code_idx[i, 2 * j]
            assert comp.code_idx[i, 2 * j + 1] == n and dist[n] == min(dist)
            mg = comp.code_margin[i, 2 * j]
            for _ in range(16):
                a = rng.uniform(0, 2 * math.pi)
                zp = zb + 0.999 * mg * np.array([math.cos(a), math.sin(a)])
                assert int(np.argmin(((zp - cb) ** 2).sum(axis=1))) == n
            # the nearest bisector: step towards each other codeword's cell
            moved = False
            for k in range(len(cb)):
                if k == n:
                    continue
                e = (cb[k] - cb[n]) / np.linalg.norm(cb[k] - cb[n])
                zp = zb + 1.001 * mg * e
                moved |= int(np.argmin(((zp - cb) ** 2).sum(axis=1))) != n
            assert moved


def test_fibquant_decoder_error_matches_design_distortion():
    # E ||x - x_hat||^2 / ||x||^2 = (per-block distortion) / 2 per coordinate
    d = 64
    c = O.make_codec(d, (1,), 0, 0, vq_bits=5)
    x = np.random.default_rng(9).standard_t(3, size=(3000, d))
    comp = O.quantize(x, c)
    rel = np.sum((x - O.dequantize(comp, c)) ** 2, axis=1) / np.sum(x * x, axis=1)
    want = O.fibquant_distortion(O.fibquant_source_points(d, 16384), c.vq_cb.astype(np.float64)) / 2
    assert abs(rel.mean() - want) < 0.05 * want, (rel.mean(), want)


def test_fibquant_qjl_estimator_is_unbiased_monte_carlo():
    # the QJL stage corrects whatever the first stage leaves: over S, the
    # estimator's mean is <q, x> with the vector codes too
    d, m, N = 16, 32, 6000
    rng = np.random.default_rng(31)
    x = rng.standard_t(3, size=(1, d))
    q = rng.standard_normal((1, 1, d))
    c0 = O.make_codec(d, (1,), m, 0, S=np.zeros((m, d)), vq_bits=3)
    exact = float(q[0, 0] @ x[0])
    est = np.empty(N)
    for k in range(N):
        c = O.make_codec(d, (1,), m, 0, D=c0.D, S=rng.standard_normal((m, d)), vq_bits=3)
        est[k] = O.estimate_scores(q, O.quantize(x, c), c, 1, 1, 1, 1)[0, 0, 0]
    se = est.std() / math.sqrt(N)
    assert abs(est.mean() - exact) < 4 * se + 1e-6 * abs(exact), (est.mean(), exact, se)
    comp0 = O.quantize(x, c0)
    mse_only = np.linalg.norm(x) * float((q[0, 0] @ c0.Pi.T) @ c0.coord_cen(comp0.code_idx)[0]) / math.sqrt(d)
    assert abs(mse_only - exact) > 10 * se


def test_fibquant_d4_block_law_is_uniform_on_the_disc():
    # at d = 4 the density of (z_1, z_2) is constant on the disc |z| < 2
    # (exponent (d - 4)/2 = 0): the quasi-Monte-Carlo radii are the uniform
    # disc's quantiles |z|^2 = 4 (i + 1/2)/M, and the Bennett-Gersho spiral
    # (density f^(1/2), also uniform) puts codeword n at |z|^2 = 4 (n + 1/2)/N
    M, N = 1000, 16
    pts = O.fibquant_source_points(4, M)
    assert np.allclose((pts ** 2).sum(axis=1), 4.0 * (np.arange(M) + 0.5) / M, rtol=0, atol=1e-12)
    cb = O.fibquant_init(N, 4)
    assert np.allclose((cb ** 2).sum(axis=1), 4.0 * (np.arange(N) + 0.5) / N, rtol=0, atol=1e-12)
    # N = 1 would sit at the mean 0; with N = 2 on a uniform disc Lloyd's
    # optimum is two antipodal points at 4 rho / (3 pi) (half-disc centroid)
    cb2 = O.fibquant_codebook.__wrapped__(1, 4, M=16384, iters=40, restarts=3).astype(np.float64)
    want = 4.0 * 2.0 / (3.0 * math.pi)
    assert np.allclose(np.linalg.norm(cb2, axis=1), want, rtol=3e-3), (np.linalg.norm(cb2, axis=1), want)
