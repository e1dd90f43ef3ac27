"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- values printed on the pages (tests/golden/), closed forms,
special cases that reduce to a textbook or library routine, Monte Carlo
expectations with standard-error bounds, and brute force on tiny inputs."""
import math

import numpy as np
import pytest
from scipy import integrate
from scipy.linalg import hadamard
from scipy.special import softmax

from oracle import tq_oracle as o
from tests.conftest import load_golden

G = load_golden("expl_printed_constants.txt")


def _vals(key):
    vals, tol = G[key]
    return [float(v.split(":")[-1]) for v in vals], tol


# ---------------------------------------------------------------- density


def test_density_normalized_and_variance():
    # Lemma 1 density integrates to 1 and has variance 1/d (the explainer's
    # std 1/sqrt(d) argument, §0 primer), by adaptive quadrature.
    for d in (4, 10, 64, 128, 1536):
        f = lambda x: o.beta_marginal_pdf(np.array([x]), d)[0]
        tot = integrate.quad(f, -1, 1, epsabs=0, epsrel=1e-12, limit=400, points=[0.0])[0]
        var = integrate.quad(lambda x: x * x * f(x), -1, 1, epsabs=0, epsrel=1e-12, limit=400,
                             points=[0.0])[0]
        assert abs(tot - 1) < 1e-9
        assert abs(var * d - 1) < 1e-8


def test_density_low_dim_special_cases():
    # §4: in 2-D the marginal is the arcsine law 1/(pi sqrt(1-x^2)); in 3-D it
    # is uniform on [-1, 1].
    x = np.linspace(-0.95, 0.95, 39)
    assert np.allclose(o.beta_marginal_pdf(x, 2), 1 / (math.pi * np.sqrt(1 - x * x)), rtol=1e-12)
    assert np.allclose(o.beta_marginal_pdf(x, 3), 0.5, rtol=1e-12)
    assert np.allclose(o.beta_marginal_cdf(x, 3), (x + 1) / 2, rtol=1e-12)


def test_cdf_and_moment_against_quadrature():
    for d in (5, 128, 1536):
        f = lambda t: o.beta_marginal_pdf(np.array([t]), d)[0]
        for a, b in ((-0.3, -0.01), (-0.02, 0.05), (0.01, 0.2), (0.1, 1.0)):
            pts = [p for p in (0.0,) if a < p < b]
            m0 = integrate.quad(f, a, b, epsabs=0, epsrel=1e-12, limit=400, points=pts or None)[0]
            m1 = integrate.quad(lambda t: t * f(t), a, b, epsabs=0, epsrel=1e-12, limit=400,
                                points=pts or None)[0]
            assert abs(o.beta_marginal_cdf(b, d) - o.beta_marginal_cdf(a, d) - m0) < 1e-11
            assert abs(o.beta_marginal_first_moment(a, b, d) - m1) < 1e-11


def test_coordinate_std_printed():
    # §0 primer: coordinate std of a random unit vector is 1/sqrt(d) -- the
    # printed 0.316 / 0.1 / 0.032 at d = 10 / 100 / 1000 (Monte Carlo over
    # points drawn with a Haar rotation of e_1).
    vals, tol = G["coordinate_std"]
    rng = np.random.default_rng(5)
    for item in vals:
        d, want = item.split(":")
        d = int(d)
        n = 4000
        pts = np.array([o.haar_rotation(rng.standard_normal((d, d)))[:, 0] for _ in range(60)]) \
            if d <= 100 else rng.standard_normal((n, d))
        if d > 100:
            pts = pts / np.linalg.norm(pts, axis=1, keepdims=True)
        std = pts.std()
        assert abs(std - float(want)) < max(tol, 0.02 * float(want))


# ---------------------------------------------------------------- codebook


def test_gaussian_codebook_printed():
    # §0.9 / §5: N(0,1) Lloyd-Max centroids {±0.798} (b=1), {±0.453, ±1.510} (b=2).
    for bits, key in ((1, "gaussian_codebook_b1_pos"), (2, "gaussian_codebook_b2_pos")):
        want, tol = _vals(key)
        c, _ = o.codebook_gaussian(bits)
        assert np.allclose(c[len(c) // 2:], want, atol=tol)
    c1, _ = o.codebook_gaussian(1)
    assert abs(c1[1] - math.sqrt(2 / math.pi)) < 1e-12


def test_codebook_d3_is_uniform_quantizer():
    # §4: the 3-D marginal is uniform, so Lloyd-Max must return the uniform
    # quantizer c_i = -1 + (2i - 1) / 2^b (textbook result for a uniform law).
    for bits in (1, 2, 3, 4):
        c, B = o.codebook(3, bits)
        n = 1 << bits
        want = -1 + (2 * np.arange(1, n + 1) - 1) / n
        assert np.allclose(c, want, atol=1e-12)
        assert np.allclose(B, -1 + 2 * np.arange(1, n) / n, atol=1e-12)


def test_codebook_one_bit_is_half_mean():
    # b = 1: the positive centroid is E[x | x > 0] = 2 * integral_0^1 x f(x) dx,
    # computed here by quadrature.
    for d in (3, 16, 128, 256, 1536):
        f = lambda x: o.beta_marginal_pdf(np.array([x]), d)[0]
        want = 2 * integrate.quad(lambda x: x * f(x), 0, 1, epsabs=0, epsrel=1e-13, limit=400)[0]
        c, B = o.codebook(d, 1)
        assert abs(c[1] - want) < 1e-12 and abs(c[0] + want) < 1e-12 and B[0] == 0.0


def test_codebook_tends_to_gaussian():
    # §4/§5: the marginal tends to N(0, 1/d), so sqrt(d) c(Beta, d) -> N(0,1) codebook.
    for bits in (1, 2, 3, 4):
        g, _ = o.codebook_gaussian(bits)
        c128 = o.codebook(128, bits)[0] * math.sqrt(128)
        c1536 = o.codebook(1536, bits)[0] * math.sqrt(1536)
        assert np.max(np.abs(c128 / g - 1)) < 0.02
        assert np.max(np.abs(c1536 / g - 1)) < 0.004


def test_codebook_lloyd_conditions_and_monte_carlo():
    # Lloyd optimality checked by sampling uniform points on the sphere: the
    # conditional mean of each cell equals its centroid and the empirical MSE
    # equals codebook_mse, both within 4 standard errors.
    rng = np.random.default_rng(11)
    d = 32
    n = 400_000
    x = rng.standard_normal((n, d))
    x1 = x[:, 0] / np.linalg.norm(x, axis=1)
    for bits in (1, 2, 3):
        c, B = o.codebook(d, bits)
        idx = np.searchsorted(B, x1)
        for i in range(len(c)):
            sel = x1[idx == i]
            se = sel.std() / math.sqrt(len(sel))
            assert abs(sel.mean() - c[i]) < 4 * se + 1e-12
        err = (x1 - c[idx]) ** 2
        assert abs(err.mean() - o.codebook_mse(d, bits)) < 4 * err.std() / math.sqrt(n)


def test_shrinkage_printed():
    # §7: lambda_b = 0.64 / 0.88 / 0.97 / 0.99 (b = 1..4), exactly 2/pi at one
    # bit in the Gaussian limit.
    want, tol = _vals("shrinkage_b1_to_b4")
    for bits, w in zip((1, 2, 3, 4), want):
        assert abs(o.shrinkage(128, bits) - w) < tol
    lim, tol1 = _vals("shrinkage_b1_limit")
    assert abs(o.shrinkage(100_000, 1) - lim[0]) < 2e-5
    assert abs(2 / math.pi - lim[0]) < tol1


def test_distortion_bounds_and_rate():
    # §5 / §9: d * D_b <= (sqrt(3) pi / 2) 4^-b; ratio to the 4^-b lower bound
    # ~1.45 at b=1; [digest] "each extra bit cuts the MSE four-fold" -> ratio in [3, 4.2].
    const, _ = _vals("mse_upper_const")
    assert abs(math.sqrt(3) * math.pi / 2 - const[0]) < 1e-12
    ratio1, tol = _vals("mse_ratio_b1")
    for d in (128, 1536):
        dd = [d * o.codebook_mse(d, b) for b in (1, 2, 3, 4)]
        for b, v in zip((1, 2, 3, 4), dd):
            assert 4.0 ** -b <= v <= const[0] * 4.0 ** -b
        for b in range(3):
            assert 3.0 <= dd[b] / dd[b + 1] <= 4.2
    big = 100_000 * o.codebook_mse(100_000, 1)
    assert abs(big / 0.25 - ratio1[0]) < tol


# ---------------------------------------------------------------- rotation


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_equals_sylvester_matrix(n):
    rng = np.random.default_rng(n)
    a = rng.standard_normal((5, n))
    assert np.allclose(o.fwht(a), a @ hadamard(n).T, atol=1e-11)


def test_hadamard_rotation_orthogonal_and_padding():
    # §3: the rotation preserves lengths and inner products; a 192-d vector is
    # zero-padded to the 256-point transform.
    rng = np.random.default_rng(3)
    for d in (128, 192):
        dp = o.next_pow2(d)
        D = np.where(rng.integers(0, 2, dp) == 0, 1.0, -1.0)
        R = o.Rotation(d, signs=D)
        x = rng.standard_normal((7, d))
        y = R.apply(x)
        assert y.shape == (7, dp)
        assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
        assert np.allclose(y @ y.T, x @ x.T, atol=1e-10)
        assert np.allclose(R.apply_t(y), x, atol=1e-12)
        # explicit matrix: H D / sqrt(d_pad)
        M = hadamard(dp) * D[None, :] / math.sqrt(dp)
        assert np.allclose(y, R.pad(x) @ M.T, atol=1e-12)


def test_haar_rotation_orthogonal_and_sign_fixed():
    # §3: QR of a Gaussian matrix, orthogonal factor; with the sign fix the
    # first column is the normalized first Gaussian column, so E[Pi_00] = 0 and
    # E[Pi_00^2] = 1/d (a plain LAPACK Q has Pi_00 of one fixed sign).
    rng = np.random.default_rng(9)
    d = 6
    v = []
    for _ in range(3000):
        Gm = rng.standard_normal((d, d))
        P = o.haar_rotation(Gm)
        v.append(P[0, 0])
        assert np.allclose(P[:, 0], Gm[:, 0] / np.linalg.norm(Gm[:, 0]), atol=1e-12)
    P = o.haar_rotation(rng.standard_normal((64, 64)))
    assert np.allclose(P.T @ P, np.eye(64), atol=1e-12)
    v = np.array(v)
    assert abs(v.mean()) < 4 * v.std() / math.sqrt(len(v))
    assert abs((v * v).mean() - 1 / d) < 4 * (v * v).std() / math.sqrt(len(v))


# ---------------------------------------------------------------- quantize and pack


def _draws(d, m, seed, dense=False, f64=False):
    rng = np.random.default_rng(seed)
    dp = d if dense else o.next_pow2(d)
    S = rng.standard_normal((m, dp))
    return {"signs": np.where(rng.integers(0, 2, dp) == 0, 1, -1),
            "S": S if f64 else S.astype(np.float16).astype(np.float32),
            "G": rng.standard_normal((d, d)) if dense else None}


def test_quantize_brute_force_product_codebook():
    # Tiny d_pad: the nearest point of the full product codebook (all 2^(b d)
    # points) equals the per-coordinate nearest centroid (separability).
    rng = np.random.default_rng(1)
    for d, bits in ((4, 1), (4, 2), (8, 1), (8, 2)):
        q = o.Quantizer(d, bits, prod=False, draws=_draws(d, 32, 0))
        c = q.centroids
        grid = np.array(np.meshgrid(*([np.arange(len(c))] * d), indexing="ij")).reshape(d, -1).T
        pts = c[grid]
        y = rng.standard_normal((50, d)) / math.sqrt(d)
        brute = np.argmin(((y[:, None, :] - pts[None]) ** 2).sum(-1), axis=1)
        assert np.array_equal(grid[brute], q.quantize(y))


def test_quantize_tie_goes_to_lower_cell():
    q = o.Quantizer(128, 3, prod=False, draws=_draws(128, 32, 0))
    B = q.boundaries
    assert np.array_equal(q.quantize(B), np.arange(len(B)))
    assert np.array_equal(q.quantize(np.nextafter(B, 1)), np.arange(1, len(B) + 1))
    assert q.quantize(np.array([0.0]))[0] == (len(B) // 2)


def test_pack_layout_bit_positions_and_roundtrip():
    rng = np.random.default_rng(2)
    for k, dp in ((1, 128), (2, 128), (3, 128), (4, 256), (3, 1536)):
        idx = rng.integers(0, 1 << k, size=(45, dp))
        w = o.pack_row(idx, k)
        assert w.shape == (45, k * dp // 32) and w.dtype == np.uint32
        assert np.array_equal(o.unpack_row(w, k, dp), idx)
        # explicit bit position: plane p, word j // 32, bit j % 32
        for t, j, p in ((0, 0, 0), (3, 37, k - 1), (44, dp - 1, 0)):
            bit = (int(w[t, p * dp // 32 + j // 32]) >> (j % 32)) & 1
            assert bit == (idx[t, j] >> p) & 1
        wb = o.pack_block32(idx, k)
        assert wb.shape == (2, k * dp)
        assert np.array_equal(o.unpack_block32(wb, k, dp, 45), idx)
        for t, j, p in ((0, 0, 0), (33, 5, k - 1), (44, dp - 1, 0)):
            bit = (int(wb[t // 32, p * dp + j]) >> (t % 32)) & 1
            assert bit == (idx[t, j] >> p) & 1
        assert np.all(wb[1] >> np.uint32(13) == 0)  # missing vectors of a ragged block are zero
    s = rng.integers(0, 2, size=(9, 128))
    assert np.array_equal(o.unpack_signs(o.pack_signs(s), 128), s)


def test_zero_vector_encoding():
    q = o.Quantizer(128, 3, prod=True, draws=_draws(128, 128, 4))
    e = q.encode(np.zeros((2, 128)))
    assert np.all(e["norms"] == 0) and np.all(e["rnorms"] >= 0)
    mid = (1 << q.k) // 2 - 1  # y = 0 sits on the middle boundary -> lower cell
    assert np.all(e["idx"] == mid)


# ---------------------------------------------------------------- estimators


def test_half_gaussian_identity():
    # §8: E[(s.y) sign(s.x)] = sqrt(2/pi) <x, y> / ||x|| for s ~ N(0, I).
    rng = np.random.default_rng(7)
    d = 16
    x = rng.standard_normal(d)
    y = rng.standard_normal(d)
    S = rng.standard_normal((400_000, d))
    v = (S @ y) * np.where(S @ x >= 0, 1.0, -1.0)
    want = math.sqrt(2 / math.pi) * x @ y / np.linalg.norm(x)
    assert abs(v.mean() - want) < 4 * v.std() / math.sqrt(len(v))


def test_qprod_unbiased_over_seeds_of_S():
    # [NOTES] eq. (3) / Q_prod: for fixed x, q, Pi the estimator averaged over
    # >= 1e4 independent draws of S equals <q, x> (bias below 3 standard
    # errors), and its variance obeys the QJL bound pi/(2m) ||r||^2 ||q'||^2 n^2.
    rng = np.random.default_rng(21)
    d, m, bits = 32, 32, 3
    x = rng.standard_normal(d) * 3.0
    qv = rng.standard_normal(d)
    base = _draws(d, m, 0, f64=True)
    est = []
    q0 = o.Quantizer(d, bits, prod=True, draws=base)
    n, y = q0.rotate_unit(x[None])
    r = y - q0.centroids[q0.quantize(y)]
    for s in range(12000):
        dr = dict(base)
        dr["S"] = np.random.default_rng([21, s]).standard_normal((m, d))
        q = o.Quantizer(d, bits, prod=True, draws=dr)
        e = q.encode(x[None])
        est.append(q.scores(qv[None], e["idx"], e["norms"], e["signs"], e["rnorms"])[0, 0])
    est = np.array(est)
    truth = qv @ x
    se = est.std() / math.sqrt(len(est))
    assert abs(est.mean() - truth) < 3 * se
    qp = q0.rot.apply(qv)
    bound = math.pi / (2 * m) * float(r[0] @ r[0]) * float(qp @ qp) * float(n[0] ** 2)
    assert est.var() <= bound * 1.05


def _fp16_gaussian(rng, shape):
    # the library's S: standard normal draws rounded to the nearest IEEE
    # binary16 value (round to nearest even), held exactly in fp32
    return rng.standard_normal(shape).astype(np.float16).astype(np.float32)


def test_half_gaussian_identity_fp16_rounded_draws():
    # The identity behind the QJL estimator (§8) with the rows of S that the
    # library accepts: N(0, 1) entries rounded to fp16.  Rounding moves each
    # entry by at most 2^-11 of its value, far inside the Monte Carlo error
    # at 4e5 draws, so the identity must still hold within 4 standard errors.
    rng = np.random.default_rng(8)
    d = 16
    x = rng.standard_normal(d)
    y = rng.standard_normal(d)
    S = _fp16_gaussian(rng, (400_000, d)).astype(np.float64)
    v = (S @ y) * np.where(S @ x >= 0, 1.0, -1.0)
    want = math.sqrt(2 / math.pi) * x @ y / np.linalg.norm(x)
    assert abs(v.mean() - want) < 4 * v.std() / math.sqrt(len(v))
    # the second moment that the variance bound uses is unchanged too:
    # E[(s.y)^2] = ||y||^2 within 4 standard errors
    w = (S @ y) ** 2
    assert abs(w.mean() - y @ y) < 4 * w.std() / math.sqrt(len(w))


def test_qprod_unbiased_over_seeds_of_fp16_S():
    # [NOTES] eq. (3) / Q_prod with the fp16-rounded Gaussian S the library
    # requires: for fixed x, q, Pi the estimator averaged over 12,000
    # independent fp16-rounded draws of S equals <q, x> within 3 standard
    # errors, and its variance obeys the QJL bound pi/(2m) ||r||^2 ||q'||^2 n^2
    # (explainer §8, Lemma 4 and the half-Gaussian identity).
    rng = np.random.default_rng(22)
    d, m, bits = 32, 32, 3
    x = rng.standard_normal(d) * 2.0
    qv = rng.standard_normal(d)
    base = _draws(d, m, 1, f64=True)
    q0 = o.Quantizer(d, bits, prod=True, draws=base)
    n, y = q0.rotate_unit(x[None])
    r = y - q0.centroids[q0.quantize(y)]
    est = []
    for s in range(12000):
        dr = dict(base)
        dr["S"] = _fp16_gaussian(np.random.default_rng([22, s]), (m, d))
        assert np.array_equal(dr["S"], dr["S"].astype(np.float16).astype(np.float32))
        q = o.Quantizer(d, bits, prod=True, draws=dr)
        e = q.encode(x[None])
        est.append(q.scores(qv[None], e["idx"], e["norms"], e["signs"], e["rnorms"])[0, 0])
    est = np.array(est)
    truth = qv @ x
    se = est.std() / math.sqrt(len(est))
    assert abs(est.mean() - truth) < 3 * se
    qp = q0.rot.apply(qv)
    bound = math.pi / (2 * m) * float(r[0] @ r[0]) * float(qp @ qp) * float(n[0] ** 2)
    assert est.var() <= bound * 1.05


def test_qmse_shrinkage_over_haar_rotations():
    # §7: with a uniformly random rotation, E<y, x~> = lambda_b <y, x>, with
    # lambda_b = d sum_i c_i^2 P_i from the codebook (within 3 standard errors).
    rng = np.random.default_rng(31)
    d, bits = 24, 1
    x = rng.standard_normal(d)
    yv = x + 0.5 * rng.standard_normal(d)
    ratio = []
    for s in range(10000):
        dr = {"signs": None, "S": None, "G": np.random.default_rng([31, s]).standard_normal((d, d))}
        q = o.Quantizer(d, bits, prod=False, draws=dr)
        e = q.encode(x[None])
        xt = q.decode(e["idx"], e["norms"])[0]
        ratio.append(yv @ xt / (yv @ x))
    ratio = np.array(ratio)
    lam = o.shrinkage(d, bits)
    assert abs(ratio.mean() - lam) < 3 * ratio.std() / math.sqrt(len(ratio))
    assert abs(lam - 2 / math.pi) < 0.02


# ---------------------------------------------------------------- unbiased (EDEN / DRIVE) scale


@pytest.mark.parametrize("d,bits,dense", [(24, 1, True), (24, 3, True), (100, 2, False),
                                          (128, 4, False), (192, 3, False)])
def test_unbiased_scale_keeps_the_component_along_x(d, bits, dense):
    # x~ = S Pi^T C[idx] with S = ||x||^2 / <Pi x, C[idx]> (EDEN's scale): the
    # component of x~ along x is x itself for every rotation, <x~, x> = ||x||^2,
    # up to the fp32 rounding of the stored scale.  The plain norm (Q_MSE) or
    # the least-squares scale n <y, C> / ||C||^2 both miss it.
    rng = np.random.default_rng(51)
    q = o.Quantizer(d, bits, prod=False, draws=_draws(d, 32, 3, dense=dense), unbiased=True)
    x = rng.standard_normal((200, d)) * rng.lognormal(0, 1, size=(200, 1))
    x[7] = 0.0
    e = q.encode(x)
    xt = q.decode(e["idx"], e["norms"])
    got, want = np.sum(xt * x, axis=1), np.sum(x * x, axis=1)
    nz = want > 0
    assert np.max(np.abs(got[nz] / want[nz] - 1.0)) < 3e-7
    assert e["norms"][7] == 0.0 and np.all(xt[7] == 0.0)
    plain = o.Quantizer(d, bits, prod=False, draws=_draws(d, 32, 3, dense=dense))
    pe = plain.encode(x)
    assert np.array_equal(pe["idx"], e["idx"])  # same codes, only the scale differs
    xp = plain.decode(pe["idx"], pe["norms"])
    assert np.min(np.abs(np.sum(xp * x, axis=1)[nz] / want[nz] - 1.0)) > 1e-4


@pytest.mark.parametrize("dense", [True, False])
def test_unbiased_scale_one_bit_is_drive(dense):
    # One bit: C[idx] = +-c1 sign(y), and the scale reduces to DRIVE's unbiased
    # S = ||x||^2 / ||R x||_1 applied to sign(R x): x~ = S R^T sign(R x), with R
    # written out here as an explicit matrix.
    rng = np.random.default_rng(52)
    d = 40
    q = o.Quantizer(d, 1, prod=False, draws=_draws(d, 32, 4, dense=dense), unbiased=True)
    R = q.rot.apply(np.eye(d)).T  # column i = R e_i
    x = rng.standard_normal((50, d)) * 2.5
    e = q.encode(x)
    xt = q.decode(e["idx"], e["norms"])
    Rx = x @ R.T
    S = np.sum(x * x, axis=1) / np.sum(np.abs(Rx), axis=1)
    drive = S[:, None] * (np.sign(Rx) @ R)
    np.testing.assert_allclose(xt, drive, rtol=3e-7, atol=3e-7 * np.abs(drive).max())


def test_unbiased_scale_over_haar_rotations():
    # EDEN: over uniformly random rotations the reconstruction is unbiased,
    # E[x~] = x (each coordinate within 4 standard errors), where the plain
    # norm shrinks it by lambda_b.
    rng = np.random.default_rng(61)
    d, bits, n = 16, 2, 10000
    x = rng.standard_normal(d)
    xs = np.empty((n, d))
    for s in range(n):
        dr = {"signs": None, "S": None, "G": np.random.default_rng([61, s]).standard_normal((d, d))}
        q = o.Quantizer(d, bits, prod=False, draws=dr, unbiased=True)
        e = q.encode(x[None])
        xs[s] = q.decode(e["idx"], e["norms"])[0]
    se = xs.std(axis=0) / math.sqrt(n)
    assert np.all(np.abs(xs.mean(axis=0) - x) < 4 * se)
    lam = o.shrinkage(d, bits)
    assert np.any(np.abs(lam * x - x) > 8 * se)  # the test separates the biased decoder


def _fp16_round_reference(v):
    """Nearest IEEE binary16 value of positive doubles, ties to even, from the
    format's definition (11 significant bits; exponents -14..15; below 2^-14
    a fixed step of 2^-24), independent of numpy's float16 cast."""
    out = []
    for x in v:
        x = float(x)
        if x == 0.0:
            out.append(0.0)
            continue
        e = max(math.floor(math.log2(x)), -14)
        step = 2.0 ** (e - 10)
        q, r = divmod(x, step)
        if r > step / 2 or (r == step / 2 and int(q) % 2 == 1):
            q += 1
        out.append(q * step)
    return np.array(out)


def test_fp16_residual_norms_round_to_nearest_even():
    # storage variant: rho kept as binary16; checked against the format's
    # definition, including exact ties and subnormal residual norms
    d, bits = 128, 3
    q16 = o.Quantizer(d, bits, prod=True, draws=_draws(d, 64, 5), rnorm_f16=True)
    x = np.random.default_rng(71).standard_normal((300, d)) * 7.0
    e = q16.encode(x)
    assert e["rnorms"].dtype == np.float16
    np.testing.assert_array_equal(e["rnorms"].astype(np.float64), _fp16_round_reference(e["rho64"]))
    rel = np.abs(e["rnorms"].astype(np.float64) / e["rho64"] - 1.0)
    assert rel.max() <= 2.0 ** -11
    ties = np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 0.5 + 2.0 ** -12, 3.0 * 2.0 ** -25])
    np.testing.assert_array_equal(ties.astype(np.float16).astype(np.float64), _fp16_round_reference(ties))
    # codes, signs and norms are those of the fp32 variant
    q32 = o.Quantizer(d, bits, prod=True, draws=_draws(d, 64, 5))
    e32 = q32.encode(x)
    for k in ("codes", "signs", "norms"):
        assert np.array_equal(e[k], e32[k])


def test_residual_norm_expectation():
    # Residual energy: E||r||^2 = d_pad * C(f, b-1) over random unit inputs
    # (the notes' E||r|| = sqrt(C) read as the second moment); dense Haar
    # rotation so the coordinates follow Lemma 1 exactly.
    rng = np.random.default_rng(41)
    d, bits = 48, 3
    q = o.Quantizer(d, bits, prod=True, draws=_draws(d, 32, 1, dense=True))
    x = rng.standard_normal((60000, d))
    e = q.encode(x)
    rr = e["rho64"] ** 2
    want = d * o.codebook_mse(d, bits - 1)
    assert abs(rr.mean() - want) < 4 * rr.std() / math.sqrt(len(rr))


def test_decode_against_explicit_matrices():
    # Q_MSE^{-1}: x~ = n Pi^T C[idx] ([NOTES] Q_MSE), with Pi^T written out as an
    # explicit matrix (scipy Sylvester Hadamard, or the dense factor) and the
    # padding dropped.
    rng = np.random.default_rng(8)
    for d, dense in ((128, False), (192, False), (40, True)):
        dr = _draws(d, 32, 2, dense=dense)
        q = o.Quantizer(d, 3, prod=False, draws=dr)
        idx = rng.integers(0, 8, size=(5, q.d_pad))
        n = rng.uniform(0.5, 3.0, size=5)
        if dense:
            M = q.rot.Pi
        else:
            M = hadamard(q.d_pad) * np.asarray(dr["signs"], float)[None, :] / math.sqrt(q.d_pad)
        want = n[:, None] * (q.centroids[idx] @ M)[:, :d]
        assert np.allclose(q.decode(idx, n), want, atol=1e-12)
        # encode of a decoded direction returns the same cells when it is a
        # codebook point scaled to unit length and the cells are wide enough
        x = want[0]
        e = q.encode(x[None])
        assert abs(e["norms"][0] - np.linalg.norm(x)) <= 1e-6 * np.linalg.norm(x)


def test_scores_match_full_dequantization():
    # The score estimator equals <q, x~_prod> with the Q_prod dequantization
    # n Pi^T (C[idx] + kappa rho S^T sign): linearity of Pi^T and S^T.
    rng = np.random.default_rng(12)
    for d, dense in ((128, False), (192, False), (48, True)):
        q = o.Quantizer(d, 3, prod=True, draws=_draws(d, 64 if not dense else 48, 3, dense=dense))
        x = rng.standard_normal((20, d))
        qq = rng.standard_normal((3, d))
        e = q.encode(x)
        s = q.scores(qq, e["idx"], e["norms"], e["signs"], e["rnorms"])
        xt = q.decode(e["idx"], e["norms"], e["signs"], e["rnorms"])
        assert np.allclose(s, qq @ xt.T, rtol=1e-10, atol=1e-10)


def test_softmax_attend_is_textbook():
    rng = np.random.default_rng(13)
    s = rng.standard_normal((4, 300)) * 5
    v = rng.standard_normal((300, 16))
    assert np.allclose(o.softmax_attend(s, v), softmax(s, axis=-1) @ v, rtol=1e-12, atol=1e-12)


def test_decode_attention_rotated_domain_equals_original_domain():
    # [PYT] Pattern 1 decompresses every value and averages in the original
    # domain; the oracle averages in the rotated domain and rotates once.
    rng = np.random.default_rng(14)
    d, seq, grp = 192, 300, 4
    kq = o.Quantizer(d, 4, prod=True, draws=_draws(d, 256, 5))
    vq = o.Quantizer(d, 4, prod=False, draws=_draws(d, 32, 6))
    K = rng.standard_normal((seq, d))
    V = rng.standard_normal((seq, d)) * 2
    qh = rng.standard_normal((grp, d))
    ke = kq.encode(K)
    ve = vq.encode(V, layout="block32")
    out = o.decode_attention(qh, kq, vq, ke, ve, 1 / math.sqrt(d), grp)
    s = kq.scores(qh, ke["idx"], ke["norms"], ke["signs"], ke["rnorms"]) / math.sqrt(d)
    vals = vq.decode(ve["idx"], ve["norms"])
    assert np.allclose(out, softmax(s, axis=-1) @ vals, rtol=1e-10, atol=1e-10)
    # and with exact (unquantized) scores/values it is plain attention
    exact = o.softmax_attend(qh @ K.T / math.sqrt(d), V)
    assert np.allclose(exact, softmax(qh @ K.T / math.sqrt(d), axis=-1) @ V)


def test_topk_brute_force():
    rng = np.random.default_rng(15)
    s = rng.integers(0, 20, size=(6, 200)).astype(np.float64)  # many ties
    v, i = o.topk(s, 10)
    for r in range(6):
        want = sorted(range(200), key=lambda j: (-s[r, j], j))[:10]
        assert list(i[r]) == want
        assert np.array_equal(v[r], s[r, want])
