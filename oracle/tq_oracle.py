"""CPU oracle for the TurboQuant hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct restatement of what the method computes, in
float64 (numpy/scipy).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never imports, links or calls anything here, and this file
imports nothing from the library: the two share no code.  The only common
dependency is the seeded input generator module ``synth`` (random draws and
workload tensors, no method arithmetic).

Sources (page titles as given; sections / equations on each page):

* [NOTES]  "[2026 ICLR] TurboQuant: Online Vector Quantization with
  Near-optimal Distortion Rate", blog notes (july-h5kf3.github.io):
  eq. (1)-(4), Lemma 1, the residual definition, the Q_prod estimator and
  the definition of Q_prod.
* [EXPL]   "TurboQuant interactive explainer", Traditional-Chinese copy
  (news.myit.tw/news/z9s33f): §3 rotation, §4 Beta marginal, §5 Lloyd-Max,
  §6 TurboQuant-MSE, §7 shrinkage, §8 QJL and TurboQuant-prod, §0.9 prior
  work (DRIVE's randomized Hadamard).
* [PYT]    "turboquant-pytorch" skill page (skill4agent.com): Core API
  (codebook, TurboQuantMSE, TurboQuantProd, compressors), Pattern 1
  (compressed-cache attention).
* [FVQ]    FastVQ README (Zapdev-labs/turboquant): sign-flipped Hadamard
  backend and padding of the trailing dimension.

Readings taken where the pages are silent or garbled:

* Codebook for a padded Hadamard vector uses d = d_pad.
* Rotation: y = H (D * pad(x)) / sqrt(d_pad), H the Sylvester matrix in
  natural order, one round of sign flips D.  Dense: y = Pi x with
  Pi = Q diag(sign(diag R)) from the QR of a Gaussian matrix.
* Tie rule: a value equal to a boundary goes to the lower cell
  (idx = #{k : B_k < y}); sign(0) = +1 for the QJL bits.
* The residual norm enters the Q_prod estimator with exponent 1 (the notes'
  squared norm is read as a typo: only the first power makes the estimator
  unbiased, by the half-Gaussian identity of [EXPL] §8).
* QJL scale sqrt(pi/2)/m with m rows of S ([EXPL] §8 has m = d).
* The residual and S act in the rotated domain ([EXPL] §8: r = Pi x - y_mse).
* A zero vector has norm 0 and is encoded from the zero rotated vector.
* fp16 residual norms (storage variant): rho rounded to the nearest IEEE
  binary16 value, ties to even.
* Unbiased per-vector scale (EDEN; DRIVE at one bit): the Q_MSE codes are
  kept and the stored scale is S = ||x||^2 / <Pi x, C[idx]> = n / <y, C[idx]>
  in place of n, so that the unchanged decoder n Pi^T C[idx] becomes
  S Pi^T C[idx].  The codebook stays the Beta(d_pad) one (TurboQuant is EDEN
  with the scale fixed; the pages' decoder-split discussion).  A vector with
  <y, C[idx]> = 0 (only the zero vector) stores 0.

Every function below has a pin in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import functools
import math

import numpy as np
from scipy.special import betainc, gammaln
from scipy.stats import norm as _normal

# ---------------------------------------------------------------------------
# Lemma 1 and eq. (4): the coordinate density and its Lloyd-Max codebook
# ---------------------------------------------------------------------------


def beta_marginal_pdf(x, d: int):
    """Density of one coordinate of a uniform point on S^{d-1} ([NOTES] Lemma 1;
    [EXPL] §4): Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1-x^2)^((d-3)/2) on [-1, 1]."""
    x = np.asarray(x, dtype=np.float64)
    logk = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
    inside = np.abs(x) < 1.0
    out = np.zeros_like(x)
    out[inside] = np.exp(logk + (d - 3) / 2.0 * np.log1p(-x[inside] ** 2))
    return out


def beta_marginal_cdf(x, d: int):
    """CDF of the Lemma 1 density.  With t = (1+x)/2 the density becomes the
    symmetric Beta((d-1)/2, (d-1)/2) law, whose CDF is the regularized
    incomplete beta function (a library primitive)."""
    x = np.clip(np.asarray(x, dtype=np.float64), -1.0, 1.0)
    a = (d - 1) / 2.0
    return betainc(a, a, (1.0 + x) / 2.0)


def beta_marginal_first_moment(a, b, d: int):
    """Integral of x f(x) over [a, b] for the Lemma 1 density.

    d/dx (1-x^2)^((d-1)/2) = -(d-1) x (1-x^2)^((d-3)/2), so the integral is
    K [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1), K the density's constant.
    """
    logk = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)

    def g(t):
        t = np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0)
        out = np.zeros_like(t)
        inside = np.abs(t) < 1.0
        out[inside] = np.exp((d - 1) / 2.0 * np.log1p(-t[inside] ** 2))
        return out

    return math.exp(logk) * (g(a) - g(b)) / (d - 1)


def _lloyd_max(mass, moment, init, support, tol=1e-15, max_iter=200000):
    """1-D continuous k-means ([NOTES] eq. (4); [EXPL] §5): alternate
    boundaries <- midpoints of adjacent centroids and centroids <- conditional
    means of their cells, until the centroids stop moving.  ``mass(a, b)`` and
    ``moment(a, b)`` integrate f and x f over [a, b]."""
    c = np.array(init, dtype=np.float64)
    lo, hi = support
    for _ in range(max_iter):
        bnd = 0.5 * (c[1:] + c[:-1])
        edges = np.concatenate([[lo], bnd, [hi]])
        p = mass(edges[:-1], edges[1:])
        mom = moment(edges[:-1], edges[1:])
        new = mom / p
        new = 0.5 * (new - new[::-1])  # the density is even: keep the codebook odd
        if np.max(np.abs(new - c)) <= tol * np.max(np.abs(new)):
            c = new
            break
        c = new
    bnd = 0.5 * (c[1:] + c[:-1])
    return c, bnd


@functools.lru_cache(maxsize=None)
def _codebook_cached(d: int, bits: int):
    c, b = _codebook_solve(d, bits)
    c.setflags(write=False)
    b.setflags(write=False)
    return c, b


def codebook(d: int, bits: int):
    """Lloyd-Max codebook for the Lemma 1 density (cached copy of
    ``_codebook_solve``)."""
    c, b = _codebook_cached(int(d), int(bits))
    return c.copy(), b.copy()


def _codebook_solve(d: int, bits: int):
    """Lloyd-Max codebook for the Lemma 1 density in dimension d with 2^bits
    levels ([NOTES] eq. (4); [PYT] ``build_lloyd_max_codebook(dim, bits)``
    returning (boundaries, centroids)).

    Returns (centroids [2^bits] ascending, boundaries [2^bits - 1]) in float64.
    """
    n = 1 << bits
    # start at equal-probability quantiles of N(0, 1/d)
    init = _normal.ppf((np.arange(n) + 0.5) / n) / math.sqrt(d)
    init = np.clip(init, -0.999, 0.999)

    def mass(a, b):
        return beta_marginal_cdf(b, d) - beta_marginal_cdf(a, d)

    def moment(a, b):
        return beta_marginal_first_moment(a, b, d)

    return _lloyd_max(mass, moment, init, (-1.0, 1.0))


def codebook_gaussian(bits: int):
    """Lloyd-Max codebook for N(0, 1) ([EXPL] §0.9 EDEN paragraph and §5: the
    normalized Beta codebook tends to it)."""
    n = 1 << bits
    init = _normal.ppf((np.arange(n) + 0.5) / n)

    def mass(a, b):
        return _normal.cdf(b) - _normal.cdf(a)

    def moment(a, b):
        return _normal.pdf(a) - _normal.pdf(b)

    return _lloyd_max(mass, moment, init, (-np.inf, np.inf))


def codebook_mse(d: int, bits: int):
    """Per-coordinate distortion C(f_X, b) of the codebook ([NOTES] eq. (4)):
    E[x^2] - sum_i c_i^2 P_i (the centroid condition makes the cross term
    collapse); E[x^2] = 1/d for the Lemma 1 density."""
    c, bnd = codebook(d, bits)
    edges = np.concatenate([[-1.0], bnd, [1.0]])
    p = beta_marginal_cdf(edges[1:], d) - beta_marginal_cdf(edges[:-1], d)
    return 1.0 / d - float(np.sum(c * c * p))


def shrinkage(d: int, bits: int):
    """lambda_b = E[y_tilde^2] / sigma^2 with sigma^2 = 1/d ([EXPL] §7)."""
    c, bnd = codebook(d, bits)
    edges = np.concatenate([[-1.0], bnd, [1.0]])
    p = beta_marginal_cdf(edges[1:], d) - beta_marginal_cdf(edges[:-1], d)
    return d * float(np.sum(c * c * p))


# ---------------------------------------------------------------------------
# §3 rotation
# ---------------------------------------------------------------------------


def next_pow2(d: int) -> int:
    p = 1
    while p < d:
        p *= 2
    return p


def fwht(a):
    """Unnormalized Walsh-Hadamard transform along the last axis, Sylvester
    (natural) order: y_i = sum_j (-1)^popcount(i & j) a_j."""
    a = np.array(a, dtype=np.float64, copy=True)
    n = a.shape[-1]
    lead = a.shape[:-1]
    h = 1
    while h < n:
        v = a.reshape(lead + (n // (2 * h), 2, h))
        x = v[..., 0, :].copy()
        y = v[..., 1, :].copy()
        v[..., 0, :] = x + y
        v[..., 1, :] = x - y
        a = v.reshape(lead + (n,))
        h *= 2
    return a


def haar_rotation(G):
    """Dense rotation from a Gaussian draw ([EXPL] §3: QR of an iid N(0,1)
    d x d matrix, keep the orthogonal factor).  The factor is made unique with
    Q diag(sign(diag R)) so that Pi is Haar-distributed."""
    Q, R = np.linalg.qr(np.asarray(G, dtype=np.float64))
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


class Rotation:
    """Pi: either the randomized Hadamard H D / sqrt(d_pad) ([EXPL] §0.9,
    DRIVE §6; [FVQ] sign-flipped Hadamard, padded trailing dimension) or a
    dense Haar matrix from ``haar_rotation``."""

    def __init__(self, d: int, *, signs=None, G=None):
        self.d = d
        if G is not None:
            self.kind = "dense"
            self.Pi = haar_rotation(G)
            self.d_pad = d
        else:
            self.kind = "hadamard"
            self.d_pad = next_pow2(d)
            self.D = np.asarray(signs, dtype=np.float64)
            assert self.D.shape == (self.d_pad,)

    def pad(self, x):
        x = np.asarray(x, dtype=np.float64)
        if x.shape[-1] == self.d_pad:
            return x
        out = np.zeros(x.shape[:-1] + (self.d_pad,))
        out[..., : x.shape[-1]] = x
        return out

    def apply(self, x):
        """y = Pi pad(x) along the last axis."""
        if self.kind == "dense":
            return np.asarray(x, dtype=np.float64) @ self.Pi.T
        return fwht(self.pad(x) * self.D) / math.sqrt(self.d_pad)

    def apply_t(self, y):
        """Pi^T y, truncated to the first d coordinates."""
        y = np.asarray(y, dtype=np.float64)
        if self.kind == "dense":
            return y @ self.Pi
        return (self.D * fwht(y) / math.sqrt(self.d_pad))[..., : self.d]


# ---------------------------------------------------------------------------
# Bit layouts (the storage format of codes and sign bits)
# ---------------------------------------------------------------------------
#
# ROW layout: per vector, plane p (bit p of the index, p = 0 is the LSB) is a
# little-endian bit string of d_pad bits: bit i of 32-bit word w holds
# coordinate 32 w + i.  Planes are stored one after another, so a row is
# k * d_pad / 32 words.  QJL signs use the same order over the m rows of S.
#
# BLOCK32 layout: vectors are grouped in blocks of 32 consecutive vectors;
# block b holds k * d_pad words, word (p * d_pad + j) carries bit p of the
# index of coordinate j for the 32 vectors, bit t <-> vector 32 b + t.  A
# ragged last block has zero bits for the missing vectors.


def _bits_to_words(bits_le):
    """bits_le [..., n] of 0/1 -> uint32 [..., ceil(n/32)], bit i of word w =
    element 32w+i (a partial last word has zero high bits)."""
    bits_le = np.asarray(bits_le)
    n = bits_le.shape[-1]
    pad = (-n) % 32
    if pad:
        bits_le = np.concatenate([bits_le, np.zeros(bits_le.shape[:-1] + (pad,), bits_le.dtype)], -1)
    b = np.asarray(bits_le, dtype=np.uint64).reshape(bits_le.shape[:-1] + (-1, 32))
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (b * weights).sum(axis=-1).astype(np.uint32)


def _words_to_bits(words, nbits):
    w = np.asarray(words, dtype=np.uint32)[..., None]
    bits = (w >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return bits.reshape(words.shape[:-1] + (-1,))[..., :nbits].astype(np.int64)


def pack_row(idx, k: int):
    """idx [N, d_pad] ints in [0, 2^k) -> uint32 [N, k * ceil(d_pad / 32)]."""
    idx = np.asarray(idx, dtype=np.int64)
    planes = [_bits_to_words((idx >> p) & 1) for p in range(k)]
    return np.concatenate(planes, axis=-1)


def unpack_row(words, k: int, d_pad: int):
    words = np.asarray(words, dtype=np.uint32)
    wpp = (d_pad + 31) // 32
    idx = np.zeros(words.shape[:-1] + (d_pad,), dtype=np.int64)
    for p in range(k):
        idx |= _words_to_bits(words[..., p * wpp:(p + 1) * wpp], d_pad) << p
    return idx


def pack_signs(sig):
    """sig [N, m] of 0/1 (1 <-> z >= 0) -> uint32 [N, m / 32]."""
    return _bits_to_words(np.asarray(sig, dtype=np.int64))


def unpack_signs(words, m: int):
    return _words_to_bits(np.asarray(words, dtype=np.uint32), m)


def pack_block32(idx, k: int):
    """idx [N, d_pad] -> uint32 [ceil(N/32), k * d_pad] (BLOCK32 layout)."""
    idx = np.asarray(idx, dtype=np.int64)
    N, d_pad = idx.shape
    nb = (N + 31) // 32
    padded = np.zeros((nb * 32, d_pad), dtype=np.int64)
    padded[:N] = idx
    blocks = padded.reshape(nb, 32, d_pad)
    out = np.zeros((nb, k, d_pad), dtype=np.uint64)
    for p in range(k):
        bit = (blocks >> p) & 1  # [nb, 32, d_pad]
        out[:, p, :] = (bit.astype(np.uint64) << np.arange(32, dtype=np.uint64)[None, :, None]).sum(axis=1)
    return out.astype(np.uint32).reshape(nb, k * d_pad)


def unpack_block32(words, k: int, d_pad: int, n: int):
    words = np.asarray(words, dtype=np.uint32)
    nb = words.shape[0]
    w = words.reshape(nb, k, d_pad)
    idx = np.zeros((nb, 32, d_pad), dtype=np.int64)
    for p in range(k):
        bits = (w[:, p, None, :] >> np.arange(32, dtype=np.uint32)[None, :, None]) & np.uint32(1)
        idx |= bits.astype(np.int64) << p
    return idx.reshape(nb * 32, d_pad)[:n]


# ---------------------------------------------------------------------------
# Quantizers: TurboQuant-MSE and TurboQuant-prod
# ---------------------------------------------------------------------------


class Quantizer:
    """One quantizer configuration: rotation, codebook, and (for Q_prod) S.

    ``bits`` is the total budget b.  Q_MSE spends all b bits on the codebook
    ([EXPL] §6; [NOTES] Q_MSE).  Q_prod spends b-1 bits on the codebook and 1
    bit per row of S on the QJL signs of the residual ([EXPL] §8; [NOTES]
    definition of Q_prod).
    """

    def __init__(self, d: int, bits: int, *, prod: bool, draws: dict, unbiased: bool = False,
                 rnorm_f16: bool = False):
        self.d = d
        self.bits = bits
        self.prod = prod
        # Q_MSE with EDEN's unbiased per-vector scale in place of the norm
        self.unbiased = bool(unbiased) and not prod
        # Q_prod storage variant: residual norms kept as IEEE fp16 ([PYT]
        # Pattern 4 memory formula, one float16 residual norm per key)
        self.rnorm_f16 = bool(rnorm_f16) and prod
        self.k = bits - 1 if prod else bits
        if draws.get("G") is not None:
            self.rot = Rotation(d, G=draws["G"])
        else:
            self.rot = Rotation(d, signs=draws["signs"])
        self.d_pad = self.rot.d_pad
        self.centroids, self.boundaries = codebook(self.d_pad, self.k) if self.k > 0 else (
            np.zeros(1), np.zeros(0))
        if prod:
            self.S = np.asarray(draws["S"], dtype=np.float64)
            self.m = self.S.shape[0]
            assert self.S.shape[1] == self.d_pad
            # [EXPL] §8: sqrt(pi/2) undoes the half-Gaussian shrinkage, 1/m
            # averages over the m rows of S.
            self.kappa = math.sqrt(math.pi / 2.0) / self.m

    # -- encode ------------------------------------------------------------

    def rotate_unit(self, x):
        """Norms n = ||x|| and y = Pi (x / n) ([NOTES] assumption ||x|| = 1,
        otherwise store the L2 norm; [PYT] compressors normalize internally)."""
        x = np.asarray(x, dtype=np.float64)
        n = np.sqrt(np.sum(x * x, axis=-1))
        safe = np.where(n > 0, n, 1.0)
        xh = np.where((n > 0)[..., None], x / safe[..., None], 0.0)
        return n, self.rot.apply(xh)

    def quantize(self, y):
        """Nearest centroid by boundary count: idx = #{k : B_k < y}
        ([NOTES] Q_MSE: nearest centroid per coordinate; ties to the lower cell)."""
        return np.searchsorted(self.boundaries, y, side="left")

    def encode(self, x, layout: str = "row"):
        """Returns a dict with codes (packed), norms (fp32) and, for Q_prod,
        signs (packed) and rnorms (fp32).  Also returns the float64
        intermediates (y, z) so tests can find coordinates that sit near a
        decision boundary."""
        n, y = self.rotate_unit(x)
        idx = self.quantize(y)
        out = {"norms": n.astype(np.float32), "idx": idx, "y": y}
        if self.unbiased:
            out["norms"] = self.unbiased_scale(n, y, idx).astype(np.float32)
        pack = pack_row if layout == "row" else pack_block32
        out["codes"] = pack(idx, self.k)
        if self.prod:
            # [NOTES] residual r = x - Q_mse^{-1}(Q_mse(x)) in the rotated
            # domain ([EXPL] §8), its norm, and sign(S r) ([EXPL] §8 QJL).
            r = y - self.centroids[idx]
            rho = np.sqrt(np.sum(r * r, axis=-1))
            z = r @ self.S.T
            sig = (z >= 0).astype(np.int64)
            out.update(rnorms=rho.astype(np.float16 if self.rnorm_f16 else np.float32),
                       signs=pack_signs(sig), z=z, rho64=rho)
        return out

    def unbiased_scale(self, n, y, idx):
        """EDEN's per-vector scale ([EXPL] prior work, EDEN paragraph:
        S = ||x||^2 / <R(x), Q(R(x))>, which makes S R^T Q(R(x)) unbiased; DRIVE
        is the one-bit case, S = ||x||^2 / ||R(x)||_1 with sign codes).  Here
        R(x) = Pi x = n y and Q(R(x)) = n C[idx] up to the codebook's fixed
        scale, which cancels between the scale and the decoder:
        S = n^2 / (n <y, C[idx]>) = n / <y, C[idx]>."""
        dot = np.sum(y * self.centroids[idx], axis=-1)
        ok = dot > 0
        return np.where(ok, np.asarray(n, np.float64) / np.where(ok, dot, 1.0), 0.0)

    # -- decode / estimate -------------------------------------------------

    def dequant_rotated(self, idx):
        return self.centroids[np.asarray(idx)]

    def decode(self, idx, norms, signs=None, rnorms=None):
        """x_tilde = n Pi^T (C[idx] [+ kappa rho S^T (2 sigma - 1)]) ([NOTES]
        Q_MSE^{-1}: centroids then Pi^T; QJL dequantization map of [EXPL] §8)."""
        yt = self.dequant_rotated(idx)
        if signs is not None and self.prod:
            sgn = 2.0 * unpack_signs(signs, self.m) - 1.0
            yt = yt + self.kappa * np.asarray(rnorms, np.float64)[..., None] * (sgn @ self.S)
        return np.asarray(norms, np.float64)[..., None] * self.rot.apply_t(yt)

    def query_prep(self, q):
        """q' = Pi q (the query is rotated, not normalized) and u = S q'."""
        qp = self.rot.apply(np.asarray(q, dtype=np.float64))
        u = qp @ self.S.T if self.prod else None
        return qp, u

    def scores(self, q, idx, norms, signs=None, rnorms=None):
        """Inner-product estimates <q_a, x_t> for queries [Q, d] against encoded
        vectors, [Q, N] ([NOTES] unbiased estimator with the residual norm to the
        first power; [EXPL] §8 QJL decoder; [PYT] ``inner_product`` /
        ``asymmetric_attention_scores``)."""
        qp, u = self.query_prep(np.atleast_2d(q))
        mse = qp @ self.dequant_rotated(idx).T
        s = mse
        if self.prod:
            sgn = 2.0 * unpack_signs(signs, self.m) - 1.0
            s = s + self.kappa * (u @ sgn.T) * np.asarray(rnorms, np.float64)[None, :]
        return s * np.asarray(norms, np.float64)[None, :]


# ---------------------------------------------------------------------------
# Decode attention over a compressed cache ([PYT] Pattern 1)
# ---------------------------------------------------------------------------


def softmax_attend(scores, values):
    """softmax over the last axis of ``scores`` (two passes: max, then sum of
    exponentials), then the weighted sum of ``values`` rows ([PYT] Pattern 1:
    ``torch.softmax`` then ``einsum('hs,hsd->hd')``)."""
    s = np.asarray(scores, dtype=np.float64)
    mx = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - mx)
    p = e / np.sum(e, axis=-1, keepdims=True)
    return p @ np.asarray(values, dtype=np.float64)


def decode_attention(q, kq: Quantizer, vq: Quantizer, kenc, venc, scale: float, group: int):
    """One decode step for one (layer, batch, kv-head) and its ``group`` query
    heads: scores from the compressed keys (Q_prod estimator), softmax with
    ``scale``, values reconstructed by Q_MSE^{-1} and averaged.

    q [group, d]; kenc / venc hold idx (unpacked), norms, signs, rnorms.
    The value average is formed in the rotated domain and rotated back once:
    sum_t p_t n_t Pi^T C[i_t] = Pi^T sum_t p_t n_t C[i_t] (Pi^T is linear).
    Returns [group, d].
    """
    s = kq.scores(q, kenc["idx"], kenc["norms"], kenc.get("signs"), kenc.get("rnorms"))
    vrot = vq.dequant_rotated(venc["idx"]) * np.asarray(venc["norms"], np.float64)[:, None]
    orot = softmax_attend(scale * s, vrot)
    return vq.rot.apply_t(orot)


def topk(scores, k: int):
    """Top-k per row by (score descending, index ascending).  Returns
    (values [Q, k], indices [Q, k])."""
    s = np.asarray(scores)
    n = s.shape[-1]
    order = np.lexsort((np.broadcast_to(np.arange(n), s.shape), -s), axis=-1)[..., :k]
    return np.take_along_axis(s, order, axis=-1), order
