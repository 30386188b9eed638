"""Pins for the float64 oracle: each checks it against something other than
itself -- closed forms, library routines (numpy / scipy), brute force and the
published Lloyd-Max table -- chosen so that a dropped term, a wrong sign or
index, or a transposed operand fails at least one of them.

Sources: HARP (gist.science paper 2605.29843) sections 1, 2.1, 2.2, 5;
PolarQuant (gist.science paper 2603.29078) sections 1 and 2.
"""

import math
import os

import numpy as np
import pytest

import oracle
from rotation_preconditioned_bit_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def rand_orth(b, rng):
    q, r = np.linalg.qr(rng.standard_normal((b, b)))
    return q * np.sign(np.diag(r))


def sylvester_closed_form(d):
    i = np.arange(d)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0) / math.sqrt(d)


def hadamard_processor(radix, signs=None):
    d = int(np.prod(radix))
    blocks = [np.broadcast_to(oracle.sylvester(b), (d // b, b, b)) for b in radix]
    return oracle.Processor(radix, blocks, signs)


def random_processor(radix, rng, signs=True, identical=False):
    d = int(np.prod(radix))
    blocks = []
    for b in radix:
        if identical:
            blocks.append(np.broadcast_to(rand_orth(b, rng), (d // b, b, b)))
        else:
            blocks.append(np.stack([rand_orth(b, rng) for _ in range(d // b)]))
    s = rng.choice([-1.0, 1.0], size=d) if signs else None
    return oracle.Processor(radix, blocks, s)


def tensor_axis_apply(P, x):
    """Independent statement of the stages: view x as a tensor with axes
    (b_0, ..., b_{m-1}) in C order (axis 0 is the largest stride); stage t
    multiplies along axis t, with the block chosen by the flattened index of
    the other axes (in order)."""
    radix = [int(b) for b in P.radix]
    v = x * (P.signs if P.signs is not None else 1.0)
    T = v.reshape(radix)
    for t, b in enumerate(radix):
        blk = P.stage_blocks(t)                       # [d/b, b, b]
        moved = np.moveaxis(T, t, -1)                 # other axes first, in order
        shp = moved.shape
        flat = moved.reshape(-1, b)                   # row index = group c
        out = np.einsum("ckj,cj->ck", blk, flat)
        T = np.moveaxis(out.reshape(shp), -1, t)
    return T.reshape(-1)


# ------------------------------------------------------------ block makers

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64])
def test_sylvester_closed_form(b):
    np.testing.assert_allclose(oracle.sylvester(b), sylvester_closed_form(b), atol=1e-15)


@pytest.mark.parametrize("b", [2, 3, 5, 7, 16, 43])
def test_qr_q_matches_library_with_positive_r(b):
    G = RNG.standard_normal((b, b))
    Q = oracle.qr_q(G)
    q, r = np.linalg.qr(G)
    ref = q * np.sign(np.diag(r))
    np.testing.assert_allclose(Q, ref, atol=1e-11)
    np.testing.assert_allclose(Q.T @ Q, np.eye(b), atol=1e-13)
    R = Q.T @ G
    assert np.all(np.diag(R) > 0)
    np.testing.assert_allclose(np.tril(R, -1), 0.0, atol=1e-11)


@pytest.mark.parametrize("b", [3, 8, 16])
def test_cayley_matches_library_solve(b):
    import scipy.linalg
    g = RNG.standard_normal((b, b))
    A = 0.3 * (np.triu(g, 1) - np.triu(g, 1).T)
    Q = oracle.cayley(A)
    ref = scipy.linalg.solve(np.eye(b) - A, np.eye(b) + A)
    np.testing.assert_allclose(Q, ref, atol=1e-12)
    np.testing.assert_allclose(Q.T @ Q, np.eye(b), atol=1e-12)
    np.testing.assert_allclose(oracle.cayley(np.zeros((b, b))), np.eye(b), atol=0)
    # first-order behaviour: Q = I + 2A + O(A^2)
    eps = 1e-6
    np.testing.assert_allclose((oracle.cayley(eps * A) - np.eye(b)) / eps, 2 * A, atol=1e-5)


def test_givens():
    np.testing.assert_allclose(oracle.givens(0.0), np.eye(2), atol=0)
    a = 0.37
    Q = oracle.givens(a)
    np.testing.assert_allclose(Q @ np.array([1.0, 0.0]), [math.cos(a), math.sin(a)], atol=1e-15)
    np.testing.assert_allclose(np.linalg.det(Q), 1.0, atol=1e-15)


def test_stage_blocks_kinds():
    b, n = 8, 5
    g = RNG.standard_normal((n, b, b))
    had = oracle.stage_blocks("hadamard", b, n)
    np.testing.assert_allclose(had, np.broadcast_to(sylvester_closed_form(b), (n, b, b)), atol=1e-15)
    # theta = 0 gives back the base mixer exactly (HARP 2.2 initialisation)
    zero = oracle.stage_blocks("cayley_hadamard", b, n, g, None, 0.0)
    np.testing.assert_allclose(zero, had, atol=0)
    qr = oracle.stage_blocks("qr", b, n, g)
    for c in range(n):
        q, r = np.linalg.qr(g[c])
        np.testing.assert_allclose(qr[c], q * np.sign(np.diag(r)), atol=1e-12)
    cay = oracle.stage_blocks("cayley_hadamard", b, n, g, None, 0.05)
    for c in range(n):
        A = 0.05 * (np.triu(g[c], 1) - np.triu(g[c], 1).T)
        ref = np.linalg.solve(np.eye(b) - A, np.eye(b) + A) @ sylvester_closed_form(b)
        np.testing.assert_allclose(cay[c], ref, atol=1e-12)
    # non-power-of-two base mixer: Q of the stage's fixed Gaussian
    base = RNG.standard_normal((5, 5))
    had5 = oracle.stage_blocks("hadamard", 5, 3, None, base)
    q, r = np.linalg.qr(base)
    np.testing.assert_allclose(had5[1], q * np.sign(np.diag(r)), atol=1e-12)
    # b = 2 uses a Givens rotation by skew_scale * g[0][1]
    g2 = RNG.standard_normal((1, 2, 2))
    cg = oracle.stage_blocks("cayley_hadamard", 2, 1, g2, None, 0.5)
    np.testing.assert_allclose(cg[0], oracle.givens(0.5 * g2[0, 0, 1]) @ sylvester_closed_form(2),
                               atol=1e-15)


# ------------------------------------------------------------ int8-stored parameters

def test_theta_quantize_reading():
    theta = 0.05 * RNG.standard_normal(1000)
    theta[17] = -0.4                                  # the stage's absmax
    q, s = oracle.theta_quantize(theta)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert s == np.float32(0.4 / 127)
    assert q[17] == -127 and np.abs(q).max() == 127
    # round to nearest: every stored value within half a step of the original
    assert np.all(np.abs(theta - np.float64(s) * q) <= 0.5 * np.float64(s) * (1 + 1e-12))
    q0, s0 = oracle.theta_quantize(np.zeros(12))
    assert s0 == 0 and not q0.any()


def _skew_from_upper(b, vals):
    """Skew-symmetric matrix whose strict upper triangle, read row by row, is
    vals (numpy's triu_indices order)."""
    A = np.zeros((b, b))
    iu = np.triu_indices(b, 1)
    A[iu] = vals
    return A - A.T


@pytest.mark.parametrize("b", [3, 4, 16, 32])
def test_theta_blocks_cayley_against_library_solve(b):
    n, P = 4, b * (b - 1) // 2
    q = RNG.integers(-127, 128, size=(n, P)).astype(np.int8)
    scale = np.float32(0.002)
    if (b & (b - 1)) == 0:
        G = sylvester_closed_form(b)
        B = oracle.theta_blocks(b, q, scale)
    else:
        G = np.linalg.qr(RNG.standard_normal((b, b)))[0]
        B = oracle.theta_blocks(b, q, scale, G)
    for c in range(n):
        A = _skew_from_upper(b, np.float64(scale) * q[c].astype(np.float64))
        ref = np.linalg.solve(np.eye(b) - A, np.eye(b) + A) @ G
        np.testing.assert_allclose(B[c], ref, atol=1e-13)
        np.testing.assert_allclose(B[c].T @ B[c], np.eye(b), atol=1e-13)
    # a single nonzero generator entry (0, 2): A = a(E02 - E20); the Cayley map
    # of a plane rotation generator is the rotation by 2 atan(a) in that plane
    qs = np.zeros((1, P), np.int8)
    qs[0, 1] = 100
    a = np.float64(scale) * 100
    R = np.eye(b)
    phi = 2 * math.atan(a)
    R[0, 0] = R[2, 2] = math.cos(phi)
    R[0, 2], R[2, 0] = math.sin(phi), -math.sin(phi)      # A[0][2] = +a
    Gp = None if (b & (b - 1)) == 0 else G
    np.testing.assert_allclose(oracle.theta_blocks(b, qs, scale, Gp)[0], R @ G, atol=1e-14)


def test_theta_blocks_zero_givens_and_trivial():
    # theta = 0 gives back the base mixer exactly (HARP 2.2 initialisation)
    for b in (2, 8, 16, 64):
        P = max(b * (b - 1) // 2, 1)
        Z = oracle.theta_blocks(b, np.zeros((3, P), np.int8), np.float32(0.01))
        np.testing.assert_array_equal(Z, np.broadcast_to(sylvester_closed_form(b), (3, b, b)))
    # b = 2: Givens rotation by scale * q times H_2, closed form
    q = np.array([[37], [-128], [0]], np.int8)
    s = np.float32(0.01)
    B = oracle.theta_blocks(2, q, s)
    for c in range(3):
        a = np.float64(s) * int(q[c, 0])
        ca, sa = math.cos(a), math.sin(a)
        ref = np.array([[ca - sa, ca + sa], [sa + ca, sa - ca]]) / math.sqrt(2)
        np.testing.assert_allclose(B[c], ref, atol=1e-15)
    # b = 1: every block is [1] (no parameters)
    np.testing.assert_array_equal(oracle.theta_blocks(1, np.zeros((5, 0), np.int8), s),
                                  np.ones((5, 1, 1)))


# ------------------------------------------------------------ processor

@pytest.mark.parametrize("radix", [(16, 16), (2, 4, 8), (4, 4, 4, 4), (256,), (2,) * 8])
def test_hadamard_blocks_with_signs_equal_sylvester_rht(radix):
    """HARP 2.2: theta = 0 recovers the fixed RHT; with power-of-two radices
    the product of Sylvester stages is exactly the Sylvester H_d (closed form
    (-1)^popcount(i & j) / sqrt(d)), applied after the random signs."""
    d = int(np.prod(radix))
    s = synth.signs(0, synth.S_SIGNS_R, d).astype(np.float64)
    P = hadamard_processor(radix, s)
    M = P.dense()
    np.testing.assert_allclose(M, sylvester_closed_form(d) * s[None, :], atol=1e-13)
    x = RNG.standard_normal(d)
    np.testing.assert_allclose(P.apply(x), sylvester_closed_form(d) @ (s * x), atol=1e-12)


def test_hadamard_rht_large_d():
    radix = (8, 8, 8, 8)
    d = 4096
    s = synth.signs(3, synth.S_SIGNS_R, d).astype(np.float64)
    P = hadamard_processor(radix, s)
    X = RNG.standard_normal((3, d))
    H = sylvester_closed_form(d)
    np.testing.assert_allclose(P.rotate_rows(X), (X * s) @ H.T, atol=1e-12)


@pytest.mark.parametrize("radix", [(16, 16), (4, 8, 2)])
def test_hadamard_without_signs_is_involution(radix):
    """PolarQuant 2: H^-1 = H for the normalised Walsh-Hadamard matrix."""
    P = hadamard_processor(radix)
    x = RNG.standard_normal(int(np.prod(radix)))
    np.testing.assert_allclose(P.apply(P.apply(x)), x, atol=1e-13)


@pytest.mark.parametrize("radix", [(2, 3, 5), (3, 7), (5, 2, 4), (7, 16), (3, 3, 3)])
def test_identical_blocks_give_kronecker_product(radix):
    """With the same (non-symmetric) block in every group of a stage, the
    processor is the Kronecker product B_0 x B_1 x ... x B_{m-1} times D
    (stage 0 acts on the most significant digit)."""
    P = random_processor(radix, RNG, identical=True)
    K = np.array([[1.0]])
    for t in range(len(radix)):
        K = np.kron(K, P.stage_blocks(t)[0])
    np.testing.assert_allclose(P.dense(), K * P.signs[None, :], atol=1e-13)


@pytest.mark.parametrize("radix", [(2, 3, 5), (4, 3), (3, 3, 3), (7, 4, 2), (16, 16), (5, 8)])
def test_stage_loop_matches_tensor_axis_statement(radix):
    P = random_processor(radix, RNG)
    for _ in range(3):
        x = RNG.standard_normal(P.d)
        np.testing.assert_allclose(P.apply(x), tensor_axis_apply(P, x), atol=1e-13)


@pytest.mark.parametrize("radix", [(2, 3, 5), (16, 16), (7, 4, 2)])
def test_dense_matches_loop_and_is_orthogonal(radix):
    P = random_processor(radix, RNG)
    M = P.dense()
    E = np.eye(P.d)
    cols = np.stack([P.apply(E[i]) for i in range(P.d)], axis=1)
    np.testing.assert_allclose(M, cols, atol=1e-13)
    np.testing.assert_allclose(M.T @ M, np.eye(P.d), atol=1e-12)
    inv_cols = np.stack([P.apply(E[i], inverse=True) for i in range(P.d)], axis=1)
    np.testing.assert_allclose(inv_cols, M.T, atol=1e-13)


@pytest.mark.parametrize("radix", [(16, 16, 16), (43, 16, 16), (7, 16, 16, 16), (32, 16, 16),
                                   (8, 8, 8, 5, 2)])
def test_norm_preservation_and_inverse(radix):
    """HARP 1 and 5: an exact orthogonal change of basis; ||Mx|| = ||x|| and
    inverse(forward(x)) = x to 1e-12 with float64 blocks."""
    P = random_processor(radix, RNG)
    x = RNG.standard_normal(P.d)
    y = P.apply(x)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-12 * np.linalg.norm(x)
    np.testing.assert_allclose(P.apply(y, inverse=True), x, atol=1e-12)


def test_mixed_radix_schedules_from_the_pages():
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "harp_mixed_radix_schedules.txt"))
            if ln.strip() and not ln.startswith("#")]
    for r in rows:
        d, radix = r[0], tuple(r[1:])
        assert int(np.prod(radix)) == d
    d, radix = rows[0][0], tuple(rows[0][1:])
    assert (d, radix) == (5120, (8, 8, 8, 5, 2))
    side = synth.side_draws(9, radix, "cayley_hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R, 0.05)
    P = oracle.processor(side)
    x = RNG.standard_normal(d)
    np.testing.assert_allclose(P.apply(P.apply(x), inverse=True), x, atol=1e-12)
    side0 = synth.side_draws(9, radix, "cayley_hadamard", synth.S_SIGNS_R, synth.S_BLOCKS_R, 0.0)
    P0 = oracle.processor(side0)
    # theta = 0: every block equals the base mixer of its radix
    for t, b in enumerate(radix):
        np.testing.assert_allclose(P0.stage_blocks(t)[7], P0.stage_blocks(t)[0], atol=0)


def test_rows_and_cols_sides():
    Pr = random_processor((4, 3), RNG)
    Pl = random_processor((2, 5), RNG)
    X = RNG.standard_normal((10, 12))
    Mr, Ml = Pr.dense(), Pl.dense()
    np.testing.assert_allclose(Pr.rotate_rows(X), X @ Mr.T, atol=1e-13)
    np.testing.assert_allclose(Pl.rotate_cols(X), Ml @ X, atol=1e-13)
    np.testing.assert_allclose(Pr.rotate_rows(X, inverse=True), X @ Mr, atol=1e-13)
    np.testing.assert_allclose(Pl.rotate_cols(X, inverse=True), Ml.T @ X, atol=1e-13)


def test_sampled_two_sided_rows():
    Pr = random_processor((4, 2, 3), RNG)
    Pl = random_processor((3, 5), RNG)
    W = RNG.standard_normal((15, 24))
    full = Pl.rotate_cols(Pr.rotate_rows(W))
    which = np.array([0, 7, 14, 3])
    np.testing.assert_allclose(oracle.two_sided_rows(W, Pl, Pr, which), full[which], atol=1e-13)
    np.testing.assert_allclose(oracle.two_sided_rows(W, None, Pr, which), Pr.rotate_rows(W)[which],
                               atol=1e-13)
    inv = Pl.rotate_cols(Pr.rotate_rows(full, inverse=True), inverse=True)
    np.testing.assert_allclose(oracle.inverse_rows(full, Pl, Pr, which), inv[which], atol=1e-13)
    np.testing.assert_allclose(inv, W, atol=1e-12)


def test_processor_from_workload_draws():
    w = synth.workload("c1")
    P = oracle.processor(w.right)
    M = P.dense()
    np.testing.assert_allclose(M, sylvester_closed_form(256) * w.right.signs[None, :].astype(np.float64),
                               atol=1e-13)


# ------------------------------------------------------------ Lloyd-Max

def _golden_lloyd_max():
    out = {}
    for ln in open(os.path.join(GOLDEN, "max1960_gaussian_lloyd_max.txt")):
        if ln.strip() and not ln.startswith("#"):
            v = ln.split()
            # tolerance per level: half a unit of the printed last digit plus
            # the 1e-4 error Max's table is known to carry
            tol = np.array([0.5 * 10.0 ** -len(a.split(".")[1]) + 1e-4 for a in v[2:]])
            out[int(v[0])] = (float(v[1]), np.array([float(a) for a in v[2:]]), tol)
    return out


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_max_matches_published_table(bits):
    mse_pub, levels, tol = _golden_lloyd_max()[bits]
    c, _ = oracle.lloyd_max(bits)
    K = 1 << bits
    assert np.all(np.abs(c[K // 2:] - levels) <= tol)
    assert np.all(np.abs(c[:K // 2] + levels[::-1]) <= tol[::-1])
    mse = _mse(c)
    assert abs(mse - mse_pub) < 2e-4 * max(1.0, mse_pub / 0.01)


def _mse(c):
    """E[(Z - Q(Z))^2] by adaptive quadrature (scipy), Q = nearest level."""
    from scipy import integrate
    K = c.size
    t = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    phi = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    return sum(integrate.quad(lambda z, k=k: (z - c[k]) ** 2 * phi(z), t[k], t[k + 1],
                              epsabs=1e-14, epsrel=1e-12)[0] for k in range(K))


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_lloyd_max_fixed_point_by_quadrature(bits):
    """PolarQuant 2: MSE-optimal centroids for N(0,1): every level is the
    conditional mean of its cell (checked by numerical integration, not the
    oracle's closed form) and the cells are bounded by midpoints."""
    from scipy import integrate
    c, _ = oracle.lloyd_max(bits)
    K = c.size
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(c, -c[::-1], atol=0)
    t = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    phi = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    for k in range(K):
        m0 = integrate.quad(phi, t[k], t[k + 1], epsabs=1e-15, epsrel=1e-13)[0]
        m1 = integrate.quad(lambda z: z * phi(z), t[k], t[k + 1], epsabs=1e-15, epsrel=1e-13)[0]
        assert abs(m1 / m0 - c[k]) < 1e-10
    # better than the best uniform quantiser with the same number of levels
    best_uniform = min(_mse((np.arange(K) - (K - 1) / 2) * step) for step in np.linspace(0.2, 1.5, 27))
    assert _mse(c) < best_uniform


# ------------------------------------------------------------ fp16 scales

def test_f16_rounding_matches_numpy():
    vals = np.concatenate([
        np.exp(RNG.uniform(np.log(1e-9), np.log(7e4), 4000)),
        [0.0, 6.103515625e-05, 6.0e-08, 5.96e-08, 2.98e-08, 65504.0, 65519.0, 1e9, 1.0, 0.1],
    ])
    # exact ties between neighbouring fp16 values must round to even
    h = RNG.integers(1, 0x7BFE, 500).astype(np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).view(np.float16).astype(np.float64)
    vals = np.concatenate([vals, 0.5 * (a + b)])
    for v in vals:
        got = oracle.f16_bits(v)
        with np.errstate(over="ignore"):
            ref = np.array(v, dtype=np.float64).astype(np.float16)
        if not np.isfinite(ref):
            assert got == 0x7BFF               # saturation reading
        else:
            assert got == int(ref.view(np.uint16)), v
            assert oracle.f16_value(got) == float(ref)


# ------------------------------------------------------------ quantiser

def _brute_nearest(z, levels):
    return np.argmin(np.abs(z[..., None] - levels[None, :]), axis=-1)


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (4, 128), (4, 32), (5, 128)])
def test_lloyd_max_codes_are_nearest_centroid(bits, group):
    X = synth.small_matrix(11 + bits, 16, 512, outlier_cols=3, scale=0.02)
    codes, scales, margin, smargin = oracle.quantize("lloyd_max", bits, group, X)
    c, _ = oracle.lloyd_max(bits)
    cent = c.astype(np.float32).astype(np.float64)
    s = np.repeat(np.array([[oracle.f16_value(v) for v in row] for row in scales]), group, axis=1)
    z = X / s
    brute = _brute_nearest(z, cent)
    safe = margin > 1e-9
    assert np.mean(safe) > 0.999
    np.testing.assert_array_equal(codes[safe], brute[safe])
    # scale = RMS of the group, rounded to fp16
    rms = np.sqrt((X.reshape(16, -1, group) ** 2).mean(axis=2))
    np.testing.assert_array_equal(scales, rms.astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (4, 128), (5, 128)])
def test_lloyd_max_absmax_scale_mode(bits, group):
    """The alternative Lloyd-Max scale (largest magnitude onto the outermost
    centroid): the stored scale is fp16(max|x| / c_{K-1}) computed with
    numpy; codes are still the nearest centroid of x/s (brute force); the
    group's largest-magnitude element gets an outermost code; the mode is
    refused for absmax codebooks."""
    X = synth.small_matrix(31 + bits, 12, 512, outlier_cols=3, scale=0.02)
    codes, scales, margin, smargin = oracle.quantize("lloyd_max", bits, group, X, scale_mode="absmax")
    c, _ = oracle.lloyd_max(bits)
    cent = c.astype(np.float32).astype(np.float64)
    K = 1 << bits
    amax = np.abs(X.reshape(12, -1, group)).max(axis=2)
    np.testing.assert_array_equal(scales, (amax / cent[-1]).astype(np.float16).view(np.uint16))
    s = np.repeat(np.array([[oracle.f16_value(v) for v in row] for row in scales]), group, axis=1)
    brute = _brute_nearest(X / s, cent)
    safe = margin > 1e-9
    assert np.mean(safe) > 0.999
    np.testing.assert_array_equal(codes[safe], brute[safe])
    Xg = X.reshape(12, -1, group)
    cg = codes.reshape(12, -1, group)
    im = np.argmax(np.abs(Xg), axis=2)
    for r in range(12):
        for g in range(Xg.shape[1]):
            i = im[r, g]
            assert cg[r, g, i] == (K - 1 if Xg[r, g, i] > 0 else 0)
    # differs from the default RMS reading
    codes0, scales0, _, _ = oracle.quantize("lloyd_max", bits, group, X)
    assert not np.array_equal(scales, scales0)
    with pytest.raises(ValueError):
        oracle.quantize("absmax", bits, group, X, scale_mode="absmax")


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_absmax_codes(bits):
    X = synth.small_matrix(21 + bits, 8, 256, outlier_cols=2)
    group = 128
    codes, scales, margin, _ = oracle.quantize("absmax", bits, group, X)
    qmax = (1 << (bits - 1)) - 1
    s = np.repeat(np.array([[oracle.f16_value(v) for v in row] for row in scales]), group, axis=1)
    xh = oracle.dequantize("absmax", bits, group, codes, scales)
    assert np.all(np.abs(X - xh) <= 0.5 * s * (1 + 1e-2))
    assert codes.min() >= 1 and codes.max() <= 2 * qmax + 1
    Xg = X.reshape(8, -1, group)
    cg = codes.reshape(8, -1, group).astype(int) - (1 << (bits - 1))
    amax = np.argmax(np.abs(Xg), axis=2)
    for r in range(8):
        for g in range(Xg.shape[1]):
            i = amax[r, g]
            assert cg[r, g, i] == int(np.sign(Xg[r, g, i])) * qmax
    ref = np.clip(np.rint(X / s), -qmax, qmax)
    safe = margin > 1e-9
    np.testing.assert_array_equal((codes.astype(int) - (1 << (bits - 1)))[safe], ref[safe])


def test_zero_group_and_dequantize():
    X = np.zeros((2, 256))
    X[1, 128:] = RNG.standard_normal(128)
    for kind, mid in (("lloyd_max", 4), ("absmax", 4)):
        codes, scales, _, _ = oracle.quantize(kind, 3, 128, X)
        assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
        assert np.all(codes[0] == mid) and np.all(codes[1, :128] == mid)
        xh = oracle.dequantize(kind, 3, 128, codes, scales)
        assert np.all(xh[0] == 0) and np.all(xh[1, :128] == 0)


def test_lloyd_max_dequantize_is_scaled_centroid():
    X = synth.small_matrix(5, 4, 128)
    codes, scales, _, _ = oracle.quantize("lloyd_max", 4, 128, X)
    c, _ = oracle.lloyd_max(4)
    xh = oracle.dequantize("lloyd_max", 4, 128, codes, scales)
    s = np.array([oracle.f16_value(v) for v in scales[:, 0]])
    np.testing.assert_array_equal(xh, s[:, None] * c.astype(np.float32).astype(np.float64)[codes])


# ------------------------------------------------------------ packing

@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_pack_matches_bitstream_brute_force(bits):
    cols = 64
    codes = RNG.integers(0, 1 << bits, (5, cols)).astype(np.uint8)
    packed = oracle.pack(bits, codes)
    assert packed.shape == (5, cols * bits // 8)
    for r in range(5):
        big = sum(int(v) << (bits * i) for i, v in enumerate(codes[r]))
        ref = np.frombuffer(big.to_bytes(cols * bits // 8, "little"), dtype=np.uint8)
        np.testing.assert_array_equal(packed[r], ref)
    np.testing.assert_array_equal(oracle.unpack(bits, packed, cols), codes)


def test_pack_known_bytes():
    # 4-bit: two codes per byte, first code in the low nibble
    np.testing.assert_array_equal(oracle.pack(4, np.array([[1, 2, 15, 0]], np.uint8)), [[0x21, 0x0F]])
    # 2-bit: four codes per byte, LSB first
    np.testing.assert_array_equal(oracle.pack(2, np.array([[1, 2, 3, 0]], np.uint8)), [[0b00111001]])
    # 3-bit: eight codes in three bytes
    codes = np.array([[7, 0, 1, 2, 3, 4, 5, 6]], np.uint8)
    big = sum(int(v) << (3 * i) for i, v in enumerate(codes[0]))
    np.testing.assert_array_equal(oracle.pack(3, codes)[0], list(big.to_bytes(3, "little")))


# ------------------------------------------------------------ round trip

def test_frobenius_invariant_two_sided():
    """HARP 5: an exact change of basis, so the quantisation error measured in
    the rotated basis equals the error after un-rotating."""
    Pr = random_processor((4, 2, 8), RNG)
    Pl = random_processor((3, 4), RNG)
    W = synth.small_matrix(3, 12, 64, outlier_cols=2, scale=0.02)
    Wp, codes, packed, scales, _, _ = oracle.rotate_quantize(W, Pl, Pr, "lloyd_max", 3, 32)
    Wph = oracle.dequantize("lloyd_max", 3, 32, codes, scales)
    Wh = oracle.dequantize_unrotate(codes, scales, Pl, Pr, "lloyd_max", 3, 32)
    e1 = np.linalg.norm(W - Wh)
    e2 = np.linalg.norm(Wp - Wph)
    assert abs(e1 - e2) <= 1e-10 * e2
    np.testing.assert_array_equal(oracle.unpack(3, packed, 64), codes)


def test_rotation_gaussianises_heavy_tails():
    """PolarQuant 2 (statistical sanity, not a parity pin): after the RHT the
    coordinates of heavy-tailed rows are close to Gaussian (kurtosis near 3)."""
    d = 1024
    x = 0.02 * synth.student_t(8, 3, 16 * d).reshape(16, d)
    s = synth.signs(8, synth.S_SIGNS_R, d).astype(np.float64)
    P = hadamard_processor((32, 32), s)
    y = P.rotate_rows(x)
    kx = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    ky = np.mean(y ** 4) / np.mean(y ** 2) ** 2
    assert kx > 6 and abs(ky - 3.0) < 0.5


# ------------------------------------------------------------ two-stage codec

def test_round_mid_against_library_casts():
    import torch
    x = np.concatenate([RNG.standard_normal(4000) * 10.0 ** RNG.integers(-6, 4, 4000),
                        [0.0, -0.0, 65504.0, -65504.0]]).astype(np.float32).astype(np.float64)
    f16 = oracle.round_mid("f16", x)
    np.testing.assert_array_equal(f16, x.astype(np.float16).astype(np.float64))
    # saturation past the largest fp16 (the reading used for the scales too)
    np.testing.assert_array_equal(oracle.round_mid("f16", np.array([1e6, -70000.0])), [65504.0, -65504.0])
    # bf16 from float32-representable values: one rounding, as torch's cast
    bf = oracle.round_mid("bf16", x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(bf, ref)
    # exact ties go to the even neighbour (8 significant bits)
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 3 * 2.0 ** -9 * 2.0 ** -7])
    np.testing.assert_array_equal(oracle.round_mid("bf16", ties)[:3], [1.0, 1 + 2.0 ** -6, -1.0])
    np.testing.assert_array_equal(oracle.round_mid("f32", x[:10] + 1e-12),
                                  (x[:10] + 1e-12).astype(np.float32).astype(np.float64))


def test_requantize_order_of_steps():
    """PolarQuant sections 2-3: first-stage codes are dequantised, rotated
    back (rows: r -> M^T r, i.e. X -> X M with the dense processor matrix),
    stored as fp16, then quantised by the second quantiser without rotation."""
    P = random_processor((8, 4, 4), RNG)
    d = P.d
    rows = 6
    X = synth.small_matrix(3, rows, d, outlier_cols=2)
    codes, scales, _, _ = oracle.quantize("lloyd_max", 5, 128, P.rotate_rows(X))
    Y, c2, packed, s2, margin, _ = oracle.requantize(codes, scales, P, "lloyd_max", 5, 128,
                                                     "f16", "absmax", 4, 64)
    Xh = oracle.dequantize("lloyd_max", 5, 128, codes, scales)
    np.testing.assert_allclose(Y, (Xh @ P.dense()).astype(np.float16), rtol=1e-3, atol=1e-6)
    np.testing.assert_array_equal(Y, Y.astype(np.float16).astype(np.float64))
    # the second stage is plain absmax on the restored fp16 weights
    s = np.repeat(np.array([[oracle.f16_value(v) for v in r] for r in s2]), 64, axis=1)
    Yg = np.abs(Y).reshape(rows, -1, 64).max(axis=2)
    np.testing.assert_allclose(s[:, ::64], Yg / 7, rtol=1e-3)
    assert np.all(np.abs(Y - s * (c2.astype(int) - 8)) <= 0.5 * s * (1 + 1e-2))
    np.testing.assert_array_equal(packed, oracle.pack(4, c2))
