"""Pins for the CPU oracle: each test checks the oracle against something other than itself
(values published for the method or its building blocks, closed forms, invariants the pages
state, library routines the oracle does not call, or brute force on tiny inputs)."""
import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats
import torch

import oracle as O
from tests.conftest import golden_path


def _read_rows(name):
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


# ------------------------------------------------------------------ random numbers
def test_splitmix64_reference_vectors():
    want = [int(r, 16) for r in _read_rows("splitmix64_seed0.txt")]
    assert O.splitmix64(0, 5) == want


def test_splitmix64_first_output_matches_independent_implementation():
    # numba's xoroshiro128+ seeding runs one SplitMix64 step (its own code, not ours).
    from numba.cuda.random import init_xoroshiro128p_states_cpu, xoroshiro128p_dtype
    st = np.zeros(1, dtype=xoroshiro128p_dtype)
    for seed in (0, 1, 12345, 987654321, 2**62 + 7):
        init_xoroshiro128p_states_cpu(st, seed, 0)
        assert int(st["s0"][0]) == O.splitmix64(seed, 1)[0]


def test_rotation_signs_are_balanced_and_d_bits():
    # d bits of storage (16 bytes at d=128, "What the Paper Doesn't Tell You", Finding 4);
    # a fair generator gives about half -1.
    s = np.concatenate([O.rotation_signs(seed, 128) for seed in range(200)])
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(np.mean(s == -1.0) - 0.5) < 0.01
    w = O.splitmix64(7, 2)
    s7 = O.rotation_signs(7, 128)
    bits = [(w[i // 64] >> (i % 64)) & 1 for i in range(128)]
    assert np.array_equal(s7 == -1.0, np.array(bits) == 1)


def test_qjl_matrix_is_standard_gaussian():
    s = O.qjl_matrix(1, 64, 64).ravel()
    assert s.dtype == np.float64
    assert np.array_equal(s, s.astype(np.float32).astype(np.float64))
    ks = scipy.stats.kstest(s, "norm")
    assert ks.pvalue > 1e-3
    assert abs(s.mean()) < 0.05 and abs(s.var() - 1.0) < 0.06
    assert not np.array_equal(O.qjl_matrix(1, 8, 16), O.qjl_matrix(2, 8, 16))


# ------------------------------------------------------------------ rotation
@pytest.mark.parametrize("d", [8, 16, 64, 128, 256])
def test_hadamard_matches_sylvester_construction(d):
    assert np.array_equal(O.hadamard(d), scipy.linalg.hadamard(d).astype(np.float64))


@pytest.mark.parametrize("d", [16, 64, 128])
def test_rotation_preserves_norms_and_inner_products(d):
    # "The rotation preserves inner products perfectly" (Three-Step Summary, Step 1).
    rng = np.random.default_rng(d)
    x, y = rng.standard_normal((2, 50, d))
    rx, ry = O.rotate(x, 3), O.rotate(y, 3)
    assert np.allclose(np.linalg.norm(rx, axis=1), np.linalg.norm(x, axis=1), rtol=0, atol=1e-6)
    assert np.allclose(np.sum(rx * ry, 1), np.sum(x * y, 1), rtol=0, atol=1e-6)
    assert np.allclose(O.inverse_rotate(rx, 3), x, atol=1e-12)


def test_rotation_applies_signs_before_transform():
    # R e_0 = H D e_0 / sqrt(d) = D_00 * (first column of H) / sqrt(d): constant entries.
    d = 64
    e0 = np.zeros((1, d))
    e0[0, 0] = 1.0
    r = O.rotate(e0, 5)[0]
    assert np.allclose(r, O.rotation_signs(5, d)[0] / math.sqrt(d))
    # and R^T e_0 = D H e_0 / sqrt(d) carries the sign pattern
    assert np.allclose(O.inverse_rotate(e0, 5)[0], O.rotation_signs(5, d) / math.sqrt(d))


def test_rotation_gaussianises_heavy_tailed_inputs():
    # "kurtosis 900 -> 2.9" on real KV tensors ("What the Paper Doesn't Tell You",
    # Finding 4). Synthetic stand-in: dense Gaussian vectors with 4 channels x3 and a
    # log-normal per-token scale (raw kurtosis > 100). Dividing by the norm alone leaves the
    # channel outliers (kurtosis > 5); after the rotation z = H D x / ||x|| the coordinates
    # behave like those of a random point on the sphere of radius sqrt(d), whose kurtosis is
    # 3 d / (d + 2) = 2.95 at d = 128.
    rng = np.random.default_rng(0)
    d = 128
    x = rng.standard_normal((4000, d))
    x[:, rng.permutation(d)[:4]] *= 3.0
    x *= np.exp(rng.standard_normal((4000, 1)))
    raw = scipy.stats.kurtosis(x.ravel(), fisher=False)
    unrot = x / np.linalg.norm(x, axis=1, keepdims=True) * math.sqrt(d)
    rec = O.quantize(x, 4)
    rot = scipy.stats.kurtosis(rec.z.ravel(), fisher=False)
    assert raw > 100.0
    assert scipy.stats.kurtosis(unrot.ravel(), fisher=False) > 5.0
    assert abs(rot - 3.0 * d / (d + 2)) < 0.1
    assert np.allclose(np.sum(rec.z ** 2, axis=1), d)


# ------------------------------------------------------------------ Lloyd-Max codebook
def test_codebook_matches_max_table():
    for row in _read_rows("max1960_gaussian_quantizer.txt"):
        parts = row.split()
        bits, kind, vals = int(parts[0]), parts[1], [float(v) for v in parts[2:]]
        c, _, dist = O.lloyd_max_gaussian(bits)
        if kind == "centroid":
            half = c[len(c) // 2:]
            assert np.allclose(half, vals, atol=1.5e-4), (bits, half, vals)
            assert np.allclose(c[: len(c) // 2], -half[::-1], atol=1e-12)
        else:
            assert abs(dist - vals[0]) / vals[0] < 2e-3, (bits, dist, vals)


def test_boundary_distance_against_published_boundaries():
    # The decision boundaries are the midpoints of adjacent optimum levels; Max's table (four
    # decimals) fixes them to within 1e-4. Coordinates placed at a published boundary plus a
    # small offset must report that offset; a record without Lloyd-Max codes reports +inf.
    import dataclasses
    pub = {}
    for row in _read_rows("max1960_gaussian_quantizer.txt"):
        parts = row.split()
        if parts[1] == "centroid":
            half = [float(v) for v in parts[2:]]
            full = [-v for v in half[::-1]] + half
            pub[int(parts[0])] = [(a + b) / 2 for a, b in zip(full[:-1], full[1:])]
    base = O.quantize(np.ones((1, 8)), 4)
    for bits, beta in pub.items():
        offsets = np.array([0.003, -0.004, 0.01, -0.02])
        z = (np.asarray(beta)[:, None] + offsets[None, :]).reshape(1, -1)
        rec = dataclasses.replace(base, bits=bits, mode=O.MSE, z=z)
        got = O.boundary_distance(rec)
        want = np.broadcast_to(np.abs(offsets), (len(beta), len(offsets))).reshape(1, -1)
        assert np.all(np.abs(got - want) <= 2e-4), (bits, got, want)
        # half-way between two neighbouring boundaries: half the gap
        if len(beta) > 1:
            mid = np.array([[(beta[1] + beta[2]) / 2 if len(beta) > 2 else (beta[0] + beta[1]) / 2]])
            gap = (beta[2] - beta[1]) / 2 if len(beta) > 2 else (beta[1] - beta[0]) / 2
            got_mid = O.boundary_distance(dataclasses.replace(base, bits=bits, mode=O.MSE, z=mid))
            assert abs(got_mid[0, 0] - gap) <= 2e-4
    # TurboQuant_prod at 2 bits decides with the 1-bit codebook (boundary 0 only)
    z = np.array([[0.9, -0.25, 1e-6]])
    got = O.boundary_distance(dataclasses.replace(base, bits=2, mode=O.PROD, z=z))
    assert np.allclose(got, [[0.9, 0.25, 1e-6]], atol=1e-12)
    # 1-bit TurboQuant_prod stores no Lloyd-Max codes: nothing to exempt
    got = O.boundary_distance(dataclasses.replace(base, bits=1, mode=O.PROD, z=z))
    assert np.all(np.isinf(got)) and got.shape == z.shape


def test_codebook_one_bit_closed_form():
    c, beta, dist = O.lloyd_max_gaussian(1)
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-12)
    assert abs(beta[0]) < 1e-15
    assert abs(dist - (1 - 2 / math.pi)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_optimality_conditions_by_quadrature(bits):
    # each centroid is the conditional mean of its cell (checked by numerical integration,
    # not by the oracle's closed-form pdf/cdf), and boundaries are midpoints
    c, beta, dist = O.lloyd_max_gaussian(bits)
    edges = np.concatenate([[-np.inf], beta, [np.inf]])
    assert np.allclose(beta, (c[:-1] + c[1:]) / 2, atol=1e-15)
    pdf = scipy.stats.norm.pdf
    mse = 0.0
    for j in range(len(c)):
        mass = scipy.integrate.quad(pdf, edges[j], edges[j + 1])[0]
        mean = scipy.integrate.quad(lambda t: t * pdf(t), edges[j], edges[j + 1])[0] / mass
        assert abs(mean - c[j]) < 1e-8
        mse += scipy.integrate.quad(lambda t: (t - c[j]) ** 2 * pdf(t), edges[j], edges[j + 1])[0]
    assert abs(mse - dist) < 1e-8


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_distortion_monte_carlo_and_information_bound(bits):
    # Monte Carlo MSE on N(0,1) within 2% of the analytic value; and the pages' guarantee
    # "within 2.72x of the information-theoretic limit" (Three-Step Summary, Step 2):
    # 4^-b <= D_b <= (sqrt(3) pi / 2) 4^-b, with sqrt(3) pi / 2 = 2.7207.
    c, beta, dist = O.lloyd_max_gaussian(bits)
    z = np.random.default_rng(bits).standard_normal(400_000)
    q = c[np.argmin(np.abs(z[:, None] - c[None, :]), axis=1)]
    mc = np.mean((z - q) ** 2)
    assert abs(mc - dist) / dist < 0.02
    assert 4.0 ** -bits <= dist <= (math.sqrt(3) * math.pi / 2) * 4.0 ** -bits
    assert abs(math.sqrt(3) * math.pi / 2 - 2.72) < 1e-3


def _gaussian_mse(levels):
    """MSE of nearest-level quantisation of N(0,1) by numerical integration over the cells."""
    levels = np.sort(np.asarray(levels, dtype=np.float64))
    edges = np.concatenate([[-np.inf], (levels[1:] + levels[:-1]) / 2, [np.inf]])
    pdf = scipy.stats.norm.pdf
    return sum(scipy.integrate.quad(lambda t: (t - l) ** 2 * pdf(t), edges[j], edges[j + 1])[0]
               for j, l in enumerate(levels))


def test_e2m1_grid_cannot_hold_the_four_bit_codebook():
    # The open question of mapping the Lloyd-Max centroids onto Blackwell's FP4 (E2M1) format
    # ("Where This Fits in the Inference Stack", Blackwell FP4). E2M1 holds 0, 0.5, 1, 1.5, 2,
    # 3, 4, 6 and their negatives (15 values); a per-block scale s only stretches the grid.
    c, _, dist = O.lloyd_max_gaussian(4)
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6.0])
    grid = np.unique(np.concatenate([-e2m1, e2m1]))
    assert grid.size == 15
    # (1) as a quantiser, the best stretched grid has a third more MSE than Lloyd-Max
    scales = np.linspace(0.3, 0.8, 201)
    mses = np.array([_gaussian_mse(grid * s) for s in scales])
    best = mses.min()
    assert abs(_gaussian_mse(c) - dist) < 1e-8
    assert best > 1.30 * dist and 0.45 < scales[mses.argmin()] < 0.52
    # ... and breaks the pages' guarantee D_b <= (sqrt(3) pi / 2) 4^-b (Three-Step Summary)
    assert best > (math.sqrt(3) * math.pi / 2) * 4.0 ** -4 > dist
    # (2) keeping the codes and moving each centroid to the nearest stretched E2M1 value merges
    # two pairs of levels and moves some centroid by more than 0.1 at every scale
    for s in scales:
        mapped = (grid * s)[np.abs(c[:, None] - (grid * s)[None, :]).argmin(axis=1)]
        assert np.unique(mapped).size < 16
        assert np.abs(mapped - c).max() > 0.1


def test_e2m1_codebook_is_the_mse_optimal_stretch_of_the_fp4_grid():
    # The E2M1 reading of the FP4 question ("Where This Fits in the Inference Stack", Blackwell
    # FP4): 16 ascending levels s * grid with both zeros, the stretch s minimising the Gaussian
    # MSE, boundaries at the midpoints.
    c, beta, dist, s = O.e2m1_codebook()
    # (1) the levels are the OCP E2M1 values, decoded from their bit patterns by the format
    #     definition (sign, 2-bit exponent with bias 1, 1-bit mantissa), times s, and the code
    #     order maps onto the bit patterns one to one
    bits = O.code_to_e2m1(np.arange(16))
    assert sorted(bits.tolist()) == list(range(16))
    vals = np.array([O.e2m1_value(int(b)) for b in bits])
    assert np.array_equal(np.sign(vals) * np.abs(vals), np.array(
        [-6, -4, -3, -2, -1.5, -1, -0.5, -0.0, 0.0, 0.5, 1, 1.5, 2, 3, 4, 6]))
    assert np.signbit(vals[7]) and not np.signbit(vals[8])
    assert np.array_equal(c, vals * s)
    assert np.allclose(beta, (c[1:] + c[:-1]) / 2) and beta[7] == 0.0
    # (2) its MSE is the numerically integrated one, and s is the minimiser: a dense scan of
    #     the stretch (scipy quadrature, independent of the oracle's closed-form moments) finds
    #     nothing lower, and moving s either way raises the MSE
    assert abs(_gaussian_mse(c) - dist) < 1e-9
    scan = [(_gaussian_mse(vals * t), t) for t in np.linspace(0.45, 0.52, 71)]
    assert min(scan)[0] >= dist - 1e-9 and abs(min(scan)[1] - s) < 1e-3
    for ds in (-1e-3, 1e-3):
        assert _gaussian_mse(vals * (s + ds)) > dist
    # (3) a third more distortion than the 4-bit Lloyd-Max codebook (the CPU study above)
    assert 1.33 < dist / O.lloyd_max_gaussian(4)[2] < 1.34


def test_e2m1_quantise_takes_the_zero_of_each_sign_and_dequantises_on_the_grid():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((200, 64))
    x[0] = 0.0
    rec = O.quantize(x, 4, O.E2M1, seed=3)
    c, beta, _, _ = O.e2m1_codebook()
    z = rec.z
    # brute force: a nearest level of each coordinate, with the zero of z's sign
    dist = np.abs(z[:, :, None] - c[None, None, :])
    assert np.all(np.take_along_axis(dist, rec.codes[:, :, None], axis=2)[:, :, 0] <= dist.min(axis=2) + 1e-15)
    small = np.abs(z) < beta[8]
    assert np.all(rec.codes[small & (z > 0)] == 8) and np.all(rec.codes[small & (z < 0)] == 7)
    assert np.all(rec.codes[0] == 7)  # the zero vector: z = 0 takes the lower zero
    # the record is a 4-bit MSE record laid out the same way
    assert rec.packed.shape == (200, 32) and O.record_bytes(64, 4, O.E2M1) == O.record_bytes(64, 4, O.MSE)
    # dequantisation: norm * D H (c[code]) / d, against the explicit inverse of H D
    xh = O.dequantize(rec)
    hd = O.hadamard(64) * O.rotation_signs(3, 64)[None, :]
    want = rec.norm16.astype(np.float64)[:, None] * np.linalg.solve(hd, c[rec.codes].T).T
    assert np.allclose(xh, want, atol=1e-12)
    with pytest.raises(ValueError):
        O.quantize(x, 3, O.E2M1)


def test_codebook_scales_with_inverse_sqrt_d():
    # "codebook centroids scale with 1/sqrt(d) for your specific head dimension"
    for d in (64, 128):
        c, beta = O.codebook(3, d)
        c0, beta0, _ = O.lloyd_max_gaussian(3)
        assert np.allclose(c * math.sqrt(d), c0) and np.allclose(beta * math.sqrt(d), beta0)


# ------------------------------------------------------------------ packing and sizes
def test_packing_hand_worked_examples():
    for row in _read_rows("pack_3bit_d8.txt"):
        left, right = row.split("|")
        nums = [int(v) for v in left.split()]
        width, d, codes = nums[0], nums[1], nums[2:]
        want = bytes(int(v, 16) for v in right.split())
        got = O.pack_bits(np.array([codes]), width)
        assert got.tobytes() == want
        assert np.array_equal(O.unpack_bits(got, width, d)[0], codes)


@pytest.mark.parametrize("width", [1, 2, 3, 4])
def test_packing_round_trip(width):
    rng = np.random.default_rng(width)
    v = rng.integers(0, 1 << width, size=(33, 128))
    p = O.pack_bits(v, width)
    assert p.shape == (33, 128 * width // 8)
    assert np.array_equal(O.unpack_bits(p, width, 128), v)


def test_three_and_a_half_bit_reading_of_the_headline_rate():
    # "3.5 bits per coordinate ... 4.6x over FP16" (One-Slide Version; Finding 3) read as 4-bit
    # keys and 3-bit values: 3.5 code bits per cached coordinate, 16 / 3.5 = 4.57x on the codes
    # alone, 4.41x with the fp16 norms of both records
    d = 128
    code_bits = (O.code_bytes(d, 4, O.MSE) + O.code_bytes(d, 3, O.MSE)) * 8
    assert code_bits / (2 * d) == 3.5
    assert round(2 * d * 16 / code_bits, 1) == 4.6
    rec = O.record_bytes(d, 4, O.MSE) + O.record_bytes(d, 3, O.MSE)
    assert rec == 116 and 4.4 < 2 * d * 2 / rec < 4.42


def test_record_sizes_match_published_compression_ratios():
    # "3 bits ... (block_size=128: 5.12x)", "4 bits ... ~4x" (Finding 3): per 128-vector,
    # fp16 costs 256 bytes.
    assert O.record_bytes(128, 3, O.MSE) == 50 and 256 / 50 == 5.12
    assert O.record_bytes(128, 4, O.MSE) == 66 and 3.8 < 256 / 66 < 4.0
    assert O.record_bytes(128, 2, O.MSE) == 34
    # TurboQuant_prod at 2 bits, d=64, m=64: 8 B codes + 8 B signs + 2 + 2
    assert O.record_bytes(64, 2, O.PROD, 64) == 20


# ------------------------------------------------------------------ quantise / dequantise
@pytest.mark.parametrize("bits", [1, 2])
def test_codes_are_exhaustive_nearest_codeword_tiny(bits):
    # brute force over every codeword of a d=8 vector: the oracle's codes minimise
    # ||z - c[codes]|| over all (2^bits)^8 code vectors
    rng = np.random.default_rng(11)
    c, _, _ = O.lloyd_max_gaussian(bits)
    levels = len(c)
    grid = np.array(np.meshgrid(*[np.arange(levels)] * 8, indexing="ij")).reshape(8, -1).T
    for _ in range(3):
        x = rng.standard_normal((1, 8))
        rec = O.quantize(x, bits)
        err = np.sum((rec.z[0][None, :] - c[grid]) ** 2, axis=1)
        best = grid[np.argmin(err)]
        assert np.array_equal(rec.codes[0], best)


def test_codeword_input_round_trips_exactly():
    # x built from a codeword (x = n R^-1 c[codes] / sqrt(d)) quantises back to the same codes
    # and dequantises to x up to the float16 rounding of its norm
    rng = np.random.default_rng(5)
    d, bits, seed = 128, 3, 9
    c, beta, _ = O.lloyd_max_gaussian(bits)
    # codes drawn with the Gaussian cell probabilities, so ||c[codes]|| ~= sqrt(d) and the
    # rescaled codeword z = sqrt(d) c / ||c|| stays inside every code's cell
    cell = np.diff(scipy.stats.norm.cdf(np.concatenate([[-np.inf], beta, [np.inf]])))
    codes = rng.choice(len(c), size=(20, d), p=cell)
    y = c[codes]
    lam = math.sqrt(d) / np.linalg.norm(y, axis=1)
    assert np.all((lam > 0.85) & (lam < 1.3))
    n = rng.uniform(0.5, 40.0, size=20)
    unit = O.inverse_rotate(y / np.linalg.norm(y, axis=1, keepdims=True), seed)
    x = unit * n[:, None]
    rec = O.quantize(x, bits, seed=seed)
    assert np.array_equal(rec.codes, codes)
    xh = O.dequantize(rec)
    scale_y = np.linalg.norm(y, axis=1) / math.sqrt(d)
    rel = np.abs(rec.norm16.astype(float) - n) / n
    assert np.all(rel <= 2.0 ** -11)
    assert np.allclose(xh, x * (rec.norm16.astype(float) / n)[:, None] * scale_y[:, None],
                       atol=1e-9)


def test_norm_rounds_to_fp16_and_saturates_to_inf():
    # the stored norm is the IEEE round-to-nearest fp16 of the float32 norm: 65504 is the
    # largest finite fp16 value, the halfway point 65520 and anything above round to +inf
    d = 16
    e0 = np.zeros((4, d))
    e0[:, 3] = [65504.0, 65519.0, 65520.0, 1.0e6]
    r = O.quantize(e0, 3, O.MSE, seed=0)
    got = r.norm16.astype(np.float64)
    assert got[0] == 65504.0 and got[1] == 65504.0
    assert np.isinf(got[2]) and np.isinf(got[3]) and np.all(got[2:] > 0)
    # the codes are those of the unit vector, whatever the norm
    r1 = O.quantize(e0[:1] / 65504.0, 3, O.MSE, seed=0)
    assert np.array_equal(r.codes, np.repeat(r1.codes, 4, axis=0))


def test_zero_vector():
    x = np.zeros((2, 64))
    x[1, 3] = 1.0
    for bits, mode in ((4, O.MSE), (2, O.PROD), (1, O.PROD)):
        rec = O.quantize(x, bits, mode, m=64)
        assert rec.norm16[0] == 0
        wbits = bits if mode == O.MSE else bits - 1
        if wbits:
            assert np.all(rec.codes[0] == (1 << (wbits - 1)) - 1)
        assert np.all(O.dequantize(rec)[0] == 0)
        if mode == O.PROD and bits == 1:
            # no Lloyd-Max codes: r = z = 0, S r = 0 and sign(0) = +1 gives bit 0
            assert np.all(rec.qjl_bits[0] == 0) and rec.rnorm16[0] == 0


def test_mse_mode_inner_product_bias_about_three_percent():
    # "Above 3 bits, the bias is small enough (~3%)" (Three-Step Summary, Step 3). For a
    # Lloyd-Max quantiser E[z Q(z)] = 1 - D, so <q, x_hat> ~= (1 - D_b) <q, x>; at b = 3
    # that is 0.9655.
    rng = np.random.default_rng(1)
    d, bits = 128, 3
    _, _, dist = O.lloyd_max_gaussian(bits)
    ratios = []
    for seed in range(40):
        x = rng.standard_normal((64, d))
        rec = O.quantize(x, bits, seed=seed)
        xh = O.dequantize(rec)
        ratios.append(np.sum(xh * x) / np.sum(x * x))
    assert abs(np.mean(ratios) - (1 - dist)) < 0.01
    assert 0.02 < 1 - np.mean(ratios) < 0.045


def test_qjl_estimator_is_unbiased_and_variance_shrinks_with_m():
    # QJL "eliminates the systematic bias" (Three-Step Summary, Step 3): averaged over the
    # random projection, <q, x_hat> -> <q, x>. With sign bits of S r, E[s_j (S q)_j] =
    # sqrt(2/pi) <q, r>/||r||, so the 1/m sum scaled by gamma sqrt(pi/2) is unbiased; its
    # variance falls as 1/m.
    rng = np.random.default_rng(3)
    d = 16
    x = rng.standard_normal((1, d))
    q = rng.standard_normal(d)
    exact = float(q @ x[0])
    est = {}
    for m in (16, 64):
        vals = []
        for s in range(1500):
            rec = O.quantize(x, 2, O.PROD, seed=4, qjl_seed=1000 + s, m=m)
            vals.append(float(q @ O.dequantize(rec)[0]))
        est[m] = np.array(vals)
        z = (est[m].mean() - exact) / (est[m].std() / math.sqrt(len(vals)))
        assert abs(z) < 4.0, (m, est[m].mean(), exact)
    # the MSE-only 1-bit estimate is biased by (1 - D_1) = 0.636, far outside these bands
    ratio = est[16].var() / est[64].var()
    assert 2.8 < ratio < 5.5


def test_prod_one_bit_residual_is_whole_vector():
    # b = 1 in TurboQuant_prod: no Lloyd-Max codes, the residual is the unit vector itself
    x = np.random.default_rng(2).standard_normal((10, 32))
    rec = O.quantize(x, 1, O.PROD, m=32)
    assert rec.packed.shape == (10, 0)
    assert np.allclose(rec.rnorm, 1.0)
    assert np.allclose(rec.proj, (rec.z / math.sqrt(32)) @ O.qjl_matrix(1, 32, 32).T)


def test_high_bit_dequantisation_converges_to_input():
    x = np.random.default_rng(8).standard_normal((50, 64)) * 3.0
    errs = [np.linalg.norm(O.dequantize(O.quantize(x, b)) - x) / np.linalg.norm(x)
            for b in (2, 4, 5, 6)]
    for b, e in zip((2, 4, 5, 6), errs):
        _, _, dist = O.lloyd_max_gaussian(b)
        assert abs(e - math.sqrt(dist)) < 0.15 * math.sqrt(dist) + 1e-3
    assert errs == sorted(errs, reverse=True)


def test_quantize_is_deterministic_and_row_independent():
    # the rotation is fixed per seed, so re-quantising reproduces the bytes (prefix-cache
    # reuse, "Why the KV Cache Exists", Prefix Caching); rows are independent (a head slice
    # quantised alone gives the same bytes: per-shard quantisation, "Where This Fits",
    # Production Deployment: Tensor Parallelism)
    x = np.random.default_rng(4).standard_normal((40, 64))
    a = O.quantize(x, 2, O.PROD, seed=3, qjl_seed=8, m=32)
    b = O.quantize(x[10:20], 2, O.PROD, seed=3, qjl_seed=8, m=32)
    assert np.array_equal(a.packed[10:20], b.packed)
    assert np.array_equal(a.qjl_packed[10:20], b.qjl_packed)
    c = O.quantize(x, 2, O.PROD, seed=3, qjl_seed=8, m=32)
    assert np.array_equal(a.packed, c.packed) and np.array_equal(a.norm16, c.norm16)


def test_records_from_packed_round_trip():
    x = np.random.default_rng(6).standard_normal((7, 64))
    a = O.quantize(x, 2, O.PROD, m=64)
    r = O.records_from_packed(2, O.PROD, 64, a.packed, a.norm16, a.qjl_packed, a.rnorm16, m=64)
    assert np.array_equal(O.dequantize(r), O.dequantize(a))


# ------------------------------------------------------------------ attention
def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(9)
    b, hq, hkv, t, d = 2, 8, 2, 37, 32
    q = rng.standard_normal((b, hq, d))
    k = rng.standard_normal((b, hkv, t, d)) * 2
    v = rng.standard_normal((b, hkv, t, d))
    out = O.gqa_decode(q, k, v, 1 / math.sqrt(d))
    g = hq // hkv
    kt = torch.tensor(k).repeat_interleave(g, dim=1)
    vt = torch.tensor(v).repeat_interleave(g, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[:, :, None, :], kt, vt)[:, :, 0, :].numpy()
    assert np.allclose(out, ref, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(10)
    v = rng.standard_normal((5, 16))
    k = rng.standard_normal((5, 16))
    assert np.allclose(O.attention(rng.standard_normal(16), k[:1], v[:1], 0.3), v[0])
    assert np.allclose(O.attention(np.zeros(16), k, v, 0.3), v.mean(0))
    kk = np.repeat(k[:1], 5, axis=0)
    assert np.allclose(O.attention(rng.standard_normal(16), kk, v, 0.3), v.mean(0))
    # a dominant key selects its value
    k2 = k.copy()
    k2[2] = 1000.0 * np.ones(16)
    assert np.allclose(O.attention(np.ones(16), k2, v, 1.0), v[2])


def test_compressed_attention_converges_with_bits():
    # each extra bit roughly halves the reconstruction error (D_b ~ 4^-b), so the attention
    # output over the dequantised cache approaches exact attention at that rate
    rng = np.random.default_rng(12)
    b, hq, hkv, t, d = 1, 4, 1, 64, 32
    q = rng.standard_normal((b, hq, d))
    k = rng.standard_normal((b * hkv * t, d))
    v = rng.standard_normal((b * hkv * t, d))
    exact = O.gqa_decode(q, k.reshape(b, hkv, t, d), v.reshape(b, hkv, t, d), 1 / math.sqrt(d))
    errs = []
    for bits in (2, 3, 4, 5, 6):
        out = O.decode_compressed(q, [O.quantize(k, bits)], [O.quantize(v, bits)], b, hkv,
                                  1 / math.sqrt(d))
        errs.append(np.linalg.norm(out - exact) / np.linalg.norm(exact))
    ratios = np.array(errs[:-1]) / np.array(errs[1:])
    assert np.all((ratios > 1.4) & (ratios < 2.6)), errs
    assert errs[-1] < 0.06


def test_prefill_reduces_to_decode_and_is_causal():
    # prefill over the compressed cache (S16, Decode Throughput vs. TTFT): the last query of a
    # chunk that ends the cache is a decode query; a query never sees later positions; the
    # first position of a sequence attends to itself alone
    rng = np.random.default_rng(21)
    B, Hkv, G, T, d, lq = 2, 2, 3, 40, 32, 5
    K, V = rng.standard_normal((2, B, Hkv, T, d))
    k_recs = [O.quantize(K[b, h], 3) for b in range(B) for h in range(Hkv)]
    v_recs = [O.quantize(V[b, h], 2) for b in range(B) for h in range(Hkv)]
    q = rng.standard_normal((B, lq, Hkv * G, d))
    t0 = T - lq
    out = O.prefill_compressed(q, k_recs, v_recs, B, Hkv, t0, d ** -0.5)
    assert out.shape == (B, lq, Hkv * G, d)
    # (1) the chunk's last query over the whole cache is the decode of that query
    dec = O.decode_compressed(q[:, -1], k_recs, v_recs, B, Hkv, d ** -0.5)
    np.testing.assert_allclose(out[:, -1], dec, rtol=0, atol=1e-13)
    # (2) causality: other keys and values after position t0 + i leave query i unchanged
    K2, V2 = K.copy(), V.copy()
    K2[:, :, t0 + 2:] = 5.0 * rng.standard_normal(K2[:, :, t0 + 2:].shape)
    V2[:, :, t0 + 2:] = rng.standard_normal(V2[:, :, t0 + 2:].shape)
    k2 = [O.quantize(K2[b, h], 3) for b in range(B) for h in range(Hkv)]
    v2 = [O.quantize(V2[b, h], 2) for b in range(B) for h in range(Hkv)]
    out2 = O.prefill_compressed(q, k2, v2, B, Hkv, t0, d ** -0.5)
    np.testing.assert_array_equal(out2[:, :2], out[:, :2])
    assert np.abs(out2[:, 2:] - out[:, 2:]).max() > 1e-3
    # (3) a chunk at the start of a sequence: position 0 sees only itself, so its output is
    # the dequantised value of token 0 whatever the query
    first = O.prefill_compressed(q[:, :1] * 100.0, k_recs, v_recs, B, Hkv, 0, d ** -0.5)
    for b in range(B):
        for h in range(Hkv * G):
            np.testing.assert_allclose(first[b, 0, h], O.dequantize(v_recs[b * Hkv + h // G])[0],
                                       rtol=0, atol=1e-14)

