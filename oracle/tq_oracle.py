"""Plain, slow CPU oracle (NumPy, float64) for TurboQuant-style KV-cache compression and for
decode attention over the compressed cache.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``; never by the product path. It shares no code, table or
constant generator with the CUDA library. Inputs reach it as arrays; it draws its own random
signs and projection matrix from the seed with its own SplitMix64 (a published counter-based
generator), exactly as the library does independently on its side.

Sources (web pages on TurboQuant, cited by title and section):
  [S17] "Closing - The Three-Step Summary": Step 1 Rotate, Step 2 Quantize, Step 3 Correct,
        The One-Slide Version.
  [S15] "What the Paper Doesn't Tell You": Finding 1 (keys vs values), Finding 2 (QJL),
        Finding 3 (bit-widths, block 128), Finding 4 (rotation implementation).
  [S04] "Why the KV Cache Exists": What's in the KV Cache; Prefix Caching.
  [S16] "Where This Fits in the Inference Stack": TensorRT-LLM (dequantise inside the
        attention kernel); Decode Throughput vs. Time to First Token.

Every step the pages leave open takes a stated reading; each reading is marked "Reading:".

Parity pins: every public function here is pinned by tests/test_oracle.py against values
the pages print, closed forms, invariants, library routines the oracle does not use, or
brute force on tiny inputs; boundary_distance (the exemption band of the bit-exact code
comparison) is pinned against the decision boundaries of Max's published Gaussian quantiser.
"""
from __future__ import annotations

import functools
import math
from dataclasses import dataclass
from statistics import NormalDist

import numpy as np

__all__ = [
    "MSE", "PROD", "E2M1", "e2m1_value", "e2m1_codebook", "code_to_e2m1", "splitmix64", "rotation_signs", "hadamard", "rotate", "inverse_rotate",
    "qjl_matrix", "lloyd_max_gaussian", "codebook", "Records", "quantize", "dequantize",
    "pack_bits", "unpack_bits", "code_bytes", "sign_bytes", "record_bytes",
    "boundary_distance", "attention", "gqa_decode", "decode_compressed", "records_from_packed",
    "prefill_compressed",
]

MSE = 0   # TurboQuant_mse: b-bit Lloyd-Max codes only
PROD = 1  # TurboQuant_prod: (b-1)-bit Lloyd-Max codes + 1-bit QJL residual sketch
E2M1 = 2  # TurboQuant_mse with 4-bit codes on Blackwell's FP4 (E2M1) grid [S16 Blackwell FP4]

_MASK64 = (1 << 64) - 1
_ROWS = 1024  # vectors per chunk in quantize/boundary_distance (memory only)
_GAMMA = 0x9E3779B97F4A7C15


# ----------------------------------------------------------------------------------------
# Random numbers. Reading: the pages say only "random signs" [S17 Step 1] and "a random sign
# vector (16 bytes)" [S15 Finding 4]; the generator is SplitMix64 (Steele, Lea & Flood,
# "Fast splittable pseudorandom number generators", OOPSLA 2014), whose k-th output (k>=0)
# from seed s is mix(s + (k+1)*0x9E3779B97F4A7C15).
# ----------------------------------------------------------------------------------------
def splitmix64(seed: int, n: int) -> list[int]:
    """First ``n`` 64-bit outputs of SplitMix64 started from ``seed``."""
    out = []
    state = seed & _MASK64
    for _ in range(n):
        state = (state + _GAMMA) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def rotation_signs(seed: int, d: int) -> np.ndarray:
    """Diagonal of D as +-1.0 (length d).

    Reading: bit i of the SplitMix64 stream (bit i%64 of output i//64) set means D_ii = -1.
    d bits of storage: 16 bytes at d=128 [S15 Finding 4].
    """
    words = splitmix64(seed, (d + 63) // 64)
    return np.array([-1.0 if (words[i // 64] >> (i % 64)) & 1 else 1.0 for i in range(d)])


def hadamard(d: int) -> np.ndarray:
    """Explicit natural-order (Sylvester) Hadamard matrix, H_ij = (-1)^popcount(i & j).

    Unnormalised (entries +-1); H @ H = d * I. Reading: natural order, signs applied first
    [S17 Step 1: "Walsh-Hadamard Transform + random signs"].
    """
    return _hadamard_cached(d).copy()


@functools.lru_cache(maxsize=None)
def _hadamard_cached(d: int) -> np.ndarray:
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    idx = range(d)
    parity = np.array([[bin(a & b).count("1") & 1 for b in idx] for a in idx])
    return np.where(parity == 1, -1.0, 1.0)


def rotate(x: np.ndarray, seed: int) -> np.ndarray:
    """Orthonormal rotation R x = H D x / sqrt(d), rows of ``x`` are vectors [S17 Step 1]."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    return (x * rotation_signs(seed, d)) @ hadamard(d).T / math.sqrt(d)


def inverse_rotate(y: np.ndarray, seed: int) -> np.ndarray:
    """R^-1 y = D H y / sqrt(d) (R is orthogonal and H symmetric)."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    return (y @ hadamard(d).T) * rotation_signs(seed, d) / math.sqrt(d)


def qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    """QJL projection S (m x d), i.i.d. N(0,1) entries, values rounded to float32.

    Reading: the pages give only "a 1-bit QJL sketch of the residual" [S17 Step 3]. S is
    drawn row-major from SplitMix64(seed): uniform u = (word >> 11) * 2^-53 in [0,1); entries
    2k and 2k+1 come from the Box-Muller transform (Box & Muller 1958) of the pair
    (u_2k, u_2k+1): rho = sqrt(-2 ln(1 - u_2k)), theta = 2 pi u_2k+1,
    e_2k = rho cos(theta), e_2k+1 = rho sin(theta); computed in double, rounded to float32.
    """
    return _qjl_cached(seed, m, d).copy()


@functools.lru_cache(maxsize=None)
def _qjl_cached(seed: int, m: int, d: int) -> np.ndarray:
    n = m * d
    if n % 2:
        raise ValueError("m*d must be even")
    words = splitmix64(seed, n)
    u = np.array([(w >> 11) * (1.0 / 9007199254740992.0) for w in words])
    out = np.empty(n)
    for k in range(n // 2):
        rho = math.sqrt(-2.0 * math.log(1.0 - u[2 * k]))
        theta = 2.0 * math.pi * u[2 * k + 1]
        out[2 * k] = rho * math.cos(theta)
        out[2 * k + 1] = rho * math.sin(theta)
    return out.astype(np.float32).astype(np.float64).reshape(m, d)


# ----------------------------------------------------------------------------------------
# Lloyd-Max codebook for N(0,1) [S17 Step 2: "Lloyd-Max scalar quantization ... the
# codebook is optimal for that distribution ... centroids scale with 1/sqrt(d)"].
# ----------------------------------------------------------------------------------------
def _pdf(x: float) -> float:
    return 0.0 if math.isinf(x) else math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _cdf(x: float) -> float:
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


@functools.lru_cache(maxsize=None)
def _lloyd_max_cached(bits: int, tol: float, max_iter: int):
    return _lloyd_max(bits, tol, max_iter)


def lloyd_max_gaussian(bits: int, tol: float = 1e-13, max_iter: int = 200000):
    """See :func:`_lloyd_max`; cached per arguments (returns fresh copies)."""
    c, beta, dist = _lloyd_max_cached(bits, tol, max_iter)
    return c.copy(), beta.copy(), dist


def _lloyd_max(bits: int, tol: float, max_iter: int):
    """Lloyd-Max quantiser of N(0,1) with 2^bits levels.

    Alternates the two optimality conditions: each boundary is the midpoint of its two
    neighbouring centroids; each centroid is the conditional mean of N(0,1) on its cell,
    (pdf(lo) - pdf(hi)) / (cdf(hi) - cdf(lo)). Starts from the centroids of the 2^bits
    equal-probability cells' midpoint quantiles and stops when no centroid moves by more
    than ``tol``. Returns (centroids ascending, boundaries ascending, distortion D), with
    D = E[(z - Q(z))^2] = 1 - sum_j c_j^2 P_j (valid at the fixed point, where E[z Q(z)] =
    E[Q(z)^2]).
    """
    if not 1 <= bits <= 6:
        raise ValueError("bits must be in 1..6")
    levels = 1 << bits
    c = [NormalDist().inv_cdf((j + 0.5) / levels) for j in range(levels)]
    for _ in range(max_iter):
        beta = [(c[j] + c[j + 1]) / 2.0 for j in range(levels - 1)]
        edges = [-math.inf] + beta + [math.inf]
        new = [(_pdf(edges[j]) - _pdf(edges[j + 1])) / (_cdf(edges[j + 1]) - _cdf(edges[j]))
               for j in range(levels)]
        moved = max(abs(a - b) for a, b in zip(c, new))
        c = new
        if moved < tol:
            break
    else:
        raise RuntimeError("Lloyd-Max did not converge")
    # N(0,1) is symmetric, so the fixed point is: c_j = -c_{L-1-j}. Make that exact, which
    # puts the middle boundary exactly at 0 (a zero coordinate then ties to the lower level).
    c = [(c[j] - c[levels - 1 - j]) / 2.0 for j in range(levels)]
    beta = [(c[j] + c[j + 1]) / 2.0 for j in range(levels - 1)]
    edges = [-math.inf] + beta + [math.inf]
    dist = 1.0 - sum(c[j] ** 2 * (_cdf(edges[j + 1]) - _cdf(edges[j])) for j in range(levels))
    return np.array(c), np.array(beta), dist


# ----------------------------------------------------------------------------------------
# The E2M1 grid [S16 "Blackwell FP4: The Natural Convergence Point": whether the Lloyd-Max
# centroids map onto NVFP4's E2M1 values is left open there]. E2M1 is the 4-bit float of
# the OCP microscaling formats: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; it
# holds 0, 0.5, 1, 1.5, 2, 3, 4, 6 with either sign (+0 and -0 both exist).
# Reading: the rotated coordinates are i.i.d. N(0,1) for every block, so one stretch s of the
# grid (no per-block scale) is the quantiser: 16 levels s * (-6, -4, -3, -2, -1.5, -1, -0.5,
# -0, +0, 0.5, 1, 1.5, 2, 3, 4, 6) in ascending order, the two zeros kept as two codes (a
# coordinate takes the zero of its own sign), boundaries at the midpoints (0 between the two
# zeros), s minimising the Gaussian MSE. Code i is stored like a Lloyd-Max code (its index in
# that order); its E2M1 bit pattern is code_to_e2m1(i).
# ----------------------------------------------------------------------------------------
_E2M1_SORTED = (-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, -0.0, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def e2m1_value(bits: int) -> float:
    """The value of a 4-bit E2M1 pattern: (-1)^s * (m / 2 if e == 0 else 2^(e-1) * (1 + m/2))."""
    sign = -1.0 if (bits >> 3) & 1 else 1.0
    e, m = (bits >> 1) & 3, bits & 1
    return sign * (m / 2.0 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0))


def code_to_e2m1(code):
    """E2M1 bit pattern of code i of the ascending E2M1 codebook: the positive half (i >= 8)
    is i - 8, the negative half the magnitude order reversed under the sign bit."""
    code = np.asarray(code, dtype=np.int64)
    return np.where(code >= 8, code - 8, 8 + (7 - code))


def _grid_mse(levels: np.ndarray) -> float:
    """E[(z - Q(z))^2] for z ~ N(0,1) and the nearest-level quantiser on ascending ``levels``
    (cells between the midpoints), from the exact Gaussian moments of each cell."""
    edges = [-math.inf] + [(levels[j] + levels[j + 1]) / 2.0 for j in range(len(levels) - 1)] + [math.inf]
    total = 0.0
    for j, c in enumerate(levels):
        a, b = edges[j], edges[j + 1]
        p = _cdf(b) - _cdf(a)
        m1 = _pdf(a) - _pdf(b)
        m2 = p + (0.0 if math.isinf(a) else a * _pdf(a)) - (0.0 if math.isinf(b) else b * _pdf(b))
        total += m2 - 2.0 * c * m1 + c * c * p
    return total


@functools.lru_cache(maxsize=None)
def _e2m1_cached():
    grid = np.array(_E2M1_SORTED)
    lo, hi = 0.3, 0.8  # the Gaussian MSE of the stretched grid is unimodal here
    g = (math.sqrt(5.0) - 1.0) / 2.0
    a, b = hi - g * (hi - lo), lo + g * (hi - lo)
    fa, fb = _grid_mse(grid * a), _grid_mse(grid * b)
    while hi - lo > 1e-12:  # golden-section search
        if fa < fb:
            hi, b, fb = b, a, fa
            a = hi - g * (hi - lo)
            fa = _grid_mse(grid * a)
        else:
            lo, a, fa = a, b, fb
            b = lo + g * (hi - lo)
            fb = _grid_mse(grid * b)
    s = (lo + hi) / 2.0
    c = grid * s
    beta = np.array([(c[j] + c[j + 1]) / 2.0 for j in range(15)])
    beta[7] = 0.0
    return c, beta, _grid_mse(c), s


def e2m1_codebook():
    """(levels ascending [16], boundaries ascending [15], Gaussian MSE, stretch s) of the E2M1
    codebook on the N(0,1) scale (see the reading above)."""
    c, beta, dist, s = _e2m1_cached()
    return c.copy(), beta.copy(), dist, s


def _levels(wbits: int, mode: int):
    """Centroids and boundaries (N(0,1) scale) of a tensor's codes."""
    if mode == E2M1:
        c, beta, _, _ = e2m1_codebook()
        return c, beta
    c, beta, _ = lloyd_max_gaussian(wbits)
    return c, beta


def codebook(bits: int, d: int):
    """Centroids and boundaries for a unit-norm vector's rotated coordinates: the N(0,1)
    Lloyd-Max codebook scaled by 1/sqrt(d) [S17 Step 2; One-Slide Version]."""
    c, beta, _ = lloyd_max_gaussian(bits)
    return c / math.sqrt(d), beta / math.sqrt(d)


# ----------------------------------------------------------------------------------------
# Bit packing. Reading: code i of a record occupies bits [i*w, i*w + w) of a little-endian
# bit stream (stream bit k is bit k%8 of byte k//8). QJL sign j is stream bit j of its own
# record; bit = 1 means (S r)_j < 0.
# ----------------------------------------------------------------------------------------
def pack_bits(vals: np.ndarray, width: int) -> np.ndarray:
    """Pack non-negative ints [N, k] (< 2^width) into bytes [N, k*width/8]."""
    vals = np.asarray(vals, dtype=np.int64)
    n, k = vals.shape
    if (k * width) % 8:
        raise ValueError("record is not a whole number of bytes")
    if width == 0:
        return np.zeros((n, 0), dtype=np.uint8)
    stream = ((vals[:, :, None] >> np.arange(width)) & 1).reshape(n, k * width)
    return np.packbits(stream.astype(np.uint8), axis=1, bitorder="little")


def unpack_bits(packed: np.ndarray, width: int, k: int) -> np.ndarray:
    """Inverse of :func:`pack_bits`: bytes [N, k*width/8] -> ints [N, k]."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    if width == 0:
        return np.zeros((n, k), dtype=np.int64)
    stream = np.unpackbits(packed, axis=1, bitorder="little")[:, : k * width]
    stream = stream.reshape(n, k, width).astype(np.int64)
    return (stream << np.arange(width)).sum(axis=2)


def _mse_bits(bits: int, mode: int) -> int:
    return bits - 1 if mode == PROD else bits


def code_bytes(d: int, bits: int, mode: int) -> int:
    """Bytes of packed Lloyd-Max codes per vector."""
    return d * _mse_bits(bits, mode) // 8


def sign_bytes(d: int, bits: int, mode: int, m: int | None = None) -> int:
    """Bytes of QJL sign bits per vector (0 in MSE mode)."""
    return (m or d) // 8 if mode == PROD else 0


def record_bytes(d: int, bits: int, mode: int, m: int | None = None) -> int:
    """Stored bytes per vector: codes + signs + fp16 norm (+ fp16 residual norm in PROD).

    At d=128 a 3-bit MSE record is 48 + 2 = 50 bytes, 5.12x smaller than 256 bytes of fp16
    [S15 Finding 3, "block_size=128: 5.12x"]; a 4-bit record is 66 bytes (~4x).
    """
    extra = 4 if mode == PROD else 2
    return code_bytes(d, bits, mode) + sign_bytes(d, bits, mode, m) + extra


def _fp16_of(v: np.ndarray) -> np.ndarray:
    """Round a float64 value to float32 then float16 (both round-to-nearest-even); values at or
    above 65520 in magnitude become infinite, as IEEE rounding prescribes."""
    with np.errstate(over="ignore"):
        return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float16)


# ----------------------------------------------------------------------------------------
# Quantise [S17 Steps 1-3; S15 Findings 1-3]
# ----------------------------------------------------------------------------------------
@dataclass
class Records:
    """Compressed records for N vectors of dimension d (one tensor: keys or values)."""
    bits: int
    mode: int
    d: int
    m: int
    seed: int
    qjl_seed: int
    codes: np.ndarray        # [N, d] Lloyd-Max code indices (ascending level order)
    packed: np.ndarray       # [N, code_bytes] uint8
    norm16: np.ndarray       # [N] float16, ||x||
    qjl_bits: np.ndarray     # [N, m] 0/1 (PROD) or [N, 0]
    qjl_packed: np.ndarray   # [N, m/8] uint8 (PROD) or [N, 0]
    rnorm16: np.ndarray      # [N] float16 residual norm gamma (PROD) or zeros
    z: np.ndarray            # [N, d] rotated coordinates on the N(0,1) scale (H D x / ||x||)
    proj: np.ndarray         # [N, m] S r (PROD) or [N, 0]
    rnorm: np.ndarray        # [N] exact residual norm (PROD) or zeros
    norm: np.ndarray         # [N] exact float64 norm ||x||


def quantize(x: np.ndarray, bits: int, mode: int = MSE, seed: int = 0, qjl_seed: int = 1,
             m: int | None = None) -> Records:
    """Compress the rows of ``x`` ([N, d], any real dtype; values taken exactly).

    1. n = ||x||_2 in float64; stored as float16 (via float32).
    2. z = H D x / n: the unnormalised Walsh-Hadamard transform of the sign-flipped vector,
       divided by the norm, so each coordinate is near N(0,1) [S17 Step 1].
       Reading: a zero vector gets z = 0.
    3. MSE: code_i = the nearest centroid of the ``bits``-bit N(0,1) Lloyd-Max codebook,
       found by brute force over all centroids; an exact tie goes to the lower index
       [S17 Step 2]. This equals the count of boundaries strictly below z_i (checked).
    3''. E2M1 (bits = 4): as 3 on the E2M1 codebook; a coordinate between the two zero levels
       takes the zero of its own sign (the count of boundaries strictly below z; 0 -> -0).
    3'. PROD (b <= 2, [S17 Step 3; S15 Finding 2]): (bits-1)-bit codes as in 3 (none when
       bits = 1); residual r = (z - c[code]) / sqrt(d) in the unit-norm rotated domain;
       gamma = ||r|| stored as float16; QJL bit j = 1 iff (S r)_j < 0 (sign(0) = +1).
    """
    x = np.asarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("x must be [N, d]")
    n_vec, d = x.shape
    m = d if (m is None or m == 0) else m
    wbits = _mse_bits(bits, mode)
    if mode not in (MSE, PROD, E2M1) or bits < 1 or wbits < 0 or (mode == E2M1 and bits != 4):
        raise ValueError("bad bits/mode")

    norm = np.sqrt(np.sum(x * x, axis=1))
    norm16 = _fp16_of(norm)
    y = (x * rotation_signs(seed, d)) @ hadamard(d).T
    z = np.zeros_like(y)
    nz = norm > 0
    z[nz] = y[nz] / norm[nz, None]

    if wbits > 0:
        cent, beta = _levels(wbits, mode)
        codes = np.empty(z.shape, dtype=np.int64)
        for lo in range(0, n_vec, _ROWS):  # rows are independent; chunks bound the temporaries
            zc = z[lo:lo + _ROWS]
            dist_all = np.abs(zc[:, :, None] - cent[None, None, :])
            nearest = np.argmin(dist_all, axis=2)
            counted = np.searchsorted(beta, zc, side="left")
            exact_tie = np.min(np.abs(zc[:, :, None] - beta[None, None, :]), axis=2) < 1e-12
            if mode == E2M1:
                # the two zero levels are equally near; the count picks the zero of z's sign
                codes[lo:lo + _ROWS] = counted
                got = np.take_along_axis(dist_all, counted[:, :, None], axis=2)[:, :, 0]
                assert np.all((got == dist_all.min(axis=2)) | exact_tie), "count is not a nearest level"
            else:
                codes[lo:lo + _ROWS] = nearest
                assert np.all((nearest == counted) | exact_tie), "nearest centroid != boundary count"
        chat = cent[codes]
    else:
        codes = np.zeros((n_vec, d), dtype=np.int64)
        chat = np.zeros((n_vec, d))
    packed = pack_bits(codes, wbits)

    if mode == PROD:
        s_mat = qjl_matrix(qjl_seed, m, d)
        r = (z - chat) / math.sqrt(d)
        rnorm = np.sqrt(np.sum(r * r, axis=1))
        proj = r @ s_mat.T
        qbits = (proj < 0).astype(np.int64)
        qpacked = pack_bits(qbits, 1)
        rnorm16 = _fp16_of(rnorm)
    else:
        rnorm = np.zeros(n_vec)
        proj = np.zeros((n_vec, 0))
        qbits = np.zeros((n_vec, 0), dtype=np.int64)
        qpacked = np.zeros((n_vec, 0), dtype=np.uint8)
        rnorm16 = np.zeros(n_vec, dtype=np.float16)
    return Records(bits, mode, d, m, seed, qjl_seed, codes, packed, norm16, qbits, qpacked,
                   rnorm16, z, proj, rnorm, norm)


def records_from_packed(bits: int, mode: int, d: int, packed: np.ndarray, norm16: np.ndarray,
                        qjl_packed: np.ndarray | None = None,
                        rnorm16: np.ndarray | None = None, seed: int = 0, qjl_seed: int = 1,
                        m: int | None = None) -> Records:
    """Rebuild :class:`Records` from stored bytes (for dequantising stored caches)."""
    m = d if (m is None or m == 0) else m
    n_vec = packed.shape[0]
    codes = unpack_bits(packed, _mse_bits(bits, mode), d)
    if mode == PROD:
        qbits = unpack_bits(qjl_packed, 1, m)
    else:
        qbits = np.zeros((n_vec, 0), dtype=np.int64)
        qjl_packed = np.zeros((n_vec, 0), dtype=np.uint8)
        rnorm16 = np.zeros(n_vec, dtype=np.float16)
    return Records(bits, mode, d, m, seed, qjl_seed, codes, np.asarray(packed),
                   np.asarray(norm16, dtype=np.float16), qbits, np.asarray(qjl_packed),
                   np.asarray(rnorm16, dtype=np.float16), np.zeros((n_vec, d)),
                   np.zeros((n_vec, 0)), np.zeros(n_vec),
                   np.asarray(norm16, dtype=np.float16).astype(np.float64))


def dequantize(rec: Records) -> np.ndarray:
    """Reconstruct x_hat [N, d] in the original domain from the stored record.

    MSE: x_hat = n * R^-1 (c[code] / sqrt(d)) = n * D H c[code] / d.
    PROD: the unit-domain estimate is c[code]/sqrt(d) + gamma * sqrt(pi/2)/m * S^T s with
    s_j = +-1 from the sign bits; the QJL term is the unbiased inner-product reconstruction
    of the residual [S17 Step 3]; so x_hat = n * D H (c[code] + sqrt(d) gamma sqrt(pi/2)/m
    S^T s) / d. Uses the stored float16 norms.
    """
    d = rec.d
    wbits = _mse_bits(rec.bits, rec.mode)
    inner = _levels(wbits, rec.mode)[0][rec.codes] if wbits > 0 else np.zeros(rec.codes.shape)
    if rec.mode == PROD:
        s_mat = qjl_matrix(rec.qjl_seed, rec.m, d)
        signs = 1.0 - 2.0 * rec.qjl_bits
        gamma = rec.rnorm16.astype(np.float64)
        inner = inner + (math.sqrt(d) * math.sqrt(math.pi / 2.0) / rec.m) * gamma[:, None] * (
            signs @ s_mat)
    n16 = rec.norm16.astype(np.float64)
    return n16[:, None] * ((inner @ hadamard(d).T) * rotation_signs(rec.seed, d)) / d


def boundary_distance(rec: Records) -> np.ndarray:
    """Distance of every z_i to the nearest decision boundary (N(0,1) scale); +inf when the
    record has no Lloyd-Max codes. Used to exempt coordinates within 1e-5 of a boundary from
    bit-exact comparison (the two sides decide them in different precisions)."""
    wbits = _mse_bits(rec.bits, rec.mode)
    if wbits == 0:
        return np.full(rec.z.shape, np.inf)
    beta = _levels(wbits, rec.mode)[1]
    out = np.empty(rec.z.shape)
    for lo in range(0, rec.z.shape[0], _ROWS):
        zc = rec.z[lo:lo + _ROWS]
        out[lo:lo + _ROWS] = np.min(np.abs(zc[:, :, None] - beta[None, None, :]), axis=2)
    return out


# ----------------------------------------------------------------------------------------
# Attention [S04 What's in the KV Cache; S16 Decode Throughput vs. TTFT]
# ----------------------------------------------------------------------------------------
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Single-query attention, naive two-pass softmax: s_t = scale * q.k_t; first pass takes
    max_t s_t, second pass p_t = exp(s_t - max), out = sum_t p_t v_t / sum_t p_t.
    q [d]; k, v [T, d]. No causal mask: a decode query attends to every cached token."""
    s = scale * (np.asarray(k, np.float64) @ np.asarray(q, np.float64))
    p = np.exp(s - s.max())
    return (p @ np.asarray(v, np.float64)) / p.sum()


def gqa_decode(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Grouped-query decode: q [B, Hq, d]; k, v [B, Hkv, T, d]; query head h reads KV head
    h // (Hq/Hkv) (consecutive query heads share a KV head). Returns [B, Hq, d]."""
    b_sz, hq, d = q.shape
    hkv = k.shape[1]
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = hq // hkv
    out = np.empty((b_sz, hq, d))
    for b in range(b_sz):
        for h in range(hq):
            out[b, h] = attention(q[b, h], k[b, h // g], v[b, h // g], scale)
    return out


def decode_compressed(q: np.ndarray, k_recs: list, v_recs: list, b_sz: int, hkv: int,
                      scale: float) -> np.ndarray:
    """Attention over the dequantised cache. ``k_recs``/``v_recs`` are :class:`Records` per
    (b, h) in row-major [B][Hkv] order, each holding that head's T tokens."""
    t_len = k_recs[0].codes.shape[0]
    d = q.shape[-1]
    kh = np.stack([dequantize(r) for r in k_recs]).reshape(b_sz, hkv, t_len, d)
    vh = np.stack([dequantize(r) for r in v_recs]).reshape(b_sz, hkv, t_len, d)
    return gqa_decode(q, kh, vh, scale)


def prefill_compressed(q: np.ndarray, k_recs: list, v_recs: list, b_sz: int, hkv: int, t0: int,
                       scale: float) -> np.ndarray:
    """Prefill attention of a chunk over the compressed cache [S16 Decode Throughput vs. Time
    to First Token: at long contexts the attention layers of prefill read the cache too].

    q [B, Lq, Hq, d] holds the queries of positions t0 .. t0 + Lq - 1; ``k_recs``/``v_recs``
    (row-major [B][Hkv] Records) hold at least t0 + Lq tokens. Reading: the chunk's own keys
    and values are written to the cache first and read back compressed like the prefix, and
    query i attends causally to positions 0 .. t0 + i. Returns [B, Lq, Hq, d]."""
    b_q, lq, hq, d = q.shape
    if b_q != b_sz or hq % hkv:
        raise ValueError("q must be [B, Lq, Hq, d] with Hq a multiple of Hkv")
    t_len = k_recs[0].codes.shape[0]
    if t0 < 0 or t0 + lq > t_len:
        raise ValueError("the records must hold positions 0 .. t0 + Lq - 1")
    g = hq // hkv
    kh = np.stack([dequantize(r) for r in k_recs]).reshape(b_sz, hkv, t_len, d)
    vh = np.stack([dequantize(r) for r in v_recs]).reshape(b_sz, hkv, t_len, d)
    out = np.empty((b_sz, lq, hq, d))
    for b in range(b_sz):
        for i in range(lq):
            n = t0 + i + 1
            for h in range(hq):
                out[b, i, h] = attention(q[b, i, h], kh[b, h // g, :n], vh[b, h // g, :n], scale)
    return out
