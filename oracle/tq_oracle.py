"""Plain numpy float64 oracle of the TurboQuant packed-KV hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.

Pages cited (by title and section):

* [TorbuQuant]         ginkgoq.github.io/TurboQuant -- "TQ4 page tensor" diagram
                       (page tensor, slot arithmetic, slot regions, byte formula),
                       the four-stage list "Quantize / Store / Attend / Measure",
                       and the "Current Status" table (exact Beta-sphere and Gaussian
                       Lloyd-Max codebooks; QR and RHT rotations).
* [turboquant_serve]   turboquant_serve 0.1.2 -- "Architecture" (update/_decode tree,
                       "Rotation", "Keys vs values", "Codebook sharing").
* [tq-kv]              shadowgraph.io tq-kv -- "How It Works" step [3] (Randomized
                       Hadamard Transform), "Library API" (generate_signs,
                       pre_rotate_query_with_signs, fused_attention_scores),
                       "Custom CUDA Kernel Stack" (flash decode v2, fused TQ attention).
* [turboquant_pro]     turboquant_pro 1.4.2 -- "How It Works" (norm preserved
                       alongside bits; 8 x 3-bit = 3 bytes), "TurboQuant -- rotate +
                       scalar-quantize", "Fused CUDA decode".

Readings taken where the pages are silent (each is a convention, stated once
here and in the docstring that applies it):

* signs: s_j = -1 if the top bit of the j-th SplitMix64 output (seeded with
  ``sign_seed``) is set, else +1; sign flips are applied before the FWHT;
* FWHT in natural (Sylvester) order, H[i][j] = (-1)^popcount(i & j), scaled 1/sqrt(D);
* the stored norm is the L2 norm of the input row (equal to the rotated row's);
* encode: idx = #{i : b_i < u} against the fp32 boundary table (ties go to the
  lower cell); a zero row stores norm 0 and encodes u = 0;
* a row holding a non-finite value stores all-zero indices and a quiet-NaN norm;
* packing: index j occupies bits [j*b, (j+1)*b) of a little-endian bit stream
  (bit p is bit p % 8 of byte p // 8), followed by the fp32 norm, little endian;
* GQA: query head h reads KV head h // (H_q / H_kv);
* codebooks: the unique Lloyd-Max quantizer of the density, reached by Lloyd's
  iteration from Panter-Dite starting points, mirrored so that c[L-1-i] = -c[i],
  then rounded to fp32 (boundaries = fp32 of the fp64 midpoints).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy import special

U64 = np.uint64
_MASK64 = (1 << 64) - 1

# ---------------------------------------------------------------------------
# Sign vector: SplitMix64
# ---------------------------------------------------------------------------

SPLITMIX64_GAMMA = 0x9E3779B97F4A7C15


def splitmix64_outputs(seed: int, n: int) -> np.ndarray:
    """First ``n`` outputs of SplitMix64 seeded with ``seed`` (uint64 array).

    [tq-kv, "Library API"]: the rotation signs come from a seeded generator
    (``hadamard::generate_signs(dim, seed)``); the pages do not name it.  The
    generator used here is SplitMix64 as published by Steele, Lea and Flood
    (2014): state advances by the golden-ratio increment, and each output is the
    state passed through the two xor-shift-multiply rounds.  Written with Python
    integers so every step is exact mod 2^64.
    """
    out = np.empty(n, dtype=np.uint64)
    state = seed & _MASK64
    for j in range(n):
        state = (state + SPLITMIX64_GAMMA) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        z = z ^ (z >> 31)
        out[j] = z
    return out


def rht_signs(dim: int, sign_seed: int) -> np.ndarray:
    """Sign vector s in {+1, -1}^dim of the randomized Hadamard transform.

    [tq-kv, "How It Works" step 3; "Library API" ``generate_signs``].
    Convention: s_j = -1 when bit 63 of the j-th SplitMix64 output is 1.
    """
    z = splitmix64_outputs(sign_seed, dim)
    return np.where((z >> U64(63)) == 1, -1.0, 1.0)


# ---------------------------------------------------------------------------
# Rotation: randomized Hadamard transform
# ---------------------------------------------------------------------------


def hadamard_matrix(dim: int) -> np.ndarray:
    """Explicit Sylvester Hadamard matrix, H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(dim)[:, None]
    j = np.arange(dim)[None, :]
    bits = np.bitwise_and(i, j)
    pop = np.zeros_like(bits)
    while np.any(bits):
        pop += bits & 1
        bits = bits >> 1
    return np.where(pop % 2 == 0, 1.0, -1.0)


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis.

    Natural (Sylvester) order: the result equals ``x @ hadamard_matrix(D).T``.
    Butterfly stages h = 1, 2, 4, ..., D/2 each replace (a, b) at positions
    (i, i + h) by (a + b, a - b).
    """
    x = np.array(x, dtype=np.float64, copy=True)
    d = x.shape[-1]
    if d & (d - 1):
        raise ValueError("FWHT length must be a power of two")
    lead = x.shape[:-1]
    h = 1
    while h < d:
        y = x.reshape(*lead, d // (2 * h), 2, h)
        a = y[..., 0, :].copy()
        b = y[..., 1, :]
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        x = y.reshape(*lead, d)
        h *= 2
    return x


def rht_forward(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = (1/sqrt(D)) H (s * x) along the last axis.

    [tq-kv, "How It Works" step 3: randomized Hadamard transform, O(d log d)];
    [turboquant_serve, "Architecture": rotate k and v before encoding].
    """
    d = x.shape[-1]
    return fwht(np.asarray(x, dtype=np.float64) * signs) / math.sqrt(d)


def rht_inverse(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """x = (1/sqrt(D)) s * (H y): the transpose (= inverse) of ``rht_forward``.

    [turboquant_serve, "Architecture": ``_decode`` multiplies by R transposed].
    """
    d = y.shape[-1]
    return signs * fwht(np.asarray(y, dtype=np.float64)) / math.sqrt(d)


def rht_matrix(dim: int, signs: np.ndarray) -> np.ndarray:
    """Explicit rotation matrix R with rht_forward(x) = R @ x (for checks)."""
    return hadamard_matrix(dim) * signs[None, :] / math.sqrt(dim)


# ---------------------------------------------------------------------------
# Rotation: dense random orthogonal matrix (QR)
# ---------------------------------------------------------------------------


def haar_orthogonal(dim: int, seed: int) -> np.ndarray:
    """Random orthogonal D x D matrix, Haar distributed, float64.

    [turboquant_serve, "Architecture" / "Rotation": a fixed random orthogonal
    matrix, seeded by head_dim]; [TorbuQuant, "Current Status": QR rotation].  The
    pages name no generator: G is a D x D matrix of standard normals from numpy's
    PCG64 generator seeded with ``seed``; with G = Q R its QR factorisation
    (numpy.linalg.qr), the columns of Q are multiplied by the signs of diag(R), which
    makes the factorisation unique and the result Haar distributed (Mezzadri, 2007).
    """
    g = np.random.default_rng(seed).standard_normal((dim, dim))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (round to nearest even), returned as float64.
    Through float32 (exact for the bf16 grid once the float32 value is rounded once)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


@dataclass
class DenseRotation:
    """The dense rotation as both paths use it: R = hi + lo with hi = bf16(f) and
    lo = bf16(f - hi), f = fp32(H) and H the float64 Haar matrix (f - hi is exact in
    float32, so lo is a multiple of hi's float32 ulp and hi + lo is exact in float32).
    R is within 2^-17 of H entry by entry (orthogonal to about 1e-5); the tensor-core
    path multiplies by hi and by lo exactly."""

    dim: int
    seed: int
    haar: np.ndarray    # float64 H
    hi: np.ndarray      # float64 values on the bf16 grid
    lo: np.ndarray

    @property
    def matrix(self) -> np.ndarray:
        return self.hi + self.lo

    def forward(self, x: np.ndarray) -> np.ndarray:
        """y = R x along the last axis."""
        return np.asarray(x, dtype=np.float64) @ self.matrix.T

    def inverse(self, y: np.ndarray) -> np.ndarray:
        """R^T y along the last axis (the transpose stands in for the inverse)."""
        return np.asarray(y, dtype=np.float64) @ self.matrix


def dense_rotation(dim: int, seed: int) -> DenseRotation:
    h = haar_orthogonal(dim, seed)
    f = h.astype(np.float32).astype(np.float64)
    hi = bf16_round(f)
    lo = bf16_round((f.astype(np.float32) - hi.astype(np.float32)).astype(np.float64))
    return DenseRotation(dim=dim, seed=seed, haar=h, hi=hi, lo=lo)


def rotate_forward(x: np.ndarray, rot) -> np.ndarray:
    """R x with ``rot`` a DenseRotation, or the RHT when ``rot`` is its sign vector."""
    return rot.forward(x) if isinstance(rot, DenseRotation) else rht_forward(x, rot)


def rotate_inverse(y: np.ndarray, rot) -> np.ndarray:
    """R^T y with ``rot`` a DenseRotation, or the RHT when ``rot`` is its sign vector."""
    return rot.inverse(y) if isinstance(rot, DenseRotation) else rht_inverse(y, rot)


# ---------------------------------------------------------------------------
# Lloyd-Max codebooks
# ---------------------------------------------------------------------------


class BetaSphereDensity:
    """Density of one coordinate of a uniform point on the sphere S^{D-1}.

    f_D(x) = Gamma(D/2) / (sqrt(pi) Gamma((D-1)/2)) (1 - x^2)^((D-3)/2), |x| < 1.
    [TorbuQuant, "Current Status": "exact Beta-sphere" Lloyd-Max codebooks];
    [turboquant_serve, "Keys vs values": MSE-optimal for the Beta prior on
    rotated unit vectors].  (x + 1)/2 follows Beta((D-1)/2, (D-1)/2).
    """

    density_id = 0

    def __init__(self, dim: int):
        if dim < 3:
            raise ValueError("Beta-sphere density needs D >= 3")
        self.dim = dim
        self.a = (dim - 3) / 2.0
        self.k = math.exp(math.lgamma(dim / 2.0) - 0.5 * math.log(math.pi)
                          - math.lgamma((dim - 1) / 2.0))
        self.support_hi = 1.0

    def pdf(self, x):
        x = np.asarray(x, dtype=np.float64)
        return self.k * np.power(np.clip(1.0 - x * x, 0.0, None), self.a)

    def survival(self, x):
        """P(X > x), from the regularised incomplete beta function."""
        p = self.a + 1.0
        return special.betainc(p, p, np.clip((1.0 - np.asarray(x)) / 2.0, 0.0, 1.0))

    def mass(self, lo, hi):
        """Integral of f over [lo, hi] (0 <= lo <= hi <= 1)."""
        return self.survival(lo) - self.survival(hi)

    def first_moment(self, lo, hi):
        """Integral of x f(x) over [lo, hi]: closed form K[(1-lo^2)^(a+1) - (1-hi^2)^(a+1)]/(2(a+1))."""
        lo = np.asarray(lo, dtype=np.float64)
        hi = np.asarray(hi, dtype=np.float64)
        p = self.a + 1.0
        return self.k * (np.power(1.0 - lo * lo, p) - np.power(1.0 - hi * hi, p)) / (2.0 * p)

    def panter_dite_quantile(self, q):
        """Quantile of the density proportional to f^(1/3) (high-rate point density)."""
        p = self.a / 3.0 + 1.0
        return 2.0 * special.betaincinv(p, p, q) - 1.0


class GaussianDensity:
    """Standard normal density, for the Gaussian-approximation codebook.

    [TorbuQuant, "Current Status": Gaussian-approximation Lloyd-Max].
    """

    density_id = 1

    def __init__(self):
        self.support_hi = math.inf

    def pdf(self, x):
        x = np.asarray(x, dtype=np.float64)
        return np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)

    def mass(self, lo, hi):
        return special.ndtr(-np.asarray(lo)) - special.ndtr(-np.asarray(hi))

    def first_moment(self, lo, hi):
        return self.pdf(lo) - self.pdf(hi)

    def panter_dite_quantile(self, q):
        return math.sqrt(3.0) * special.ndtri(q)


@dataclass
class Codebook:
    """Lloyd-Max quantizer: L centroids and L-1 boundaries (float64)."""

    centroids: np.ndarray
    boundaries: np.ndarray
    iterations_run: int
    n_iter: int

    @property
    def levels(self) -> int:
        return self.centroids.size


def lloyd_max(density, bits: int, n_iter: int) -> Codebook:
    """Lloyd-Max scalar quantizer of a symmetric density with 2^bits levels.

    The two Lloyd-Max conditions: every boundary is the midpoint of its two
    neighbouring centroids, and every centroid is the conditional mean of the
    density over its cell.  Lloyd's iteration alternates them: boundaries from
    centroids, then centroids from boundaries.  By symmetry only the upper half
    (cells above 0) is iterated; the lower half is its mirror image, so the
    middle boundary is exactly 0.  Starting points are the Panter-Dite
    high-rate points (quantiles of f^(1/3)).  ``n_iter`` iterations are run; the
    loop stops early only when an iteration leaves every centroid bit-identical
    (a floating-point fixed point, after which further iterations change
    nothing).

    [turboquant_serve, "Keys vs values" and "Codebook sharing": codebooks are
    fitted once and shared]; [TorbuQuant, "Current Status"];
    [turboquant_pro, "TurboQuant -- rotate + scalar-quantize": precomputed
    Lloyd-Max boundaries].
    """
    levels = 1 << bits
    half = levels // 2
    q = (half + np.arange(half) + 0.5) / levels
    c = np.asarray(density.panter_dite_quantile(q), dtype=np.float64)
    iters = 0
    for it in range(n_iter):
        edges = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [density.support_hi]])
        lo, hi = edges[:-1], edges[1:]
        c_new = density.first_moment(lo, hi) / density.mass(lo, hi)
        iters = it + 1
        if np.array_equal(c_new, c):
            break
        c = c_new
    upper_mid = 0.5 * (c[:-1] + c[1:])
    centroids = np.concatenate([-c[::-1], c])
    boundaries = np.concatenate([-upper_mid[::-1], [0.0], upper_mid])
    return Codebook(centroids=centroids, boundaries=boundaries,
                    iterations_run=iters, n_iter=n_iter)


def lloyd_max_beta(dim: int, bits: int, n_iter: int) -> Codebook:
    """Lloyd-Max codebook for the D-dimensional Beta-sphere coordinate density."""
    return lloyd_max(BetaSphereDensity(dim), bits, n_iter)


def lloyd_max_gaussian(bits: int, n_iter: int) -> Codebook:
    """Lloyd-Max codebook for N(0, 1)."""
    return lloyd_max(GaussianDensity(), bits, n_iter)


def lloyd_max_gaussian_dim(dim: int, bits: int, n_iter: int) -> Codebook:
    """Gaussian-approximation codebook of dimension D: the Lloyd-Max quantizer of
    N(0, 1/D), the large-D limit of one coordinate of a uniform unit vector.

    [TorbuQuant, "Current Status": Lloyd-Max codebooks, "exact Beta-sphere and
    Gaussian approximation"].  The optimal quantizer of sigma X is sigma times that of
    X (the two Lloyd-Max conditions are scale-equivariant), so this is the N(0, 1)
    codebook with centroids and boundaries multiplied by 1/sqrt(D).
    """
    cb = lloyd_max_gaussian(bits, n_iter)
    s = 1.0 / math.sqrt(dim)
    return Codebook(centroids=cb.centroids * s, boundaries=cb.boundaries * s,
                    iterations_run=cb.iterations_run, n_iter=cb.n_iter)


def codebook_distortion(density, cb: Codebook) -> float:
    """Mean squared error E[(X - Q(X))^2] of a codebook under ``density``.

    Per cell: E[x^2] - 2 c E[x] + c^2 P, with E[x^2] by composite Gauss-Legendre.
    """
    edges = np.concatenate([[-density.support_hi], cb.boundaries, [density.support_hi]])
    nodes, weights = np.polynomial.legendre.leggauss(64)
    total = 0.0
    for i, ci in enumerate(cb.centroids):
        lo, hi = edges[i], edges[i + 1]
        if math.isinf(lo):
            lo = -12.0
        if math.isinf(hi):
            hi = 12.0
        panels = np.linspace(lo, hi, 17)
        for a, b in zip(panels[:-1], panels[1:]):
            x = 0.5 * (b - a) * nodes + 0.5 * (b + a)
            total += 0.5 * (b - a) * np.sum(weights * (x - ci) ** 2 * density.pdf(x))
    return float(total)


@dataclass
class CodebookTable:
    """fp32 table consumed by both paths: centroids (L) and boundaries (L-1)."""

    dim: int
    bits: int
    density_id: int
    n_iter: int
    iterations_run: int
    centroids: np.ndarray   # float32, length L
    boundaries: np.ndarray  # float32, length L-1


def to_fp32_table(cb: Codebook, dim: int, bits: int, density_id: int) -> CodebookTable:
    """Round a float64 codebook to the fp32 table (round to nearest even)."""
    return CodebookTable(dim=dim, bits=bits, density_id=density_id, n_iter=cb.n_iter,
                         iterations_run=cb.iterations_run,
                         centroids=cb.centroids.astype(np.float32),
                         boundaries=cb.boundaries.astype(np.float32))


# ---------------------------------------------------------------------------
# Slot layout
# ---------------------------------------------------------------------------


def region_bytes(dim: int, bits: int) -> int:
    """Bytes of one K or V region: ceil(D * bits / 8) packed index bytes + 4 norm bytes.

    [TorbuQuant, "TQ4 page tensor": K bytes ceil(D*k_bits/8)+4, V bytes
    ceil(D*v_bits/8)+4].
    """
    return (dim * bits + 7) // 8 + 4


def slot_bytes(dim: int, k_bits: int, v_bits: int) -> int:
    """slot_bytes = K bytes + V bytes (before any padding). [TorbuQuant, "TQ4 page tensor"]."""
    return region_bytes(dim, k_bits) + region_bytes(dim, v_bits)


def slot_position(slot: int, block_size: int):
    """(block, row) of a slot: block = slot // block_size, row = slot % block_size.

    [TorbuQuant, "TQ4 page tensor"].
    """
    return slot // block_size, slot % block_size


# ---------------------------------------------------------------------------
# Encode, pack, unpack
# ---------------------------------------------------------------------------


def encode(u: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """Cell index of each coordinate: idx = #{i : b_i < u} (ties to the lower cell).

    [turboquant_pro, "TurboQuant -- rotate + scalar-quantize": quantize each
    coordinate with precomputed Lloyd-Max boundaries].  ``boundaries`` are the
    fp32 table values, compared exactly as float64.
    """
    b = np.asarray(boundaries, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    return np.sum(b[None, :] < u.reshape(-1, 1), axis=1).reshape(u.shape).astype(np.int64)


def pack_bits(idx: np.ndarray, bits: int) -> np.ndarray:
    """Pack the last axis of ``idx`` into ceil(D*bits/8) bytes, LSB-first.

    Index j fills bits [j*bits, (j+1)*bits) of the stream; stream bit p is bit
    p % 8 of byte p // 8.  [turboquant_pro, "How It Works": 8 x 3-bit = 3 bytes];
    [TorbuQuant, "TQ4 page tensor": packed K / V indices].
    """
    idx = np.asarray(idx, dtype=np.int64)
    d = idx.shape[-1]
    lead = idx.shape[:-1]
    flat = idx.reshape(-1, d)
    nbytes = (d * bits + 7) // 8
    out = np.zeros((flat.shape[0], nbytes), dtype=np.uint8)
    for j in range(d):
        for k in range(bits):
            p = j * bits + k
            bit = (flat[:, j] >> k) & 1
            out[:, p // 8] |= (bit << (p % 8)).astype(np.uint8)
    return out.reshape(*lead, nbytes)


def unpack_bits(packed: np.ndarray, dim: int, bits: int) -> np.ndarray:
    """Inverse of ``pack_bits``: read ``dim`` indices of ``bits`` bits each."""
    packed = np.asarray(packed, dtype=np.uint8)
    lead = packed.shape[:-1]
    flat = packed.reshape(-1, packed.shape[-1]).astype(np.int64)
    out = np.zeros((flat.shape[0], dim), dtype=np.int64)
    for j in range(dim):
        for k in range(bits):
            p = j * bits + k
            out[:, j] |= ((flat[:, p // 8] >> (p % 8)) & 1) << k
    return out.reshape(*lead, dim)


# ---------------------------------------------------------------------------
# Quantize a row and build its slot region
# ---------------------------------------------------------------------------

QUIET_NAN_F32 = np.array([0x7FC00000], dtype=np.uint32).view(np.float32)[0]


def quantize_rows(x: np.ndarray, signs: np.ndarray, table: CodebookTable):
    """Rotate, take the norm, normalise and encode each row of ``x`` (..., D).

    Returns (idx int64 (..., D), norm float32 (...), u float64 (..., D),
    nonfinite bool (...)).

    Steps [TorbuQuant, "Quantize": rotate, normalize, codebook-encode, pack];
    [turboquant_pro, "How It Works": the L2 norm is preserved alongside the
    bits]:
      y = (1/sqrt(D)) H (s * x);  n = ||x||_2;  u = y / n;  idx = encode(u).
    ``signs`` is the RHT sign vector, or a DenseRotation (then y = R x).
    A zero row stores n = 0 and encodes u = 0.  A row with a non-finite value
    stores all-zero indices and a quiet-NaN norm.
    """
    x = np.asarray(x, dtype=np.float64)
    lead = x.shape[:-1]
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    nonfinite = ~np.all(np.isfinite(rows), axis=1)
    safe = np.where(nonfinite[:, None], 0.0, rows)
    y = rotate_forward(safe, signs)
    n = np.sqrt(np.sum(safe * safe, axis=1))
    u = np.where(n[:, None] > 0, y / np.where(n > 0, n, 1.0)[:, None], 0.0)
    idx = encode(u, table.boundaries)
    idx[nonfinite] = 0
    norm32 = n.astype(np.float32)
    norm32[nonfinite] = QUIET_NAN_F32
    return (idx.reshape(*lead, d), norm32.reshape(lead), u.reshape(*lead, d),
            nonfinite.reshape(lead))


def encode_region(idx: np.ndarray, norm32: np.ndarray, bits: int) -> np.ndarray:
    """Region bytes: packed indices, then the fp32 norm in little-endian order.

    [TorbuQuant, "TQ4 page tensor": K region = packed K indices, fp32 norm].
    """
    packed = pack_bits(idx, bits)
    nb = np.asarray(norm32, dtype="<f4").reshape(*packed.shape[:-1], 1).view(np.uint8)
    return np.concatenate([packed, nb.reshape(*packed.shape[:-1], 4)], axis=-1)


def decode_region(region: np.ndarray, dim: int, bits: int):
    """Split region bytes into (idx int64 (..., D), norm float32 (...)).

    [TorbuQuant, "TQ4 page tensor": a K or V region is the packed indices, then
    the fp32 norm].  The first ceil(D*bits/8) bytes are unpacked LSB-first
    (``unpack_bits``); the next four bytes are the norm, little endian.  Pinned
    against regions laid out by hand, bit by bit, with the norm written by
    ``struct`` (tests/test_oracle_pack_encode.py).
    """
    region = np.asarray(region, dtype=np.uint8)
    nb = (dim * bits + 7) // 8
    idx = unpack_bits(region[..., :nb], dim, bits)
    norm = np.ascontiguousarray(region[..., nb:nb + 4]).view("<f4")[..., 0]
    return idx, norm.astype(np.float32)


# ---------------------------------------------------------------------------
# Quantize-append into pages
# ---------------------------------------------------------------------------


def quantize_append(pages: np.ndarray, slot_mapping: np.ndarray, k: np.ndarray,
                    v: np.ndarray, k_table: CodebookTable, v_table: CodebookTable,
                    sign_seed: int, rotation=None) -> np.ndarray:
    """Quantize every (token, KV head) row of K and V and store it in its slot.

    pages        uint8 [num_blocks, block_size, H_kv, slot_stride] (a copy is returned)
    slot_mapping int   [T]; entries < 0 are skipped
    k, v         [T, H_kv, D] (any real dtype; converted exactly to float64)

    Slot of token t: block = slot // block_size, row = slot % block_size; its
    bytes are page[block, row, h, :]: K region then V region; padding bytes
    beyond slot_bytes are left untouched.  [TorbuQuant, "TQ4 page tensor" and
    the "Store" stage]; [turboquant_serve, "Architecture": update() rotates,
    encodes and stores both k and v].  The same sign vector serves K and V and
    every head ([turboquant_serve, "Rotation": one fixed matrix per head_dim]).
    ``rotation``: a DenseRotation to use instead of the RHT of ``sign_seed``.
    """
    pages = np.array(pages, dtype=np.uint8, copy=True)
    num_blocks, block_size, h_kv, stride = pages.shape
    t, hk, d = k.shape
    assert hk == h_kv and v.shape == k.shape
    kb = region_bytes(d, k_table.bits)
    vb = region_bytes(d, v_table.bits)
    assert kb + vb <= stride
    signs = rotation if rotation is not None else rht_signs(d, sign_seed)
    ki, kn, _, _ = quantize_rows(np.asarray(k, dtype=np.float64), signs, k_table)
    vi, vn, _, _ = quantize_rows(np.asarray(v, dtype=np.float64), signs, v_table)
    kreg = encode_region(ki, kn, k_table.bits)
    vreg = encode_region(vi, vn, v_table.bits)
    for tok in range(t):
        slot = int(slot_mapping[tok])
        if slot < 0:
            continue
        blk, row = slot_position(slot, block_size)
        if blk >= num_blocks:
            raise IndexError("slot outside the page pool")
        pages[blk, row, :, :kb] = kreg[tok]
        pages[blk, row, :, kb:kb + vb] = vreg[tok]
    return pages


# ---------------------------------------------------------------------------
# Dequantize and attend
# ---------------------------------------------------------------------------


def dequantize_rows(idx: np.ndarray, norm32: np.ndarray, table: CodebookTable,
                    signs: np.ndarray) -> np.ndarray:
    """x_hat = norm * R^T c[idx] in float64 on the fp32 table values (``signs``: the
    RHT sign vector, or a DenseRotation).

    [turboquant_serve, "Architecture": unpack + Lloyd-Max decode -> restore
    magnitude -> multiply by R transposed]; [turboquant_pro, "How It Works":
    then invert].
    """
    c = np.asarray(table.centroids, dtype=np.float64)[np.asarray(idx)]
    return np.asarray(norm32, dtype=np.float64)[..., None] * rotate_inverse(c, signs)


def gather_sequence(pages: np.ndarray, block_table_row: np.ndarray, seq_len: int):
    """Slot bytes of tokens 0..seq_len-1 of one sequence: [seq_len, H_kv, slot_stride].

    Token t lives in block block_table_row[t // block_size], row t % block_size.
    [TorbuQuant, "TQ4 page tensor": slot -> block, row].
    """
    block_size = pages.shape[1]
    tok = np.arange(seq_len)
    blocks = np.asarray(block_table_row)[tok // block_size]
    return pages[blocks, tok % block_size]


def paged_decode(q: np.ndarray, pages: np.ndarray, block_table: np.ndarray,
                 seq_lens: np.ndarray, k_table: CodebookTable,
                 v_table: CodebookTable, sign_seed: int, scale: float,
                 rotation=None) -> np.ndarray:
    """One decode step over packed pages, by the plain definition.

    q [B, H_q, D]; returns o [B, H_q, D] float64.  For each sequence b and query
    head h (KV head h // G): dequantize every cached K and V row, then
    s_t = scale <q, k_hat_t>, p = softmax(s) (max-subtracted, float64),
    o = sum_t p_t v_hat_t.  A sequence of length 0 gives o = 0.

    [turboquant_serve, "Architecture": _decode then attention];
    [tq-kv, "Library API": scores from the compressed keys with a softmax scale].
    ``rotation``: a DenseRotation to use instead of the RHT of ``sign_seed``.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, h_q, d = q.shape
    h_kv = pages.shape[2]
    g = h_q // h_kv
    kb = region_bytes(d, k_table.bits)
    vb = region_bytes(d, v_table.bits)
    signs = rotation if rotation is not None else rht_signs(d, sign_seed)
    out = np.zeros((bsz, h_q, d), dtype=np.float64)
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        slots = gather_sequence(pages, block_table[b], n)          # [n, H_kv, stride]
        ki, kn = decode_region(slots[..., :kb], d, k_table.bits)
        vi, vn = decode_region(slots[..., kb:kb + vb], d, v_table.bits)
        khat = dequantize_rows(ki, kn, k_table, signs)               # [n, H_kv, D]
        vhat = dequantize_rows(vi, vn, v_table, signs)
        for h in range(h_q):
            kv = h // g
            s = scale * (khat[:, kv, :] @ q[b, h])
            s = s - np.max(s)
            p = np.exp(s)
            p /= np.sum(p)
            out[b, h] = p @ vhat[:, kv, :]
    return out


def rotated_domain_partial(q_rot: np.ndarray, k_idx: np.ndarray, k_norm: np.ndarray,
                           v_idx: np.ndarray, v_norm: np.ndarray, k_table: CodebookTable,
                           v_table: CodebookTable, scale: float):
    """Attention of one query over a token range, computed on the codes.

    q_rot [D] is the rotated query R q.  Scores s_t = scale * n_K,t * sum_j
    q_rot_j c_K[idx_t,j]; returns the un-normalised partial (m, l, O') with
    m = max s, l = sum exp(s - m), O' = sum exp(s - m) n_V,t c_V[idx_t] (still in
    the rotated domain).  [tq-kv, "Library API": pre_rotate_query_with_signs and
    fused_attention_scores]; [tq-kv, "Custom CUDA Kernel Stack": flash decode v2
    with split-KV and online softmax].
    """
    ck = np.asarray(k_table.centroids, dtype=np.float64)[k_idx]
    cv = np.asarray(v_table.centroids, dtype=np.float64)[v_idx]
    s = scale * np.asarray(k_norm, dtype=np.float64) * (ck @ q_rot)
    m = np.max(s)
    e = np.exp(s - m)
    return m, np.sum(e), (e * np.asarray(v_norm, dtype=np.float64)) @ cv


def merge_partials(parts):
    """Combine split partials (m_i, l_i, O'_i): m = max m_i, l = sum e^(m_i-m) l_i,
    O' = sum e^(m_i-m) O'_i / l.  [tq-kv, "Custom CUDA Kernel Stack": split-KV]."""
    m = max(p[0] for p in parts)
    l = sum(math.exp(p[0] - m) * p[1] for p in parts)
    o = sum(math.exp(p[0] - m) * p[2] for p in parts)
    return o / l


def paged_decode_rotated(q: np.ndarray, pages: np.ndarray, block_table: np.ndarray,
                         seq_lens: np.ndarray, k_table: CodebookTable,
                         v_table: CodebookTable, sign_seed: int, scale: float,
                         split_tokens: int = 0) -> np.ndarray:
    """The decode as the fused kernels compute it: rotate q once, score on codes,
    online softmax over token splits, V in the rotated domain, one inverse
    rotation of the output.  Equal to ``paged_decode`` in exact arithmetic.

    [tq-kv, "Library API"]; [turboquant_pro, "Fused CUDA decode": split-K decode
    on the codes without reconstruction].
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, h_q, d = q.shape
    h_kv = pages.shape[2]
    g = h_q // h_kv
    kb = region_bytes(d, k_table.bits)
    vb = region_bytes(d, v_table.bits)
    signs = rht_signs(d, sign_seed)
    out = np.zeros((bsz, h_q, d), dtype=np.float64)
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        slots = gather_sequence(pages, block_table[b], n)
        ki, kn = decode_region(slots[..., :kb], d, k_table.bits)
        vi, vn = decode_region(slots[..., kb:kb + vb], d, v_table.bits)
        step = split_tokens if split_tokens > 0 else n
        for h in range(h_q):
            kv = h // g
            qr = rht_forward(q[b, h], signs)
            parts = [rotated_domain_partial(qr, ki[s:s + step, kv], kn[s:s + step, kv],
                                            vi[s:s + step, kv], vn[s:s + step, kv],
                                            k_table, v_table, scale)
                     for s in range(0, n, step)]
            out[b, h] = rht_inverse(merge_partials(parts), signs)
    return out


# ---------------------------------------------------------------------------
# Decode with an uncompressed hot window
# ---------------------------------------------------------------------------


def paged_decode_hot(q: np.ndarray, pages: np.ndarray, block_table: np.ndarray,
                     seq_lens: np.ndarray, hot_k: np.ndarray, hot_v: np.ndarray,
                     hot_lens: np.ndarray, k_table: CodebookTable, v_table: CodebookTable,
                     sign_seed: int, scale: float, rotation=None) -> np.ndarray:
    """One decode step over the packed pages plus an uncompressed hot window.

    [turboquant_pro, "Fused CUDA decode": the fp16 hot window is merged with the
    compressed tokens through the online softmax; "Streaming cache": recent tokens
    stay uncompressed]; [tq-kv, "How It Works", "3-Fix for GGUF Models": the sink
    tokens stay in FP16 and the current token is lossless].

    q [B, H_q, D]; hot_k, hot_v [B, W, H_kv, D] (any real dtype, read exactly);
    hot_lens [B]: sequence b attends to its seq_lens[b] packed tokens (dequantized
    as in ``paged_decode``) and to hot tokens 0 .. hot_lens[b]-1, in one softmax over
    all of them: s_t = scale <q, k_t>, o = sum_t softmax(s)_t v_t.  Which positions the
    hot tokens held (the first few, the most recent) does not enter the result.  A
    sequence with no tokens at all gives 0.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, h_q, d = q.shape
    h_kv = pages.shape[2]
    g = h_q // h_kv
    kb = region_bytes(d, k_table.bits)
    vb = region_bytes(d, v_table.bits)
    signs = rht_signs(d, sign_seed)
    if rotation is not None:
        signs = rotation
    hk = np.asarray(hot_k, dtype=np.float64)
    hv = np.asarray(hot_v, dtype=np.float64)
    out = np.zeros((bsz, h_q, d), dtype=np.float64)
    for b in range(bsz):
        n, w = int(seq_lens[b]), int(hot_lens[b])
        if n + w == 0:
            continue
        keys = np.zeros((0, h_kv, d))
        vals = np.zeros((0, h_kv, d))
        if n > 0:
            slots = gather_sequence(pages, block_table[b], n)
            ki, kn = decode_region(slots[..., :kb], d, k_table.bits)
            vi, vn = decode_region(slots[..., kb:kb + vb], d, v_table.bits)
            keys = dequantize_rows(ki, kn, k_table, signs)
            vals = dequantize_rows(vi, vn, v_table, signs)
        keys = np.concatenate([keys, hk[b, :w]], axis=0)            # [n + w, H_kv, D]
        vals = np.concatenate([vals, hv[b, :w]], axis=0)
        for h in range(h_q):
            kv = h // g
            s = scale * (keys[:, kv, :] @ q[b, h])
            p = np.exp(s - np.max(s))
            out[b, h] = (p / np.sum(p)) @ vals[:, kv, :]
    return out


# ---------------------------------------------------------------------------
# QJL residual sketch of the keys
# ---------------------------------------------------------------------------

QJL_CONST = math.sqrt(math.pi / 2.0)


def qjl_region_bytes(dim: int) -> int:
    """Bytes the QJL sketch adds to a K region: D sign bits, then the fp32 residual norm."""
    return dim // 8 + 4


def k_region_bytes(dim: int, bits: int, qjl: bool) -> int:
    return region_bytes(dim, bits) + (qjl_region_bytes(dim) if qjl else 0)


def qjl_sketch(r: np.ndarray, qjl_signs: np.ndarray):
    """1-bit sketch of the residual r (..., D): z = [S r >= 0] with S = (1/sqrt(D)) H
    diag(s'), a second randomized Hadamard transform with its own seeded signs
    (tq-kv, "How It Works" step [5]: SRHT QJL error correction; TorbuQuant, "Current
    Status": QJL residual).  Returns (z int64 (..., D) in {0, 1}, gamma = ||r||_2)."""
    r = np.asarray(r, dtype=np.float64)
    z = (rht_forward(r, qjl_signs) >= 0.0).astype(np.int64)
    return z, np.sqrt(np.sum(r * r, axis=-1))


def qjl_correction(z: np.ndarray, gamma: np.ndarray, qjl_signs: np.ndarray) -> np.ndarray:
    """The residual estimate gamma sqrt(pi/2) / sqrt(D) S^T (2z - 1), in the rotated
    domain: its inner product with a rotated query y is the QJL estimator
    gamma sqrt(pi/2) / sqrt(D) <S y, sign(S r)> of <y, r> (unbiased over the sketch's
    signs for large D)."""
    d = np.asarray(z).shape[-1]
    zpm = 2.0 * np.asarray(z, dtype=np.float64) - 1.0
    return (np.asarray(gamma, dtype=np.float64)[..., None] * QJL_CONST / math.sqrt(d)
            * rht_inverse(zpm, qjl_signs))


def quantize_keys_qjl(x: np.ndarray, rot, table: CodebookTable, qjl_signs: np.ndarray):
    """Keys with the QJL residual: the MSE quantizer of ``quantize_rows``, then the 1-bit
    sketch of the rotated-domain residual r = u - c[idx].  Returns (idx, norm float32,
    z, gamma float32, u, nonfinite); a non-finite row stores z = 0 and gamma = 0."""
    idx, n32, u, bad = quantize_rows(x, rot, table)
    c = np.asarray(table.centroids, dtype=np.float64)[idx]
    r = np.where(bad[..., None], 0.0, u - c)
    z, gamma = qjl_sketch(r, qjl_signs)
    z = np.where(bad[..., None], 0, z)
    return idx, n32, z, gamma.astype(np.float32), u, bad


def encode_k_region_qjl(idx, norm32, z, gamma32, bits: int) -> np.ndarray:
    """K region with the sketch: packed codes, fp32 norm, D sign bits (LSB-first, bit j
    = z_j), fp32 residual norm gamma (little endian)."""
    head = encode_region(idx, norm32, bits)
    zb = pack_bits(z, 1)
    g = np.asarray(gamma32, dtype="<f4").reshape(*zb.shape[:-1], 1).view(np.uint8)
    return np.concatenate([head, zb, g.reshape(*zb.shape[:-1], 4)], axis=-1)


def decode_k_region_qjl(region: np.ndarray, dim: int, bits: int):
    """(idx, norm float32, z, gamma float32) of a K region written by encode_k_region_qjl."""
    region = np.asarray(region, dtype=np.uint8)
    rb = region_bytes(dim, bits)
    idx, norm = decode_region(region[..., :rb], dim, bits)
    z = unpack_bits(region[..., rb:rb + dim // 8], dim, 1)
    g = np.ascontiguousarray(region[..., rb + dim // 8:rb + dim // 8 + 4]).view("<f4")[..., 0]
    return idx, norm, z, g.astype(np.float32)


def dequantize_keys_qjl(idx, norm32, z, gamma32, table: CodebookTable, rot,
                        qjl_signs: np.ndarray) -> np.ndarray:
    """k_hat = norm R^T (c[idx] + qjl_correction): the key whose inner product with any q
    is the QJL-corrected score norm (<R q, c> + gamma sqrt(pi/2)/sqrt(D) <S R q, 2z-1>)."""
    c = np.asarray(table.centroids, dtype=np.float64)[np.asarray(idx)]
    w = c + qjl_correction(z, gamma32, qjl_signs)
    return np.asarray(norm32, dtype=np.float64)[..., None] * rotate_inverse(w, rot)


def quantize_append_qjl(pages: np.ndarray, slot_mapping: np.ndarray, k: np.ndarray,
                        v: np.ndarray, k_table: CodebookTable, v_table: CodebookTable,
                        sign_seed: int, qjl_seed: int) -> np.ndarray:
    """quantize_append with the QJL sketch in the K region: slot = [K codes | K norm |
    sketch bits | gamma][V codes | V norm] (the V region as before)."""
    pages = np.array(pages, dtype=np.uint8, copy=True)
    num_blocks, block_size, h_kv, stride = pages.shape
    t, hk, d = k.shape
    kb = k_region_bytes(d, k_table.bits, True)
    vb = region_bytes(d, v_table.bits)
    assert hk == h_kv and kb + vb <= stride
    signs = rht_signs(d, sign_seed)
    ki, kn, kz, kg, _, _ = quantize_keys_qjl(np.asarray(k, dtype=np.float64), signs, k_table,
                                             rht_signs(d, qjl_seed))
    vi, vn, _, _ = quantize_rows(np.asarray(v, dtype=np.float64), signs, v_table)
    kreg = encode_k_region_qjl(ki, kn, kz, kg, k_table.bits)
    vreg = encode_region(vi, vn, v_table.bits)
    for tok in range(t):
        slot = int(slot_mapping[tok])
        if slot < 0:
            continue
        blk, row = slot_position(slot, block_size)
        pages[blk, row, :, :kb] = kreg[tok]
        pages[blk, row, :, kb:kb + vb] = vreg[tok]
    return pages


def paged_decode_qjl(q: np.ndarray, pages: np.ndarray, block_table: np.ndarray,
                     seq_lens: np.ndarray, k_table: CodebookTable, v_table: CodebookTable,
                     sign_seed: int, qjl_seed: int, scale: float) -> np.ndarray:
    """paged_decode over slots written by quantize_append_qjl: the keys dequantized with
    their QJL correction, then plain softmax attention."""
    q = np.asarray(q, dtype=np.float64)
    bsz, h_q, d = q.shape
    h_kv = pages.shape[2]
    g = h_q // h_kv
    kb = k_region_bytes(d, k_table.bits, True)
    vb = region_bytes(d, v_table.bits)
    signs = rht_signs(d, sign_seed)
    qs = rht_signs(d, qjl_seed)
    out = np.zeros((bsz, h_q, d), dtype=np.float64)
    for b in range(bsz):
        n = int(seq_lens[b])
        if n == 0:
            continue
        slots = gather_sequence(pages, block_table[b], n)
        ki, kn, kz, kg = decode_k_region_qjl(slots[..., :kb], d, k_table.bits)
        vi, vn = decode_region(slots[..., kb:kb + vb], d, v_table.bits)
        khat = dequantize_keys_qjl(ki, kn, kz, kg, k_table, signs, qs)
        vhat = dequantize_rows(vi, vn, v_table, signs)
        for h in range(h_q):
            kv = h // g
            s = scale * (khat[:, kv, :] @ q[b, h])
            p = np.exp(s - np.max(s))
            out[b, h] = (p / np.sum(p)) @ vhat[:, kv, :]
    return out
