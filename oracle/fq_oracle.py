"""FibQuant CPU oracle: a plain, slow, fp64 restatement of the method (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may import this
module.  The product path (the CUDA library and its Python binding) never imports, links or
runs it, and it shares no code, header, table generator or helper with that path.

Sources (cited by page and section):
  [FQ]   "FibQuant: Universal Vector Quantization for Random-Access KV-Cache Compression",
         gist.science technical summary (zh and fr editions, same section numbering) and the
         paper's English abstract on its Hugging Face paper page.
  [TQ]   "TurboQuant: Online Vector Quantization with Near-optimal Distortion Rate", blog notes
         (leeon-k.github.io), the scalar codec that FibQuant's k = 1 case reduces to.
  [BQ]   "Block Sphere Vector Quantization", NeurIPS 2026 paper notes (papernotes.org), an
         independent block-sphere VQ with the same canonical block source.

Conventions: a vector x has d coordinates; blocks have k coordinates; d' = k * ceil(d / k)
(x is zero-padded to d' when k does not divide d); m = d' / k blocks; N codewords; B = log2 N
bits per block index; P = ceil(m B / 8) payload bytes per record.  The rotation acts on
column vectors, z = Pi x.  Everything is float64 unless a step fixes another precision.

Parity status of each part is listed in the test files that pin it; every function below
except ``attention_*`` on real-model weights (not available) is pinned by at least one
check against a closed form, an invariant, a printed number or brute force.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
from scipy import special
from scipy.spatial import cKDTree

PHI = (1.0 + math.sqrt(5.0)) / 2.0
GOLDEN_ANGLE = 2.0 * math.pi * (2.0 - PHI)  # 2.39996... rad


# --------------------------------------------------------------------------------------
# Parameters: rate and record size.  [FQ] sec. 2.3 "rate": b = log2(N) / k bits per coordinate;
# [FQ] sec. 1: records are fixed-size at fixed addresses (random access).
# --------------------------------------------------------------------------------------

def padded_dim(d: int, k: int) -> int:
    """d' = k ceil(d / k): zero padding when k does not divide d (a reading: [FQ] sec. 2.3
    speaks of d/k blocks, and [BQ] 'limitations' requires the block size to divide d)."""
    return k * ((d + k - 1) // k)


def index_bits(N: int) -> int:
    B = int(round(math.log2(N)))
    if N < 2 or (1 << B) != N or N > 65536:
        raise ValueError("N must be a power of two in [2, 65536]")
    return B


def payload_bytes(d: int, k: int, N: int) -> int:
    m = padded_dim(d, k) // k
    return (m * index_bits(N) + 7) // 8


def rate_bits_per_coord(k: int, N: int) -> float:
    """[FQ] sec. 2.3: b = log2(N) / k."""
    return math.log2(N) / k


# --------------------------------------------------------------------------------------
# Haar rotation.  [TQ] sec. 3.1: draw a matrix with iid N(0,1) entries and take its QR
# decomposition.  The sign correction Q diag(sign(diag R)) makes Q exactly Haar
# (standard result; a plain QR alone is not Haar).
# --------------------------------------------------------------------------------------

def haar_rotation(dp: int, seed: int, sign_fix: bool = True) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    G = rng.standard_normal((dp, dp))
    Q, R = np.linalg.qr(G)
    if sign_fix:
        s = np.sign(np.diag(R))
        s[s == 0] = 1.0
        Q = Q * s[None, :]
    return Q


# --------------------------------------------------------------------------------------
# The canonical source.  [FQ] sec. 2.1 / Thm 1: after normalisation and a Haar rotation,
# any k consecutive coordinates follow the spherical-Beta density f_{d,k} on the unit ball.
# [BQ] key design 1 gives the density
#     f_{d,k}(z) = Gamma(d/2) / (pi^{k/2} Gamma((d-k)/2)) (1 - |z|^2)^{(d-k-2)/2},
# with |z|^2 ~ Beta(k/2, (d-k)/2) independent of a uniform direction.
# [TQ] sec. 2 lemma: the k = 1 case, f_X(x) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1-x^2)^{(d-3)/2}.
# --------------------------------------------------------------------------------------

def block_density(z: np.ndarray, d: int, k: int) -> np.ndarray:
    r2 = np.sum(np.asarray(z, dtype=np.float64) ** 2, axis=-1)
    logc = special.gammaln(d / 2) - (k / 2) * math.log(math.pi) - special.gammaln((d - k) / 2)
    out = np.zeros_like(r2)
    inside = r2 < 1.0
    out[inside] = np.exp(logc + ((d - k - 2) / 2) * np.log1p(-r2[inside]))
    return out


def coord_density(x: np.ndarray, d: int) -> np.ndarray:
    return block_density(np.asarray(x, dtype=np.float64)[..., None], d, 1)


def block_r2_law(d: int, k: int) -> tuple[float, float]:
    """Beta parameters of |z_j|^2 for a k-block of a uniform point on S^{d-1}."""
    return k / 2.0, (d - k) / 2.0


def sample_source_blocks(M: int, d: int, k: int, rng: np.random.Generator) -> np.ndarray:
    """M iid draws from f_{d,k}: radius^2 ~ Beta(k/2,(d-k)/2) times a uniform direction.  For
    the full-vector block (k = d) the block is the whole unit vector: radius 1, uniform on the
    sphere (the Beta law degenerates at b = 0)."""
    a, b = block_r2_law(d, k)
    r = np.sqrt(rng.beta(a, b, size=M)) if k < d else np.ones(M)
    u = rng.standard_normal((M, k))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    return u * r[:, None]


# --------------------------------------------------------------------------------------
# Codebook initialisation.  [FQ] sec. 2.2: radii from Bennett-Gersho companding of the
# radial density (closed form for k = 2), directions from a planar Fibonacci spiral (k = 2),
# a Fibonacci sphere (k = 3) or a Roberts-Kronecker sequence (k >= 4).
#
# Companding (a reading; the summary names the rule, not the formula): the Bennett-Gersho
# optimal point density in k dimensions is lambda ~ f^{k/(k+2)}.  For f_{d,k} this is
# (1 - r^2)^{a} with a = k (d-k-2) / (2 (k+2)); in polar form the squared radius of a point
# drawn from lambda is Beta(k/2, a + 1).  Radii are its quantiles at levels (n + 1/2) / N.
# For k = 2 the Beta(1, beta) quantile is closed form: r^2 = 1 - (1 - q)^{1/beta}, beta = d/4.
# --------------------------------------------------------------------------------------

def companded_r2_law(d: int, k: int) -> tuple[float, float]:
    return k / 2.0, 1.0 + k * (d - k - 2) / (2.0 * (k + 2))


def quantile_levels(N: int) -> np.ndarray:
    return (np.arange(N, dtype=np.float64) + 0.5) / N


def init_radii(d: int, k: int, N: int) -> np.ndarray:
    """Companded Beta-quantile radii, increasing in n (general path: inverse incomplete beta).
    Full-vector codes (k = d) put every codeword on the unit sphere: the block is the whole unit
    vector, so all bits go to the angular packing ([FQ] sec. 4.2 on full-vector codes)."""
    if k >= d:
        return np.ones(N)
    a, b = companded_r2_law(d, k)
    return np.sqrt(special.betaincinv(a, b, quantile_levels(N)))


def init_radii_k2_closed_form(d: int, N: int) -> np.ndarray:
    """k = 2 closed form of the same quantiles ([FQ] sec. 2.2 says k = 2 is closed form)."""
    beta = companded_r2_law(d, 2)[1]
    q = quantile_levels(N)
    return np.sqrt(1.0 - (1.0 - q) ** (1.0 / beta))


def bit_reverse(n: np.ndarray, bits: int) -> np.ndarray:
    n = np.asarray(n, dtype=np.int64)
    out = np.zeros_like(n)
    for b in range(bits):
        out |= ((n >> b) & 1) << (bits - 1 - b)
    return out


def roberts_root(k: int) -> float:
    """Positive root g of g^{k+1} = g + 1 (the generalised golden ratio of the R_k sequence)."""
    g = 1.5
    for _ in range(200):
        g -= (g ** (k + 1) - g - 1.0) / ((k + 1) * g ** k - 1.0)
    return g


def init_directions(k: int, N: int) -> np.ndarray:
    """Unit directions u_n, n = 0..N-1.

    k = 2: angle n * golden angle (Vogel / sunflower spiral, the 'golden quantizer').
    k = 3: Fibonacci sphere: height 1 - (2n+1)/N, azimuth n * golden angle.
    k >= 4: Roberts-Kronecker points t_n = frac(1/2 + (n+1) alpha), alpha_i = g^{-i}, mapped to
            the sphere through the normal quantile function and normalisation.
    """
    n = np.arange(N, dtype=np.float64)
    if k == 2:
        th = n * GOLDEN_ANGLE
        return np.stack([np.cos(th), np.sin(th)], axis=1)
    if k == 3:
        h = 1.0 - (2.0 * n + 1.0) / N
        rho = np.sqrt(np.maximum(0.0, 1.0 - h * h))
        ph = n * GOLDEN_ANGLE
        return np.stack([rho * np.cos(ph), rho * np.sin(ph), h], axis=1)
    if k >= 4:
        g = roberts_root(k)
        alpha = g ** (-np.arange(1, k + 1, dtype=np.float64))
        t = np.mod(0.5 + (n[:, None] + 1.0) * alpha[None, :], 1.0)
        v = special.ndtri(t)
        return v / np.linalg.norm(v, axis=1, keepdims=True)
    raise ValueError("k >= 2 for vector directions")


def init_codebook(d: int, k: int, N: int) -> np.ndarray:
    """Deterministic radial-angular initial codebook C0 [N, k] (fp64).

    k = 2 pairs radius n with direction n (radius grows along the spiral).  For k >= 3 the
    radius of codeword n takes quantile level bitrev(n) (a reading: pairing is not given;
    bit reversal decorrelates radius from the direction sequence).
    """
    r = init_radii(d, k, N)
    u = init_directions(k, N)
    if k >= 3:
        r = r[bit_reverse(np.arange(N), index_bits(N))]
    return u * r[:, None]


# --------------------------------------------------------------------------------------
# Scalar Lloyd-Max on the coordinate law ([TQ] sec. 3.1: a 1-D continuous k-means on f_X,
# boundaries at midpoints of sorted centroids).  Solved on the continuous density, not on
# samples: cell probability and first moment are closed form, the cost uses quadrature.
# --------------------------------------------------------------------------------------

def _coord_cdf(x: np.ndarray, d: int) -> np.ndarray:
    a = (d - 1) / 2.0
    return special.betainc(a, a, np.clip((1.0 + np.asarray(x)) / 2.0, 0.0, 1.0))


def _coord_first_moment(lo: np.ndarray, hi: np.ndarray, d: int) -> np.ndarray:
    """int_lo^hi x f_X(x) dx = C_d/(d-1) [(1-lo^2)^{(d-1)/2} - (1-hi^2)^{(d-1)/2}]."""
    logc = special.gammaln(d / 2) - 0.5 * math.log(math.pi) - special.gammaln((d - 1) / 2)
    e = (d - 1) / 2.0
    f = lambda t: np.power(np.clip(1.0 - t * t, 0.0, None), e)
    return math.exp(logc) / (d - 1) * (f(lo) - f(hi))


def scalar_lloyd(d: int, N1: int, iters: int = 2000, tol: float = 1e-15) -> np.ndarray:
    """Optimal N1-level scalar quantizer of f_X at dimension d (sorted centroids)."""
    from scipy.special import betaincinv
    a = (d - 1) / 2.0
    c = 2.0 * betaincinv(a, a, quantile_levels(N1)) - 1.0
    for _ in range(iters):
        edges = np.concatenate([[-1.0], (c[1:] + c[:-1]) / 2.0, [1.0]])
        p = _coord_cdf(edges[1:], d) - _coord_cdf(edges[:-1], d)
        m1 = _coord_first_moment(edges[:-1], edges[1:], d)
        c_new = m1 / p
        if np.max(np.abs(c_new - c)) < tol:
            c = c_new
            break
        c = c_new
    return c


def scalar_mse_per_coord(c: np.ndarray, d: int) -> float:
    """E (X - Q(X))^2 under f_X for the scalar quantizer with sorted centroids c."""
    from scipy.integrate import quad
    edges = np.concatenate([[-1.0], (c[1:] + c[:-1]) / 2.0, [1.0]])
    tot = 0.0
    for i, ci in enumerate(c):
        val, _ = quad(lambda x: (x - ci) ** 2 * coord_density(np.array(x), d), edges[i],
                      edges[i + 1], epsabs=1e-15, epsrel=1e-12, limit=200)
        tot += val
    return tot


def product_codebook(c1: np.ndarray, k: int) -> np.ndarray:
    """k-fold Cartesian product of a scalar codebook (the scalar product specialisation)."""
    grids = np.meshgrid(*([c1] * k), indexing="ij")
    return np.stack([g.reshape(-1) for g in grids], axis=1)


# --------------------------------------------------------------------------------------
# Multi-restart Lloyd-Max refinement ([FQ] sec. 2.2; objective: [BQ] key design 1, k-means
# under f_{d,k}).  Hyper-parameters are not on the pages (readings):
#   training set: M = max(2^18, 256 N) seeded draws from f_{d,k};
#   iteration: exact nearest-codeword assignment, centroid = cell mean, an empty cell keeps
#   its codeword; stop when the relative drop of the training MSE is below 1e-7 or after
#   max_iter iterations;
#   restarts: 0 = deterministic init; 1..R-2 = init + Gaussian jitter of 0.25 x the median
#   nearest-neighbour spacing; R-1 = the scalar product codebook when N = N1^k, else one
#   more jitter restart; the restart with the lowest training MSE wins.
# --------------------------------------------------------------------------------------

def assign_exact(samples: np.ndarray, C: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Exact nearest codeword (ties have probability zero on continuous samples).  A k-d tree
    for small blocks; for blocks of more than 8 coordinates (where a tree prunes nothing) plain
    brute force by chunked matrix products, argmin of |c|^2 - 2 s.c, then the direct-form
    squared distance of the chosen codeword."""
    C = np.asarray(C, dtype=np.float64)
    if C.shape[1] <= 8:
        dist, idx = cKDTree(C).query(samples, k=1, workers=-1)
        return idx.astype(np.int64), dist * dist
    cc = np.sum(C * C, axis=1)
    idx = np.empty(samples.shape[0], dtype=np.int64)
    step = max(1, (1 << 25) // C.shape[0])
    for s0 in range(0, samples.shape[0], step):
        blk = samples[s0:s0 + step]
        idx[s0:s0 + step] = np.argmin(cc[None, :] - 2.0 * (blk @ C.T), axis=1)
    d2 = np.sum((samples - C[idx]) ** 2, axis=1)
    return idx, d2


def lloyd(C0: np.ndarray, samples: np.ndarray, max_iter: int = 300, tol: float = 1e-7):
    """Returns (C, history of training MSE per block, one entry per assignment)."""
    C = np.array(C0, dtype=np.float64, copy=True)
    N, k = C.shape
    idx, d2 = assign_exact(samples, C)
    mse = float(d2.mean())
    hist = [mse]
    for _ in range(max_iter):
        cnt = np.bincount(idx, minlength=N).astype(np.float64)
        sums = np.zeros_like(C)
        for i in range(k):
            sums[:, i] = np.bincount(idx, weights=samples[:, i], minlength=N)
        nz = cnt > 0
        C[nz] = sums[nz] / cnt[nz, None]
        idx, d2 = assign_exact(samples, C)
        new = float(d2.mean())
        hist.append(new)
        done = (mse - new) <= tol * mse
        mse = new
        if done:
            break
    return C, hist


def _perfect_root(N: int, k: int) -> int | None:
    r = int(round(N ** (1.0 / k)))
    for c in (r - 1, r, r + 1):
        if c >= 2 and c ** k == N:
            return c
    return None


def median_nn_spacing(C: np.ndarray) -> float:
    dist, _ = cKDTree(C).query(C, k=2)
    return float(np.median(dist[:, 1]))


@dataclass
class CodebookInfo:
    d: int
    k: int
    N: int
    seed: int
    restarts: int
    max_iter: int
    M: int
    train_mse: list = field(default_factory=list)   # final training MSE per restart
    iters: list = field(default_factory=list)
    best: int = 0


def build_codebook(d: int, k: int, N: int, seed: int = 101, restarts: int = 8,
                   max_iter: int = 300, M: int | None = None, tol: float = 1e-7):
    """FibQuant codebook for (d', k, N): returns (C [N,k] float64, CodebookInfo)."""
    if M is None:
        M = max(1 << 18, 256 * N)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, d, k, N])))
    samples = sample_source_blocks(M, d, k, rng)
    C0 = init_codebook(d, k, N)
    spacing = median_nn_spacing(C0)
    N1 = _perfect_root(N, k)
    info = CodebookInfo(d, k, N, seed, restarts, max_iter, M)
    best = None
    for r in range(restarts):
        if r == 0:
            init = C0
        elif r == restarts - 1 and N1 is not None and restarts > 1:
            init = product_codebook(scalar_lloyd(d, N1), k)
        else:
            jr = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, d, k, N, r])))
            init = C0 + 0.25 * spacing * jr.standard_normal(C0.shape)
        C, hist = lloyd(init, samples, max_iter=max_iter, tol=tol)
        info.train_mse.append(hist[-1])
        info.iters.append(len(hist) - 1)
        if best is None or hist[-1] < best[1]:
            best = (C, hist[-1], r)
    info.best = best[2]
    return best[0], info


def block_mse(samples: np.ndarray, C: np.ndarray) -> float:
    """Mean squared error per block of the nearest-codeword quantizer C on samples."""
    return float(assign_exact(samples, C)[1].mean())


# --------------------------------------------------------------------------------------
# Encoder ([FQ] sec. 2.3): nu = |x|_2, unit vector rotated, z = Pi x / nu, split into
# m blocks of k consecutive coordinates, nearest codeword per block in the shared codebook.
# The norm is stored as fp16 (round to nearest even).  Readings: a zero vector (outside
# Thm 1, which covers nonzero inputs) encodes as all-zero indices and norm +0; ties go to
# the lowest index; distances use the direct form sum (z - c)^2.
# --------------------------------------------------------------------------------------

@dataclass
class Encoded:
    idx: np.ndarray     # [n, m] int64
    norms: np.ndarray   # [n] float16 (bits: norms.view(np.uint16))
    gap: np.ndarray     # [n, m] second-best minus best squared distance (inf when N == 1)
    z: np.ndarray       # [n, d'] unit rotated vectors (zeros for nu = 0)
    nu: np.ndarray      # [n] exact norms (float64)


def rotate_unit(x: np.ndarray, rot: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    dp = padded_dim(d, k)
    R = np.asarray(rot, dtype=np.float64)
    assert R.shape == (dp, dp)
    xp = np.zeros((n, dp))
    xp[:, :d] = x
    nu = np.sqrt(np.sum(x * x, axis=1))
    z = xp @ R.T
    nz = nu > 0
    z[nz] /= nu[nz, None]
    z[~nz] = 0.0
    return z, nu


def nearest_codeword(zb: np.ndarray, C: np.ndarray, chunk: int = 1 << 16):
    """Brute force over all N codewords: (argmin, gap) for blocks zb [.., k]."""
    C = np.asarray(C, dtype=np.float64)
    chunk = max(1, min(chunk, (1 << 24) // (C.shape[0] * C.shape[1])))  # bounded temporaries
    flat = zb.reshape(-1, C.shape[1])
    idx = np.empty(flat.shape[0], dtype=np.int64)
    gap = np.empty(flat.shape[0])
    for s in range(0, flat.shape[0], chunk):
        blk = flat[s:s + chunk]
        dist = np.sum((blk[:, None, :] - C[None, :, :]) ** 2, axis=2)
        i = np.argmin(dist, axis=1)  # first occurrence = lowest index on ties
        idx[s:s + chunk] = i
        if C.shape[0] > 1:
            two = np.partition(dist, 1, axis=1)[:, :2]
            gap[s:s + chunk] = two[:, 1] - two[:, 0]
        else:
            gap[s:s + chunk] = np.inf
    return idx.reshape(zb.shape[:-1]), gap.reshape(zb.shape[:-1])


def encode(x: np.ndarray, rot: np.ndarray, codebook: np.ndarray, k: int) -> Encoded:
    C = np.asarray(codebook, dtype=np.float64)
    z, nu = rotate_unit(x, rot, k)
    n, dp = z.shape
    m = dp // k
    idx, gap = nearest_codeword(z.reshape(n, m, k), C)
    idx[nu == 0] = 0
    norms = nu.astype(np.float16)  # NumPy converts float64 -> float16 with round-half-even
    return Encoded(idx, norms, gap, z, nu)


# --------------------------------------------------------------------------------------
# Fixed-rate record ([FQ] sec. 1 and 2.3).  Reading of the layout: index j occupies record
# bits [jB, (j+1)B), least significant bit first; record bit i lives in byte i // 8 at bit
# i % 8; unused tail bits are zero.  Norms live in a separate fp16 plane at the same token
# offset (structure-of-arrays; every token is still at a fixed address).
# --------------------------------------------------------------------------------------

def pack(idx: np.ndarray, N: int) -> np.ndarray:
    B = index_bits(N)
    n, m = idx.shape
    P = (m * B + 7) // 8
    codes = np.zeros((n, P), dtype=np.uint8)
    idx = np.asarray(idx, dtype=np.int64)
    for j in range(m):
        for b in range(B):
            pos = j * B + b
            bit = ((idx[:, j] >> b) & 1).astype(np.uint8)
            codes[:, pos // 8] |= (bit << (pos % 8)).astype(np.uint8)
    return codes


def unpack(codes: np.ndarray, m: int, N: int) -> np.ndarray:
    B = index_bits(N)
    codes = np.asarray(codes, dtype=np.uint8)
    idx = np.zeros((codes.shape[0], m), dtype=np.int64)
    for j in range(m):
        for b in range(B):
            pos = j * B + b
            bit = (codes[:, pos // 8] >> (pos % 8)) & 1
            idx[:, j] |= bit.astype(np.int64) << b
    return idx


# --------------------------------------------------------------------------------------
# Decoder ([FQ] sec. 2.3): fetch the codewords, concatenate the blocks, apply the inverse
# rotation Pi^T ([TQ] sec. 3.1), scale by the stored norm; padded coordinates are dropped.
# --------------------------------------------------------------------------------------

def decode_idx(idx: np.ndarray, norms_f16: np.ndarray, rot: np.ndarray, codebook: np.ndarray,
               d: int) -> np.ndarray:
    C = np.asarray(codebook, dtype=np.float64)
    n, m = idx.shape
    zhat = C[idx].reshape(n, m * C.shape[1])
    xr = zhat @ np.asarray(rot, dtype=np.float64)  # rows: (Pi^T zhat)^T = zhat^T Pi
    nu = np.asarray(norms_f16, dtype=np.float16).astype(np.float64)
    return nu[:, None] * xr[:, :d]


def decode(codes: np.ndarray, norms_f16: np.ndarray, rot: np.ndarray, codebook: np.ndarray,
           d: int, k: int, N: int) -> np.ndarray:
    m = padded_dim(d, k) // k
    return decode_idx(unpack(codes, m, N), norms_f16, rot, codebook, d)


# --------------------------------------------------------------------------------------
# Decode attention over a compressed cache (the consumer that [FQ] sec. 5 says the fixed-
# address interface keeps fusable).  Readings: one query token per (batch, head); query head
# h reads kv head h // (Hq / Hkv); scores q.k * scale with scale = 1/sqrt(d) of the original
# d; no mask; softmax with the maximum subtracted.
# --------------------------------------------------------------------------------------

def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - np.max(s, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_exact(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(q K^T scale) V for q [B,Hq,d], K/V [B,Hkv,T,d] (any float dtype, fp64 math)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Bn, Hq, d = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.empty((Bn, Hq, V.shape[-1]))
    for b in range(Bn):
        for h in range(Hq):
            g = h // G
            p = _softmax(K[b, g] @ q[b, h] * scale)
            out[b, h] = p @ V[b, g]
    return out


@dataclass
class CompressedKV:
    codes: np.ndarray   # [B, Hkv, T, P] uint8
    norms: np.ndarray   # [B, Hkv, T] float16
    rot: np.ndarray     # [d', d'] (fp32 data)
    codebook: np.ndarray
    k: int
    N: int


def attention_decoded(q: np.ndarray, Kc: CompressedKV, Vc: CompressedKV, d: int,
                      scale: float) -> np.ndarray:
    """Attention over the fully decoded caches (what the CUDA attention is checked against)."""
    Bn, Hkv, T, _ = Kc.codes.shape
    Kh = decode(Kc.codes.reshape(-1, Kc.codes.shape[-1]), Kc.norms.reshape(-1), Kc.rot,
                Kc.codebook, d, Kc.k, Kc.N).reshape(Bn, Hkv, T, d)
    Vh = decode(Vc.codes.reshape(-1, Vc.codes.shape[-1]), Vc.norms.reshape(-1), Vc.rot,
                Vc.codebook, d, Vc.k, Vc.N).reshape(Bn, Hkv, T, d)
    return attention_exact(q, Kh, Vh, scale)


def attention_lut(q: np.ndarray, Kc: CompressedKV, Vc: CompressedKV, d: int,
                  scale: float) -> np.ndarray:
    """The rotated-domain form: q~ = Pi_K pad(q) once; per-block LUT[j][c] = q~_j . C_K[c];
    s_t = nu_t sum_j LUT[j][idx_tj] scale; values accumulated as sum_t p_t nu_t zhat_t in the
    rotated domain and inverse-rotated once.  Algebraically identical to attention_decoded."""
    q = np.asarray(q, dtype=np.float64)
    Bn, Hq, _ = q.shape
    _, Hkv, T, _ = Kc.codes.shape
    G = Hq // Hkv
    dpk = padded_dim(d, Kc.k)
    dpv = padded_dim(d, Vc.k)
    mk, mv = dpk // Kc.k, dpv // Vc.k
    CK = np.asarray(Kc.codebook, dtype=np.float64)
    CV = np.asarray(Vc.codebook, dtype=np.float64)
    RK = np.asarray(Kc.rot, dtype=np.float64)
    RV = np.asarray(Vc.rot, dtype=np.float64)
    out = np.empty((Bn, Hq, d))
    for b in range(Bn):
        for g in range(Hkv):
            ik = unpack(Kc.codes[b, g], mk, Kc.N)
            iv = unpack(Vc.codes[b, g], mv, Vc.N)
            nk = Kc.norms[b, g].astype(np.float64)
            nv = Vc.norms[b, g].astype(np.float64)
            zv = CV[iv].reshape(T, dpv)
            for h in range(g * G, (g + 1) * G):
                qp = np.zeros(dpk)
                qp[:d] = q[b, h]
                qt = RK @ qp
                lut = qt.reshape(mk, Kc.k) @ CK.T                      # [mk, N]
                s = nk * lut[np.arange(mk)[None, :], ik].sum(axis=1) * scale
                p = _softmax(s)
                acc = (p * nv) @ zv                                   # rotated domain
                out[b, h] = (RV.T @ acc)[:d]
    return out


def cosine(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.sum(a * b, -1) / (np.linalg.norm(a, axis=-1) * np.linalg.norm(b, axis=-1))


# --------------------------------------------------------------------------------------
# Cartesian grid-LUT candidate pruning ([BQ] key design 2): partition the block space into a
# grid of L cells per axis, keep for every cell the c codewords nearest its centre, and
# search only those.  Approximate by design.  Readings: the grid spans [-R, R]^k with
# R = max |codeword coordinate| + 3/sqrt(d'); coordinates outside clamp to the edge cell;
# cell i covers [-R + i h, -R + (i+1) h), h = 2R / L; candidates are ordered by distance to
# the centre (ties: lower index); the search keeps the lowest index on distance ties.
# --------------------------------------------------------------------------------------

def grid_range(codebook: np.ndarray, dp: int) -> float:
    return float(np.max(np.abs(codebook))) + 3.0 / math.sqrt(dp)


def grid_cells(zb: np.ndarray, R: float, L: int) -> np.ndarray:
    h = 2.0 * R / L
    c = np.floor((np.asarray(zb, dtype=np.float64) + R) / h).astype(np.int64)
    return np.clip(c, 0, L - 1)


def grid_topc_table(codebook: np.ndarray, R: float, L: int, c: int) -> np.ndarray:
    """[L^k, c] candidate ids; the flat cell id is sum_i cell_i L^i (axis 0 fastest)."""
    C = np.asarray(codebook, dtype=np.float64)
    k = C.shape[1]
    h = 2.0 * R / L
    f = np.arange(L ** k, dtype=np.int64)
    cells = np.stack([(f // L ** i) % L for i in range(k)], axis=1)
    centres = -R + (cells + 0.5) * h
    table = np.empty((centres.shape[0], c), dtype=np.int64)
    for s in range(0, centres.shape[0], 4096):
        cc = centres[s:s + 4096]
        dist = np.sum((cc[:, None, :] - C[None, :, :]) ** 2, axis=2)
        order = np.argsort(dist, axis=1, kind="stable")
        table[s:s + 4096] = order[:, :c]
    return table


def flat_cell(cells: np.ndarray, L: int) -> np.ndarray:
    k = cells.shape[-1]
    w = L ** np.arange(k)
    return np.sum(cells * w, axis=-1)


def encode_grid_topc(x: np.ndarray, rot: np.ndarray, codebook: np.ndarray, k: int, L: int,
                     c: int):
    """Encoder with the approximate grid search.  Returns (Encoded, boundary distance per
    block: the smallest distance of z_j to a cell face it could cross, for parity exemptions)."""
    C = np.asarray(codebook, dtype=np.float64)
    z, nu = rotate_unit(x, rot, k)
    n, dp = z.shape
    m = dp // k
    R = grid_range(C, dp)
    h = 2.0 * R / L
    table = grid_topc_table(C, R, L, c)
    zb = z.reshape(n, m, k)
    cells = grid_cells(zb, R, L)
    fid = flat_cell(cells, L)
    cand = table[fid]                                     # [n, m, c]
    cz = C[cand]                                          # [n, m, c, k]
    dist = np.sum((zb[:, :, None, :] - cz) ** 2, axis=3)  # [n, m, c]
    # lowest codeword index among equal distances
    best = np.full((n, m), np.inf)
    idx = np.zeros((n, m), dtype=np.int64)
    for i in range(c):
        better = (dist[:, :, i] < best) | ((dist[:, :, i] == best) & (cand[:, :, i] < idx))
        best = np.where(better, dist[:, :, i], best)
        idx = np.where(better, cand[:, :, i], idx)
    idx[nu == 0] = 0
    gap = np.full((n, m), np.inf)
    if c > 1:
        two = np.partition(dist, 1, axis=2)[:, :, :2]
        gap = two[:, :, 1] - two[:, :, 0]
    t = (zb + R) / h
    nearest_face = np.clip(np.round(t), 1, L - 1)
    bd = (np.abs(t - nearest_face) * h).min(axis=2)
    norms = nu.astype(np.float16)
    return Encoded(idx, norms, gap, z, nu), bd


# --------------------------------------------------------------------------------------
# Variants (not on the measured path yet).
#
# [BQ] key design 3, target-aware scalar rescale: after the inverse rotation the unscaled
# reconstruction xbar = Pi^T zbar of a unit vector has a shrunk norm.  With the alignment
# rho = <z, zbar> (= <x, xbar> for unit x) the decoder scales xbar by
#   S = rho / |xbar|^2   (least squared reconstruction error),
#   S = 1 / rho          (inner products unbiased: the component along x becomes exact),
#   S = 1                (plain reconstruction, the rule of the measured path).
# rho is one more stored scalar per vector.  Readings: |xbar| = |zbar| (Pi is orthogonal, and
# the padded coordinates are kept before the final truncation to d); a zero vector stores
# rho = 1.
# --------------------------------------------------------------------------------------

RESCALE_RULES = ("mse", "unbiased", "plain")


def rescale_factor(rho: np.ndarray, zbar_sq: np.ndarray, rule: str) -> np.ndarray:
    """S of [BQ] key design 3 for alignment rho and squared reconstruction norm |zbar|^2."""
    rho = np.asarray(rho, dtype=np.float64)
    if rule == "mse":
        return rho / np.asarray(zbar_sq, dtype=np.float64)
    if rule == "unbiased":
        return 1.0 / rho
    if rule == "plain":
        return np.ones_like(rho)
    raise ValueError(rule)


def encode_rescaled(x: np.ndarray, rot: np.ndarray, codebook: np.ndarray, k: int):
    """The encoder plus rho = <z, zbar> per vector.  Returns (Encoded, rho)."""
    enc = encode(x, rot, codebook, k)
    C = np.asarray(codebook, dtype=np.float64)
    n, dp = enc.z.shape
    zbar = C[enc.idx].reshape(n, dp)
    rho = np.sum(enc.z * zbar, axis=1)
    rho[enc.nu == 0] = 1.0
    return enc, rho


def decode_rescaled(idx: np.ndarray, norms_f16: np.ndarray, rho: np.ndarray, rot: np.ndarray,
                    codebook: np.ndarray, d: int, rule: str) -> np.ndarray:
    """x_hat = nu * S * (Pi^T zbar)[0:d] with S from `rule` ([BQ] key design 3)."""
    C = np.asarray(codebook, dtype=np.float64)
    n, m = idx.shape
    zbar = C[idx].reshape(n, m * C.shape[1])
    S = rescale_factor(rho, np.sum(zbar * zbar, axis=1), rule)
    xr = zbar @ np.asarray(rot, dtype=np.float64)
    nu = np.asarray(norms_f16, dtype=np.float16).astype(np.float64)
    return (nu * S)[:, None] * xr[:, :d]


# --------------------------------------------------------------------------------------
# [TQ] sec. 2.2 (QJL, a 1-bit inner-product quantizer): for x in R^d,
#   Q_qjl(x) = sign(S x),  Q_qjl^{-1}(q) = sqrt(pi/2) / d * S^T q,
# with S a d x d matrix of iid N(0, 1) entries (drawn here from a seeded PCG64 generator and
# passed in).  Reading: sign(0) = +1.
# [TQ] sec. 3.1 (TurboQuant_mse): y = Pi x, each coordinate of y to its nearest centroid of the
# scalar Lloyd-Max codebook c1 of the coordinate law; dequantize Pi^T c1[idx].
# [TQ] sec. 3.2 (TurboQuant_prod, inner-product optimal, b bits): Q_mse at b - 1 bits, then
# Q_qjl of the residual r = x - Q_mse^{-1}(Q_mse(x)) and gamma = |r|_2; the estimate is
#   Q_mse^{-1}(Q_mse(x)) + gamma * Q_qjl^{-1}(Q_qjl(r)).
# All vectors are rows; x is on the unit sphere (the norm is stored separately, as above).
# --------------------------------------------------------------------------------------

def qjl_matrix(d: int, seed: int) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal((d, d))


def qjl_quantize(x: np.ndarray, S: np.ndarray) -> np.ndarray:
    s = np.atleast_2d(np.asarray(x, dtype=np.float64)) @ S.T   # rows of (S x)^T
    return np.where(s >= 0.0, 1.0, -1.0)


def qjl_dequantize(q: np.ndarray, S: np.ndarray) -> np.ndarray:
    d = S.shape[0]
    return math.sqrt(math.pi / 2.0) / d * (np.atleast_2d(q) @ S)  # rows of (S^T q)^T


def turboquant_mse_quantize(x: np.ndarray, rot: np.ndarray, c1: np.ndarray) -> np.ndarray:
    y = np.atleast_2d(np.asarray(x, dtype=np.float64)) @ np.asarray(rot, dtype=np.float64).T
    return np.argmin(np.abs(y[:, :, None] - np.asarray(c1)[None, None, :]), axis=2)


def turboquant_mse_dequantize(idx: np.ndarray, rot: np.ndarray, c1: np.ndarray) -> np.ndarray:
    return np.asarray(c1, dtype=np.float64)[idx] @ np.asarray(rot, dtype=np.float64)


def turboquant_prod_quantize(x: np.ndarray, rot: np.ndarray, c1: np.ndarray, S: np.ndarray):
    """(idx of Q_mse at the bits of c1, QJL signs of the residual, gamma = |residual|)."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    idx = turboquant_mse_quantize(x, rot, c1)
    r = x - turboquant_mse_dequantize(idx, rot, c1)
    return idx, qjl_quantize(r, S), np.linalg.norm(r, axis=1)


def turboquant_prod_dequantize(idx: np.ndarray, q: np.ndarray, gamma: np.ndarray,
                               rot: np.ndarray, c1: np.ndarray, S: np.ndarray) -> np.ndarray:
    return (turboquant_mse_dequantize(idx, rot, c1) +
            np.asarray(gamma, dtype=np.float64)[:, None] * qjl_dequantize(q, S))


# --------------------------------------------------------------------------------------
# Random access and the decode-step write path (not on the measured path yet).  [FQ] sec. 1:
# records are fixed-size at fixed addresses, so any token decodes alone (gather-decode of a
# token list) and a sequence can end at any length (per-sequence context lengths).  A decode
# step that appends its own token encodes that token's key and value into the next record slot
# of its sequence and attends over the cache including it.  Readings: a length counts tokens
# from position 0; records past a sequence's length are never read (they may hold anything).
# --------------------------------------------------------------------------------------

def decode_tokens(codes: np.ndarray, norms_f16: np.ndarray, token_ids, rot: np.ndarray,
                  codebook: np.ndarray, d: int, k: int, N: int) -> np.ndarray:
    """Decode only the records at token_ids (any order, repeats allowed) of a [T, P] plane."""
    ids = np.asarray(token_ids, dtype=np.int64)
    return decode(np.asarray(codes)[ids], np.asarray(norms_f16)[ids], rot, codebook, d, k, N)


def _slice_cache(c: CompressedKV, b: int, length: int) -> CompressedKV:
    return CompressedKV(c.codes[b:b + 1, :, :length], c.norms[b:b + 1, :, :length], c.rot,
                        c.codebook, c.k, c.N)


def attention_decoded_lengths(q: np.ndarray, Kc: CompressedKV, Vc: CompressedKV, d: int,
                              scale: float, lengths) -> np.ndarray:
    """attention_decoded with sequence b limited to its first lengths[b] >= 1 tokens."""
    q = np.asarray(q, dtype=np.float64)
    out = np.empty(q.shape)
    for b, length in enumerate(np.asarray(lengths, dtype=np.int64)):
        out[b:b + 1] = attention_decoded(q[b:b + 1], _slice_cache(Kc, b, int(length)),
                                         _slice_cache(Vc, b, int(length)), d, scale)
    return out


def _write_token(c: CompressedKV, x_new: np.ndarray, lengths: np.ndarray) -> CompressedKV:
    """Encode x_new [B, Hkv, d] and store each row in record slot lengths[b] of its sequence."""
    Bn, Hkv, d = x_new.shape
    enc = encode(x_new.reshape(Bn * Hkv, d), c.rot, c.codebook, c.k)
    rec = pack(enc.idx, c.N).reshape(Bn, Hkv, -1)
    codes, norms = c.codes.copy(), c.norms.copy()
    for b in range(Bn):
        codes[b, :, lengths[b]] = rec[b]
        norms[b, :, lengths[b]] = enc.norms.reshape(Bn, Hkv)[b]
    return CompressedKV(codes, norms, c.rot, c.codebook, c.k, c.N)


def append_and_attend(q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, Kc: CompressedKV,
                      Vc: CompressedKV, d: int, scale: float, lengths):
    """One decode step with its own token: k_new, v_new [B, Hkv, d] are encoded into slot
    lengths[b] of each sequence (the caches need room), then the step attends over
    lengths[b] + 1 tokens.  Returns (out, new key cache, new value cache, new lengths)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    K2 = _write_token(Kc, np.asarray(k_new), lengths)
    V2 = _write_token(Vc, np.asarray(v_new), lengths)
    return attention_decoded_lengths(q, K2, V2, d, scale, lengths + 1), K2, V2, lengths + 1
