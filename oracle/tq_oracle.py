"""Plain fp64 CPU oracle for TurboQuant KV-cache quantization and decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it.  It shares no code, tables or constants with the
CUDA library; the two meet only through the seeded input generators in
``kv_inputs.py`` (which hold none of the method's arithmetic).

Everything here is written for a reader checking it against the pages by eye:
fp64 throughout, whole-array numpy steps, no blocking or fusion.

Sources (page title, section):
  [P3] "TurboQuant-MLX: quantizzare pesi e KV cache per LLM open-weight su Mac",
       sections "Il metodo TurboQuant, in breve", "Cosa aggiunge turboquant-mlx",
       "I numeri dichiarati".
  [P2] "Greetings from TurboQuant-MLX & Some Insights to Share!" (turboquant_plus
       issue 59), items 1-3 (attention sink, 64-token chunks, sparse V).
  [P5] "Why TurboQuant saves DGX twice" (NVIDIA developer forum): PolarQuant +
       QJL residual correction, 3.5-bit, no calibration, online per token.

Readings where the pages are silent are marked [reading] where they are
used.  Pins: every function below is checked by
``tests/test_oracle_pins.py`` against something other than itself; none is
"parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from functools import lru_cache
from statistics import NormalDist

import numpy as np

# ---------------------------------------------------------------------------
# Counter-based random numbers: SplitMix64 (Steele, Lea, Flood 2014) and
# Box-Muller.  [reading] The pages only say the rotation is random and seeded
# ("lo si ruota prima a caso", [P3] "Il metodo TurboQuant, in breve"); the
# generator is our choice, implemented independently on each side from the
# published definition.
# ---------------------------------------------------------------------------
MASK64 = (1 << 64) - 1
SPLITMIX_GAMMA = 0x9E3779B97F4A7C15
TAG_ROTATION = 0
TAG_QJL = 1
TAG_HADAMARD_SIGNS = 2


def splitmix64(state0: int, count: int, start: int = 0) -> np.ndarray:
    """Outputs start..start+count-1 of SplitMix64 seeded with ``state0``.

    Output i is mix(state0 + (i+1)*gamma) with the published mixing function
    (xor-shift 30, multiply, xor-shift 27, multiply, xor-shift 31).
    """
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(state0 & MASK64) + i * np.uint64(SPLITMIX_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def stream_state(seed: int, tag: int) -> int:
    """Initial SplitMix64 state for one named stream: seed xor (tag << 32)."""
    return (int(seed) ^ (int(tag) << 32)) & MASK64


def uniforms(state0: int, count: int) -> np.ndarray:
    """Uniform doubles in (0, 1): ((z >> 11) + 0.5) * 2^-53."""
    z = splitmix64(state0, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def gaussians(seed: int, tag: int, count: int) -> np.ndarray:
    """Standard normals by Box-Muller on consecutive uniform pairs (u1, u2).

    Pair k gives r*cos(2*pi*u2) then r*sin(2*pi*u2), r = sqrt(-2 ln u1).
    """
    pairs = (count + 1) // 2
    u = uniforms(stream_state(seed, tag), 2 * pairs)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    theta = 2.0 * math.pi * u2
    out = np.empty(2 * pairs)
    out[0::2] = r * np.cos(theta)
    out[1::2] = r * np.sin(theta)
    return out[:count]


# ---------------------------------------------------------------------------
# Random rotation Pi and QJL matrix S.
# [P3] "Il metodo TurboQuant, in breve": rotate first, at random.  A dense Haar
# orthogonal matrix (QR of a Gaussian matrix with the sign of diag(R) folded
# into Q, Mezzadri 2007) is the plainest reading.  The port in [P3] "Cosa
# aggiunge turboquant-mlx" uses a Hadamard transform instead.
# ---------------------------------------------------------------------------

def rotation(seed: int, d: int) -> np.ndarray:
    """Pi (d x d, row-major), y = Pi @ u.  G = N(0,1)^{d x d} row-major fill."""
    g = gaussians(seed, TAG_ROTATION, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[None, :]


def hadamard_signs(seed: int, d: int) -> np.ndarray:
    """The random sign flips of the Hadamard rotation: s_j = -1 when the top
    bit of SplitMix64 output j of stream (seed, TAG_HADAMARD_SIGNS) is set,
    +1 otherwise."""
    z = splitmix64(stream_state(seed, TAG_HADAMARD_SIGNS), d)
    return np.where((z >> np.uint64(63)) == 1, -1.0, 1.0)


def walsh_hadamard(d: int) -> np.ndarray:
    """Sylvester's Walsh-Hadamard matrix: H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(d)
    bits = np.bitwise_and(i[:, None], i[None, :])
    pop = np.zeros_like(bits)
    while bits.any():
        pop += bits & 1
        bits >>= 1
    return np.where(pop % 2 == 1, -1.0, 1.0)


def hadamard_rotation(seed: int, d: int) -> np.ndarray:
    """[P3] "Cosa aggiunge turboquant-mlx": the port realizes the random
    rotation with a Hadamard transform.  Randomized with sign flips (the page
    gives no detail; the plainest reading): Pi = H D / sqrt(d), D = diag(s),
    so y = Pi u is the normalized Walsh-Hadamard transform of the sign-flipped
    u.  d must be a power of two."""
    if d <= 0 or d & (d - 1):
        raise ValueError("the Hadamard rotation needs d a power of two")
    return walsh_hadamard(d) * hadamard_signs(seed, d)[None, :] / math.sqrt(d)


def qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    """S (m x d) with i.i.d. N(0,1) entries, row-major fill."""
    return gaussians(seed, TAG_QJL, m * d).reshape(m, d)


# ---------------------------------------------------------------------------
# Lloyd-Max codebook for one coordinate of a uniform point on S^{d-1}.
# [P3] "Il metodo TurboQuant, in breve": after the rotation the coordinates
# follow a known distribution and each is quantized on its own with an optimal
# scalar quantizer; [P3] "Cosa aggiunge turboquant-mlx": Lloyd-Max codebook.
# Density f(x) = C (1 - x^2)^((d-3)/2) on [-1, 1],
# C = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)).
# ---------------------------------------------------------------------------
_GL_NODES, _GL_WEIGHTS = np.polynomial.legendre.leggauss(64)
_GL_PIECES = 16


def coord_log_const(d: int) -> float:
    return math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0)


def coord_density(x: np.ndarray, d: int) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    inside = np.abs(x) < 1.0
    xx = np.where(inside, x, 0.0)
    val = np.exp(coord_log_const(d) + 0.5 * (d - 3) * np.log1p(-xx * xx))
    return np.where(inside, val, 0.0)


def _support(d: int) -> float:
    """Half-width beyond which f is below exp(-750) of its peak."""
    return min(1.0, math.sqrt(-math.expm1(-1500.0 / max(d - 3, 1))))


def integrate(fun, a: np.ndarray, b: np.ndarray, d: int) -> np.ndarray:
    """Composite Gauss-Legendre integral of fun over [a_k, b_k] (vectorised).

    Limits are clipped to the support of f, where the integrands live.
    """
    lim = _support(d)
    a = np.clip(np.asarray(a, dtype=np.float64), -lim, lim)
    b = np.clip(np.asarray(b, dtype=np.float64), -lim, lim)
    edges = a[:, None] + (b - a)[:, None] * np.linspace(0.0, 1.0, _GL_PIECES + 1)[None, :]
    lo, hi = edges[:, :-1], edges[:, 1:]
    mid, half = 0.5 * (lo + hi), 0.5 * (hi - lo)
    x = mid[..., None] + half[..., None] * _GL_NODES
    return (fun(x) * _GL_WEIGHTS * half[..., None]).sum(axis=(-1, -2))


def cell_mass(a, b, d: int) -> np.ndarray:
    return integrate(lambda x: coord_density(x, d), a, b, d)


def cell_first_moment(a, b, d: int) -> np.ndarray:
    """int_a^b x f(x) dx = C/(d-1) [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)]."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)

    def prim(t):
        inside = np.abs(t) < 1.0
        tt = np.where(inside, t, 0.0)
        v = np.exp(coord_log_const(d) + 0.5 * (d - 1) * np.log1p(-tt * tt)) / (d - 1)
        return np.where(inside, v, 0.0)

    return prim(a) - prim(b)


@dataclass
class Codebook:
    d: int
    bits: int
    centroids: np.ndarray  # (2^bits,) ascending
    bounds: np.ndarray     # (2^bits - 1,) midpoints
    iterations: int


@lru_cache(maxsize=None)
def lloyd_max(d: int, bits: int, tol: float = 1e-15, max_iter: int = 100000) -> Codebook:
    """Lloyd-Max iteration for the coordinate density f.

    Start at Gaussian quantiles (variance 1/d); alternate
      t_k = (c_k + c_{k+1}) / 2             (nearest-neighbour boundaries)
      c_k = int x f / int f over [t_{k-1}, t_k]  (centroid condition)
    until no centroid moves by more than ``tol`` (relative to max |c|).
    Above 4 bits the plain iteration converges too slowly (its contraction
    approaches 1 as the levels grow), so the same two conditions are solved
    by Newton's method instead (lloyd_max_newton).
    """
    if bits > 4:
        return lloyd_max_newton(d, bits, tol)
    return lloyd_iteration(d, bits, tol, max_iter)


def lloyd_iteration(d: int, bits: int, tol: float = 1e-15, max_iter: int = 100000) -> Codebook:
    """The plain Lloyd-Max iteration of lloyd_max, for any number of bits."""
    levels = 1 << bits
    nd = NormalDist()
    c = np.array([nd.inv_cdf((k + 0.5) / levels) for k in range(levels)]) / math.sqrt(d)
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate(([-1.0], t))
        hi = np.concatenate((t, [1.0]))
        c_new = cell_first_moment(lo, hi, d) / cell_mass(lo, hi, d)
        moved = np.max(np.abs(c_new - c))
        c = c_new
        if moved <= tol * np.max(np.abs(c)):
            break
    return Codebook(d, bits, c, 0.5 * (c[:-1] + c[1:]), it)


def lloyd_max_newton(d: int, bits: int, tol: float = 1e-15, max_iter: int = 100, warm: int = 50) -> Codebook:
    """The fixed point of the Lloyd map of lloyd_max, T_k(c) = M1_k / M0_k
    (first moment over mass of f over [t_{k-1}, t_k], t_k the midpoints),
    found by Newton's method on G(c) = c - T(c).  With f_k = f(t_k):
      dT_k/dc_{k+1} = f_k (t_k - T_k) / (2 M0_k)
      dT_k/dc_{k-1} = f_{k-1} (T_k - t_{k-1}) / (2 M0_k)
      dT_k/dc_k     = the sum of the two
    so the Jacobian I - dT is tridiagonal.  Start: the high-resolution optimum
    for a Gaussian of variance 1/d (point density proportional to f^(1/3):
    Gaussian quantiles of variance 3/d), then ``warm`` plain Lloyd steps.
    Steps are halved while they do not reduce max |G| or break the order of
    the centroids.
    """
    levels = 1 << bits
    nd = NormalDist()
    c = np.array([nd.inv_cdf((k + 0.5) / levels) for k in range(levels)]) * math.sqrt(3.0 / d)

    def lloyd_map(c):
        t = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate(([-1.0], t))
        hi = np.concatenate((t, [1.0]))
        m0 = cell_mass(lo, hi, d)
        return cell_first_moment(lo, hi, d) / m0, m0, t

    for _ in range(warm):
        c = lloyd_map(c)[0]
    T, m0, t = lloyd_map(c)
    G = c - T
    it = 0
    for it in range(1, max_iter + 1):
        ft = coord_density(t, d)
        up = ft * (t - T[:-1]) / (2 * m0[:-1])   # dT_k/dc_{k+1}, k < L-1
        lo = ft * (T[1:] - t) / (2 * m0[1:])     # dT_{k+1}/dc_k
        jac = np.eye(levels)
        jac -= np.diag(np.concatenate((up, [0.0])) + np.concatenate(([0.0], lo)))
        jac -= np.diag(up, 1) + np.diag(lo, -1)
        step = np.linalg.solve(jac, -G)
        lam = 1.0
        while True:
            cn = c + lam * step
            if np.all(np.diff(cn) > 0) and cn[0] > -1.0 and cn[-1] < 1.0:
                Tn, m0n, tn = lloyd_map(cn)
                Gn = cn - Tn
                if np.max(np.abs(Gn)) < np.max(np.abs(G)) or lam < 1e-6:
                    break
            lam *= 0.5
        moved = np.max(np.abs(cn - c))
        c, T, m0, t, G = cn, Tn, m0n, tn, Gn
        if moved <= tol * np.max(np.abs(c)):
            break
    return Codebook(d, bits, c, 0.5 * (c[:-1] + c[1:]), it)


def mse_distortion(cb: Codebook) -> float:
    """D = d * sum_k int_{cell k} (x - c_k)^2 f(x) dx  (unit-vector MSE)."""
    c = cb.centroids
    lo = np.concatenate(([-1.0], cb.bounds))
    hi = np.concatenate((cb.bounds, [1.0]))
    per_cell = [
        integrate(lambda x, ck=ck: (x - ck) ** 2 * coord_density(x, cb.d),
                  lo[k:k + 1], hi[k:k + 1], cb.d)[0]
        for k, ck in enumerate(c)
    ]
    return cb.d * float(np.sum(per_cell))


# ---------------------------------------------------------------------------
# Row formats.  [reading] The pages fix only that codes are packed at "odd" bit
# widths ([P5]); the layout is ours: code j at bit offset j*b of the row, bits
# least-significant first inside little-endian bytes.  Mixed rows ([P3] "Il
# metodo TurboQuant, in breve": 3.5 bits per channel) put the first d/2
# rotated coordinates at b+1 bits, the rest at b bits.
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Format:
    bits: int          # total bits per channel (prod includes the QJL bit)
    prod: bool = False  # inner-product variant: (bits-1)-bit MSE + 1-bit QJL
    mixed: bool = False  # first d/2 coordinates at bits+1 (MSE only)

    def mse_bits(self, j: int, d: int) -> int:
        b = self.bits - 1 if self.prod else self.bits
        return b + 1 if (self.mixed and j < d // 2) else b

    def code_bytes(self, d: int) -> int:
        return sum(self.mse_bits(j, d) for j in range(d)) // 8


def pack_codes(idx: np.ndarray, widths: list[int]) -> np.ndarray:
    """Pack rows of codes (n, d) with per-coordinate widths into bytes."""
    n, d = idx.shape
    bits = []
    for j in range(d):
        w = widths[j]
        for k in range(w):
            bits.append((idx[:, j] >> k) & 1)
    if not bits:
        return np.zeros((n, 0), dtype=np.uint8)
    stream = np.stack(bits, axis=1).astype(np.uint8)
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_codes(packed: np.ndarray, widths: list[int]) -> np.ndarray:
    n = packed.shape[0]
    stream = np.unpackbits(packed, axis=1, bitorder="little").astype(np.int64)
    out = np.zeros((n, len(widths)), dtype=np.int64)
    pos = 0
    for j, w in enumerate(widths):
        for k in range(w):
            out[:, j] |= stream[:, pos] << k
            pos += 1
    return out


# ---------------------------------------------------------------------------
# Quantizer.
# ---------------------------------------------------------------------------

@dataclass
class Params:
    d: int
    fmt_k: Format
    fmt_v: Format
    seed: int = 0
    m: int = 128
    rotation: str = "haar"   # "haar" (dense Haar Pi) or "hadamard" (sign flips + Walsh-Hadamard)
    pi: np.ndarray = field(init=False)
    s: np.ndarray = field(init=False)
    books: dict = field(init=False)

    def __post_init__(self):
        if self.rotation == "haar":
            self.pi = rotation(self.seed, self.d)
        elif self.rotation == "hadamard":
            self.pi = hadamard_rotation(self.seed, self.d)
        else:
            raise ValueError(f"unknown rotation {self.rotation!r}")
        self.s = qjl_matrix(self.seed, self.m, self.d)
        self.books = {}
        for f in (self.fmt_k, self.fmt_v):
            for j in range(self.d):
                b = f.mse_bits(j, self.d)
                if b > 0 and b not in self.books:
                    self.books[b] = lloyd_max(self.d, b)

    def fmt(self, which: str) -> Format:
        return self.fmt_k if which == "k" else self.fmt_v


@dataclass
class Packed:
    codes: np.ndarray      # (n, code_bytes) uint8
    norms: np.ndarray      # (n,) float32, nu = ||x||
    qjl: np.ndarray        # (n, m/8) uint8 (prod) or (n, 0)
    res_norms: np.ndarray  # (n,) float32, gamma = ||r|| (prod) or zeros


def quantize(p: Params, x: np.ndarray, which: str = "k") -> Packed:
    """Rotate, quantize each coordinate, pack; prod adds the QJL sign sketch.

    [P3] "Il metodo TurboQuant, in breve":
      nu = ||x||, u = x / nu  ([reading] the known density is that of a unit
      vector, so the norm is kept on the side in fp32)
      y = Pi u
      idx_j = #{k : t_k < y_j}  (nearest centroid; a tie goes to the lower index)
    Inner-product variant (same section, and [P5] "QJL residual correction"):
      MSE stage with bits-1 bits, c_u = Pi^T c[idx], r = u - c_u, gamma = ||r||,
      z = sign(S r) with sign(0) = +1, stored as bit 1 for +1.
    A zero vector gets nu = 0, all codes 0, gamma = 0 and QJL bits 0.
    """
    fmt = p.fmt(which)
    d = p.d
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    nu = np.sqrt(np.sum(x * x, axis=1))
    zero = nu == 0.0
    u = x / np.where(zero, 1.0, nu)[:, None]
    u[zero] = 0.0
    y = u @ p.pi.T
    widths = [fmt.mse_bits(j, d) for j in range(d)]
    idx = np.zeros((n, d), dtype=np.int64)
    chat = np.zeros((n, d))
    for j in range(d):
        w = widths[j]
        if w == 0:
            continue
        cb = p.books[w]
        idx[:, j] = np.sum(y[:, j:j + 1] > cb.bounds[None, :], axis=1)
        chat[:, j] = cb.centroids[idx[:, j]]
    idx[zero] = 0
    chat[zero] = 0.0
    codes = pack_codes(idx, widths)
    if fmt.prod:
        c_u = chat @ p.pi          # Pi^T c  as a row vector
        r = u - c_u
        gamma = np.sqrt(np.sum(r * r, axis=1))
        proj = r @ p.s.T           # S r
        zbits = (proj >= 0.0).astype(np.int64)
        zbits[zero] = 0
        gamma[zero] = 0.0
        qjl = pack_codes(zbits, [1] * p.m)
    else:
        gamma = np.zeros(n)
        qjl = np.zeros((n, 0), dtype=np.uint8)
    return Packed(codes, nu.astype(np.float32), qjl, gamma.astype(np.float32))


QJL_SCALE_NUM = math.sqrt(math.pi / 2.0)  # sqrt(pi/2); divided by m at use


def dequantize(p: Params, pk: Packed, which: str = "k") -> np.ndarray:
    """x_hat = nu * (Pi^T c[idx] + sqrt(pi/2)/m * gamma * S^T z).

    The QJL constant follows from E[(s.q) sign(s.r)] = sqrt(2/pi) <q, r>/||r||
    for s ~ N(0, I): it is the one that makes <q, x_hat> unbiased
    ([P3] "Il metodo TurboQuant, in breve": the sketch makes the inner-product
    estimate unbiased).  KV dequantized before attention: [P3] "Cosa aggiunge
    turboquant-mlx".
    """
    fmt = p.fmt(which)
    d = p.d
    widths = [fmt.mse_bits(j, d) for j in range(d)]
    idx = unpack_codes(pk.codes, widths)
    chat = np.zeros(idx.shape)
    for j in range(d):
        if widths[j]:
            chat[:, j] = p.books[widths[j]].centroids[idx[:, j]]
    u_hat = chat @ p.pi
    if fmt.prod:
        z = 2.0 * unpack_codes(pk.qjl, [1] * p.m) - 1.0
        u_hat = u_hat + (QJL_SCALE_NUM / p.m) * pk.res_norms.astype(np.float64)[:, None] * (z @ p.s)
    return pk.norms.astype(np.float64)[:, None] * u_hat


# ---------------------------------------------------------------------------
# Decode attention over the quantized cache.
# [reading] Standard scaled dot-product attention for one decode step:
# score 1/sqrt(d), GQA q-head h reads kv-head h // (Hq/Hkv), softmax over all
# tokens held.  Attention sink ([P2] item 1): the first n_sink tokens are kept
# unquantized (bf16 here).  Sparse V ([P2] item 3): the V of a quantized token
# whose final softmax weight is below the threshold is left out of the
# weighted sum; the denominator keeps it; sink tokens are never skipped.
# ---------------------------------------------------------------------------

def attend_one(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
               n_sink: int, sparse_v_threshold: float = 0.0) -> np.ndarray:
    """One query (d,) over keys/values (T, d) already in the original domain."""
    d = q.shape[0]
    t = keys.shape[0]
    if t == 0:
        return np.zeros(d)
    s = keys @ q / math.sqrt(d)
    e = np.exp(s - np.max(s))
    prob = e / np.sum(e)
    keep = np.ones(t, dtype=bool)
    if sparse_v_threshold > 0.0:
        keep = prob >= sparse_v_threshold
        keep[:min(n_sink, t)] = True
    return (prob * keep) @ values


@dataclass
class Cache:
    """Oracle-side cache: one entry per (seq, kv-head), each holding the
    sink rows (bf16 values as fp64) and the packed rows of the quantized
    tokens, for K and V."""
    n_sink: int
    k_sink: dict = field(default_factory=dict)
    v_sink: dict = field(default_factory=dict)
    k_rows: dict = field(default_factory=dict)
    v_rows: dict = field(default_factory=dict)


def cache_from_vectors(p: Params, k: np.ndarray, v: np.ndarray, n_sink: int) -> Cache:
    """Build a cache from k, v of shape (B, Hkv, T, d) (values already in the
    input precision): tokens t < n_sink go to the sink, the rest are quantized."""
    c = Cache(n_sink)
    B, Hkv = k.shape[0], k.shape[1]
    for b in range(B):
        for h in range(Hkv):
            ns = min(n_sink, k.shape[2])
            c.k_sink[b, h] = np.asarray(k[b, h, :ns], dtype=np.float64)
            c.v_sink[b, h] = np.asarray(v[b, h, :ns], dtype=np.float64)
            c.k_rows[b, h] = quantize(p, k[b, h, ns:], "k")
            c.v_rows[b, h] = quantize(p, v[b, h, ns:], "v")
    return c


def decode_attention(p: Params, q: np.ndarray, cache: Cache, lens, hkv: int,
                     sparse_v_threshold: float = 0.0, heads=None) -> np.ndarray:
    """Outputs (B, Hq, d) for queries q (B, Hq, d); only ``heads`` (a list of
    (b, h) pairs) are computed when given, the rest stay zero."""
    q = np.asarray(q, dtype=np.float64)
    B, hq, d = q.shape
    group = hq // hkv
    out = np.zeros((B, hq, d))
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(hq)]
    by_kv = {}
    for b, h in todo:
        by_kv.setdefault((b, h // group), []).append(h)
    for (b, g), hs in by_kv.items():
        length = int(lens[b])
        ns = min(cache.n_sink, length)
        nq = length - ns
        kr, vr = cache.k_rows[b, g], cache.v_rows[b, g]
        k_hat = dequantize(p, Packed(kr.codes[:nq], kr.norms[:nq], kr.qjl[:nq], kr.res_norms[:nq]), "k")
        v_hat = dequantize(p, Packed(vr.codes[:nq], vr.norms[:nq], vr.qjl[:nq], vr.res_norms[:nq]), "v")
        keys = np.concatenate([cache.k_sink[b, g][:ns], k_hat], axis=0)
        vals = np.concatenate([cache.v_sink[b, g][:ns], v_hat], axis=0)
        for h in hs:
            out[b, h] = attend_one(q[b, h], keys, vals, ns, sparse_v_threshold)
    return out


# ---------------------------------------------------------------------------
# Inner-product search over a quantized database.  [P3] "Il metodo TurboQuant,
# in breve": besides the KV cache, the paper applies the quantizer to
# similarity search, in place of product quantization.  [reading] The score of
# a database row for a query is the inner product of the query with the row's
# reconstruction, <q, x_hat> (in prod mode the unbiased estimate of <q, x>);
# a search returns the k best rows per query, larger score first, equal scores
# in row order, and pads with score -inf and row -1 when the database holds
# fewer than k rows.
# ---------------------------------------------------------------------------

def ip_scores(p: Params, q: np.ndarray, pk: Packed, which: str = "k") -> np.ndarray:
    """Scores (Q, n) of queries q (Q, d) against the packed rows pk."""
    return np.asarray(q, dtype=np.float64) @ dequantize(p, pk, which).T


def ip_search(p: Params, q: np.ndarray, pk: Packed, k: int, which: str = "k"):
    """Top-k rows per query: (scores (Q, k), rows (Q, k))."""
    s = ip_scores(p, q, pk, which)
    nq, n = s.shape
    scores = np.full((nq, k), -np.inf)
    rows = np.full((nq, k), -1, dtype=np.int64)
    for i in range(nq):
        order = np.lexsort((np.arange(n), -s[i]))[:k]  # score descending, then row ascending
        scores[i, :order.size] = s[i, order]
        rows[i, :order.size] = order
    return scores, rows
