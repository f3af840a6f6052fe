"""Pins for the oracle: each test checks it against something other than itself
(published values, closed forms, an independent library routine, brute force
or a statistical law), so that a dropped term, a wrong sign or a transposed
operand anywhere in it fails here."""
import math
import os
from functools import lru_cache

import numpy as np
import pytest
import torch
from scipy import special, stats

import kv_inputs
from oracle import tq_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def _kv(name):
    return {a.strip(): b.strip() for a, b in (r.split("|") for r in _table(name))}


@lru_cache(maxsize=None)
def book(d, b):
    return o.lloyd_max(d, b)


# ---- random numbers -------------------------------------------------------

def test_splitmix64_published_outputs():
    want = [int(r, 16) for r in _table("splitmix64_seed0.txt")]
    got = [int(z) for z in o.splitmix64(0, 3)]
    assert got == want


def test_gaussians_are_standard_normal():
    g = o.gaussians(7, 3, 1 << 20)
    n = g.size
    assert abs(g.mean()) < 5 / math.sqrt(n)
    assert abs(g.var() - 1.0) < 5 * math.sqrt(2.0 / n)
    assert abs(stats.kurtosis(g, fisher=False) - 3.0) < 5 * math.sqrt(24.0 / n)
    assert stats.kstest(g[:200000], "norm").pvalue > 1e-4
    # streams with different tags are different
    assert not np.allclose(o.gaussians(7, 0, 16), o.gaussians(7, 1, 16))


# ---- rotation -------------------------------------------------------------

def test_rotation_orthogonal_det_pm1():
    pi = o.rotation(0, 128)
    assert np.max(np.abs(pi.T @ pi - np.eye(128))) < 1e-13
    assert abs(abs(np.linalg.det(pi)) - 1.0) < 1e-10


def test_rotation_is_gram_schmidt_of_gaussian_columns():
    # Independent characterisation: Q with positive diag(R) is the
    # Gram-Schmidt orthonormalisation of the columns of G.
    d = 12
    g = o.gaussians(5, o.TAG_ROTATION, d * d).reshape(d, d)
    q = np.zeros((d, d))
    for j in range(d):
        v = g[:, j].copy()
        for _ in range(2):  # re-orthogonalise once for fp64 accuracy
            for i in range(j):
                v -= (q[:, i] @ v) * q[:, i]
        q[:, j] = v / np.linalg.norm(v)
    assert np.max(np.abs(o.rotation(5, d) - q)) < 1e-12


def test_rotation_is_haar():
    # One entry of a Haar matrix in dimension d is a coordinate of a uniform
    # point on S^{d-1}: (1 + x)/2 ~ Beta((d-1)/2, (d-1)/2).
    d = 16
    xs = np.array([o.rotation(seed, d)[3, 5] for seed in range(1500)])
    a = (d - 1) / 2
    assert stats.kstest((1 + xs) / 2, stats.beta(a, a).cdf).pvalue > 1e-4


# ---- Hadamard rotation ([P3] "Cosa aggiunge turboquant-mlx") ---------------

def _sylvester(d):
    # Independent construction of the Walsh-Hadamard matrix: H_1 = [1],
    # H_2n = [[H_n, H_n], [H_n, -H_n]].
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def _fwht(v):
    # In-place butterflies (an O(d log d) algorithm, not a matrix product).
    v = v.copy()
    n, hlen = v.shape[0], 1
    while hlen < n:
        for i in range(0, n, 2 * hlen):
            a, b = v[i:i + hlen].copy(), v[i + hlen:i + 2 * hlen].copy()
            v[i:i + hlen], v[i + hlen:i + 2 * hlen] = a + b, a - b
        hlen *= 2
    return v


def test_hadamard_rotation_orthogonal_with_entries_pm_inv_sqrt_d():
    for d in (8, 128, 512):
        pi = o.hadamard_rotation(3, d)
        assert np.max(np.abs(pi @ pi.T - np.eye(d))) < 1e-14
        assert np.all(np.abs(np.abs(pi) - 1 / math.sqrt(d)) < 1e-16)
        assert np.array_equal(o.walsh_hadamard(d), _sylvester(d))


def test_hadamard_rotation_is_signed_fast_transform():
    # y = Pi u is the normalised fast Walsh-Hadamard transform of the
    # sign-flipped u: catches a transposed Pi (signs on rows, not columns).
    d = 128
    rng = np.random.default_rng(11)
    s = o.hadamard_signs(7, d)
    for _ in range(4):
        u = rng.standard_normal(d)
        want = _fwht(s * u) / math.sqrt(d)
        assert np.max(np.abs(o.hadamard_rotation(7, d) @ u - want)) < 1e-13


def test_hadamard_signs_balanced_and_seeded():
    s = o.hadamard_signs(0, 1 << 14)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 5 / math.sqrt(s.size)
    assert not np.array_equal(o.hadamard_signs(0, 128), o.hadamard_signs(1, 128))


@pytest.mark.parametrize("fmt", [o.Format(3), o.Format(3, mixed=True), o.Format(2, prod=True)])
def test_hadamard_quantize_is_nearest_centroid_and_rotates_back(fmt):
    p = o.Params(128, fmt, fmt, rotation="hadamard")
    x = kv_inputs.kv_vectors(32, 128, key="hd", dtype=torch.bfloat16).double().numpy()
    pk = o.quantize(p, x, "k")
    widths = [fmt.mse_bits(j, 128) for j in range(128)]
    idx = o.unpack_codes(pk.codes, widths)
    y = (x / np.linalg.norm(x, axis=1, keepdims=True)) @ p.pi.T
    for v in range(32):
        for j in range(128):
            if widths[j]:
                assert idx[v, j] == int(np.argmin(np.abs(y[v, j] - p.books[widths[j]].centroids)))
    if not fmt.prod:
        xh = o.dequantize(p, pk, "k")
        c = np.array([[p.books[widths[j]].centroids[idx[v, j]] for j in range(128)] for v in range(32)])
        assert np.max(np.abs(xh @ p.pi.T / pk.norms.astype(np.float64)[:, None] - c)) < 1e-13


def test_qjl_matrix_standard_normal_rows():
    s = o.qjl_matrix(0, 128, 128)
    assert s.shape == (128, 128)
    assert abs(s.mean()) < 5 / 128
    assert abs(s.var() - 1) < 5 * math.sqrt(2 / s.size)
    assert not np.allclose(s, o.rotation(0, 128))


# ---- coordinate density and codebook ---------------------------------------

@pytest.mark.parametrize("d", [8, 64, 128, 512])
def test_density_is_beta_law(d):
    a = (d - 1) / 2
    assert abs(o.cell_mass(np.array([-1.0]), np.array([1.0]), d)[0] - 1.0) < 1e-13
    for x in (-0.3, -0.05, 0.0, 0.02, 0.1, 0.25):
        want = special.betainc(a, a, (1 + x) / 2)
        got = o.cell_mass(np.array([-1.0]), np.array([x]), d)[0]
        assert abs(got - want) < 1e-12


@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_one_bit_centroid_closed_form(d):
    # For b = 1 the cells are [-1,0] and [0,1]; E[x | x > 0] has the closed
    # form Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)) -> sqrt(2/(pi d)).
    c = math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))
    cb = book(d, 1)
    assert np.max(np.abs(cb.centroids - np.array([-c, c]))) < 1e-12
    assert abs(c / math.sqrt(2 / (math.pi * d)) - 1) < 1 / (2 * d)


def test_large_d_limit_is_max_gaussian_table():
    d = 1_000_000
    for row in _table("lloyd_max_gaussian_max1960.txt"):
        levels, vals = row.split("|")
        b = int(levels).bit_length() - 1
        want = np.array([float(v) for v in vals.split()])
        got = o.lloyd_max(d, b).centroids[(1 << b) // 2:] * math.sqrt(d)
        assert np.max(np.abs(got - want) / want) < 1.5e-3, (b, got, want)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_codebook_conditions_by_monte_carlo(b):
    # Sample the first coordinate of a uniform point on S^{127} directly
    # (g0 / sqrt(g0^2 + chi2_127)) and check each centroid is the mean of its
    # cell and that d * MSE equals the quadrature distortion.
    d = 128
    rng = np.random.default_rng(100 + b)
    n = 1 << 21
    g0 = rng.standard_normal(n)
    x = g0 / np.sqrt(g0 * g0 + rng.chisquare(d - 1, n))
    cb = book(d, b)
    idx = np.searchsorted(cb.bounds, x)
    for k, ck in enumerate(cb.centroids):
        sel = x[idx == k]
        se = sel.std() / math.sqrt(sel.size)
        assert abs(sel.mean() - ck) < 5 * se + 1e-12
    err = d * (x - cb.centroids[idx]) ** 2
    assert abs(err.mean() - o.mse_distortion(cb)) < 5 * err.std() / math.sqrt(n)
    # symmetry of the density
    assert np.max(np.abs(cb.centroids + cb.centroids[::-1])) < 1e-14


def test_distortion_bounds_and_page_cosines():
    # "within about 2.7x of the information-theoretic minimum" (article,
    # "Il metodo TurboQuant, in breve"): 4^-b <= D_b <= sqrt(3) pi / 2 * 4^-b.
    for b in (1, 2, 3, 4):
        dist = o.mse_distortion(book(128, b))
        assert 4.0 ** -b <= dist <= math.sqrt(3) * math.pi / 2 * 4.0 ** -b
    for row in _table("pages_cosine.txt"):
        b, cos = row.split("|")
        b, cos = int(b), float(cos)
        assert round(math.sqrt(1 - o.mse_distortion(book(128, b))), 3) == cos


@pytest.mark.parametrize("b", [2, 3])
def test_mixed_row_distortion_is_mean_of_its_two_widths(b):
    # "3.5 / 2.5 bits per channel" (article, "Il metodo TurboQuant, in
    # breve"): half the rotated coordinates at b+1 bits, half at b.  For
    # uniform unit vectors every rotated coordinate follows the sphere law, so
    # the expected squared error of the round trip is (D_b + D_{b+1}) / 2.
    fmt = o.Format(b, mixed=True)
    p = o.Params(128, fmt, fmt)
    rng = np.random.default_rng(40 + b)
    u = rng.standard_normal((8192, 128))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    err = np.sum((o.dequantize(p, o.quantize(p, u, "k"), "k") - u) ** 2, axis=1)
    want = 0.5 * (o.mse_distortion(book(128, b)) + o.mse_distortion(book(128, b + 1)))
    assert abs(err.mean() - want) < 5 * err.std() / math.sqrt(err.size)
    # and it lies strictly between the two uniform widths' distortions
    assert o.mse_distortion(book(128, b + 1)) < err.mean() < o.mse_distortion(book(128, b))


def test_end_to_end_cosine_matches_pages():
    p = o.Params(128, o.Format(3), o.Format(4))
    for row in _table("pages_cosine.txt"):
        b, cos = row.split("|")
        which = "k" if int(b) == 3 else "v"
        x = kv_inputs.kv_vectors(4096, 128, key=("cos", int(b))).double().numpy()
        xh = o.dequantize(p, o.quantize(p, x, which), which)
        c = np.sum(x * xh, 1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1)
        assert round(float(c.mean()), 3) == float(cos)


# ---- quantize / pack -------------------------------------------------------

@pytest.mark.parametrize("fmt", [o.Format(1), o.Format(2), o.Format(3), o.Format(4),
                                 o.Format(3, mixed=True), o.Format(2, mixed=True), o.Format(3, prod=True),
                                 o.Format(8)])
def test_quantize_is_brute_force_nearest_centroid(fmt):
    p = o.Params(128, fmt, fmt)
    x = kv_inputs.kv_vectors(64, 128, key="bf", dtype=torch.bfloat16).double().numpy()
    pk = o.quantize(p, x, "k")
    widths = [fmt.mse_bits(j, 128) for j in range(128)]
    idx = o.unpack_codes(pk.codes, widths)
    for v in range(64):
        y = p.pi @ (x[v] / np.linalg.norm(x[v]))
        for j in range(128):
            if widths[j] == 0:
                continue
            c = p.books[widths[j]].centroids
            assert idx[v, j] == int(np.argmin(np.abs(y[j] - c)))
    assert np.allclose(pk.norms, np.linalg.norm(x, axis=1), rtol=1e-7)


def test_pack_golden_b3():
    rows = _kv("pack_b3.txt")
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, :8] = [int(c) for c in rows["codes"].split()]
    want = bytes.fromhex("".join(rows["bytes"].split())) + bytes(45)
    got = o.pack_codes(codes, [3] * 128)
    assert got.tobytes() == want
    assert np.array_equal(o.unpack_codes(got, [3] * 128), codes)


@pytest.mark.parametrize("name,bits,row", [("pack_mixed43.txt", 3, 56), ("pack_mixed32.txt", 2, 40)])
def test_pack_golden_mixed(name, bits, row):
    rows = _kv(name)
    codes = np.zeros((1, 128), dtype=np.int64)
    for kv in rows["set"].split():
        j, c = kv.split("=")
        codes[0, int(j)] = int(c)
    want = bytearray(row)
    for kv in rows["bytes"].split():
        i, v = kv.split("=")
        want[int(i)] = int(v, 16)
    fmt = o.Format(bits, mixed=True)
    widths = [fmt.mse_bits(j, 128) for j in range(128)]
    assert fmt.code_bytes(128) == row
    got = o.pack_codes(codes, widths)
    assert got.tobytes() == bytes(want)
    assert np.array_equal(o.unpack_codes(got, widths), codes)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_pack_roundtrip(b):
    rng = np.random.default_rng(b)
    idx = rng.integers(0, 1 << b, size=(33, 128))
    assert np.array_equal(o.unpack_codes(o.pack_codes(idx, [b] * 128), [b] * 128), idx)


def test_zero_vector():
    fmt = o.Format(3, prod=True)
    p = o.Params(128, fmt, fmt)
    pk = o.quantize(p, np.zeros((2, 128)), "k")
    assert not pk.codes.any() and not pk.qjl.any()
    assert not pk.norms.any() and not pk.res_norms.any()
    assert not o.dequantize(p, pk, "k").any()


# ---- dequantize ------------------------------------------------------------

def test_mse_dequant_rotates_back_to_centroids():
    # Dequantizing packed rows built by hand must give x_hat with
    # Pi x_hat / nu = c[idx] (the forward rotation undoes the inverse one, so a
    # transposed Pi fails) and ||x_hat|| = nu ||c[idx]||.
    fmt = o.Format(4)
    p = o.Params(128, fmt, fmt)
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 16, size=(16, 128))
    nu = rng.uniform(0.5, 50, size=16).astype(np.float32)
    pk = o.Packed(o.pack_codes(idx, [4] * 128), nu, np.zeros((16, 0), np.uint8), np.zeros(16, np.float32))
    xh = o.dequantize(p, pk, "k")
    c = p.books[4].centroids[idx]
    assert np.max(np.abs(xh @ p.pi.T / nu.astype(np.float64)[:, None] - c)) < 1e-13
    assert np.allclose(np.linalg.norm(xh, axis=1), nu * np.linalg.norm(c, axis=1), rtol=1e-12)


def test_mse_stage_shrinks_inner_products():
    # For the MSE quantizer E<u, u_hat> = E||u_hat||^2 = 1 - D_b: the bias the
    # QJL stage removes (article, "Il metodo TurboQuant, in breve").
    fmt = o.Format(1)
    p = o.Params(128, fmt, fmt)
    x = kv_inputs.kv_vectors(20000, 128, key="bias").double().numpy()
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    uh = o.dequantize(p, o.quantize(p, x, "k"), "k") / np.linalg.norm(x, axis=1, keepdims=True)
    ip = np.sum(u * uh, axis=1)
    want = 1 - o.mse_distortion(p.books[1])
    assert abs(ip.mean() - want) < 5 * ip.std() / math.sqrt(ip.size)
    assert abs(want - 2 / math.pi) < 0.01


@pytest.mark.parametrize("bits", [1, 3])
def test_qjl_inner_product_is_unbiased_with_exact_variance(bits):
    # Over random S, <q, x_hat> - <q, x> has mean 0 and variance
    # nu^2 (pi/(2m)) gamma^2 (||q||^2 - (2/pi) <q, r/gamma>^2)
    # (sign identity E[(s.q) sign(s.r)] = sqrt(2/pi) <q, r>/||r||).
    fmt = o.Format(bits, prod=True)
    p = o.Params(128, fmt, fmt)
    x = kv_inputs.kv_vectors(1, 128, key=("qjl", bits)).double().numpy()
    q = kv_inputs.queries((128,), key=("qjl", bits), dtype=torch.float64).numpy()
    nu = np.linalg.norm(x)
    u = x[0] / nu
    errs = []
    for seed in range(1, 1201):
        p.s = o.qjl_matrix(seed, p.m, 128)
        pk = o.quantize(p, x, "k")
        errs.append(q @ o.dequantize(p, pk, "k")[0] - q @ x[0])
    errs = np.array(errs)
    pk = o.quantize(p, x, "k")
    widths = [fmt.mse_bits(j, 128) for j in range(128)]
    chat = np.zeros(128)
    if bits > 1:
        chat = p.books[bits - 1].centroids[o.unpack_codes(pk.codes, widths)[0]]
    r = u - chat @ p.pi
    g = np.linalg.norm(r)
    var = nu ** 2 * (math.pi / (2 * p.m)) * g ** 2 * (q @ q - (2 / math.pi) * (q @ r / g) ** 2)
    n = errs.size
    assert abs(errs.mean()) < 5 * math.sqrt(var / n)
    assert abs(errs.var() / var - 1) < 5 * math.sqrt(2 / n)


# ---- attention -------------------------------------------------------------

def _loops_attention(q, keys, vals, n_sink, thr):
    """Pure-Python loops, tiny T only."""
    d = len(q)
    s = [sum(q[i] * k[i] for i in range(d)) / math.sqrt(d) for k in keys]
    mx = max(s)
    e = [math.exp(v - mx) for v in s]
    tot = sum(e)
    out = [0.0] * d
    for t, v in enumerate(vals):
        p = e[t] / tot
        if thr > 0 and t >= n_sink and p < thr:
            continue
        for i in range(d):
            out[i] += p * v[i]
    return np.array(out)


def test_attention_brute_force_tiny():
    rng = np.random.default_rng(0)
    for t in (1, 2, 5, 8):
        q = rng.standard_normal(16)
        k = 3 * rng.standard_normal((t, 16))
        v = rng.standard_normal((t, 16))
        for thr in (0.0, 0.05):
            want = _loops_attention(q, k, v, 1, thr)
            assert np.allclose(o.attend_one(q, k, v, 1, thr), want, atol=1e-14)


def test_attention_special_cases():
    rng = np.random.default_rng(1)
    q = rng.standard_normal(8)
    v = rng.standard_normal((6, 8))
    same = np.tile(rng.standard_normal(8), (6, 1))
    assert np.allclose(o.attend_one(q, same, v, 0), v.mean(axis=0), atol=1e-14)
    assert np.allclose(o.attend_one(q, same[:1], v[:1], 0), v[0], atol=1e-14)
    assert not o.attend_one(q, np.zeros((0, 8)), np.zeros((0, 8)), 0).any()


def test_sparse_v_error_bound():
    rng = np.random.default_rng(2)
    q = rng.standard_normal(32)
    k = 4 * rng.standard_normal((500, 32))
    v = rng.standard_normal((500, 32))
    full = o.attend_one(q, k, v, 4, 0.0)
    thr = 1e-3
    sparse = o.attend_one(q, k, v, 4, thr)
    s = k @ q / math.sqrt(32)
    p = np.exp(s - s.max()); p /= p.sum()
    skipped = (p < thr); skipped[:4] = False
    assert skipped.any()
    bound = np.sum(p[skipped]) * np.max(np.linalg.norm(v, axis=1))
    assert 0 < np.linalg.norm(full - sparse) <= bound + 1e-15


def test_decode_attention_gqa_sink_and_rotated_domain_identity():
    fmt_k, fmt_v = o.Format(4), o.Format(3)
    p = o.Params(128, fmt_k, fmt_v)
    B, hkv, hq, T, ns = 2, 2, 4, 40, 5
    k = kv_inputs.kv_vectors(B * hkv * T, 128, key="ak", dtype=torch.bfloat16)
    v = kv_inputs.kv_vectors(B * hkv * T, 128, key="av", dtype=torch.bfloat16)
    k = k.double().numpy().reshape(B, hkv, T, 128)
    v = v.double().numpy().reshape(B, hkv, T, 128)
    q = kv_inputs.queries((B, hq, 128), key="aq").double().numpy()
    cache = o.cache_from_vectors(p, k, v, ns)
    lens = [T, 23]
    out = o.decode_attention(p, q, cache, lens, hkv)
    for b in range(B):
        for h in range(hq):
            g = h // 2
            n = lens[b]
            kr, vr = cache.k_rows[b, g], cache.v_rows[b, g]
            # keys through the rotated domain: s = nu <Pi q, c[idx]>
            idx = o.unpack_codes(kr.codes, [4] * 128)[:n - ns]
            c = p.books[4].centroids[idx]
            s_rot = kr.norms[:n - ns].astype(np.float64) * (c @ (p.pi @ q[b, h]))
            keys = np.concatenate([k[b, g, :ns], o.dequantize(p, kr, "k")[:n - ns]])
            assert np.allclose(keys[ns:] @ q[b, h], s_rot, rtol=1e-10, atol=1e-10)
            vals = np.concatenate([v[b, g, :ns], o.dequantize(p, vr, "v")[:n - ns]])
            assert np.allclose(out[b, h], _loops_attention(q[b, h], keys, vals, ns, 0.0), atol=1e-12)


# ---- inner-product search ----------------------------------------------------

@pytest.mark.parametrize("fmt", [o.Format(3), o.Format(2, mixed=True)])
def test_ip_search_is_brute_force_top_k(fmt):
    # brute force in the rotated domain: score = nu * sum_j (Pi q)_j c[idx_j]
    # (no reconstruction, no Pi^T), then a plain sort by (-score, row)
    p = o.Params(128, fmt, fmt)
    x = kv_inputs.kv_vectors(61, 128, key="ipb").double().numpy()
    x[40] = x[3]  # exact ties: the lower row comes first
    x[41] = x[3]
    pk = o.quantize(p, x, "k")
    widths = [fmt.mse_bits(j, 128) for j in range(128)]
    idx = o.unpack_codes(pk.codes, widths)
    q = np.random.default_rng(6).standard_normal((4, 128))
    q[1] = 3.0 * x[3] / np.linalg.norm(x[3])  # the tied rows are this query's best
    want_s = np.zeros((4, 61))
    for i in range(4):
        qr = p.pi @ q[i]
        for r in range(61):
            acc = 0.0
            for j in range(128):
                acc += qr[j] * p.books[widths[j]].centroids[idx[r, j]]
            want_s[i, r] = float(pk.norms[r]) * acc
    assert np.max(np.abs(o.ip_scores(p, q, pk) - want_s)) < 1e-12 * np.max(np.abs(want_s))
    scores, rows = o.ip_search(p, q, pk, 9)
    for i in range(4):
        brute = sorted(range(61), key=lambda r: (-want_s[i, r], r))[:9]
        assert rows[i].tolist() == brute
        assert np.allclose(scores[i], want_s[i, brute], rtol=1e-12, atol=0)
    assert rows[1, :3].tolist() == [3, 40, 41]


def test_ip_search_pads_short_databases():
    fmt = o.Format(2, prod=True)
    p = o.Params(128, fmt, fmt)
    x = kv_inputs.kv_vectors(3, 128, key="ips").double().numpy()
    q = np.random.default_rng(7).standard_normal((2, 128))
    scores, rows = o.ip_search(p, q, o.quantize(p, x, "k"), 5)
    assert (rows[:, 3:] == -1).all() and np.isneginf(scores[:, 3:]).all()
    assert sorted(rows[0, :3].tolist()) == [0, 1, 2]
    empty = o.quantize(p, np.zeros((0, 128)), "k")
    scores, rows = o.ip_search(p, q, empty, 4)
    assert (rows == -1).all() and np.isneginf(scores).all()


# ---- codebooks above 4 bits (Newton on the Lloyd conditions) ----------------

@pytest.mark.parametrize("b", [2, 3, 4, 5])
def test_newton_reaches_the_lloyd_iteration_fixed_point(b):
    # two algorithms for the same conditions: the plain iteration (run to
    # convergence) and Newton's method from the high-resolution start
    it = o.lloyd_iteration(128, b)
    nw = o.lloyd_max_newton(128, b)
    assert np.max(np.abs(it.centroids - nw.centroids)) < 1e-13


@pytest.mark.parametrize("b", [6, 8])
def test_many_level_codebook_conditions(b):
    d = 128
    cb = book(d, b)
    c = cb.centroids
    assert np.all(np.diff(c) > 0) and np.max(np.abs(c + c[::-1])) < 1e-13
    lo = np.concatenate(([-1.0], cb.bounds))
    hi = np.concatenate((cb.bounds, [1.0]))
    # centroid condition, cell by cell, against an independent quadrature
    from scipy import integrate as si
    for k in (0, 1, len(c) // 2 - 1, len(c) // 2, len(c) - 1):
        m0 = si.quad(lambda x: o.coord_density(x, d), lo[k], hi[k], epsabs=0, epsrel=1e-13)[0]
        m1 = si.quad(lambda x: x * o.coord_density(x, d), lo[k], hi[k], epsabs=0, epsrel=1e-13)[0]
        assert abs(m1 / m0 - c[k]) < 1e-12 * max(abs(c[k]), 1e-3)
    # the rate-distortion sandwich of the article ("within about 2.7x")
    dist = o.mse_distortion(cb)
    assert 4.0 ** -b <= dist <= math.sqrt(3) * math.pi / 2 * 4.0 ** -b


def test_eight_bit_rows_are_bytes():
    # 8-bit codes (the K8 setting of the article's "Cosa aggiunge"): code j is byte j
    fmt = o.Format(8)
    assert fmt.code_bytes(128) == 128
    idx = np.random.default_rng(9).integers(0, 256, size=(5, 128))
    packed = o.pack_codes(idx, [8] * 128)
    assert np.array_equal(packed, idx.astype(np.uint8))
