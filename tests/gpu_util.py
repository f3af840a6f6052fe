"""Helpers shared by the GPU parity tests: build matching GPU / oracle
parameter sets, move packed rows between the two, and compare results with
the tolerances of the parity contract."""
from __future__ import annotations

import numpy as np
import torch

import online_vector_quantization_b200 as tq
from oracle import tq_oracle as o

# Tolerances (the parity contract).
BOUNDARY_EPS = 1e-5        # codes may differ only within this distance of a bound
MISMATCH_FRACTION = 1e-4   # ... and on fewer than this fraction of coordinates
DEQUANT_ATOL = 1e-5        # fp32 dequantization on identical packed input
ATTN_REL_L2 = 2e-3         # decode attention, bf16 queries and outputs


def fmt(bits, prod=False, mixed=False):
    return o.Format(bits, prod=prod, mixed=mixed)


def make_params(fk: o.Format, fv: o.Format, seed: int = 0, rotation: str = "haar"):
    kind = {"haar": tq.TQ_ROT_HAAR, "hadamard": tq.TQ_ROT_HADAMARD}[rotation]
    gp = tq.Params(fk.bits, fv.bits, tq.TQ_MODE_PROD if fk.prod else tq.TQ_MODE_MSE,
                   tq.TQ_MODE_PROD if fv.prod else tq.TQ_MODE_MSE, int(fk.mixed), int(fv.mixed), seed=seed,
                   rotation=kind)
    op = o.Params(128, fk, fv, seed=seed, rotation=rotation)
    return gp, op


def widths(f: o.Format):
    return [f.mse_bits(j, 128) for j in range(128)]


def gpu_packed_to_numpy(pk: tq.Packed) -> o.Packed:
    n = pk.norms.shape[0]
    codes = pk.codes.cpu().numpy() if pk.codes is not None else np.zeros((n, 0), np.uint8)
    qjl = pk.qjl.cpu().numpy() if pk.qjl is not None else np.zeros((n, 0), np.uint8)
    res = pk.res_norms.cpu().numpy() if pk.res_norms is not None else np.zeros(n, np.float32)
    return o.Packed(codes, pk.norms.cpu().numpy(), qjl, res)


def numpy_packed_to_gpu(pk: o.Packed) -> tq.Packed:
    def t(a, dtype):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dtype=dtype, device="cuda")
    n = pk.norms.shape[0]
    return tq.Packed(t(pk.codes, torch.uint8) if pk.codes.shape[1] else None,
                     t(pk.norms, torch.float32),
                     t(pk.qjl, torch.uint8) if pk.qjl.shape[1] else None,
                     t(pk.res_norms, torch.float32) if pk.qjl.shape[1] else None)


def rotated_unit(op: o.Params, x: np.ndarray) -> np.ndarray:
    nu = np.linalg.norm(x, axis=1, keepdims=True)
    return (x / np.where(nu == 0, 1, nu)) @ op.pi.T


def mismatch_fraction(f: o.Format) -> float:
    """MISMATCH_FRACTION for rows of up to 4 bits.  A code can flip only where
    the coordinate lies within the two sides' rounding difference of a bound,
    so the rate grows with the number of bounds per coordinate: 8-bit codes
    (255 bounds against 15) get the fraction scaled by 255 / 15."""
    nb = max((1 << b) - 1 for b in widths(f))
    return MISMATCH_FRACTION * max(1.0, nb / 15)


def compare_codes(op: o.Params, f: o.Format, x: np.ndarray, got: o.Packed, want: o.Packed):
    """Codes bit-exact except coordinates within BOUNDARY_EPS of a bound, and
    those fewer than mismatch_fraction(f) of all.  Returns the set of vectors
    whose codes differ (their QJL sketch legitimately differs too)."""
    w = widths(f)
    gi = o.unpack_codes(got.codes, w)
    wi = o.unpack_codes(want.codes, w)
    bad = np.argwhere(gi != wi)
    y = rotated_unit(op, x)
    for v, j in bad:
        b = op.books[w[j]].bounds
        assert np.min(np.abs(y[v, j] - b)) < BOUNDARY_EPS, (v, j, y[v, j], gi[v, j], wi[v, j])
    total = gi.size
    assert len(bad) <= max(1, mismatch_fraction(f) * total), (len(bad), total)
    return set(int(v) for v in bad[:, 0])


def compare_qjl(op: o.Params, f: o.Format, x: np.ndarray, got: o.Packed, want: o.Packed, skip: set):
    if not f.prod:
        return
    gb = o.unpack_codes(got.qjl, [1] * 128)
    wb = o.unpack_codes(want.qjl, [1] * 128)
    # S r in fp64 from the oracle's own codes
    chat = np.zeros((x.shape[0], 128))
    wi = o.unpack_codes(want.codes, widths(f)) if want.codes.shape[1] else None
    for j, wj in enumerate(widths(f)):
        if wj:
            chat[:, j] = op.books[wj].centroids[wi[:, j]]
    nu = np.linalg.norm(x, axis=1, keepdims=True)
    u = x / np.where(nu == 0, 1, nu)
    proj = (u - chat @ op.pi) @ op.s.T
    for v, i in np.argwhere(gb != wb):
        if int(v) in skip:
            continue
        assert abs(proj[v, i]) < BOUNDARY_EPS, (v, i, proj[v, i])
    keep = np.array([v not in skip for v in range(x.shape[0])])
    assert np.allclose(got.res_norms[keep], want.res_norms[keep], rtol=1e-5, atol=1e-6)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def side_id(side: str) -> int:
    return tq.TQ_K if side == "k" else tq.TQ_V


def read_unit_rows(cache: tq.Cache, f: o.Format, side: str, b: int, h: int, row0: int, n: int) -> o.Packed:
    """Quantized rows row0 .. row0 + n - 1 of unit (b, h), as packed rows
    (tq_cache_read_rows: the code planes are tiled)."""
    out = tq.Packed.empty(cache.params, max(n, 1), side_id(side))
    tq.tq_cache_read_rows(cache.params, cache, side_id(side), b, h, row0, out, n)
    torch.cuda.synchronize()
    pk = gpu_packed_to_numpy(out)
    return o.Packed(pk.codes[:n], pk.norms[:n], pk.qjl[:n], pk.res_norms[:n])


def write_unit_rows(cache: tq.Cache, side: str, b: int, h: int, row0: int, pk: o.Packed):
    n = pk.norms.shape[0]
    if n:
        tq.tq_cache_write_rows(cache.params, cache, side_id(side), b, h, row0, numpy_packed_to_gpu(pk), n)


def fill_cache_from_oracle(cache: tq.Cache, op: o.Params, ocache: o.Cache, lens, B, hkv):
    """Write oracle-packed rows (tq_cache_write_rows) and bf16 sink rows into a
    GPU cache."""
    sinks = {side: cache.plane(side + "_sink", torch.bfloat16, 128) for side in ("k", "v")}
    for b in range(B):
        for h in range(hkv):
            ns = min(cache.n_sink, lens[b])
            nq = lens[b] - ns
            for side, rows, sink in (("k", ocache.k_rows[b, h], ocache.k_sink[b, h]),
                                     ("v", ocache.v_rows[b, h], ocache.v_sink[b, h])):
                write_unit_rows(cache, side, b, h, 0,
                                o.Packed(rows.codes[:nq], rows.norms[:nq], rows.qjl[:nq], rows.res_norms[:nq]))
                if ns:
                    sinks[side][b, h, :ns] = torch.from_numpy(sink[:ns]).to(torch.bfloat16).cuda()
    torch.cuda.synchronize()
    cache.lens.copy_(torch.tensor(lens, dtype=torch.int32))
