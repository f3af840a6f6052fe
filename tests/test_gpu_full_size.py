"""GPU parity at the full sizes of the measured workloads, in the launch
configuration bench.py times (same inputs, same grid: every persistent CTA
busy), checked on sampled outputs the oracle computes one by one:

- the quantize sweep (1M bf16 vectors with outlier channels): every format,
  4096 sampled rows against the oracle's quantizer;
- prod 3-bit GQA decode (B=1, 32 q / 8 kv heads, T=32768): two sampled
  kv-heads, codes against the oracle and the attention of their 8 query heads
  against the oracle's attention over the very same packed rows;
- long-context K4/V3 decode with a 128-token bf16 sink, planted keys and
  sparse V (B=4, 64 q / 8 kv, T=131072): two sampled (sequence, kv-head) units;
- the streaming step (16 sequences, U[8192, 65536] contexts, mixed 3.5-bit,
  prefill, one 64-token append, one decode): two sampled units;
- the inner-product search (2^22 prod 3-bit rows, 8 queries, top-10): the
  returned rows against the oracle's scores and a 200,000-row sample.
"""
import numpy as np
import pytest
import torch

import kv_inputs
from oracle import tq_oracle as o

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, run on the GPU machine
    pytest.skip("needs a CUDA device", allow_module_level=True)

import online_vector_quantization_b200 as tq  # noqa: E402
import gpu_util as gu  # noqa: E402

D = 128


def unit_packed(cache, f: o.Format, side: str, b: int, h: int, rows: int) -> o.Packed:
    """The packed rows [0, rows) of plane side (k or v) of unit (b, h)."""
    return gu.read_unit_rows(cache, f, side, b, h, 0, rows)


def oracle_cache_from_gpu(cache, fk, fv, units, lens):
    """Oracle cache holding exactly the GPU's packed rows (and bf16 sink) of
    the sampled units, so the attention comparison isolates the decode."""
    oc = o.Cache(cache.n_sink)
    for b, h in units:
        ns = min(cache.n_sink, lens[b])
        nq = lens[b] - ns
        if cache.n_sink:
            oc.k_sink[b, h] = cache.plane("k_sink", torch.bfloat16, D)[b, h, :ns].double().cpu().numpy()
            oc.v_sink[b, h] = cache.plane("v_sink", torch.bfloat16, D)[b, h, :ns].double().cpu().numpy()
        else:
            oc.k_sink[b, h] = np.zeros((0, D))
            oc.v_sink[b, h] = np.zeros((0, D))
        oc.k_rows[b, h] = unit_packed(cache, fk, "k", b, h, nq)
        oc.v_rows[b, h] = unit_packed(cache, fv, "v", b, h, nq)
    return oc


def check_unit_codes(op, f, side, x_unit, got):
    """GPU-quantized rows of one unit against the oracle's quantizer."""
    want = o.quantize(op, x_unit, side)
    skip = gu.compare_codes(op, f, x_unit, got, want) if f.code_bytes(D) else set()
    assert np.allclose(got.norms, want.norms, rtol=1e-6, atol=0)
    gu.compare_qjl(op, f, x_unit, got, want, skip)


def check_attention(op, q, oc, lens, hkv, units, out, thr=0.0):
    group = q.shape[1] // hkv
    heads = [(b, h * group + j) for b, h in units for j in range(group)]
    want = o.decode_attention(op, q.double().numpy(), oc, lens, hkv, thr, heads)
    got = out.float().cpu().numpy()
    for b, h in units:
        sl = slice(h * group, (h + 1) * group)
        err = gu.rel_l2(got[b, sl], want[b, sl])
        assert err < gu.ATTN_REL_L2, (b, h, err)


SWEEP = [gu.fmt(b) for b in (1, 2, 3, 4)] + [gu.fmt(b, prod=True) for b in (1, 2, 3, 4)]


@pytest.fixture(scope="module")
def sweep_input():
    n = 32 * 32768
    x = kv_inputs.kv_vectors(n, D, key="sweep", device="cuda", dtype=torch.bfloat16, outliers=True)
    rows = np.sort(np.random.default_rng(2).choice(n, 4096, replace=False))
    return x, rows, x[torch.from_numpy(rows).cuda()].double().cpu().numpy()


@pytest.mark.parametrize("f", SWEEP, ids=["mse1", "mse2", "mse3", "mse4", "prod1", "prod2", "prod3", "prod4"])
def test_full_quantize_sweep_sampled(sweep_input, f):
    x, rows, xs = sweep_input
    gp, op = gu.make_params(f, f)
    pk = tq.Packed.empty(gp, x.shape[0], tq.TQ_K)
    tq.tq_quantize(gp, x, tq.TQ_K, pk)
    torch.cuda.synchronize()
    assert gp.status() == 0
    idx = torch.from_numpy(rows).cuda()
    got = o.Packed(pk.codes[idx].cpu().numpy() if pk.codes is not None else np.zeros((len(rows), 0), np.uint8),
                   pk.norms[idx].cpu().numpy(),
                   pk.qjl[idx].cpu().numpy() if pk.qjl is not None else np.zeros((len(rows), 0), np.uint8),
                   pk.res_norms[idx].cpu().numpy() if pk.res_norms is not None else np.zeros(len(rows), np.float32))
    check_unit_codes(op, f, "k", xs, got)


def test_full_prod3_gqa_decode_sampled():
    T, hkv, hq = 32768, 8, 32
    f = gu.fmt(3, prod=True)
    gp, op = gu.make_params(f, f)
    cache = tq.Cache(gp, 1, hkv, T, 0)
    k = kv_inputs.kv_vectors(T * hkv, D, key="c3k", device="cuda").view(1, T, hkv, D)
    v = kv_inputs.kv_vectors(T * hkv, D, key="c3v", device="cuda").view(1, T, hkv, D)
    tq.tq_append(gp, cache, torch.zeros(1, dtype=torch.int32, device="cuda"), k, v)
    q = kv_inputs.queries((1, hq, D), key="c3q", device="cuda")
    ws = tq.decode_workspace(gp, 1, hq, hkv, T)
    out = torch.empty(1, hq, D, dtype=torch.bfloat16, device="cuda")
    tq.tq_decode_attn(gp, q, cache, T, out, ws)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    units = [(0, 1), (0, 6)]
    for b, h in units:
        check_unit_codes(op, f, "k", k[b, :, h].double().cpu().numpy(), unit_packed(cache, f, "k", b, h, T))
    oc = oracle_cache_from_gpu(cache, f, f, units, [T])
    check_attention(op, q.cpu(), oc, [T], hkv, units, out)


def test_full_k4v3_sink_sparse_decode_sampled():
    B, T, hkv, hq, n_sink = 4, 131072, 8, 64, 128
    fk, fv = gu.fmt(4), gu.fmt(3)
    gp, op = gu.make_params(fk, fv)
    cache = tq.Cache(gp, B, hkv, T - n_sink, n_sink)
    q = kv_inputs.queries((B, hq, D), key="c4q", device="cuda")
    units = [(1, 3), (3, 6)]
    kept = {}
    for s in range(B):
        ids = torch.tensor([s], dtype=torch.int32, device="cuda")
        ks, vs = [], []
        for h in range(hkv):
            kk = kv_inputs.kv_vectors(T, D, key=("c4k", s, h), device="cuda", dtype=torch.bfloat16)
            kk = kv_inputs.planted_keys(kk, q[s, 8 * h:8 * h + 8], 8, n_sink, key=("c4p", s, h))
            ks.append(kk)
            vs.append(kv_inputs.kv_vectors(T, D, key=("c4v", s, h), device="cuda", dtype=torch.bfloat16))
        for b, h in units:
            if b == s:
                kept[b, h] = (ks[h].double().cpu().numpy(), vs[h].double().cpu().numpy())
        kt = torch.stack(ks, 1).view(1, T, hkv, D)
        vt = torch.stack(vs, 1).view(1, T, hkv, D)
        del ks, vs
        for c0 in range(0, T, 32768):
            tq.tq_append(gp, cache, ids, kt[:, c0:c0 + 32768].contiguous(), vt[:, c0:c0 + 32768].contiguous())
        del kt, vt
    ws = tq.decode_workspace(gp, B, hq, hkv, T)
    out = torch.empty(B, hq, D, dtype=torch.bfloat16, device="cuda")
    tq.tq_decode_attn(gp, q, cache, T, out, ws, 1e-6)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    for b, h in units:
        kx, vx = kept[b, h]
        check_unit_codes(op, fk, "k", kx[n_sink:], unit_packed(cache, fk, "k", b, h, T - n_sink))
        check_unit_codes(op, fv, "v", vx[n_sink:], unit_packed(cache, fv, "v", b, h, T - n_sink))
    oc = oracle_cache_from_gpu(cache, fk, fv, units, [T] * B)
    check_attention(op, q.cpu(), oc, [T] * B, hkv, units, out, 1e-6)


def test_full_stream_step_sampled():
    import bench

    st = bench.build_stream_workload(tq, torch, kv_inputs, 0, 1, torch.device("cuda", 0))
    params, cache = st["params"], st["cache"]
    tq.tq_append(params, cache, st["ids"], st["ck"][0], st["cv"][0])
    tq.tq_decode_attn(params, st["qs"][0], cache, st["cap"], st["out"], st["ws"])
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    lens = cache.lens.cpu().tolist()
    f = gu.fmt(3, mixed=True)
    _, op = gu.make_params(f, f)
    units = [(6, 2), (13, 5)]  # sequences of 55,659 and 12,624 tokens before the append
    oc = oracle_cache_from_gpu(cache, f, f, units, lens)
    check_attention(op, st["qs"][0].cpu(), oc, lens, bench.HKV, units, st["out"])
    # the appended chunk of the sampled units, against the oracle's quantizer
    for b, h in units:
        rows = np.arange(lens[b] - bench.CHUNK, lens[b])
        got = unit_packed(cache, f, "k", b, h, lens[b])
        got = o.Packed(got.codes[rows], got.norms[rows], got.qjl[rows], got.res_norms[rows])
        check_unit_codes(op, f, "k", st["ck"][0][b, :, h].double().cpu().numpy(), got)


def test_full_search_sampled():
    """The search workload bench.py times (2^22 prod 3-bit rows, 8 queries,
    top-10): the returned rows' scores against the oracle's, and no row of a
    200,000-row sample (plus every returned row) beats the returned ones by
    more than the score tolerance."""
    import test_gpu_search as ts

    n, nq, k = 1 << 22, 8, 10
    f = gu.fmt(3, prod=True)
    gp, op = gu.make_params(f, f)
    x = kv_inputs.kv_vectors(n, D, key="search-db", device="cuda", dtype=torch.bfloat16, outliers=True)
    pk = tq.Packed.empty(gp, n, tq.TQ_K)
    tq.tq_quantize(gp, x, tq.TQ_K, pk)
    q = kv_inputs.queries((nq, D), key=("search-q", nq), device="cuda")
    sc = torch.empty(nq, k, device="cuda")
    rw = torch.empty(nq, k, dtype=torch.int64, device="cuda")
    tq.tq_search(gp, tq.TQ_K, pk, n, q, k, sc, rw, tq.search_workspace())
    torch.cuda.synchronize()
    assert gp.status() == 0
    got_s, got_r = sc.cpu().numpy(), rw.cpu().numpy()
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(n, 200000, replace=False), got_r.ravel()]))
    idx = torch.from_numpy(rows).cuda()
    sub = o.Packed(pk.codes[idx].cpu().numpy(), pk.norms[idx].cpu().numpy(), pk.qjl[idx].cpu().numpy(),
                   pk.res_norms[idx].cpu().numpy())
    qd = q.double().cpu().numpy()
    all_s = o.ip_scores(op, qd, sub, "k")
    ts.check_topk(qd, got_s, got_r, all_s, pk.norms.cpu().numpy(), k, cand_rows=rows)
