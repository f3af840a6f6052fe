"""GPU parity of tq_search (top-k inner-product search over a quantized
database) against the oracle's search over the very same packed rows.

Scores are compared element by element within a tolerance derived from the
kernel's arithmetic (fp16 centroids and query halves, fp32 accumulation);
where scores lie closer than that tolerance the order of rows is not unique,
so the returned set is checked for validity instead: nothing left out beats
the returned rows by more than the tolerance, and the rows are distinct,
in range and sorted by the kernel's own scores."""
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
# score tolerance per unit of ||q|| * max ||x||: the query in fp16 (high
# halves only for more than 4 queries: at most 2^-12 relative per coordinate,
# about 2^-12 / sqrt(128) summed with random signs), centroids near-exact in
# fp16 after the per-width scaling, fp32 accumulation
SCORE_TOL = 2e-4


def build_db(f, n, key, which=tq.TQ_K, fv=None, boost=()):
    """n database rows; the rows in `boost` are scaled by 8, so that a query
    along one of them has that row as its clear best."""
    gp, op = gu.make_params(f, fv or f)
    x = kv_inputs.kv_vectors(max(n, 1), D, key=key, dtype=torch.bfloat16, outliers=True)[:n].clone()
    for r in boost:
        x[r] = x[r] * 8
    pk = tq.Packed.empty(gp, max(n, 1), which)
    if n:
        tq.tq_quantize(gp, x.cuda(), which, pk)
    torch.cuda.synchronize()
    return gp, op, x, pk


def run_search(gp, which, pk, n, q, k):
    ws = tq.search_workspace()
    scores = torch.full((q.shape[0], k), float("nan"), device="cuda")
    rows = torch.full((q.shape[0], k), -7, dtype=torch.int64, device="cuda")
    tq.tq_search(gp, which, pk, n, q.cuda(), k, scores, rows, ws)
    torch.cuda.synchronize()
    assert gp.status() == 0
    return scores.cpu().numpy(), rows.cpu().numpy()


def to_oracle(pk, n):
    return o.Packed(pk.codes[:n].cpu().numpy() if pk.codes is not None else np.zeros((n, 0), np.uint8),
                    pk.norms[:n].cpu().numpy(),
                    pk.qjl[:n].cpu().numpy() if pk.qjl is not None else np.zeros((n, 0), np.uint8),
                    pk.res_norms[:n].cpu().numpy() if pk.res_norms is not None else np.zeros(n, np.float32))


def check_topk(qd, got_s, got_r, all_s, norms, k, cand_rows=None):
    """all_s: oracle scores (Q, m) of rows cand_rows (default: all rows)."""
    n = all_s.shape[1] if cand_rows is None else None
    for i in range(qd.shape[0]):
        tau = SCORE_TOL * np.linalg.norm(qd[i]) * float(np.max(norms)) if norms.size else 0.0
        kk = k if n is None else min(k, n)
        r = got_r[i, :kk]
        assert (got_r[i, kk:] == -1).all() and np.isneginf(got_s[i, kk:]).all()
        assert len(set(r.tolist())) == kk and r.min() >= 0
        # sorted by the kernel's own scores, equal scores in row order
        for j in range(kk - 1):
            assert got_s[i, j] > got_s[i, j + 1] or (got_s[i, j] == got_s[i, j + 1] and r[j] < r[j + 1])
        if cand_rows is None:
            want = all_s[i, r]
            others = np.delete(all_s[i], r)
        else:
            pos = {int(c): j for j, c in enumerate(cand_rows)}
            want = np.array([all_s[i, pos[int(x)]] for x in r])
            others = all_s[i, [j for j, c in enumerate(cand_rows) if int(c) not in set(r.tolist())]]
        assert np.max(np.abs(got_s[i, :kk] - want)) <= tau, (i, np.max(np.abs(got_s[i, :kk] - want)), tau)
        if others.size:
            assert np.max(others) <= np.min(want) + 2 * tau
            # what is unique: every row that beats all rows outside the
            # oracle's top kk by more than the tolerance is returned
            cand = np.arange(all_s.shape[1]) if cand_rows is None else np.asarray(cand_rows)
            order = np.argsort(-all_s[i], kind="stable")
            if order.size > kk:
                edge = all_s[i, order[kk]]
                sure = cand[order[:kk]][all_s[i, order[:kk]] > edge + 2 * tau]
                assert set(sure.tolist()) <= set(r.tolist())


def queries(xd, nq, key, planted=()):
    """nq queries N(0, 1); query j of `planted` (j, row) points along row."""
    q = kv_inputs.queries((nq, D), key=key, dtype=torch.float32).double().numpy()
    for j, row in planted:
        q[j] = 2.0 * xd[row] / np.linalg.norm(xd[row])
    return q


SEARCH_FORMATS = [gu.fmt(1), gu.fmt(3), gu.fmt(4), gu.fmt(3, mixed=True), gu.fmt(2, mixed=True),
                  gu.fmt(1, prod=True), gu.fmt(3, prod=True), gu.fmt(4, prod=True), gu.fmt(8)]
SEARCH_IDS = ["mse1", "mse3", "mse4", "mixed3.5", "mixed2.5", "prod1", "prod3", "prod4", "mse8"]


@pytest.mark.parametrize("f", SEARCH_FORMATS, ids=SEARCH_IDS)
@pytest.mark.parametrize("nq,k", [(3, 10), (8, 32), (11, 1)], ids=["q3k10", "q8k32", "q11k1"])
def test_search_parity(f, nq, k):
    # several chunks per CTA of the persistent grid and a ragged tail of 3 rows
    n = 148 * 480 * 2 + 4 * 7 + 3
    gp, op, x, pk = build_db(f, n, ("srch", str(f)), boost=(12345, n - 1))
    xd = x.double().numpy()
    qd = queries(xd, nq, ("srq", str(f), nq), planted=[(0, 12345), (nq - 1, n - 1)])
    q = torch.from_numpy(qd).to(torch.bfloat16 if nq != 8 else torch.float32)
    qd = q.double().numpy()
    got_s, got_r = run_search(gp, tq.TQ_K, pk, n, q, k)
    opk = to_oracle(pk, n)
    all_s = o.ip_scores(op, qd, opk, "k")
    check_topk(qd, got_s, got_r, all_s, opk.norms, k)


def test_search_values_side_and_ties():
    # the V format of asymmetric parameters, and exact ties (duplicated rows)
    fk, fv = gu.fmt(4), gu.fmt(2, prod=True)
    n = 5000
    gp, op, x, pk = build_db(fk, n, "srv", which=tq.TQ_V, fv=fv, boost=(77,))
    for name in ("codes", "norms", "qjl", "res_norms"):
        t = getattr(pk, name)
        t[4000] = t[77]
        t[4001] = t[77]
    xd = x.double().numpy()
    qd = queries(xd, 4, "srvq", planted=[(2, 77)])
    q = torch.from_numpy(qd).float()
    got_s, got_r = run_search(gp, tq.TQ_V, pk, n, q, 8)
    opk = to_oracle(pk, n)
    all_s = o.ip_scores(op, qd, opk, "v")
    check_topk(qd, got_s, got_r, all_s, opk.norms, 8)
    assert got_r[2, :3].tolist() == [77, 4000, 4001]
    assert got_s[2, 0] == got_s[2, 1] == got_s[2, 2]


@pytest.mark.parametrize("n", [0, 1, 3, 5, 9], ids=lambda n: f"n{n}")
def test_search_short_databases(n):
    f = gu.fmt(3, prod=True)
    gp, op, x, pk = build_db(f, n, ("srs", n))
    qd = kv_inputs.queries((2, D), key=("srsq", n), dtype=torch.float32).double().numpy()
    got_s, got_r = run_search(gp, tq.TQ_K, pk, n, torch.from_numpy(qd).float(), 6)
    want_s, want_r = o.ip_search(op, qd, to_oracle(pk, n), 6, "k")
    assert (got_r[:, n:] == -1).all() and np.isneginf(got_s[:, n:]).all()
    if n:
        all_s = o.ip_scores(op, qd, to_oracle(pk, n), "k")
        check_topk(qd, got_s, got_r, all_s, pk.norms[:n].cpu().numpy(), 6)


def test_search_rejects_bad_arguments():
    f = gu.fmt(3)
    gp, op, x, pk = build_db(f, 64, "srb")
    q = torch.zeros(2, D, device="cuda")
    ws = tq.search_workspace()
    s = torch.zeros(2, 40, device="cuda")
    r = torch.zeros(2, 40, dtype=torch.int64, device="cuda")
    with pytest.raises(tq.TqError) as e:
        tq.tq_search(gp, tq.TQ_K, pk, 64, q, 33, s, r, ws)
    assert e.value.status == 2
    with pytest.raises(tq.TqError) as e:
        tq.tq_search(gp, tq.TQ_K, pk, 64, q, 0, s, r, ws)
    assert e.value.status == 1
    with pytest.raises(tq.TqError) as e:
        tq.tq_search(gp, tq.TQ_K, pk, 64, q, 4, s, r, ws[:100])
    assert e.value.status == 4


def test_search_with_bound_pass():
    # a database large enough for the leading-rows pass that seeds the bound
    f = gu.fmt(3)
    n = 8 * 148 * 480 + 1001
    gp, op, x, pk = build_db(f, n, "srl", boost=(70000, n - 2))
    xd = x.double().numpy()
    qd = queries(xd, 5, "srlq", planted=[(1, 70000), (3, n - 2)])
    q = torch.from_numpy(qd).to(torch.bfloat16)
    qd = q.double().numpy()
    got_s, got_r = run_search(gp, tq.TQ_K, pk, n, q, 16)
    opk = to_oracle(pk, n)
    check_topk(qd, got_s, got_r, o.ip_scores(op, qd, opk, "k"), opk.norms, 16)
