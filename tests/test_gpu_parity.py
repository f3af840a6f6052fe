"""GPU parity: every call of the C ABI against the oracle on the same seeded
inputs, at sizes the oracle finishes in seconds that still span several
tiles and a ragged tail, plus the edge cases of the method."""
import math

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

FORMATS = [gu.fmt(1), gu.fmt(2), gu.fmt(3), gu.fmt(4), gu.fmt(3, mixed=True), gu.fmt(2, mixed=True),
           gu.fmt(1, prod=True), gu.fmt(2, prod=True), gu.fmt(3, prod=True), gu.fmt(4, prod=True)]
FMT_IDS = ["mse1", "mse2", "mse3", "mse4", "mixed3.5", "mixed2.5", "prod1", "prod2", "prod3", "prod4"]


@pytest.mark.parametrize("f", FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_quantize_parity(f, dtype):
    gp, op = gu.make_params(f, f)
    n = 1000  # 15 full 64-vector tiles and a ragged tail of 40
    x = kv_inputs.kv_vectors(n, 128, key=("qp", f.bits, f.prod, f.mixed), dtype=dtype, outliers=True)
    x[7] = 0  # a zero vector
    xg = x.cuda()
    out = tq.Packed.empty(gp, n, tq.TQ_K)
    tq.tq_quantize(gp, xg, tq.TQ_K, out)
    torch.cuda.synchronize()
    got = gu.gpu_packed_to_numpy(out)
    xd = x.double().numpy()
    want = o.quantize(op, xd, "k")
    skip = gu.compare_codes(op, f, xd, got, want) if f.code_bytes(128) else set()
    assert np.allclose(got.norms, want.norms, rtol=1e-6, atol=0)
    gu.compare_qjl(op, f, xd, got, want, skip)
    assert not got.codes[7].any() and got.norms[7] == 0


@pytest.mark.parametrize("f", FORMATS, ids=FMT_IDS)
def test_quantize_many_tiles_per_cta(f):
    """bf16 rows run on the tensor-core kernels: enough 128-row tiles that
    every CTA of the persistent grid cycles its input ring, both accumulators
    and (prod) the residual tiles several times, plus a ragged tail."""
    gp, op = gu.make_params(f, f)
    n = 148 * 128 * 9 + 77
    x = kv_inputs.kv_vectors(n, 128, key=("qtc", f.bits, f.mixed), dtype=torch.bfloat16, outliers=True)
    x[12345] = 0
    out = tq.Packed.empty(gp, n, tq.TQ_V)
    tq.tq_quantize(gp, x.cuda(), tq.TQ_V, out)
    torch.cuda.synchronize()
    assert gp.status() == 0
    got = gu.gpu_packed_to_numpy(out)
    xd = x.double().numpy()
    want = o.quantize(op, xd, "v")
    skip = gu.compare_codes(op, f, xd, got, want) if f.code_bytes(128) else set()
    assert np.allclose(got.norms, want.norms, rtol=1e-6, atol=0)
    gu.compare_qjl(op, f, xd, got, want, skip)
    assert not got.codes[12345].any() and got.norms[12345] == 0


@pytest.mark.parametrize("f", FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_quantize_parity_hadamard_rotation(f, dtype):
    """The randomized Hadamard rotation (sign flips, then the normalized
    Walsh-Hadamard transform) in place of the Haar rotation: both quantize
    kernels (SIMT for fp32, tensor cores for bf16) across several tiles of
    the persistent grid and a ragged tail."""
    gp, op = gu.make_params(f, f, seed=11, rotation="hadamard")
    n = 148 * 128 + 333
    x = kv_inputs.kv_vectors(n, 128, key=("qh", f.bits, f.prod, f.mixed), dtype=dtype, outliers=True)
    x[5] = 0
    out = tq.Packed.empty(gp, n, tq.TQ_K)
    tq.tq_quantize(gp, x.cuda(), tq.TQ_K, out)
    torch.cuda.synchronize()
    assert gp.status() == 0
    got = gu.gpu_packed_to_numpy(out)
    xd = x.double().numpy()
    want = o.quantize(op, xd, "k")
    skip = gu.compare_codes(op, f, xd, got, want) if f.code_bytes(128) else set()
    assert np.allclose(got.norms, want.norms, rtol=1e-6, atol=0)
    gu.compare_qjl(op, f, xd, got, want, skip)
    assert not got.codes[5].any() and got.norms[5] == 0


@pytest.mark.parametrize("f", FORMATS, ids=FMT_IDS)
def test_dequantize_parity(f):
    gp, op = gu.make_params(f, f)
    n = 777
    x = kv_inputs.kv_vectors(n, 128, key=("dq", f.bits, f.prod, f.mixed), dtype=torch.bfloat16, outliers=True)
    want_pk = o.quantize(op, x.double().numpy(), "v")
    want = o.dequantize(op, want_pk, "v")
    out = torch.empty(n, 128, dtype=torch.float32, device="cuda")
    tq.tq_dequantize(gp, gu.numpy_packed_to_gpu(want_pk), n, tq.TQ_V, out)
    got = out.cpu().numpy()
    assert np.max(np.abs(got - want)) <= gu.DEQUANT_ATOL


def _decode_case(fk, fv, B, hq, hkv, T, lens, n_sink, thr, q_dtype=torch.bfloat16, out_dtype=torch.bfloat16,
                 key="dec", rotation="haar"):
    gp, op = gu.make_params(fk, fv, rotation=rotation)
    k = kv_inputs.kv_vectors(B * hkv * T, 128, key=(key, "k"), dtype=torch.bfloat16)
    v = kv_inputs.kv_vectors(B * hkv * T, 128, key=(key, "v"), dtype=torch.bfloat16)
    kd = k.double().numpy().reshape(B, hkv, T, 128)
    vd = v.double().numpy().reshape(B, hkv, T, 128)
    q = kv_inputs.queries((B, hq, 128), key=(key, "q"), dtype=q_dtype)
    ocache = o.cache_from_vectors(op, kd, vd, n_sink)
    want = o.decode_attention(op, q.double().numpy(), ocache, lens, hkv, thr)
    cap = ((T + 63) // 64) * 64
    cache = tq.Cache(gp, B, hkv, cap, n_sink)
    gu.fill_cache_from_oracle(cache, op, ocache, lens, B, hkv)
    max_len = max(max(lens), 1)
    ws = tq.decode_workspace(gp, B, hq, hkv, max_len)
    out = torch.full((B, hq, 128), float("nan"), dtype=out_dtype, device="cuda")
    tq.tq_decode_attn(gp, q.cuda(), cache, max_len, out, ws, thr)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert int(cache.status.item()) == 0
    if out_dtype == torch.bfloat16:
        floor = gu.rel_l2(torch.from_numpy(want).to(torch.bfloat16).double().numpy(), want)
        print(f"decode rel L2 {gu.rel_l2(got, want):.3e} (bf16 rounding of the exact output alone: {floor:.3e})")
    return got, want, (gp, op, cache, ws, q, out, max_len)


DECODE_FORMATS = [
    (gu.fmt(3), gu.fmt(3)),
    (gu.fmt(4), gu.fmt(3)),
    (gu.fmt(4), gu.fmt(4)),
    (gu.fmt(2), gu.fmt(2)),
    (gu.fmt(1), gu.fmt(1)),
    (gu.fmt(3), gu.fmt(2)),
    (gu.fmt(4), gu.fmt(2)),
    (gu.fmt(3, mixed=True), gu.fmt(3, mixed=True)),
    (gu.fmt(2, mixed=True), gu.fmt(2, mixed=True)),
    (gu.fmt(3, prod=True), gu.fmt(3, prod=True)),
    (gu.fmt(2, prod=True), gu.fmt(2, prod=True)),
    (gu.fmt(4, prod=True), gu.fmt(4, prod=True)),
    (gu.fmt(1, prod=True), gu.fmt(1, prod=True)),
    (gu.fmt(8), gu.fmt(3)),
]
DEC_IDS = ["k3v3", "k4v3", "k4v4", "k2v2", "k1v1", "k3v2", "k4v2", "mixed", "mixed2.5", "prod3", "prod2", "prod4", "prod1",
           "k8v3"]


@pytest.mark.parametrize("fk,fv", DECODE_FORMATS, ids=DEC_IDS)
def test_decode_parity_formats(fk, fv):
    # several splits per sequence, ragged lengths, GQA group of 4
    got, want, _ = _decode_case(fk, fv, B=2, hq=8, hkv=2, T=2500, lens=[2500, 1777], n_sink=0, thr=0.0,
                                key=("fmt", str(fk), str(fv)))
    assert gu.rel_l2(got, want) < gu.ATTN_REL_L2


@pytest.mark.parametrize("fk,fv", [(gu.fmt(4), gu.fmt(3)), (gu.fmt(3, mixed=True), gu.fmt(3, mixed=True)),
                                   (gu.fmt(3, prod=True), gu.fmt(3, prod=True))], ids=["k4v3", "mixed", "prod3"])
def test_decode_parity_hadamard_rotation(fk, fv):
    # the query rotation and the output un-rotation use the Hadamard Pi
    got, want, _ = _decode_case(fk, fv, B=2, hq=8, hkv=2, T=1500, lens=[1500, 999], n_sink=16, thr=0.0,
                                key=("had", str(fk), str(fv)), rotation="hadamard")
    assert gu.rel_l2(got, want) < gu.ATTN_REL_L2


def test_decode_sink_sparse_v_gqa8():
    # config-4-like: G = 8, bf16 sink, sparse V at 1e-6, lengths around the sink
    lens = [700, 129, 128, 50]
    got, want, _ = _decode_case(gu.fmt(4), gu.fmt(3), B=4, hq=16, hkv=2, T=700, lens=lens, n_sink=128,
                                thr=1e-6, key="sink")
    assert gu.rel_l2(got, want) < gu.ATTN_REL_L2


def test_decode_fp32_single_head():
    # config-1-like: one fp32 query head, fp32 output
    got, want, _ = _decode_case(gu.fmt(3), gu.fmt(3), B=1, hq=1, hkv=1, T=4096, lens=[4096], n_sink=0, thr=0.0,
                                q_dtype=torch.float32, out_dtype=torch.float32, key="f32")
    err = gu.rel_l2(got, want)
    print(f"fp32 decode rel L2 = {err:.3e}")
    assert err < gu.ATTN_REL_L2


def test_decode_empty_and_tiny_sequences():
    lens = [0, 1, 17, 300]
    got, want, (gp, op, cache, ws, q, out, max_len) = _decode_case(
        gu.fmt(3), gu.fmt(3), B=4, hq=4, hkv=2, T=320, lens=lens, n_sink=0, thr=0.0, key="tiny")
    assert not np.any(got[0])
    assert gu.rel_l2(got[1:], want[1:]) < gu.ATTN_REL_L2
    # the workspace is left ready: a second call gives the same result
    tq.tq_decode_attn(gp, q.cuda(), cache, max_len, out, ws, 0.0)
    torch.cuda.synchronize()
    assert np.array_equal(out.float().cpu().numpy(), got)


def test_decode_length_above_bound_sets_status():
    got, want, (gp, op, cache, ws, q, out, max_len) = _decode_case(
        gu.fmt(3), gu.fmt(3), B=1, hq=2, hkv=1, T=256, lens=[256], n_sink=0, thr=0.0, key="bound")
    tq.tq_decode_attn(gp, q.cuda(), cache, 200, out, ws, 0.0)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & 2


@pytest.mark.parametrize("fk,fv,n_sink", [(gu.fmt(4), gu.fmt(3), 8), (gu.fmt(3, mixed=True), gu.fmt(3, mixed=True), 0),
                                          (gu.fmt(2, mixed=True), gu.fmt(2, mixed=True), 4),
                                          (gu.fmt(3, prod=True), gu.fmt(3, prod=True), 0),
                                          (gu.fmt(8), gu.fmt(3), 8)],
                         ids=["k4v3sink", "mixed", "mixed2.5sink", "prod3", "k8v3sink"])
def test_append_parity(fk, fv, n_sink):
    gp, op = gu.make_params(fk, fv)
    n_seq, hkv, cap = 3, 2, 256
    cache = tq.Cache(gp, n_seq, hkv, cap, n_sink)
    start = [0, 5, 100]
    cache.lens.copy_(torch.tensor(start, dtype=torch.int32))
    n_tok = 64
    k = kv_inputs.kv_vectors(n_seq * n_tok * hkv, 128, key=("ap", "k"), dtype=torch.bfloat16).view(n_seq, n_tok, hkv, 128)
    v = kv_inputs.kv_vectors(n_seq * n_tok * hkv, 128, key=("ap", "v"), dtype=torch.bfloat16).view(n_seq, n_tok, hkv, 128)
    seq_ids = torch.tensor([2, 0, 1], dtype=torch.int32, device="cuda")  # input row s -> cache sequence
    tq.tq_append(gp, cache, seq_ids, k.cuda(), v.cuda())
    torch.cuda.synchronize()
    lens = cache.lens.cpu().tolist()
    order = [2, 0, 1]
    assert lens == [start[i] + n_tok for i in range(3)]
    for s_in, seq in enumerate(order):
        for h in range(hkv):
            for side, x, f in (("k", k, fk), ("v", v, fv)):
                xs = x[s_in, :, h].double().numpy()
                pos = np.arange(start[seq], start[seq] + n_tok)
                qpos = pos[pos >= n_sink] - n_sink
                if len(qpos):
                    want = o.quantize(op, xs[pos >= n_sink], side)
                    got = gu.read_unit_rows(cache, f, side, seq, h, int(qpos[0]), len(qpos))
                    xq = xs[pos >= n_sink]
                    skip = gu.compare_codes(op, f, xq, got, want) if f.code_bytes(128) else set()
                    assert np.allclose(got.norms, want.norms, rtol=1e-6)
                    gu.compare_qjl(op, f, xq, got, want, skip)
                if n_sink and (pos < n_sink).any():
                    sink = cache.plane(side + "_sink", torch.bfloat16, 128)
                    sp = pos[pos < n_sink]
                    assert torch.equal(sink[seq, h, sp].cpu(), x[s_in, pos < n_sink, h].to(torch.bfloat16))
    # an append past capacity is refused as a whole and flagged
    big = torch.zeros(1, 200, hkv, 128, dtype=torch.bfloat16, device="cuda")
    tq.tq_append(gp, cache, torch.tensor([2], dtype=torch.int32, device="cuda"), big, big)
    torch.cuda.synchronize()
    assert cache.lens.cpu().tolist() == lens
    assert int(cache.status.item()) & 1


def test_gpu_built_cache_attention_matches_oracle_built():
    # append-built cache (GPU quantize) vs the oracle's own cache and attention
    fk = fv = gu.fmt(3, mixed=True)
    gp, op = gu.make_params(fk, fv)
    B, hkv, hq, T = 2, 2, 8, 640
    k = kv_inputs.kv_vectors(B * T * hkv, 128, key=("gb", "k"), dtype=torch.bfloat16).view(B, T, hkv, 128)
    v = kv_inputs.kv_vectors(B * T * hkv, 128, key=("gb", "v"), dtype=torch.bfloat16).view(B, T, hkv, 128)
    q = kv_inputs.queries((B, hq, 128), key=("gb", "q"))
    cache = tq.Cache(gp, B, hkv, T, 0)
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    for c0 in range(0, T, 64):
        tq.tq_append(gp, cache, ids, k[:, c0:c0 + 64].contiguous().cuda(), v[:, c0:c0 + 64].contiguous().cuda())
    ws = tq.decode_workspace(gp, B, hq, hkv, T)
    out = torch.empty(B, hq, 128, dtype=torch.bfloat16, device="cuda")
    tq.tq_decode_attn(gp, q.cuda(), cache, T, out, ws)
    torch.cuda.synchronize()
    kd = k.double().numpy().transpose(0, 2, 1, 3)
    vd = v.double().numpy().transpose(0, 2, 1, 3)
    ocache = o.cache_from_vectors(op, kd, vd, 0)
    want = o.decode_attention(op, q.double().numpy(), ocache, [T, T], hkv)
    assert gu.rel_l2(out.float().cpu().numpy(), want) < gu.ATTN_REL_L2


GQA_FORMATS = [(gu.fmt(3, mixed=True), gu.fmt(3, mixed=True)), (gu.fmt(4), gu.fmt(3)),
               (gu.fmt(3, prod=True), gu.fmt(3, prod=True)), (gu.fmt(1), gu.fmt(1)), (gu.fmt(8), gu.fmt(3))]


@pytest.mark.parametrize("group", [1, 2, 3, 5, 6, 7, 8])
@pytest.mark.parametrize("fk,fv", GQA_FORMATS, ids=["mixed", "k4v3", "prod3", "k1v1", "k8v3"])
def test_decode_parity_gqa_groups(fk, fv, group):
    """Every query-head group size the boundary accepts: groups of up to 4 pack
    the query's high and low halves into spare MMA columns (3 leaves two of the
    eight columns empty), larger groups run unpacked with 8 - group empty
    columns."""
    got, want, _ = _decode_case(fk, fv, B=2, hq=2 * group, hkv=2, T=1100, lens=[1100, 613], n_sink=0, thr=0.0,
                                key=("gqa", str(fk), group))
    assert gu.rel_l2(got, want) < gu.ATTN_REL_L2


def _oracle_weights(op, q, ocache, b, kvh, group, nq):
    """Final softmax weights (group, nq) of the quantized tokens of one unit
    (no sink), by plain attention over the oracle's dequantized keys."""
    kr = ocache.k_rows[b, kvh]
    keys = o.dequantize(op, o.Packed(kr.codes[:nq], kr.norms[:nq], kr.qjl[:nq], kr.res_norms[:nq]), "k")
    s = q[b, kvh * group:(kvh + 1) * group] @ keys.T / math.sqrt(128)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("fk,fv,group", [(gu.fmt(4), gu.fmt(3), 4), (gu.fmt(4), gu.fmt(3), 8),
                                         (gu.fmt(3, mixed=True), gu.fmt(3, mixed=True), 4)],
                         ids=["k4v3g4", "k4v3g8", "mixedg4"])
def test_decode_sparse_v_drops_and_matches_oracle(fk, fv, group):
    """Peaked queries (N(0,1) scaled by 8): most softmax weights fall below
    1e-6, the kernel drops their values and skips whole tiles, and the output
    still matches the oracle's exact rule (drop a token's value when its final
    weight is below the threshold).  The kernel's bound is conservative: every
    weight it drops is one the exact rule drops."""
    B, hkv, T, thr = 2, 2, 3000, 1e-6
    hq = hkv * group
    gp, op = gu.make_params(fk, fv)
    key = ("sparse", str(fk), group)
    k = kv_inputs.kv_vectors(B * hkv * T, 128, key=(key, "k"), dtype=torch.bfloat16)
    v = kv_inputs.kv_vectors(B * hkv * T, 128, key=(key, "v"), dtype=torch.bfloat16)
    q = (kv_inputs.queries((B, hq, 128), key=(key, "q"), dtype=torch.float32) * 8).to(torch.bfloat16)
    ocache = o.cache_from_vectors(op, k.double().numpy().reshape(B, hkv, T, 128),
                                  v.double().numpy().reshape(B, hkv, T, 128), 0)
    lens = [T, 2345]
    qd = q.double().numpy()
    want = o.decode_attention(op, qd, ocache, lens, hkv, thr)
    cache = tq.Cache(gp, B, hkv, ((T + 63) // 64) * 64, 0)
    gu.fill_cache_from_oracle(cache, op, ocache, lens, B, hkv)
    ws = tq.decode_workspace(gp, B, hq, hkv, T)
    out = torch.empty(B, hq, 128, dtype=torch.bfloat16, device="cuda")
    stats = torch.zeros(4, dtype=torch.int64, device="cuda")
    tq.tq_decode_attn(gp, q.cuda(), cache, T, out, ws, thr, sparse_v_stats=stats)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    examined, dropped, tiles, skipped = (int(x) for x in stats.cpu())
    exact_dropped = sum(int((_oracle_weights(op, qd, ocache, b, h, group, lens[b]) < thr).sum())
                        for b in range(B) for h in range(hkv))
    print(f"sparse V: kernel dropped {dropped}/{examined} weights ({dropped / examined:.3f}), exact rule "
          f"{exact_dropped / examined:.3f}; tiles skipped {skipped}/{tiles} ({skipped / tiles:.3f})")
    assert examined == sum(lens) * hkv * group
    assert dropped / examined > 0.5
    assert dropped <= exact_dropped
    assert gu.rel_l2(out.float().cpu().numpy(), want) < gu.ATTN_REL_L2


def test_decode_sparse_v_skips_whole_tiles():
    """A value tile's work is skipped only when all its (token, head) weights
    are dropped, and a warp can only tell once it has met a large score.  One
    unit of 6 x 148 x 480 tokens (several 480-token chunks per CTA of the
    persistent grid): in every third chunk the first token of every 32-token
    tile is a strong key (norm 30, cos 0.99 with the query); the rest are
    ordinary keys, whose scores sit ~20 below.  Warps meet a strong key early in
    their range and then skip the tiles of ordinary keys after it, whatever
    the exact chunk ranges of the CTAs; the output matches the oracle's exact
    rule."""
    fk, fv = gu.fmt(4), gu.fmt(3)
    gp, op = gu.make_params(fk, fv)
    T, thr = 6 * 148 * 480, 1e-6
    q = kv_inputs.queries((1, 1, 128), key=("skip", "q"), dtype=torch.float32)
    k = kv_inputs.kv_vectors(T, 128, key=("skip", "k"), dtype=torch.float32)
    v = kv_inputs.kv_vectors(T, 128, key=("skip", "v"), dtype=torch.float32)
    pos = np.arange(T)
    strong = ((pos // 480) % 3 == 0) & (pos % 32 == 0)
    qh = q[0, 0] / q[0, 0].norm()
    w = kv_inputs.kv_vectors(int(strong.sum()), 128, key=("skip", "w"), dtype=torch.float32)
    w = w - (w @ qh)[:, None] * qh[None]
    w = w / w.norm(dim=1, keepdim=True)
    k[torch.from_numpy(strong)] = 30.0 * (0.99 * qh[None] + (1 - 0.99 ** 2) ** 0.5 * w)
    k = k.to(torch.bfloat16)
    v = v.to(torch.bfloat16)
    q = q.to(torch.bfloat16)
    ocache = o.cache_from_vectors(op, k.double().numpy()[None, None], v.double().numpy()[None, None], 0)
    want = o.decode_attention(op, q.double().numpy(), ocache, [T], 1, thr)
    cache = tq.Cache(gp, 1, 1, T, 0)
    gu.fill_cache_from_oracle(cache, op, ocache, [T], 1, 1)
    ws = tq.decode_workspace(gp, 1, 1, 1, T)
    out = torch.empty(1, 1, 128, dtype=torch.bfloat16, device="cuda")
    stats = torch.zeros(4, dtype=torch.int64, device="cuda")
    tq.tq_decode_attn(gp, q.cuda(), cache, T, out, ws, thr, sparse_v_stats=stats)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    examined, dropped, tiles, skipped = (int(x) for x in stats.cpu())
    print(f"sparse V, planted keys: dropped {dropped}/{examined}, tiles skipped {skipped}/{tiles}")
    assert examined == T and tiles == T // 32
    assert skipped / tiles > 0.3 and dropped / examined > 0.6
    assert gu.rel_l2(out.float().cpu().numpy(), want) < gu.ATTN_REL_L2


def test_tiny_fp32_quantize_append_decode_end_to_end():
    """The tiny MSE-only configuration as stated: 4096 fp32 vectors (d = 128,
    lognormal norms), 3-bit codes quantized on the GPU, dequantized, then
    appended to a one-head cache as keys and values alike and attended by one
    fp32 query; the GPU-built cache against the oracle's own."""
    f = gu.fmt(3)
    gp, op = gu.make_params(f, f)
    n = 4096
    x = kv_inputs.kv_vectors(n, 128, key="c1")
    xd = x.double().numpy()
    pk = tq.Packed.empty(gp, n, tq.TQ_K)
    tq.tq_quantize(gp, x.cuda(), tq.TQ_K, pk)
    torch.cuda.synchronize()
    got = gu.gpu_packed_to_numpy(pk)
    want_pk = o.quantize(op, xd, "k")
    gu.compare_codes(op, f, xd, got, want_pk)
    assert np.allclose(got.norms, want_pk.norms, rtol=1e-6, atol=0)
    # dequantization of the GPU's codes, against the oracle's on the same codes
    xh = torch.empty(n, 128, dtype=torch.float32, device="cuda")
    tq.tq_dequantize(gp, pk, n, tq.TQ_K, xh)
    torch.cuda.synchronize()
    assert np.max(np.abs(xh.cpu().numpy() - o.dequantize(op, got, "k"))) <= gu.DEQUANT_ATOL
    # K = V = the same vectors through the streaming append (fp32 input)
    cache = tq.Cache(gp, 1, 1, n, 0)
    xs = x.view(1, n, 1, 128).cuda()
    tq.tq_append(gp, cache, torch.zeros(1, dtype=torch.int32, device="cuda"), xs, xs)
    torch.cuda.synchronize()
    assert cache.lens.cpu().tolist() == [n] and int(cache.status.item()) == 0
    assert np.array_equal(gu.read_unit_rows(cache, f, "k", 0, 0, 0, n).codes, got.codes)
    assert np.array_equal(gu.read_unit_rows(cache, f, "v", 0, 0, 0, n).codes, got.codes)
    q = kv_inputs.queries((1, 1, 128), key="c1q", dtype=torch.float32)
    ws = tq.decode_workspace(gp, 1, 1, 1, n)
    out = torch.empty(1, 1, 128, dtype=torch.float32, device="cuda")
    tq.tq_decode_attn(gp, q.cuda(), cache, n, out, ws)
    torch.cuda.synchronize()
    ocache = o.cache_from_vectors(op, xd[None, None], xd[None, None], 0)
    want = o.decode_attention(op, q.double().numpy(), ocache, [n], 1)
    err = gu.rel_l2(out.cpu().numpy(), want)
    print(f"tiny fp32 case (4096 vectors, fp32 query and output, GPU-built cache vs the oracle's): rel L2 {err:.3e}")
    assert err < gu.ATTN_REL_L2


ALL_CODE_FORMATS = [gu.fmt(1), gu.fmt(2), gu.fmt(3), gu.fmt(4), gu.fmt(3, mixed=True), gu.fmt(2, mixed=True),
                    gu.fmt(2, prod=True), gu.fmt(3, prod=True), gu.fmt(4, prod=True), gu.fmt(8)]
ALL_CODE_IDS = ["mse1", "mse2", "mse3", "mse4", "mixed3.5", "mixed2.5", "prod2", "prod3", "prod4", "mse8"]


def _tile_spec_offsets(f, side):
    """The tiled code layout as include/tq.h states it, written out on its
    own: for token i (0..15) of a tile, the tile byte of every byte of its
    packed row.  Lane L = 4g + t; a key lane owns tokens g, g + 8 and quarter
    t of each segment, a value lane tokens 2t, 2t+1, 2t+8, 2t+9 and eighth g;
    lane blocks of code_bytes / 2 bytes are stored as 16-byte columns while
    16 bytes remain, then an 8- and a 4-byte column as needed."""
    cb = f.code_bytes(128)
    w = [f.mse_bits(j, 128) for j in range(128)]
    segs = [(0, 64), (64, 128)] if f.mixed else [(0, 128)]
    seg_start = [sum(w[:a]) // 8 for a, _ in segs]
    seg_bytes = [sum(w[a:b]) // 8 for a, b in segs]
    lb = cb // 2
    cols = [16] * (lb // 16)
    rest = lb % 16
    for width in (8, 4):
        if rest >= width:
            cols.append(width)
            rest -= width
    assert rest == 0

    def tile_byte(lane, p):
        base = 0
        for width in cols:
            if p < width:
                return base + lane * width + p
            p -= width
            base += 32 * width
        raise AssertionError

    table = {}
    for tok in range(16):
        m = {}
        for si, (sb, nb) in enumerate(zip(seg_start, seg_bytes)):
            if side == "k":
                g, role, parts = tok % 8, tok // 8, 4
                piece = nb // 4
                prior = sum(2 * (seg_bytes[x] // 4) for x in range(si))
                for t in range(parts):
                    for i in range(piece):
                        m[sb + t * piece + i] = tile_byte(4 * g + t, prior + role * piece + i)
            else:
                t, member = (tok % 8) // 2, tok % 2 + 2 * (tok // 8)
                piece = nb // 8
                prior = sum(4 * (seg_bytes[x] // 8) for x in range(si))
                for g in range(8):
                    for i in range(piece):
                        m[sb + g * piece + i] = tile_byte(4 * g + t, prior + member * piece + i)
        assert sorted(m) == list(range(cb))
        table[tok] = m
    assert sorted(v for m in table.values() for v in m.values()) == list(range(16 * cb))
    return table


@pytest.mark.parametrize("f", ALL_CODE_FORMATS, ids=ALL_CODE_IDS)
@pytest.mark.parametrize("side", ["k", "v"])
def test_cache_rows_round_trip_and_tile_layout(f, side):
    """tq_cache_write_rows / tq_cache_read_rows round-trip arbitrary packed rows
    at a ragged offset, and the code plane holds them exactly as the tile
    layout of include/tq.h says."""
    fk = f if side == "k" else gu.fmt(1)
    fv = f if side == "v" else gu.fmt(1)
    gp, op = gu.make_params(fk, fv)
    cap, n, row0 = 256, 150, 37
    cache = tq.Cache(gp, 2, 3, cap, 0)
    rng = np.random.default_rng(7)
    cb = f.code_bytes(128)
    pk = o.Packed(rng.integers(0, 256, (n, cb), dtype=np.uint8), rng.random(n).astype(np.float32),
                  rng.integers(0, 256, (n, 16 if f.prod else 0), dtype=np.uint8),
                  rng.random(n).astype(np.float32) if f.prod else np.zeros(n, np.float32))
    gu.write_unit_rows(cache, side, 1, 2, row0, pk)
    back = gu.read_unit_rows(cache, f, side, 1, 2, row0, n)
    assert np.array_equal(back.codes, pk.codes) and np.array_equal(back.norms, pk.norms)
    if f.prod:
        assert np.array_equal(back.qjl, pk.qjl) and np.array_equal(back.res_norms, pk.res_norms)
    # the raw code plane of unit (1, 2) against the stated layout
    plane = cache.buffer[getattr(cache.struct, side + "_codes") - cache.buffer.data_ptr():]
    unit = plane[(1 * 3 + 2) * cap * cb:(1 * 3 + 2 + 1) * cap * cb].cpu().numpy().reshape(cap // 16, 16 * cb)
    spec = _tile_spec_offsets(f, side)
    for r in range(n):
        pos = row0 + r
        tile, tok = divmod(pos, 16)
        offs = spec[tok]
        assert all(unit[tile, offs[j]] == pk.codes[r, j] for j in range(cb)), r
    # the other units are untouched
    other = plane[:cap * cb].cpu().numpy()
    assert not other.any()


@pytest.mark.parametrize("fk,fv", [(gu.fmt(3, mixed=True), gu.fmt(3, mixed=True)), (gu.fmt(4), gu.fmt(3)),
                                   (gu.fmt(3, prod=True), gu.fmt(3, prod=True)), (gu.fmt(2, mixed=True),
                                                                                  gu.fmt(2, mixed=True)),
                                   (gu.fmt(8), gu.fmt(3))],
                         ids=["mixed3.5", "k4v3", "prod3", "mixed2.5", "k8v3"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_append_rows_equal_quantize_rows(fk, fv, dtype):
    """Appending in ragged 64-token chunks stores, bit for bit, the rows
    tq_quantize produces for the same vectors (both kernels families: tensor
    cores for bf16, SIMT for fp32), at every tile position."""
    gp, _ = gu.make_params(fk, fv)
    hkv, T = 2, 203
    cache = tq.Cache(gp, 1, hkv, 256, 3)
    k = kv_inputs.kv_vectors(T * hkv, 128, key=("ar", "k"), dtype=dtype).view(1, T, hkv, 128).cuda()
    v = kv_inputs.kv_vectors(T * hkv, 128, key=("ar", "v"), dtype=dtype).view(1, T, hkv, 128).cuda()
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    for c0 in range(0, T, 64):
        tq.tq_append(gp, cache, ids, k[:, c0:c0 + 64].contiguous(), v[:, c0:c0 + 64].contiguous())
    torch.cuda.synchronize()
    assert cache.lens.cpu().tolist() == [T] and int(cache.status.item()) == 0
    for side, x, which in (("k", k, tq.TQ_K), ("v", v, tq.TQ_V)):
        f = fk if side == "k" else fv
        for h in range(hkv):
            xs = x[0, 3:, h].contiguous()
            ref = tq.Packed.empty(gp, T - 3, which)
            tq.tq_quantize(gp, xs, which, ref)
            torch.cuda.synchronize()
            want = gu.gpu_packed_to_numpy(ref)
            got = gu.read_unit_rows(cache, f, side, 0, h, 0, T - 3)
            assert np.array_equal(got.codes, want.codes), (side, h)
            assert np.array_equal(got.norms, want.norms)
            if f.prod:
                assert np.array_equal(got.qjl, want.qjl) and np.array_equal(got.res_norms, want.res_norms)


# ---------------------------------------------------------------------------
# 8-bit codes (256 centroids, one byte per coordinate): the fp32 path rotates
# in fp64 on the SIMT cores, the bf16 path on the tensor cores with a
# three-term split of Pi; both search the codebook through uniform cells.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("rotation", ["haar", "hadamard"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_quantize_parity_8bit(dtype, rotation):
    f = gu.fmt(8)
    gp, op = gu.make_params(f, gu.fmt(3), seed=5, rotation=rotation)
    # bf16: several 128-row tiles per CTA of the persistent grid and a ragged
    # tail; fp32: one vector per block, a ragged count
    n = 148 * 128 * 3 + 77 if dtype == torch.bfloat16 else 3001
    x = kv_inputs.kv_vectors(n, 128, key=("q8", rotation), dtype=dtype, outliers=True)
    x[9] = 0
    out = tq.Packed.empty(gp, n, tq.TQ_K)
    tq.tq_quantize(gp, x.cuda(), tq.TQ_K, out)
    torch.cuda.synchronize()
    assert gp.status() == 0
    got = gu.gpu_packed_to_numpy(out)
    xd = x.double().numpy()
    want = o.quantize(op, xd, "k")
    gu.compare_codes(op, f, xd, got, want)
    assert np.allclose(got.norms, want.norms, rtol=1e-6, atol=0)
    assert not got.codes[9].any() and got.norms[9] == 0
    # the levels are reached across the range (all 256 on the larger bf16
    # set; the outermost few are rare in 3001 vectors)
    assert len(np.unique(got.codes)) >= (256 if n > 10000 else 248)


def test_dequantize_parity_8bit():
    gp, op = gu.make_params(gu.fmt(8), gu.fmt(3))
    n = 555
    x = kv_inputs.kv_vectors(n, 128, key="dq8", dtype=torch.bfloat16, outliers=True)
    want_pk = o.quantize(op, x.double().numpy(), "k")
    want = o.dequantize(op, want_pk, "k")
    out = torch.empty(n, 128, dtype=torch.float32, device="cuda")
    tq.tq_dequantize(gp, gu.numpy_packed_to_gpu(want_pk), n, tq.TQ_K, out)
    assert np.max(np.abs(out.cpu().numpy() - want)) <= gu.DEQUANT_ATOL


def test_decode_k8v3_beats_k4v3_on_the_same_vectors():
    """8-bit keys reach the exact (unquantized-key) attention more closely
    than 4-bit keys over the same values: the decode kernel reads the wider
    codes without losing what they add."""
    B, hq, hkv, T = 2, 8, 2, 1500
    lens = [1500, 1111]
    k = kv_inputs.kv_vectors(B * hkv * T, 128, key=("k8cmp", "k"), dtype=torch.bfloat16)
    v = kv_inputs.kv_vectors(B * hkv * T, 128, key=("k8cmp", "v"), dtype=torch.bfloat16)
    q = kv_inputs.queries((B, hq, 128), key=("k8cmp", "q"))
    kd = k.double().numpy().reshape(B, hkv, T, 128)
    vd = v.double().numpy().reshape(B, hkv, T, 128)
    errs = {}
    for kb in (4, 8):
        gp, op = gu.make_params(gu.fmt(kb), gu.fmt(3))
        ocache = o.cache_from_vectors(op, kd, vd, 0)
        # exact keys, the values as quantized: isolates the keys' error
        exact = np.zeros((B, hq, 128))
        group = hq // hkv
        for b in range(B):
            for h in range(hq):
                kvh = h // group
                vr = ocache.v_rows[b, kvh]
                n = lens[b]
                vals = o.dequantize(op, o.Packed(vr.codes[:n], vr.norms[:n], vr.qjl[:n], vr.res_norms[:n]), "v")
                s = kd[b, kvh, :n] @ q[b, h].double().numpy() / math.sqrt(128)
                w = np.exp(s - s.max())
                exact[b, h] = (w / w.sum()) @ vals
        cache = tq.Cache(gp, B, hkv, ((T + 63) // 64) * 64, 0)
        gu.fill_cache_from_oracle(cache, op, ocache, lens, B, hkv)
        ws = tq.decode_workspace(gp, B, hq, hkv, T)
        out = torch.empty(B, hq, 128, dtype=torch.float32, device="cuda")
        tq.tq_decode_attn(gp, q.cuda(), cache, T, out, ws)
        torch.cuda.synchronize()
        errs[kb] = gu.rel_l2(out.cpu().numpy(), exact)
    print(f"rel L2 vs exact keys: K4 {errs[4]:.3e}  K8 {errs[8]:.3e}")
    assert errs[8] < 0.25 * errs[4]


@pytest.mark.parametrize("fk,fv,dtype", [(gu.fmt(3, mixed=True), gu.fmt(3, mixed=True), torch.bfloat16),
                                         (gu.fmt(3, prod=True), gu.fmt(3, prod=True), torch.bfloat16),
                                         (gu.fmt(4), gu.fmt(3), torch.bfloat16),
                                         (gu.fmt(3, mixed=True), gu.fmt(3, mixed=True), torch.float32),
                                         (gu.fmt(8), gu.fmt(3), torch.float32)],
                         ids=["mixed-one-launch", "prod3-one-launch", "k4v3-two-kernels", "mixed-f32", "k8v3-f32"])
def test_append_length_update_folded(fk, fv, dtype):
    """The last CTA of an append updates lens (no separate launch): ragged
    appends to shuffled subsets of the sequences leave every length exact,
    the stored rows equal to tq_quantize's, and the status word (the CTA count
    in its high half included) back at zero; an append that does not fit
    leaves its sequence's length alone and sets bit 1 only."""
    gp, _ = gu.make_params(fk, fv)
    n_seq, hkv, cap, n_sink = 5, 2, 512, 4
    cache = tq.Cache(gp, n_seq, hkv, cap, n_sink)
    rng = np.random.default_rng(31)
    expect = [0] * n_seq
    held = {s: [] for s in range(n_seq)}  # (k, v) chunks per sequence, in order
    for step in range(12):
        n_tok = int(rng.integers(1, 41))
        seqs = [int(s) for s in rng.permutation(n_seq)[:int(rng.integers(1, n_seq + 1))]]
        k = kv_inputs.kv_vectors(len(seqs) * n_tok * hkv, 128, key=("fold", "k", step), dtype=dtype)
        v = kv_inputs.kv_vectors(len(seqs) * n_tok * hkv, 128, key=("fold", "v", step), dtype=dtype)
        k = k.view(len(seqs), n_tok, hkv, 128)
        v = v.view(len(seqs), n_tok, hkv, 128)
        tq.tq_append(gp, cache, torch.tensor(seqs, dtype=torch.int32, device="cuda"), k.cuda(), v.cuda())
        for i, s in enumerate(seqs):
            expect[s] += n_tok
            held[s].append((k[i], v[i]))
        torch.cuda.synchronize()
        assert cache.lens.cpu().tolist() == expect, step
        assert int(cache.status.item()) == 0, step
    # the quantized rows of two sequences against tq_quantize of the same vectors
    for s in (0, 3):
        if expect[s] <= n_sink:
            continue
        for side, which, f in (("k", tq.TQ_K, fk), ("v", tq.TQ_V, fv)):
            x = torch.cat([kv[0 if side == "k" else 1] for kv in held[s]], 0)  # (len, hkv, d)
            for h in range(hkv):
                xs = x[n_sink:, h].contiguous().cuda()
                ref = tq.Packed.empty(gp, xs.shape[0], which)
                tq.tq_quantize(gp, xs, which, ref)
                torch.cuda.synchronize()
                want = gu.gpu_packed_to_numpy(ref)
                got = gu.read_unit_rows(cache, f, side, s, h, 0, xs.shape[0])
                assert np.array_equal(got.codes, want.codes), (s, side, h)
                assert np.array_equal(got.norms, want.norms)
    # refused: neither sequence 2 nor 4 can take 600 more tokens; then 8 fit
    big = kv_inputs.kv_vectors(2 * 600 * hkv, 128, key="fold-big", dtype=dtype).view(2, 600, hkv, 128)
    seqs = torch.tensor([2, 4], dtype=torch.int32, device="cuda")
    tq.tq_append(gp, cache, seqs, big.cuda(), big.cuda())
    torch.cuda.synchronize()
    assert cache.lens.cpu().tolist() == expect
    assert int(cache.status.item()) == 1
    small = big[:, :8].contiguous().cuda()
    cache.status.zero_()
    tq.tq_append(gp, cache, torch.tensor([4], dtype=torch.int32, device="cuda"), small[:1], small[:1])
    torch.cuda.synchronize()
    expect[4] += 8
    assert cache.lens.cpu().tolist() == expect and int(cache.status.item()) == 0


def test_decode_reads_query_and_cache_written_just_before():
    """The decode call's kernels start under programmatic stream
    serialization, overlapping the previous kernel's tail: a query produced by
    the kernel right before the call, after an append that filled the cache,
    must still be read as written.  Each call is compared with the same call
    made after a full synchronization."""
    fk = fv = gu.fmt(3, mixed=True)
    gp, _ = gu.make_params(fk, fv)
    B, hkv, hq, T = 3, 2, 8, 700
    k = kv_inputs.kv_vectors(B * T * hkv, 128, key=("pdl", "k"), dtype=torch.bfloat16).view(B, T, hkv, 128).cuda()
    v = kv_inputs.kv_vectors(B * T * hkv, 128, key=("pdl", "v"), dtype=torch.bfloat16).view(B, T, hkv, 128).cuda()
    base = kv_inputs.queries((B, hq, 128), key=("pdl", "q"), dtype=torch.float32).cuda()
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    ws = tq.decode_workspace(gp, B, hq, hkv, T)
    for trial in range(3):
        cache = tq.Cache(gp, B, hkv, 704, 0)
        out_fast = torch.empty(B, hq, 128, dtype=torch.bfloat16, device="cuda")
        for c0 in range(0, T, 64):
            c1 = min(T, c0 + 64)
            tq.tq_append(gp, cache, ids, k[:, c0:c1].contiguous(), v[:, c0:c1].contiguous())
        # the query comes from a kernel launched just before the decode call
        q = (base * (1.0 + 0.5 * trial)).to(torch.bfloat16)
        tq.tq_decode_attn(gp, q, cache, T, out_fast, ws)
        torch.cuda.synchronize()
        out_sync = torch.empty_like(out_fast)
        q2 = q.clone()
        torch.cuda.synchronize()
        tq.tq_decode_attn(gp, q2, cache, T, out_sync, ws)
        torch.cuda.synchronize()
        assert torch.equal(out_fast, out_sync), trial
        assert cache.lens.cpu().tolist() == [T] * B and int(cache.status.item()) == 0


def test_back_to_back_steps_match_synchronized_steps():
    """The append's kernel starts under programmatic stream serialization
    right after the previous step's merge (which lets it launch early), and
    its input comes from the kernel just before it: step after step without a
    synchronization, every decode output and the final lengths must equal
    those of the same steps with a full synchronization around every call."""
    fk = fv = gu.fmt(3, mixed=True)
    gp, _ = gu.make_params(fk, fv)
    B, hkv, hq, chunk, steps = 4, 2, 8, 48, 6
    lens0 = [130, 0, 515, 64]
    k = kv_inputs.kv_vectors(steps * B * chunk * hkv, 128, key=("b2b", "k"), dtype=torch.float32).view(steps, B, chunk, hkv, 128).cuda()
    v = kv_inputs.kv_vectors(steps * B * chunk * hkv, 128, key=("b2b", "v"), dtype=torch.float32).view(steps, B, chunk, hkv, 128).cuda()
    qs = kv_inputs.queries((steps, B, hq, 128), key=("b2b", "q"), dtype=torch.float32).cuda()
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    cap = 896

    def prefilled():
        cache = tq.Cache(gp, B, hkv, cap, 0)
        for s, n in enumerate(lens0):
            if n:
                x = kv_inputs.kv_vectors(n * hkv, 128, key=("b2b-pre", s), dtype=torch.bfloat16).view(1, n, hkv, 128).cuda()
                tq.tq_append(gp, cache, torch.tensor([s], dtype=torch.int32, device="cuda"), x, x)
        torch.cuda.synchronize()
        return cache

    outs = {}
    for mode in ("sync", "fast"):
        cache = prefilled()
        ws = tq.decode_workspace(gp, B, hq, hkv, cap)
        outs[mode] = []
        for i in range(steps):
            # the chunk and the query are written by the kernels just before the calls
            kc, vc = k[i].to(torch.bfloat16), v[i].to(torch.bfloat16)
            q = qs[i].to(torch.bfloat16)
            if mode == "sync":
                torch.cuda.synchronize()
            tq.tq_append(gp, cache, ids, kc, vc)
            if mode == "sync":
                torch.cuda.synchronize()
            out = torch.empty(B, hq, 128, dtype=torch.bfloat16, device="cuda")
            tq.tq_decode_attn(gp, q, cache, cap, out, ws)
            if mode == "sync":
                torch.cuda.synchronize()
            outs[mode].append(out)
        torch.cuda.synchronize()
        assert cache.lens.cpu().tolist() == [n + steps * chunk for n in lens0], mode
        assert int(cache.status.item()) == 0, mode
    for i in range(steps):
        assert torch.equal(outs["fast"][i], outs["sync"][i]), i
