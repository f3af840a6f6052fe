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
]
DEC_IDS = ["k3v3", "k4v3", "k4v4", "k2v2", "k1v1", "k3v2", "k4v2", "mixed", "mixed2.5", "prod3", "prod2", "prod4", "prod1"]


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
                                          (gu.fmt(3, prod=True), gu.fmt(3, prod=True), 0)],
                         ids=["k4v3sink", "mixed", "mixed2.5sink", "prod3"])
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
                want = o.quantize(op, xs[pos >= n_sink], side)
                codes = cache.plane(side + "_codes", torch.uint8, f.code_bytes(128))
                norms = cache.plane(side + "_norms", torch.float32, 1)
                got = o.Packed(codes[seq, h, qpos].cpu().numpy() if codes is not None else np.zeros((len(qpos), 0), np.uint8),
                               norms[seq, h, qpos, 0].cpu().numpy(),
                               cache.plane(side + "_qjl", torch.uint8, 16)[seq, h, qpos].cpu().numpy() if f.prod else np.zeros((len(qpos), 0), np.uint8),
                               cache.plane(side + "_res_norms", torch.float32, 1)[seq, h, qpos, 0].cpu().numpy() if f.prod else np.zeros(len(qpos), np.float32))
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
