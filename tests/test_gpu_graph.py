"""The public calls inside a CUDA graph.  tq_append and tq_decode_attn only
launch kernels on the caller's stream (the append's side stream, used when
the K and V formats differ, forks from and joins back into it): they allocate
nothing and never synchronize, so a step of append + decode can be captured
once and replayed.  A replay must give the same bits as the same calls made
eagerly, advance the lengths by the chunk each time, and leave the status
word at zero."""
from __future__ import annotations

import pytest
import torch

import kv_inputs
import online_vector_quantization_b200 as tq
import gpu_util as gu

pytestmark = pytest.mark.gpu

GRAPH_FORMATS = [
    (gu.fmt(3, mixed=True), gu.fmt(3, mixed=True)),  # one append kernel for K and V
    (gu.fmt(3, prod=True), gu.fmt(3, prod=True)),    # prod rows: quantize kernels on a side stream
    (gu.fmt(8), gu.fmt(3)),                          # K and V formats differ: fork / join
]


def _prefilled(gp, lens, hkv, cap, n_sink):
    cache = tq.Cache(gp, len(lens), hkv, cap, n_sink)
    for s, n in enumerate(lens):
        k = kv_inputs.kv_vectors(n * hkv, 128, key=("graph-pre", "k", s), dtype=torch.bfloat16).view(1, n, hkv, 128)
        v = kv_inputs.kv_vectors(n * hkv, 128, key=("graph-pre", "v", s), dtype=torch.bfloat16).view(1, n, hkv, 128)
        tq.tq_append(gp, cache, torch.tensor([s], dtype=torch.int32, device="cuda"), k.cuda(), v.cuda())
    return cache


@pytest.mark.parametrize("fk,fv", GRAPH_FORMATS, ids=["mixed3.5", "prod3", "k8v3"])
def test_captured_append_decode_step_replays_like_eager_calls(fk, fv):
    gp, _ = gu.make_params(fk, fv)
    lens, hkv, hq, cap, n_sink, chunk, steps = [300, 517, 9], 2, 8, 1024, 4, 16, 3
    n_seq = len(lens)
    ids = torch.arange(n_seq, dtype=torch.int32, device="cuda")
    ks = [kv_inputs.kv_vectors(n_seq * chunk * hkv, 128, key=("graph", "k", i), dtype=torch.bfloat16)
          .view(n_seq, chunk, hkv, 128).cuda() for i in range(steps)]
    vs = [kv_inputs.kv_vectors(n_seq * chunk * hkv, 128, key=("graph", "v", i), dtype=torch.bfloat16)
          .view(n_seq, chunk, hkv, 128).cuda() for i in range(steps)]
    qs = [kv_inputs.queries((n_seq, hq, 128), key=("graph", "q", i)).cuda() for i in range(steps)]

    # eager calls (these also set up the library's per-kernel attributes and
    # its side stream before any capture)
    ca = _prefilled(gp, lens, hkv, cap, n_sink)
    ws_a = tq.decode_workspace(gp, n_seq, hq, hkv, cap)
    want = []
    for i in range(steps):
        out = torch.empty(n_seq, hq, 128, dtype=torch.bfloat16, device="cuda")
        tq.tq_append(gp, ca, ids, ks[i], vs[i])
        tq.tq_decode_attn(gp, qs[i], ca, cap, out, ws_a)
        want.append(out)
    torch.cuda.synchronize()
    assert int(ca.status.item()) == 0

    # the same step captured once, replayed with each step's inputs copied in
    cb = _prefilled(gp, lens, hkv, cap, n_sink)
    ws_b = tq.decode_workspace(gp, n_seq, hq, hkv, cap)
    dk, dv, dq = torch.empty_like(ks[0]), torch.empty_like(vs[0]), torch.empty_like(qs[0])
    out_g = torch.empty(n_seq, hq, 128, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    lens_before = cb.lens.cpu().tolist()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tq.tq_append(gp, cb, ids, dk, dv)
        tq.tq_decode_attn(gp, dq, cb, cap, out_g, ws_b)
    torch.cuda.synchronize()
    assert cb.lens.cpu().tolist() == lens_before, "capturing must not run the append"
    for i in range(steps):
        dk.copy_(ks[i])
        dv.copy_(vs[i])
        dq.copy_(qs[i])
        g.replay()
        torch.cuda.synchronize()
        assert cb.lens.cpu().tolist() == [n + chunk * (i + 1) for n in lens], i
        assert torch.equal(out_g, want[i]), (i, (out_g.float() - want[i].float()).abs().max().item())
    assert int(cb.status.item()) == 0
    assert torch.equal(cb.lens, ca.lens)
    del g
