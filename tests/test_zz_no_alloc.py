"""The no-allocation decode entry point (tq_decode_attn_noalloc) against the
regular one (tq_decode_attn with a caller workspace), through the C ABI.

Callers that cannot allocate device memory use this entry point; its
workspace is a fixed array the library defines in device memory.  This file is
collected last on purpose, and the test also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import kv_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import online_vector_quantization_b200 as tq  # noqa: E402

REL_L2 = 2e-3  # the decode-attention tolerance of the parity tests


def _rel(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / b.norm())


def test_noalloc_matches_workspace_entry_point_twice():
    p = tq.Params(4, 3)
    B, hkv, hq, T, n_sink = 3, 4, 16, 900, 16
    cache = tq.Cache(p, B, hkv, 1024, n_sink)
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    k = kv_inputs.kv_vectors(B * T * hkv, 128, key="na-k", device="cuda", dtype=torch.bfloat16).view(B, T, hkv, 128)
    v = kv_inputs.kv_vectors(B * T * hkv, 128, key="na-v", device="cuda", dtype=torch.bfloat16).view(B, T, hkv, 128)
    tq.tq_append(p, cache, ids, k, v)
    cache.lens.copy_(torch.tensor([T, 517, 33], dtype=torch.int32))
    ws = tq.decode_workspace(p, B, hq, hkv, T)
    for call in range(2):
        q = kv_inputs.queries((B, hq, 128), key=("na-q", call), device="cuda")
        want = torch.empty(B, hq, 128, dtype=torch.bfloat16, device="cuda")
        got = torch.full((B, hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        tq.tq_decode_attn(p, q, cache, T, want, ws, 1e-6)
        tq.tq_decode_attn_noalloc(p, q, cache, T, got, 1e-6)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert _rel(got, want) < REL_L2, call
    assert int(cache.status.item()) == 0


def test_noalloc_rejects_a_call_beyond_the_static_scratch():
    p = tq.Params(3, 3)
    cache = tq.Cache(p, 256, 8, 64, 0)  # 2048 (sequence, kv-head) units need more than 8 MiB
    q = torch.zeros(256, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(tq.TqError) as e:
        tq.tq_decode_attn_noalloc(p, q, cache, 64, out)
    assert e.value.status == 4
