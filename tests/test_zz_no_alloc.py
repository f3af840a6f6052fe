"""The no-allocation decode entry point (tq_decode_attn_noalloc) against the
regular one (tq_decode_attn with a caller workspace), through the C ABI.

Callers that cannot allocate device memory (an engine that owns all device
memory in its own pool and calls this library from plugin code, or a decode
loop that cannot afford cudaMalloc's implicit synchronization) use this entry
point; its workspace is a fixed array the library defines in device memory.
Both entry points run the same kernels on the same inputs, so their outputs
must be identical.  This file is collected last on purpose, and the tests
also pass alone in a fresh process."""
import ctypes

import pytest
import torch

import kv_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import online_vector_quantization_b200 as tq  # noqa: E402

STATIC_SCRATCH_BYTES = 8 << 20


def _two_calls_match(p, B, hkv, hq, T, lens, n_sink, thr, key):
    cache = tq.Cache(p, B, hkv, ((T + 63) // 64) * 64, n_sink)
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    k = kv_inputs.kv_vectors(B * T * hkv, 128, key=(key, "k"), device="cuda", dtype=torch.bfloat16).view(B, T, hkv, 128)
    v = kv_inputs.kv_vectors(B * T * hkv, 128, key=(key, "v"), device="cuda", dtype=torch.bfloat16).view(B, T, hkv, 128)
    tq.tq_append(p, cache, ids, k, v)
    cache.lens.copy_(torch.tensor(lens, dtype=torch.int32))
    ws = tq.decode_workspace(p, B, hq, hkv, T)
    for call in range(2):
        q = kv_inputs.queries((B, hq, 128), key=(key, "q", call), device="cuda")
        want = torch.empty(B, hq, 128, dtype=torch.bfloat16, device="cuda")
        got = torch.full((B, hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        tq.tq_decode_attn(p, q, cache, T, want, ws, thr)
        tq.tq_decode_attn_noalloc(p, q, cache, T, got, thr)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all(), call
        assert torch.equal(got, want), (call, float((got.float() - want.float()).abs().max()))
    assert int(cache.status.item()) == 0


def test_noalloc_matches_workspace_entry_point_twice():
    # K4/V3 with a bf16 sink and sparse V, ragged lengths, GQA group of 4
    _two_calls_match(tq.Params(4, 3), B=3, hkv=4, hq=16, T=900, lens=[900, 517, 33], n_sink=16, thr=1e-6,
                     key="na-k4v3")


def test_noalloc_prod3_gqa_matches_workspace_entry_point_twice():
    # prod formats: wider partial slots (rotated + sketch accumulators), QJL
    # and residual-norm planes; GQA group of 4 over 2 kv-heads
    p = tq.Params(3, 3, tq.TQ_MODE_PROD, tq.TQ_MODE_PROD)
    _two_calls_match(p, B=2, hkv=2, hq=8, T=1300, lens=[1300, 611], n_sink=0, thr=0.0, key="na-prod3")


def test_noalloc_rejects_a_call_beyond_the_static_scratch():
    p = tq.Params(3, 3)
    cache = tq.Cache(p, 256, 8, 64, 0)  # 2048 (sequence, kv-head) units need more than 8 MiB
    q = torch.zeros(256, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    assert tq.tq_decode_workspace_bytes(p, 256, 64, 8, 64) > STATIC_SCRATCH_BYTES
    with pytest.raises(tq.TqError) as e:
        tq.tq_decode_attn_noalloc(p, q, cache, 64, out)
    assert e.value.status == 4


def test_noalloc_capacity_as_documented():
    # 780 (sequence, kv-head) units in MSE mode and 625 in prod mode with
    # groups of 4 query heads fit the 8 MiB scratch
    mse = tq.Params(3, 3)
    prod = tq.Params(3, 3, tq.TQ_MODE_PROD, tq.TQ_MODE_PROD)
    assert tq.tq_decode_workspace_bytes(mse, 780, 4, 1, 65536) <= STATIC_SCRATCH_BYTES
    assert tq.tq_decode_workspace_bytes(prod, 625, 4, 1, 65536) <= STATIC_SCRATCH_BYTES


def test_noalloc_checks_the_cache_like_the_workspace_entry_point():
    # a cache with a NULL code plane, and one with a misaligned norm plane: both
    # entry points refuse them on the host before anything is launched
    p = tq.Params(4, 3)
    cache = tq.Cache(p, 1, 1, 64, 0)
    cache.lens.fill_(10)
    q = torch.zeros(1, 1, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    flags = tq.TqAttnFlags(0.0, 0)
    ws = tq.decode_workspace(p, 1, 1, 1, 64)
    stream = torch.cuda.current_stream().cuda_stream

    def both(struct):
        a = tq._lib.tq_decode_attn_noalloc(p.handle, q.data_ptr(), tq.TQ_BF16, ctypes.byref(struct), 1, 1, 64,
                                           out.data_ptr(), tq.TQ_BF16, ctypes.byref(flags), stream)
        b = tq._lib.tq_decode_attn(p.handle, q.data_ptr(), tq.TQ_BF16, ctypes.byref(struct), 1, 1, 64,
                                   out.data_ptr(), tq.TQ_BF16, ws.data_ptr(), ws.numel(), ctypes.byref(flags),
                                   stream)
        return a, b

    no_codes = tq.TqCache.from_buffer_copy(cache.struct)
    no_codes.k_codes = None
    assert both(no_codes) == (1, 1)  # TQ_ERR_ARG
    bad_align = tq.TqCache.from_buffer_copy(cache.struct)
    bad_align.v_norms = cache.struct.v_norms + 4
    assert both(bad_align) == (3, 3)  # TQ_ERR_ALIGN
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
