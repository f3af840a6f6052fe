"""Seeded synthetic inputs shaped like the KV-cache workloads of the pages.

Shared by the tests, the oracle checks and bench.py.  It holds none of the
method's arithmetic: only random vectors, queries and sequence lengths.

Recipe (the pages give no data; quality suites such as LongBench, NIAH and
RULER named in the NVIDIA forum post are not used and these inputs stand in
for real KV caches):
  head vector x = s * g, g ~ N(0, I_d), s = exp(0.5 * N(0, 1)) per vector
  (a lognormal(0, 0.5) scale); optional outlier channels are multiplied by 8
  before the scaling; the result is cast to the requested dtype.
  queries ~ N(0, I_d).
Every tensor is a pure function of (key, device): the same key gives the same
values on the same device type (CPU and CUDA streams differ).
"""
from __future__ import annotations

import hashlib

import torch

OUTLIER_CHANNELS = (5, 37, 70, 101)
OUTLIER_GAIN = 8.0
LOGNORMAL_SIGMA = 0.5


def _generator(key, device) -> torch.Generator:
    h = hashlib.sha256(repr(key).encode()).digest()
    gen = torch.Generator(device=device)
    gen.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return gen


def kv_vectors(n: int, d: int, key, device="cpu", dtype=torch.float32,
               outliers: bool = False) -> torch.Tensor:
    """(n, d) head vectors x = s * g as described in the module docstring."""
    gen = _generator(("kv", key), device)
    g = torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    if outliers:
        g[:, list(OUTLIER_CHANNELS)] *= OUTLIER_GAIN
    s = torch.exp(LOGNORMAL_SIGMA * torch.randn(n, generator=gen, device=device, dtype=torch.float32))
    return (g * s[:, None]).to(dtype)


def queries(shape, key, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    gen = _generator(("q", key), device)
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def planted_keys(k: torch.Tensor, q: torch.Tensor, group: int, lo: int, key,
                 cos: float = 0.9) -> torch.Tensor:
    """For one (sequence, kv-head): k (T, d), q (G, d) its query heads.

    Each query head h gets one position t_h >= lo (distinct, seeded) whose key
    is replaced by ||k_t|| (cos * q_h/||q_h|| + sqrt(1 - cos^2) w), w a random
    unit vector orthogonal to q_h: a key that the head attends to strongly.
    Returns a new tensor in k's dtype.
    """
    t_total, d = k.shape
    gen = _generator(("plant", key), "cpu")
    pos = torch.randperm(t_total - lo, generator=gen)[:group] + lo
    out = k.clone()
    kf = k.float()
    for h in range(group):
        qh = q[h].float()
        qh = qh / qh.norm()
        w = torch.randn(d, generator=gen).to(k.device)
        w = w - (w @ qh) * qh
        w = w / w.norm()
        t = int(pos[h])
        out[t] = (kf[t].norm() * (cos * qh + (1.0 - cos * cos) ** 0.5 * w)).to(k.dtype)
    return out


def sequence_lengths(n: int, lo: int, hi: int, key) -> list[int]:
    """n lengths uniform in [lo, hi] (inclusive)."""
    gen = _generator(("len", key), "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]
