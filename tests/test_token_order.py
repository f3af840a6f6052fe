"""The decode kernel's per-format token orders (token_order in
tq_decode_common.cuh) against the shared-memory bank model that produced them
(csrc/bank_perm.py): each committed order is a permutation of the 16 tokens
of a subtile and costs no more wavefronts than the identity; formats without
an entry use the identity."""
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "online_vector_quantization_b200", "csrc")
sys.path.insert(0, CSRC)
import bank_perm as bp  # noqa: E402


def committed_orders():
    src = open(os.path.join(CSRC, "tq_decode_common.cuh")).read()
    body = src[src.index("constexpr uint64_t token_order("):]
    body = body[:body.index(";")]
    return {(int(k), int(v)): int(w, 16) for k, v, w in re.findall(r"kf == (\d+) && vf == (\d+)\s*\?\s*0x([0-9A-F]+)ull", body)}


ORDERS = committed_orders()


def test_every_order_has_a_model_entry():
    pairs = {(kf, vf) for kf, vf, *_ in bp.PAIRS}
    assert ORDERS and set(ORDERS) <= pairs


@pytest.mark.parametrize("kf,vf,fk,fv,chunk", bp.PAIRS, ids=[f"k{p[0]}v{p[1]}" for p in bp.PAIRS])
def test_order_is_a_permutation_no_worse_than_identity(kf, vf, fk, fv, chunk):
    ident = list(range(16))
    word = ORDERS.get((kf, vf))
    if word is None:
        return  # identity order
    pi = [(word >> (4 * k)) & 15 for k in range(16)]
    assert sorted(pi) == ident
    assert bp.cost(pi, fk, fv, chunk) <= bp.cost(ident, fk, fv, chunk)
