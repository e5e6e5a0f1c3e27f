"""Plant plausible mistakes in the oracle and check that a pin catches each.

This is what makes the pins worth trusting: a dropped term, a wrong sign, a
swapped index or a reversed tie-break in the oracle must fail at least one of
them.  Mutations are applied with monkeypatch to the oracle module only.
"""
import numpy as np
import pytest

from oracle import dsa_ref as R
from tests import test_oracle as P


def _bad_mla_no_rope(q, kv, d_c, sm_scale):
    return R_orig_mla(q[:, :d_c], kv[:, :d_c], d_c, sm_scale)


def _bad_mla_values_include_rope(q, kv, d_c, sm_scale):
    o, lse = R_orig_mla(q, kv, kv.shape[1], sm_scale)
    return o[:, 1:d_c + 1], lse


def _bad_indexer_min(q, w, k):
    return np.minimum(k @ q.T, 0.0) @ w


def _bad_indexer_no_relu(q, w, k):
    return (k @ q.T) @ w


def _bad_topk_upper_tie(scores, k):
    n = scores.shape[0]
    pos = np.arange(n)
    order = np.lexsort((-pos, -np.asarray(scores, dtype=np.float64)))
    take = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int64)
    out[: take.shape[0]] = take
    return out


def _bad_e4m3_bias8(codes):
    return R_orig_e4m3(codes) / 2.0


R_orig_mla = R.sparse_mla_row
R_orig_e4m3 = R.e4m3_decode

CASES = [
    ("sparse_mla_row", _bad_mla_no_rope, [P.test_absorbed_equals_unabsorbed]),
    ("sparse_mla_row", _bad_mla_values_include_rope, [P.test_absorbed_equals_unabsorbed,
                                                      P.test_mla_brute_force]),
    ("indexer_row", _bad_indexer_min, [P.test_indexer_brute_force_fp8,
                                       P.test_indexer_weights_and_heads_not_transposed]),
    ("indexer_row", _bad_indexer_no_relu, [P.test_indexer_brute_force_fp8]),
    ("topk_row", _bad_topk_upper_tie, [P.test_topk_signed_zero_and_degenerate]),
    ("e4m3_decode", _bad_e4m3_bias8, [P.test_e4m3_decoder_matches_torch_on_all_codes]),
]


@pytest.mark.parametrize("name,bad,pins", CASES, ids=[c[1].__name__ for c in CASES])
def test_pin_catches_mutation(monkeypatch, name, bad, pins):
    monkeypatch.setattr(R, name, bad)
    for pin in pins:
        with pytest.raises(AssertionError):
            pin()
