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


def _encode_variant(y, half_away=False, sat=448.0, min_exp=-6):
    """The oracle's encoder with one slip switched on."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, min_exp)
    quantum = np.ldexp(1.0, e - 3)
    q = a / quantum
    v = (np.floor(q + 0.5) if half_away else np.rint(q)) * quantum
    v = np.minimum(v, sat)
    _, vex = np.frexp(v)
    ve = vex - 1
    normal = v >= 2.0 ** min_exp
    e_field = np.where(normal, ve + 7, 0)
    mant = np.where(normal, v / np.ldexp(1.0, ve) - 1.0, v / 2.0 ** min_exp) * 8.0
    mag = (e_field.astype(np.int64) << 3) | mant.astype(np.int64)
    return ((np.signbit(y).astype(np.int64) << 7) | mag).astype(np.uint8)


def _bad_encode_half_away(y):
    return _encode_variant(y, half_away=True)


def _bad_encode_no_saturation(y):
    return _encode_variant(y, sat=480.0)


def _bad_encode_subnormal_exponent(y):
    return _encode_variant(y, min_exp=-7)


def _bad_quantise_scale_240(k):
    k = np.asarray(k, dtype=np.float32)
    s = (np.max(np.abs(k), axis=1) / np.float32(240)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1)).astype(np.float32)
    return R.e4m3_encode((k / s[:, None]).astype(np.float32)), s


def _bad_physical_rows_mirrored_offset(seq, s, cache):
    s = np.asarray(s, dtype=np.int64)
    bt = cache.get("block_table")
    if bt is not None:
        page = int(cache["page_size"])
        return np.asarray(bt)[seq, s // page].astype(np.int64) * page + (page - 1 - s % page)
    return R_orig_rows(seq, s, cache)


def _bad_outproj_dim_major(o, w_uv, w_out):
    u = np.einsum("ivc,ic->iv", w_uv, o)
    return u, w_out @ u.T.reshape(-1)


def _bad_outproj_head0_weights(o, w_uv, w_out):
    u = np.einsum("vc,ic->iv", w_uv[0], o)
    return u, w_out @ u.reshape(-1)


def _bad_kl_grad_sign(p, scores):
    kl, g = R_orig_kl(p, scores)
    return kl, -g


def _bad_teacher_unnormalised(a):
    return a.sum(axis=0)


def _bad_backward_no_relu_mask(q, w, k, g):
    d = k @ q.T
    dw = np.maximum(d, 0.0).T @ g
    gd = g[:, None] * w[None, :]
    return gd.T @ k, dw, gd @ q


def _bad_backward_dk_without_w(q, w, k, g):
    dq, dw, _ = R_orig_bwd(q, w, k, g)
    on = (k @ q.T > 0).astype(np.float64)
    return dq, dw, (g[:, None] * on) @ q


R_orig_kl = R.indexer_kl_row
R_orig_bwd = R.indexer_backward_row
R_orig_rows = R.physical_rows
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
    ("e4m3_encode", _bad_encode_half_away, [P.test_e4m3_encode_is_nearest_value_ties_to_even,
                                            P.test_e4m3_encode_matches_torch_cast_in_range]),
    ("e4m3_encode", _bad_encode_no_saturation, [P.test_e4m3_encode_special_values,
                                                P.test_e4m3_encode_is_nearest_value_ties_to_even]),
    ("e4m3_encode", _bad_encode_subnormal_exponent,
     [P.test_e4m3_encode_inverts_decode_on_every_finite_code,
      P.test_e4m3_encode_matches_torch_cast_in_range]),
    ("quantise_keys", _bad_quantise_scale_240, [P.test_quantise_keys_error_bound_and_scale,
                                                P.test_quantise_keys_matches_generator_cast]),
    ("output_projection_row", _bad_outproj_dim_major,
     [P.test_output_projection_brute_force, P.test_output_projection_completes_the_pages_module]),
    ("output_projection_row", _bad_outproj_head0_weights,
     [P.test_output_projection_brute_force, P.test_output_projection_completes_the_pages_module]),
    ("indexer_kl_row", _bad_kl_grad_sign,
     [P.test_kl_gradient_against_finite_differences_and_autograd,
      P.test_indexer_backward_against_autograd]),
    ("teacher_distribution", _bad_teacher_unnormalised,
     [P.test_teacher_is_the_head_mean_of_the_dense_attention, P.test_indexer_backward_against_autograd]),
    ("indexer_backward_row", _bad_backward_no_relu_mask, [P.test_indexer_backward_against_autograd]),
    ("indexer_backward_row", _bad_backward_dk_without_w, [P.test_indexer_backward_against_autograd]),
    ("physical_rows", _bad_physical_rows_mirrored_offset,
     [lambda: P.test_cache_append_writes_where_the_layout_says(True)]),
]


@pytest.mark.parametrize("name,bad,pins", CASES, ids=[c[1].__name__ for c in CASES])
def test_pin_catches_mutation(monkeypatch, name, bad, pins):
    monkeypatch.setattr(R, name, bad)
    for pin in pins:
        with pytest.raises(AssertionError):
            pin()
