"""Pins for the float64 oracle: it is checked against things other than itself.

Each test states what it pins and which plausible slip it would catch.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats

from oracle import dsa_ref as R
from long_context_sparse_04_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# P8: number formats against an independent decoder (torch casts)
# --------------------------------------------------------------------------

def test_e4m3_decoder_matches_torch_on_all_codes():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = R.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                      # 0x7F and 0xFF only
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x80] == 0.0


def test_bf16_decoder_matches_torch():
    import torch
    bits = np.random.default_rng(0).integers(0, 2 ** 16, size=5000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]     # drop inf/nan patterns
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ref, R.bf16_decode(bits))


# --------------------------------------------------------------------------
# P1: brute force, pure Python loops, L <= 64
# --------------------------------------------------------------------------

def _brute_indexer(q8, qs, w, k8, ks, klen):
    """Scalar loops over the definition, decoding each byte on its own."""
    def dec(c):                                  # OCP e4m3, written again by hand
        s = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 15, c & 7
        return s * (2.0 ** -6) * m / 8 if e == 0 else s * 2.0 ** (e - 7) * (1 + m / 8)
    out = []
    for s_ in range(klen):
        acc = 0.0
        for j in range(len(w)):
            dot = 0.0
            for d in range(len(k8[s_])):
                dot += dec(int(q8[j][d])) * float(qs[j]) * dec(int(k8[s_][d])) * float(ks[s_])
            acc += float(w[j]) * (dot if dot > 0 else 0.0)
        out.append(acc)
    return out


def test_indexer_brute_force_fp8():
    cfg = I.CONFIGS["prefill_8k"].replace(seq_len=48, h_idx=3, d_idx=16, topk=8,
                                         n_heads=2, d_c=8, d_r=4, plant_frac=0.1)
    inp = I.generate(cfg, threads=1)
    for t in (0, 5, 31, 47):
        got = R.row_scores(inp, t)
        ref = _brute_indexer(inp["q_idx"][t], inp["q_scale"][t], inp["w"][t],
                             inp["k_idx"], inp["k_scale"], t + 1)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_mla_brute_force():
    rng = np.random.default_rng(1)
    H, dc, dr, n = 3, 6, 2, 9
    q = rng.standard_normal((H, dc + dr))
    kv = rng.standard_normal((n, dc + dr))
    scale = 0.37
    o, lse = R.sparse_mla_row(q, kv, dc, scale)
    for i in range(H):
        z = [scale * sum(q[i][d] * kv[s][d] for d in range(dc + dr)) for s in range(n)]
        den = sum(math.exp(v) for v in z)
        assert abs(lse[i] - math.log(den)) < 1e-12
        for d in range(dc):
            ref = sum(math.exp(z[s]) / den * kv[s][d] for s in range(n))
            assert abs(o[i][d] - ref) < 1e-12


def test_lse_matches_library_logsumexp():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 10)) * 3
    kv = rng.standard_normal((50, 10))
    _, lse = R.sparse_mla_row(q, kv, 7, 0.9)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(0.9 * q @ kv.T, axis=1), rtol=1e-13)


# --------------------------------------------------------------------------
# P2: top-k equals a full stable sort, with ties and signed zeros
# --------------------------------------------------------------------------

def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda s: (-float(scores[s]), s))[:k]
    order = sorted(order)
    return order + [-1] * (k - len(order))


@pytest.mark.parametrize("seed", range(12))
def test_topk_equals_stable_sort(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 40))
    vals = rng.choice([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 2.0, 3.5], size=n) \
        if seed % 2 else rng.standard_normal(n).round(1)
    for k in (1, 3, 7, 40, 64):
        assert list(R.topk_row(vals, k)) == _brute_topk(vals, k)


def test_topk_signed_zero_and_degenerate():
    v = np.array([0.0, -0.0, 0.0, -0.0, -1.0])
    assert list(R.topk_row(v, 2)) == [0, 1]          # -0 == +0: lower index wins
    assert list(R.topk_row(np.zeros(0), 4)) == [-1, -1, -1, -1]
    assert list(R.topk_row(np.array([5.0, 1.0]), 4)) == [0, 1, -1, -1]
    assert R.kth_score(np.array([3.0, 9.0, 1.0, 7.0]), 2) == 7.0
    assert R.kth_score(np.array([3.0, 9.0]), 5) == 3.0


# --------------------------------------------------------------------------
# P3: k >= visible keys makes sparse MLA the dense MLA
# --------------------------------------------------------------------------

def test_full_k_equals_dense_attention():
    inp = I.generate(I.CONFIGS["tiny_fp32"].replace(seq_len=40), threads=1)
    res = R.dsa_forward_rows(inp, range(40), topk=64)
    lat = inp["latent"].astype(np.float64)
    for t, idx, o, lse in zip(res["rows"], res["idx"], res["out"], res["lse"]):
        assert list(idx[: t + 1]) == list(range(t + 1)) and (idx[t + 1:] == -1).all()
        z = inp["sm_scale"] * inp["q"][t].astype(np.float64) @ lat[: t + 1].T
        p = scipy.special.softmax(z, axis=1)
        np.testing.assert_allclose(o, p @ lat[: t + 1, :64], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, scipy.special.logsumexp(z, axis=1), rtol=1e-13)


# --------------------------------------------------------------------------
# P4: outputs are convex combinations of the selected value latents
# --------------------------------------------------------------------------

def test_output_is_convex_combination():
    inp = I.generate(I.CONFIGS["tiny_fp32"], threads=1)
    res = R.dsa_forward_rows(inp, [3, 100, 255])
    lat = inp["latent"].astype(np.float64)
    for t, idx, o, lse in zip(res["rows"], res["idx"], res["out"], res["lse"]):
        sel = idx[idx >= 0]
        assert len(sel) == min(64, t + 1)
        c = lat[sel, :64]
        assert (o >= c.min(axis=0) - 1e-12).all() and (o <= c.max(axis=0) + 1e-12).all()
        z = inp["sm_scale"] * inp["q"][t].astype(np.float64) @ lat[sel].T
        np.testing.assert_allclose(np.exp(z - lse[:, None]).sum(axis=1), 1.0, rtol=1e-12)


# --------------------------------------------------------------------------
# P5: the page's single-head ReLU(q.k/sqrt(d_I)) is the H_I=1 special case
# --------------------------------------------------------------------------

def test_single_head_reduction():
    rng = np.random.default_rng(3)
    for d in (32, 64, 128):
        q = rng.standard_normal(d)
        k = rng.standard_normal((100, d))
        np.testing.assert_allclose(R.indexer_row(q[None], np.array([1 / math.sqrt(d)]), k),
                                   R.indexer_row_single_head(q, k), rtol=1e-13, atol=1e-15)


def test_indexer_weights_and_heads_not_transposed():
    # distinct per-head weights: a swapped (t, j) index or a dropped head changes I
    q = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    w = np.array([2.0, -3.0, 0.5])
    k = np.array([[1.0, 2.0], [-1.0, 1.0], [-1.0, -1.0]])
    # hand evaluation: s0 dots (1,2,3) -> 2-6+1.5; s1 (-1,1,0) -> -3; s2 all <= 0 -> 0
    np.testing.assert_allclose(R.indexer_row(q, w, k), [-2.5, -3.0, 0.0])


# --------------------------------------------------------------------------
# P6: absorbed MLA equals MLA with explicit W_UK / W_UV up-projections
# --------------------------------------------------------------------------

def test_absorbed_equals_unabsorbed():
    rng = np.random.default_rng(4)
    H, d_h, d_v, d_c, d_r, n = 4, 12, 10, 16, 6, 30
    c = rng.standard_normal((n, d_c))
    kr = rng.standard_normal((n, d_r))
    qn = rng.standard_normal((H, d_h))
    qr = rng.standard_normal((H, d_r))
    w_uk = rng.standard_normal((H, d_h, d_c)) / 3
    w_uv = rng.standard_normal((H, d_v, d_c)) / 3
    u_ref = R.unabsorbed_mla_row(qn, qr, c, kr, w_uk, w_uv)
    q_abs = np.concatenate([np.einsum("hdc,hd->hc", w_uk, qn), qr], axis=1)
    o, _ = R.sparse_mla_row(q_abs, np.concatenate([c, kr], axis=1), d_c, 1 / math.sqrt(d_h + d_r))
    u = np.einsum("hvc,hc->hv", w_uv, o)
    np.testing.assert_allclose(u, u_ref, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# P7: counts the pages print
# --------------------------------------------------------------------------

def test_page_counts():
    g = json.load(open(os.path.join(GOLDEN, "page_counts.json")))
    e = g["causal_pairs_131072"]
    cfg = I.CONFIGS["prefill_64k"].replace(seq_len=e["L"])
    _, klen = I.row_layout(cfg)
    pairs = int(klen.astype(np.int64).sum())
    assert pairs == 8_590_000_128
    assert abs(pairs - e["value"]) <= e["rel_tol"] * e["value"]
    s = g["sparsity_k2048_L131072"]
    assert 1 - s["k"] / s["L"] > s["value"]
    f = g["fraction_k2048_L128000"]
    assert abs(f["k"] / f["L"] - f["value"]) <= f["rel_tol"] * f["value"]
    assert I.CONFIGS["decode_128k_paged"].topk == g["topk_value"]["value"]


# --------------------------------------------------------------------------
# cache addressing: a paged layout and a contiguous layout of the same blocks
# give the same results (block table indirection done right)
# --------------------------------------------------------------------------

def test_paged_equals_contiguous():
    base = I.CONFIGS["decode_128k_paged"].replace(
        ctx_lo=150, ctx_hi=300, n_seqs=3, h_idx=4, d_idx=16, topk=32, n_heads=2, d_c=8, d_r=4)
    a = I.generate(base, threads=1)
    b = I.generate(base.replace(paged=False), threads=1)
    assert (a["row_klen"] == b["row_klen"]).all()
    assert a["cache"]["block_table"] is not None and b["cache"]["block_table"] is None
    ra = R.dsa_forward_rows(a, range(6))
    rb = R.dsa_forward_rows(b, range(6))
    for x, y in zip(ra["scores"], rb["scores"]):
        np.testing.assert_array_equal(x, y)
    for x, y in zip(ra["out"], rb["out"]):
        np.testing.assert_array_equal(x, y)


def test_generator_layout_rules():
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=100, ctx_hi=200, n_seqs=4,
                                                h_idx=2, d_idx=16, n_heads=2, d_c=8, d_r=8)
    seq, klen = I.row_layout(cfg)
    ctx = I.context_lengths(cfg)
    assert list(seq) == [0, 0, 1, 1, 2, 2, 3, 3]
    assert list(klen) == [int(c) - 1 + j for c in ctx for j in (0, 1)]
    inp = I.generate(cfg, threads=1)
    bt = inp["cache"]["block_table"]
    used = bt[bt >= 0]
    assert sorted(used) == list(range(inp["cache"]["num_pages"]))   # a permutation
    # FP8 quantisation: |codes| <= 448 and dequantised keys within one e4m3 step
    k = R.dequant_keys(inp, np.arange(64))
    assert np.isfinite(k).all()
    assert np.abs(R.e4m3_decode(inp["k_idx"])).max() <= 448


def test_planted_keys_point_at_their_query():
    cfg = I.CONFIGS["prefill_8k"].replace(seq_len=256, h_idx=4, plant_frac=0.05)
    found = 0
    for chunk in range(1):
        for off, tgt, head in I._plant_targets(cfg, 0, chunk):
            s = chunk * I.CHUNK + off
            assert s <= tgt < 256
            kc, ks, _ = I.key_chunk(cfg, 0, chunk)
            kv = R.e4m3_decode(kc[off]) * ks[off]
            qv = I.qidx_rows_f32(cfg, [tgt])[0, head].astype(np.float64)
            cos = kv @ qv / np.linalg.norm(kv) / np.linalg.norm(qv)
            assert cos > 0.99 and abs(np.linalg.norm(kv) - 4 * math.sqrt(128)) < 2.0
            found += 1
    assert found > 0


# --------------------------------------------------------------------------
# P9: FP8 quantisation and the cache append
# --------------------------------------------------------------------------

_FINITE_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def test_e4m3_encode_inverts_decode_on_every_finite_code():
    # every representable value maps back to its own code, -0.0 included
    assert np.array_equal(R.e4m3_encode(R.e4m3_decode(_FINITE_CODES)), _FINITE_CODES)


def test_e4m3_encode_is_nearest_value_ties_to_even():
    """Brute force over the 254 finite codes: the code of y is the one whose
    value is nearest; of two equally near, the one with an even mantissa; above
    448, the largest (saturation).  Ties are planted at every midpoint."""
    vals = R.e4m3_decode(_FINITE_CODES)
    pos = np.unique(vals[vals >= 0])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(7)
    y = np.concatenate([mids, -mids, rng.uniform(-470, 470, 4000),
                        rng.standard_normal(2000) * 2.0 ** rng.integers(-12, 6, 2000),
                        [0.0, 448.0, 448.1, 463.9, 464.0, 1e30, -1e30]])
    got = R.e4m3_encode(y)
    for yi, g in zip(y, got):
        d = np.abs(vals - min(abs(yi), 448.0) * (1 if yi >= 0 else -1))
        cand = _FINITE_CODES[d == d.min()]
        cand = cand[(cand >> 7) == (1 if np.signbit(yi) else 0)] if len(cand) > 1 else cand
        if len(cand) > 1:
            cand = cand[(cand & 1) == 0]
        assert len(cand) == 1 and g == cand[0], (yi, hex(g), [hex(c) for c in cand])


def test_e4m3_encode_matches_torch_cast_in_range():
    # torch's float8 cast rounds to nearest even but turns overflow into NaN,
    # so it is compared on [-448, 448]
    import torch
    rng = np.random.default_rng(8)
    pos = np.unique(np.abs(R.e4m3_decode(_FINITE_CODES)))
    mids = (pos[1:] + pos[:-1]) / 2                  # every tie, exact in fp32
    y = np.concatenate([mids, -mids, rng.uniform(-448, 448, 20000),
                        rng.standard_normal(20000) * 2.0 ** rng.integers(-14, 8, 20000)])
    y = np.clip(y, -448, 448).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(R.e4m3_encode(y.astype(np.float64)), ref)


def test_e4m3_encode_special_values():
    cases = {448.0: 0x7E, 449.0: 0x7E, 1e9: 0x7E, -1e9: 0xFE, 2.0 ** -9: 0x01,
             2.0 ** -10: 0x00, 3 * 2.0 ** -10: 0x02, 1.0: 0x38, -2.0: 0xC0, 0.0: 0x00,
             1.0625: 0x38, 1.1875: 0x3A, 2.0 ** -6: 0x08, 7 * 2.0 ** -9: 0x07}
    for y, c in cases.items():
        assert R.e4m3_encode(np.array([y]))[0] == c, y
    assert R.e4m3_encode(np.array([-0.0]))[0] == 0x80
    assert R.e4m3_encode(np.array([-1e-6]))[0] == 0x80
    with pytest.raises(ValueError):
        R.e4m3_encode(np.array([np.nan]))


def test_quantise_keys_error_bound_and_scale():
    """Dequantised keys are within half a step of the input: relative 2^-4 in
    the normal range, absolute 2^-10 * s below it; the largest magnitude of a
    token lands on +-448; an all-zero token gets scale 1 and zero codes."""
    rng = np.random.default_rng(9)
    k = (rng.standard_normal((300, 128)) * np.exp(rng.uniform(-20, 8, (300, 1)))).astype(np.float32)
    k[0] = 0.0
    k[1, :] = 0.0
    k[1, 5] = -3.0
    codes, s = R.quantise_keys(k)
    assert s.dtype == np.float32 and s[0] == 1.0 and not codes[0].any()
    deq = R.e4m3_decode(codes) * s[:, None].astype(np.float64)
    bound = np.maximum(2.0 ** -4 * np.abs(k.astype(np.float64)), 2.0 ** -10 * s[:, None])
    assert np.all(np.abs(deq - k) <= bound * (1 + 1e-6))
    assert np.all(np.abs(R.e4m3_decode(codes[1:])).max(axis=1) == 448.0)
    assert codes[1, 5] == 0xFE and s[1] == np.float32(3.0) / np.float32(448)


def test_quantise_keys_matches_generator_cast():
    # the input generator quantises with torch's cast after a clip: another
    # implementation of the same rule
    rng = np.random.default_rng(10)
    k = (rng.standard_normal((500, 128)) * 3).astype(np.float32)
    codes, s = R.quantise_keys(k)
    g_codes, g_s = I.to_e4m3_rows(k)
    assert np.array_equal(codes, g_codes) and np.array_equal(s, g_s)


def _logical_view(inp, seq, arr):
    """A sequence's cache rows in logical order, built by concatenating its
    pages in block-table order (paged) or slicing from its start."""
    c = inp["cache"]
    if c["block_table"] is not None:
        pg = c["page_size"]
        pages = [p for p in c["block_table"][seq] if p >= 0]
        return np.concatenate([arr[p * pg:(p + 1) * pg] for p in pages])
    return arr[int(c["seq_start"][seq]):]


@pytest.mark.parametrize("paged", [True, False])
def test_cache_append_writes_where_the_layout_says(paged):
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=100, ctx_hi=300, n_seqs=3, paged=paged,
                                                h_idx=2, d_idx=16, n_heads=2, d_c=8, d_r=8)
    inp = I.generate(cfg, threads=1)
    ctx = I.context_lengths(cfg)
    rng = np.random.default_rng(11)
    tok_seq = np.array([0, 2, 1, 2, 0, 1], dtype=np.int32)
    tok_pos = np.array([0, int(ctx[2]) - 1, 65, 64, 63, int(ctx[1]) - 2], dtype=np.int32)
    k_new = rng.standard_normal((6, 16)).astype(np.float32)
    lat_new = rng.integers(0, 2 ** 15, (6, 16)).astype(np.uint16)
    ki, ks, lat, bad = R.cache_append(inp, 3, tok_seq, tok_pos, k_new, lat_new)
    assert bad == set()
    codes, s = I.to_e4m3_rows(k_new)
    written = set()
    for n in range(6):
        b, p = int(tok_seq[n]), int(tok_pos[n])
        assert np.array_equal(_logical_view(inp, b, ki)[p], codes[n])
        assert _logical_view(inp, b, ks)[p] == s[n]
        assert np.array_equal(_logical_view(inp, b, lat)[p], lat_new[n])
        written.add((b, p))
    # every other row is untouched
    changed = np.nonzero((ki != inp["k_idx"]).any(1) | (lat != inp["latent"]).any(1))[0]
    assert len(changed) <= 6
    for b in range(3):
        v0, v1 = _logical_view(inp, b, inp["latent"]), _logical_view(inp, b, lat)
        for p in range(int(ctx[b])):
            if (b, p) not in written:
                assert np.array_equal(v0[p], v1[p])


def test_cache_append_rejects_out_of_range_and_non_finite():
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=100, ctx_hi=130, n_seqs=2,
                                                h_idx=2, d_idx=16, n_heads=2, d_c=8, d_r=8)
    inp = I.generate(cfg, threads=1)
    bt = inp["cache"]["block_table"]
    bt[1, 1] = inp["cache"]["num_pages"]            # a page id past the pool
    width = bt.shape[1] * 64
    k_new = np.ones((8, 16), np.float32)
    k_new[5, 3] = np.inf
    lat_new = np.ones((8, 16), np.uint16)
    # token:   0 ok, 1 seq<0, 2 seq>=2, 3 pos<0, 4 past the table, 5 inf key,
    #          6 ok, 7 bad page id
    tok_seq = [0, -1, 2, 1, 1, 1, 0, 1]
    tok_pos = [3, 0, 0, -5, width, 7, 9, 70]
    ki, ks, lat, bad = R.cache_append(inp, 2, tok_seq, tok_pos, k_new, lat_new)
    assert bad == {1, 2, 3, 4, 5, 7}
    changed = np.nonzero((ki != inp["k_idx"]).any(1) | (lat != inp["latent"]).any(1))[0]
    assert sorted(changed) == sorted([bt[0, 0] * 64 + 3, bt[0, 0] * 64 + 9])


# --------------------------------------------------------------------------
# P10: the output projection (W_UV per head, then W_out)
# --------------------------------------------------------------------------

def test_output_projection_brute_force():
    """Scalar loops over the definition: u[i][v] = sum_c W_UV[i][v][c] o[i][c],
    y[m] = sum_i sum_v W_out[m][i*d_v + v] u[i][v]."""
    rng = np.random.default_rng(20)
    H, d_c, d_v, d_model = 3, 5, 4, 6
    o = rng.standard_normal((H, d_c))
    w_uv = rng.standard_normal((H, d_v, d_c))
    w_out = rng.standard_normal((d_model, H * d_v))
    u_ref = [[sum(w_uv[i][v][c] * o[i][c] for c in range(d_c)) for v in range(d_v)] for i in range(H)]
    y_ref = [sum(w_out[m][i * d_v + v] * u_ref[i][v] for i in range(H) for v in range(d_v))
             for m in range(d_model)]
    u, y = R.output_projection_row(o, w_uv, w_out)
    np.testing.assert_allclose(u, np.array(u_ref), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(y, np.array(y_ref), rtol=1e-13, atol=1e-13)


def test_output_projection_completes_the_pages_module():
    """The page's module: values uncompressed per selected row by one linear
    layer (H*d_v outputs, viewed as [H, d_v]), weighted by the softmax, heads
    concatenated in order, then the output linear layer; written with torch
    library routines.  The oracle's path (sparse MLA latent output, then the
    projection) must give the same y."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(21)
    H, d_c, d_r, d_v, d_model, n = 4, 12, 6, 5, 7, 9
    q = rng.standard_normal((H, d_c + d_r)) * 0.3
    kv = rng.standard_normal((n, d_c + d_r))
    w_uv = rng.standard_normal((H, d_v, d_c))
    w_out = rng.standard_normal((d_model, H * d_v))
    sm = 1 / math.sqrt(d_c + d_r)
    o, _ = R.sparse_mla_row(q, kv, d_c, sm)
    _, y = R.output_projection_row(o, w_uv, w_out)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    c = t(kv[:, :d_c])
    p = torch.softmax(t(q) @ t(kv).T * sm, dim=-1)                   # [H, n]
    v = F.linear(c, t(w_uv.reshape(H * d_v, d_c))).view(n, H, d_v)    # per selected row
    attn = torch.einsum("is,siv->iv", p, v).reshape(H * d_v)
    y_page = F.linear(attn, t(w_out)).numpy()
    np.testing.assert_allclose(y, y_page, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# P11: indexer warm-up loss (KL to the dense attention) and its backward
# --------------------------------------------------------------------------

def _warmup_case(seed=22, H=3, D=10, H_I=4, d_I=6, n=9):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((H, D)), rng.standard_normal((n, D)), rng.standard_normal((H_I, d_I)),
            rng.standard_normal(H_I), rng.standard_normal((n, d_I)))


def test_teacher_is_the_head_mean_of_the_dense_attention():
    # every head's probabilities sum to 1 over the keys, so the normaliser of
    # the page's teacher is H: p is the mean over heads
    q, kv, _, _, _ = _warmup_case()
    a = R.dense_attention_probs(q, kv, 0.3)
    np.testing.assert_allclose(a.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    p = R.teacher_distribution(a)
    np.testing.assert_allclose(p, a.mean(axis=0), rtol=1e-14)
    np.testing.assert_allclose(p.sum(), 1.0, rtol=0, atol=1e-14)
    # the dense probabilities equal scipy's softmax of the same logits
    np.testing.assert_allclose(a, scipy.special.softmax(0.3 * q @ kv.T, axis=1), rtol=1e-13)


def test_kl_matches_scipy_and_vanishes_at_the_teacher():
    rng = np.random.default_rng(23)
    p = rng.random(12)
    p[3] = 0.0                                   # a key with no teacher mass
    p /= p.sum()
    scores = rng.standard_normal(12) * 2
    kl, _ = R.indexer_kl_row(p, scores)
    ref = scipy.stats.entropy(p, scipy.special.softmax(scores))
    assert abs(kl - ref) <= 1e-13 * max(1.0, ref) and kl > 0
    pp = p + 1e-3
    pp /= pp.sum()
    kl0, g0 = R.indexer_kl_row(pp, np.log(pp) + 7.5)      # softmax(log p + c) = p
    assert abs(kl0) < 1e-14 and np.abs(g0).max() < 1e-14


def test_kl_gradient_against_finite_differences_and_autograd():
    import torch
    rng = np.random.default_rng(24)
    p = rng.random(7)
    p /= p.sum()
    scores = rng.standard_normal(7)
    _, g = R.indexer_kl_row(p, scores)
    h = 1e-6
    fd = np.array([(R.indexer_kl_row(p, scores + h * e)[0] - R.indexer_kl_row(p, scores - h * e)[0]) / (2 * h)
                   for e in np.eye(7)])
    np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-9)
    s = torch.tensor(scores, requires_grad=True)
    torch.nn.functional.kl_div(torch.log_softmax(s, 0), torch.tensor(p), reduction="sum").backward()
    np.testing.assert_allclose(g, s.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_indexer_backward_against_autograd():
    """The warm-up chain for two rows, differentiated by torch autograd: teacher
    from the dense attention, scores from the indexer definition, KL summed over
    rows; the oracle's composed gradients must match for q_I, w and k_I."""
    import torch
    rng = np.random.default_rng(25)
    H, D, H_I, d_I, n, T = 3, 10, 4, 6, 9, 2
    qm = rng.standard_normal((T, H, D))
    kv = rng.standard_normal((n, D))
    qi = rng.standard_normal((T, H_I, d_I))
    w = rng.standard_normal((T, H_I))
    k = rng.standard_normal((n, d_I))
    klen = [6, 9]                                 # causal: row t sees its first klen keys
    dq_o, dw_o, dk_o, loss_o = np.zeros_like(qi), np.zeros_like(w), np.zeros_like(k), 0.0
    for t in range(T):
        p = R.teacher_distribution(R.dense_attention_probs(qm[t], kv[:klen[t]], 0.25))
        sc = R.indexer_row(qi[t], w[t], k[:klen[t]])
        kl, g = R.indexer_kl_row(p, sc)
        dq, dw, dk = R.indexer_backward_row(qi[t], w[t], k[:klen[t]], g)
        dq_o[t], dw_o[t] = dq, dw
        dk_o[:klen[t]] += dk
        loss_o += kl
    tq, tw, tk = (torch.tensor(x, requires_grad=True) for x in (qi, w, k))
    loss = 0
    for t in range(T):
        a = torch.softmax(0.25 * torch.tensor(qm[t]) @ torch.tensor(kv[:klen[t]]).T, dim=1)
        p = a.sum(0) / a.sum()
        sc = torch.relu(tk[:klen[t]] @ tq[t].T) @ tw[t]
        loss = loss + torch.nn.functional.kl_div(torch.log_softmax(sc, 0), p, reduction="sum")
    loss.backward()
    assert abs(loss.item() - loss_o) <= 1e-12 * abs(loss_o)
    np.testing.assert_allclose(dq_o, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw_o, tw.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk_o, tk.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_mask_argument_is_the_relu_decision():
    # passing the ReLU decision explicitly changes nothing when it is the one
    # the float64 dot products give; for FP8 operands the exact decision (the
    # sign of the codes' dot product, scales being positive) agrees with them
    # except where the float64 dot product is within rounding of zero
    rng = np.random.default_rng(26)
    q, w, k = rng.standard_normal((4, 6)), rng.standard_normal(4), rng.standard_normal((9, 6))
    g = rng.standard_normal(9)
    a = R.indexer_backward_row(q, w, k, g)
    b = R.indexer_backward_row(q, w, k, g, on=(k @ q.T) > 0)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    codes_q = rng.integers(0, 256, (64, 128)).astype(np.uint8)
    codes_k = rng.integers(0, 256, (50, 128)).astype(np.uint8)
    codes_q[(codes_q & 0x7F) == 0x7F] = 0                       # no NaN codes
    codes_k[(codes_k & 0x7F) == 0x7F] = 0
    qs, ks = rng.random(64) + 0.5, rng.random(50) + 0.5
    qc, kc = R.e4m3_decode(codes_q), R.e4m3_decode(codes_k)
    exact = (kc @ qc.T) > 0
    d = (kc * ks[:, None]) @ (qc * qs[:, None]).T
    near = np.abs(d) <= 1e-12 * (np.abs(kc * ks[:, None]) @ np.abs(qc * qs[:, None]).T)
    assert np.array_equal(exact[~near], (d > 0)[~near])
