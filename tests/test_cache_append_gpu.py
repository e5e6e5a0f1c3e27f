"""GPU parity of the fused FP8 quantise + cache append (dsa_cache_append).

Every byte of the three caches after the call is compared with the oracle's
cache_append run on the same starting caches: the e4m3 codes and fp32 scales
bit for bit (the codes are an integer decision that both sides take in fp32:
fl32(amax / 448), fl32(k / s), one round to nearest even), the latent rows as
bit copies, and every row that is not a destination unchanged.
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from oracle import dsa_ref as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def _num_seqs(inp):
    c = inp["cache"]
    return int(c["block_table"].shape[0] if c["block_table"] is not None else len(c["seq_start"]))


def _special_keys(n, d, rng):
    """Random keys over 70 binades, plus rows that reach every corner of the
    rule: all zero, a scale that underflows to 0, and rows with amax = 448
    (so s = 1 and k / s = k) that hold every rounding tie, signed zeros and
    subnormal codes."""
    k = (rng.standard_normal((n, d)) * np.exp(rng.uniform(-30, 10, (n, 1)))).astype(np.float32)
    vals = np.unique(np.abs(R.e4m3_decode(np.arange(0x7F, dtype=np.uint8))))
    mids = (vals[1:] + vals[:-1]) / 2
    k[0] = 0.0
    k[1] = 0.0
    k[1, d // 2] = 1e-42                                  # s = fl32(1e-42 / 448) = 0 -> 1
    row = np.resize(np.concatenate([mids, -mids]), d).astype(np.float32)
    row[0], row[-1] = 448.0, -1e-4                        # amax 448; -1e-4 -> 0x80
    k[2] = row
    k[3] = -row[::-1]
    k[4] = rng.uniform(2.0 ** -11, 2.0 ** -6, d).astype(np.float32) * rng.choice([-1, 1], d)
    k[4, 1] = 448.0                                       # subnormal codes
    k[5] = rng.uniform(-1, 1, d).astype(np.float32)
    k[5, 7] = -3.0e38                                     # near the fp32 maximum
    return k


def _latent_rows(inp, n, rng):
    w = inp["latent"].shape[1]
    if inp["mla_dtype"] == "bf16":
        return rng.integers(0, 2 ** 16, (n, w)).astype(np.uint16)
    return rng.standard_normal((n, w)).astype(np.float32)


def _run(N, inp, tok_seq, tok_pos, k_new, lat_new):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload, to_device
    wl = DeviceWorkload(inp)
    dev = wl.device
    wl.append(to_device(np.asarray(tok_seq, np.int32), dev), to_device(np.asarray(tok_pos, np.int32), dev),
              to_device(np.asarray(k_new, np.float32), dev), to_device(lat_new, dev))
    torch.cuda.synchronize()
    st = wl.status(N.DSA_OP_CACHE_APPEND)
    ran = wl.kernels_ran(N.DSA_OP_CACHE_APPEND)
    return wl.caches_to_host(), st, ran


def _compare(got, want):
    (gk, gs, gl), (wk, ws, wl_) = got, want
    assert np.array_equal(gk.view(np.uint8) if gk.dtype == np.uint8 else gk.view(np.uint32),
                          wk.view(np.uint8) if wk.dtype == np.uint8 else wk.view(np.uint32))
    if ws is not None:
        assert np.array_equal(gs.view(np.uint32), ws.view(np.uint32))
    assert np.array_equal(gl.view(np.uint16 if gl.dtype == np.uint16 else np.uint32),
                          wl_.view(np.uint16 if wl_.dtype == np.uint16 else np.uint32))


def _scattered_tokens(inp, cfg, n, rng):
    """n distinct (seq, pos) pairs inside the sequences' pages, the last
    position of every sequence among them.  Each position stays inside its own
    sequence's rows: the generator gives every sequence a page-rounded region
    (contiguous layout: seq_start[b] is a multiple of 64 and the region holds
    ceil(ctx/64)*64 rows), and positions are drawn below that size."""
    ctx = I.context_lengths(cfg)
    pages = -(-ctx // I.BLOCK) * I.BLOCK
    pairs = {(b, int(ctx[b]) - 1) for b in range(len(ctx))}
    while len(pairs) < n:
        b = int(rng.integers(0, len(ctx)))
        pairs.add((b, int(rng.integers(0, pages[b]))))
    pairs = list(pairs)
    rng.shuffle(pairs)
    return np.array([p[0] for p in pairs], np.int32), np.array([p[1] for p in pairs], np.int32)


CASES = {
    # d_I 128 / latent 576 bf16, paged (the production layout)
    "paged_d128": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=200, ctx_hi=900, n_seqs=5),
    # contiguous layout
    "contig_d128": I.CONFIGS["decode_16k"].replace(ctx_lo=100, ctx_hi=700, n_seqs=4),
    # d_I 512 (four key chunks per lane), latent 1088 bf16 (a second latent group)
    "paged_d512_wide": I.CONFIGS["decode_128k_paged"].replace(
        ctx_lo=100, ctx_hi=300, n_seqs=3, d_idx=512, d_c=1024, h_idx=4, n_heads=2),
    # d_I 36 (a ragged key row), fp32 caches: copies, no scale
    "contig_f32": I.CONFIGS["tiny_fp32"].replace(d_idx=36),
}


@pytest.mark.parametrize("name", list(CASES))
def test_append_matches_oracle(N, name):
    cfg = CASES[name]
    rng = np.random.default_rng(list(CASES).index(name) + 100)
    inp = I.generate(cfg, with_q=False, threads=4)
    n = 197
    tok_seq, tok_pos = _scattered_tokens(inp, cfg, n, rng)
    k_new = _special_keys(n, cfg.d_idx, rng)
    lat_new = _latent_rows(inp, n, rng)
    got, st, ran = _run(N, inp, tok_seq, tok_pos, k_new, lat_new)
    assert st == (0, -1) and ran & N.DSA_KERNEL_CACHE_APPEND
    ki, ks, lat, bad = R.cache_append(inp, _num_seqs(inp), tok_seq, tok_pos, k_new, lat_new)
    assert bad == set()
    _compare(got, (ki, ks, lat))


def test_append_empty_is_a_no_op(N):
    cfg = CASES["paged_d128"]
    inp = I.generate(cfg, with_q=False, threads=4)
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    wl = DeviceWorkload(inp)
    e = torch.empty(0, dtype=torch.int32, device=wl.device)
    wl.append(e, e, torch.empty((0, cfg.d_idx), device=wl.device),
              torch.empty((0, cfg.d_qk), dtype=torch.bfloat16, device=wl.device))
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_CACHE_APPEND) == (0, -1)
    assert wl.kernels_ran(N.DSA_OP_CACHE_APPEND) == 0
    _compare(wl.caches_to_host(), (inp["k_idx"], inp["k_scale"], inp["latent"]))


@pytest.mark.parametrize("kind", ["seq_neg", "seq_big", "pos_neg", "past_table", "bad_page",
                                  "past_contig", "inf", "nan"])
def test_append_rejects_one_bad_token(N, kind):
    """One bad token among good ones: it is not written, the status word names
    it, and every other token is written as the oracle writes it."""
    contig = kind == "past_contig"
    cfg = (CASES["contig_d128"] if contig else CASES["paged_d128"])
    inp = I.generate(cfg, with_q=False, threads=4)
    rng = np.random.default_rng(5)
    n, bad_n = 40, 17
    tok_seq, tok_pos = _scattered_tokens(inp, cfg, n, rng)
    k_new = _special_keys(n, cfg.d_idx, rng)
    lat_new = _latent_rows(inp, n, rng)
    code = N.DSA_ERR_OUT_OF_RANGE
    if kind == "seq_neg":
        tok_seq[bad_n] = -1
    elif kind == "seq_big":
        tok_seq[bad_n] = _num_seqs(inp)
    elif kind == "pos_neg":
        tok_pos[bad_n] = -3
    elif kind == "past_table":
        tok_pos[bad_n] = inp["cache"]["block_table"].shape[1] * I.BLOCK
    elif kind == "bad_page":
        b = int(tok_seq[bad_n])
        inp["cache"]["block_table"][b, int(tok_pos[bad_n]) // I.BLOCK] = inp["cache"]["num_pages"]
        # no other token may use that page entry
        same = (tok_seq == b) & (tok_pos // I.BLOCK == tok_pos[bad_n] // I.BLOCK)
        keep = ~same
        keep[bad_n] = True
        tok_seq, tok_pos, k_new, lat_new = tok_seq[keep], tok_pos[keep], k_new[keep], lat_new[keep]
        bad_n = int(np.nonzero(np.nonzero(keep)[0] == bad_n)[0][0])
    elif kind == "past_contig":
        tok_seq[bad_n] = len(inp["cache"]["seq_start"]) - 1
        tok_pos[bad_n] = inp["latent"].shape[0]
    else:
        k_new[bad_n, 3] = np.inf if kind == "inf" else np.nan
        code = N.DSA_ERR_INVALID_ARG
    got, st, ran = _run(N, inp, tok_seq, tok_pos, k_new, lat_new)
    assert st == (code, bad_n)
    ki, ks, lat, bad = R.cache_append(inp, _num_seqs(inp), tok_seq, tok_pos, k_new, lat_new)
    assert bad == {bad_n}
    _compare(got, (ki, ks, lat))


@pytest.mark.parametrize("name", ["decode_128k_paged", "prefill_64k"])
def test_append_full_size(N, name):
    """The workloads' own new tokens at full size: a decode step's 32 tokens
    into the 128K paged caches, and all 65,536 tokens of the 64K prefill into
    zeroed caches.  The result must equal the oracle's quantisation of the same
    fp32 keys (which is also what the input generator stored)."""
    cfg = I.CONFIGS[name]
    inp = I.generate(cfg, with_q=False, rows=[])       # the caches only
    tok_seq, tok_pos = I.new_tokens(cfg)
    k_new, lat_new = I.token_keys(cfg, tok_seq, tok_pos)
    start = dict(inp)
    if cfg.prefill:
        start["k_idx"] = np.zeros_like(inp["k_idx"])
        start["k_scale"] = np.zeros_like(inp["k_scale"])
        start["latent"] = np.zeros_like(inp["latent"])
    got, st, ran = _run(N, start, tok_seq, tok_pos, k_new, lat_new)
    assert st == (0, -1)
    rows = np.array([R.physical_rows(int(b), np.array([int(p)]), inp["cache"])[0]
                     for b, p in zip(tok_seq, tok_pos)])
    codes, s = R.quantise_keys(k_new)
    gk, gs, gl = got
    assert np.array_equal(gk[rows], codes)
    assert np.array_equal(gs[rows].view(np.uint32), s.view(np.uint32))
    assert np.array_equal(gl[rows], lat_new)
    # and the caches as a whole: the generator's caches, bit for bit
    _compare(got, (inp["k_idx"], inp["k_scale"], inp["latent"]))
