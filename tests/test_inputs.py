"""The seeded input generator: a subset of query rows is bit-identical to the
same rows of the whole workload (the full-size parity tests rely on it)."""
import numpy as np

from long_context_sparse_04_b200 import inputs as I


def test_row_subset_matches_whole_workload():
    cfg = I.CONFIGS["prefill_8k"].replace(seq_len=700)
    whole = I.generate(cfg)
    rows = [0, 3, 255, 256, 699]
    sub = I.generate(cfg, rows=rows)
    for key in ("row_seq", "row_klen", "q_idx", "q_scale", "w", "q"):
        assert np.array_equal(sub[key], whole[key][rows]), key
    for key in ("k_idx", "k_scale", "latent"):
        assert np.array_equal(sub[key], whole[key]), key


def test_row_subset_paged_decode():
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=3000, ctx_hi=5000, n_seqs=3)
    whole = I.generate(cfg)
    rows = [1, 4]
    sub = I.generate(cfg, rows=rows)
    for key in ("row_seq", "row_klen", "q_idx", "q_scale", "w", "q"):
        assert np.array_equal(sub[key], whole[key][rows]), key
    assert np.array_equal(sub["cache"]["block_table"], whole["cache"]["block_table"])


def test_new_tokens_are_each_sequences_last_positions():
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=3000, ctx_hi=5000, n_seqs=3)
    ctx = I.context_lengths(cfg)
    seq, pos = I.new_tokens(cfg)
    assert list(seq) == [0, 0, 1, 1, 2, 2]
    assert list(pos) == [int(c) - 2 + j for c in ctx for j in (0, 1)]
    pre = I.CONFIGS["prefill_8k"].replace(seq_len=300)
    seq, pos = I.new_tokens(pre)
    assert (seq == 0).all() and list(pos) == list(range(300))


def test_token_keys_are_the_stored_keys_before_the_casts():
    # the stored caches are the storage casts of exactly these fp32 values, so a
    # cache append of them rewrites the caches with the same bytes
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=1100, ctx_hi=2500, n_seqs=2)
    inp = I.generate(cfg, with_q=False, rows=[])
    seq, pos = I.new_tokens(cfg)
    k, lat = I.token_keys(cfg, seq, pos)
    bt = inp["cache"]["block_table"]
    rows = [int(bt[b, p // I.BLOCK]) * I.BLOCK + p % I.BLOCK for b, p in zip(seq, pos)]
    codes, scale = I.to_e4m3_rows(k)
    assert np.array_equal(codes, inp["k_idx"][rows]) and np.array_equal(scale, inp["k_scale"][rows])
    assert np.array_equal(lat, inp["latent"][rows])


def test_projection_inputs_are_seeded_per_row():
    cfg = I.CONFIGS["decode_16k"].replace(n_heads=4, d_c=64, d_v=32, d_model=96)
    a = I.latent_out_rows(cfg, range(6))
    assert np.array_equal(I.latent_out_rows(cfg, [3, 5]), a[[3, 5]])
    w1, o1 = I.out_proj_weights(cfg)
    w2, o2 = I.out_proj_weights(cfg)
    assert np.array_equal(w1, w2) and np.array_equal(o1, o2)
    assert w1.shape == (4, 32, 64) and o1.shape == (96, 128)
    w3, _ = I.out_proj_weights(cfg.replace(seed=cfg.seed + 1))
    assert not np.array_equal(w1, w3)
