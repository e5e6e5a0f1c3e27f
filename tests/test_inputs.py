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
