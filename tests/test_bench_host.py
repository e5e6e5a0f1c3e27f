"""Host-side arithmetic of bench.py: the algorithmic bytes and FLOPs that the
roofline fractions divide by, against the per-unit figures stated for each
kernel (CPU only)."""
import numpy as np

import bench
from long_context_sparse_04_b200 import inputs as I


def test_cache_append_bytes_per_token():
    cfg = I.CONFIGS["prefill_64k"]
    # read: fp32 key 512 + bf16 latent 1152 + (seq, pos) 8 + one map entry 4;
    # written: 128 codes + 4 scale + 1152 latent
    assert bench.append_bytes_per_token(cfg) == 512 + 1152 + 8 + 4 + 128 + 4 + 1152 == 2960
    f32 = I.CONFIGS["tiny_fp32"]
    assert bench.append_bytes_per_token(f32) == 4 * 32 + 80 * 4 + 12 + 4 * 32 + 80 * 4


def test_output_projection_flops_and_bytes():
    cfg = I.CONFIGS["decode_128k_paged"]
    flops, by = bench.proj_algorithmic(cfg, 32)
    assert flops == 2 * 32 * 128 * 128 * (512 + 7168)
    weights = 2 * (128 * 128 * 512 + 7168 * 128 * 128)
    assert by == weights + 2 * 32 * (128 * 512 + 2 * 128 * 128 + 7168) == 258_408_448
    f64k, _ = bench.proj_algorithmic(I.CONFIGS["prefill_64k"], 65536)
    assert f64k == 16_492_674_416_640


def test_path_stage_units():
    cfg = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=300, ctx_hi=700, n_seqs=3)
    inp = I.generate(cfg, with_q=False, threads=2)
    klen = inp["row_klen"].astype(np.int64)
    ctx = I.context_lengths(cfg)
    idx = bench.algorithmic(cfg, inp, "indexer")
    # each sequence's keys once (132 B: e4m3 row + scale) for both of its rows
    assert idx["bytes"] == int(ctx.sum()) * 132
    assert idx["flops"] == 2 * 64 * 128 * int(klen.sum())
    tk = bench.algorithmic(cfg, inp, "topk")
    assert tk["bytes"] == 4 * int(klen.sum()) + 4 * 2048 * len(klen)
    mla = bench.algorithmic(cfg, inp, "mla")
    sel = np.minimum(klen, 2048)
    assert mla["bytes"] == int(sel.sum()) * 1152 + len(klen) * 128 * (576 + 512) * 2
    assert mla["flops"] == int(sel.sum()) * 2 * 128 * (576 + 512)


def test_warmup_flops():
    cfg = I.CONFIGS["decode_16k"].replace(ctx_lo=300, ctx_hi=700, n_seqs=3)
    inp = I.generate(cfg, with_q=False, threads=2)
    fl = bench.warmup_flops(inp)
    pairs = int(inp["row_klen"].astype(np.int64).sum())
    # the 64 x 128 dot products twice (dq/dw, dk) and the dq and dk contractions
    assert fl == {"fp32": 4 * 2 * 64 * 128 * pairs, "pairs": pairs}


def test_path_launches():
    import types
    n = types.SimpleNamespace(DSA_KERNEL_MLA_COMBINE=0x20)
    # decode: indexer, top-k, attention (the split merge runs inside the attention kernel)
    assert bench.path_launches(n, 0x20 | 0x10, 32, prefill=False) == 3
    # prefill: the three kernels per 512-row chunk
    assert bench.path_launches(n, 0, 65536, prefill=True) == 3 * 128
    assert bench.path_launches(n, 0, 513, prefill=True) == 6
