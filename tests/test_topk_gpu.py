"""dsa_topk on fp32 score rows given directly, against the oracle's selection.

The scores are exact fp32 values, so the selection is compared bit for bit:
the k largest, ties to the lower position, ascending, -1 padded.  The rows
cover the regimes of the kernel: one CTA or a cluster of 2-8 CTAs per row,
segments longer than the shared-memory cache (rows past 8 * 16384 keys),
short rows (klen <= k), and score distributions that stress the radix digits:
massive ties, one crowded histogram bin, signed zeros, infinities, all
negative values.
"""
import ctypes

import numpy as np
import pytest

from oracle import dsa_ref as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def _rows(kind, lengths, seed):
    rng = np.random.default_rng(seed)
    out = []
    for n in lengths:
        if kind == "normal":
            s = rng.standard_normal(n)
        elif kind == "all_equal":
            s = np.full(n, 1.5)
        elif kind == "few_values":
            s = rng.choice(np.array([-1.0, 0.0, 0.5, 2.0]), size=n, p=[0.4, 0.3, 0.25, 0.05])
        elif kind == "signed_zero":
            s = rng.choice(np.array([-0.0, 0.0, -1e-30, 1e-30, -3.0]), size=n)
        elif kind == "crowded_bin":
            # every score inside one 12-bit key bin: [1, 1 + 2^-4) shares sign,
            # exponent and the top three mantissa bits
            s = 1.0 + rng.random(n) * 0.0624
        elif kind == "infinities":
            s = rng.standard_normal(n)
            s[rng.random(n) < 0.01] = np.inf
            s[rng.random(n) < 0.01] = -np.inf
        elif kind == "negative":
            s = -np.abs(rng.standard_normal(n)) - 1.0
        elif kind == "planted":
            s = rng.standard_normal(n) * 0.1
            hot = rng.choice(n, size=min(n, 3000), replace=False)
            s[hot] += 5.0 + rng.random(hot.shape[0])
        else:
            raise ValueError(kind)
        out.append(s.astype(np.float32))
    return out


def _run(N, rows_np, k):
    import torch
    T = len(rows_np)
    max_klen = max(max(r.shape[0] for r in rows_np), 1)
    ld = (max_klen + 127) // 128 * 128
    host = np.full((T, ld), np.nan, dtype=np.float32)   # past klen: never read
    for t, r in enumerate(rows_np):
        host[t, : r.shape[0]] = r
    dev = torch.device("cuda")
    scores = torch.from_numpy(host).to(dev)
    klen = torch.tensor([r.shape[0] for r in rows_np], dtype=torch.int32, device=dev)
    seq = torch.zeros(T, dtype=torch.int32, device=dev)
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    dims = N.dsa_dims(n_idx_heads=64, d_idx=128, n_heads=128, d_c=512, d_r=64, topk=k,
                      idx_dtype=N.DSA_FP8_E4M3, mla_dtype=N.DSA_BF16, sm_scale=0.1,
                      algo=N.DSA_ALGO_AUTO)
    vp = lambda x: ctypes.c_void_p(x.data_ptr())
    rows = N.dsa_rows(num_rows=T, row_seq=vp(seq), row_klen=vp(klen), max_klen=max_klen, q_group=1)
    nws = N.dsa_workspace_size(dims, rows, N.DSA_OP_TOPK)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    N.dsa_workspace_init(vp(ws), nws, stream)
    N.dsa_topk(dims, rows, vp(scores), ld, vp(idx), vp(ws), nws, stream)
    torch.cuda.synchronize()
    assert N.dsa_read_device_status(vp(ws), stream) == (0, -1)
    return idx.cpu().numpy()


LENGTHS = [1, 2047, 2048, 2049, 5000, 16384, 16385, 40000, 131072]
KINDS = ["normal", "all_equal", "few_values", "signed_zero", "crowded_bin", "infinities",
         "negative", "planted"]


@pytest.mark.parametrize("kind", KINDS)
def test_topk_matches_oracle(N, kind):
    rows = _rows(kind, LENGTHS, seed=KINDS.index(kind))
    got = _run(N, rows, 2048)
    for t, r in enumerate(rows):
        want = R.topk_row(r.astype(np.float64), 2048)
        assert np.array_equal(got[t], want), (kind, r.shape[0],
                                              np.flatnonzero(got[t] != want)[:5])


@pytest.mark.parametrize("k", [1, 7, 100, 1000])
def test_topk_small_k(N, k):
    rows = _rows("normal", [1, 50, 999, 1000, 1001, 20000, 70000], seed=k)
    got = _run(N, rows, k)
    for t, r in enumerate(rows):
        assert np.array_equal(got[t], R.topk_row(r.astype(np.float64), k)), (k, r.shape[0])


@pytest.mark.parametrize("kind", ["normal", "few_values", "crowded_bin"])
def test_topk_rows_beyond_the_cluster_cache(N, kind):
    # 8 CTAs x 16384 cached keys: longer rows read the rest of their segment
    # from global memory
    rows = _rows(kind, [131073, 200003, 262144], seed=11)
    got = _run(N, rows, 2048)
    for t, r in enumerate(rows):
        assert np.array_equal(got[t], R.topk_row(r.astype(np.float64), 2048)), (kind, r.shape[0])


@pytest.mark.parametrize("k", [2048, 64])
def test_topk_many_rows(N, k):
    """A batch of hundreds of rows, some past one CTA's cache, runs one CTA
    per row streaming the scores (the cluster kernel above runs the few-row
    batches and batches of short rows): every kind of row,
    lengths around k and well past it, and bins far over the threshold-bin
    capacity (all_equal, crowded_bin), each against the oracle."""
    lengths = [1, k - 1, k, k + 1, 3000, 4097, 6000, 9000, 20000, 40000]
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows = []
    i = 0
    while len(rows) < 2 * sms + 8:
        kind = KINDS[i % len(KINDS)]
        rows += _rows(kind, [lengths[(i + j) % len(lengths)] for j in range(2)], seed=100 + i)
        i += 1
    got = _run(N, rows, k)
    for t, r in enumerate(rows):
        want = R.topk_row(r.astype(np.float64), k)
        assert np.array_equal(got[t], want), (t, r.shape[0], np.flatnonzero(got[t] != want)[:5])
