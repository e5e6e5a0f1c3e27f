"""The fused indexer -> top-k of dsa_decode_step (and dsa_forward) with
q_group <= 2: the indexer's epilogue builds each row's histogram of its
scores' top 12 key bits, and top-k starts from it instead of its own first
pass ("DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 1:
The Lightning Indexer", item "Separable Streaming Top-k").

Checks, through the C ABI:
  - the selection is the oracle's rule on the GPU's own scores, bit for bit,
    and within the tie band of the oracle's own selection (tests/parity.py);
  - it equals the staged path (standalone top-k) bit for bit, scores and
    attention outputs included;
  - repeated calls on one workspace agree (every top-k leaves the row
    histograms zeroed for the next call);
  - rows that tie massively (all-zero head weights: every score is +0) and
    rows of non-positive scores (negative head weights: many zeros) select
    the lowest positions among equals;
  - a CTA whose key range spans more groups than it keeps histograms for
    adds the rest to the global histograms directly.
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "decode_small": I.CONFIGS["decode_16k"].replace(ctx_lo=2100, ctx_hi=5000, n_seqs=6),
    "decode_short_rows": I.CONFIGS["decode_16k"].replace(ctx_lo=1, ctx_hi=2600, n_seqs=8),
    "paged_small": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=2040, ctx_hi=6000, n_seqs=4),
    # rows longer than one CTA's shared-memory segment: 2-4 CTA clusters
    "decode_cluster": I.CONFIGS["decode_16k"].replace(ctx_lo=17000, ctx_hi=40000, n_seqs=3),
    "paged_cluster": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=30000, ctx_hi=70000, n_seqs=2),
    # 600 sequences of 2-5 key tiles: each indexer CTA spans more groups than
    # its shared-memory histograms cover; k = 64 so these rows still select
    "many_groups_k64": I.CONFIGS["decode_16k"].replace(ctx_lo=200, ctx_hi=520, n_seqs=600,
                                                         topk=64),
}


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


_cache = {}


def _inputs(name):
    if name not in _cache:
        _cache[name] = I.generate(CASES[name])
    return _cache[name]


def _decode(N, inp, algo, reps=1):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    wl = DeviceWorkload(inp, algo=algo)
    res = []
    for _ in range(reps):
        out, lse, sc, idx = wl.decode_step(debug=True)
        torch.cuda.synchronize()
        res.append(tuple(P.to_np(x) for x in (sc, idx, out, lse)))
    assert wl.status(N.DSA_OP_DECODE_STEP) == (0, -1)
    ran = wl.kernels_ran(N.DSA_OP_DECODE_STEP)
    assert ran & N.DSA_KERNEL_INDEXER_TC and ran & N.DSA_KERNEL_TOPK and ran & N.DSA_KERNEL_MLA_TC, hex(ran)
    return res


def _rows(T):
    return range(T) if T <= 64 else sorted(set(np.linspace(0, T - 1, 40).astype(int)) | {T - 1})


@pytest.mark.parametrize("name", list(CASES))
def test_fused_selection_matches_oracle(N, name):
    inp = _inputs(name)
    (sc, idx, out, lse), = _decode(N, inp, N.DSA_ALGO_AUTO)
    P.check_rows(inp, _rows(len(inp["row_klen"])), sc, idx, out, lse)


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_staged(N, name):
    inp = _inputs(name)
    a = _decode(N, inp, N.DSA_ALGO_AUTO, reps=3)
    b, = _decode(N, inp, N.DSA_ALGO_STAGED)
    klen = inp["row_klen"]
    for r in a:                                   # every call, the first and the repeats
        for t in range(len(klen)):
            assert np.array_equal(r[0][t, : klen[t]], b[0][t, : klen[t]]), f"scores row {t}"
        for x, y in zip(r[1:], b[1:]):
            np.testing.assert_array_equal(x, y)


def test_fused_ties_and_signed_zeros(N):
    inp = dict(_inputs("paged_small"))
    w = inp["w"].copy()
    w[0] = 0.0                                    # every score of row 0 is +0: all tie
    w[1] = -np.abs(w[1])                          # row 1: scores <= 0, exact zeros common
    w[2, ::2] = 0.0                               # row 2: half the heads off
    inp["w"] = w
    (sc, idx, out, lse), = _decode(N, inp, N.DSA_ALGO_AUTO, reps=1)
    k = int(inp["topk"])
    for t in range(3):
        klen = int(inp["row_klen"][t])
        P.check_topk(idx[t], sc[t, :klen], _oracle_scores(inp, t), k, f"row {t}")
    # row 0: the lowest k positions
    assert np.array_equal(idx[0], np.arange(k))


def _oracle_scores(inp, t):
    from oracle import dsa_ref as R
    return R.row_scores(inp, t)


def test_workspace_reused_across_plans(N):
    """One workspace serves decode steps of different row counts with other
    ops in between, whose data lands where a later step keeps its histograms;
    every step gives the bits of a step on a freshly initialised workspace
    (the library clears a histogram region it cannot vouch for)."""
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload, _vp

    wl = DeviceWorkload(_inputs("paged_small"))
    assert wl.rows.q_group == 2
    big = max(N.dsa_workspace_size(wl.dims, wl.rows, op)
              for op in (N.DSA_OP_DECODE_STEP, N.DSA_OP_INDEXER, N.DSA_OP_SPARSE_MLA))
    shared = torch.empty(big, dtype=torch.uint8, device="cuda")
    N.dsa_workspace_init(_vp(shared), big, wl.stream)

    def rows_of(k):
        return N.dsa_rows(num_rows=k, row_seq=_vp(wl.row_seq), row_klen=_vp(wl.row_klen),
                          max_klen=wl.max_klen, q_group=2)

    def step(rows, k, ws, n):
        out = torch.full((k, wl.H, wl.d_c), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((k, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((k, wl.topk), -7, dtype=torch.int32, device="cuda")
        N.dsa_decode_step(wl.dims, rows, wl.cache, _vp(wl.q_idx), _vp(wl.q_scale), _vp(wl.w),
                          _vp(wl.q), _vp(out), _vp(lse), None, _vp(idx), _vp(ws), n, wl.stream)
        assert N.dsa_read_device_status(_vp(ws), wl.stream) == (0, -1)
        return out, lse, idx

    for k in (8, 4, 8, 2, 6):
        rows = rows_of(k)
        need = N.dsa_workspace_size(wl.dims, rows, N.DSA_OP_DECODE_STEP)
        fresh = torch.empty(need, dtype=torch.uint8, device="cuda")
        N.dsa_workspace_init(_vp(fresh), need, wl.stream)
        ref = step(rows, k, fresh, need)
        got = step(rows, k, shared, big)
        assert torch.equal(ref[2], got[2]), k
        assert torch.equal(ref[0].view(torch.int16), got[0].view(torch.int16)), k
        assert torch.equal(ref[1].view(torch.int32), got[1].view(torch.int32)), k
        # another op writes its own data over the shared workspace before the next step
        scores = torch.empty((wl.T, wl.ld), dtype=torch.float32, device="cuda")
        n_idx = N.dsa_workspace_size(wl.dims, wl.rows, N.DSA_OP_INDEXER)
        N.dsa_indexer_scores(wl.dims, wl.rows, wl.cache, _vp(wl.q_idx), _vp(wl.q_scale), _vp(wl.w),
                             _vp(scores), wl.ld, _vp(shared), n_idx, wl.stream)
        shared[256:].random_(0, 256)      # stale bytes everywhere past the status block
    torch.cuda.synchronize()
