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
