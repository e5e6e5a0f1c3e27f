"""Parity at the full sizes of the five workloads, on sampled rows.

The decode workloads run whole through dsa_decode_step, the call bench.py
times, with the scores and indices also written out; every row is checked for
the properties that hold at any size and a sample of rows against the oracle.
The 8K and 64K prefills run whole through dsa_forward (512-row chunks), the
call bench.py times; the scores of their sampled rows come from a second,
stage-by-stage run on those rows alone (per-row results do not depend on the
batch, which the tests also check).  The 64K outputs are too large to copy out,
so their every-row properties are checked on the device.  The 64K prefill also
runs its sampled query rows alone against the full 64K-token caches.
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def _check_selection_properties(inp, idx, out, lse):
    """What holds for every row at any size: k' = min(k, klen) ascending valid
    positions then -1, finite outputs."""
    k = int(inp["topk"])
    for t, klen in enumerate(inp["row_klen"]):
        kk = min(k, int(klen))
        sel = idx[t, :kk]
        assert np.all(sel >= 0) and np.all(sel < klen), f"row {t}: index out of range"
        assert np.all(np.diff(sel) > 0), f"row {t}: not strictly ascending"
        assert np.all(idx[t, kk:] == -1), f"row {t}: padding"
        if klen <= k:
            assert np.array_equal(sel, np.arange(klen)), f"row {t}: short row takes every key"
    assert np.all(np.isfinite(out)), "non-finite output"
    assert np.all(np.isfinite(lse)), "non-finite lse"


def _decode_full(N, name, rows):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    inp = I.generate(I.CONFIGS[name])
    wl = DeviceWorkload(inp)
    out, lse, sc, idx = wl.decode_step(debug=True)
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_DECODE_STEP) == (0, -1)
    ran = wl.kernels_ran(N.DSA_OP_DECODE_STEP)
    assert ran & N.DSA_KERNEL_INDEXER_TC and ran & N.DSA_KERNEL_TOPK and ran & N.DSA_KERNEL_MLA_TC
    sc, idx, out, lse = P.to_np(sc), P.to_np(idx), P.to_np(out), P.to_np(lse)
    _check_selection_properties(inp, idx, out, lse)
    P.check_rows(inp, rows, sc, idx, out, lse)


def test_decode_128k_paged_full(N):
    # the workload bench.py times: 16 sequences x 2 rows, 96K-128K context, paged
    _decode_full(N, "decode_128k_paged", [0, 1, 14, 30, 31])


def test_decode_16k_full(N):
    _decode_full(N, "decode_16k", [0, 13, 31])


def test_prefill_8k_full(N):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    cfg = I.CONFIGS["prefill_8k"]
    sample = [0, 1, 2047, 2048, 4095, 8191]
    inp = I.generate(cfg)
    wl = DeviceWorkload(inp)
    out, lse, idx = wl.forward()
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_FORWARD) == (0, -1)
    idx, out, lse = P.to_np(idx), P.to_np(out), P.to_np(lse)
    _check_selection_properties(inp, idx, out, lse)
    del wl
    # the sampled rows alone, stage by stage: scores for the oracle comparison
    sub = I.generate(cfg, rows=sample)
    ws = DeviceWorkload(sub)
    s_sc = ws.indexer()
    s_idx = ws.topk_(s_sc)
    torch.cuda.synchronize()
    s_sc, s_idx = P.to_np(s_sc), P.to_np(s_idx)
    assert np.array_equal(s_idx, idx[sample]), "selection depends on the batch"
    P.check_rows(sub, range(len(sample)), s_sc, idx[sample], out[sample], lse[sample])


def _check_selection_properties_device(row_klen, k, idx, out, lse):
    """_check_selection_properties for workloads too large to copy out: the
    same checks on every row, as tensor reductions on the device."""
    import torch
    T = idx.shape[0]
    klen = torch.as_tensor(np.asarray(row_klen, dtype=np.int64), device=idx.device).view(T, 1)
    col = torch.arange(k, device=idx.device, dtype=torch.int64).view(1, k)
    kk = torch.clamp(klen, max=k)
    sel = col < kk
    ix = idx.to(torch.int64)
    assert bool(((ix >= 0) & (ix < klen))[sel].all()), "index out of range"
    asc = ix[:, 1:] > ix[:, :-1]
    assert bool(asc[sel[:, 1:]].all()), "not strictly ascending"
    assert bool((ix[~sel] == -1).all()), "padding"
    short = (klen <= k).view(T, 1) & sel
    assert bool((ix == col)[short].all()), "short row takes every key"
    assert bool(torch.isfinite(out).all()), "non-finite output"
    assert bool(torch.isfinite(lse).all()), "non-finite lse"


def test_prefill_64k_full(N):
    # the call bench.py times for the 64K prefill: one dsa_forward over all
    # 65,536 rows (128 chunks of 512 rows, query groups of 4)
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    cfg = I.CONFIGS["prefill_64k"]
    sample = [0, 1, 2046, 2047, 2048, 9999, 30000, 45001, 65534, 65535]
    inp = I.generate(cfg, threads=16)
    wl = DeviceWorkload(inp)
    out, lse, idx = wl.forward()
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_FORWARD) == (0, -1)
    ran = wl.kernels_ran(N.DSA_OP_FORWARD)
    assert ran & N.DSA_KERNEL_INDEXER_TC and ran & N.DSA_KERNEL_TOPK and ran & N.DSA_KERNEL_MLA_TC
    _check_selection_properties_device(inp["row_klen"], int(inp["topk"]), idx, out, lse)
    s_out, s_lse, s_idx = (P.to_np(x[sample]) for x in (out, lse, idx))
    del wl, out, lse, idx, inp
    torch.cuda.empty_cache()
    # the sampled rows alone, stage by stage: their scores for the oracle
    # comparison; the selection must not depend on the batch
    sub = I.generate(cfg, rows=sample, threads=16)
    ws = DeviceWorkload(sub)
    r_sc = ws.indexer()
    r_idx = ws.topk_(r_sc)
    torch.cuda.synchronize()
    r_sc, r_idx = P.to_np(r_sc), P.to_np(r_idx)
    assert np.array_equal(r_idx, s_idx), "selection depends on the batch"
    P.check_rows(sub, range(len(sample)), r_sc, s_idx, s_out, s_lse)


def test_prefill_64k_sampled_rows(N):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    cfg = I.CONFIGS["prefill_64k"]
    sample = [0, 2047, 2048, 30000, 65535]
    sub = I.generate(cfg, rows=sample)
    wl = DeviceWorkload(sub)
    sc = wl.indexer()
    idx = wl.topk_(sc)
    out, lse = wl.mla(idx)
    torch.cuda.synchronize()
    for op in (N.DSA_OP_INDEXER, N.DSA_OP_TOPK, N.DSA_OP_SPARSE_MLA):
        assert wl.status(op) == (0, -1)
    sc, idx, out, lse = P.to_np(sc), P.to_np(idx), P.to_np(out), P.to_np(lse)
    _check_selection_properties(sub, idx, out, lse)
    P.check_rows(sub, range(len(sample)), sc, idx, out, lse)
