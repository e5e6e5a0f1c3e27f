"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Small workloads with the shapes and distributions of the five configurations
(several tiles, ragged tails, rows shorter than k), every row checked.
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_fp32": I.CONFIGS["tiny_fp32"],
    "decode_small": I.CONFIGS["decode_16k"].replace(ctx_lo=2100, ctx_hi=5000, n_seqs=6),
    "decode_short_rows": I.CONFIGS["decode_16k"].replace(ctx_lo=1, ctx_hi=2600, n_seqs=8),
    "prefill_small": I.CONFIGS["prefill_8k"].replace(seq_len=2500),
    "paged_small": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=2040, ctx_hi=6000, n_seqs=4),
    # rows longer than one CTA's shared-memory segment: top-k runs as a 2-4 CTA cluster
    "decode_cluster": I.CONFIGS["decode_16k"].replace(ctx_lo=17000, ctx_hi=40000, n_seqs=3),
    "paged_cluster": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=30000, ctx_hi=70000, n_seqs=2),
    # logits with std 8: block maxima move by more than 2^8, so O is rescaled mid-row
    "decode_sharp": I.CONFIGS["decode_16k"].replace(ctx_lo=2100, ctx_hi=5000, n_seqs=4, std_q=8.0),
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
        _cache[name] = I.generate(SMALL[name])
    return _cache[name]


def _run_stages(N, inp, algo):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    wl = DeviceWorkload(inp, algo=algo)
    scores = wl.indexer()
    idx = wl.topk_(scores)
    out, lse = wl.mla(idx)
    torch.cuda.synchronize()
    for op in (N.DSA_OP_INDEXER, N.DSA_OP_TOPK, N.DSA_OP_SPARSE_MLA):
        assert wl.status(op) == (0, -1)
    # the intended kernels ran (no silent fallback)
    ran_idx = wl.kernels_ran(N.DSA_OP_INDEXER)
    fp8 = inp["idx_dtype"] == "e4m3"
    want = N.DSA_KERNEL_INDEXER_TC if (fp8 and algo == N.DSA_ALGO_AUTO) else N.DSA_KERNEL_INDEXER_SIMT
    assert ran_idx == want, hex(ran_idx)
    assert wl.kernels_ran(N.DSA_OP_TOPK) == N.DSA_KERNEL_TOPK
    ran_mla = wl.kernels_ran(N.DSA_OP_SPARSE_MLA)
    if algo == N.DSA_ALGO_SIMT or inp["mla_dtype"] != "bf16":
        assert ran_mla == N.DSA_KERNEL_MLA_SIMT, hex(ran_mla)
    else:
        assert ran_mla & N.DSA_KERNEL_MLA_TC and not ran_mla & N.DSA_KERNEL_MLA_SIMT, hex(ran_mla)
    return wl, P.to_np(scores), P.to_np(idx), P.to_np(out), P.to_np(lse)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("algo", ["auto", "simt"])
def test_stagewise_parity(N, name, algo):
    inp = _inputs(name)
    a = N.DSA_ALGO_AUTO if algo == "auto" else N.DSA_ALGO_SIMT
    _, sc, idx, out, lse = _run_stages(N, inp, a)
    T = inp["row_seq"].shape[0]
    rows = range(T) if T <= 64 else sorted(set(np.linspace(0, T - 1, 48).astype(int)) | {T - 1})
    P.check_rows(inp, rows, sc, idx, out, lse)


@pytest.mark.parametrize("name", ["decode_small", "paged_small", "tiny_fp32"])
def test_decode_step_equals_stages(N, name):
    import torch
    inp = _inputs(name)
    wl, sc, idx, out, lse = _run_stages(N, inp, N.DSA_ALGO_AUTO)
    o2, l2, s2, i2 = wl.decode_step(debug=True)
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_DECODE_STEP) == (0, -1)
    klen = inp["row_klen"]
    s2 = P.to_np(s2)
    for t in range(len(klen)):
        assert np.array_equal(s2[t, : klen[t]], sc[t, : klen[t]])
    assert np.array_equal(P.to_np(i2), idx)
    np.testing.assert_array_equal(P.to_np(o2), out)
    np.testing.assert_array_equal(P.to_np(l2), lse)


@pytest.mark.parametrize("name", ["prefill_small", "tiny_fp32"])
def test_forward_equals_stages(N, name):
    import torch
    inp = _inputs(name)
    wl, sc, idx, out, lse = _run_stages(N, inp, N.DSA_ALGO_AUTO)
    o2, l2, i2 = wl.forward()
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_FORWARD) == (0, -1)
    assert np.array_equal(P.to_np(i2), idx)
    np.testing.assert_array_equal(P.to_np(o2), out)


def test_deterministic(N):
    inp = _inputs("paged_small")
    a = _run_stages(N, inp, N.DSA_ALGO_AUTO)
    b = _run_stages(N, inp, N.DSA_ALGO_AUTO)
    for x, y in zip(a[1:], b[1:]):
        np.testing.assert_array_equal(x, y)


def test_block_table_out_of_range_is_reported(N):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    inp = dict(_inputs("paged_small"))
    cache = dict(inp["cache"])
    bt = cache["block_table"].copy()
    bt[1, 3] = cache["num_pages"] + 7          # a page that does not exist
    cache["block_table"] = bt
    inp["cache"] = cache
    wl = DeviceWorkload(inp)
    wl.indexer()
    torch.cuda.synchronize()
    st, det = wl.status(N.DSA_OP_INDEXER)
    assert st == N.DSA_ERR_OUT_OF_RANGE and det == cache["num_pages"] + 7


def test_split_merge_on_a_reused_workspace(N):
    """The key splits of a decode row are merged inside the attention kernel by
    the last split to arrive, counted through arrival tickets in the workspace.
    A workspace holding stale bytes, reused by calls with different split plans
    and by repeated calls, gives the bits of a freshly initialised one."""
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload, _vp

    wl = DeviceWorkload(I.generate(SMALL["paged_small"]))
    idx = wl.topk_(wl.indexer())
    torch.cuda.synchronize()
    need = {k: N.dsa_workspace_size(wl.dims, N.dsa_rows(
        num_rows=k, row_seq=_vp(wl.row_seq), row_klen=_vp(wl.row_klen),
        max_klen=wl.max_klen, q_group=wl.rows.q_group), N.DSA_OP_SPARSE_MLA) for k in (1, 3, 8)}
    gen = torch.Generator(device="cuda").manual_seed(7)
    stale = torch.randint(0, 256, (max(need.values()),), dtype=torch.uint8, device="cuda",
                          generator=gen)
    N.dsa_workspace_init(_vp(stale), 256, wl.stream)          # the status block only
    for k in (8, 1, 3, 8, 3):
        rows = N.dsa_rows(num_rows=k, row_seq=_vp(wl.row_seq), row_klen=_vp(wl.row_klen),
                          max_klen=wl.max_klen, q_group=wl.rows.q_group)
        fresh = torch.empty(need[k], dtype=torch.uint8, device="cuda")
        N.dsa_workspace_init(_vp(fresh), need[k], wl.stream)
        outs = []
        for ws in (fresh, stale):
            out = torch.full((k, wl.H, wl.d_c), float("nan"), dtype=torch.bfloat16, device="cuda")
            lse = torch.full((k, wl.H), float("nan"), dtype=torch.float32, device="cuda")
            N.dsa_sparse_mla_fwd(wl.dims, rows, wl.cache, _vp(wl.q), _vp(idx), _vp(out), _vp(lse),
                                 _vp(ws), need[k], wl.stream)
            assert N.dsa_read_device_status(_vp(ws), wl.stream) == (0, -1)
            ran = N.dsa_read_kernel_trace(_vp(ws), wl.stream)
            assert ran & N.DSA_KERNEL_MLA_TC, hex(ran)
            # a plan with key splits merges them (and says so)
            assert bool(ran & N.DSA_KERNEL_MLA_COMBINE) == (need[k] > 256), (k, hex(ran))
            outs.append((out, lse))
        assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16)), k
        assert torch.equal(outs[0][1].view(torch.int32), outs[1][1].view(torch.int32)), k
        assert not torch.isnan(outs[1][0].float()).any(), k
