"""dsa_sparse_mla_fwd_noalloc (static device scratch) against dsa_sparse_mla_fwd.

The file name sorts last so that the static scratch is exercised both after
every other GPU test and, run on its own, in a fresh process.
"""
import ctypes

import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = {
    # 8 rows: the split plan gives several key splits per row, so the
    # partials live in the scratch and every split holds keys
    "paged_8rows": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=6000, ctx_hi=9000, n_seqs=4),
    # 3 rows, some shorter than k: splits with few or no keys
    "decode_3rows": I.CONFIGS["decode_16k"].replace(ctx_lo=1500, ctx_hi=4000, n_seqs=3),
}


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def _vp(x):
    return ctypes.c_void_p(x.data_ptr())


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_call(N, name):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload

    wl = DeviceWorkload(I.generate(CASES[name]))
    # the split plan keeps partials beyond the 256-byte status block
    assert N.dsa_workspace_size(wl.dims, wl.rows, N.DSA_OP_SPARSE_MLA) > 256
    idx = wl.topk_(wl.indexer())
    ref_out, ref_lse = wl.mla(idx)
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_SPARSE_MLA) == (0, -1)
    assert wl.kernels_ran(N.DSA_OP_SPARSE_MLA) & N.DSA_KERNEL_MLA_TC

    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        N.dsa_sparse_mla_fwd_noalloc(wl.dims, wl.rows, wl.cache, _vp(wl.q), _vp(idx), _vp(out),
                                     _vp(lse), wl.stream)
        torch.cuda.synchronize()
        if call == 1:  # the first call may still load modules; later ones allocate nothing
            assert torch.cuda.mem_get_info()[0] == free_before
        # same kernels, same split plan: identical bits
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"call {call}"
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"call {call}"


def test_noalloc_rejects_plans_beyond_the_scratch(N):
    import torch

    # d_c = 8192 with 128 heads: one row in 8 key splits needs ~32 MiB of
    # partials, beyond the 20 MiB array; the call must refuse before launching
    dev = torch.device("cuda")
    buf = torch.zeros(1 << 16, dtype=torch.float32, device=dev)
    p = _vp(buf)
    dims = N.dsa_dims(n_idx_heads=64, d_idx=128, n_heads=128, d_c=8192, d_r=64, topk=2048,
                      idx_dtype=N.DSA_FP8_E4M3, mla_dtype=N.DSA_BF16, sm_scale=0.1,
                      algo=N.DSA_ALGO_AUTO)
    rows = N.dsa_rows(num_rows=1, row_seq=p, row_klen=p, max_klen=4096, q_group=1)
    cache = N.dsa_cache(latent=p, num_seqs=1, num_tokens=4096)
    need = N.dsa_workspace_size(dims, rows, N.DSA_OP_SPARSE_MLA)
    assert need > 20 << 20
    st = N.dsa_sparse_mla_fwd_noalloc(dims, rows, cache, p, p, p, None,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                      check=False)
    assert st == N.DSA_ERR_WORKSPACE
    msg = N.LIB.dsa_last_error().decode()
    assert "static scratch" in msg and str(need) in msg, msg
    torch.cuda.synchronize()
    assert np.all(buf.cpu().numpy() == 0)  # nothing ran
