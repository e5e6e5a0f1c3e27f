"""The bounded waits end a kernel whose pipeline can no longer make progress.

A test-only fault makes the tensor-core indexer's epilogue withhold its
accumulator releases, with a short spin limit per wait.  The MMA issuer's wait
for a free accumulator must run out, record DSA_ERR_TIMEOUT at one of the
indexer's wait sites, and let the kernel return (the call completes and the
context stays usable: the next, fault-free call gives correct scores).
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from tests import parity as P

pytestmark = pytest.mark.gpu

# wait sites of the indexer kernel: producer (1, 2), MMA issuer (3, 4, 5),
# epilogue (6), producer tail (7, 8, 9, 10), key-scale warp (11)
INDEXER_SITES = set(range(1, 12))


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def test_indexer_wait_runs_out_and_reports(N):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload
    from oracle import dsa_ref as R
    # two sequences of ~100K keys: every CTA gets more tiles than accumulators,
    # so its MMA issuer reaches the withheld release
    cfg = I.CONFIGS["decode_128k_paged"].replace(n_seqs=2)
    inp = I.generate(cfg, threads=8)
    wl = DeviceWorkload(inp)
    N.dsa_set_fault_injection(1 << 10, N.DSA_FAULT_INDEXER_ACC_RELEASE)
    try:
        wl.indexer()
        torch.cuda.synchronize()
    finally:
        N.dsa_set_fault_injection(0, 0)
    code, site = wl.status(N.DSA_OP_INDEXER)
    assert code == N.DSA_ERR_TIMEOUT, (code, site)
    assert site in INDEXER_SITES, site
    # the context is intact: the same call without the fault is correct
    sc = P.to_np(wl.indexer())
    torch.cuda.synchronize()
    assert wl.status(N.DSA_OP_INDEXER) == (0, -1)
    for t in (0, wl.T - 1):
        klen = int(inp["row_klen"][t])
        P.check_scores(sc[t, :klen], R.row_scores(inp, t), f"row {t}")
