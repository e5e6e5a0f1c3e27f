"""GPU parity of the indexer warm-up ("DeepSeek Sparse Attention DSA
Architecture Guide", section "Training Mechanics: Dense Warm-Up and KL
Alignment", Phase 1): dsa_indexer_kl (loss and dL/dI per row) and
dsa_indexer_backward (dq_I, dw, dk_I), through the C ABI, against the
float64 oracle (oracle/dsa_ref.py: indexer_kl_row, indexer_backward_row).

Each stage is checked on the GPU's own inputs (the KL on the GPU's scores,
the backward on the GPU's gradient), so the comparison isolates that stage.
The ReLU mask is decided exactly on both sides (the dot product of e4m3 codes
is exact in fp64), so every difference is fp32 rounding:
  loss:     |d| <= 1e-4 |ref| + 1e-6
  dL/dI:    |d| <= 1e-5 (softmax(I)_s + p_s) + 1e-9
  dq,dw,dk: |d| <= 1e-5 A + 1e-6 rms(ref), where A is the same sum taken over
            the absolute values of its terms (a sum of n fp32 terms is within
            about sqrt(n) * 2^-24 * A of exact; the terms have both signs, the
            head weights being signed, so A, not the result, sets the scale)
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from oracle import dsa_ref as R
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    # decode rows, two per sequence, paged caches: every key seen by 1-2 rows
    "paged_decode": I.CONFIGS["decode_128k_paged"].replace(ctx_lo=1500, ctx_hi=5200, n_seqs=3),
    # one causal sequence: key s is seen by every row t >= s (dk sums over rows)
    "prefill": I.CONFIGS["prefill_8k"].replace(seq_len=700),
    # fp32 indexer operands (no FP8, no scales), contiguous cache
    "decode_f32": I.CONFIGS["decode_16k"].replace(ctx_lo=900, ctx_hi=2100, n_seqs=3, fp8=False),
}


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def _teacher(klen, rng):
    """A row's teacher: positive weights with some exact zeros, summing to 1."""
    p = rng.random(klen) ** 3
    p[rng.random(klen) < 0.1] = 0.0
    p[0] = max(p[0], 1e-3)
    return p / p.sum()


def _rms(x):
    return float(np.sqrt(np.mean(np.square(x)))) if x.size else 0.0


def _close(got, ref, abs_sum, what):
    tol = 1e-5 * abs_sum + 1e-6 * _rms(ref)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {ref.size} outside; worst {np.abs(got - ref).max():.3e}"


def _run(N, name):
    import torch
    from long_context_sparse_04_b200.workload import DeviceWorkload, _vp
    inp = I.generate(CASES[name], with_q=False, threads=8)
    wl = DeviceWorkload(inp)
    T, ld = wl.T, wl.ld
    rng = np.random.default_rng(list(CASES).index(name) + 40)
    klen = inp["row_klen"].astype(int)
    p = np.zeros((T, ld), np.float32)
    for t in range(T):
        p[t, : klen[t]] = _teacher(klen[t], rng)
    dev = wl.device
    scores = wl.indexer()
    p_d = torch.from_numpy(p).to(dev)
    grad = torch.full((T, ld), float("nan"), dtype=torch.float32, device=dev)
    loss = torch.empty(T, dtype=torch.float32, device=dev)
    n = N.dsa_workspace_size(wl.dims, wl.rows, N.DSA_OP_INDEXER_KL)
    ws_kl = torch.zeros(n, dtype=torch.uint8, device=dev)
    N.dsa_indexer_kl(wl.rows, _vp(scores), ld, _vp(p_d), ld, _vp(grad), ld, _vp(loss), _vp(ws_kl), n,
                     wl.stream)
    H_I, d_I = wl.dims.n_idx_heads, wl.dims.d_idx
    dq = torch.empty((T, H_I, d_I), dtype=torch.float32, device=dev)
    dw = torch.empty((T, H_I), dtype=torch.float32, device=dev)
    dk = torch.zeros((int(inp["k_idx"].shape[0]), d_I), dtype=torch.float32, device=dev)
    n = N.dsa_workspace_size(wl.dims, wl.rows, N.DSA_OP_INDEXER_BACKWARD)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)

    def backward():
        N.dsa_indexer_backward(wl.dims, wl.rows, wl.cache, _vp(wl.q_idx), _vp(wl.q_scale), _vp(wl.w),
                               _vp(grad), ld, _vp(dq), _vp(dw), _vp(dk), _vp(ws), n, wl.stream)
        torch.cuda.synchronize()
        return P.to_np(dq).copy(), P.to_np(dw).copy(), P.to_np(dk).copy()

    out = backward()
    assert N.dsa_read_device_status(_vp(ws), wl.stream) == (0, -1)
    assert N.dsa_read_kernel_trace(_vp(ws), wl.stream) & N.DSA_KERNEL_WARMUP
    assert N.dsa_read_device_status(_vp(ws_kl), wl.stream) == (0, -1)
    again = backward()
    for x, y in zip(out, again):                          # deterministic run to run
        np.testing.assert_array_equal(x, y)
    return inp, p, P.to_np(scores), P.to_np(grad), P.to_np(loss), out


@pytest.mark.parametrize("name", list(CASES))
def test_warmup_kl_and_backward(N, name):
    inp, p, sc, g, loss, (dq, dw, dk) = _run(N, name)
    klen = inp["row_klen"].astype(int)
    T = len(klen)
    dk_ref = np.zeros_like(dk, dtype=np.float64)
    dk_abs = np.zeros_like(dk_ref)
    seen = np.zeros(dk.shape[0], bool)
    for t in range(T):
        n = klen[t]
        kl, g_ref = R.indexer_kl_row(p[t, :n].astype(np.float64), sc[t, :n].astype(np.float64))
        assert abs(loss[t] - kl) <= 1e-4 * abs(kl) + 1e-6, f"loss row {t}: {loss[t]} vs {kl}"
        q_soft = g_ref + p[t, :n]
        tol = 1e-5 * (np.abs(q_soft) + p[t, :n]) + 1e-9
        assert (np.abs(g[t, :n] - g_ref) <= tol).all(), f"grad row {t}"
        # backward on the GPU's own gradient
        rows = R.physical_rows(int(inp["row_seq"][t]), np.arange(n), inp["cache"])
        qd = R.dequant_queries(inp, t)
        kd = R.dequant_keys(inp, rows)
        w = np.asarray(inp["w"][t], dtype=np.float32).astype(np.float64)
        gt = g[t, :n].astype(np.float64)
        # ReLU's mask taken exactly, as the kernel takes it: the sign of the dot
        # product of the stored values (e4m3 codes or fp32), exact in float64
        # for e4m3 (the scales are positive and do not change it)
        kc = R.as_f64(inp["k_idx"][rows], inp["idx_dtype"])
        qc = R.as_f64(inp["q_idx"][t], inp["idx_dtype"])
        on = (kc @ qc.T) > 0
        dq_r, dw_r, dk_r = R.indexer_backward_row(qd, w, kd, gt, on=on)
        # the same sums over the absolute values of their terms
        ga = np.abs(gt)[:, None] * on * np.abs(w)[None, :]
        _close(dq[t], dq_r, ga.T @ np.abs(kd), f"dq row {t}")
        _close(dw[t], dw_r, (np.maximum(kd @ qd.T, 0) * on).T @ np.abs(gt), f"dw row {t}")
        np.add.at(dk_ref, rows, dk_r)
        np.add.at(dk_abs, rows, ga @ np.abs(qd))
        seen[rows] = True
    _close(dk[seen], dk_ref[seen], dk_abs[seen], "dk")
    assert np.all(dk[~seen] == 0), "keys no row sees are written"
