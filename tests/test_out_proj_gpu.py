"""GPU parity of the output projection (dsa_output_projection) against the
oracle's output_projection_row, on the same bf16 inputs.

Tolerances come from the arithmetic.  u is one fp32-accumulated dot product
per element rounded to bf16 once: within 2^-9 of |u| (the fp32 sums over
K = d_c terms add far less), so the test allows 2^-8 |u| + 2^-10 rms(u row).
y is computed from the bf16 u, so each u's rounding (relative, at most 2^-9,
signs independent) enters y as a sum over K = H*d_v terms whose size is about
2^-9/sqrt(3) rms(y row); y is then rounded to bf16 once more (2^-9 |y|).  The
test allows 2^-7 (|y| + rms(y row)), about seven standard deviations of the
first term.  A dropped K block of 64 out of 16,384 would show as ~6% of
rms(y), far outside it.
"""
import numpy as np
import pytest

from long_context_sparse_04_b200 import inputs as I
from oracle import dsa_ref as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def N():
    from long_context_sparse_04_b200 import build
    build.build()
    from long_context_sparse_04_b200 import _native
    return _native


def _bf16(bits):
    return R.bf16_decode(bits)


def _run(N, o_bits, w_uv_bits, w_out_bits, d_v, d_model, o_dev=None):
    import ctypes
    import torch
    from long_context_sparse_04_b200.workload import to_device
    dev = torch.device("cuda")
    T, H, d_c = o_bits.shape if o_dev is None else o_dev.shape
    dims = N.dsa_proj_dims(n_heads=H, d_c=d_c, d_v=d_v, d_model=d_model)
    o = to_device(o_bits, dev) if o_dev is None else o_dev
    w_uv = to_device(w_uv_bits, dev)
    w_out = to_device(w_out_bits, dev)
    u = torch.full((T, H, d_v), float("nan"), dtype=torch.bfloat16, device=dev)
    y = torch.full((T, d_model), float("nan"), dtype=torch.bfloat16, device=dev)
    nbytes = N.dsa_output_projection_ws_size(dims, T)
    assert nbytes > 0
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    vp = lambda x: ctypes.c_void_p(x.data_ptr())
    N.dsa_output_projection(dims, T, vp(o), vp(w_uv), vp(w_out), vp(u), vp(y), vp(ws), nbytes, stream)
    torch.cuda.synchronize()
    st = N.dsa_read_device_status(vp(ws), stream)
    ran = N.dsa_read_kernel_trace(vp(ws), stream)
    return u, y, st, ran


def _check(rows, w_uv_bits, w_out_bits, u_gpu, y_gpu):
    w_uv, w_out = _bf16(w_uv_bits), _bf16(w_out_bits)
    for t, ob in rows:
        u_ref, y_ref = R.output_projection_row(_bf16(ob), w_uv, w_out)
        ug = u_gpu[t].float().cpu().numpy().astype(np.float64)
        yg = y_gpu[t].float().cpu().numpy().astype(np.float64)
        u_rms = np.sqrt(np.mean(u_ref ** 2))
        y_rms = np.sqrt(np.mean(y_ref ** 2))
        du = np.abs(ug - u_ref) - (2.0 ** -8 * np.abs(u_ref) + 2.0 ** -10 * u_rms)
        dy = np.abs(yg - y_ref) - 2.0 ** -7 * (np.abs(y_ref) + y_rms)
        assert du.max() <= 0, f"row {t}: u off by {du.max():.3e} beyond the bound"
        assert dy.max() <= 0, f"row {t}: y off by {dy.max():.3e} beyond the bound"


# (T, H, d_c, d_v, d_model): ragged row tiles, a ragged column tile, a K split,
# d_v = 256 (one full N tile per head), and the decode shape at full size
SHAPES = {
    "small": (37, 4, 128, 64, 96),
    "split_ragged": (200, 8, 512, 128, 544),
    "dv256": (130, 2, 192, 256, 64),
    "decode_full": (32, 128, 512, 128, 7168),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_out_proj_matches_oracle(N, name):
    T, H, d_c, d_v, d_model = SHAPES[name]
    cfg = I.CONFIGS["decode_128k_paged"].replace(n_heads=H, d_c=d_c, d_v=d_v, d_model=d_model,
                                                seed=30 + list(SHAPES).index(name))
    w_uv, w_out = I.out_proj_weights(cfg)
    o = I.latent_out_rows(cfg, range(T))
    u, y, st, ran = _run(N, o, w_uv, w_out, d_v, d_model)
    assert st == (0, -1)
    assert ran & N.DSA_KERNEL_OUT_PROJ
    import torch
    assert not torch.isnan(u).any() and not torch.isnan(y).any(), "an output was not written"
    _check([(t, o[t]) for t in range(T)], w_uv, w_out, u, y)


def test_out_proj_split_reduce_runs(N):
    # the decode shape splits K over the SMs; the sum kernel must have run
    T, H, d_c, d_v, d_model = SHAPES["decode_full"]
    cfg = I.CONFIGS["decode_128k_paged"].replace(n_heads=H, d_c=d_c, d_v=d_v, d_model=d_model)
    w_uv, w_out = I.out_proj_weights(cfg)
    o = I.latent_out_rows(cfg, range(T))
    u1, y1, st, ran = _run(N, o, w_uv, w_out, d_v, d_model)
    assert ran & N.DSA_KERNEL_OUT_PROJ_REDUCE
    u2, y2, _, _ = _run(N, o, w_uv, w_out, d_v, d_model)
    import torch
    assert torch.equal(u1.view(torch.int16), u2.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "not deterministic"


def test_out_proj_empty_and_rejections(N):
    import ctypes
    dims = N.dsa_proj_dims(n_heads=4, d_c=128, d_v=64, d_model=96)
    assert N.dsa_output_projection_ws_size(dims, 0) == 256
    bad = N.dsa_proj_dims(n_heads=4, d_c=100, d_v=64, d_model=96)
    assert N.dsa_output_projection_ws_size(bad, 8) == 0
    import torch
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = N.dsa_output_projection(dims, 0, None, None, None, None, None,
                                 ctypes.c_void_p(ws.data_ptr()), 256, None, check=False)
    assert st == N.DSA_OK
    st = N.dsa_output_projection(bad, 8, None, None, None, None, None,
                                 ctypes.c_void_p(ws.data_ptr()), 256, None, check=False)
    assert st == N.DSA_ERR_UNSUPPORTED


def test_out_proj_prefill_64k_full(N):
    """All 65,536 rows of the 64K prefill at the production shape.  o is a
    1,024-row seeded block repeated down the rows: sampled rows are checked
    against the oracle, and rows with equal inputs must give bit-equal outputs
    wherever they sit among the 512 row tiles."""
    import torch
    cfg = I.CONFIGS["prefill_64k"]
    T, blk = cfg.seq_len, 1024
    w_uv, w_out = I.out_proj_weights(cfg)
    o_blk = I.latent_out_rows(cfg, range(blk))
    from long_context_sparse_04_b200.workload import to_device
    o_dev = to_device(o_blk, torch.device("cuda")).repeat(T // blk, 1, 1)
    u, y, st, ran = _run(N, None, w_uv, w_out, cfg.d_v, cfg.d_model, o_dev=o_dev)
    assert st == (0, -1) and ran & N.DSA_KERNEL_OUT_PROJ
    sample = [0, 127, 128, 1023, 1024, 40000, 65535]
    _check([(t, o_blk[t % blk]) for t in sample], w_uv, w_out, u, y)
    for t in [1024 + 5, 33 * 1024 + 900, 65535]:
        assert torch.equal(y[t].view(torch.int16), y[t % blk].view(torch.int16))
        assert torch.equal(u[t].view(torch.int16), u[t % blk].view(torch.int16))
