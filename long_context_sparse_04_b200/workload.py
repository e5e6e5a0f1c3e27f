"""Device-side plumbing: put a workload's tensors in HBM and call the C ABI.

PyTorch provides device memory and streams only; every stage runs in
libdsa.so through the binding in ``_native``.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _native as N


def _vp(x):
    return None if x is None else ctypes.c_void_p(x.data_ptr())


def to_device(a: np.ndarray | None, device):
    import torch
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:                       # bf16 bit patterns
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def q_group_for(cfg) -> int:
    if cfg.prefill:
        return 4
    return cfg.rows_per_seq if cfg.rows_per_seq in (1, 2, 4) else 1


class DeviceWorkload:
    """One workload resident on a CUDA device, with the C-ABI descriptors."""

    def __init__(self, inp: dict, device="cuda", algo: int = N.DSA_ALGO_AUTO,
                 q_group: int | None = None):
        import torch
        self.torch = torch
        self.inp = inp
        self.device = torch.device(device)
        cfg = inp["cfg"]
        self.cfg = cfg
        dev = self.device
        self.row_seq = to_device(inp["row_seq"].astype(np.int32), dev)
        self.row_klen = to_device(inp["row_klen"].astype(np.int32), dev)
        self.q_idx = to_device(inp["q_idx"], dev)
        self.q_scale = to_device(inp["q_scale"], dev)
        self.w = to_device(inp["w"].astype(np.float32), dev)
        self.k_idx = to_device(inp["k_idx"], dev)
        self.k_scale = to_device(inp["k_scale"], dev)
        self.latent = to_device(inp["latent"], dev)
        self.q = to_device(inp["q"], dev) if inp.get("q") is not None else None
        c = inp["cache"]
        self.seq_start = to_device(c["seq_start"], dev) if c.get("seq_start") is not None else None
        self.block_table = to_device(c["block_table"], dev) if c.get("block_table") is not None else None
        T = int(inp["row_seq"].shape[0])
        self.T = T
        self.max_klen = int(inp["row_klen"].max()) if T else 0
        self.ld = ((self.max_klen + 127) // 128) * 128
        self.topk = int(inp["topk"])
        self.H = int(inp["n_heads"])
        self.d_c = int(inp["d_c"])
        self.mla_bf16 = inp["mla_dtype"] == "bf16"
        self.dims = N.dsa_dims(
            n_idx_heads=int(inp["h_idx"]), d_idx=int(inp["d_idx"]), n_heads=self.H,
            d_c=self.d_c, d_r=int(inp["d_r"]), topk=self.topk,
            idx_dtype=N.DSA_FP8_E4M3 if inp["idx_dtype"] == "e4m3" else N.DSA_F32,
            mla_dtype=N.DSA_BF16 if self.mla_bf16 else N.DSA_F32,
            sm_scale=float(inp["sm_scale"]), algo=algo)
        self.rows = N.dsa_rows(num_rows=T, row_seq=_vp(self.row_seq), row_klen=_vp(self.row_klen),
                               max_klen=self.max_klen,
                               q_group=q_group if q_group is not None else q_group_for(cfg))
        n_tok = int(inp["k_idx"].shape[0])
        bt = c.get("block_table")
        self.cache = N.dsa_cache(
            latent=_vp(self.latent), idx_k=_vp(self.k_idx), idx_k_scale=_vp(self.k_scale),
            seq_start=_vp(self.seq_start), block_table=_vp(self.block_table),
            page_size=int(c["page_size"]) if bt is not None else 0,
            max_pages_per_seq=int(bt.shape[1]) if bt is not None else 0,
            num_seqs=int(len(c["seq_start"]) if bt is None else bt.shape[0]), num_tokens=n_tok)
        self._ws = {}

    # ------------------------------------------------------------------ helpers
    @property
    def stream(self):
        return ctypes.c_void_p(self.torch.cuda.current_stream(self.device).cuda_stream)

    def workspace(self, op: int):
        if op not in self._ws:
            n = N.dsa_workspace_size(self.dims, self.rows, op)
            assert n > 0, "dsa_workspace_size returned 0"
            ws = self.torch.empty(n, dtype=self.torch.uint8, device=self.device)
            N.dsa_workspace_init(_vp(ws), n, self.stream)
            self._ws[op] = (ws, n)
        return self._ws[op]

    def status(self, op: int):
        ws, _ = self.workspace(op)
        return N.dsa_read_device_status(_vp(ws), self.stream)

    def kernels_ran(self, op: int) -> int:
        ws, _ = self.workspace(op)
        return N.dsa_read_kernel_trace(_vp(ws), self.stream)

    def out_dtype(self):
        return self.torch.bfloat16 if self.mla_bf16 else self.torch.float32

    # ------------------------------------------------------------------ stages
    def indexer(self, scores=None):
        torch = self.torch
        if scores is None:
            scores = torch.full((self.T, self.ld), float("nan"), dtype=torch.float32, device=self.device)
        ws, n = self.workspace(N.DSA_OP_INDEXER)
        N.dsa_indexer_scores(self.dims, self.rows, self.cache, _vp(self.q_idx), _vp(self.q_scale),
                             _vp(self.w), _vp(scores), self.ld, _vp(ws), n, self.stream)
        return scores

    def topk_(self, scores, idx=None):
        torch = self.torch
        if idx is None:
            idx = torch.empty((self.T, self.topk), dtype=torch.int32, device=self.device)
        ws, n = self.workspace(N.DSA_OP_TOPK)
        N.dsa_topk(self.dims, self.rows, _vp(scores), scores.shape[1], _vp(idx), _vp(ws), n,
                   self.stream)
        return idx

    def mla(self, idx, out=None, lse=None):
        torch = self.torch
        if out is None:
            out = torch.empty((self.T, self.H, self.d_c), dtype=self.out_dtype(), device=self.device)
        if lse is None:
            lse = torch.empty((self.T, self.H), dtype=torch.float32, device=self.device)
        ws, n = self.workspace(N.DSA_OP_SPARSE_MLA)
        N.dsa_sparse_mla_fwd(self.dims, self.rows, self.cache, _vp(self.q), _vp(idx), _vp(out),
                             _vp(lse), _vp(ws), n, self.stream)
        return out, lse

    def decode_step(self, out=None, lse=None, debug=False):
        torch = self.torch
        if out is None:
            out = torch.empty((self.T, self.H, self.d_c), dtype=self.out_dtype(), device=self.device)
        if lse is None:
            lse = torch.empty((self.T, self.H), dtype=torch.float32, device=self.device)
        dbg_s = dbg_i = None
        if debug:
            dbg_s = torch.full((self.T, self.ld), float("nan"), dtype=torch.float32, device=self.device)
            dbg_i = torch.empty((self.T, self.topk), dtype=torch.int32, device=self.device)
        ws, n = self.workspace(N.DSA_OP_DECODE_STEP)
        N.dsa_decode_step(self.dims, self.rows, self.cache, _vp(self.q_idx), _vp(self.q_scale),
                          _vp(self.w), _vp(self.q), _vp(out), _vp(lse), _vp(dbg_s), _vp(dbg_i),
                          _vp(ws), n, self.stream)
        return out, lse, dbg_s, dbg_i

    def forward(self, out=None, lse=None, idx=None):
        torch = self.torch
        if out is None:
            out = torch.empty((self.T, self.H, self.d_c), dtype=self.out_dtype(), device=self.device)
        if lse is None:
            lse = torch.empty((self.T, self.H), dtype=torch.float32, device=self.device)
        if idx is None:
            idx = torch.empty((self.T, self.topk), dtype=torch.int32, device=self.device)
        ws, n = self.workspace(N.DSA_OP_FORWARD)
        N.dsa_forward(self.dims, self.rows, self.cache, _vp(self.q_idx), _vp(self.q_scale),
                      _vp(self.w), _vp(self.q), _vp(out), _vp(lse), _vp(idx), _vp(ws), n,
                      self.stream)
        return out, lse, idx

    def append(self, tok_seq, tok_pos, k_new, latent_new, check=True):
        """dsa_cache_append of new tokens (device tensors: int32 [n], int32 [n],
        fp32 [n, d_I], latent rows [n, d_c+d_r]) into this workload's caches."""
        ws, n = self.workspace(N.DSA_OP_CACHE_APPEND)
        return N.dsa_cache_append(self.dims, self.cache, int(tok_seq.shape[0]), _vp(tok_seq),
                                  _vp(tok_pos), _vp(k_new), _vp(latent_new), _vp(ws), n,
                                  self.stream, check=check)

    def caches_to_host(self):
        """(k_idx, k_scale, latent) in their storage formats (bf16 as uint16 bits)."""
        torch = self.torch
        lat = self.latent
        lat = lat.view(torch.int16).cpu().numpy().view(np.uint16) if lat.dtype == torch.bfloat16 \
            else lat.cpu().numpy()
        ks = None if self.k_scale is None else self.k_scale.cpu().numpy()
        return self.k_idx.cpu().numpy(), ks, lat
