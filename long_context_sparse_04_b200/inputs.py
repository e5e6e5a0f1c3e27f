"""Seeded synthetic inputs for the DSA forward path.

This module holds no arithmetic of the method.  It draws the random tensors,
casts them to their storage formats (FP8 e4m3 with per-row fp32 scales for the
indexer, bf16 or fp32 for the MLA side) and lays out the caches (contiguous,
or 64-token pages under a shuffled block table).  The CUDA path and the CPU
oracle both receive exactly these bytes.

Every tensor is drawn piece by piece from
``numpy.random.Generator(PCG64(SeedSequence([seed, tensor_id, *piece])))`` so
that any query row, or any chunk of 1024 keys (16 pages of 64) of a sequence,
can be regenerated alone.

The workloads follow the five shapes the pages' DSA description is measured
at: a tiny fp32 prefill, 8K-16K decode, 8K and 64K causal prefill, and 96K-128K
paged decode with two query tokens per sequence.  Where the pages leave a
distribution open, the choices are: the second parameter of N(mu, x) is the
standard deviation; latents and RoPE keys are N(0, 1); 5% of key positions of
the prefill workloads carry a "planted" indexer key aligned with a random later
query head (norm 4 * sqrt(d_I)), set before FP8 quantisation.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# tensor ids of the seed sequences
TID_QIDX, TID_W, TID_KIDX, TID_LATENT, TID_Q, TID_PLANT, TID_LEN, TID_TABLE = range(1, 9)
TID_WUV, TID_WOUT, TID_O = 9, 10, 11
BLOCK = 64          # tokens per page of paged caches
CHUNK = 1024        # keys per seeded chunk of a sequence (a multiple of BLOCK)
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class DSAConfig:
    name: str
    prefill: bool           # True: one causal sequence, row t sees t+1 keys
    seq_len: int            # prefill length L (prefill) or upper context bound
    ctx_lo: int             # decode: context drawn uniformly from [ctx_lo, ctx_hi]
    ctx_hi: int
    n_seqs: int
    rows_per_seq: int       # decode query rows per sequence (1, or 2 for MTP)
    h_idx: int
    d_idx: int
    topk: int
    n_heads: int
    d_c: int
    d_r: int
    fp8: bool               # indexer in e4m3 + scales (else fp32)
    bf16: bool              # MLA operands in bf16 (else fp32)
    paged: bool
    plant_frac: float
    std_qidx: float
    std_kidx: float
    std_w: float
    std_q: float
    std_kv: float
    seed: int
    d_v: int = 128          # value head width after W_UV (output projection)
    d_model: int = 7168     # model width after W_out (output projection)

    @property
    def d_qk(self) -> int:
        return self.d_c + self.d_r

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_c + self.d_r)

    @property
    def n_rows(self) -> int:
        return self.seq_len if self.prefill else self.n_seqs * self.rows_per_seq

    def replace(self, **kw) -> "DSAConfig":
        return dataclasses.replace(self, **kw)


_BIG = dict(h_idx=64, d_idx=128, topk=2048, n_heads=128, d_c=512, d_r=64,
            fp8=True, bf16=True, std_qidx=1.0, std_kidx=1.0, std_w=1.0 / 8,
            std_q=0.05, std_kv=1.0)

CONFIGS = {
    # one causal sequence, fp32 throughout
    "tiny_fp32": DSAConfig(
        name="tiny_fp32", prefill=True, seq_len=256, ctx_lo=0, ctx_hi=0, n_seqs=1,
        rows_per_seq=256, h_idx=4, d_idx=32, topk=64, n_heads=8, d_c=64, d_r=16,
        fp8=False, bf16=False, paged=False, plant_frac=0.0, std_qidx=1.0,
        std_kidx=1.0, std_w=0.25, std_q=1.0 / math.sqrt(80), std_kv=1.0 / math.sqrt(80),
        seed=0),
    # 32 sequences x 1 new token, contexts 8K-16K, contiguous cache
    "decode_16k": DSAConfig(
        name="decode_16k", prefill=False, seq_len=16384, ctx_lo=8192, ctx_hi=16384,
        n_seqs=32, rows_per_seq=1, paged=False, plant_frac=0.0, seed=1, **_BIG),
    # one causal sequence of 8192 tokens with planted keys
    "prefill_8k": DSAConfig(
        name="prefill_8k", prefill=True, seq_len=8192, ctx_lo=0, ctx_hi=0, n_seqs=1,
        rows_per_seq=8192, paged=False, plant_frac=0.05, seed=2, **_BIG),
    # one causal sequence of 65536 tokens with planted keys
    "prefill_64k": DSAConfig(
        name="prefill_64k", prefill=True, seq_len=65536, ctx_lo=0, ctx_hi=0, n_seqs=1,
        rows_per_seq=65536, paged=False, plant_frac=0.05, seed=3, **_BIG),
    # 16 sequences x 2 query tokens, contexts 96K-128K, 64-token pages
    "decode_128k_paged": DSAConfig(
        name="decode_128k_paged", prefill=False, seq_len=131072, ctx_lo=98304,
        ctx_hi=131072, n_seqs=16, rows_per_seq=2, paged=True, plant_frac=0.0,
        seed=4, **_BIG),
}


# ----------------------------------------------------------------------------
# random streams
# ----------------------------------------------------------------------------

def _rng(seed: int, tid: int, *block: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, *block])))


def _normal(seed, tid, block, shape, std) -> np.ndarray:
    x = _rng(seed, tid, *block).standard_normal(size=shape, dtype=np.float32)
    return x * np.float32(std)


# ----------------------------------------------------------------------------
# storage casts (round to nearest even; FP8 saturates at +-448)
# ----------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def to_e4m3_rows(x: np.ndarray):
    """Quantise along the last axis: scale = amax/448 per row, codes = e4m3(x/scale)."""
    import torch
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = np.clip(x / scale[..., None], -E4M3_MAX, E4M3_MAX)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


# ----------------------------------------------------------------------------
# per-row / per-block generators
# ----------------------------------------------------------------------------

def qidx_rows_f32(cfg: DSAConfig, rows) -> np.ndarray:
    """Indexer queries before quantisation, [len(rows), H_I, d_I] float32."""
    return np.stack([_normal(cfg.seed, TID_QIDX, (int(t),), (cfg.h_idx, cfg.d_idx), cfg.std_qidx)
                     for t in rows]) if len(rows) else np.zeros((0, cfg.h_idx, cfg.d_idx), np.float32)


def w_rows(cfg: DSAConfig, rows) -> np.ndarray:
    if len(rows) == 0:
        return np.zeros((0, cfg.h_idx), np.float32)
    return np.stack([_normal(cfg.seed, TID_W, (int(t),), (cfg.h_idx,), cfg.std_w) for t in rows])


def q_rows(cfg: DSAConfig, rows) -> np.ndarray:
    """MLA queries [len(rows), H, d_c+d_r], storage format (bf16 bits or f32)."""
    x = np.stack([_normal(cfg.seed, TID_Q, (int(t),), (cfg.n_heads, cfg.d_qk), cfg.std_q)
                  for t in rows])
    return to_bf16_bits(x) if cfg.bf16 else x


def _plant_targets(cfg: DSAConfig, seq: int, chunk: int):
    """Planted positions in a 1024-key chunk: list of (offset, target row, target head)."""
    if cfg.plant_frac <= 0:
        return []
    r = _rng(cfg.seed, TID_PLANT, seq, chunk)
    mask = r.random(CHUNK) < cfg.plant_frac
    out = []
    for off in np.nonzero(mask)[0]:
        s = chunk * CHUNK + int(off)
        if s >= cfg.seq_len:
            continue
        tgt = int(r.integers(s, cfg.seq_len))
        head = int(r.integers(0, cfg.h_idx))
        out.append((int(off), tgt, head))
    return out


def key_chunk_f32(cfg: DSAConfig, seq: int, chunk: int):
    """Keys [1024*chunk, 1024*chunk + 1024) of sequence `seq` before the storage
    casts: (k_I float32 [1024, d_I], latent float32 [1024, d_c+d_r])."""
    k = _normal(cfg.seed, TID_KIDX, (seq, chunk), (CHUNK, cfg.d_idx), cfg.std_kidx)
    for off, tgt, head in _plant_targets(cfg, seq, chunk):
        qv = qidx_rows_f32(cfg, [tgt])[0, head]
        k[off] = np.float32(4.0 * math.sqrt(cfg.d_idx)) * qv / np.float32(np.linalg.norm(qv))
    lat = _normal(cfg.seed, TID_LATENT, (seq, chunk), (CHUNK, cfg.d_qk), cfg.std_kv)
    return k, lat


def key_chunk(cfg: DSAConfig, seq: int, chunk: int):
    """Keys [1024*chunk, 1024*chunk + 1024) of sequence `seq`, both caches.

    Returns (k_idx codes or f32 [1024, d_I], k_scale [1024] or None,
    latent [1024, d_c+d_r] in storage format).
    """
    k, lat = key_chunk_f32(cfg, seq, chunk)
    if cfg.fp8:
        kc, ks = to_e4m3_rows(k)
    else:
        kc, ks = k, None
    lat = to_bf16_bits(lat) if cfg.bf16 else lat
    return kc, ks, lat


def token_keys(cfg: DSAConfig, tok_seq, tok_pos):
    """The generator's keys of tokens (tok_seq[n], tok_pos[n]) before the FP8
    cast: (k_I float32 [n, d_I], latent [n, d_c+d_r] in storage format).  These
    are what a cache append of those tokens takes as input."""
    tok_seq = np.asarray(tok_seq, dtype=np.int64)
    tok_pos = np.asarray(tok_pos, dtype=np.int64)
    n = tok_seq.shape[0]
    k = np.zeros((n, cfg.d_idx), np.float32)
    lat = np.zeros((n, cfg.d_qk), np.float32)
    cache = {}
    for i in range(n):
        key = (int(tok_seq[i]), int(tok_pos[i]) // CHUNK)
        if key not in cache:
            cache = {key: key_chunk_f32(cfg, *key)}
        kc, lc = cache[key]
        k[i] = kc[tok_pos[i] % CHUNK]
        lat[i] = lc[tok_pos[i] % CHUNK]
    return k, (to_bf16_bits(lat) if cfg.bf16 else lat)


def new_tokens(cfg: DSAConfig):
    """The tokens a decode step of the workload appends before it attends: the
    last rows_per_seq positions of every sequence (prefill: every position).
    Returns (tok_seq int32 [n], tok_pos int32 [n])."""
    ctx = context_lengths(cfg)
    if cfg.prefill:
        return np.zeros(cfg.seq_len, np.int32), np.arange(cfg.seq_len, dtype=np.int32)
    nq = cfg.rows_per_seq
    seq = np.repeat(np.arange(cfg.n_seqs, dtype=np.int32), nq)
    j = np.tile(np.arange(nq), cfg.n_seqs)
    return seq, (ctx[seq] - nq + j).astype(np.int32)


def out_proj_weights(cfg: DSAConfig):
    """W_UV [H, d_v, d_c] ~ N(0, 1/d_c) and W_out [d_model, H*d_v] ~ N(0, 1/(H*d_v))
    (variances), as bf16 bit patterns: unit-scale projections of unit-scale
    inputs."""
    w_uv = _normal(cfg.seed, TID_WUV, (0,), (cfg.n_heads, cfg.d_v, cfg.d_c), 1 / math.sqrt(cfg.d_c))
    w_out = np.empty((cfg.d_model, cfg.n_heads * cfg.d_v), np.float32)
    step = 512
    for i in range(0, cfg.d_model, step):
        r = min(step, cfg.d_model - i)
        w_out[i:i + r] = _normal(cfg.seed, TID_WOUT, (i // step,), (r, cfg.n_heads * cfg.d_v),
                                 1 / math.sqrt(cfg.n_heads * cfg.d_v))
    return to_bf16_bits(w_uv), to_bf16_bits(w_out)


def latent_out_rows(cfg: DSAConfig, rows) -> np.ndarray:
    """Stand-ins for the sparse attention's latent output o [len(rows), H, d_c]
    (a softmax-weighted mean of unit-variance latent rows, so smaller than
    one): N(0, 0.1^2), bf16 bit patterns, seeded per row."""
    if len(rows) == 0:
        return np.zeros((0, cfg.n_heads, cfg.d_c), np.uint16)
    return to_bf16_bits(np.stack([_normal(cfg.seed, TID_O, (int(t),), (cfg.n_heads, cfg.d_c), 0.1)
                                  for t in rows]))


def context_lengths(cfg: DSAConfig) -> np.ndarray:
    if cfg.prefill:
        return np.array([cfg.seq_len], dtype=np.int64)
    r = _rng(cfg.seed, TID_LEN, 0)
    return r.integers(cfg.ctx_lo, cfg.ctx_hi + 1, size=cfg.n_seqs).astype(np.int64)


def row_layout(cfg: DSAConfig):
    """row_seq, row_klen (int32 [T]).  Decode row j of n_q sees ctx-(n_q-1-j)."""
    if cfg.prefill:
        t = np.arange(cfg.seq_len, dtype=np.int32)
        return np.zeros(cfg.seq_len, np.int32), t + 1
    ctx = context_lengths(cfg)
    nq = cfg.rows_per_seq
    seq = np.repeat(np.arange(cfg.n_seqs, dtype=np.int32), nq)
    j = np.tile(np.arange(nq), cfg.n_seqs)
    klen = (ctx[seq] - (nq - 1 - j)).astype(np.int32)
    return seq, klen


# ----------------------------------------------------------------------------
# whole workload
# ----------------------------------------------------------------------------

def generate(cfg: DSAConfig, with_q: bool = True, threads: int = 8, rows=None) -> dict:
    """All inputs of one workload as host numpy arrays (storage formats).

    Keys: row_seq, row_klen, q_idx, q_scale, w, k_idx, k_scale, latent, q,
    cache (seq_start | block_table, page_size, num_pages), topk, d_c, d_r,
    sm_scale, idx_dtype, mla_dtype, n_heads, h_idx, d_idx, cfg.

    rows: a subset of the workload's query rows (their indices), or None for
    all.  Every query row is seeded on its own, so a subset's rows are
    bit-identical to the same rows of the whole workload; the caches are always
    generated whole.
    """
    row_seq, row_klen = row_layout(cfg)
    qrows = np.arange(row_seq.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    row_seq, row_klen = row_seq[qrows], row_klen[qrows]
    T = row_seq.shape[0]
    ctx = context_lengths(cfg)
    nblk = [(int(c) + BLOCK - 1) // BLOCK for c in ctx]
    total_blocks = sum(nblk)
    n_tok = total_blocks * BLOCK

    # block placement: logical (seq, blk) -> physical block id
    if cfg.paged:
        perm = _rng(cfg.seed, TID_TABLE, 0).permutation(total_blocks).astype(np.int32)
        max_pages = max(nblk)
        table = np.full((cfg.n_seqs, max_pages), -1, dtype=np.int32)
        placements, o = [], 0
        for b in range(len(ctx)):
            table[b, : nblk[b]] = perm[o: o + nblk[b]]
            placements += [(b, lb, int(perm[o + lb])) for lb in range(nblk[b])]
            o += nblk[b]
        cache = {"block_table": table, "page_size": BLOCK, "num_pages": total_blocks,
                 "seq_start": None}
    else:
        starts = np.zeros(len(ctx), dtype=np.int64)
        placements, o = [], 0
        for b in range(len(ctx)):
            starts[b] = o * BLOCK
            placements += [(b, lb, o + lb) for lb in range(nblk[b])]
            o += nblk[b]
        cache = {"block_table": None, "page_size": BLOCK, "num_pages": total_blocks,
                 "seq_start": starts.astype(np.int32)}

    kdt = np.uint8 if cfg.fp8 else np.float32
    ldt = np.uint16 if cfg.bf16 else np.float32
    k_idx = np.zeros((n_tok, cfg.d_idx), dtype=kdt)
    k_scale = np.ones(n_tok, dtype=np.float32) if cfg.fp8 else None
    latent = np.zeros((n_tok, cfg.d_qk), dtype=ldt)

    # logical block (seq, lb) -> physical block, then fill chunk by chunk
    phys_of = {(b, lb): ph for b, lb, ph in placements}
    per = CHUNK // BLOCK

    def fill(job):
        b, c = job
        kc, ks, lat = key_chunk(cfg, b, c)
        for i in range(per):
            ph = phys_of.get((b, c * per + i))
            if ph is None:
                break
            src_sl = slice(i * BLOCK, (i + 1) * BLOCK)
            dst = slice(ph * BLOCK, (ph + 1) * BLOCK)
            k_idx[dst] = kc[src_sl]
            if ks is not None:
                k_scale[dst] = ks[src_sl]
            latent[dst] = lat[src_sl]

    jobs = [(b, c) for b in range(len(ctx)) for c in range((nblk[b] + per - 1) // per)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, jobs))

    # indexer queries, in row chunks on the thread pool (every row is seeded on
    # its own and quantised on its own, so the chunking changes no byte)
    def qidx_chunk(r):
        qf = qidx_rows_f32(cfg, r)
        return to_e4m3_rows(qf) if cfg.fp8 else (qf, None)

    chunks = [qrows[i: i + 1024] for i in range(0, T, 1024)] or [qrows]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(qidx_chunk, chunks))
    q_idx = np.concatenate([p[0] for p in parts])
    q_scale = np.concatenate([p[1] for p in parts]) if cfg.fp8 else None
    w = w_rows(cfg, qrows)
    inp = dict(row_seq=row_seq, row_klen=row_klen, q_idx=q_idx, q_scale=q_scale, w=w,
               k_idx=k_idx, k_scale=k_scale, latent=latent, cache=cache,
               topk=cfg.topk, d_c=cfg.d_c, d_r=cfg.d_r, sm_scale=cfg.sm_scale,
               idx_dtype="e4m3" if cfg.fp8 else "f32", mla_dtype="bf16" if cfg.bf16 else "f32",
               n_heads=cfg.n_heads, h_idx=cfg.h_idx, d_idx=cfg.d_idx, cfg=cfg)
    if with_q:
        chunks = [qrows[i: i + 256] for i in range(0, T, 256)]
        with ThreadPoolExecutor(max_workers=threads) as ex:
            parts = list(ex.map(lambda r: q_rows(cfg, r), chunks))
        inp["q"] = np.concatenate(parts) if parts else None
    else:
        inp["q"] = None
    return inp
