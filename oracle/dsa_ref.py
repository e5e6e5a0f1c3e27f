"""Float64 CPU oracle for the DeepSeek Sparse Attention (DSA) forward hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) may import, call or link this module; only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` use it.  It shares no code with the CUDA path: the only thing the
two sides have in common is the seeded input generator, which hands both the
same bytes.

What is computed, and where the definition comes from (page title, then the
section and equation on that page):

* "DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 1: The
  Lightning Indexer", index-score equation I = ReLU(q_I . k_I / sqrt(d_I)),
  generalised to H_I weighted heads  I[t,s] = sum_j w[t,j] ReLU(q[t,j] . k[s]).
  The single-head form is the special case H_I = 1, w = 1/sqrt(d_I), because
  ReLU is positively homogeneous (pinned in the tests).
* same page, same section, item "Native FP8 Precision": the indexer operands
  are FP8.  The oracle never quantises; it decodes the e4m3 bytes it is given
  (OCP FP8 E4M3: bias 7, no infinities, S.1111.111 is NaN) and multiplies by
  the per-row fp32 scale.
* same page, section "Stage 2: Fine-Grained Token Selection and Output
  Computation", selection equation S_t = TopK({I[t,s]}_{s<=t}, k); ties go to
  the lower position; the selected positions are returned in ascending order
  (the page's PyTorch listing sorts them "to preserve temporal order") and, as
  in that listing, k is clipped to the number of visible keys.
* same section, output equation u_{t,i} = sum_{s in S_t} softmax_s(A) W_UV c_s,
  here in absorbed form: the query already carries W_UK, so a logit is
  sm_scale * (q[t,i] . [c_s || k^R_s]) over the 576 (or d_c + d_R) latent
  dims and the output is the latent sum_s p_s c_s (width d_c).
* section "The Classical Multi-Head Latent Attention (MLA) Mechanism", logit
  equation A_{t,s,i}: the dense MLA that sparse MLA must equal when k covers
  every visible key, and the un-absorbed form used for the absorbed ==
  un-absorbed identity.

Every function is a direct transcription of its definition: no blocking, no
fusion, no reordering beyond one library matmul per contraction.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------

E4M3_EXP_BIAS = 7


def _e4m3_value(code: int) -> float:
    """Value of one OCP FP8 E4M3 code.

    Bit layout S EEEE MMM.  Exponent field 0 is subnormal:
    (-1)^S * 2^(1-7) * M/8.  Otherwise (-1)^S * 2^(E-7) * (1 + M/8), except
    E = 15, M = 7, which is NaN (the format has no infinities).
    """
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return sign * 2.0 ** (1 - E4M3_EXP_BIAS) * (m / 8.0)
    return sign * 2.0 ** (e - E4M3_EXP_BIAS) * (1.0 + m / 8.0)


_E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3 byte codes to float64 (each code through _e4m3_value)."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64: the high half of a float32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def as_f64(x: np.ndarray, kind: str) -> np.ndarray:
    """Exact float64 value of a stored tensor: kind is 'f32', 'bf16' or 'e4m3'."""
    if kind == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if kind == "bf16":
        return bf16_decode(x)
    if kind == "e4m3":
        return e4m3_decode(x)
    raise ValueError(kind)


# ----------------------------------------------------------------------------
# Cache addressing: logical key position s of sequence b -> physical cache row
# ----------------------------------------------------------------------------

def physical_rows(seq: int, s: np.ndarray, cache: dict) -> np.ndarray:
    """Physical cache row of logical key positions ``s`` of sequence ``seq``.

    Paged cache: row = block_table[seq, s // page] * page + s % page.
    Contiguous cache: row = seq_start[seq] + s (seq_start absent: 0).
    """
    s = np.asarray(s, dtype=np.int64)
    bt = cache.get("block_table")
    if bt is not None:
        page = int(cache["page_size"])
        pages = np.asarray(bt)[seq, s // page].astype(np.int64)
        return pages * page + s % page
    start = cache.get("seq_start")
    base = 0 if start is None else int(np.asarray(start)[seq])
    return base + s


# ----------------------------------------------------------------------------
# Stage 1: lightning indexer
# ----------------------------------------------------------------------------

def indexer_row(q: np.ndarray, w: np.ndarray, k: np.ndarray) -> np.ndarray:
    """I[s] = sum_j w[j] * max(0, q[j] . k[s]) for one query row.

    q: [H_I, d_I] float64 (dequantised), w: [H_I], k: [n_keys, d_I]
    (dequantised).  Returns [n_keys] float64.
    """
    dots = k @ q.T                          # [n_keys, H_I]
    return np.maximum(dots, 0.0) @ w        # [n_keys]


def indexer_row_single_head(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """The page's single-head form ReLU(q . k / sqrt(d_I)); q: [d_I]."""
    d_i = q.shape[0]
    return np.maximum((k @ q) / math.sqrt(d_i), 0.0)


# ----------------------------------------------------------------------------
# Stage 2a: top-k selection
# ----------------------------------------------------------------------------

def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Positions of the k largest scores among the visible keys.

    Order keys by (-score, position) with a stable sort, keep the first
    min(k, n), return them ascending, padded with -1 to length k.  -0.0 and
    +0.0 compare equal, so equal scores keep the lower position.
    """
    n = scores.shape[0]
    pos = np.arange(n, dtype=np.int64)
    order = np.lexsort((pos, -np.asarray(scores, dtype=np.float64)))
    take = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int64)
    out[: take.shape[0]] = take
    return out


def kth_score(scores: np.ndarray, k: int) -> float:
    """tau: the k-th largest visible score (the last one the selection keeps)."""
    n = scores.shape[0]
    if n == 0:
        return float("nan")
    srt = np.sort(np.asarray(scores, dtype=np.float64))[::-1]
    return float(srt[min(k, n) - 1])


# ----------------------------------------------------------------------------
# Stage 2b: sparse MLA (absorbed / MQA form)
# ----------------------------------------------------------------------------

def sparse_mla_row(q: np.ndarray, kv: np.ndarray, d_c: int, sm_scale: float):
    """Absorbed MLA over the selected latent rows of one query row.

    q: [H, D] (D = d_c + d_R), kv: [n_sel, D] rows c_s || k^R_s.
    z[i,s] = sm_scale * q[i] . kv[s];  p = softmax_s(z);
    o[i] = sum_s p[i,s] * c_s  (c_s = kv[s, :d_c]);  lse[i] = log sum_s e^z.
    Returns (o [H, d_c], lse [H]).  With no selected rows the output is 0 and
    lse is -inf.
    """
    h = q.shape[0]
    if kv.shape[0] == 0:
        return np.zeros((h, d_c)), np.full(h, -np.inf)
    z = sm_scale * (q @ kv.T)                       # [H, n_sel]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    den = e.sum(axis=1, keepdims=True)
    p = e / den
    o = p @ kv[:, :d_c]
    lse = (m + np.log(den))[:, 0]
    return o, lse


def unabsorbed_mla_row(q_nope, q_rope, c, k_rope, w_uk, w_uv):
    """MLA as the pages write it, with explicit up-projections.

    q_nope: [H, d_h], q_rope: [H, d_R], c: [n, d_c], k_rope: [n, d_R],
    w_uk: [H, d_h, d_c], w_uv: [H, d_v, d_c].
    A[i,s] = (q_i . (W_UK,i c_s) + q^R_i . k^R_s) / sqrt(d_h + d_R);
    u_i = sum_s softmax_s(A[i]) W_UV,i c_s.   Returns u: [H, d_v].
    """
    h, d_h = q_nope.shape
    d_r = q_rope.shape[1]
    out = []
    for i in range(h):
        keys = c @ w_uk[i].T                         # [n, d_h]
        a = (keys @ q_nope[i] + k_rope @ q_rope[i]) / math.sqrt(d_h + d_r)
        a = a - a.max()
        p = np.exp(a) / np.exp(a).sum()
        vals = c @ w_uv[i].T                         # [n, d_v]
        out.append(p @ vals)
    return np.stack(out)


# ----------------------------------------------------------------------------
# Whole path, row by row
# ----------------------------------------------------------------------------

def dequant_queries(inp: dict, t: int) -> np.ndarray:
    """Indexer query of row t as float64 [H_I, d_I] (e4m3 * per-head scale)."""
    q = as_f64(inp["q_idx"][t], inp["idx_dtype"])
    if inp.get("q_scale") is not None:
        q = q * np.asarray(inp["q_scale"][t], dtype=np.float32).astype(np.float64)[:, None]
    return q


def dequant_keys(inp: dict, rows: np.ndarray) -> np.ndarray:
    """Indexer keys at physical rows as float64 [n, d_I] (e4m3 * per-token scale)."""
    k = as_f64(inp["k_idx"][rows], inp["idx_dtype"])
    if inp.get("k_scale") is not None:
        k = k * np.asarray(inp["k_scale"][rows], dtype=np.float32).astype(np.float64)[:, None]
    return k


def row_scores(inp: dict, t: int) -> np.ndarray:
    """Indexer scores I[t, 0:klen[t]] of one row, float64."""
    seq = int(inp["row_seq"][t])
    klen = int(inp["row_klen"][t])
    rows = physical_rows(seq, np.arange(klen), inp["cache"])
    k = dequant_keys(inp, rows)
    q = dequant_queries(inp, t)
    w = np.asarray(inp["w"][t], dtype=np.float32).astype(np.float64)
    return indexer_row(q, w, k)


def row_attention(inp: dict, t: int, idx: np.ndarray):
    """Sparse MLA of row t over the selected logical positions idx (-1 = none)."""
    seq = int(inp["row_seq"][t])
    sel = np.asarray(idx, dtype=np.int64)
    sel = sel[sel >= 0]
    rows = physical_rows(seq, sel, inp["cache"])
    kv = as_f64(inp["latent"][rows], inp["mla_dtype"])
    q = as_f64(inp["q"][t], inp["mla_dtype"])
    return sparse_mla_row(q, kv, int(inp["d_c"]), float(inp["sm_scale"]))


def dsa_forward_rows(inp: dict, rows, topk: int | None = None):
    """Run the three stages for the listed rows.

    Returns dict with per-row lists: scores (float64 [klen]), idx (int64 [k]),
    out (float64 [H, d_c]), lse (float64 [H]).
    """
    k = int(inp["topk"] if topk is None else topk)
    res = {"rows": list(rows), "scores": [], "idx": [], "out": [], "lse": []}
    for t in rows:
        sc = row_scores(inp, t)
        sel = topk_row(sc, k)
        o, lse = row_attention(inp, t, sel)
        res["scores"].append(sc)
        res["idx"].append(sel)
        res["out"].append(o)
        res["lse"].append(lse)
    return res
