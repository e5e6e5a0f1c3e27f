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
* same page, item "Native FP8 Precision", with "Sparse Attention in Large
  Language Models: Architecture Evolution and Engineering Practice", section 4,
  item "Memory Management and KV Cache Optimization" (paged caches), and
  "Sparse Attention Architectures for Long-Context Inference: Evolution and
  Engineering Practices", section 6, item "Incremental inference adaptation"
  (each decoding step writes its new tokens into the caches): the cache
  append.  New indexer keys are quantised to e4m3 with one fp32 scale per
  token (an encoder written from the OCP definition: nearest value, ties to
  the even code, saturating at +-448) and written with their latent rows at
  the rows the block table gives.
* same section, output equation, with the page's "End-to-End Implementation"
  module: the output projection after the path, u_{t,i} = W_UV,i o_{t,i} per
  head (W_UV,i is constant in s, so it moves out of the softmax sum) and
  y_t = W_out [u_{t,1}; ...; u_{t,H}].
* section "Training Mechanics: Dense Warm-Up and KL Alignment", Phase 1: the
  teacher distribution (dense attention probabilities summed over heads and
  normalised over the keys), the KL loss of the indexer's softmax against it,
  and the backward of that loss through the indexer to q_I, w and k_I.
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


# ----------------------------------------------------------------------------
# Cache append: FP8 quantisation of new indexer keys, then the paged write
# ----------------------------------------------------------------------------
#
# "DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 1: The
# Lightning Indexer", item "Native FP8 Precision": indexer keys are stored as
# 8-bit floats.  "Sparse Attention in Large Language Models: Architecture
# Evolution and Engineering Practice", section 4, item "Memory Management and
# KV Cache Optimization": the caches are paged.  "Sparse Attention
# Architectures for Long-Context Inference: Evolution and Engineering
# Practices", section 6, item "Incremental inference adaptation": every
# decoding step writes the new tokens into the caches before attending.
# The pages fix neither the scale rule nor the rounding; the reading taken
# here is one fp32 scale per token, s = amax / 448 (1 when that is 0), and
# code = E4M3(k / s) with k / s in fp32 and one round-to-nearest-even,
# saturating at +-448.

E4M3_MAX = 448.0          # largest finite E4M3 magnitude, 2^8 * (1 + 6/8)
E4M3_MIN_EXP = 1 - E4M3_EXP_BIAS   # exponent of the smallest normal, -6
E4M3_MANT_BITS = 3


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 code of each (finite) value: round to nearest, ties to
    the even code, magnitudes above 448 saturate to 448; the sign bit is the
    value's sign bit (so -0.0 and negatives that round to zero give 0x80).

    In the binade [2^e, 2^(e+1)), e >= -6, the representable magnitudes are
    the multiples of 2^(e-3); below 2^-6 (the subnormals) the multiples of
    2^-9.  The nearest multiple is the rounded quotient, exact in float64.
    """
    y = np.asarray(y, dtype=np.float64)
    if not np.all(np.isfinite(y)):
        raise ValueError("e4m3_encode: non-finite input")
    a = np.abs(y)
    _, ex = np.frexp(a)                         # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, E4M3_MIN_EXP)        # floor(log2 a), clamped at the subnormals
    quantum = np.ldexp(1.0, e - E4M3_MANT_BITS)
    v = np.rint(a / quantum) * quantum          # np.rint: half to even
    v = np.minimum(v, E4M3_MAX)
    # code of the magnitude v
    _, vex = np.frexp(v)
    ve = vex - 1
    normal = v >= 2.0 ** E4M3_MIN_EXP
    e_field = np.where(normal, ve + E4M3_EXP_BIAS, 0)
    mant = np.where(normal, v / np.ldexp(1.0, ve) - 1.0, v / 2.0 ** E4M3_MIN_EXP) * 8.0
    mag = (e_field.astype(np.int64) << 3) | mant.astype(np.int64)
    sign = np.signbit(y).astype(np.int64) << 7
    return (sign | mag).astype(np.uint8)


def quantise_keys(k: np.ndarray):
    """Per-token FP8 quantisation of indexer keys k [n, d_I] (float32).

    s[n] = fl32(amax_n / 448), replaced by 1 when it is 0 (an all-zero key, or
    an amax so small that the quotient underflows); codes = E4M3(fl32(k / s)).
    Returns (codes uint8 [n, d_I], s float32 [n]).  Non-finite keys raise.
    """
    k = np.asarray(k, dtype=np.float32)
    if not np.all(np.isfinite(k)):
        raise ValueError("quantise_keys: non-finite key")
    amax = np.max(np.abs(k), axis=1) if k.shape[1] else np.zeros(k.shape[0], np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    y = (k / s[:, None]).astype(np.float32)
    return e4m3_encode(y), s


def append_destination(seq: int, pos: int, cache: dict, num_seqs: int, num_tokens: int):
    """Physical row that token (seq, pos) is written to, or None when the
    sequence, the position, the block-table slot or the page is out of range."""
    if not (0 <= seq < num_seqs) or pos < 0:
        return None
    bt = cache.get("block_table")
    if bt is not None:
        page = int(cache["page_size"])
        bt = np.asarray(bt)
        if pos // page >= bt.shape[1]:
            return None
        p = int(bt[seq, pos // page])
        if not (0 <= p < num_tokens // page):
            return None
    row = int(physical_rows(seq, np.array([pos]), cache)[0])
    return row if 0 <= row < num_tokens else None


def cache_append(inp: dict, num_seqs: int, tok_seq, tok_pos, k_new, latent_new):
    """Write new tokens into copies of the caches of ``inp`` (num_seqs sequences).

    Token n goes to physical row append_destination(tok_seq[n], tok_pos[n]):
    its indexer key quantised by quantise_keys (e4m3 caches) or copied (f32
    caches), its scale, and its latent row c || k^R copied bit for bit.  A
    token whose destination is out of range, or whose key is not finite, is
    not written and is listed in the returned ``bad`` set.  Destinations must
    be distinct.  Returns (k_idx, k_scale, latent, bad).
    """
    k_idx = np.array(inp["k_idx"], copy=True)
    k_scale = None if inp.get("k_scale") is None else np.array(inp["k_scale"], copy=True)
    latent = np.array(inp["latent"], copy=True)
    cache = inp["cache"]
    num_tokens = latent.shape[0]
    k_new = np.asarray(k_new, dtype=np.float32)
    bad, seen = set(), set()
    for n in range(len(tok_seq)):
        row = append_destination(int(tok_seq[n]), int(tok_pos[n]), cache, num_seqs, num_tokens)
        if row is None or not np.all(np.isfinite(k_new[n])):
            bad.add(n)
            continue
        assert row not in seen, "two appended tokens share a destination"
        seen.add(row)
        if inp["idx_dtype"] == "e4m3":
            codes, s = quantise_keys(k_new[n:n + 1])
            k_idx[row] = codes[0]
            k_scale[row] = s[0]
        else:
            k_idx[row] = k_new[n]
        latent[row] = latent_new[n]
    return k_idx, k_scale, latent, bad


# ----------------------------------------------------------------------------
# Output projection: W_UV per head, then W_out over the concatenated heads
# ----------------------------------------------------------------------------
#
# "DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 2:
# Fine-Grained Token Selection and Output Computation", output equation:
# u_{t,i} = sum_s softmax_s(.) W_{UV,i} c_s.  W_{UV,i} does not depend on s, so
# u_{t,i} = W_{UV,i} o_{t,i} with o_{t,i} = sum_s softmax_s(.) c_s, the latent
# output of the sparse attention.  The page's module ("End-to-End
# Implementation") then concatenates the heads in head order and applies its
# output projection w_out.

def output_projection_row(o: np.ndarray, w_uv: np.ndarray, w_out: np.ndarray):
    """o [H, d_c], w_uv [H, d_v, d_c], w_out [d_model, H*d_v] (float64).
    u[i] = W_UV[i] @ o[i];  y = W_out @ [u[0]; u[1]; ...; u[H-1]].
    Returns (u [H, d_v], y [d_model])."""
    u = np.einsum("ivc,ic->iv", w_uv, o)
    y = w_out @ u.reshape(-1)
    return u, y


# ----------------------------------------------------------------------------
# Indexer warm-up: KL loss against the dense attention, and its backward
# ----------------------------------------------------------------------------
#
# "DeepSeek Sparse Attention DSA Architecture Guide", section "Training
# Mechanics: Dense Warm-Up and KL Alignment", "Phase 1: Dense Warm-Up via
# Teacher-Student Distillation": the teacher distribution of row t is the
# dense attention probabilities summed over the heads and normalised over the
# visible keys, p_{t,s} = sum_i A_{t,s,i} / sum_{s'} sum_i A_{t,s',i}, and the
# indexer minimises L^I = sum_t KL(p_{t,:} || Softmax(I_{t,:})).  Only the
# indexer's inputs (its queries, keys and head weights) receive gradients.

def dense_attention_probs(q: np.ndarray, kv: np.ndarray, sm_scale: float) -> np.ndarray:
    """A[i, s] = softmax_s(sm_scale * q[i] . kv[s]) over all given keys (the
    row's visible keys), q [H, D], kv [n, D].  Returns [H, n]."""
    z = sm_scale * (q @ kv.T)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def teacher_distribution(a: np.ndarray) -> np.ndarray:
    """p[s] = sum_i A[i, s] / sum_s' sum_i A[i, s'] for one row, A [H, n]."""
    tot = a.sum(axis=0)
    return tot / tot.sum()


def indexer_kl_row(p: np.ndarray, scores: np.ndarray):
    """KL(p || softmax(I)) of one row and its gradient with respect to I.

    KL = sum_s p_s (log p_s - log softmax(I)_s), with 0 log 0 = 0.  Since
    sum_s p_s = 1, dKL/dI_s = softmax(I)_s - p_s.  Returns (kl, grad [n])."""
    p = np.asarray(p, dtype=np.float64)
    scores = np.asarray(scores, dtype=np.float64)
    m = scores.max()
    log_z = m + np.log(np.exp(scores - m).sum())
    log_q = scores - log_z
    nz = p > 0
    kl = float(np.sum(p[nz] * (np.log(p[nz]) - log_q[nz])))
    return kl, np.exp(log_q) - p


def indexer_backward_row(q: np.ndarray, w: np.ndarray, k: np.ndarray, g: np.ndarray, on=None):
    """Backward of I[s] = sum_j w[j] ReLU(q[j] . k[s]) for one row, given
    g[s] = dL/dI[s].  q [H_I, d_I], w [H_I], k [n, d_I], g [n].  ReLU's
    derivative is 1 where its argument is > 0 and 0 elsewhere (0 at 0).
    `on` [n, H_I] (optional) gives that decision, [q[j] . k[s] > 0], taken
    exactly elsewhere (for FP8 operands: the sign of the dot product of the
    codes, as the scales are positive); by default it is taken from the
    float64 dot products here.
    Returns (dq [H_I, d_I], dw [H_I], dk [n, d_I])."""
    d = k @ q.T                               # [n, H_I]
    on = (d > 0).astype(np.float64) if on is None else np.asarray(on, dtype=np.float64)
    dw = np.maximum(d, 0.0).T @ g             # [H_I]
    gd = (g[:, None] * on) * w[None, :]       # dL/d(q_j . k_s), [n, H_I]
    dq = gd.T @ k                             # [H_I, d_I]
    dk = gd @ q                               # [n, d_I]
    return dq, dw, dk
