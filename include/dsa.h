/*
 * dsa.h - C ABI of the B200 DeepSeek Sparse Attention (DSA) forward path.
 *
 * The path has three stages, as the DSA description defines them
 * ("DeepSeek Sparse Attention DSA Architecture Guide"):
 *
 *   1. lightning indexer ("Stage 1: The Lightning Indexer", index-score
 *      equation, generalised to H_I weighted heads):
 *          I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]),   s < klen[t]
 *      with q_I and k_I in FP8 e4m3 and one fp32 scale per query head row and
 *      per key token ("Native FP8 Precision").
 *   2. top-k ("Stage 2: Fine-Grained Token Selection and Output Computation",
 *      selection equation S_t = TopK(I[t,:], k)): the k largest scores, ties
 *      to the lower position, returned in ascending position order and padded
 *      with -1 when klen < k (the page's listing clips k to the sequence and
 *      sorts the positions to keep temporal order).
 *   3. sparse MLA in absorbed form (same section, output equation; logit of
 *      "The Classical Multi-Head Latent Attention (MLA) Mechanism"):
 *          z[i,s] = sm_scale * q[t,i] . (c_s || kR_s),  s in S_t
 *          out[t,i] = sum_s softmax_s(z[i,:]) * c_s,     lse[t,i] = log sum_s e^z
 *      The query already carries W_UK; W_UV and the output projection are
 *      dense GEMMs after this path and are not part of it.
 *
 * Conventions (every entry point):
 *  - All pointers except the dsa_* descriptor structs are DEVICE pointers owned
 *    by the caller.  The library allocates no device memory: scratch comes from
 *    the caller's workspace `ws` (size from dsa_workspace_size, 256-byte
 *    aligned), or for dsa_sparse_mla_fwd_noalloc from a static array inside
 *    the library.  Descriptor structs are read on the host during the call only.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  No entry point synchronises, except
 *    dsa_read_device_status.
 *  - The return code reports what the host can see: null or misaligned
 *    pointers, unsupported shapes, a workspace that is too small, CUDA launch
 *    errors.  Errors found on the device (a block-table entry outside
 *    [0, num_pages), a bounded wait that ran out) are recorded in a status
 *    word inside `ws`; read it with dsa_read_device_status.  Nothing traps.
 *  - Results are deterministic run to run (no floating-point atomics).
 *  - Row t of a call sees keys s in [0, klen[t]) of sequence row_seq[t].
 *    Prefill row t of a sequence sees klen = t + 1; decode row j of n_q new
 *    rows of a sequence with ctx cached tokens sees klen = ctx - (n_q - 1 - j).
 *  - Top-k indices are logical positions within the sequence.  Only the
 *    attention stage translates them through the block table.
 */
#ifndef DSA_B200_DSA_H_
#define DSA_B200_DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so callers need no CUDA headers. */
typedef struct CUstream_st* dsa_stream_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, bad layout */
  DSA_ERR_UNSUPPORTED = 2,   /* shape/dtype combination the library does not run */
  DSA_ERR_CUDA = 3,          /* a CUDA call or kernel launch failed               */
  DSA_ERR_OUT_OF_RANGE = 4,  /* device: block-table entry outside [0, num_pages)   */
  DSA_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel ran out     */
  DSA_ERR_WORKSPACE = 6      /* ws is NULL, misaligned or smaller than required    */
} dsa_status;

typedef enum {
  DSA_F32 = 0,
  DSA_BF16 = 1,
  DSA_FP8_E4M3 = 2
} dsa_dtype;

/* Which kernels to run.  AUTO picks the tensor-core kernels (tcgen05) for the
 * FP8 indexer with H_I*group <= 256, d_I = 128, and for bf16 MLA with
 * H = 128, d_c = 512, d_r = 64; everything else runs the SIMT kernels.  With
 * AUTO, dsa_decode_step and dsa_forward fuse the indexer and top-k when the
 * tensor-core indexer runs and q_group <= 2: the indexer's epilogue also
 * builds each row's histogram of its scores' top 12 order-preserving key bits
 * (the first pass of the radix selection), and top-k starts from it
 * ("DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 1: The
 * Lightning Indexer", item "Separable Streaming Top-k": the selection is
 * folded into the indexer's pass).  STAGED runs the same tensor-core kernels
 * without that fusion (top-k builds its own histogram), as dsa_topk does. */
typedef enum {
  DSA_ALGO_AUTO = 0,
  DSA_ALGO_SIMT = 1,
  DSA_ALGO_STAGED = 2
} dsa_algo;

/* Problem dimensions. */
typedef struct {
  int32_t n_idx_heads;   /* H_I: indexer heads                          */
  int32_t d_idx;         /* d_I: indexer head width (bytes per e4m3 key) */
  int32_t n_heads;       /* H: MLA query heads                          */
  int32_t d_c;           /* latent width = value width                  */
  int32_t d_r;           /* decoupled RoPE key width                    */
  int32_t topk;          /* k, 1 <= k <= 2048                           */
  dsa_dtype idx_dtype;   /* DSA_FP8_E4M3 (scales required) or DSA_F32   */
  dsa_dtype mla_dtype;   /* DSA_BF16 or DSA_F32                         */
  float sm_scale;        /* softmax scale, e.g. 1/sqrt(d_c + d_r)       */
  dsa_algo algo;
} dsa_dims;

/* Query rows.  Any mix of sequences. */
typedef struct {
  int32_t num_rows;          /* T >= 0                                          */
  const int32_t* row_seq;    /* [T] device: sequence of row t, in [0, num_seqs)  */
  const int32_t* row_klen;   /* [T] device: visible keys of row t, in [0, max_klen] */
  int32_t max_klen;          /* host: upper bound of row_klen (sizes the grid)   */
  int32_t q_group;           /* 1, 2 or 4: rows [g*q_group, (g+1)*q_group) belong
                                to one sequence; the indexer scores such a group
                                against one pass over its keys.  A group that
                                mixes sequences is reported as
                                DSA_ERR_INVALID_ARG in the device status word.  */
} dsa_rows;

/* The two caches of the layer: the latent cache (c || kR per token) and the
 * indexer key cache (k_I per token + its fp32 scale).  Physical row of logical
 * key s of sequence b:
 *   paged (block_table != NULL): block_table[b*max_pages_per_seq + s/page_size]
 *                                * page_size + s % page_size
 *   contiguous:                  seq_start[b] + s   (seq_start NULL: s)        */
typedef struct {
  const void* latent;         /* [num_tokens, d_c + d_r] bf16 | f32, row-major  */
  const void* idx_k;          /* [num_tokens, d_idx] e4m3 | f32, row-major      */
  const float* idx_k_scale;   /* [num_tokens] (required for e4m3, else NULL)     */
  const int32_t* seq_start;   /* [num_seqs] or NULL (contiguous layout)          */
  const int32_t* block_table; /* [num_seqs, max_pages_per_seq] or NULL           */
  int32_t page_size;          /* paged: tokens per page, a multiple of 64        */
  int32_t max_pages_per_seq;  /* paged: row stride of block_table                */
  int32_t num_seqs;
  int64_t num_tokens;         /* rows of latent / idx_k (paged: num_pages*page)  */
} dsa_cache;

typedef enum {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_MLA = 2,
  DSA_OP_DECODE_STEP = 3,
  DSA_OP_FORWARD = 4,
  DSA_OP_CACHE_APPEND = 5,
  DSA_OP_INDEXER_KL = 6,
  DSA_OP_INDEXER_BACKWARD = 7
} dsa_op;

/* Human-readable name of a status code (static storage). */
const char* dsa_status_string(dsa_status s);

/* Text of the last host-side error on the calling thread ("" if none). */
const char* dsa_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int32_t dsa_version(void);

/* Bytes of workspace `op` needs for these dimensions and rows (host only; it
 * reads the current device's SM count, which sets the decode key splits, and
 * uses 148 when no device is present).  Returns 0 for invalid arguments.
 * DSA_OP_CACHE_APPEND needs only the status block; `rows` may be NULL for it. */
size_t dsa_workspace_size(const dsa_dims* dims, const dsa_rows* rows, dsa_op op);

/* Zero the workspace `ws` (ws_bytes bytes, async on stream): the device status
 * word at its head and, for dsa_decode_step and dsa_forward, the per-row
 * score histograms of the fused indexer -> top-k, which every top-k leaves
 * zeroed for the next call.  Call it once before the first use of a
 * workspace, and again after a call that recorded a device error (a call cut
 * short may leave histograms behind).  A workspace may then serve calls of
 * other ops or other rows in any order: the library records, per workspace
 * address on the host, which bytes its calls left zeroed, and a call whose
 * histogram region is not among them clears it first (one memset).  A fused
 * call on a workspace never initialised may select wrongly (its histograms
 * hold other counts) but accesses nothing out of bounds. */
dsa_status dsa_workspace_init(void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Synchronise `stream`, copy the device status word of `ws` to *status_out
 * (one of dsa_status) and clear it.  *detail_out (may be NULL) receives the
 * row or page that raised it, or -1. */
dsa_status dsa_read_device_status(void* ws, dsa_stream_t stream, int32_t* status_out,
                                  int32_t* detail_out);

/* Kernel trace: every kernel sets its bit in the workspace's status block when
 * it runs, so a caller (or a test) can tell which implementation ran. */
#define DSA_KERNEL_INDEXER_SIMT 0x01u
#define DSA_KERNEL_INDEXER_TC   0x02u   /* tcgen05 FP8 indexer */
#define DSA_KERNEL_TOPK         0x04u
#define DSA_KERNEL_MLA_SIMT     0x08u
#define DSA_KERNEL_MLA_TC       0x10u   /* tcgen05 bf16 sparse MLA */
#define DSA_KERNEL_MLA_COMBINE  0x20u   /* split-K combine of the sparse MLA (inside its kernel) */
#define DSA_KERNEL_CACHE_APPEND 0x40u   /* fused FP8 quantise + cache write */
#define DSA_KERNEL_OUT_PROJ     0x80u   /* tcgen05 output projection GEMM */
#define DSA_KERNEL_OUT_PROJ_REDUCE 0x100u   /* split-K sum of the W_out product */
#define DSA_KERNEL_WARMUP       0x200u   /* indexer warm-up: KL and backward kernels */

/* Synchronise `stream`, return the kernel trace of `ws` in *mask_out and clear it. */
dsa_status dsa_read_kernel_trace(void* ws, dsa_stream_t stream, uint32_t* mask_out);

/* Per-stage timing of dsa_decode_step on the calling thread.  `events` holds
 * n_events = 4 cudaEvent_t handles created by the caller; each later
 * dsa_decode_step on this thread records them on its stream before the
 * indexer, after the indexer, after top-k and after the attention stage.
 * n_events = 0 turns this off.  The handles are not owned by the library. */
dsa_status dsa_set_stage_events(void* const* events, int32_t n_events);

/* Profiling trace on the calling thread.  When `dev_buf` (device memory, at
 * least 896 int64 = 7168 bytes, zeroed by the caller) is set, the tensor-core
 * kernels record clock64() stamps of their pipeline events there, each in its
 * own region: int64 [0, 512) the sparse-MLA kernel's first CTA pair
 * ([2 CTAs][8 events][32 blocks]: decoded, after the max barrier, S issued,
 * PV issued, S read by the softmax, peer logits arrived, P stored, exp done),
 * [512, 640) top-k's first cluster ([8 CTAs][16 events], phase ends; the
 * cluster kernel only), and
 * [640, 896) the indexer's CTA 0 ([8 events][32 tiles]: stage free, TMA
 * issued, MMA ready, MMA committed, accumulator ready, key data landed,
 * accumulator loaded, scores stored).  Stamps of one SM's clock; compare
 * within a region.  dev_buf = NULL turns it off.  For performance analysis
 * only. */
dsa_status dsa_set_trace_buffer(void* dev_buf, size_t bytes);

/* Fault injection, for tests of the failure paths only (never set it in
 * production).  Every wait inside the kernels is bounded: after a number of
 * polls it records DSA_ERR_TIMEOUT (detail = the wait's site) in the device
 * status word and the kernel winds down and returns, with every asynchronous
 * copy and tensor-core operation it started complete.  On the calling host
 * thread, later launches use `spin_limit` polls per wait (0 = the built-in
 * limit) and inject the faults in `faults`:
 *   DSA_FAULT_INDEXER_ACC_RELEASE  the tensor-core indexer's epilogue never
 *       releases its accumulators, so its MMA issuer's wait for a free
 *       accumulator runs out (and then the epilogue's and the producer's
 *       waits for tiles that are never computed).
 * Returns DSA_ERR_INVALID_ARG for unknown fault bits.  (0, 0) switches it off. */
#define DSA_FAULT_INDEXER_ACC_RELEASE 0x1u
dsa_status dsa_set_fault_injection(uint32_t spin_limit, uint32_t faults);

/* Stage 1: indexer scores.
 *   q_idx   [T, H_I, d_I] e4m3 | f32
 *   q_scale [T, H_I] fp32 (e4m3 only, else NULL): dequantised q = e4m3 * scale
 *   w       [T, H_I] fp32 head weights
 *   scores  [T, ld_scores] fp32 out; entries s >= klen[t] are left unspecified.
 *           ld_scores >= max_klen and a multiple of 4.
 * The scale factors are folded exactly: I = k_scale[s] * sum_j (w*q_scale)[t,j]
 * * ReLU(q8 . k8), since both scales are positive and ReLU is positively
 * homogeneous. */
dsa_status dsa_indexer_scores(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                              const void* q_idx, const float* q_scale, const float* w,
                              float* scores, int64_t ld_scores,
                              void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Stage 2: top-k selection.
 *   scores [T, ld_scores] fp32 (only s < klen[t] is read)
 *   idx    [T, topk] int32 out: ascending logical positions, -1 padded.
 * Comparison is on the fp32 value (-0.0 == +0.0); equal values go to the
 * lower position.  NaN scores are unsupported. */
dsa_status dsa_topk(const dsa_dims* dims, const dsa_rows* rows, const float* scores,
                    int64_t ld_scores, int32_t* idx, void* ws, size_t ws_bytes,
                    dsa_stream_t stream);

/* Stage 3: sparse absorbed MLA over the selected rows.
 *   q   [T, H, d_c + d_r] bf16 | f32
 *   idx [T, topk] int32 logical positions (entries < 0 are skipped; entries
 *       >= klen[t] are a caller error and are read as given)
 *   out [T, H, d_c] bf16 | f32 (same dtype as q)
 *   lse [T, H] fp32 natural-log sum of exp(z) (may be NULL); -inf and out = 0
 *       for a row with no selected key. */
dsa_status dsa_sparse_mla_fwd(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                              const void* q, const int32_t* idx, void* out, float* lse,
                              void* ws, size_t ws_bytes, dsa_stream_t stream);

/* dsa_sparse_mla_fwd without a caller workspace, for callers that cannot hand
 * out device memory.  The sparse attention pages have no counterpart of this
 * call: it is a deployment convenience.  Arguments, layouts and results are
 * those of dsa_sparse_mla_fwd, bit for bit (same kernels, same split plan).
 * Scratch: a file-scope static device array of 20 MiB (256-byte status block
 * + split-K partials) inside the library.  Nothing is allocated: no
 * cudaMalloc/cudaFree, no allocating library routine.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it; make that
 *     first call before any stream capture.  Later calls may be captured.
 *   - Each call clears the status block (cudaMemsetAsync on `stream`); the
 *     partials need no clearing, every split writes its own.  Device-side
 *     range errors are recorded there but cannot be read back through this
 *     call: use dsa_sparse_mla_fwd with a workspace for checked runs.
 *   - Every call on a device shares the one array, so calls that overlap
 *     (different streams, or host threads racing on one device) race on it
 *     and corrupt each other's partials.  Serialise them.
 * Returns DSA_ERR_WORKSPACE, with the sizes in dsa_last_error(), when the
 * split plan needs more than the 20 MiB (more rows x splits than the array
 * holds), and the argument errors of dsa_sparse_mla_fwd. */
dsa_status dsa_sparse_mla_fwd_noalloc(const dsa_dims* dims, const dsa_rows* rows,
                                      const dsa_cache* cache, const void* q, const int32_t* idx,
                                      void* out, float* lse, dsa_stream_t stream);

/* The three stages for a batch of decode rows (few rows per sequence), one
 * enqueue, no host synchronisation.  Scores and indices live in ws unless
 * dbg_scores [T, round_up(max_klen,128)] / dbg_idx [T, topk] are given, in
 * which case they are written there. */
dsa_status dsa_decode_step(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                           const void* q_idx, const float* q_scale, const float* w,
                           const void* q, void* out, float* lse,
                           float* dbg_scores, int32_t* dbg_idx,
                           void* ws, size_t ws_bytes, dsa_stream_t stream);

/* The three stages for any rows (prefill): rows are processed in chunks whose
 * score buffer fits the workspace; `idx_out` [T, topk] (may be NULL) receives
 * the selections. */
dsa_status dsa_forward(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                       const void* q_idx, const float* q_scale, const float* w,
                       const void* q, void* out, float* lse, int32_t* idx_out,
                       void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Cache append: the write that precedes the three stages of every decoding
 * step ("Sparse Attention Architectures for Long-Context Inference: Evolution
 * and Engineering Practices", section 6, item "Incremental inference
 * adaptation": the caches are updated with each step's new tokens), into the
 * paged caches of "Sparse Attention in Large Language Models: Architecture
 * Evolution and Engineering Practice", section 4, item "Memory Management and
 * KV Cache Optimization", with the indexer keys in FP8 ("DeepSeek Sparse
 * Attention DSA Architecture Guide", section "Stage 1: The Lightning
 * Indexer", item "Native FP8 Precision").  One kernel quantises and writes.
 *
 * Token n (0 <= n < n_new) goes to the physical row of logical position
 * tok_pos[n] of sequence tok_seq[n], through the map every other call reads:
 *   idx_k[row]       = E4M3(fl32(k_new[n, :] / s)),  s = fl32(amax_n / 448),
 *                      s = 1 when that is 0; E4M3 rounds to nearest, ties to
 *                      the even code, and saturates at +-448 (the OCP FP8
 *                      encoding; -0.0 and negatives that round to 0 give 0x80)
 *   idx_k_scale[row] = s
 *   latent[row]      = latent_new[n, :]   (bit copy)
 * With idx_dtype = DSA_F32 the key is copied and idx_k_scale is not used.
 *   tok_seq, tok_pos [n_new] int32, device
 *   k_new      [n_new, d_idx] fp32, device, 16-byte aligned; d_idx <= 512
 *   latent_new [n_new, d_c + d_r] in mla_dtype, device, 16-byte aligned
 * The caches that `cache` describes (latent, idx_k, idx_k_scale) are WRITTEN
 * here and must be writable device memory; the descriptor's const qualifiers
 * describe the other calls, which only read them.  Destinations must be
 * distinct within one call (two tokens with one destination race).
 * A token whose sequence is outside [0, num_seqs), whose position is negative
 * or beyond the block table's width, whose block-table entry is outside
 * [0, num_pages), or whose contiguous row is outside [0, num_tokens), is not
 * written and is recorded in the device status word as DSA_ERR_OUT_OF_RANGE
 * with detail n; a token whose key holds an infinity or NaN is not written
 * either, and is recorded as DSA_ERR_INVALID_ARG with detail n (the first
 * error of a launch wins).  The other tokens are written.
 * Contiguous layout: the library knows where each sequence's rows start
 * (seq_start) but not where they end, so the only range check is
 * [0, num_tokens).  A position past the end of sequence b's own rows is
 * written into the rows that follow them (the next sequence's, in the usual
 * layout) without an error: the caller keeps tok_pos[n] below the capacity of
 * its sequence.  The paged layout has no such hazard (a position beyond the
 * block table's width is refused).
 * ws: at least dsa_workspace_size(dims, NULL, DSA_OP_CACHE_APPEND) bytes (the
 * status block), zeroed once by dsa_workspace_init.  n_new = 0 launches
 * nothing. */
dsa_status dsa_cache_append(const dsa_dims* dims, const dsa_cache* cache, int32_t n_new,
                            const int32_t* tok_seq, const int32_t* tok_pos,
                            const float* k_new, const void* latent_new,
                            void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Output projection: the two GEMMs after the path that complete u_t
 * ("DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 2:
 * Fine-Grained Token Selection and Output Computation", output equation
 * u_{t,i} = sum_s softmax_s(.) W_{UV,i} c_s; W_{UV,i} does not depend on s, so
 * it applies once to the latent output o of dsa_sparse_mla_fwd; then the
 * output projection of the page's module, "End-to-End Implementation", over
 * the heads concatenated in order):
 *     u[t,i,:] = W_UV[i] o[t,i,:]                     (i < H)
 *     y[t,:]   = W_out [u[t,0,:]; u[t,1,:]; ...; u[t,H-1,:]]
 * bf16 operands, fp32 accumulation on the tensor cores; u is rounded to bf16
 * once and y is computed from that bf16 u, then rounded to bf16 once (a K
 * split adds its fp32 partials in a fixed order first). */
typedef struct {
  int32_t n_heads;   /* H                                                        */
  int32_t d_c;       /* latent width per head (the attention output), a multiple of 64 */
  int32_t d_v;       /* value head width after W_UV: a multiple of 32, at most 256,
                        with H * d_v a multiple of 64                             */
  int32_t d_model;   /* output width after W_out, a multiple of 32               */
} dsa_proj_dims;

/* Workspace bytes of dsa_output_projection for num_rows rows (host only; it
 * reads the current device's SM count, which sets the K splits of small
 * batches).  Returns 0 for invalid dimensions. */
size_t dsa_output_projection_ws_size(const dsa_proj_dims* dims, int32_t num_rows);

/*   o     [T, H, d_c] bf16: the latent attention output (dsa_sparse_mla_fwd's out)
 *   w_uv  [H, d_v, d_c] bf16, row-major: W_UV[i] is a d_v x d_c matrix
 *   w_out [d_model, H*d_v] bf16, row-major: column i*d_v + v multiplies u[t,i,v]
 *   u     [T, H, d_v] bf16 out (the per-head values, kept for the caller)
 *   y     [T, d_model] bf16 out
 * All device pointers, 16-byte aligned, owned by the caller; u and y must not
 * overlap the inputs.  ws: dsa_output_projection_ws_size bytes, 256-byte
 * aligned (status block, then split-K partials); zero its status block once
 * with dsa_workspace_init.  A bounded wait that runs out is recorded there
 * (DSA_ERR_TIMEOUT).  T = 0 launches nothing. */
dsa_status dsa_output_projection(const dsa_proj_dims* dims, int32_t num_rows, const void* o,
                                 const void* w_uv, const void* w_out, void* u, void* y,
                                 void* ws, size_t ws_bytes, dsa_stream_t stream);

/* Indexer warm-up ("DeepSeek Sparse Attention DSA Architecture Guide",
 * section "Training Mechanics: Dense Warm-Up and KL Alignment", Phase 1): the
 * indexer learns to match the dense attention.  The teacher p_t of query row
 * t is the dense attention probabilities of the row summed over heads and
 * normalised over its visible keys (so it sums to 1); the loss is
 * L^I = sum_t KL(p_t || softmax(I_t)).
 *
 * dsa_indexer_kl: for every row t, over s < klen[t],
 *     loss[t]    = sum_s p[t,s] (log p[t,s] - log softmax(I[t,:])_s)   (0 log 0 = 0)
 *     grad[t,s]  = softmax(I[t,:])_s - p[t,s]        ( = dL/dI[t,s] )
 *   scores  [T, ld_scores] fp32, e.g. dsa_indexer_scores' output
 *   teacher [T, ld_teacher] fp32, p[t,s] >= 0, summing to 1 over s < klen[t]
 *   grad    [T, ld_grad] fp32 out (entries s >= klen[t] untouched); loss [T] fp32 out
 * fp32 arithmetic (expf/logf).  ws: the status block
 * (dsa_workspace_size(..., DSA_OP_INDEXER_KL)).  dims may be NULL. */
dsa_status dsa_indexer_kl(const dsa_rows* rows, const float* scores, int64_t ld_scores,
                          const float* teacher, int64_t ld_teacher, float* grad, int64_t ld_grad,
                          float* loss, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* dsa_indexer_backward: given g = dL/dI (e.g. dsa_indexer_kl's grad), the
 * gradients of I[t,s] = sum_j w[t,j] ReLU(q[t,j] . k[s]) with respect to the
 * dequantised operands (e4m3 code times its scale; the FP8 cast is not
 * differentiated):
 *     dw[t,j]   = sum_{s<klen[t]} g[t,s] ReLU(q[t,j] . k[s])
 *     dq[t,j,:] = sum_{s<klen[t]} g[t,s] w[t,j] [q[t,j] . k[s] > 0] k[s]
 *     dk[s,:]   = sum over the rows t of s's sequence with klen[t] > s of
 *                 sum_j g[t,s] w[t,j] [q[t,j] . k[s] > 0] q[t,j]
 *   q_idx, q_scale, w, cache: as dsa_indexer_scores (H_I = 64, d_I = 128)
 *   grad [T, ld_grad] fp32
 *   dq [T, H_I, d_I], dw [T, H_I] fp32 out
 *   dk [num_tokens, d_I] fp32 out, indexed by the key's physical cache row;
 *      only rows that some query row of the call sees are written
 * The ReLU mask is decided exactly (the dot product of the e4m3 codes is exact
 * in fp64), the rest is fp32 with every sum in a fixed order (deterministic).
 * CUDA-core kernels.  ws: dsa_workspace_size(dims, rows,
 * DSA_OP_INDEXER_BACKWARD) bytes (status block + per-row partial sums). */
dsa_status dsa_indexer_backward(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                                const void* q_idx, const float* q_scale, const float* w,
                                const float* grad, int64_t ld_grad, float* dq, float* dw, float* dk,
                                void* ws, size_t ws_bytes, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_DSA_H_ */
