// api.cu - the C ABI of the DSA forward path: argument checks, workspace
// planning, kernel selection and launches.  No entry point allocates device
// memory; only dsa_read_device_status and dsa_read_kernel_trace synchronise.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "dsa_kernels.cuh"

namespace dsa {

static thread_local char g_err[512] = "";
static thread_local cudaEvent_t g_stage_ev[4] = {nullptr, nullptr, nullptr, nullptr};
static thread_local int g_n_stage_ev = 0;

static thread_local long long* g_trace = nullptr;
static thread_local uint32_t g_fault_spin = 0, g_fault_inject = 0;

static void stage_event(int i, cudaStream_t s) {
  if (g_n_stage_ev == 4 && g_stage_ev[i] != nullptr) cudaEventRecord(g_stage_ev[i], s);
}

long long* trace_buffer() { return g_trace; }
uint32_t fault_spin_limit() { return g_fault_spin ? g_fault_spin : kSpinLimit; }
uint32_t fault_inject() { return g_fault_inject; }

dsa_status set_smem_limit_once(const void* fn, size_t bytes, std::atomic<bool> (&done)[kMaxDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_error("no current CUDA device");
    return DSA_ERR_CUDA;
  }
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && done[dev].load(std::memory_order_acquire)) return DSA_OK;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) {
    set_error("cannot allow %zu bytes of shared memory: %s", bytes, cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  if (cached) done[dev].store(true, std::memory_order_release);
  return DSA_OK;
}

int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

namespace {

constexpr size_t kAlign = 256;
constexpr int kForwardChunkRows = 512;
constexpr int kWarmupChunkKeys = 512;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int64_t scores_ld(int max_klen) { return ((int64_t)max_klen + 127) / 128 * 128; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define CHECK_ARG(cond, ...)          \
  do {                                \
    if (!(cond)) {                    \
      set_error(__VA_ARGS__);         \
      return DSA_ERR_INVALID_ARG;     \
    }                                 \
  } while (0)

dsa_status check_dims(const dsa_dims* d) {
  CHECK_ARG(d != nullptr, "dims is NULL");
  CHECK_ARG(d->n_idx_heads > 0 && d->d_idx > 0 && d->n_heads > 0 && d->d_c > 0 && d->d_r >= 0,
            "non-positive dimension");
  CHECK_ARG(d->topk >= 1 && d->topk <= 2048, "topk %d outside [1, 2048]", d->topk);
  CHECK_ARG(d->idx_dtype == DSA_FP8_E4M3 || d->idx_dtype == DSA_F32, "idx_dtype must be e4m3 or f32");
  CHECK_ARG(d->mla_dtype == DSA_BF16 || d->mla_dtype == DSA_F32, "mla_dtype must be bf16 or f32");
  CHECK_ARG(d->algo == DSA_ALGO_AUTO || d->algo == DSA_ALGO_SIMT || d->algo == DSA_ALGO_STAGED,
            "unknown algo");
  CHECK_ARG(d->sm_scale > 0.f, "sm_scale must be > 0");
  if (d->d_idx % 4 != 0 || (d->d_c + d->d_r) % 8 != 0) {
    set_error("d_idx must be a multiple of 4 and d_c + d_r a multiple of 8");
    return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

dsa_status check_rows(const dsa_rows* r) {
  CHECK_ARG(r != nullptr, "rows is NULL");
  CHECK_ARG(r->num_rows >= 0 && r->max_klen >= 0, "negative num_rows or max_klen");
  CHECK_ARG(r->q_group == 1 || r->q_group == 2 || r->q_group == 4, "q_group must be 1, 2 or 4");
  if (r->num_rows > 0) {
    CHECK_ARG(r->row_seq != nullptr && r->row_klen != nullptr, "row_seq / row_klen is NULL");
  }
  return DSA_OK;
}

dsa_status check_cache(const dsa_cache* c, const dsa_dims* d, bool need_idx, bool need_latent) {
  CHECK_ARG(c != nullptr, "cache is NULL");
  CHECK_ARG(c->num_seqs > 0 && c->num_tokens >= 0, "cache needs num_seqs > 0");
  if (need_idx) {
    CHECK_ARG(c->idx_k != nullptr, "idx_k is NULL");
    CHECK_ARG(aligned(c->idx_k, 16), "idx_k must be 16-byte aligned");
    if (d->idx_dtype == DSA_FP8_E4M3) CHECK_ARG(c->idx_k_scale != nullptr, "idx_k_scale is NULL");
  }
  if (need_latent) {
    CHECK_ARG(c->latent != nullptr, "latent is NULL");
    CHECK_ARG(aligned(c->latent, 16), "latent must be 16-byte aligned");
  }
  if (c->block_table) {
    CHECK_ARG(c->page_size > 0 && c->max_pages_per_seq > 0, "paged cache needs page_size > 0");
    CHECK_ARG(c->num_tokens % c->page_size == 0, "num_tokens must be num_pages * page_size");
    CHECK_ARG(c->num_tokens / c->page_size <= INT32_MAX, "too many pages");
  }
  return DSA_OK;
}

dsa_status check_proj(const dsa_proj_dims* d) {
  CHECK_ARG(d != nullptr, "dims is NULL");
  CHECK_ARG(d->n_heads > 0 && d->d_c > 0 && d->d_v > 0 && d->d_model > 0, "non-positive dimension");
  if (d->d_c % 64 != 0 || d->d_v % 32 != 0 || d->d_v > 256 || (d->n_heads * d->d_v) % 64 != 0 ||
      d->d_model % 32 != 0) {
    set_error("output projection takes d_c %% 64 == 0, d_v %% 32 == 0, d_v <= 256, "
              "H*d_v %% 64 == 0, d_model %% 32 == 0");
    return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

size_t proj_partial_bytes(const dsa_proj_dims* d, int32_t T) {
  const int splits = out_proj_splits(T, d->d_model, d->n_heads * d->d_v / 64);
  return splits > 1 ? align_up((size_t)splits * (size_t)T * (size_t)d->d_model * sizeof(float)) : 0;
}

CacheMap make_map(const dsa_cache* c) {
  CacheMap m{};
  m.seq_start = c->seq_start;
  m.block_table = c->block_table;
  m.page_size = c->block_table ? c->page_size : 1;
  m.page_shift = -1;
  if (c->block_table && (c->page_size & (c->page_size - 1)) == 0) {
    int s = 0;
    while ((1 << s) < c->page_size) ++s;
    m.page_shift = s;
  }
  m.max_pages_per_seq = c->max_pages_per_seq;
  m.num_pages = c->block_table ? (int32_t)(c->num_tokens / c->page_size) : 0;
  m.num_tokens = c->num_tokens;
  return m;
}

// Workspace layout (offsets from ws, each 256-byte aligned).
struct WsPlan {
  size_t status = 0;
  size_t indexer = 0, indexer_bytes = 0;
  size_t scores = 0, scores_bytes = 0;
  size_t idx = 0, idx_bytes = 0;
  size_t mla = 0, mla_bytes = 0;
  size_t hist = 0, hist_bytes = 0;
  size_t bwd = 0, bwd_bytes = 0;
  size_t total = 0;
  int64_t ld = 0;
  int chunk_rows = 0;
  int splits = 1;
};

WsPlan plan(const dsa_dims* d, const dsa_rows* r, dsa_op op) {
  WsPlan p;
  size_t off = kStatusBytes;
  const int T = r->num_rows;
  int rows = T;
  if (op == DSA_OP_FORWARD) rows = T < kForwardChunkRows ? T : kForwardChunkRows;
  p.chunk_rows = rows;
  p.ld = scores_ld(r->max_klen);
  const bool need_idx = op == DSA_OP_INDEXER || op == DSA_OP_DECODE_STEP || op == DSA_OP_FORWARD;
  const bool need_buf = op == DSA_OP_DECODE_STEP || op == DSA_OP_FORWARD;
  const bool need_mla = op == DSA_OP_SPARSE_MLA || need_buf;
  if (need_idx) {
    p.indexer = off;
    p.indexer_bytes = align_up(indexer_ws_bytes(rows, r->q_group));
    off += p.indexer_bytes;
  }
  if (need_buf) {
    p.scores = off;
    p.scores_bytes = align_up((size_t)rows * (size_t)p.ld * sizeof(float));
    off += p.scores_bytes;
    p.idx = off;
    p.idx_bytes = align_up((size_t)rows * (size_t)d->topk * sizeof(int32_t));
    off += p.idx_bytes;
  }
  if (need_mla) {
    p.splits = (op == DSA_OP_DECODE_STEP || op == DSA_OP_SPARSE_MLA) ? mla_tc_splits(rows) : 1;
    p.mla = off;
    p.mla_bytes = align_up(mla_ws_bytes(rows, d->n_heads, d->d_c, p.splits));
    off += p.mla_bytes;
  }
  // per-row score histograms of the fused indexer -> top-k (query groups of
  // at most 2 rows); zeroed by dsa_workspace_init and left zeroed by each top-k
  if (need_buf && r->q_group <= 2) {
    p.hist = off;
    p.hist_bytes = align_up((size_t)rows * 4096 * sizeof(uint32_t));
    off += p.hist_bytes;
  }
  if (op == DSA_OP_INDEXER_BACKWARD) {
    p.bwd = off;
    p.bwd_bytes = align_up(warmup_ws_bytes(T, r->max_klen, kWarmupChunkKeys));
    off += p.bwd_bytes;
  }
  p.total = off;
  return p;
}

dsa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned(ws, kAlign)) {
    set_error("workspace must be non-NULL and 256-byte aligned");
    return DSA_ERR_WORKSPACE;
  }
  if (ws_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", ws_bytes, need);
    return DSA_ERR_WORKSPACE;
  }
  return DSA_OK;
}

uint8_t* at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

IndexerArgs indexer_args(const dsa_dims* d, const dsa_rows* r, const dsa_cache* c,
                         const void* q_idx, const float* q_scale, const float* w, float* scores,
                         int64_t ld, void* ws, const WsPlan& p) {
  IndexerArgs a{};
  a.num_rows = r->num_rows;
  a.max_klen = r->max_klen;
  a.q_group = r->q_group;
  a.row_seq = r->row_seq;
  a.row_klen = r->row_klen;
  a.n_idx_heads = d->n_idx_heads;
  a.d_idx = d->d_idx;
  a.idx_dtype = d->idx_dtype;
  a.q_idx = q_idx;
  a.q_scale = q_scale;
  a.w = w;
  a.idx_k = c->idx_k;
  a.idx_k_scale = c->idx_k_scale;
  a.map = make_map(c);
  a.scores = scores;
  a.ld_scores = ld;
  a.num_seqs = c->num_seqs;
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  a.tile_offsets = reinterpret_cast<int32_t*>(at(ws, p.indexer));
  return a;
}

bool indexer_runs_tc(const dsa_dims* d, const IndexerArgs& a) {
  return d->algo != DSA_ALGO_SIMT && indexer_tc_supported(a);
}

dsa_status run_indexer(const dsa_dims* d, IndexerArgs& a, void* ws, const WsPlan& p,
                       cudaStream_t s) {
  if (indexer_runs_tc(d, a))
    return launch_indexer_tc(a, at(ws, p.indexer), p.indexer_bytes, s);
  return launch_indexer_simt(a, s);
}

// The fused indexer -> top-k: the indexer builds each row's histogram of its
// scores' top 12 key bits, and top-k starts from it.
// Which bytes of a workspace are known to be zero, per workspace address: all
// of it after dsa_workspace_init, the histogram region after a call whose
// top-k cleared it, nothing after any other call that writes the workspace.
// The fused histograms are accumulated into, so a call whose histogram region
// is not vouched for (a workspace reused with other rows or another op, whose
// data may lie there) clears it first.
struct ZeroSpan {
  size_t off = 0, bytes = 0;
};
std::mutex g_zero_mu;
std::unordered_map<const void*, ZeroSpan> g_zero;

void ws_zero_set(const void* ws, size_t off, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_zero_mu);
  g_zero[ws] = ZeroSpan{off, bytes};
}
void ws_zero_forget(const void* ws) { ws_zero_set(ws, 0, 0); }
bool ws_zero_covers(const void* ws, size_t off, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_zero_mu);
  const auto it = g_zero.find(ws);
  return it != g_zero.end() && it->second.off <= off && off + bytes <= it->second.off + it->second.bytes;
}
// Before a fused call: the histogram region is zero (cleared now if not vouched for).
dsa_status ws_hist_ready(void* ws, const WsPlan& p, cudaStream_t s) {
  if (ws_zero_covers(ws, p.hist, p.hist_bytes)) return DSA_OK;
  if (cudaMemsetAsync(at(ws, p.hist), 0, p.hist_bytes, s) != cudaSuccess) {
    set_error("clearing the histogram region failed: %s", cudaGetErrorString(cudaGetLastError()));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

uint32_t* fused_hist(const dsa_dims* d, const IndexerArgs& ia, void* ws, const WsPlan& p) {
  if (d->algo != DSA_ALGO_AUTO || p.hist_bytes == 0 || !indexer_tc_hist_supported(ia)) return nullptr;
  return reinterpret_cast<uint32_t*>(at(ws, p.hist));
}

MlaArgs mla_args(const dsa_dims* d, const dsa_rows* r, const dsa_cache* c, const void* q,
                 const int32_t* idx, void* out, float* lse, void* ws, const WsPlan& p) {
  MlaArgs a{};
  a.num_rows = r->num_rows;
  a.row_seq = r->row_seq;
  a.row_klen = r->row_klen;
  a.n_heads = d->n_heads;
  a.d_c = d->d_c;
  a.d_r = d->d_r;
  a.topk = d->topk;
  a.mla_dtype = d->mla_dtype;
  a.sm_scale = d->sm_scale;
  a.q = q;
  a.idx = idx;
  a.latent = c->latent;
  a.map = make_map(c);
  a.out = out;
  a.lse = lse;
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  a.splits = p.splits;
  a.part_o = at(ws, p.mla);
  a.part_ml = reinterpret_cast<float*>(
      at(ws, p.mla + (size_t)r->num_rows * p.splits * d->n_heads * d->d_c * sizeof(float)));
  a.part_cnt = reinterpret_cast<unsigned long long*>(a.part_ml + (size_t)r->num_rows * p.splits * d->n_heads * 4);
  a.trace = trace_buffer() ? trace_buffer() + kTraceMla : nullptr;
  return a;
}

dsa_status run_mla(const dsa_dims* d, MlaArgs& a, cudaStream_t s) {
  if (d->algo != DSA_ALGO_SIMT && mla_tc_supported(a)) return launch_mla_tc(a, s);
  return launch_mla_simt(a, s);
}

// Scratch of dsa_sparse_mla_fwd_noalloc: the 256-byte status block followed
// by the split-K partials, laid out as the caller workspace of
// dsa_sparse_mla_fwd.  20 MiB holds every split plan of the tensor-core path
// (H = 128, d_c = 512) on a 148-SM device: one CTA pair per (row, split), so
// rows * splits <= 74, 74 * 128 * 2064 bytes = 18.6 MiB (plus 16 bytes of
// arrival tickets per row).
constexpr size_t kNoAllocScratchBytes = size_t(20) << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device and kept.
dsa_status noalloc_scratch(void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* ptr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_error("no current CUDA device (or device index >= %d)", kMaxDevices);
    return DSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      return DSA_ERR_CUDA;
    }
    ptr[dev] = p;
  }
  *out = ptr[dev];
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_OUT_OF_RANGE: return "DSA_ERR_OUT_OF_RANGE";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
  }
  return "DSA_UNKNOWN_STATUS";
}

const char* dsa_last_error(void) { return g_err; }

int32_t dsa_version(void) { return 100; }

size_t dsa_workspace_size(const dsa_dims* dims, const dsa_rows* rows, dsa_op op) {
  if (op == DSA_OP_CACHE_APPEND) return check_dims(dims) == DSA_OK ? kStatusBytes : 0;
  if (op == DSA_OP_INDEXER_KL) return kStatusBytes;
  if (check_dims(dims) != DSA_OK || check_rows(rows) != DSA_OK) return 0;
  if (op < DSA_OP_INDEXER || op > DSA_OP_INDEXER_BACKWARD || op == DSA_OP_CACHE_APPEND) return 0;
  return plan(dims, rows, op).total;
}

dsa_status dsa_workspace_init(void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (check_ws(ws, ws_bytes, kStatusBytes) != DSA_OK) return DSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) != cudaSuccess) {
    set_error("cudaMemsetAsync failed");
    return DSA_ERR_CUDA;
  }
  ws_zero_set(ws, 0, ws_bytes);
  return DSA_OK;
}

dsa_status dsa_read_device_status(void* ws, dsa_stream_t stream, int32_t* status_out,
                                  int32_t* detail_out) {
  if (status_out == nullptr) {
    set_error("status_out is NULL");
    return DSA_ERR_INVALID_ARG;
  }
  if (check_ws(ws, kStatusBytes, kStatusBytes) != DSA_OK) return DSA_ERR_WORKSPACE;
  int32_t h[2] = {0, 0};
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess ||
      cudaMemsetAsync(ws, 0, 2 * sizeof(int32_t), s) != cudaSuccess) {
    set_error("reading the device status failed: %s", cudaGetErrorString(cudaGetLastError()));
    return DSA_ERR_CUDA;
  }
  *status_out = h[0];
  if (detail_out) *detail_out = h[0] ? h[1] : -1;
  return DSA_OK;
}

dsa_status dsa_read_kernel_trace(void* ws, dsa_stream_t stream, uint32_t* mask_out) {
  if (mask_out == nullptr) {
    set_error("mask_out is NULL");
    return DSA_ERR_INVALID_ARG;
  }
  if (check_ws(ws, kStatusBytes, kStatusBytes) != DSA_OK) return DSA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t* dev = &reinterpret_cast<DeviceStatus*>(ws)->ran;
  uint32_t h = 0;
  if (cudaMemcpyAsync(&h, dev, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(dev, 0, sizeof(h), s) != cudaSuccess) {
    set_error("reading the kernel trace failed");
    return DSA_ERR_CUDA;
  }
  *mask_out = h;
  return DSA_OK;
}

dsa_status dsa_set_stage_events(void* const* events, int32_t n_events) {
  if (n_events == 0) {
    g_n_stage_ev = 0;
    return DSA_OK;
  }
  if (n_events != 4 || events == nullptr) {
    set_error("dsa_set_stage_events takes 0 or 4 events");
    return DSA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < 4; ++i) g_stage_ev[i] = static_cast<cudaEvent_t>(events[i]);
  g_n_stage_ev = 4;
  return DSA_OK;
}

dsa_status dsa_set_trace_buffer(void* dev_buf, size_t bytes) {
  if (dev_buf != nullptr && bytes < sizeof(long long) * kTraceLen) {
    set_error("trace buffer needs %zu bytes", sizeof(long long) * kTraceLen);
    return DSA_ERR_INVALID_ARG;
  }
  g_trace = static_cast<long long*>(dev_buf);
  return DSA_OK;
}

dsa_status dsa_set_fault_injection(uint32_t spin_limit, uint32_t faults) {
  if ((faults & ~(uint32_t)DSA_FAULT_INDEXER_ACC_RELEASE) != 0) {
    set_error("unknown fault bits 0x%x", faults);
    return DSA_ERR_INVALID_ARG;
  }
  g_fault_spin = spin_limit;
  g_fault_inject = faults;
  return DSA_OK;
}

dsa_status dsa_indexer_scores(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                              const void* q_idx, const float* q_scale, const float* w,
                              float* scores, int64_t ld_scores, void* ws, size_t ws_bytes,
                              dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows)) ||
      (st = check_cache(cache, dims, true, false)))
    return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(q_idx && w && scores, "q_idx / w / scores is NULL");
    CHECK_ARG(dims->idx_dtype != DSA_FP8_E4M3 || q_scale, "q_scale is NULL for e4m3");
    CHECK_ARG(aligned(q_idx, 16) && aligned(scores, 16), "q_idx and scores must be 16-byte aligned");
  }
  CHECK_ARG(ld_scores >= rows->max_klen && ld_scores % 4 == 0,
            "ld_scores must be >= max_klen and a multiple of 4");
  const WsPlan p = plan(dims, rows, DSA_OP_INDEXER);
  if ((st = check_ws(ws, ws_bytes, p.total))) return st;
  IndexerArgs a = indexer_args(dims, rows, cache, q_idx, q_scale, w, scores, ld_scores, ws, p);
  ws_zero_forget(ws);
  return run_indexer(dims, a, ws, p, (cudaStream_t)stream);
}

dsa_status dsa_topk(const dsa_dims* dims, const dsa_rows* rows, const float* scores,
                    int64_t ld_scores, int32_t* idx, void* ws, size_t ws_bytes,
                    dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows))) return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(scores && idx, "scores / idx is NULL");
    CHECK_ARG(aligned(scores, 16), "scores must be 16-byte aligned");
  }
  CHECK_ARG(ld_scores >= rows->max_klen && ld_scores % 4 == 0,
            "ld_scores must be >= max_klen and a multiple of 4");
  const WsPlan p = plan(dims, rows, DSA_OP_TOPK);
  if ((st = check_ws(ws, ws_bytes, p.total))) return st;
  TopkArgs a{};
  a.num_rows = rows->num_rows;
  a.row_klen = rows->row_klen;
  a.scores = scores;
  a.ld_scores = ld_scores;
  a.topk = dims->topk;
  a.idx = idx;
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  a.trace = trace_buffer() ? trace_buffer() + kTraceTopk : nullptr;
  ws_zero_forget(ws);
  return launch_topk(a, rows->max_klen, (cudaStream_t)stream);
}

dsa_status dsa_sparse_mla_fwd(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                              const void* q, const int32_t* idx, void* out, float* lse, void* ws,
                              size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows)) ||
      (st = check_cache(cache, dims, false, true)))
    return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(q && idx && out, "q / idx / out is NULL");
    CHECK_ARG(aligned(q, 16) && aligned(out, 16), "q and out must be 16-byte aligned");
  }
  const WsPlan p = plan(dims, rows, DSA_OP_SPARSE_MLA);
  if ((st = check_ws(ws, ws_bytes, p.total))) return st;
  MlaArgs a = mla_args(dims, rows, cache, q, idx, out, lse, ws, p);
  ws_zero_forget(ws);
  return run_mla(dims, a, (cudaStream_t)stream);
}

dsa_status dsa_sparse_mla_fwd_noalloc(const dsa_dims* dims, const dsa_rows* rows,
                                      const dsa_cache* cache, const void* q, const int32_t* idx,
                                      void* out, float* lse, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows)) ||
      (st = check_cache(cache, dims, false, true)))
    return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(q && idx && out, "q / idx / out is NULL");
    CHECK_ARG(aligned(q, 16) && aligned(out, 16), "q and out must be 16-byte aligned");
  }
  const WsPlan p = plan(dims, rows, DSA_OP_SPARSE_MLA);
  if (p.total > kNoAllocScratchBytes) {
    set_error("sparse MLA of %d rows needs %zu bytes of scratch; the static scratch holds %zu",
              rows->num_rows, p.total, kNoAllocScratchBytes);
    return DSA_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  if ((st = noalloc_scratch(&ws))) return st;
  if (cudaMemsetAsync(ws, 0, kStatusBytes, (cudaStream_t)stream) != cudaSuccess) {
    set_error("clearing the status block failed: %s", cudaGetErrorString(cudaGetLastError()));
    return DSA_ERR_CUDA;
  }
  MlaArgs a = mla_args(dims, rows, cache, q, idx, out, lse, ws, p);
  ws_zero_forget(ws);
  return run_mla(dims, a, (cudaStream_t)stream);
}

dsa_status dsa_decode_step(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                           const void* q_idx, const float* q_scale, const float* w, const void* q,
                           void* out, float* lse, float* dbg_scores, int32_t* dbg_idx, void* ws,
                           size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows)) ||
      (st = check_cache(cache, dims, true, true)))
    return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(q_idx && w && q && out, "q_idx / w / q / out is NULL");
    CHECK_ARG(dims->idx_dtype != DSA_FP8_E4M3 || q_scale, "q_scale is NULL for e4m3");
    CHECK_ARG(aligned(q_idx, 16) && aligned(q, 16) && aligned(out, 16),
              "q_idx, q and out must be 16-byte aligned");
    CHECK_ARG(dbg_scores == nullptr || aligned(dbg_scores, 16), "dbg_scores must be 16-byte aligned");
  }
  const WsPlan p = plan(dims, rows, DSA_OP_DECODE_STEP);
  if ((st = check_ws(ws, ws_bytes, p.total))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  float* scores = dbg_scores ? dbg_scores : reinterpret_cast<float*>(at(ws, p.scores));
  int32_t* idx = dbg_idx ? dbg_idx : reinterpret_cast<int32_t*>(at(ws, p.idx));
  IndexerArgs ia = indexer_args(dims, rows, cache, q_idx, q_scale, w, scores, p.ld, ws, p);
  ia.hist = fused_hist(dims, ia, ws, p);
  if (ia.hist && (st = ws_hist_ready(ws, p, s))) return st;
  ws_zero_forget(ws);
  // a cluster top-k follows: the indexer lets it launch only at its end
  ia.late_trigger = indexer_runs_tc(dims, ia) && topk_uses_clusters(rows->num_rows, rows->max_klen);
  stage_event(0, s);
  if ((st = run_indexer(dims, ia, ws, p, s))) return st;
  stage_event(1, s);
  TopkArgs ta{};
  ta.num_rows = rows->num_rows;
  ta.row_klen = rows->row_klen;
  ta.scores = scores;
  ta.ld_scores = p.ld;
  ta.topk = dims->topk;
  ta.idx = idx;
  ta.status = reinterpret_cast<DeviceStatus*>(ws);
  ta.trace = trace_buffer() ? trace_buffer() + kTraceTopk : nullptr;
  ta.hist = ia.hist;
  ta.after_late_trigger = ia.late_trigger;
  if ((st = launch_topk(ta, rows->max_klen, s))) return st;
  stage_event(2, s);
  MlaArgs ma = mla_args(dims, rows, cache, q, idx, out, lse, ws, p);
  st = run_mla(dims, ma, s);
  stage_event(3, s);
  // the top-k left the histogram region zeroed
  if (st == DSA_OK && ia.hist) ws_zero_set(ws, p.hist, p.hist_bytes);
  return st;
}

dsa_status dsa_forward(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                       const void* q_idx, const float* q_scale, const float* w, const void* q,
                       void* out, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes,
                       dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows)) ||
      (st = check_cache(cache, dims, true, true)))
    return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(q_idx && w && q && out, "q_idx / w / q / out is NULL");
    CHECK_ARG(dims->idx_dtype != DSA_FP8_E4M3 || q_scale, "q_scale is NULL for e4m3");
    CHECK_ARG(aligned(q_idx, 16) && aligned(q, 16) && aligned(out, 16),
              "q_idx, q and out must be 16-byte aligned");
  }
  const WsPlan p = plan(dims, rows, DSA_OP_FORWARD);
  if ((st = check_ws(ws, ws_bytes, p.total))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int T = rows->num_rows;
  const int H_I = dims->n_idx_heads, D_I = dims->d_idx, H = dims->n_heads;
  const int DQK = dims->d_c + dims->d_r;
  const size_t qi_el = dims->idx_dtype == DSA_FP8_E4M3 ? 1 : 4;
  const size_t mla_el = dims->mla_dtype == DSA_BF16 ? 2 : 4;
  float* scores = reinterpret_cast<float*>(at(ws, p.scores));
  int32_t* idx_ws = reinterpret_cast<int32_t*>(at(ws, p.idx));
  bool used_hist = false;
  for (int r0 = 0; r0 < T; r0 += p.chunk_rows) {
    const int n = (T - r0) < p.chunk_rows ? (T - r0) : p.chunk_rows;
    dsa_rows cr = *rows;
    cr.num_rows = n;
    cr.row_seq = rows->row_seq + r0;
    cr.row_klen = rows->row_klen + r0;
    const uint8_t* qi = static_cast<const uint8_t*>(q_idx) + (size_t)r0 * H_I * D_I * qi_el;
    const float* qs = q_scale ? q_scale + (size_t)r0 * H_I : nullptr;
    const float* wr = w + (size_t)r0 * H_I;
    const uint8_t* qq = static_cast<const uint8_t*>(q) + (size_t)r0 * H * DQK * mla_el;
    uint8_t* oo = static_cast<uint8_t*>(out) + (size_t)r0 * H * dims->d_c * mla_el;
    float* ll = lse ? lse + (size_t)r0 * H : nullptr;
    int32_t* idx = idx_out ? idx_out + (size_t)r0 * dims->topk : idx_ws;
    IndexerArgs ia = indexer_args(dims, &cr, cache, qi, qs, wr, scores, p.ld, ws, p);
    ia.hist = fused_hist(dims, ia, ws, p);
    if (ia.hist && !used_hist && (st = ws_hist_ready(ws, p, s))) return st;
    if (r0 == 0) ws_zero_forget(ws);
    used_hist = used_hist || ia.hist != nullptr;
    ia.late_trigger = indexer_runs_tc(dims, ia) && topk_uses_clusters(n, rows->max_klen);
    if ((st = run_indexer(dims, ia, ws, p, s))) return st;
    TopkArgs ta{};
    ta.num_rows = n;
    ta.row_klen = cr.row_klen;
    ta.scores = scores;
    ta.ld_scores = p.ld;
    ta.topk = dims->topk;
    ta.idx = idx;
    ta.status = reinterpret_cast<DeviceStatus*>(ws);
    ta.trace = trace_buffer() ? trace_buffer() + kTraceTopk : nullptr;
    ta.hist = ia.hist;
    ta.after_late_trigger = ia.late_trigger;
    if ((st = launch_topk(ta, rows->max_klen, s))) return st;
    MlaArgs ma = mla_args(dims, &cr, cache, qq, idx, oo, ll, ws, p);
    if ((st = run_mla(dims, ma, s))) return st;
  }
  // every chunk's top-k left the histogram region zeroed
  if (used_hist) ws_zero_set(ws, p.hist, p.hist_bytes);
  return DSA_OK;
}

dsa_status dsa_cache_append(const dsa_dims* dims, const dsa_cache* cache, int32_t n_new,
                            const int32_t* tok_seq, const int32_t* tok_pos,
                            const float* k_new, const void* latent_new,
                            void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) != DSA_OK) return st;
  if ((st = check_cache(cache, dims, true, true)) != DSA_OK) return st;
  CHECK_ARG(n_new >= 0, "n_new must be >= 0");
  if ((st = check_ws(ws, ws_bytes, kStatusBytes)) != DSA_OK) return st;
  if (dims->d_idx > cache_append_max_d_idx()) {
    set_error("cache append takes d_idx <= %d", cache_append_max_d_idx());
    return DSA_ERR_UNSUPPORTED;
  }
  if (n_new == 0) return DSA_OK;
  CHECK_ARG(tok_seq != nullptr && tok_pos != nullptr, "tok_seq / tok_pos is NULL");
  CHECK_ARG(k_new != nullptr && aligned(k_new, 16), "k_new must be non-NULL and 16-byte aligned");
  CHECK_ARG(latent_new != nullptr && aligned(latent_new, 16),
            "latent_new must be non-NULL and 16-byte aligned");
  AppendArgs a{};
  a.n_new = n_new;
  a.tok_seq = tok_seq;
  a.tok_pos = tok_pos;
  a.k_new = k_new;
  a.latent_new = latent_new;
  a.d_idx = dims->d_idx;
  a.latent_row_bytes = (dims->d_c + dims->d_r) * (dims->mla_dtype == DSA_BF16 ? 2 : 4);
  a.idx_dtype = dims->idx_dtype;
  // the caches are written here; the descriptor is shared with the read-only calls
  a.idx_k = const_cast<void*>(cache->idx_k);
  a.idx_k_scale = const_cast<float*>(cache->idx_k_scale);
  a.latent = const_cast<void*>(cache->latent);
  a.map = make_map(cache);
  a.num_seqs = cache->num_seqs;
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  return launch_cache_append(a, (cudaStream_t)stream);
}

dsa_status dsa_indexer_kl(const dsa_rows* rows, const float* scores, int64_t ld_scores,
                          const float* teacher, int64_t ld_teacher, float* grad, int64_t ld_grad,
                          float* loss, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_rows(rows))) return st;
  if ((st = check_ws(ws, ws_bytes, kStatusBytes))) return st;
  if (rows->num_rows > 0) CHECK_ARG(scores && teacher && grad && loss, "a tensor pointer is NULL");
  CHECK_ARG(ld_scores >= rows->max_klen && ld_teacher >= rows->max_klen && ld_grad >= rows->max_klen,
            "leading dimensions must be >= max_klen");
  WarmupArgs a{};
  a.num_rows = rows->num_rows;
  a.row_seq = rows->row_seq;
  a.row_klen = rows->row_klen;
  a.scores = scores;
  a.ld_scores = ld_scores;
  a.teacher = teacher;
  a.ld_teacher = ld_teacher;
  a.grad = grad;
  a.ld_grad = ld_grad;
  a.loss = loss;
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  return launch_indexer_kl(a, (cudaStream_t)stream);
}

dsa_status dsa_indexer_backward(const dsa_dims* dims, const dsa_rows* rows, const dsa_cache* cache,
                                const void* q_idx, const float* q_scale, const float* w,
                                const float* grad, int64_t ld_grad, float* dq, float* dw, float* dk,
                                void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_dims(dims)) || (st = check_rows(rows)) ||
      (st = check_cache(cache, dims, true, false)))
    return st;
  if (rows->num_rows > 0) {
    CHECK_ARG(q_idx && w && grad && dq && dw && dk, "a tensor pointer is NULL");
    CHECK_ARG(dims->idx_dtype != DSA_FP8_E4M3 || q_scale, "q_scale is NULL for e4m3");
  }
  CHECK_ARG(ld_grad >= rows->max_klen, "ld_grad must be >= max_klen");
  const WsPlan p = plan(dims, rows, DSA_OP_INDEXER_BACKWARD);
  if ((st = check_ws(ws, ws_bytes, p.total))) return st;
  WarmupArgs a{};
  a.num_rows = rows->num_rows;
  a.row_seq = rows->row_seq;
  a.row_klen = rows->row_klen;
  a.n_idx_heads = dims->n_idx_heads;
  a.d_idx = dims->d_idx;
  a.idx_dtype = dims->idx_dtype;
  a.q_idx = q_idx;
  a.q_scale = dims->idx_dtype == DSA_FP8_E4M3 ? q_scale : nullptr;
  a.w = w;
  a.idx_k = cache->idx_k;
  a.idx_k_scale = dims->idx_dtype == DSA_FP8_E4M3 ? cache->idx_k_scale : nullptr;
  a.map = make_map(cache);
  a.grad = const_cast<float*>(grad);
  a.ld_grad = ld_grad;
  a.dq = dq;
  a.dw = dw;
  a.dk = dk;
  a.partial = reinterpret_cast<float*>(at(ws, p.bwd));
  ws_zero_forget(ws);
  a.chunk_keys = kWarmupChunkKeys;
  a.n_chunks = (rows->max_klen + kWarmupChunkKeys - 1) / kWarmupChunkKeys;
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  if (!warmup_supported(a)) {
    set_error("indexer backward runs H_I = 64, d_I = 128 (e4m3 or f32)");
    return DSA_ERR_UNSUPPORTED;
  }
  return launch_indexer_backward(a, rows->max_klen, cache->num_seqs, (cudaStream_t)stream);
}

size_t dsa_output_projection_ws_size(const dsa_proj_dims* dims, int32_t num_rows) {
  if (check_proj(dims) != DSA_OK || num_rows < 0) return 0;
  return kStatusBytes + proj_partial_bytes(dims, num_rows);
}

dsa_status dsa_output_projection(const dsa_proj_dims* dims, int32_t num_rows, const void* o,
                                 const void* w_uv, const void* w_out, void* u, void* y,
                                 void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st;
  if ((st = check_proj(dims)) != DSA_OK) return st;
  CHECK_ARG(num_rows >= 0, "num_rows must be >= 0");
  if ((st = check_ws(ws, ws_bytes, kStatusBytes + proj_partial_bytes(dims, num_rows))) != DSA_OK)
    return st;
  ws_zero_forget(ws);
  if (num_rows == 0) return DSA_OK;
  CHECK_ARG(o && w_uv && w_out && u && y, "a tensor pointer is NULL");
  CHECK_ARG(aligned(o, 16) && aligned(w_uv, 16) && aligned(w_out, 16) && aligned(u, 16) &&
                aligned(y, 16),
            "tensors must be 16-byte aligned");
  if (tensor_map_encoder() == nullptr) {
    set_error("output projection needs cuTensorMapEncodeTiled from the driver");
    return DSA_ERR_UNSUPPORTED;
  }
  ProjArgs a{};
  a.num_rows = num_rows;
  a.n_heads = dims->n_heads;
  a.d_c = dims->d_c;
  a.d_v = dims->d_v;
  a.d_model = dims->d_model;
  a.o = o;
  a.w_uv = w_uv;
  a.w_out = w_out;
  a.u = u;
  a.y = y;
  a.partial = reinterpret_cast<float*>(at(ws, kStatusBytes));
  a.status = reinterpret_cast<DeviceStatus*>(ws);
  return launch_out_proj(a, (cudaStream_t)stream);
}

}  // extern "C"
