// dsa_kernels.cuh - argument blocks and launchers of the DSA kernels.
#pragma once

#include <atomic>

#include "dsa_common.cuh"

namespace dsa {

struct IndexerArgs {
  int num_rows, max_klen, q_group;
  const int32_t* row_seq;
  const int32_t* row_klen;
  int n_idx_heads, d_idx;
  dsa_dtype idx_dtype;
  const void* q_idx;          // [T, H_I, d_I]
  const float* q_scale;       // [T, H_I] or null
  const float* w;             // [T, H_I]
  const void* idx_k;          // [num_tokens, d_I]
  const float* idx_k_scale;   // [num_tokens] or null
  CacheMap map;
  float* scores;
  int64_t ld_scores;
  int num_seqs;
  DeviceStatus* status;
  int32_t* tile_offsets;      // workspace: [n_groups + 1] exclusive scan of key tiles
  uint32_t* hist;             // [num_rows, 4096] score-key histograms (zeroed), or null
  int late_trigger;           // tensor-core kernel: let dependents launch only once a CTA's
                              // tiles are done (the next kernel is a cluster top-k)
};

struct TopkArgs {
  int num_rows;
  const int32_t* row_klen;
  const float* scores;
  int64_t ld_scores;
  int topk;
  int32_t* idx;               // [T, topk]
  DeviceStatus* status;
  long long* trace;           // profiling stamps or null
  uint32_t* hist;             // [T, 4096] histograms of the scores' top 12 key bits from the
                              // indexer (read, then zeroed), or null: top-k builds its own
  int after_late_trigger;     // the previous kernel lets dependents launch at its end only
};

struct MlaArgs {
  int num_rows;
  const int32_t* row_seq;
  const int32_t* row_klen;
  int n_heads, d_c, d_r, topk;
  dsa_dtype mla_dtype;
  float sm_scale;
  const void* q;              // [T, H, d_c + d_r]
  const int32_t* idx;         // [T, topk]
  const void* latent;         // [num_tokens, d_c + d_r]
  CacheMap map;
  void* out;                  // [T, H, d_c]
  float* lse;                 // [T, H] or null
  DeviceStatus* status;
  // split-K scratch (tensor-core path)
  void* part_o;               // [T, splits, 2 ranks, 64, H] float4: unnormalised O, dims
                              // 4i..4i+3 of the rank's 256 for head h
  float* part_ml;             // [T, splits, 2, H, 2]  (max, sum) per CTA of the pair
  unsigned long long* part_cnt;   // [T, 2] arrival tickets: launch id << 32 | arrivals
  uint32_t launch_id;         // nonzero, distinct for consecutive launches
  int splits;
  int merge_in_cluster;       // 2 splits in one 4-CTA cluster, merged through shared memory
  long long* trace;           // profiling stamps or null
};

struct AppendArgs {
  int n_new;
  const int32_t* tok_seq;     // [n_new]
  const int32_t* tok_pos;     // [n_new]
  const float* k_new;         // [n_new, d_I] fp32
  const void* latent_new;     // [n_new, d_c + d_r] in the latent cache's dtype
  int d_idx;
  int latent_row_bytes;       // (d_c + d_r) * element size, a multiple of 16
  dsa_dtype idx_dtype;
  void* idx_k;                // written: [num_tokens, d_I] e4m3 | f32
  float* idx_k_scale;         // written: [num_tokens] (e4m3 only)
  void* latent;               // written: [num_tokens, d_c + d_r]
  CacheMap map;
  int num_seqs;
  DeviceStatus* status;
};

// Profiling trace buffer registered on the calling host thread (or null).
// Layout (int64 clock64 stamps): [0, 512) the attention kernel's first CTA
// pair ([2 CTAs][8 events][32 blocks]), [512, 640) top-k's first cluster
// ([8 CTAs][16 events]), [640, 896) the indexer's CTA 0 ([8 events][32 tiles]).
long long* trace_buffer();
constexpr int kTraceMla = 0, kTraceTopk = 512, kTraceIdx = 640, kTraceLen = 896;
// Test-only fault injection of the calling host thread (dsa_set_fault_injection):
// the spin limit of the kernels' bounded waits (kSpinLimit unless set) and the
// DSA_FAULT_* bits to inject.
uint32_t fault_spin_limit();
uint32_t fault_inject();
static constexpr int kTraceEvents = 8, kTraceBlocks = 32;

dsa_status launch_indexer_simt(const IndexerArgs& a, cudaStream_t stream);
dsa_status launch_indexer_tc(const IndexerArgs& a, void* ws_tail, size_t ws_tail_bytes,
                             cudaStream_t stream);
bool indexer_tc_supported(const IndexerArgs& a);
// The indexer builds the rows' score histograms for top-k (fused path).
bool indexer_tc_hist_supported(const IndexerArgs& a);
size_t indexer_ws_bytes(int num_rows, int q_group);

dsa_status launch_topk(const TopkArgs& a, int max_klen, cudaStream_t stream);
size_t topk_ws_bytes();

dsa_status launch_mla_simt(const MlaArgs& a, cudaStream_t stream);
dsa_status launch_mla_tc(const MlaArgs& a, cudaStream_t stream);
bool mla_tc_supported(const MlaArgs& a);
int mla_tc_splits(int num_rows);
// Whether a top-k of `num_rows` rows of at most `max_klen` keys runs as
// clusters (else one CTA per row, streaming).
bool topk_uses_clusters(int num_rows, int max_klen);
size_t mla_ws_bytes(int num_rows, int n_heads, int d_c, int splits);

dsa_status launch_cache_append(const AppendArgs& a, cudaStream_t stream);
int cache_append_max_d_idx();

// Indexer warm-up: KL(p || softmax(I)) per row, its gradient g, and the
// backward of the indexer scores to q_I, w and k_I.
struct WarmupArgs {
  int num_rows;
  const int32_t* row_seq;
  const int32_t* row_klen;
  int n_idx_heads, d_idx;
  dsa_dtype idx_dtype;
  const void* q_idx;          // [T, H_I, d_I]
  const float* q_scale;       // [T, H_I] or null
  const float* w;             // [T, H_I]
  const void* idx_k;          // [num_tokens, d_I]
  const float* idx_k_scale;   // [num_tokens] or null
  CacheMap map;
  const float* scores;        // KL: [T, ld_scores]
  int64_t ld_scores;
  const float* teacher;       // KL: [T, ld_teacher]
  int64_t ld_teacher;
  float* grad;                // KL: written; backward: read.  [T, ld_grad]
  int64_t ld_grad;
  float* loss;                // KL: [T]
  float* dq;                  // backward: [T, H_I, d_I]
  float* dw;                  // backward: [T, H_I]
  float* dk;                  // backward: [num_tokens, d_I] (rows some query sees)
  float* partial;             // backward workspace: [T, n_chunks, H_I, d_I + 1]
  int chunk_keys, n_chunks;
  DeviceStatus* status;
};
bool warmup_supported(const WarmupArgs& a);
size_t warmup_ws_bytes(int num_rows, int max_klen, int chunk_keys);
dsa_status launch_indexer_kl(const WarmupArgs& a, cudaStream_t stream);
dsa_status launch_indexer_backward(const WarmupArgs& a, int max_klen, int num_seqs, cudaStream_t stream);

// Output projection: u = W_UV,i o_i per head, then y = W_out [u_1; ...; u_H].
struct ProjArgs {
  int num_rows, n_heads, d_c, d_v, d_model;
  const void* o;              // [T, H, d_c] bf16
  const void* w_uv;           // [H, d_v, d_c] bf16
  const void* w_out;          // [d_model, H * d_v] bf16
  void* u;                    // [T, H, d_v] bf16
  void* y;                    // [T, d_model] bf16
  float* partial;             // workspace: [splits, T, d_model] fp32 (splits > 1)
  DeviceStatus* status;
};
int out_proj_splits(int num_rows, int d_model, int k_blocks);
dsa_status launch_out_proj(const ProjArgs& a, cudaStream_t stream);

// cuTensorMapEncodeTiled from the driver (null when unavailable), looked up once.
void* tensor_map_encoder();

// Per-device host state.  Kernel attributes and device properties belong to a
// device, so a process that drives several GPUs sets and caches them per
// device (the current one at the call).
constexpr int kMaxDevices = 128;
// Raises the dynamic shared-memory limit of kernel `fn` to `bytes` on the
// current device, once per device (`done` is the kernel's flag array).
dsa_status set_smem_limit_once(const void* fn, size_t bytes, std::atomic<bool> (&done)[kMaxDevices]);
// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Host-side error text of the calling thread.
void set_error(const char* fmt, ...);

}  // namespace dsa
