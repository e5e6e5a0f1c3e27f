// topk.cu - per-row top-k selection by radix select ("DeepSeek Sparse
// Attention DSA Architecture Guide", section "Stage 2: Fine-Grained Token
// Selection and Output Computation", selection equation S_t = TopK(I[t,:], k)).
//
// One cluster of `csize` CTAs (1..8, 512 threads each) per query row.  Each CTA
// copies a contiguous segment of the row into shared memory (cp.async, all
// loads in flight at once) and turns it in place into order-preserving uint32
// keys (float -> key, -0 mapped to +0).  The k-th largest key T is found digit
// by digit (12 + 10 + 10 bits, most significant first):
//   * every CTA builds a histogram of its keys that match the prefix so far;
//   * the cluster merges them as a reduce-scatter: CTA r sums bins
//     [r*B/csize, (r+1)*B/csize) over the cluster through distributed shared
//     memory, the per-CTA slice totals are exchanged, and the CTA whose slice
//     holds the k-th key finds the bin and tells the others;
//   * after the first digit only the keys of the threshold bin can matter, so
//     each CTA moves them to a candidate list and later digits scan the list.
// The output pass walks the segment in position order (lane-interleaved, so
// shared-memory loads are conflict free, with warp ballots for the ordering)
// and keeps key > T, and key == T while the running count of equal keys
// (across the cluster, in position order) is below the number still needed.
// The selected positions come out sorted ascending with ties going to the
// lower position, without a sort.  Rows with klen <= k return 0..klen-1 then -1.
#include "dsa_kernels.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins0 = 4096;       // first digit: bits 31..20
constexpr int kCacheCap = 16384;   // keys of the segment kept in smem
constexpr int kCandCap = 4096;     // candidates of the threshold bin per CTA
constexpr int kMaxCluster = 8;

__device__ __forceinline__ void kstamp(long long* tr, int ev) {
  if (tr != nullptr && blockIdx.x == 0 && threadIdx.x == 0 && ev < kTraceBlocks) tr[ev] = clock64();
}

struct TopkSmem {
  uint32_t keys[kCacheCap];
  uint32_t hist[kBins0];
  uint32_t cand_key[kCandCap];
  uint32_t slice_tot[2][kMaxCluster];   // per-CTA slice totals, by digit parity
  uint32_t counts[kMaxCluster][2];      // per-CTA (n_gt, n_eq)
  uint32_t warp_tmp[kWarps];
  uint32_t warp_cnt[kWarps][2];
  uint32_t cand_n;
  uint32_t sel[2][2];                   // (bin, need) found for digit d, by parity
};

// Exclusive prefix over the block of one value per thread (512 threads).
__device__ __forceinline__ uint32_t block_excl_prefix(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t s = tmp[w];
    before += (w < warp) ? s : 0u;
    all += s;
  }
  __syncthreads();
  if (total) *total = all;
  return before + x - v;
}

// Shared histogram increment.  Row scores spread over many bins (a 32-key
// warp round hits ~25 distinct bins), so warp-level aggregation of equal bins
// buys nothing; the shared-memory atomic unit resolves the rare collisions.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool valid, uint32_t bin) {
  if (valid) atomicAdd(&hist[bin], 1u);
}

// Cluster-wide selection of the bin holding the `need`-th largest key among
// `nbins` histogram bins (S.hist of every CTA).  Returns (bin, need within bin)
// in S.sel[par] of every CTA.  Two cluster barriers.
__device__ void cluster_select(TopkSmem& S, int nbins, uint32_t need, uint32_t csize,
                               uint32_t rank, int par) {
  const int slice = nbins / (int)csize;              // bins owned by this CTA
  const int b0 = (int)rank * slice;
  cluster_sync();                                    // all histograms complete
  // this CTA's slice, summed over the cluster: one bin per thread (slice <= 4096)
  uint32_t mine[8];
  uint32_t local = 0;
  const int per = (slice + kThreads - 1) / kThreads; // 1..8 bins per thread
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mine[i] = 0;
    if (i < per) {
      const int b = b0 + threadIdx.x * per + i;
      if (threadIdx.x * per + i < slice) {
        if (csize == 1) {
          mine[i] = S.hist[b];
        } else {
          uint32_t vv[kMaxCluster];
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r)
            vv[r] = r < (int)csize ? ld_dsmem_u32(mapa(&S.hist[b], (uint32_t)r)) : 0u;
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r) mine[i] += vv[r];
        }
      }
    }
    local += mine[i];
  }
  // suffix position of each thread's bins within the slice (bins descending = threads descending)
  uint32_t total;
  const uint32_t before = block_excl_prefix(local, S.warp_tmp, &total);
  const uint32_t above_in_slice = total - before - local;   // keys in higher bins of the slice
  // slice totals to every CTA
  if (threadIdx.x == 0) {
    for (uint32_t r = 0; r < csize; ++r) {
      if (csize == 1) S.slice_tot[par][rank] = total;
      else st_dsmem_u32(mapa(&S.slice_tot[par][rank], r), total);
    }
  }
  cluster_sync();
  // keys above this CTA's slice: all slices of higher rank
  uint32_t above = 0;
  for (uint32_t r = rank + 1; r < csize; ++r) above += S.slice_tot[par][r];
  if (above < need && above + total >= need) {       // the slice holding the need-th key
    uint32_t cum = above + above_in_slice;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (i < per) {
        const uint32_t c = mine[i];
        if (cum < need && cum + c >= need) {
          const int b = b0 + threadIdx.x * per + i;
          for (uint32_t r = 0; r < csize; ++r) {
            if (csize == 1) {
              S.sel[par][0] = (uint32_t)b;
              S.sel[par][1] = need - cum;
            } else {
              st_dsmem_u32(mapa(&S.sel[par][0], r), (uint32_t)b);
              st_dsmem_u32(mapa(&S.sel[par][1], r), need - cum);
            }
          }
        }
        cum += c;
      }
    }
  }
  cluster_sync();                                    // (bin, need) everywhere
}

__global__ void __launch_bounds__(kThreads, 2) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smraw);
  trace_kernel(a.status, DSA_KERNEL_TOPK);
  const uint32_t csize = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int t = blockIdx.x / csize;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.topk;
  const int klen = a.row_klen[t];
  int32_t* out = a.idx + (int64_t)t * k;

  kstamp(a.trace, 0);
  if (klen <= k) {  // uniform over the cluster; no DSMEM was touched
    for (int i = rank * kThreads + tid; i < k; i += csize * kThreads) out[i] = i < klen ? i : -1;
    return;
  }

  const float* row = a.scores + (int64_t)t * a.ld_scores;
  const int seg = (((klen + (int)csize - 1) / (int)csize) + 3) & ~3;
  const int lo = min((int)rank * seg, klen);
  const int hi = min(lo + seg, klen);
  const int n = hi - lo;
  const int ncache = min(n, kCacheCap);
  const float* srow = row + lo;

  // ---- the segment into shared memory: every 16-byte piece in flight at once
  {
    const int n4 = (reinterpret_cast<uintptr_t>(srow) & 15) == 0 ? (ncache >> 2) : 0;
    for (int i = tid; i < n4; i += kThreads) cp_async_16(&S.keys[4 * i], srow + 4 * i);
    for (int i = 4 * n4 + tid; i < ncache; i += kThreads)
      S.keys[i] = __float_as_uint(__ldcg(srow + i));
  }
  for (int i = tid; i < kBins0; i += kThreads) S.hist[i] = 0;
  if (tid == 0) S.cand_n = 0;
  cp_async_wait_all();
  __syncthreads();
  kstamp(a.trace, 1);

  auto key_at = [&](int i) -> uint32_t {
    return i < ncache ? S.keys[i] : float_key(__ldcg(srow + i));
  };

  // ---- digit 0: keys in place, histogram of bits 31..20
  const int nround = (n + kThreads - 1) / kThreads;
#pragma unroll 4
  for (int r = 0; r < nround; ++r) {
    const int i = r * kThreads + tid;
    const bool v = i < n;
    uint32_t key = 0;
    if (v) {
      if (i < ncache) {
        key = float_key(__uint_as_float(S.keys[i]));
        S.keys[i] = key;
      } else {
        key = float_key(__ldcg(srow + i));
      }
    }
    hist_add(S.hist, v, key >> 20);
  }
  kstamp(a.trace, 2);
  cluster_select(S, kBins0, (uint32_t)k, csize, rank, 0);
  uint32_t prefix = S.sel[0][0];
  uint32_t need = S.sel[0][1];
  kstamp(a.trace, 3);

  // ---- candidates of the threshold bin (warp-aggregated appends); this
  // CTA's own histogram still says how many there are
  const bool use_cand = S.hist[prefix] <= (uint32_t)kCandCap;
  if (use_cand) {
#pragma unroll 4
    for (int r = 0; r < nround; ++r) {
      const int i = r * kThreads + tid;
      uint32_t key = 0;
      const bool v = (i < n) && (((key = key_at(i)) >> 20) == prefix);
      const uint32_t m = __ballot_sync(0xffffffffu, v);
      uint32_t base = 0;
      if (lane == 0 && m) base = atomicAdd(&S.cand_n, (uint32_t)__popc(m));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (v) {
        const uint32_t slot = base + __popc(m & ((1u << lane) - 1));
        S.cand_key[slot] = key;
      }
    }
  }
  __syncthreads();   // every thread has read S.hist[prefix] before it is cleared
  const int ncand = use_cand ? (int)S.cand_n : n;
  kstamp(a.trace, 4);

  // ---- digits 1 and 2 (10 bits each) over the candidates (or the segment)
  int shift = 20;
#pragma unroll 1
  for (int d = 0; d < 2; ++d) {
    const int nshift = 10 - 10 * d;                  // 10, then 0
    for (int i = tid; i < 1024; i += kThreads) S.hist[i] = 0;
    __syncthreads();
    const int nr = (ncand + kThreads - 1) / kThreads;
    for (int r = 0; r < nr; ++r) {
      const int i = r * kThreads + tid;
      bool v = i < ncand;
      uint32_t key = 0;
      if (v) key = use_cand ? S.cand_key[i] : key_at(i);
      v = v && ((key >> shift) == prefix);
      hist_add(S.hist, v, (key >> nshift) & 1023u);
    }
    kstamp(a.trace, 5 + 2 * d);
    cluster_select(S, 1024, need, csize, rank, (d + 1) & 1);
    prefix = (prefix << 10) | S.sel[(d + 1) & 1][0];
    need = S.sel[(d + 1) & 1][1];
    shift = nshift;
    kstamp(a.trace, 6 + 2 * d);
  }
  const uint32_t T = prefix;     // the k-th largest key

  // ---- counts of keys > T and == T per warp chunk (positions in order:
  // warp w owns [w*chunk, (w+1)*chunk)), per CTA, shared with the cluster
  const int chunk = ((n + kWarps - 1) / kWarps + 31) & ~31;
  const int w_lo = min(warp * chunk, n), w_hi = min(w_lo + chunk, n);
  uint32_t w_gt = 0, w_eq = 0;
  for (int i = w_lo + lane; i < w_hi; i += 32) {
    const uint32_t key = key_at(i);
    w_gt += key > T;
    w_eq += key == T;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    w_gt += __shfl_xor_sync(0xffffffffu, w_gt, off);
    w_eq += __shfl_xor_sync(0xffffffffu, w_eq, off);
  }
  if (lane == 0) {
    S.warp_cnt[warp][0] = w_gt;
    S.warp_cnt[warp][1] = w_eq;
  }
  __syncthreads();
  uint32_t gw = 0, ew = 0, tot_gt = 0, tot_eq = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t g = S.warp_cnt[w][0], e = S.warp_cnt[w][1];
    gw += w < warp ? g : 0u;
    ew += w < warp ? e : 0u;
    tot_gt += g;
    tot_eq += e;
  }
  if (tid < (int)csize) {
    if (csize == 1) {
      S.counts[rank][0] = tot_gt;
      S.counts[rank][1] = tot_eq;
    } else {
      st_dsmem_u32(mapa(&S.counts[rank][0], (uint32_t)tid), tot_gt);
      st_dsmem_u32(mapa(&S.counts[rank][1], (uint32_t)tid), tot_eq);
    }
  }
  cluster_sync();
  kstamp(a.trace, 9);
  uint32_t out_base = 0, eq_base = 0;
  for (uint32_t r = 0; r < rank; ++r) {
    const uint32_t e = S.counts[r][1];
    const uint32_t take = (eq_base >= need) ? 0u : min(e, need - eq_base);
    out_base += S.counts[r][0] + take;
    eq_base += e;
  }

  // ---- ordered output: lane-interleaved rounds of 32 positions per warp;
  // ballots give the order inside a round.  An equal key is taken while the
  // number of equal keys before it (cluster-wide, in position order) < need.
  uint32_t eq_rank = eq_base + ew;
  const uint32_t eq_taken_before = (eq_base >= need) ? 0u : min(ew, need - eq_base);
  uint32_t pos = out_base + gw + eq_taken_before;
  const uint32_t lt_mask = (1u << lane) - 1;
  for (int i0 = w_lo; i0 < w_hi; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < w_hi ? key_at(i) : 0u;
    const bool gt = i < w_hi && key > T;
    const bool eq = i < w_hi && key == T;
    const uint32_t em = __ballot_sync(0xffffffffu, eq);
    const uint32_t my_eq_rank = eq_rank + __popc(em & lt_mask);
    const bool sel = gt || (eq && my_eq_rank < need);
    const uint32_t sm = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const uint32_t p = pos + __popc(sm & lt_mask);
      if (p < (uint32_t)k) out[p] = lo + i;
    }
    pos += __popc(sm);
    eq_rank += __popc(em);
  }
  kstamp(a.trace, 10);
  cluster_sync();   // keep this CTA's smem alive until the cluster's remote accesses are done
  kstamp(a.trace, 11);
}

}  // namespace

size_t topk_ws_bytes() { return 0; }

dsa_status launch_topk(const TopkArgs& a, int max_klen, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  int csize = 1;
  while (csize < kMaxCluster && (int64_t)csize * kCacheCap < (int64_t)max_klen) csize <<= 1;
  const size_t smem = sizeof(TopkSmem);
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.num_rows * csize));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, topk_kernel, a);
  if (e != cudaSuccess) {
    set_error("topk launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
