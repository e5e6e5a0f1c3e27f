// topk.cu - per-row top-k selection by radix select ("DeepSeek Sparse
// Attention DSA Architecture Guide", section "Stage 2: Fine-Grained Token
// Selection and Output Computation", selection equation S_t = TopK(I[t,:], k)).
//
// One cluster of `csize` CTAs (1..8) per query row.  Each CTA owns a
// contiguous segment of the row and keeps it in shared memory as
// order-preserving uint32 keys (float -> key with -0 mapped to +0).  The k-th
// largest key T is found digit by digit (11 + 11 + 10 bits, most significant
// first): every CTA builds a 2048-bin histogram of its keys that match the
// prefix found so far, the histograms are summed across the cluster through
// distributed shared memory, and the bin where the count from the top reaches
// k is the next digit.  After the first digit only the keys of the threshold
// bin can still matter, so they are moved to a candidate list and the later
// digits scan just that list.
//
// The output pass walks the segment in position order and keeps key > T, and
// key == T while the running count of equal keys (across the cluster, in
// position order) is below the number still needed.  That yields the selected
// positions already sorted ascending, with ties going to the lower position,
// and needs no sort.  Rows with klen <= k return 0..klen-1 then -1.
#include "dsa_kernels.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 256;
constexpr int kBins = 2048;
constexpr int kCacheCap = 16384;   // keys of the segment kept in smem
constexpr int kCandCap = 3072;     // candidates of the threshold bin
constexpr int kItems = 8;          // consecutive keys per thread in the output pass

struct TopkSmem {
  uint32_t hist[2][kBins];
  uint32_t cache[kCacheCap];
  uint32_t cand_key[kCandCap];
  int32_t cand_pos[kCandCap];
  uint32_t scan_tmp[2][kThreads / 32];
  uint32_t counts[4];              // n_gt, n_eq of this CTA (read by the cluster)
  uint32_t cand_n;
  uint32_t sel_bin;
  uint32_t sel_need;
};

__device__ __forceinline__ uint32_t excl_prefix(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    uint32_t s = tmp[w];
    before += (w < warp) ? s : 0u;
    all += s;
  }
  __syncthreads();
  if (total) *total = all;
  return before + x - v;
}

__device__ __forceinline__ uint32_t excl_suffix(uint32_t v, uint32_t* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t y = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x += y;
  }
  if (lane == 0) tmp[warp] = x;
  __syncthreads();
  uint32_t after = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) after += (w > warp) ? tmp[w] : 0u;
  __syncthreads();
  return after + x - v;
}

// Warp-aggregated shared histogram increment; every lane of the warp must call it.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool valid, uint32_t bin) {
  const uint32_t key = valid ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  const int leader = __ffs(peers) - 1;
  if (valid && (int)(threadIdx.x & 31) == leader) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Sum the cluster's histograms `which`, then find the bin where the count from
// the top reaches `need`.  Writes sel_bin / sel_need (need left inside the bin).
__device__ void select_bin(TopkSmem& S, int which, uint32_t need, uint32_t csize) {
  constexpr int per = kBins / kThreads;   // 8 consecutive bins per thread
  static_assert(per == 8, "two 16-byte loads per CTA");
  uint32_t tot[per];
  const uint32_t* mine = &S.hist[which][threadIdx.x * per];
  if (csize == 1) {
#pragma unroll
    for (int i = 0; i < per; ++i) tot[i] = mine[i];
  } else {
    // issue every remote load first, then add (the loads overlap in flight)
    uint4 v[8][2];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < (int)csize) {
        const uint32_t addr = mapa(mine, (uint32_t)r);
        v[r][0] = ld_dsmem_v4(addr);
        v[r][1] = ld_dsmem_v4(addr + 16);
      } else {
        v[r][0] = v[r][1] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int i = 0; i < per; ++i) tot[i] = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      tot[0] += v[r][0].x; tot[1] += v[r][0].y; tot[2] += v[r][0].z; tot[3] += v[r][0].w;
      tot[4] += v[r][1].x; tot[5] += v[r][1].y; tot[6] += v[r][1].z; tot[7] += v[r][1].w;
    }
  }
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) local += tot[i];
  uint32_t cum = excl_suffix(local, S.scan_tmp[0]);
#pragma unroll
  for (int i = per - 1; i >= 0; --i) {
    const uint32_t c = tot[i];
    if (cum < need && cum + c >= need) {
      S.sel_bin = threadIdx.x * per + i;
      S.sel_need = need - cum;
    }
    cum += c;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smraw);
  trace_kernel(a.status, DSA_KERNEL_TOPK);
  const uint32_t csize = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int t = blockIdx.x / csize;
  const int tid = threadIdx.x;
  const int k = a.topk;
  const int klen = a.row_klen[t];
  int32_t* out = a.idx + (int64_t)t * k;

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

  for (int i = tid; i < kBins; i += kThreads) { S.hist[0][i] = 0; S.hist[1][i] = 0; }
  if (tid == 0) S.cand_n = 0;
  __syncthreads();

  auto key_at = [&](int i) -> uint32_t {
    return i < ncache ? S.cache[i] : float_key(__ldcg(srow + i));
  };

  // ---- digit 0: load the segment, cache its keys, histogram bits 31..21
  for (int base = 0; base < n; base += kThreads * 4) {
    const int i = base + tid * 4;
    uint32_t kk[4];
    bool v[4];
    if (i + 3 < n) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(srow + i));
      kk[0] = float_key(f.x); kk[1] = float_key(f.y); kk[2] = float_key(f.z); kk[3] = float_key(f.w);
      v[0] = v[1] = v[2] = v[3] = true;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[e] = i + e < n;
        kk[e] = v[e] ? float_key(__ldcg(srow + i + e)) : 0u;
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (v[e] && i + e < kCacheCap) S.cache[i + e] = kk[e];
      hist_add(S.hist[0], v[e], kk[e] >> 21);
    }
  }
  cluster_sync();
  select_bin(S, 0, (uint32_t)k, csize);
  const uint32_t b0 = S.sel_bin;
  uint32_t need = S.sel_need;

  // ---- candidates of the threshold bin (if they fit)
  const uint32_t local_b0 = S.hist[0][b0];
  const bool use_cand = local_b0 <= (uint32_t)kCandCap;
  if (use_cand) {
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      if (i < n) {
        const uint32_t key = key_at(i);
        if ((key >> 21) == b0) {
          const uint32_t slot = atomicAdd(&S.cand_n, 1u);
          S.cand_key[slot] = key;
          S.cand_pos[slot] = i;
        }
      }
    }
    __syncthreads();
  }
  const int ncand = use_cand ? (int)S.cand_n : n;

  // ---- digits 1 and 2 over the candidates (or the whole segment)
  uint32_t prefix = b0;          // digits found so far
  int prefix_shift = 21;         // key >> prefix_shift == prefix for a match
  const int shifts[2] = {10, 0};
  const uint32_t masks[2] = {0x7FFu, 0x3FFu};
#pragma unroll
  for (int d = 0; d < 2; ++d) {
    const int which = (d == 0) ? 1 : 0;
    if (d == 1) {
      for (int i = tid; i < kBins; i += kThreads) S.hist[0][i] = 0;
      __syncthreads();
    }
    for (int base = 0; base < ncand; base += kThreads) {
      const int i = base + tid;
      bool v = i < ncand;
      uint32_t key = 0;
      if (v) key = use_cand ? S.cand_key[i] : key_at(i);
      v = v && ((key >> prefix_shift) == prefix);
      hist_add(S.hist[which], v, (key >> shifts[d]) & masks[d]);
    }
    cluster_sync();
    select_bin(S, which, need, csize);
    prefix = (prefix << (prefix_shift - shifts[d])) | S.sel_bin;
    prefix_shift = shifts[d];
    need = S.sel_need;
  }
  const uint32_t T = prefix;     // the k-th largest key

  // ---- counts of this segment, shared with the cluster
  uint32_t my_gt = 0, my_eq = 0;
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t key = key_at(i);
    my_gt += key > T;
    my_eq += key == T;
  }
  uint32_t tot_gt, tot_eq;
  excl_prefix(my_gt, S.scan_tmp[0], &tot_gt);
  excl_prefix(my_eq, S.scan_tmp[1], &tot_eq);
  if (tid == 0) { S.counts[0] = tot_gt; S.counts[1] = tot_eq; }
  cluster_sync();
  uint32_t out_base = 0, eq_base = 0;
  for (uint32_t r = 0; r < rank; ++r) {
    const uint32_t g = csize == 1 ? 0u : ld_dsmem_u32(mapa(&S.counts[0], r));
    const uint32_t e = csize == 1 ? 0u : ld_dsmem_u32(mapa(&S.counts[1], r));
    const uint32_t take = (eq_base >= need) ? 0u : min(e, need - eq_base);
    out_base += g + take;
    eq_base += e;
  }

  // ---- ordered output pass
  for (int base = 0; base < n; base += kThreads * kItems) {
    const int i0 = base + tid * kItems;
    uint32_t keys[kItems];
    uint32_t c_eq = 0;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      keys[e] = (i0 + e < n) ? key_at(i0 + e) : 0u;
      c_eq += (i0 + e < n) && keys[e] == T;
    }
    uint32_t eq_tile;
    uint32_t eq_rank = eq_base + excl_prefix(c_eq, S.scan_tmp[0], &eq_tile);
    uint32_t sel_flags = 0, c_sel = 0;
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      const bool valid = i0 + e < n;
      bool sel = valid && keys[e] > T;
      if (valid && keys[e] == T) {
        sel = eq_rank < need;
        ++eq_rank;
      }
      sel_flags |= (sel ? 1u : 0u) << e;
      c_sel += sel;
    }
    uint32_t sel_tile;
    uint32_t pos = out_base + excl_prefix(c_sel, S.scan_tmp[1], &sel_tile);
#pragma unroll
    for (int e = 0; e < kItems; ++e)
      if (sel_flags >> e & 1u) {
        if (pos < (uint32_t)k) out[pos] = lo + i0 + e;
        ++pos;
      }
    out_base += sel_tile;
    eq_base += eq_tile;
  }
  cluster_sync();   // keep this CTA's smem alive until the cluster's remote reads are done
}

}  // namespace

size_t topk_ws_bytes() { return 0; }

dsa_status launch_topk(const TopkArgs& a, int max_klen, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  int csize = 1;
  while (csize < 8 && (int64_t)csize * kCacheCap < (int64_t)max_klen) csize <<= 1;
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
