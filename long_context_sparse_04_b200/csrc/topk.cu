// topk.cu - per-row top-k selection by radix select ("DeepSeek Sparse
// Attention DSA Architecture Guide", section "Stage 2: Fine-Grained Token
// Selection and Output Computation", selection equation S_t = TopK(I[t,:], k)).
//
// One cluster of `csize` CTAs (1..8, 512 threads each) per query row.  CTA r
// copies segment r of the row into shared memory (cp.async, all pieces in
// flight at once) and turns it in place into order-preserving uint32 keys
// (float -> key, -0 mapped to +0).  Full passes read four keys per thread.
//
// 1. Histogram of the top 12 key bits; the cluster merges the histograms
//    (CTA r sums a slice of the bins over the cluster through distributed
//    shared memory) and every CTA finds the bin B0 holding the k-th largest
//    key, the rank `need0` of that key inside the bin, and the bin's size c0.
// 2. Only keys in bin B0 or above can be selected (about k plus one bin per
//    row, ~2% of the keys).  They are marked in a bitmap of the segment, one
//    32-bit word per thread; every later pass visits set bits only.
// 3. When c0 is small (the usual case) every CTA sends its keys of bin B0,
//    and its count of keys above B0, to every CTA of the cluster; after one
//    cluster barrier each CTA finishes the selection alone: two more 10-bit
//    digits over the c0 gathered keys give the k-th largest key T and the
//    number `need` of keys equal to T that are taken.  Otherwise the last two
//    digits run as cluster-wide histograms like step 1.
// 4. The output pass walks the marked keys in position order (thread w owns
//    positions [32w, 32w+32); a block scan of the per-thread counts orders
//    the threads) and keeps key > T, and key == T while the number of equal
//    keys before it (across the cluster, in position order) is below `need`.
//    The positions come out ascending with ties going to the lower position,
//    without a sort.  A segment longer than the cache (rows past 8 * 16384
//    keys) skips the bitmap and scans the segment instead, warp w owning a
//    contiguous range and warp ballots giving the order inside it.
// Rows with klen <= k return 0..klen-1 then -1.
//
// Batches of at least two rows per SM longer than one CTA's cache (long
// prefill chunks) run topk_row_kernel instead (further below): one CTA per
// row streaming the scores, no cluster.
#include "dsa_kernels.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins0 = 4096;       // first digit: bits 31..20
constexpr int kBins = 1024;        // second and third digits: bits 19..10, 9..0
constexpr int kCacheCap = 16384;   // keys of the segment kept in smem
constexpr int kMaxCluster = 8;
constexpr int kGatherCap = 2048;   // threshold-bin keys of a row gathered in every CTA
constexpr int kStampsPerCta = 16;

// clock64 stamps of the first cluster, [rank][event], when a trace buffer is set
__device__ __forceinline__ void kstamp(long long* tr, uint32_t csize, uint32_t rank, int ev) {
  if (tr != nullptr && blockIdx.x < csize && threadIdx.x == 0)
    tr[rank * kStampsPerCta + ev] = clock64();
}

struct TopkSmem {
  uint32_t keys[kCacheCap];
  uint32_t hist[kBins0];
  uint32_t slice[kBins0 / 2];            // merged slice (csize >= 2); later a local histogram
  uint32_t bits[kCacheCap / 32];         // keys in bin B0 or above
  uint32_t gather[kGatherCap];           // keys of bin B0 of the whole row, by rank
  uint32_t lhist[2][kBins];              // local histograms of the last two digits
  uint32_t above[kMaxCluster];           // keys above bin B0, per rank
  uint32_t cnt_b0[kMaxCluster];          // keys in bin B0, per rank (fused path)
  uint32_t slice_tot[kMaxCluster];       // slice totals of every CTA
  uint32_t counts[kMaxCluster][2];       // (n_gt, n_eq) of every CTA (radix path)
  uint32_t warp_tmp[kWarps];
  uint32_t warp_cnt[kWarps][2];
  uint32_t sel_bin, sel_need, sel_cnt;
  uint32_t goff, gcount;
};

// Sum over the block (512 threads); every thread gets the total.
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  uint32_t all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) all += tmp[w];
  __syncthreads();
  return all;
}

// Exclusive prefix over the block of one value per thread, in thread order.
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
  *total = all;
  return before + x - v;
}

// Among `nb` bins (higher bins hold larger keys) whose counts are at `bins` -
// in CTA `owner`'s shared memory when `remote` - find the bin holding the
// need-th largest key, given `above` keys in higher bins.  Sets S.sel_bin
// (bin_base + bin), S.sel_need (rank inside the bin), S.sel_cnt (its count).
__device__ void search_bins(TopkSmem& S, const uint32_t* bins, bool remote, uint32_t owner, int nb,
                            int bin_base, uint32_t above, uint32_t need) {
  const int tid = threadIdx.x;
  const int per = (nb + kThreads - 1) / kThreads;   // 1..8
  uint32_t mine[8];
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = tid * per + i;
    mine[i] = 0;
    if (i < per && j < nb) mine[i] = remote ? ld_dsmem_u32(mapa(&bins[j], owner)) : bins[j];
    local += mine[i];
  }
  uint32_t tot;
  const uint32_t before = block_excl_prefix(local, S.warp_tmp, &tot);
  uint32_t cum = above + (tot - before - local);      // keys in bins above this thread's
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (i < per) {
      const uint32_t c = mine[i];
      if (cum < need && cum + c >= need) {
        S.sel_bin = (uint32_t)(bin_base + tid * per + i);
        S.sel_need = need - cum;
        S.sel_cnt = c;
      }
      cum += c;
    }
  }
  __syncthreads();
}

// Warp-level search of 1024 local bins: the bin holding the need-th largest
// key, and the rank of that key inside it.  Lane L sums bins [32L, 32L+32)
// (eight 16-byte loads in a lane-rotated order, so the eight lanes of each
// load phase hit distinct banks); suffix sums over the lanes locate the lane
// L* holding the key, then the warp reads L*'s 32 bins one per lane and a
// second suffix scan locates the bin.
__device__ __forceinline__ void warp_search_1024(const uint32_t* bins, uint32_t need,
                                                 uint32_t* sel_bin, uint32_t* sel_need) {
  const int lane = threadIdx.x & 31;
  const uint4* mine = reinterpret_cast<const uint4*>(bins + 32 * lane);
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 x = mine[(i + lane) & 7];
    s += x.x + x.y + x.z + x.w;
  }
  auto suffix = [&](uint32_t v) {                      // sum over lanes >= this one
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, v, off);
      if (lane + off < 32) v += y;
    }
    return v;
  };
  const uint32_t above = suffix(s) - s;                // keys in the bins of higher lanes
  const uint32_t hit = __ballot_sync(0xffffffffu, above < need && above + s >= need);
  const int ls = __ffs(hit) - 1;                       // exactly one lane
  const uint32_t base = __shfl_sync(0xffffffffu, above, ls);
  const uint32_t c = bins[32 * ls + lane];
  const uint32_t cum = base + suffix(c) - c;           // keys in higher bins
  if (cum < need && cum + c >= need) {
    *sel_bin = (uint32_t)(32 * ls + lane);
    *sel_need = need - cum;
  }
}

// The bin of the need-th largest key among `nbins` bins of S.hist summed over
// the cluster (S.sel_* on every CTA).  Two cluster barriers.
__device__ void cluster_select(TopkSmem& S, int nbins, uint32_t need, uint32_t csize,
                               uint32_t rank) {
  const int tid = threadIdx.x;
  if (csize == 1) {
    __syncthreads();                                  // the histogram is complete
    search_bins(S, S.hist, false, 0, nbins, 0, 0, need);
    return;
  }
  const int slice = nbins / (int)csize;
  const int b0 = (int)rank * slice;
  cluster_sync();                                     // every histogram is complete
  uint32_t part = 0;
  for (int j = tid; j < slice; j += kThreads) {
    uint32_t vv[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r)
      vv[r] = r < (int)csize ? ld_dsmem_u32(mapa(&S.hist[b0 + j], (uint32_t)r)) : 0u;
    uint32_t c = 0;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) c += vv[r];
    S.slice[j] = c;
    part += c;
  }
  const uint32_t total = block_sum(part, S.warp_tmp);
  if (tid < (int)csize) st_dsmem_u32(mapa(&S.slice_tot[rank], (uint32_t)tid), total);
  cluster_sync();                                     // slices and their totals published
  uint32_t owner = 0, above = 0;                      // slices of higher rank hold higher bins
  for (int r = (int)csize - 1; r >= 0; --r) {
    const uint32_t tot = S.slice_tot[r];
    if (above + tot >= need) { owner = (uint32_t)r; break; }
    above += tot;
  }
  search_bins(S, S.slice, owner != rank, owner, slice, (int)owner * slice, above, need);
}

// kHist: the indexer has built each row's histogram of bits 31..20 (a.hist);
// the first selection pass and its cluster merge are skipped, and the row's
// histogram is zeroed once every CTA of the row has read it.
template <bool kHist>
__global__ void __launch_bounds__(kThreads, 2) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smraw);
  pdl_launch_dependents();
  pdl_wait();                                // the scores come from the previous kernel
  trace_kernel(a.status, DSA_KERNEL_TOPK);
  const uint32_t csize = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int t = blockIdx.x / csize;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.topk;
  const int klen = a.row_klen[t];
  int32_t* out = a.idx + (int64_t)t * k;

  uint32_t* const ghist = kHist ? a.hist + (int64_t)t * kBins0 : nullptr;
  kstamp(a.trace, csize, rank, 0);
  if (klen <= k) {  // uniform over the cluster; no DSMEM was touched
    for (int i = rank * kThreads + tid; i < k; i += csize * kThreads) out[i] = i < klen ? i : -1;
    if (kHist)
      for (int i = rank * kThreads + tid; i < kBins0; i += csize * kThreads) ghist[i] = 0u;
    return;
  }

  const float* row = a.scores + (int64_t)t * a.ld_scores;
  const int seg = (((klen + (int)csize - 1) / (int)csize) + 3) & ~3;
  const int lo = min((int)rank * seg, klen);
  const int n = min(lo + seg, klen) - lo;
  const int ncache = min(n, kCacheCap);     // n > kCacheCap only past 8 * 16384 keys
  const int nvec = (n + 3) >> 2;
  const float* srow = row + lo;

  // ---- the segment into shared memory: every 16-byte piece in flight at once
  {
    const int n4 = (reinterpret_cast<uintptr_t>(srow) & 15) == 0 ? (ncache >> 2) : 0;
    for (int i = tid; i < n4; i += kThreads) cp_async_16(&S.keys[4 * i], srow + 4 * i);
    for (int i = 4 * n4 + tid; i < ncache; i += kThreads)
      S.keys[i] = __float_as_uint(__ldcg(srow + i));
  }
  if (kHist) {
    // the threshold bin from the row's histogram, while the segment lands
    for (int i = tid; i < kBins0 / 4; i += kThreads)
      reinterpret_cast<uint4*>(S.hist)[i] = __ldcg(reinterpret_cast<const uint4*>(ghist) + i);
    __syncthreads();
    search_bins(S, S.hist, false, 0, kBins0, 0, 0, (uint32_t)k);
  } else {
    for (int i = tid; i < kBins0; i += kThreads) S.hist[i] = 0;
  }
  cp_async_wait_all();
  __syncthreads();
  kstamp(a.trace, csize, rank, 1);
  const bool use_bits = n <= kCacheCap;               // uniform over the CTA

  // four keys starting at 4v (converted); entries at or past n are garbage
  auto key4 = [&](int v) -> uint4 {
    if (4 * v < ncache) return *reinterpret_cast<const uint4*>(&S.keys[4 * v]);
    uint32_t q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = 4 * v + j < n ? float_key(__ldcg(srow + 4 * v + j)) : 0u;
    return make_uint4(q[0], q[1], q[2], q[3]);
  };
  auto nvalid = [&](int v) { return min(4, n - 4 * v); };

  // ---- 1. keys in place, histogram of bits 31..20, cluster-wide bin B0
  // (the fused path converts the keys in the bitmap pass below)
#pragma unroll 2
  for (int v = tid; v < ((kHist && use_bits) ? 0 : nvec); v += kThreads) {
    uint32_t q[4];
    if (4 * v < ncache) {
      const uint4 raw = *reinterpret_cast<const uint4*>(&S.keys[4 * v]);
      q[0] = float_key(__uint_as_float(raw.x));
      q[1] = float_key(__uint_as_float(raw.y));
      q[2] = float_key(__uint_as_float(raw.z));
      q[3] = float_key(__uint_as_float(raw.w));
      *reinterpret_cast<uint4*>(&S.keys[4 * v]) = make_uint4(q[0], q[1], q[2], q[3]);
    } else {
      const uint4 g = key4(v);
      q[0] = g.x; q[1] = g.y; q[2] = g.z; q[3] = g.w;
    }
    if (!kHist) {
      const int nv = nvalid(v);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j < nv) atomicAdd(&S.hist[q[j] >> 20], 1u);
    }
  }
  kstamp(a.trace, csize, rank, 2);
  if (!kHist) cluster_select(S, kBins0, (uint32_t)k, csize, rank);
  const uint32_t B0 = S.sel_bin, need0 = S.sel_need, c0 = S.sel_cnt;
  kstamp(a.trace, csize, rank, 3);

  // ---- 2. bitmap of the keys in bin B0 or above (segments held in smem):
  // lanes 8i..8i+7 of a round hold the 32 keys of one word; the fused path
  // turns the scores into keys here, in the same pass (thread tid holds the
  // same vectors tid, tid + 512, ... as the conversion loop above)
  const int nwords = (n + 31) >> 5;                   // <= 512 = kThreads when use_bits
  for (int i = tid; i < 2 * kBins; i += kThreads) (&S.lhist[0][0])[i] = 0;
  if (tid == 0) S.gcount = 0;
  uint32_t cb_local = 0, ca_local = 0;                // fused path: keys in bin B0 / above it
  if (use_bits) {
    for (int base = warp * 32; base < nvec; base += kThreads) {
      const int v = base + lane;
      const bool inb = v < nvec;
      uint4 g = inb ? *reinterpret_cast<const uint4*>(&S.keys[4 * v]) : make_uint4(0, 0, 0, 0);
      if (kHist && inb) {
        g = make_uint4(float_key(__uint_as_float(g.x)), float_key(__uint_as_float(g.y)),
                       float_key(__uint_as_float(g.z)), float_key(__uint_as_float(g.w)));
        *reinterpret_cast<uint4*>(&S.keys[4 * v]) = g;
      }
      const uint32_t q[4] = {g.x, g.y, g.z, g.w};
      const int nv = inb ? nvalid(v) : 0;
      uint32_t m = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t bin = q[j] >> 20;
        m |= (j < nv && bin >= B0) ? (1u << j) : 0u;
        if (kHist && j < nv) { cb_local += bin == B0; ca_local += bin > B0; }
      }
      m <<= 4 * (lane & 7);
      m |= __shfl_xor_sync(0xffffffffu, m, 1);
      m |= __shfl_xor_sync(0xffffffffu, m, 2);
      m |= __shfl_xor_sync(0xffffffffu, m, 4);
      if ((lane & 7) == 0 && inb) S.bits[v >> 3] = m;
    }
  }
  if (kHist && !use_bits) {
    for (int v = tid; v < nvec; v += kThreads) {
      const uint4 g = key4(v);
      const uint32_t q[4] = {g.x, g.y, g.z, g.w};
      const int nv = nvalid(v);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j < nv) { cb_local += (q[j] >> 20) == B0; ca_local += (q[j] >> 20) > B0; }
    }
  }
  __syncthreads();
  const uint32_t myword = (use_bits && tid < nwords) ? S.bits[tid] : 0u;
  const uint32_t* const mykeys = &S.keys[32 * tid];
  // fused path: this segment's counts of bin B0 and above it to every CTA of
  // the row (the staged path reads them from the per-CTA histograms), then
  // the row's global histogram is cleared for the next call
  uint32_t goff_h = 0;
  if (kHist) {
    uint32_t cb, ca;
    if (use_bits) {                                   // both counts <= 16384: one packed sum
      const uint32_t both = block_sum((ca_local << 16) | cb_local, S.warp_tmp);
      cb = both & 0xFFFFu;
      ca = both >> 16;
    } else {
      cb = block_sum(cb_local, S.warp_tmp);
      ca = block_sum(ca_local, S.warp_tmp);
    }
    if (tid < (int)csize) {
      if ((uint32_t)tid == rank) {
        S.cnt_b0[rank] = cb;
        S.above[rank] = ca;
      } else {
        st_dsmem_u32(mapa(&S.cnt_b0[rank], (uint32_t)tid), cb);
        st_dsmem_u32(mapa(&S.above[rank], (uint32_t)tid), ca);
      }
    }
    cluster_sync();                                   // every CTA has read the row's histogram
    if (rank == 0)
      for (int i = tid; i < kBins0 / 4; i += kThreads)
        reinterpret_cast<uint4*>(ghist)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (uint32_t r = 0; r < rank; ++r) goff_h += S.cnt_b0[r];

  }
  kstamp(a.trace, csize, rank, 4);

  // ---- 3. T, `need`, and this CTA's offsets in the cluster-wide order:
  // out_base = keys the lower-ranked CTAs select, eq_base = their keys == T
  uint32_t T, need, out_base = 0, eq_base = 0;
  const bool gathered = c0 <= (uint32_t)kGatherCap;   // uniform over the cluster
  if (gathered) {
    // where this CTA's bin-B0 keys go in the gathered list: after those of
    // lower ranks (their histograms still hold their counts of bin B0; the
    // fused path has exchanged the counts above)
    uint32_t goff = goff_h;
    if (!kHist) {
      if (warp == 0) {
        uint32_t hb = 0;
        if (lane < (int)rank) hb = ld_dsmem_u32(mapa(&S.hist[B0], (uint32_t)lane));
        hb = __reduce_add_sync(0xffffffffu, hb);
        if (lane == 0) S.goff = hb;
      }
      uint32_t ab = 0;                                // keys of this segment above bin B0
      for (int b = (int)B0 + 1 + tid; b < kBins0; b += kThreads) ab += S.hist[b];
      ab = block_sum(ab, S.warp_tmp);                 // also publishes S.goff
      goff = S.goff;
      if (tid < (int)csize) {
        if ((uint32_t)tid == rank) S.above[rank] = ab;
        else st_dsmem_u32(mapa(&S.above[rank], (uint32_t)tid), ab);
      }
    }
    auto send = [&](uint32_t key) {
      const uint32_t slot = goff + atomicAdd(&S.gcount, 1u);
      // only a row histogram that does not count this row's scores (a workspace
      // used before dsa_workspace_init) can overfill the list
      if (slot >= (uint32_t)kGatherCap) return;
      for (uint32_t r = 0; r < csize; ++r) {
        if (r == rank) S.gather[slot] = key;
        else st_dsmem_u32(mapa(&S.gather[slot], r), key);
      }
    };
    if (use_bits) {
      for (uint32_t w = myword; w; w &= w - 1) {
        const uint32_t key = mykeys[__ffs(w) - 1];
        if ((key >> 20) == B0) send(key);
      }
    } else {
      for (int v = tid; v < nvec; v += kThreads) {
        const uint4 g = key4(v);
        const uint32_t q[4] = {g.x, g.y, g.z, g.w};
        const int nv = nvalid(v);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nv && (q[j] >> 20) == B0) send(q[j]);
      }
    }
    // Last cluster barrier of this path: after it no CTA touches another's
    // shared memory, so each may finish and exit on its own.
    cluster_sync();
    kstamp(a.trace, csize, rank, 5);
    // the need0-th largest of the c0 gathered keys: two 10-bit digits, locally
    for (int i = tid; i < (int)c0; i += kThreads)
      atomicAdd(&S.lhist[0][(S.gather[i] >> 10) & 1023u], 1u);
    __syncthreads();
    if (warp == 0) warp_search_1024(S.lhist[0], need0, &S.sel_bin, &S.sel_need);
    __syncthreads();
    const uint32_t p1 = (B0 << 10) | S.sel_bin, n1 = S.sel_need;
    for (int i = tid; i < (int)c0; i += kThreads) {
      const uint32_t key = S.gather[i];
      if ((key >> 10) == p1) atomicAdd(&S.lhist[1][key & 1023u], 1u);
    }
    __syncthreads();
    if (warp == 0) warp_search_1024(S.lhist[1], n1, &S.sel_bin, &S.sel_need);
    __syncthreads();
    T = (p1 << 10) | S.sel_bin;
    need = S.sel_need;
    // gathered keys of lower ranks against T (> T in the high half, == T in
    // the low half; both < 2^16)
    uint32_t g = 0;
    for (int i = tid; i < (int)goff; i += kThreads) {
      const uint32_t key = S.gather[i];
      g += (key > T ? 0x10000u : 0u) + (key == T ? 1u : 0u);
    }
    g = block_sum(g, S.warp_tmp);
    uint32_t ab_before = 0;
    for (uint32_t r = 0; r < rank; ++r) ab_before += S.above[r];
    eq_base = g & 0xFFFFu;
    out_base = ab_before + (g >> 16) + min(eq_base, need);
    kstamp(a.trace, csize, rank, 6);
  } else {
    // the last two digits as cluster-wide histograms
    uint32_t prefix = B0, nd = need0;
    int shift = 20;
#pragma unroll 1
    for (int d = 0; d < 2; ++d) {
      const int nshift = shift - 10;
      for (int i = tid; i < kBins; i += kThreads) S.hist[i] = 0;
      __syncthreads();
      if (use_bits) {
        for (uint32_t w = myword; w; w &= w - 1) {
          const uint32_t key = mykeys[__ffs(w) - 1];
          if ((key >> shift) == prefix) atomicAdd(&S.hist[(key >> nshift) & 1023u], 1u);
        }
      } else {
#pragma unroll 2
        for (int v = tid; v < nvec; v += kThreads) {
          const uint4 g = key4(v);
          const uint32_t q[4] = {g.x, g.y, g.z, g.w};
          const int nv = nvalid(v);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (j < nv && (q[j] >> shift) == prefix) atomicAdd(&S.hist[(q[j] >> nshift) & 1023u], 1u);
        }
      }
      cluster_select(S, kBins, nd, csize, rank);
      prefix = (prefix << 10) | S.sel_bin;
      nd = S.sel_need;
      shift = nshift;
    }
    T = prefix;
    need = nd;
  }

  // ---- 4. counts of keys > T and == T before each thread (bitmap) or warp
  // (segment scan) in position order, and per CTA
  const int cv = ((nvec + kWarps - 1) / kWarps + 31) & ~31;   // segment scan: vectors per warp
  const int w_v0 = min(warp * cv, nvec), w_v1 = min(w_v0 + cv, nvec);
  uint32_t gt_before, eq_before, tot_gt, tot_eq;
  if (use_bits) {
    uint32_t gt_t = 0, eq_t = 0;
    for (uint32_t w = myword; w; w &= w - 1) {
      const uint32_t key = mykeys[__ffs(w) - 1];
      gt_t += key > T;
      eq_t += key == T;
    }
    uint32_t tot;   // > T in the high half, == T in the low half (both <= 16384)
    const uint32_t before = block_excl_prefix((gt_t << 16) | eq_t, S.warp_tmp, &tot);
    gt_before = before >> 16;
    eq_before = before & 0xFFFFu;
    tot_gt = tot >> 16;
    tot_eq = tot & 0xFFFFu;
  } else {
    uint32_t w_gt = 0, w_eq = 0;
#pragma unroll 2
    for (int v = w_v0 + lane; v < w_v1; v += 32) {
      const uint4 g = key4(v);
      const uint32_t q[4] = {g.x, g.y, g.z, g.w};
      const int nv = nvalid(v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w_gt += (j < nv) & (q[j] > T);
        w_eq += (j < nv) & (q[j] == T);
      }
    }
    w_gt = __reduce_add_sync(0xffffffffu, w_gt);
    w_eq = __reduce_add_sync(0xffffffffu, w_eq);
    if (lane == 0) {
      S.warp_cnt[warp][0] = w_gt;
      S.warp_cnt[warp][1] = w_eq;
    }
    __syncthreads();
    gt_before = eq_before = tot_gt = tot_eq = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t gc = S.warp_cnt[w][0], ec = S.warp_cnt[w][1];
      gt_before += w < warp ? gc : 0u;
      eq_before += w < warp ? ec : 0u;
      tot_gt += gc;
      tot_eq += ec;
    }
  }
  if (!gathered) {
    if (tid < (int)csize) {
      if ((uint32_t)tid == rank) {
        S.counts[rank][0] = tot_gt;
        S.counts[rank][1] = tot_eq;
      } else {
        st_dsmem_u32(mapa(&S.counts[rank][0], (uint32_t)tid), tot_gt);
        st_dsmem_u32(mapa(&S.counts[rank][1], (uint32_t)tid), tot_eq);
      }
    }
    // Last cluster barrier of this path (see above).
    cluster_sync();
    for (uint32_t r = 0; r < rank; ++r) {
      const uint32_t e = S.counts[r][1];
      out_base += S.counts[r][0] + ((eq_base >= need) ? 0u : min(e, need - eq_base));
      eq_base += e;
    }
  }
  kstamp(a.trace, csize, rank, 7);

  // ---- ordered output
  uint32_t eq_rank = eq_base + eq_before;             // equal keys before this thread / warp
  uint32_t pos = out_base + gt_before + ((eq_base >= need) ? 0u : min(eq_before, need - eq_base));
  if (use_bits) {
    for (uint32_t w = myword; w; w &= w - 1) {
      const int b = __ffs(w) - 1;
      const uint32_t key = mykeys[b];
      const bool eq = key == T;
      if (key > T || (eq && eq_rank < need)) {
        if (pos < (uint32_t)k) out[pos] = lo + 32 * tid + b;
        ++pos;
      }
      eq_rank += eq;
    }
  } else {
    // lane L of a round holds positions 4(v0+L) .. +3: position order is
    // lane-major, then j
    const uint32_t lt = (1u << lane) - 1;
    for (int v0 = w_v0; v0 < w_v1; v0 += 32) {
      const int v = v0 + lane;
      const bool inb = v < w_v1;
      const uint4 g = inb ? key4(v) : make_uint4(0, 0, 0, 0);
      const uint32_t q[4] = {g.x, g.y, g.z, g.w};
      const int nv = inb ? nvalid(v) : 0;
      bool gt[4], eq[4];
      uint32_t e_before = 0, e_round = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        gt[j] = j < nv && q[j] > T;
        eq[j] = j < nv && q[j] == T;
        const uint32_t bl = __ballot_sync(0xffffffffu, eq[j]);
        e_before += __popc(bl & lt);
        e_round += __popc(bl);
      }
      bool sel[4];
      uint32_t r_eq = eq_rank + e_before;
      uint32_t s_before = 0, s_round = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sel[j] = gt[j] || (eq[j] && r_eq < need);
        r_eq += eq[j];
        const uint32_t bl = __ballot_sync(0xffffffffu, sel[j]);
        s_before += __popc(bl & lt);
        s_round += __popc(bl);
      }
      uint32_t p = pos + s_before;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (sel[j]) {
          if (p < (uint32_t)k) out[p] = lo + 4 * v + j;
          ++p;
        }
      }
      pos += s_round;
      eq_rank += e_round;
    }
  }
  kstamp(a.trace, csize, rank, 8);
}


// ---------------------------------------------------------------------------
// One CTA of 1024 threads per row, no cluster and no copy of the row in shared
// memory: the scores are streamed from global memory (L2) in position order,
// warp w owning a contiguous range of the row.
//   1. The first-digit histogram (bits 31..20): the indexer's (kHist), read and
//      zeroed for the next call, or one pass that builds it.  Its bin search
//      gives B0 (the bin of the k-th largest key), the rank need0 of that key in
//      B0 and the bin's count c0.
//   2. One pass: per warp, the keys above bin B0 are counted and the keys of
//      bin B0 are collected (with the warp that saw them) in shared memory.
//   3. Two 10-bit digits over the c0 collected keys give T (the k-th largest
//      key) and `need` (how many keys equal to T are taken, lowest positions
//      first); the collected keys give each warp's counts of keys > T and == T.
//      When c0 exceeds the collection's capacity (massive ties), two more
//      passes over the row build the digit histograms and one counts per warp.
//   4. A block-wide prefix of the warps' counts gives each warp its place in
//      the output; a last pass writes the selected positions in order.
// The positions come out ascending with ties going to the lower position.
constexpr int kRowThreads = 1024;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowGatherCap = 4096;   // keys of bin B0 collected in shared memory

struct RowSmem {
  uint32_t hist[kBins0];
  uint32_t gather[kRowGatherCap];       // keys of bin B0
  uint8_t gwarp[kRowGatherCap];         // the warp that collected each
  uint32_t lhist[2][kBins];             // the last two digits
  uint32_t wcnt[kRowWarps][4];          // per warp: above B0, in B0 and > T, == T
  uint32_t warp_tmp[kRowWarps];
  uint32_t sel_bin, sel_need, sel_cnt, gcount;
};

// Among 4096 first-digit bins, the bin of the need-th largest key (every
// thread of the block gets it in S.sel_*).
__device__ void row_search0(RowSmem& S, uint32_t need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint4 m = reinterpret_cast<const uint4*>(S.hist)[tid];     // bins 4 tid .. 4 tid + 3
  const uint32_t local = m.x + m.y + m.z + m.w;
  uint32_t x = local;                                              // inclusive prefix in the warp
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.warp_tmp[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kRowWarps; ++w) {
    const uint32_t v = S.warp_tmp[w];
    before += (w < warp) ? v : 0u;
    all += v;
  }
  uint32_t cum = all - (before + x);                               // keys in higher threads' bins
  const uint32_t c[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
  for (int i = 3; i >= 0; --i) {
    if (cum < need && cum + c[i] >= need) {
      S.sel_bin = (uint32_t)(4 * tid + i);
      S.sel_need = need - cum;
      S.sel_cnt = c[i];
    }
    cum += c[i];
  }
  __syncthreads();
}

template <bool kHist>
__global__ void __launch_bounds__(kRowThreads, 1) topk_row_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  RowSmem& S = *reinterpret_cast<RowSmem*>(smraw);
  pdl_launch_dependents();
  pdl_wait();                                // the scores come from the previous kernel
  trace_kernel(a.status, DSA_KERNEL_TOPK);
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.topk;
  const int klen = a.row_klen[t];
  int32_t* out = a.idx + (int64_t)t * k;
  uint32_t* const ghist = kHist ? a.hist + (int64_t)t * kBins0 : nullptr;
  if (klen <= k) {
    for (int i = tid; i < k; i += kRowThreads) out[i] = i < klen ? i : -1;
    if (kHist)
      for (int i = tid; i < kBins0 / 4; i += kRowThreads)
        reinterpret_cast<uint4*>(ghist)[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const float* row = a.scores + (int64_t)t * a.ld_scores;
  // warp w: positions [w0, w1), w0 a multiple of 128; a round is 32 lanes x 4
  const int per_warp = ((klen + 128 * kRowWarps - 1) / (128 * kRowWarps)) * 128;
  const int w0 = min(warp * per_warp, klen), w1 = min(w0 + per_warp, klen);
  const uint32_t lt = (1u << lane) - 1;
  // four keys at position p (a multiple of 4, p < klen <= ld_scores, so the
  // 16 bytes are inside the row); positions at or past w1 give no key
  auto load4 = [&](int p) -> float4 { return __ldcg(reinterpret_cast<const float4*>(row + p)); };

  // ---- 1. first digit
  if (tid < kRowWarps) {
    S.wcnt[tid][0] = S.wcnt[tid][1] = S.wcnt[tid][2] = S.wcnt[tid][3] = 0u;
  }
  if (tid == 0) S.gcount = 0u;
  if (kHist) {
    const uint4 h = __ldcg(reinterpret_cast<const uint4*>(ghist) + tid);
    reinterpret_cast<uint4*>(S.hist)[tid] = h;
    reinterpret_cast<uint4*>(ghist)[tid] = make_uint4(0u, 0u, 0u, 0u);   // for the next call
  } else {
    reinterpret_cast<uint4*>(S.hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int p0 = w0; p0 < w1; p0 += 4 * 128) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + 128 * u + 4 * lane;
        f[u] = p < w1 ? load4(p) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + 128 * u + 4 * lane;
        const float v[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (p + j < w1) atomicAdd(&S.hist[float_key(v[j]) >> 20], 1u);
      }
    }
  }
  __syncthreads();
  row_search0(S, (uint32_t)k);
  const uint32_t B0 = S.sel_bin, need0 = S.sel_need, c0 = S.sel_cnt;
  const bool gathered = c0 <= (uint32_t)kRowGatherCap;   // uniform over the block

  // ---- 2. keys above B0 per warp; the keys of B0 collected
  {
    uint32_t above = 0;
    for (int p0 = w0; p0 < w1; p0 += 4 * 128) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + 128 * u + 4 * lane;
        f[u] = p < w1 ? load4(p) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + 128 * u + 4 * lane;
        const float v[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool in = p + j < w1;
          const uint32_t key = float_key(v[j]);
          const uint32_t bin = key >> 20;
          above += (in && bin > B0) ? 1u : 0u;
          if (gathered) {
            const bool mine = in && bin == B0;
            const uint32_t bl = __ballot_sync(0xffffffffu, mine);
            if (bl) {
              uint32_t base = 0;
              if (lane == 0) base = atomicAdd(&S.gcount, (uint32_t)__popc(bl));
              base = __shfl_sync(0xffffffffu, base, 0);
              if (mine) {
                const uint32_t slot = base + __popc(bl & lt);
                if (slot < (uint32_t)kRowGatherCap) {   // always, with consistent counts
                  S.gather[slot] = key;
                  S.gwarp[slot] = (uint8_t)warp;
                }
              }
            }
          }
        }
      }
    }
    above = __reduce_add_sync(0xffffffffu, above);
    if (lane == 0) S.wcnt[warp][0] = above;
  }
  for (int i = tid; i < 2 * kBins; i += kRowThreads) (&S.lhist[0][0])[i] = 0u;
  __syncthreads();
  // the histogram must count exactly the keys of bin B0 (a workspace used
  // before dsa_workspace_init can hold other counts)
  if (kHist && gathered && tid == 0 && S.gcount != c0) set_status(a.status, DSA_ERR_WORKSPACE, t);

  // ---- 3. T and `need`; per warp, keys of B0 above T and equal to it
  uint32_t T, need;
  if (gathered) {
    for (int i = tid; i < (int)c0; i += kRowThreads) atomicAdd(&S.lhist[0][(S.gather[i] >> 10) & 1023u], 1u);
    __syncthreads();
    if (warp == 0) warp_search_1024(S.lhist[0], need0, &S.sel_bin, &S.sel_need);
    __syncthreads();
    const uint32_t p1 = (B0 << 10) | S.sel_bin, n1 = S.sel_need;
    for (int i = tid; i < (int)c0; i += kRowThreads) {
      const uint32_t key = S.gather[i];
      if ((key >> 10) == p1) atomicAdd(&S.lhist[1][key & 1023u], 1u);
    }
    __syncthreads();
    if (warp == 0) warp_search_1024(S.lhist[1], n1, &S.sel_bin, &S.sel_need);
    __syncthreads();
    T = (p1 << 10) | S.sel_bin;
    need = S.sel_need;
    for (int i = tid; i < (int)c0; i += kRowThreads) {
      const uint32_t key = S.gather[i];
      const int w = S.gwarp[i];
      if (key > T) atomicAdd(&S.wcnt[w][1], 1u);
      else if (key == T) atomicAdd(&S.wcnt[w][2], 1u);
    }
  } else {
    // massive ties in bin B0: the last two digits and the per-warp counts by passes
    uint32_t prefix = B0, nd = need0;
#pragma unroll 1
    for (int d = 0; d < 2; ++d) {
      const int shift = 20 - 10 * d, nshift = shift - 10;
      for (int p = w0 + 4 * lane; p < w1; p += 128) {
        const float4 f = load4(p);
        const float v[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t key = float_key(v[j]);
          if (p + j < w1 && (key >> shift) == prefix) atomicAdd(&S.lhist[d][(key >> nshift) & 1023u], 1u);
        }
      }
      __syncthreads();
      if (warp == 0) warp_search_1024(S.lhist[d], nd, &S.sel_bin, &S.sel_need);
      __syncthreads();
      prefix = (prefix << 10) | S.sel_bin;
      nd = S.sel_need;
    }
    T = prefix;
    need = nd;
    uint32_t gt = 0, eq = 0;
    for (int p = w0 + 4 * lane; p < w1; p += 128) {
      const float4 f = load4(p);
      const float v[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t key = float_key(v[j]);
        const bool in = p + j < w1;
        gt += (in && (key >> 20) == B0 && key > T) ? 1u : 0u;
        eq += (in && key == T) ? 1u : 0u;
      }
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if (lane == 0) {
      S.wcnt[warp][1] = gt;
      S.wcnt[warp][2] = eq;
    }
  }
  __syncthreads();

  // ---- 4. this warp's place in the output, then the ordered output pass
  uint32_t pos = 0, eq_rank = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t e = S.wcnt[w][2];
    pos += S.wcnt[w][0] + S.wcnt[w][1] + (eq_rank >= need ? 0u : min(e, need - eq_rank));
    eq_rank += e;
  }
  for (int p00 = w0; p00 < w1; p00 += 4 * 128) {
    float4 fu[4];                            // four rounds' loads in flight
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p00 + 128 * u + 4 * lane;
      fu[u] = p < w1 ? load4(p) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int p0 = p00 + 128 * u;
    const int p = p0 + 4 * lane;
    const float4 f = fu[u];
    const float v[4] = {f.x, f.y, f.z, f.w};
    bool gt[4], eq[4];
    uint32_t e_before = 0, e_round = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t key = float_key(v[j]);
      const bool in = p + j < w1;
      gt[j] = in && key > T;
      eq[j] = in && key == T;
      const uint32_t bl = __ballot_sync(0xffffffffu, eq[j]);
      e_before += __popc(bl & lt);
      e_round += __popc(bl);
    }
    bool sel[4];
    uint32_t r_eq = eq_rank + e_before;
    uint32_t s_before = 0, s_round = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sel[j] = gt[j] || (eq[j] && r_eq < need);
      r_eq += eq[j];
      const uint32_t bl = __ballot_sync(0xffffffffu, sel[j]);
      s_before += __popc(bl & lt);
      s_round += __popc(bl);
    }
    uint32_t q = pos + s_before;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (sel[j]) {
        if (q < (uint32_t)k) out[q] = p + j;
        ++q;
      }
    }
    pos += s_round;
    eq_rank += e_round;
  }
  }
}

}  // namespace

size_t topk_ws_bytes() { return 0; }

// Clusters of `csize` CTAs of `fn` that can be resident at once (0 if the
// query fails), looked up once per device, instantiation and cluster size.
int max_topk_clusters(const void* fn, int which, int csize, size_t smem) {
  static std::atomic<int> cached[2][4][kMaxDevices];
  static std::atomic<bool> have[2][4][kMaxDevices];
  const int ci = csize >= 8 ? 3 : csize >= 4 ? 2 : csize >= 2 ? 1 : 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (have[which][ci][dev].load()) return cached[which][ci][dev].load();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)csize);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = csize;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cached[which][ci][dev].store(n);
  have[which][ci][dev].store(true);
  return n;
}

// Many long rows (a prefill chunk past 16K keys) fill the device with one CTA
// per row; a few long rows (decode) keep each row's scores in the shared
// memory of a cluster, and rows that fit one CTA's cache take one CTA with the
// row in shared memory.
bool topk_uses_clusters(int num_rows, int max_klen) {
  return num_rows < 2 * device_sm_count() || max_klen <= kCacheCap;
}

// The row kernel: one CTA per row, streaming the scores.
dsa_status launch_topk_rows(const TopkArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(RowSmem);
  static std::atomic<bool> attr_done[2][kMaxDevices] = {};
  const void* fn = a.hist ? reinterpret_cast<const void*>(topk_row_kernel<true>)
                          : reinterpret_cast<const void*>(topk_row_kernel<false>);
  if (dsa_status st = set_smem_limit_once(fn, smem, attr_done[a.hist ? 1 : 0])) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.num_rows);
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = a.hist ? cudaLaunchKernelEx(&cfg, topk_row_kernel<true>, a)
                         : cudaLaunchKernelEx(&cfg, topk_row_kernel<false>, a);
  if (e != cudaSuccess) {
    set_error("topk launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status launch_topk(const TopkArgs& a, int max_klen, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  if (!topk_uses_clusters(a.num_rows, max_klen)) return launch_topk_rows(a, stream);
  int csize = 1;
  while (csize < kMaxCluster && (int64_t)csize * kCacheCap < (int64_t)max_klen) csize <<= 1;
  const size_t smem = sizeof(TopkSmem);
  static std::atomic<bool> attr_done[2][kMaxDevices] = {};
  const void* fn = a.hist ? reinterpret_cast<const void*>(topk_kernel<true>)
                          : reinterpret_cast<const void*>(topk_kernel<false>);
  if (dsa_status st = set_smem_limit_once(fn, smem, attr_done[a.hist ? 1 : 0])) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.num_rows * csize));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // A programmatic launch places the clusters while the previous kernel's last
  // CTAs still hold SMs; clusters of four or more CTAs placed piecemeal pack
  // worse, and a grid that fits the device in one wave of clusters may then
  // need two.  Such a grid is launched once the previous kernel is done,
  // unless that kernel lets its dependents launch only at its end (the
  // indexer of this library's fused calls does).
  const bool one_wave =
      csize >= 4 && a.num_rows <= max_topk_clusters(fn, a.hist ? 1 : 0, csize, smem);
  cfg.numAttrs = (one_wave && !a.after_late_trigger) ? 1 : 2;
  cudaError_t e = a.hist ? cudaLaunchKernelEx(&cfg, topk_kernel<true>, a)
                         : cudaLaunchKernelEx(&cfg, topk_kernel<false>, a);
  if (e != cudaSuccess) {
    set_error("topk launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
