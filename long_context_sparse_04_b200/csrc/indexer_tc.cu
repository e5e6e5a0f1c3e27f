// indexer_tc.cu - FP8 lightning indexer on the 5th-generation tensor cores.
//
// Computes, for each query row t and visible key s < klen[t]
//     I[t,s] = k_scale[s] * sum_j w'[t,j] * ReLU(q8[t,j,:] . k8[s,:]),  w' = w * q_scale
// which equals sum_j w[t,j] ReLU(q[t,j] . k[s]) on the dequantised operands
// because both scales are positive and ReLU is positively homogeneous
// ("DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 1: The
// Lightning Indexer": index-score equation, FP8 operands).
//
// Shape of the contraction: one tile is 128 keys (M) x NQ*64 query-heads (N)
// x 128 (K = d_I bytes of e4m3).  A query group is NQ consecutive rows of one
// sequence; all its heads share one pass over the sequence's keys.
//
// Persistent CTAs (one per SM) each own a contiguous range of the flattened
// (group, key tile) list.  A prologue resolves, through the block table, the
// physical cache row of both 64-key halves of every tile of the range into
// shared memory, so the loops below never wait on a dependent global load.
// Roles (576 threads):
//   warp 0      producer (one thread): TMA of the two 64-row key boxes (a box
//               never crosses a 64-token page) into an 8-stage ring (6 when
//               N = 256), and of the group's queries (N x 128 B) into a double
//               buffer.  Per-tile flags computed in the prologue (first / last
//               tile of its group) keep this loop short.
//   warp 18     key scales: the 32 lanes copy each tile's 128 key scales into
//               a scale slot with cp.async, a stage at a time behind the
//               producer, so the epilogue never waits on a global load.
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//               (kind::f8f6f4, e4m3 x e4m3 -> fp32, 4 MMAs of K=32 per tile)
//               into one of four (N <= 128) or two TMEM accumulators; one
//               commit per tile frees the key stage and tells the epilogue
//               that the accumulator is ready.
//   warps 2-17  epilogue in 16/(4*NQ) sets that take alternate tiles (one
//               set's TMEM-load latency overlaps another's math): tcgen05.ld
//               of the accumulator (lane = key), ReLU, head-weighted sum with w'
//               (packed fp32x2 FMAs), times the key's scale, coalesced store.
// The L x H_I per-head score tensor lives only in TMEM.
#include <cstddef>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "dsa_kernels.cuh"

namespace dsa {
namespace {

constexpr int kTileKeys = 128;
constexpr int kDI = 128;
constexpr int kHI = 64;
constexpr int kEpiWarps = 16;
constexpr int kScaleWarp = 2 + kEpiWarps;          // warp 18: key scales into their slots
constexpr int kThreads = 64 + 32 * kEpiWarps + 32;
constexpr int kMaxGroups = 2048;
// At most 511 tiles per CTA: a row's key count inside one CTA then stays below
// 65,536, so the shared-memory score histogram can keep 16-bit counters.
constexpr int kMaxCtaTiles = 511;
constexpr int kKeyTileBytes = kTileKeys * kDI;   // 16 KB
// Key-scale slots: the producer writes tile j's scales into slot j % 16 when it
// fills the tile's key stage, and the epilogue reads them before it releases
// the tile's accumulator.  The producer reaches tile j + 16 only after the MMA
// of tile j + 16 - stages, which needs the accumulator of tile
// j + 16 - stages - accumulators >= j released: 16 >= stages + accumulators
// (10 + 4, or 6 + 2) keeps a slot from being overwritten before it is read.
constexpr int kScaleSlots = 16;

// Key-tile stages in flight: as many as shared memory allows beside the
// queries (and, for NQ <= 2, the score histograms).
template <int NQ>
constexpr int num_stages() { return NQ <= 2 ? 8 : 6; }

// Score histograms (NQ <= 2): for the first hist_slots() groups of a CTA's
// range, per query row of the group, 4096 bins of the top 12 bits of the
// order-preserving key of each score, two 16-bit counters per word.
constexpr int kHistBins = 4096;
template <int NQ>
constexpr int hist_slots() { return NQ <= 2 ? 4 / NQ : 0; }
template <int NQ>
constexpr int hist_words() { return NQ <= 2 ? 4 * kHistBins / 2 : 4; }

// TMEM accumulators per CTA: four of N columns when they fit in 512, else two.
template <int NQ>
constexpr int num_acc() { return NQ * kHI <= 128 ? 4 : 2; }

template <int NQ>
struct __align__(1024) IdxSmem {
  uint8_t keys[num_stages<NQ>()][kKeyTileBytes];
  uint8_t q[2][NQ * kHI * kDI];
  float wq[kEpiWarps][kHI];                             // per epilogue warp: w' of its heads
  float kscale[kScaleSlots][kTileKeys];                 // key scales of tile j in slot j % kScaleSlots
  uint32_t hist[hist_words<NQ>()];                      // [slot][query of group][bin / 2]
  alignas(16) int32_t tile_row[kMaxCtaTiles][2];        // physical row of each 64-key half, -1: none
  int32_t tile_info[kMaxCtaTiles];                      // group << 2 | last tile of group << 1 | first
  int32_t tile_off[kMaxGroups + 1];
  int32_t scan_tmp[kThreads / 32];
  uint64_t full[num_stages<NQ>()], empty[num_stages<NQ>()];
  uint64_t q_full[2], q_empty[2];
  uint64_t acc_empty[4];
  uint32_t tmem_base;
};

// every member the kernel reads as a vector or fills with cp.async sits on a
// 16-byte boundary (tile_row is read as int2, kscale filled 16 bytes at a time)
static_assert(offsetof(IdxSmem<1>, tile_row) % 16 == 0 && offsetof(IdxSmem<2>, tile_row) % 16 == 0 &&
                  offsetof(IdxSmem<4>, tile_row) % 16 == 0, "tile_row alignment");
static_assert(offsetof(IdxSmem<1>, kscale) % 16 == 0 && offsetof(IdxSmem<2>, kscale) % 16 == 0 &&
                  offsetof(IdxSmem<4>, kscale) % 16 == 0, "kscale alignment");
static_assert(offsetof(IdxSmem<1>, wq) % 16 == 0 && offsetof(IdxSmem<2>, wq) % 16 == 0 &&
                  offsetof(IdxSmem<4>, wq) % 16 == 0, "wq alignment");

struct TcArgs {
  long long* trace;           // profiling stamps (CTA 0, first 32 tiles) or null
  uint32_t spin_limit;        // polls of every bounded wait
  uint32_t inject;            // DSA_FAULT_* bits (tests only)
  int num_rows, n_groups;
  const int32_t* row_seq;
  const int32_t* row_klen;
  const float* q_scale;
  const float* w;
  const float* k_scale;
  CacheMap map;
  float* scores;
  int64_t ld;
  uint32_t* hist;             // [num_rows, 4096] score-key histograms to add to, or null
  DeviceStatus* status;
  int late_trigger;           // dependents launch once every CTA's tiles are done
};

// Walks the flattened (group, key tile) list from a start tile.
struct TileIter {
  const int32_t* off;
  int g, kt, ntiles, ng;
  __device__ void start(const int32_t* o, int n_groups, int tile) {
    off = o;
    ng = n_groups;
    int lo = 0, hi = n_groups;            // largest g with off[g] <= tile
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (off[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
    kt = tile - off[g];
    ntiles = off[g + 1] - off[g];
  }
  __device__ void next() {
    if (++kt >= ntiles) {
      kt = 0;
      do {
        if (++g >= ng) { ntiles = 0; return; }   // past the last tile
        ntiles = off[g + 1] - off[g];
      } while (ntiles == 0);
    }
  }
};

__device__ __forceinline__ void istamp(long long* tr, int ev, int j) {
  if (tr != nullptr && blockIdx.x == 0 && j < kTraceBlocks) tr[ev * kTraceBlocks + j] = clock64();
}

// ReLU of two fp32 bit patterns, packed low | high << 32 for an f32x2 operation.
__device__ __forceinline__ unsigned long long relu2(uint32_t a, uint32_t b) {
  return (unsigned long long)__float_as_uint(fmaxf(__uint_as_float(a), 0.f)) |
         ((unsigned long long)__float_as_uint(fmaxf(__uint_as_float(b), 0.f)) << 32);
}
// d = a * b + c on two fp32 lanes at once (fma.rn.f32x2).
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

template <int NQ>
__device__ __forceinline__ int group_max_klen(const TcArgs& a, int g) {
  int mk = 0;
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    const int r = g * NQ + i;
    if (r < a.num_rows) mk = max(mk, a.row_klen[r]);
  }
  return mk;
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  TcArgs a) {
  constexpr int N = NQ * kHI;
  constexpr int kQBytes = N * kDI;
  constexpr int kAcc = num_acc<NQ>();
  constexpr int kStages = num_stages<NQ>();
  extern __shared__ __align__(1024) uint8_t smraw[];
  IdxSmem<NQ>& S = *reinterpret_cast<IdxSmem<NQ>*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lim = a.spin_limit;
  // dependents may launch now, or (late_trigger) once this CTA's tiles are done
  if (!a.late_trigger) pdl_launch_dependents();
  pdl_wait();
  trace_kernel(a.status, DSA_KERNEL_INDEXER_TC);

  // ---- schedule: exclusive scan of key tiles per group (every CTA, redundantly)
  {
    const int chunk = (a.n_groups + kThreads - 1) / kThreads;
    const int g_lo = min(a.n_groups, (int)threadIdx.x * chunk);
    const int g_hi = min(a.n_groups, g_lo + chunk);
    int local = 0;
    for (int g = g_lo; g < g_hi; ++g) {
      const int seq0 = a.row_seq[g * NQ];
      for (int i = 1; i < NQ; ++i) {
        const int r = g * NQ + i;
        if (r < a.num_rows && a.row_seq[r] != seq0) set_status(a.status, DSA_ERR_INVALID_ARG, g);
      }
      const int nt = (group_max_klen<NQ>(a, g) + kTileKeys - 1) / kTileKeys;
      S.tile_off[g + 1] = nt;
      local += nt;
    }
    int x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) S.scan_tmp[warp] = x;
    __syncthreads();
    int run = x - local;
    for (int w2 = 0; w2 < warp; ++w2) run += S.scan_tmp[w2];
    for (int g = g_lo; g < g_hi; ++g) {
      run += S.tile_off[g + 1];
      S.tile_off[g + 1] = run;
    }
    if (threadIdx.x == 0) S.tile_off[0] = 0;
  }
  if (threadIdx.x == 32) {
    // full: the producer lane's arrive (with the key bytes as transactions)
    // plus one cp.async arrival per producer lane for the scales
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 33); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.q_full[i], 1);
      mbar_init(&S.q_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&S.acc_empty[i], 4 * NQ);     // the warps of one epilogue set
    }
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kAcc * N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int total = S.tile_off[a.n_groups];
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int t_begin = min(total, (int)blockIdx.x * per);
  const int t_end = min(total, t_begin + per);
  const int ntile = t_end - t_begin;
  const uint32_t tmem = S.tmem_base;
  if (ntile > kMaxCtaTiles) {           // the host sizes the grid so this cannot happen
    set_status(a.status, DSA_ERR_INVALID_ARG, -2);
  } else {
    // ---- physical rows of both halves of every tile of this CTA's range
    for (int i = threadIdx.x; i < 2 * ntile; i += kThreads) {
      TileIter it;
      it.start(S.tile_off, a.n_groups, t_begin + (i >> 1));
      const int s0 = it.kt * kTileKeys + (i & 1) * 64;
      int row = -1;
      if (s0 < group_max_klen<NQ>(a, it.g)) {
        bool ok = true;
        const int64_t r = a.map.row(a.row_seq[it.g * NQ], s0, a.status, &ok);
        row = ok ? (int32_t)r : -1;
      }
      S.tile_row[i >> 1][i & 1] = row;
      if ((i & 1) == 0) {
        const int j = i >> 1;
        S.tile_info[j] = (it.g << 2) | ((it.kt + 1 == it.ntiles || j + 1 == ntile) ? 2 : 0) |
                         ((it.kt == 0 || j == 0) ? 1 : 0);
      }
    }
  }
  constexpr int kHistSlots = hist_slots<NQ>();
  const bool use_hist = kHistSlots > 0 && a.hist != nullptr;
  if (use_hist)
    for (int i = threadIdx.x; i < hist_words<NQ>(); i += kThreads) S.hist[i] = 0u;
  __syncthreads();
  const bool run = ntile > 0 && ntile <= kMaxCtaTiles;
  // the group of the CTA's first tile: histogram slot of group g is g - g_first
  int g_first = 0;
  if (run) {
    TileIter it0;
    it0.start(S.tile_off, a.n_groups, t_begin);
    g_first = it0.g;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer (lane 0): TMA only
    if (run && lane == 0) {
      // A lean loop: one thread issues every load, so its instruction count
      // per tile bounds the tile rate.
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      const bool tracing = a.trace != nullptr && blockIdx.x == 0;
      int st = 0, qb = 0;
      uint32_t ph = 1, qph = 1;                       // parity to wait for on empty / q_empty
      int qcount = 0, qloads = 0, j = 0;
      bool alive = true;
      for (; j < ntile; ++j) {
        const int info = S.tile_info[j];
        const int2 rr = *reinterpret_cast<const int2*>(S.tile_row[j]);
        if (info & 1) {
          if (qcount > 0) { qb ^= 1; if (qb == 0) qph ^= 1; }
          ++qcount;
          if (!(alive = mbar_wait(&S.q_empty[qb], qph, a.status, 1, lim))) break;
          mbar_expect_tx(&S.q_full[qb], kQBytes);
          tma_load_2d(S.q[qb], &tm_q, &S.q_full[qb], 0, (info >> 2) * NQ * kHI);
          ++qloads;
        }
        if (!(alive = mbar_wait(&S.empty[st], ph, a.status, 2, lim))) break;
        if (tracing) istamp(a.trace, 0, j);
        const uint32_t bytes = (rr.x >= 0 ? kKeyTileBytes / 2 : 0) + (rr.y >= 0 ? kKeyTileBytes / 2 : 0);
        if (bytes == 0) {
          mbar_arrive(&S.full[st]);
        } else {
          mbar_expect_tx(&S.full[st], bytes);
          if (rr.x >= 0) tma_load_2d(S.keys[st], &tm_k, &S.full[st], 0, rr.x);
          if (rr.y >= 0) tma_load_2d(S.keys[st] + kKeyTileBytes / 2, &tm_k, &S.full[st], 0, rr.y);
        }
        if (tracing) istamp(a.trace, 1, j);
        if (++st == kStages) { st = 0; ph ^= 1; }
      }
      // tail: every bulk load issued has landed (also when a wait above ran
      // out and the MMA stopped consuming), then the MMAs have released every
      // stage and query buffer in use, so nothing is still in flight to this
      // CTA's shared memory at exit
      for (int s2 = 0; s2 < kStages && s2 < j; ++s2) {
        const int fills = (j - 1 - s2) / kStages + 1;
        if (!mbar_wait(&S.full[s2], (fills - 1) & 1, a.status, 9, lim)) break;
      }
      for (int q2 = 0; q2 < 2 && q2 < qloads; ++q2) {
        const int fills = (qloads - q2 + 1) / 2;
        if (!mbar_wait(&S.q_full[q2], (fills - 1) & 1, a.status, 10, lim)) break;
      }
      if (alive) {
        for (int s2 = 0; s2 < kStages && s2 < j; ++s2) {
          const int last_use = (j - 1 - s2) / kStages;
          if (!mbar_wait(&S.empty[s2], last_use & 1, a.status, 7, lim)) break;
        }
        for (int q2 = 0; q2 < 2 && q2 < qcount; ++q2) {
          const int last_use = (qcount - 1 - q2) >> 1;
          if (!mbar_wait(&S.q_empty[q2], last_use & 1, a.status, 8, lim)) break;
        }
      }
    }
  } else if (warp == kScaleWarp) {
    // ------------------------------------------------------------ key scales (32 lanes)
    // Follows the producer stage by stage: once a stage is free (the same
    // wait as the producer's), each lane copies 4 of the tile's 128 key
    // scales into the tile's scale slot with cp.async, whose completion
    // arrives on the stage's full barrier.  A separate warp keeps this work
    // out of the producer's loop.
    if (run) {
      const int half = lane >> 4, k4 = 4 * (lane & 15);
      int st = 0;
      uint32_t ph = 1;
      for (int j = 0; j < ntile; ++j) {
        const int2 rr = *reinterpret_cast<const int2*>(S.tile_row[j]);
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&S.empty[st], ph, a.status, 11, lim);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        // scales of keys [64 half + k4, +4): one 16-byte piece when aligned and
        // in range, else four 4-byte pieces (rows past the cache read as 0)
        const int row = half ? rr.y : rr.x;
        float* dst = &S.kscale[j % kScaleSlots][64 * half + k4];
        const int64_t pr = (int64_t)row + k4;
        if (row >= 0 && (reinterpret_cast<uintptr_t>(a.k_scale + pr) & 15) == 0 &&
            pr + 4 <= a.map.num_tokens) {
          cp_async_16(dst, a.k_scale + pr);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool in = row >= 0 && pr + e < a.map.num_tokens;
            cp_async_4_zfill(dst + e, a.k_scale + (in ? pr + e : 0), in);
          }
        }
        cp_async_mbar_arrive(&S.full[st]);
        if (++st == kStages) { st = 0; ph ^= 1; }
      }
      cp_async_wait_all();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && run) {
      // A lean loop (see the producer): descriptors are a base plus a stage or
      // k-step offset in their start-address field (address >> 4).
      constexpr uint32_t idesc = idesc_f8_e4m3(N);
      const bool tracing = a.trace != nullptr && blockIdx.x == 0;
      const uint64_t kd0 = sdesc_sw128(smem_u32(S.keys[0]), 16, 1024);
      const uint64_t qd0 = sdesc_sw128(smem_u32(S.q[0]), 16, 1024);
      constexpr uint64_t kStageStep = kKeyTileBytes >> 4, kQStep = kQBytes >> 4;
      int st = 0, ab = 0, qb = 1;
      uint32_t ph = 0, aph = 1, qph = 1;              // parity to wait for on full / acc_empty / q_full
      for (int j = 0; j < ntile; ++j) {
        const int info = S.tile_info[j];
        if (info & 1) {
          qb ^= 1;
          if (qb == 0) qph ^= 1;
          if (!mbar_wait(&S.q_full[qb], qph, a.status, 3, lim)) break;
        }
        if (!mbar_wait(&S.full[st], ph, a.status, 4, lim)) break;
        if (tracing) istamp(a.trace, 5, j);
        if (!mbar_wait(&S.acc_empty[ab], aph, a.status, 5, lim)) break;
        tc_fence_after();
        if (tracing) istamp(a.trace, 2, j);
        const uint64_t kd = kd0 + (uint64_t)st * kStageStep, qd = qd0 + (uint64_t)qb * kQStep;
        const uint32_t d = tmem + ab * N;
#pragma unroll
        for (int k = 0; k < kDI / 32; ++k) mma_f8(d, kd + 2 * k, qd + 2 * k, idesc, k > 0);
        mma_commit(&S.empty[st]);           // stage free, and accumulator ab ready
        if (info & 2) mma_commit(&S.q_empty[qb]);
        if (tracing) istamp(a.trace, 3, j);
        if (++st == kStages) { st = 0; ph ^= 1; }
        if (++ab == kAcc) { ab = 0; aph ^= 1; }
      }
    }
  } else if (run) {
    // ------------------------------------------------------------ epilogue (warps 2-17)
    // The 16 warps form NSET = 16 / (4*NQ) sets of 4*NQ warps; set k takes the
    // tiles j = k (mod NSET), so the sets sit in different phases and one set's
    // TMEM-load latency overlaps another's arithmetic.  Warp (lq, qi) of a set
    // reduces the 64 heads of query qi for keys 32lq..32lq+31 of its tiles.
    // A wait that times out only marks the warp dead.
    constexpr int WPS = 4 * NQ;
    constexpr int NSET = kEpiWarps / WPS;
    const int e = warp - 2;               // 0..15
    const int set = e / WPS, wi = e % WPS;
    const int lq = warp & 3;              // TMEM lane quarter this warp may access
    const int qi = wi >> 2;
    const int row_in_tile = lq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(lq * 32) << 16;
    TileIter it;
    it.start(S.tile_off, a.n_groups, t_begin);
    for (int k = 0; k < set && k < ntile; ++k) it.next();
    int klen = 0, cur_g = -1;
    bool dead = false;
    for (int j = set; j < ntile; j += NSET) {
      if (it.g != cur_g) {
        cur_g = it.g;
        const int r = it.g * NQ + qi;
        klen = r < a.num_rows ? a.row_klen[r] : 0;
        // w' = w * q_scale of this warp's query into its own slice
        __syncwarp();
        for (int q = lane; q < kHI; q += 32)
          S.wq[e][q] = r < a.num_rows ? a.w[(int64_t)r * kHI + q] * a.q_scale[(int64_t)r * kHI + q] : 0.f;
        __syncwarp();
      }
      const int ab = j % kAcc;
      // the stage's barrier completes when the tile's MMAs are done, which
      // also orders the key scales the producer copied for this tile
      dead = dead || !mbar_wait(&S.empty[j % kStages], (j / kStages) & 1, a.status, 6, lim);
      tc_fence_after();
      const float ks = S.kscale[j % kScaleSlots][row_in_tile];
      if (threadIdx.x == 64) istamp(a.trace, 4, j);
      const uint32_t col = tmem + lane_off + ab * N + qi * kHI;
      uint32_t v0[32], v1[32];
      tmem_ld32(col, v0);
      tmem_ld32(col + 32, v1);
      tmem_wait_ld_regs(v0);
      tmem_wait_ld_regs(v1);
      if (threadIdx.x == 64) istamp(a.trace, 6, j);
      tc_fence_before();
      __syncwarp();
      // values are in registers (a test may withhold the release, so that the
      // MMA issuer's bounded wait runs out)
      if (lane == 0 && !(a.inject & DSA_FAULT_INDEXER_ACC_RELEASE)) mbar_arrive(&S.acc_empty[ab]);
      // sum_h w'_h ReLU(x_h), two heads per packed fp32x2 FMA
      const ulonglong2* wv = reinterpret_cast<const ulonglong2*>(&S.wq[e][0]);
      unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int h = 0; h < 32; h += 4) {
        const ulonglong2 w0 = wv[h / 4], w1 = wv[8 + h / 4];
        acc[0] = ffma2(relu2(v0[h + 0], v0[h + 1]), w0.x, acc[0]);
        acc[1] = ffma2(relu2(v0[h + 2], v0[h + 3]), w0.y, acc[1]);
        acc[2] = ffma2(relu2(v1[h + 0], v1[h + 1]), w1.x, acc[2]);
        acc[3] = ffma2(relu2(v1[h + 2], v1[h + 3]), w1.y, acc[3]);
      }
      float lo[4], hi[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        lo[q] = __uint_as_float((uint32_t)acc[q]);
        hi[q] = __uint_as_float((uint32_t)(acc[q] >> 32));
      }
      const float sum = ((lo[0] + hi[0]) + (lo[1] + hi[1])) + ((lo[2] + hi[2]) + (lo[3] + hi[3]));
      const int s = it.kt * kTileKeys + row_in_tile;
      const float score = sum * ks;
      if (!dead && s < klen) {
        a.scores[(int64_t)(it.g * NQ + qi) * a.ld + s] = score;
        if (use_hist) {
          // the first selection pass of top-k, done here: the bin of this score
          const uint32_t bin = float_key(score) >> 20;
          const int slot = it.g - g_first;
          if (slot < kHistSlots)
            atomicAdd(&S.hist[(slot * NQ + qi) * (kHistBins / 2) + (bin >> 1)], 1u << (16 * (bin & 1)));
          else
            atomicAdd(&a.hist[(int64_t)(it.g * NQ + qi) * kHistBins + bin], 1u);
        }
      }
      if (threadIdx.x == 64) istamp(a.trace, 7, j);
      for (int k = 0; k < NSET; ++k) it.next();
    }
  }
  if (a.late_trigger) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kAcc * N);
  }
  // add this CTA's histograms of its first groups to the rows' global ones
  if (use_hist && run) {
    for (int i = threadIdx.x; i < kHistSlots * NQ * (kHistBins / 2); i += kThreads) {
      const uint32_t v = S.hist[i];
      if (v == 0u) continue;
      const int sq = i / (kHistBins / 2), w = i - sq * (kHistBins / 2);
      const int row = (g_first + sq / NQ) * NQ + sq % NQ;
      if (row >= a.num_rows) continue;
      uint32_t* dst = a.hist + (int64_t)row * kHistBins + 2 * w;
      if (v & 0xFFFFu) atomicAdd(dst, v & 0xFFFFu);
      if (v >> 16) atomicAdd(dst + 1, v >> 16);
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
}

// 2D byte tensor [rows, 128] with 128-byte rows, box 128 x box_rows, 128B swizzle.
bool make_tmap_rows128(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int NQ>
dsa_status launch_nq(const IndexerArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(IdxSmem<NQ>) + 1024;
  static std::atomic<bool> attr[kMaxDevices] = {};
  if (dsa_status st = set_smem_limit_once(reinterpret_cast<const void*>(indexer_tc_kernel<NQ>), smem, attr))
    return st;
  CUtensorMap tm_k;
  if (!make_tmap_rows128(&tm_k, a.idx_k, (uint64_t)a.map.num_tokens, 64)) {
    set_error("indexer_tc: cuTensorMapEncodeTiled failed");
    return DSA_ERR_CUDA;
  }
  const int n_groups_all = (a.num_rows + NQ - 1) / NQ;
  for (int g0 = 0; g0 < n_groups_all; g0 += kMaxGroups) {
    const int ng = min(kMaxGroups, n_groups_all - g0);
    const int r0 = g0 * NQ;
    TcArgs t{};
    t.num_rows = min(a.num_rows - r0, ng * NQ);
    t.n_groups = ng;
    t.row_seq = a.row_seq + r0;
    t.row_klen = a.row_klen + r0;
    t.q_scale = a.q_scale + (int64_t)r0 * kHI;
    t.w = a.w + (int64_t)r0 * kHI;
    t.k_scale = a.idx_k_scale;
    t.map = a.map;
    t.scores = a.scores + (int64_t)r0 * a.ld_scores;
    t.ld = a.ld_scores;
    t.hist = a.hist ? a.hist + (int64_t)r0 * kHistBins : nullptr;
    t.status = a.status;
    t.late_trigger = a.late_trigger;
    t.trace = trace_buffer() ? trace_buffer() + kTraceIdx : nullptr;
    t.spin_limit = fault_spin_limit();
    t.inject = fault_inject();
    CUtensorMap tq;
    if (!make_tmap_rows128(&tq, static_cast<const uint8_t*>(a.q_idx) + (int64_t)r0 * kHI * kDI,
                           (uint64_t)t.num_rows * kHI, NQ * kHI)) {
      set_error("indexer_tc: cuTensorMapEncodeTiled failed");
      return DSA_ERR_CUDA;
    }
    // tiles are at most groups x ceil(max_klen / 128); a CTA takes at most kMaxCtaTiles
    const int64_t tiles = (int64_t)ng * ((a.max_klen + kTileKeys - 1) / kTileKeys);
    const int64_t need = (tiles + kMaxCtaTiles - 1) / kMaxCtaTiles;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, std::max<int64_t>(device_sm_count(), need)));
    indexer_tc_kernel<NQ><<<grid, kThreads, smem, stream>>>(tm_k, tq, t);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      set_error("indexer_tc launch: %s", cudaGetErrorString(e));
      return DSA_ERR_CUDA;
    }
  }
  return DSA_OK;
}

}  // namespace

void* tensor_map_encoder() {
  // a function-local static: initialised once, safely under concurrent first calls
  static void* const fn = [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      return p;
    return static_cast<void*>(nullptr);
  }();
  return fn;
}

bool indexer_tc_supported(const IndexerArgs& a) {
  if (a.idx_dtype != DSA_FP8_E4M3 || a.d_idx != kDI || a.n_idx_heads != kHI) return false;
  if (a.q_scale == nullptr || a.idx_k_scale == nullptr) return false;
  if (a.map.block_table != nullptr && a.map.page_size % 64 != 0) return false;
  if (a.map.num_tokens >= (int64_t)INT32_MAX) return false;
  if (encode_fn() == nullptr) return false;
  return a.q_group == 1 || a.q_group == 2 || a.q_group == 4;
}

bool indexer_tc_hist_supported(const IndexerArgs& a) {
  return indexer_tc_supported(a) && a.q_group <= 2;
}

size_t indexer_ws_bytes(int num_rows, int q_group) {
  return sizeof(int32_t) * (size_t)((num_rows + q_group - 1) / q_group + 1);
}

dsa_status launch_indexer_tc(const IndexerArgs& a, void*, size_t, cudaStream_t stream) {
  if (a.num_rows == 0 || a.max_klen == 0) return DSA_OK;
  switch (a.q_group) {
    case 1: return launch_nq<1>(a, stream);
    case 2: return launch_nq<2>(a, stream);
    default: return launch_nq<4>(a, stream);
  }
}

}  // namespace dsa
