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
// Roles (320 threads):
//   warp 0      producer.  Lane 0: TMA of the two 64-row key boxes (a box never
//               crosses a 64-token page) into a 6-stage ring, and of the group's
//               queries (N x 128 B) into a double buffer.  All 32 lanes: cp.async
//               of the tile's 128 per-key scales into an 8-slot ring.
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//               (kind::f8f6f4, e4m3 x e4m3 -> fp32, 4 MMAs of K=32 per tile)
//               into one of two TMEM accumulators (2 x N columns).
//   warps 2-9   epilogue: tcgen05.ld of the accumulator (lane = key), ReLU,
//               head-weighted sum with w', times k_scale, coalesced fp32 store.
// The L x H_I per-head score tensor lives only in TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "dsa_kernels.cuh"

namespace dsa {
namespace {

constexpr int kTileKeys = 128;
constexpr int kDI = 128;
constexpr int kHI = 64;
constexpr int kStages = 6;
constexpr int kScaleSlots = 8;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 2048;
constexpr int kMaxCtaTiles = 512;
constexpr int kKeyTileBytes = kTileKeys * kDI;   // 16 KB

template <int NQ>
struct __align__(1024) IdxSmem {
  uint8_t keys[kStages][kKeyTileBytes];
  uint8_t q[2][NQ * kHI * kDI];
  float scales[kScaleSlots][kTileKeys];
  float wq[kEpiWarps][(NQ >= 2 ? NQ / 2 : 1) * kHI];   // per epilogue warp: w' of its queries
  int32_t tile_row[kMaxCtaTiles][2];                    // physical row of each 64-key half, -1: none
  int32_t tile_off[kMaxGroups + 1];
  int32_t scan_tmp[kThreads / 32];
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t sc_full[kScaleSlots], sc_empty[kScaleSlots];
  uint32_t tmem_base;
};

struct TcArgs {
  int num_rows, n_groups;
  const int32_t* row_seq;
  const int32_t* row_klen;
  const float* q_scale;
  const float* w;
  const float* k_scale;
  CacheMap map;
  float* scores;
  int64_t ld;
  DeviceStatus* status;
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
  extern __shared__ __align__(1024) uint8_t smraw[];
  IdxSmem<NQ>& S = *reinterpret_cast<IdxSmem<NQ>*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.q_full[i], 1);
      mbar_init(&S.q_empty[i], 1);
      mbar_init(&S.acc_full[i], 1);
      mbar_init(&S.acc_empty[i], kEpiWarps);
    }
    for (int i = 0; i < kScaleSlots; ++i) {
      mbar_init(&S.sc_full[i], 32);          // one cp.async arrival per producer lane
      mbar_init(&S.sc_empty[i], kEpiWarps);
    }
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 2 * N);
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
    }
  }
  __syncthreads();
  const bool run = ntile > 0 && ntile <= kMaxCtaTiles;

  if (warp == 0) {
    // ------------------------------------------------------------ producer warp
    if (run) {
      if (lane == 0) { prefetch_tmap(&tm_k); prefetch_tmap(&tm_q); }
      TileIter it;
      it.start(S.tile_off, a.n_groups, t_begin);
      int qcount = 0, j = 0;
      bool alive = true;
      for (; j < ntile; ++j, it.next()) {
        const int st = j % kStages, sl = j % kScaleSlots;
        if (lane == 0) {
          if (j == 0 || it.kt == 0) {
            const int qb = qcount & 1;
            alive = mbar_wait(&S.q_empty[qb], ((qcount >> 1) & 1) ^ 1, a.status, 1);
            if (alive) {
              mbar_expect_tx(&S.q_full[qb], kQBytes);
              tma_load_2d(S.q[qb], &tm_q, &S.q_full[qb], 0, it.g * NQ * kHI);
            }
          }
          alive = alive && mbar_wait(&S.empty[st], ((j / kStages) & 1) ^ 1, a.status, 2);
          if (alive) {
            const int r0 = S.tile_row[j][0], r1 = S.tile_row[j][1];
            const uint32_t bytes = (r0 >= 0 ? kKeyTileBytes / 2 : 0) + (r1 >= 0 ? kKeyTileBytes / 2 : 0);
            if (bytes == 0) {
              mbar_arrive(&S.full[st]);
            } else {
              mbar_expect_tx(&S.full[st], bytes);
              if (r0 >= 0) tma_load_2d(S.keys[st], &tm_k, &S.full[st], 0, r0);
              if (r1 >= 0) tma_load_2d(S.keys[st] + kKeyTileBytes / 2, &tm_k, &S.full[st], 0, r1);
            }
          }
          alive = alive && mbar_wait(&S.sc_empty[sl], ((j / kScaleSlots) & 1) ^ 1, a.status, 9);
        }
        if (j == 0 || it.kt == 0) ++qcount;
        alive = __shfl_sync(0xffffffffu, alive, 0);
        if (!alive) break;
        // the tile's 128 key scales: 4 per lane, asynchronously
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = i * 32 + lane;
          const int r = S.tile_row[j][k >> 6];
          if (r >= 0 && (int64_t)r + (k & 63) < a.map.num_tokens)
            cp_async_4(&S.scales[sl][k], a.k_scale + (int64_t)r + (k & 63));
        }
        cp_async_mbar_arrive(&S.sc_full[sl]);
      }
      // tail: wait until the MMAs have released every stage and query buffer in
      // use, so no commit is still in flight to this CTA's shared memory at exit
      if (alive && lane == 0) {
        for (int st = 0; st < kStages && st < j; ++st) {
          const int last_use = (j - 1 - st) / kStages;
          if (!mbar_wait(&S.empty[st], last_use & 1, a.status, 7)) break;
        }
        for (int qb = 0; qb < 2 && qb < qcount; ++qb) {
          const int last_use = (qcount - 1 - qb) >> 1;
          if (!mbar_wait(&S.q_empty[qb], last_use & 1, a.status, 8)) break;
        }
      }
      cp_async_wait<0>();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && run) {
      TileIter it;
      it.start(S.tile_off, a.n_groups, t_begin);
      constexpr uint32_t idesc = idesc_f8_e4m3(N);
      int qcount = -1;
      for (int j = 0; j < ntile; ++j) {
        const bool first = (j == 0 || it.kt == 0);
        if (first) {
          ++qcount;
          if (!mbar_wait(&S.q_full[qcount & 1], (qcount >> 1) & 1, a.status, 3)) break;
        }
        const int st = j % kStages, ab = j & 1;
        if (!mbar_wait(&S.full[st], (j / kStages) & 1, a.status, 4)) break;
        if (!mbar_wait(&S.acc_empty[ab], ((j >> 1) & 1) ^ 1, a.status, 5)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(S.keys[st]);
        const uint32_t qa = smem_u32(S.q[qcount & 1]);
#pragma unroll
        for (int k = 0; k < kDI / 32; ++k)
          mma_f8(tmem + ab * N, sdesc_sw128(ka + 32 * k, 16, 1024), sdesc_sw128(qa + 32 * k, 16, 1024),
                 idesc, k > 0);
        mma_commit(&S.empty[st]);
        mma_commit(&S.acc_full[ab]);
        const bool last = (it.kt + 1 == it.ntiles) || (j + 1 == ntile);
        if (last) mma_commit(&S.q_empty[qcount & 1]);
        it.next();
      }
    }
  } else if (run) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;               // 0..7
    const int lq = warp & 3;              // TMEM lane quarter this warp may access
    const int half = e >> 2;
    const int row_in_tile = lq * 32 + lane;
    constexpr int QPW = NQ >= 2 ? NQ / 2 : 1;   // queries this warp reduces
    const bool active = NQ >= 2 || half == 0;
    TileIter it;
    it.start(S.tile_off, a.n_groups, t_begin);
    int klen[QPW];
    for (int j = 0; j < ntile; ++j, it.next()) {
      if (j == 0 || it.kt == 0) {
        for (int i = 0; i < QPW; ++i) {
          const int r = it.g * NQ + half * QPW + i;
          klen[i] = (active && r < a.num_rows) ? a.row_klen[r] : 0;
        }
        // w' = w * q_scale of this warp's queries into this warp's own slice
        // (written and read by the same warp: __syncwarp orders it)
        __syncwarp();
        for (int i = lane; i < QPW * kHI; i += 32) {
          const int r = it.g * NQ + half * QPW + i / kHI, h = i % kHI;
          float v = 0.f;
          if (active && r < a.num_rows)
            v = a.w[(int64_t)r * kHI + h] * a.q_scale[(int64_t)r * kHI + h];
          S.wq[e][i] = v;
        }
        __syncwarp();
      }
      const int ab = j & 1, sl = j % kScaleSlots;
      if (!mbar_wait(&S.acc_full[ab], (j >> 1) & 1, a.status, 6)) break;
      tc_fence_after();
      const int s = it.kt * kTileKeys + row_in_tile;
      float res[QPW];
      if (active) {
#pragma unroll
        for (int i = 0; i < QPW; ++i) {
          const int qi = half * QPW + i;
          const uint32_t col = tmem + ab * N + qi * kHI + ((uint32_t)(lq * 32) << 16);
          uint32_t v0[32], v1[32];
          tmem_ld32(col, v0);
          tmem_ld32(col + 32, v1);
          tmem_wait_ld();
          const float4* wv = reinterpret_cast<const float4*>(&S.wq[e][i * kHI]);
          float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
          for (int h = 0; h < 32; h += 4) {
            const float4 w0 = wv[h / 4];
            acc0 = fmaf(fmaxf(__uint_as_float(v0[h + 0]), 0.f), w0.x, acc0);
            acc1 = fmaf(fmaxf(__uint_as_float(v0[h + 1]), 0.f), w0.y, acc1);
            acc2 = fmaf(fmaxf(__uint_as_float(v0[h + 2]), 0.f), w0.z, acc2);
            acc3 = fmaf(fmaxf(__uint_as_float(v0[h + 3]), 0.f), w0.w, acc3);
            const float4 w1 = wv[8 + h / 4];
            acc0 = fmaf(fmaxf(__uint_as_float(v1[h + 0]), 0.f), w1.x, acc0);
            acc1 = fmaf(fmaxf(__uint_as_float(v1[h + 1]), 0.f), w1.y, acc1);
            acc2 = fmaf(fmaxf(__uint_as_float(v1[h + 2]), 0.f), w1.z, acc2);
            acc3 = fmaf(fmaxf(__uint_as_float(v1[h + 3]), 0.f), w1.w, acc3);
          }
          res[i] = (acc0 + acc1) + (acc2 + acc3);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[ab]);
      if (!mbar_wait(&S.sc_full[sl], (j / kScaleSlots) & 1, a.status, 10)) break;
      const float ks = S.scales[sl][row_in_tile];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.sc_empty[sl]);
      if (active) {
#pragma unroll
        for (int i = 0; i < QPW; ++i) {
          const int r = it.g * NQ + half * QPW + i;
          if (s < klen[i]) a.scores[(int64_t)r * a.ld + s] = res[i] * ks;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * N);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
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

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int NQ>
dsa_status launch_nq(const IndexerArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(IdxSmem<NQ>) + 1024;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(indexer_tc_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess) {
      set_error("indexer_tc: cannot set %zu bytes of shared memory", smem);
      return DSA_ERR_CUDA;
    }
    attr = true;
  }
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
    t.status = a.status;
    CUtensorMap tq;
    if (!make_tmap_rows128(&tq, static_cast<const uint8_t*>(a.q_idx) + (int64_t)r0 * kHI * kDI,
                           (uint64_t)t.num_rows * kHI, NQ * kHI)) {
      set_error("indexer_tc: cuTensorMapEncodeTiled failed");
      return DSA_ERR_CUDA;
    }
    // tiles are at most groups x ceil(max_klen / 128); a CTA takes at most kMaxCtaTiles
    const int64_t tiles = (int64_t)ng * ((a.max_klen + kTileKeys - 1) / kTileKeys);
    const int64_t need = (tiles + kMaxCtaTiles - 1) / kMaxCtaTiles;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, std::max<int64_t>(num_sms(), need)));
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

bool indexer_tc_supported(const IndexerArgs& a) {
  if (a.idx_dtype != DSA_FP8_E4M3 || a.d_idx != kDI || a.n_idx_heads != kHI) return false;
  if (a.q_scale == nullptr || a.idx_k_scale == nullptr) return false;
  if (a.map.block_table != nullptr && a.map.page_size % 64 != 0) return false;
  if (a.map.num_tokens >= (int64_t)INT32_MAX) return false;
  if (encode_fn() == nullptr) return false;
  return a.q_group == 1 || a.q_group == 2 || a.q_group == 4;
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
