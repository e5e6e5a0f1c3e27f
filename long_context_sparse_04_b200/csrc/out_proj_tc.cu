// out_proj_tc.cu - the output projection after the sparse attention, on the
// 5th-generation tensor cores.
//
// "DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 2:
// Fine-Grained Token Selection and Output Computation", output equation:
// u_{t,i} = sum_s softmax_s(.) W_{UV,i} c_s = W_{UV,i} o_{t,i}, where o is the
// latent output of the absorbed attention (W_UV,i does not depend on s).  The
// page's module ("End-to-End Implementation") then applies its output
// projection to the heads concatenated in order:
//     u[t,i,:] = W_UV[i] o[t,i,:]                      (per head, K = d_c)
//     y[t,:]   = W_out [u[t,0,:]; ...; u[t,H-1,:]]      (K = H * d_v)
//
// Both are one kernel, Y[t, n] = sum_k X[t, k] W[n, k] over a batch (the heads
// for W_UV, one batch for W_out): a tile is 128 rows t (the MMA's M) x BN
// weight rows n (the MMA's N, <= 256) over K in blocks of 64 bf16 (one
// 128-byte swizzle row).  Token rows are the M side so that a thread of the
// epilogue owns one output row and stores it in 16-byte pieces; a decode batch
// (32 rows) leaves 3/4 of M idle, which costs nothing there because the
// weights' HBM stream, not the tensor pipe, bounds it.  Small batches split K
// so that every SM streams weights; a second kernel adds the fp32 partials in
// a fixed order (no atomics: results do not depend on the schedule).
//
// Persistent CTAs, 192 threads:
//   warp 0      producer (one thread): TMA of the X tile (3D map: K, head,
//               row; rows past T read as zeros) and the W tile (2D map) into
//               a 4-stage ring, 48 KB per stage.
//   warp 1      TMEM allocator + single-thread issuer of tcgen05.mma
//               (kind::f16, bf16 x bf16 -> fp32, four K=16 MMAs per stage)
//               into two 256-column accumulators (tile i+1 accumulates while
//               the epilogue drains tile i).
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (lane = row t), bf16
//               round (cvt.rn.bf16x2) and 16-byte stores, or fp32 partials.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "dsa_kernels.cuh"

namespace dsa {
namespace {

constexpr int kBM = 128;                 // rows per tile (MMA M)
constexpr int kBK = 64;                  // K elements per stage (128 bytes of bf16)
constexpr int kMaxBN = 256;              // weight rows per tile (MMA N)
constexpr int kStages = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kXTileBytes = kBM * 128;   // 16 KB
constexpr int kWTileBytes = kMaxBN * 128;   // 32 KB; a BN-row tile fills the first BN*128 B
constexpr int kMaxSplits = 16;

struct __align__(1024) ProjSmem {
  uint8_t x[kStages][kXTileBytes];
  uint8_t w[kStages][kWTileBytes];
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
};

struct GemmArgs {
  int T;                  // rows of X and Y
  int batches;            // heads (W_UV) or 1 (W_out)
  int bn;                 // weight rows per tile, a multiple of 32, <= 256
  int n_tiles;            // weight-row tiles per batch
  int n_total;            // weight rows per batch = output columns per batch
  int kb_total;           // K blocks of 64
  int splits;             // K splits; 1 writes bf16 Y directly
  int t_tiles;
  uint16_t* y;            // bf16 bits
  int64_t y_row, y_batch; // element strides of Y
  float* partial;         // [splits, T, n_total] fp32 when splits > 1 (batches == 1)
  DeviceStatus* status;
  uint32_t trace_bit;
};

struct Item {
  int b, tt, nt, s, kb_lo, kb_hi;
};

__device__ __forceinline__ Item decode_item(const GemmArgs& a, int it) {
  Item r;
  r.s = it % a.splits;
  it /= a.splits;
  r.nt = it % a.n_tiles;
  it /= a.n_tiles;
  r.tt = it % a.t_tiles;
  r.b = it / a.t_tiles;
  r.kb_lo = (int)((int64_t)r.s * a.kb_total / a.splits);
  r.kb_hi = (int)((int64_t)(r.s + 1) * a.kb_total / a.splits);
  return r;
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Two floats -> bf16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t bf16x2(uint32_t lo, uint32_t hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(__uint_as_float(hi)), "f"(__uint_as_float(lo)));
  return d;
}

__global__ void __launch_bounds__(kThreads, 1)
out_proj_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  ProjSmem& S = *reinterpret_cast<ProjSmem*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  pdl_wait();
  trace_kernel(a.status, a.trace_bit);
  if (threadIdx.x == 32) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&S.acc_full[i], 1); mbar_init(&S.acc_empty[i], kEpiWarps); }
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 2 * kMaxBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const int items = a.batches * a.t_tiles * a.n_tiles * a.splits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
      const uint32_t bytes = kXTileBytes + (uint32_t)a.bn * 128u;
      int st = 0, used = 0;
      uint32_t ph = 1;                       // parity to wait for on empty
      bool alive = true;
      for (int it = blockIdx.x; it < items && alive; it += gridDim.x) {
        const Item m = decode_item(a, it);
        for (int kb = m.kb_lo; kb < m.kb_hi; ++kb) {
          if (!(alive = mbar_wait(&S.empty[st], ph, a.status, 11))) break;
          mbar_expect_tx(&S.full[st], bytes);
          tma_load_3d(S.x[st], &tm_x, &S.full[st], kb * kBK, m.b, m.tt * kBM);
          tma_load_2d(S.w[st], &tm_w, &S.full[st], kb * kBK, m.b * a.n_total + m.nt * a.bn);
          ++used;
          if (++st == kStages) { st = 0; ph ^= 1; }
        }
      }
      // tail: wait until the MMAs have released every stage in use, so no
      // commit is still in flight to this CTA's shared memory at exit
      if (alive) {
        for (int s2 = 0; s2 < kStages && s2 < used; ++s2) {
          const int last_use = (used - 1 - s2) / kStages;
          if (!mbar_wait(&S.empty[s2], last_use & 1, a.status, 12)) break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(a.bn, false);
      const uint64_t xd0 = sdesc_sw128(smem_u32(S.x[0]), 16, 1024);
      const uint64_t wd0 = sdesc_sw128(smem_u32(S.w[0]), 16, 1024);
      constexpr uint64_t kXStep = kXTileBytes >> 4, kWStep = kWTileBytes >> 4;
      int st = 0, ab = 0;
      uint32_t ph = 0, aph = 1;              // parity to wait for on full / acc_empty
      bool alive = true;
      for (int it = blockIdx.x; it < items && alive; it += gridDim.x) {
        const Item m = decode_item(a, it);
        if (!(alive = mbar_wait(&S.acc_empty[ab], aph, a.status, 13))) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * kMaxBN;
        for (int kb = m.kb_lo; kb < m.kb_hi; ++kb) {
          if (!(alive = mbar_wait(&S.full[st], ph, a.status, 14))) break;
          tc_fence_after();
          const uint64_t xd = xd0 + (uint64_t)st * kXStep, wd = wd0 + (uint64_t)st * kWStep;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_bf16(d, xd + 2 * k, wd + 2 * k, idesc, (kb > m.kb_lo || k > 0) ? 1u : 0u);
          mma_commit(&S.empty[st]);
          if (++st == kStages) { st = 0; ph ^= 1; }
        }
        if (!alive) break;
        mma_commit(&S.acc_full[ab]);
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (4 warps)
    const int q = warp & 3;                  // the TMEM lane quarter this warp may access
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int ab = 0;
    uint32_t aph = 0;
    bool dead = false;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      const Item m = decode_item(a, it);
      dead = dead || !mbar_wait(&S.acc_full[ab], aph, a.status, 15);
      tc_fence_after();
      const int t = m.tt * kBM + q * 32 + lane;
      for (int c = 0; c < a.bn; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + ab * kMaxBN + c, v);
        tmem_wait_ld_regs(v);
        const int n = m.nt * a.bn + c;       // column within the batch
        if (dead || t >= a.T || n >= a.n_total) continue;
        if (a.splits == 1) {
          uint4* dst = reinterpret_cast<uint4*>(a.y + (int64_t)t * a.y_row + (int64_t)m.b * a.y_batch + n);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(bf16x2(v[8 * j + 0], v[8 * j + 1]), bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                bf16x2(v[8 * j + 4], v[8 * j + 5]), bf16x2(v[8 * j + 6], v[8 * j + 7]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(a.partial + ((int64_t)m.s * a.T + t) * a.n_total + n);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[ab]);
      if (++ab == 2) { ab = 0; aph ^= 1; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kMaxBN);
  }
}

// y[i] = bf16(sum_s partial[s][i]), s in order; i over T * n_total in fours.
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ partial, int splits, int64_t n4, int64_t plane,
                     uint16_t* __restrict__ y, DeviceStatus* status) {
  pdl_launch_dependents();
  pdl_wait();
  trace_kernel(status, DSA_KERNEL_OUT_PROJ_REDUCE);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(partial)[i];
    for (int s = 1; s < splits; ++s) {
      const float4 p = reinterpret_cast<const float4*>(partial + s * plane)[i];
      acc.x += p.x;
      acc.y += p.y;
      acc.z += p.z;
      acc.w += p.w;
    }
    reinterpret_cast<uint2*>(y)[i] =
        make_uint2(bf16x2(__float_as_uint(acc.x), __float_as_uint(acc.y)),
                   bf16x2(__float_as_uint(acc.z), __float_as_uint(acc.w)));
  }
}

bool make_tmap_x(CUtensorMap* m, const void* base, int k, int batches, int rows,
                 int64_t batch_stride_bytes, int64_t row_stride_bytes) {
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)k, (cuuint64_t)batches, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)batch_stride_bytes, (cuuint64_t)row_stride_bytes};
  cuuint32_t box[3] = {kBK, 1, kBM};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_w(CUtensorMap* m, const void* base, int k, int rows, int box_rows) {
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)k * 2};
  cuuint32_t box[2] = {kBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

dsa_status launch_gemm(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& g,
                       cudaStream_t stream) {
  const size_t smem = sizeof(ProjSmem) + 1024;
  static std::atomic<bool> attr[kMaxDevices] = {};
  if (dsa_status st = set_smem_limit_once(reinterpret_cast<const void*>(out_proj_kernel), smem, attr))
    return st;
  const int64_t items = (int64_t)g.batches * g.t_tiles * g.n_tiles * g.splits;
  const int grid = (int)std::min<int64_t>(items, device_sm_count());
  out_proj_kernel<<<grid, kThreads, smem, stream>>>(tx, tw, g);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("out_proj launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace

// K splits of the W_out product: enough (row tile x column tile x split) items
// to give every SM one, each split at least 8 K blocks.
int out_proj_splits(int num_rows, int d_model, int k_blocks) {
  const int64_t tiles = (int64_t)((num_rows + kBM - 1) / kBM) * ((d_model + kMaxBN - 1) / kMaxBN);
  const int sms = device_sm_count();
  if (tiles == 0 || tiles >= sms) return 1;
  int s = (int)(sms / tiles);
  s = std::min(s, std::max(1, k_blocks / 8));
  return std::max(1, std::min(s, kMaxSplits));
}

dsa_status launch_out_proj(const ProjArgs& a, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  const int T = a.num_rows, H = a.n_heads;
  const int t_tiles = (T + kBM - 1) / kBM;
  // u[t,i,:] = W_UV[i] o[t,i,:]: batches = heads, one tile of d_v weight rows
  CUtensorMap tx, tw;
  if (!make_tmap_x(&tx, a.o, a.d_c, H, T, (int64_t)a.d_c * 2, (int64_t)H * a.d_c * 2) ||
      !make_tmap_w(&tw, a.w_uv, a.d_c, H * a.d_v, a.d_v)) {
    set_error("out_proj: cuTensorMapEncodeTiled failed");
    return DSA_ERR_CUDA;
  }
  GemmArgs g{};
  g.T = T;
  g.batches = H;
  g.bn = a.d_v;
  g.n_tiles = 1;
  g.n_total = a.d_v;
  g.kb_total = a.d_c / kBK;
  g.splits = 1;
  g.t_tiles = t_tiles;
  g.y = static_cast<uint16_t*>(a.u);
  g.y_row = (int64_t)H * a.d_v;
  g.y_batch = a.d_v;
  g.status = a.status;
  g.trace_bit = DSA_KERNEL_OUT_PROJ;
  if (dsa_status st = launch_gemm(tx, tw, g, stream)) return st;

  // y[t,:] = W_out u[t,:,:] (heads concatenated): one batch, 256-row tiles
  const int K2 = H * a.d_v;
  const int bn2 = std::min(kMaxBN, a.d_model);
  if (!make_tmap_x(&tx, a.u, K2, 1, T, (int64_t)K2 * 2, (int64_t)K2 * 2) ||
      !make_tmap_w(&tw, a.w_out, K2, a.d_model, bn2)) {
    set_error("out_proj: cuTensorMapEncodeTiled failed");
    return DSA_ERR_CUDA;
  }
  g.batches = 1;
  g.bn = bn2;
  g.n_tiles = (a.d_model + bn2 - 1) / bn2;
  g.n_total = a.d_model;
  g.kb_total = K2 / kBK;
  g.splits = out_proj_splits(T, a.d_model, g.kb_total);
  g.y = static_cast<uint16_t*>(a.y);
  g.y_row = a.d_model;
  g.y_batch = 0;
  g.partial = a.partial;
  if (dsa_status st = launch_gemm(tx, tw, g, stream)) return st;
  if (g.splits > 1) {
    const int64_t n4 = (int64_t)T * a.d_model / 4;
    const int grid = (int)std::min<int64_t>((n4 + 255) / 256, 4 * (int64_t)device_sm_count());
    splitk_reduce_kernel<<<grid, 256, 0, stream>>>(a.partial, g.splits, n4, (int64_t)T * a.d_model,
                                                   static_cast<uint16_t*>(a.y), a.status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      set_error("out_proj reduce launch: %s", cudaGetErrorString(e));
      return DSA_ERR_CUDA;
    }
  }
  return DSA_OK;
}

}  // namespace dsa
