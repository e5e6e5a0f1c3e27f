// warmup.cu - the indexer's warm-up objective and its backward (CUDA cores).
//
// "DeepSeek Sparse Attention DSA Architecture Guide", section "Training
// Mechanics: Dense Warm-Up and KL Alignment", Phase 1: the indexer is trained
// to match the dense attention, the teacher p_t being the dense attention
// probabilities of row t summed over heads and normalised, and the loss
// L^I = sum_t KL(p_t || softmax(I_t)).
//
//  indexer_kl_kernel      per row t: KL(p_t || softmax(I_t)) over s < klen[t]
//                         (0 log 0 = 0) and its gradient g = softmax(I_t) - p_t.
//  indexer_bwd_dq_kernel  per (row, chunk of keys): partial dq, dw of
//                         I[s] = sum_j w_j ReLU(q_j . k_s).
//  indexer_bwd_reduce     the chunk partials of each row, summed in chunk order.
//  indexer_bwd_dk_kernel  per (sequence, tile of 32 keys): dk of every key,
//                         summed over the rows that see it, in row order.
// Gradients are taken with respect to the dequantised operands (e4m3 codes
// times their scales); the FP8 cast itself is not differentiated.  ReLU's
// derivative is 1 where its argument is > 0, else 0.  The argument's sign is
// taken exactly: q_j . k_s = q_scale_j k_scale_s sum_i e4m3(q8_ji) e4m3(k8_si),
// and that sum of products of E4M3 values (each a multiple of 2^-9 below 449)
// is exact in fp64, so the mask does not depend on summation order.  The dot
// products run in fp32 first: a sum of 128 terms accumulated with fma is
// within gamma_127 sum_i |k_i q_i| <= gamma_127 |k| |q| of exact
// (gamma_n = n u / (1 - n u), u = 2^-24; Cauchy-Schwarz for the second step),
// so its sign is the exact sign whenever its magnitude exceeds that bound; the
// few that do not are recomputed in fp64.
// Every sum is in a fixed order: results are deterministic run to run.
#include <cuda_fp8.h>

#include "dsa_kernels.cuh"

namespace dsa {
namespace {

constexpr int kHI = 64, kDI = 128;        // the shapes these kernels run (H_I x d_I)
constexpr int kTile = 32;                 // keys per inner tile
constexpr int kQP = kDI + 4;              // padded row of a query in shared memory
constexpr int kThreads = 256;

// Sixteen e4m3 codes (one 16-byte piece) as floats.
__device__ __forceinline__ void e4m3x16_to_float(uint4 v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
      const float2 x = __half22float2(__half2(r));
      f[4 * i + 2 * h] = x.x;
      f[4 * i + 2 * h + 1] = x.y;
    }
  }
}
// Elements [16 p, 16 p + 16) of an indexer tensor row block (e4m3 codes or
// f32), unscaled, as floats; `base` is 16-byte aligned.
__device__ __forceinline__ void load16(const void* base, int64_t p, bool fp8, float* f) {
  if (fp8) {
    e4m3x16_to_float(reinterpret_cast<const uint4*>(base)[p], f);
  } else {
    const float4* b = reinterpret_cast<const float4*>(base) + 4 * p;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = b[i];
      f[4 * i] = x.x; f[4 * i + 1] = x.y; f[4 * i + 2] = x.z; f[4 * i + 3] = x.w;
    }
  }
}
// fp32 filter factor: gamma_127 for u = 2^-24, rounded up with some room.
constexpr double kDotBound = 7.6e-6;

__device__ __forceinline__ float block_reduce_sum(float v, float* tmp) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) tmp[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += tmp[i];   // fixed order
  return s;
}
__device__ __forceinline__ float block_reduce_max(float v, float* tmp) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) tmp[w] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, tmp[i]);
  return m;
}

// grid T, block 256: one row.  Three passes over the row's klen entries.
__global__ void __launch_bounds__(kThreads) indexer_kl_kernel(WarmupArgs a) {
  __shared__ float tmp[kThreads / 32];
  trace_kernel(a.status, DSA_KERNEL_WARMUP);
  const int t = blockIdx.x;
  const int n = a.row_klen[t];
  const float* I = a.scores + (int64_t)t * a.ld_scores;
  const float* p = a.teacher + (int64_t)t * a.ld_teacher;
  float* g = a.grad + (int64_t)t * a.ld_grad;
  float m = -INFINITY;
  for (int s = threadIdx.x; s < n; s += kThreads) m = fmaxf(m, I[s]);
  m = block_reduce_max(m, tmp);
  float z = 0.f;
  for (int s = threadIdx.x; s < n; s += kThreads) z += expf(I[s] - m);
  z = block_reduce_sum(z, tmp);
  const float log_z = m + logf(z);
  float kl = 0.f;
  for (int s = threadIdx.x; s < n; s += kThreads) {
    const float lq = I[s] - log_z;                   // log softmax(I)_s
    const float ps = p[s];
    g[s] = expf(lq) - ps;
    if (ps > 0.f) kl += ps * (logf(ps) - lq);
  }
  kl = block_reduce_sum(kl, tmp);
  if (threadIdx.x == 0) a.loss[t] = n > 0 ? kl : 0.f;
}

// One key tile: stored key values (unscaled), their scales and the fp32
// filter bound factor kDotBound |k_s| into shared memory; keys past klen or
// unmapped read as zero with scale 0.
__device__ __forceinline__ void load_key_tile(const WarmupArgs& a, int seq, int s0, int klen,
                                              float (*kv)[kDI], float* ks, float* kn, int64_t* prow) {
  const bool fp8 = a.idx_dtype == DSA_FP8_E4M3;
  if (threadIdx.x < kTile) {
    const int s = s0 + threadIdx.x;
    int64_t r = -1;
    if (s < klen) {
      bool ok = true;
      r = a.map.row(seq, s, a.status, &ok);
      if (!ok) r = -1;
    }
    prow[threadIdx.x] = r;
    ks[threadIdx.x] = r >= 0 ? (a.idx_k_scale ? a.idx_k_scale[r] : 1.f) : 0.f;
  }
  __syncthreads();
  // 32 keys x 8 pieces of 16 elements: one piece per thread
  {
    const int j = threadIdx.x >> 3, pc = threadIdx.x & 7;
    const int64_t r = prow[j];
    float f[16];
    if (r >= 0) {
      load16(static_cast<const uint8_t*>(a.idx_k) + r * kDI * (fp8 ? 1 : 4), pc, fp8, f);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) f[e] = 0.f;
    }
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 16; ++e) ss = fma((double)f[e], (double)f[e], ss);
#pragma unroll
    for (int e = 0; e < 16; e += 4) *reinterpret_cast<float4*>(&kv[j][16 * pc + e]) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
    // |k_s|^2 over the eight pieces of the key (lanes 8j'..8j'+7 of a warp)
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (pc == 0) kn[j] = (float)(kDotBound * sqrt(ss) * (1.0 + 1e-6));
  }
  __syncthreads();
}

// The query of row t: stored values (unscaled), scales, weights, and |q_j|.
__device__ __forceinline__ void load_query(const WarmupArgs& a, int t, float (*qv)[kQP], float* qs,
                                           float* w, float* qn) {
  const bool fp8 = a.idx_dtype == DSA_FP8_E4M3;
  const uint8_t* base = static_cast<const uint8_t*>(a.q_idx) + (int64_t)t * kHI * kDI * (fp8 ? 1 : 4);
  // 64 heads x 8 pieces of 16 elements: two pieces per thread
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int piece = threadIdx.x + kThreads * h2;
    const int j = piece >> 3, pc = piece & 7;
    float f[16];
    load16(base + (int64_t)j * kDI * (fp8 ? 1 : 4), pc, fp8, f);
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 16; ++e) ss = fma((double)f[e], (double)f[e], ss);
#pragma unroll
    for (int e = 0; e < 16; e += 4) *reinterpret_cast<float4*>(&qv[j][16 * pc + e]) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (pc == 0) qn[j] = (float)(sqrt(ss) * (1.0 + 1e-6));
  }
  if (threadIdx.x < kHI) {
    qs[threadIdx.x] = a.q_scale ? a.q_scale[(int64_t)t * kHI + threadIdx.x] : 1.f;
    w[threadIdx.x] = a.w[(int64_t)t * kHI + threadIdx.x];
  }
  __syncthreads();
}

// dots[s][j] = sum_i kv[s][i] qv[j][i] for the 32 x 64 (key, head) pairs of a
// tile, with its sign exact: fp32 fma sums, and the pairs within the bound
// kn[s] qn[j] of zero recomputed in fp64 (exact for e4m3 values).  A nonzero
// exact value keeps its sign in the stored float.  Thread (warp w, lane l)
// takes keys 4w .. 4w + 3 and heads l, l + 32: per four dims, each key's
// values are one 16-byte load that the warp shares, each head's one 16-byte
// load (query rows padded to kQP floats, so the 8 lanes of a quarter warp hit
// distinct banks): 6 loads per 32 FMAs.
__device__ __forceinline__ void tile_dots(float (*kv)[kDI], float (*qv)[kQP], const float* kn,
                                          const float* qn, float (*dots)[kHI]) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float acc[4][2];
#pragma unroll
  for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll 4
  for (int i = 0; i < kDI; i += 4) {
    const float4 q0 = *reinterpret_cast<const float4*>(&qv[lane][i]);
    const float4 q1 = *reinterpret_cast<const float4*>(&qv[lane + 32][i]);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 k = *reinterpret_cast<const float4*>(&kv[4 * w + r][i]);
      acc[r][0] = fmaf(k.w, q0.w, fmaf(k.z, q0.z, fmaf(k.y, q0.y, fmaf(k.x, q0.x, acc[r][0]))));
      acc[r][1] = fmaf(k.w, q1.w, fmaf(k.z, q1.z, fmaf(k.y, q1.y, fmaf(k.x, q1.x, acc[r][1]))));
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int s = 4 * w + r;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int j = lane + 32 * c;
      float d = acc[r][c];
      if (fabsf(d) <= kn[s] * qn[j]) {             // the sign is not certain: exact sum
        double e = 0.0;
        for (int i = 0; i < kDI; ++i) e = fma((double)kv[s][i], (double)qv[j][i], e);
        d = e > 0.0 ? fmaxf((float)e, 1e-45f) : (e < 0.0 ? fminf((float)e, -1e-45f) : 0.f);
      }
      dots[s][j] = d;
    }
  }
  __syncthreads();
}

struct DqSmem {
  float qv[kHI][kQP];
  float kv[kTile][kDI];
  float dots[kTile][kHI];
  float coef[kTile][kHI];                  // g_s w_j [dot > 0] k_scale_s
  float qs[kHI], w[kHI], ks[kTile], g[kTile], kn[kTile], qn[kHI];
  int64_t prow[kTile];
};

// grid (n_chunks, T), block 256.  Thread tid accumulates dq[j][d] for
// j = tid / 4 (heads 0..63) and d = 16 i + 4 (tid % 4) + e (i < 8, e < 4: four
// dims per 16-byte load; the four threads of a head read 64 contiguous bytes),
// and (tid < 64) dw[tid].
__global__ void __launch_bounds__(kThreads) indexer_bwd_dq_kernel(WarmupArgs a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  DqSmem& S = *reinterpret_cast<DqSmem*>(smraw);
  trace_kernel(a.status, DSA_KERNEL_WARMUP);
  const int t = blockIdx.y, c = blockIdx.x;
  const int klen = a.row_klen[t], seq = a.row_seq[t];
  const int s_lo = c * a.chunk_keys, s_hi = min(klen, s_lo + a.chunk_keys);
  const int jq = threadIdx.x >> 2, d0 = 4 * (threadIdx.x & 3);
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;
  float dw = 0.f;
  if (s_lo < s_hi) {
    load_query(a, t, S.qv, S.qs, S.w, S.qn);
    const float* g = a.grad + (int64_t)t * a.ld_grad;
    for (int s0 = s_lo; s0 < s_hi; s0 += kTile) {
      load_key_tile(a, seq, s0, s_hi, S.kv, S.ks, S.kn, S.prow);
      if (threadIdx.x < kTile) S.g[threadIdx.x] = s0 + threadIdx.x < s_hi ? g[s0 + threadIdx.x] : 0.f;
      tile_dots(S.kv, S.qv, S.kn, S.qn, S.dots);
      for (int e = threadIdx.x; e < kTile * kHI; e += kThreads) {
        const int s = e / kHI, j = e - s * kHI;
        S.coef[s][j] = S.dots[s][j] > 0.f ? S.g[s] * S.w[j] * S.ks[s] : 0.f;
      }
      __syncthreads();
      if (threadIdx.x < kHI) {                        // dw_j += sum_s g_s ReLU(q_j . k_s)
        const int j = threadIdx.x;
        for (int s = 0; s < kTile; ++s)
          dw = fmaf(S.g[s] * S.ks[s] * S.qs[j], fmaxf(S.dots[s][j], 0.f), dw);
      }
      for (int s = 0; s < kTile; ++s) {               // dq_j += sum_s coef_sj k_s
        const float cf = S.coef[s][jq];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 k4 = *reinterpret_cast<const float4*>(&S.kv[s][16 * i + d0]);
          acc[4 * i] = fmaf(cf, k4.x, acc[4 * i]);
          acc[4 * i + 1] = fmaf(cf, k4.y, acc[4 * i + 1]);
          acc[4 * i + 2] = fmaf(cf, k4.z, acc[4 * i + 2]);
          acc[4 * i + 3] = fmaf(cf, k4.w, acc[4 * i + 3]);
        }
      }
      __syncthreads();
    }
  }
  // partials [T][n_chunks][64][128 + 1]: dq then dw at column 128
  float* part = a.partial + (((int64_t)t * a.n_chunks + c) * kHI) * (kDI + 1);
#pragma unroll
  for (int i = 0; i < 32; ++i) part[(int64_t)jq * (kDI + 1) + 16 * (i >> 2) + d0 + (i & 3)] = acc[i];
  if (threadIdx.x < kHI) part[(int64_t)threadIdx.x * (kDI + 1) + kDI] = dw;
}

// grid T, block 256: dq[t] and dw[t] as the sum of the row's chunk partials.
__global__ void __launch_bounds__(kThreads) indexer_bwd_reduce_kernel(WarmupArgs a) {
  const int t = blockIdx.x;
  const float* part = a.partial + (int64_t)t * a.n_chunks * kHI * (kDI + 1);
  for (int e = threadIdx.x; e < kHI * (kDI + 1); e += kThreads) {
    float s = 0.f;
    for (int c = 0; c < a.n_chunks; ++c) s += part[(int64_t)c * kHI * (kDI + 1) + e];
    const int j = e / (kDI + 1), d = e - j * (kDI + 1);
    if (d < kDI) a.dq[((int64_t)t * kHI + j) * kDI + d] = s;
    else a.dw[(int64_t)t * kHI + j] = s;
  }
}

struct DkSmem {
  float qv[kHI][kQP];
  float kv[kTile][kDI];
  float dots[kTile][kHI];
  float coef[kTile][kHI];                  // g_s w_j [dot > 0] q_scale_j
  float qs[kHI], w[kHI], ks[kTile], g[kTile], kn[kTile], qn[kHI];
  int64_t prow[kTile];
  int seen[kTile];
};

// grid (ceil(max_klen / 32), num_seqs), block 256.  Thread tid accumulates
// dk[s][d] for s = tid / 8 and d = 32 i + 4 (tid % 8) + e (i < 4, e < 4), over
// the rows of sequence b that see key s, in row order; writes the keys some
// row sees.
__global__ void __launch_bounds__(kThreads) indexer_bwd_dk_kernel(WarmupArgs a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  DkSmem& S = *reinterpret_cast<DkSmem*>(smraw);
  trace_kernel(a.status, DSA_KERNEL_WARMUP);
  const int b = blockIdx.y, s0 = blockIdx.x * kTile;
  const int sk = threadIdx.x >> 3, d0 = 4 * (threadIdx.x & 7);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  if (threadIdx.x < kTile) S.seen[threadIdx.x] = 0;
  // the keys of the tile (up to the longest row of this sequence)
  int kmax = 0;
  for (int t = threadIdx.x; t < a.num_rows; t += kThreads)
    if (a.row_seq[t] == b) kmax = max(kmax, a.row_klen[t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  __shared__ int kmax_w[kThreads / 32];
  if ((threadIdx.x & 31) == 0) kmax_w[threadIdx.x >> 5] = kmax;
  __syncthreads();
  kmax = 0;
  for (int i = 0; i < kThreads / 32; ++i) kmax = max(kmax, kmax_w[i]);
  if (s0 >= kmax) return;                            // no row of b sees this tile
  load_key_tile(a, b, s0, kmax, S.kv, S.ks, S.kn, S.prow);
  for (int t = 0; t < a.num_rows; ++t) {
    if (a.row_seq[t] != b) continue;                  // uniform over the block
    const int klen = a.row_klen[t];
    if (klen <= s0) continue;
    load_query(a, t, S.qv, S.qs, S.w, S.qn);
    const float* g = a.grad + (int64_t)t * a.ld_grad;
    if (threadIdx.x < kTile) {
      const bool vis = s0 + threadIdx.x < klen;
      S.g[threadIdx.x] = vis ? g[s0 + threadIdx.x] : 0.f;
      S.seen[threadIdx.x] |= vis ? 1 : 0;
    }
    tile_dots(S.kv, S.qv, S.kn, S.qn, S.dots);
    for (int e = threadIdx.x; e < kTile * kHI; e += kThreads) {
      const int s = e / kHI, j = e - s * kHI;
      S.coef[s][j] = S.dots[s][j] > 0.f ? S.g[s] * S.w[j] * S.qs[j] : 0.f;
    }
    __syncthreads();
    for (int j = 0; j < kHI; ++j) {                   // dk_s += sum_j coef_sj q_j
      const float cf = S.coef[sk][j];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 q4 = *reinterpret_cast<const float4*>(&S.qv[j][32 * i + d0]);
        acc[4 * i] = fmaf(cf, q4.x, acc[4 * i]);
        acc[4 * i + 1] = fmaf(cf, q4.y, acc[4 * i + 1]);
        acc[4 * i + 2] = fmaf(cf, q4.z, acc[4 * i + 2]);
        acc[4 * i + 3] = fmaf(cf, q4.w, acc[4 * i + 3]);
      }
    }
    __syncthreads();
  }
  if (S.seen[sk] && S.prow[sk] >= 0) {
    float* dst = a.dk + S.prow[sk] * kDI + d0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(dst + 32 * i) = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
  }
}

}  // namespace

bool warmup_supported(const WarmupArgs& a) {
  return a.n_idx_heads == kHI && a.d_idx == kDI &&
         (a.idx_dtype == DSA_FP8_E4M3 || a.idx_dtype == DSA_F32);
}

size_t warmup_ws_bytes(int num_rows, int max_klen, int chunk_keys) {
  const int64_t n_chunks = (max_klen + chunk_keys - 1) / chunk_keys;
  return (size_t)num_rows * (size_t)std::max<int64_t>(n_chunks, 1) * kHI * (kDI + 1) * sizeof(float);
}

dsa_status launch_indexer_kl(const WarmupArgs& a, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  indexer_kl_kernel<<<a.num_rows, kThreads, 0, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("indexer_kl launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status launch_indexer_backward(const WarmupArgs& a, int max_klen, int num_seqs, cudaStream_t stream) {
  if (a.num_rows == 0 || max_klen == 0) return DSA_OK;
  static std::atomic<bool> attr_dq[kMaxDevices] = {}, attr_dk[kMaxDevices] = {};
  if (dsa_status st = set_smem_limit_once(reinterpret_cast<const void*>(indexer_bwd_dq_kernel),
                                          sizeof(DqSmem), attr_dq))
    return st;
  if (dsa_status st = set_smem_limit_once(reinterpret_cast<const void*>(indexer_bwd_dk_kernel),
                                          sizeof(DkSmem), attr_dk))
    return st;
  indexer_bwd_dq_kernel<<<dim3((unsigned)a.n_chunks, (unsigned)a.num_rows), kThreads, sizeof(DqSmem),
                          stream>>>(a);
  indexer_bwd_reduce_kernel<<<a.num_rows, kThreads, 0, stream>>>(a);
  indexer_bwd_dk_kernel<<<dim3((unsigned)((max_klen + kTile - 1) / kTile), (unsigned)num_seqs), kThreads,
                          sizeof(DkSmem), stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("indexer backward launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
