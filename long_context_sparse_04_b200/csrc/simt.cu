// simt.cu - SIMT (CUDA-core) kernels of the DSA forward path.
//
// These run the fp32 workload (fp32 cannot use the tensor cores at a 1e-4
// tolerance) and serve as a second, independent GPU implementation of every
// stage for any dtype when DSA_ALGO_SIMT is requested.
//
//  indexer_simt: I[t,s] = k_scale[s] * sum_j (w*q_scale)[t,j] * ReLU(q[t,j] . k[s])
//                ("DeepSeek Sparse Attention DSA Architecture Guide", section
//                "Stage 1: The Lightning Indexer", index-score equation with H_I
//                weighted heads).
//  mla_simt:     absorbed sparse MLA with an online softmax over the selected
//                rows (same page, "Stage 2", output equation).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dsa_kernels.cuh"

namespace dsa {

__device__ __forceinline__ float load_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ float load_elem(const uint8_t* p, int64_t i) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(p[i]), __NV_E4M3);
  return __half2float(__half(h));
}
__device__ __forceinline__ void store_elem(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// grid (ceil(max_klen/128), T), block 128; smem: q [H_I*d_I] + w' [H_I] floats.
template <typename KT>
__global__ void __launch_bounds__(128) indexer_simt_kernel(IndexerArgs a) {
  extern __shared__ float sm[];
  pdl_wait();
  trace_kernel(a.status, DSA_KERNEL_INDEXER_SIMT);
  const int t = blockIdx.y;
  const int H = a.n_idx_heads, D = a.d_idx;
  float* q = sm;
  float* wq = sm + H * D;
  const KT* qi = static_cast<const KT*>(a.q_idx) + (int64_t)t * H * D;
  for (int i = threadIdx.x; i < H * D; i += blockDim.x) q[i] = load_elem(qi, i);
  for (int j = threadIdx.x; j < H; j += blockDim.x)
    wq[j] = a.w[(int64_t)t * H + j] * (a.q_scale ? a.q_scale[(int64_t)t * H + j] : 1.0f);
  __syncthreads();
  const int klen = a.row_klen[t];
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= klen) return;
  const int seq = a.row_seq[t];
  bool ok = true;
  const int64_t r = a.map.row(seq, s, a.status, &ok);
  if (!ok) return;
  const KT* kp = static_cast<const KT*>(a.idx_k) + r * D;
  float acc = 0.f;
  for (int j = 0; j < H; ++j) {
    float dot = 0.f;
    for (int d = 0; d < D; ++d) dot = fmaf(q[j * D + d], load_elem(kp, d), dot);
    acc = fmaf(wq[j], fmaxf(dot, 0.f), acc);
  }
  if (a.idx_k_scale) acc *= a.idx_k_scale[r];
  a.scores[(int64_t)t * a.ld_scores + s] = acc;
}

// grid (T, H/8), block 128.  Each block: one row, 8 heads.
// smem: q [8][D] + kv [16][D] + z [8][16] floats.
template <typename T>
__global__ void __launch_bounds__(128) mla_simt_kernel(MlaArgs a) {
  constexpr int HB = 8, KC = 16;
  extern __shared__ float sm[];
  pdl_wait();
  trace_kernel(a.status, DSA_KERNEL_MLA_SIMT);
  const int t = blockIdx.x;
  const int h0 = blockIdx.y * HB;
  const int D = a.d_c + a.d_r, DC = a.d_c, H = a.n_heads;
  float* q = sm;
  float* kv = q + HB * D;
  float* z = kv + KC * D;
  __shared__ float alpha_s[HB];
  const T* qp = static_cast<const T*>(a.q) + ((int64_t)t * H + h0) * D;
  for (int i = threadIdx.x; i < HB * D; i += blockDim.x) q[i] = load_elem(qp, i) * a.sm_scale;
  const int seq = a.row_seq[t];
  const int32_t* idx = a.idx + (int64_t)t * a.topk;
  // output ownership: head oh = tid / 16, dims d = tid % 16 + 16*i
  const int oh = threadIdx.x / 16, od = threadIdx.x % 16;
  const int nd = DC / 16;
  float o[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) o[i] = 0.f;
  float m = -INFINITY, l = 0.f;   // tracked by threads 0..7 (one per head), shared via smem
  __shared__ float m_s[HB], l_s[HB];
  if (threadIdx.x < HB) { m_s[threadIdx.x] = -INFINITY; l_s[threadIdx.x] = 0.f; }
  __syncthreads();
  __shared__ int64_t prow[KC];
  for (int c0 = 0; c0 < a.topk; c0 += KC) {
    if (threadIdx.x < KC) {
      const int s = (c0 + threadIdx.x < a.topk) ? idx[c0 + threadIdx.x] : -1;
      int64_t pr = -1;
      if (s >= 0) {
        bool ok = true;
        pr = a.map.row(seq, s, a.status, &ok);
        if (!ok) pr = -1;
      }
      prow[threadIdx.x] = pr;
    }
    __syncthreads();
    const T* lat = static_cast<const T*>(a.latent);
    for (int i = threadIdx.x; i < KC * D; i += blockDim.x) {
      int j = i / D, d = i - j * D;
      kv[i] = prow[j] >= 0 ? load_elem(lat, prow[j] * D + d) : 0.f;
    }
    __syncthreads();
    // logits: thread -> (head, key) pair, 8 x 16 = 128
    {
      int hh = threadIdx.x / KC, j = threadIdx.x % KC;
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc = fmaf(q[hh * D + d], kv[j * D + d], acc);
      z[hh * KC + j] = prow[j] >= 0 ? acc : -INFINITY;
    }
    __syncthreads();
    if (threadIdx.x < HB) {
      int hh = threadIdx.x;
      float mx = m_s[hh];
      for (int j = 0; j < KC; ++j) mx = fmaxf(mx, z[hh * KC + j]);
      float al = (mx == -INFINITY) ? 1.f : expf(m_s[hh] - mx);
      float sum = l_s[hh] * al;
      for (int j = 0; j < KC; ++j) {
        float p = (z[hh * KC + j] == -INFINITY) ? 0.f : expf(z[hh * KC + j] - mx);
        z[hh * KC + j] = p;
        sum += p;
      }
      m_s[hh] = mx;
      l_s[hh] = sum;
      alpha_s[hh] = al;
    }
    __syncthreads();
    {
      float al = alpha_s[oh];
      for (int i = 0; i < nd && i < 32; ++i) {
        int d = od + 16 * i;
        float acc = o[i] * al;
        for (int j = 0; j < KC; ++j) acc = fmaf(z[oh * KC + j], kv[j * D + d], acc);
        o[i] = acc;
      }
    }
    __syncthreads();
  }
  m = m_s[oh];
  l = l_s[oh];
  T* out = static_cast<T*>(a.out) + ((int64_t)t * H + h0 + oh) * DC;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  for (int i = 0; i < nd && i < 32; ++i) store_elem(out, od + 16 * i, o[i] * inv);
  if (a.lse && od == 0)
    a.lse[(int64_t)t * H + h0 + oh] = l > 0.f ? m + logf(l) : -INFINITY;
}

dsa_status launch_indexer_simt(const IndexerArgs& a, cudaStream_t stream) {
  if (a.num_rows == 0 || a.max_klen == 0) return DSA_OK;
  dim3 grid((a.max_klen + 127) / 128, a.num_rows);
  size_t smem = (size_t)(a.n_idx_heads * a.d_idx + a.n_idx_heads) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaSuccess;
    if (a.idx_dtype == DSA_FP8_E4M3)
      e = cudaFuncSetAttribute(indexer_simt_kernel<uint8_t>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else
      e = cudaFuncSetAttribute(indexer_simt_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  if (a.idx_dtype == DSA_FP8_E4M3)
    indexer_simt_kernel<uint8_t><<<grid, 128, smem, stream>>>(a);
  else
    indexer_simt_kernel<float><<<grid, 128, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status launch_mla_simt(const MlaArgs& a, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  if (a.n_heads % 8 != 0 || a.d_c % 16 != 0 || a.d_c > 512) return DSA_ERR_UNSUPPORTED;
  const int D = a.d_c + a.d_r;
  size_t smem = (size_t)(8 * D + 16 * D + 8 * 16) * sizeof(float);
  dim3 grid(a.num_rows, a.n_heads / 8);
  cudaError_t e;
  if (a.mla_dtype == DSA_BF16) {
    e = cudaFuncSetAttribute(mla_simt_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    mla_simt_kernel<__nv_bfloat16><<<grid, 128, smem, stream>>>(a);
  } else {
    e = cudaFuncSetAttribute(mla_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    mla_simt_kernel<float><<<grid, 128, smem, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
