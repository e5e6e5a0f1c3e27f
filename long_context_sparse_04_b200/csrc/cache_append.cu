// cache_append.cu - fused FP8 quantise + paged cache write of new tokens.
//
// Each decoding step writes its new tokens into the layer's caches before the
// indexer reads them ("Sparse Attention Architectures for Long-Context
// Inference: Evolution and Engineering Practices", section 6, item
// "Incremental inference adaptation").  The indexer key cache is FP8
// ("DeepSeek Sparse Attention DSA Architecture Guide", section "Stage 1: The
// Lightning Indexer", item "Native FP8 Precision") with one fp32 scale per
// token, and both caches are paged ("Sparse Attention in Large Language
// Models: Architecture Evolution and Engineering Practice", section 4, item
// "Memory Management and KV Cache Optimization").
//
// One warp per token, eight tokens per CTA.  The work is a stream: per token
// 4*d_I bytes of key and (d_c+d_r)*elt bytes of latent in, d_I codes, a scale
// and the latent row out, so the kernel is HBM-bound and its design is about
// bytes in flight: every lane issues its key float4s and its first latent
// 16-byte chunks before the destination lookup (two dependent loads through
// the block table), so the table walk overlaps the payload.  No shared
// memory, no tensor cores: nothing here is a contraction.
//
//   amax  = max |k|            (lane max, then a butterfly over the warp)
//   s     = fl32(amax / 448)   (div.rn.f32; 1 when the quotient is 0)
//   code  = E4M3(fl32(k / s))  (div.rn.f32, then cvt.rn.satfinite.e4m3x2)
//
// The divisions are IEEE round-to-nearest and take no flush-to-zero, so the
// codes are exactly those of the rule as written; the hardware conversion
// rounds to nearest even and saturates finite overflow at +-448.
#include <cfloat>

#include "dsa_kernels.cuh"

namespace dsa {
namespace {

constexpr int kWarpsPerCta = 8;     // tokens per CTA
constexpr int kMaxKeyChunks = 4;    // float4 per lane: d_I <= 4 * 32 * 4 = 512
constexpr int kLatGroup = 3;        // 16-byte latent chunks per lane in flight (1152 B rows: one group)

__device__ __forceinline__ float div_rn(float a, float b) {
  float r;
  asm("div.rn.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Four floats -> four e4m3 bytes, x0 in the lowest byte (the lowest address).
// cvt packs its first source into the upper byte of the pair.
__device__ __forceinline__ uint32_t e4m3x4(float x0, float x1, float x2, float x3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

__device__ __forceinline__ float4 ld_stream_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_stream_u4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ bool finite4(const float4& v) {
  return fabsf(v.x) <= FLT_MAX && fabsf(v.y) <= FLT_MAX && fabsf(v.z) <= FLT_MAX &&
         fabsf(v.w) <= FLT_MAX;
}

__device__ __forceinline__ float amax4(const float4& v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
cache_append_kernel(const AppendArgs a) {
  pdl_launch_dependents();
  trace_kernel(a.status, DSA_KERNEL_CACHE_APPEND);
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (n >= a.n_new) return;

  // 1. the payload: key chunks and the first latent group, all in flight
  const int kc = a.d_idx >> 2;
  const float4* ksrc = reinterpret_cast<const float4*>(a.k_new) + (int64_t)n * kc;
  float4 v[kMaxKeyChunks];
#pragma unroll
  for (int i = 0; i < kMaxKeyChunks; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < kc ? ld_stream_f4(ksrc + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int lc = a.latent_row_bytes >> 4;
  const uint4* lsrc = reinterpret_cast<const uint4*>(a.latent_new) + (int64_t)n * lc;
  uint4 t[kLatGroup];
#pragma unroll
  for (int i = 0; i < kLatGroup; ++i) {
    const int c = lane + 32 * i;
    if (c < lc) t[i] = ld_stream_u4(lsrc + c);
  }

  // 2. the destination row (the same map the attention stage reads)
  const int seq = __ldg(a.tok_seq + n);
  const int pos = __ldg(a.tok_pos + n);
  bool ok = seq >= 0 && seq < a.num_seqs && pos >= 0;
  int64_t row = 0;
  if (ok) row = a.map.row(seq, pos, nullptr, &ok);
  if (!ok) {
    if (lane == 0) set_status(a.status, DSA_ERR_OUT_OF_RANGE, n);
    return;
  }

  // 3. the key: reject non-finite, then quantise (or copy) and store
  bool fin = true;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxKeyChunks; ++i) {
    fin = fin && finite4(v[i]);
    amax = fmaxf(amax, amax4(v[i]));
  }
  if (!__all_sync(0xffffffffu, fin)) {
    if (lane == 0) set_status(a.status, DSA_ERR_INVALID_ARG, n);
    return;
  }
  if (a.idx_dtype == DSA_FP8_E4M3) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float s = div_rn(amax, 448.f);
    if (!(s > 0.f)) s = 1.f;
    uint32_t* kdst = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.idx_k) + row * a.d_idx);
#pragma unroll
    for (int i = 0; i < kMaxKeyChunks; ++i) {
      const int c = lane + 32 * i;
      if (c < kc)
        kdst[c] = e4m3x4(div_rn(v[i].x, s), div_rn(v[i].y, s), div_rn(v[i].z, s), div_rn(v[i].w, s));
    }
    if (lane == 0) a.idx_k_scale[row] = s;
  } else {
    float4* kdst = reinterpret_cast<float4*>(static_cast<float*>(a.idx_k) + row * a.d_idx);
#pragma unroll
    for (int i = 0; i < kMaxKeyChunks; ++i) {
      const int c = lane + 32 * i;
      if (c < kc) kdst[c] = v[i];
    }
  }

  // 4. the latent row: store the group in flight, load the next (rows wider
  //    than 32 * kLatGroup chunks only)
  uint4* ldst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.latent) + row * a.latent_row_bytes);
  for (int base = 0;;) {
#pragma unroll
    for (int i = 0; i < kLatGroup; ++i) {
      const int c = base + lane + 32 * i;
      if (c < lc) ldst[c] = t[i];
    }
    base += 32 * kLatGroup;
    if (base >= lc) break;
#pragma unroll
    for (int i = 0; i < kLatGroup; ++i) {
      const int c = base + lane + 32 * i;
      if (c < lc) t[i] = ld_stream_u4(lsrc + c);
    }
  }
}

}  // namespace

dsa_status launch_cache_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.n_new == 0) return DSA_OK;
  const unsigned grid = (unsigned)((a.n_new + kWarpsPerCta - 1) / kWarpsPerCta);
  cache_append_kernel<<<grid, kWarpsPerCta * 32, 0, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("cache append launch failed: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

int cache_append_max_d_idx() { return kMaxKeyChunks * 32 * 4; }

}  // namespace dsa
