// mla_tc.cu - sparse absorbed MLA on the 5th-generation tensor cores.
//
// For query row t, head i and the selected keys s in S_t ("DeepSeek Sparse
// Attention DSA Architecture Guide", section "Stage 2: Fine-Grained Token
// Selection and Output Computation", output equation, in absorbed form):
//     z[i,s] = sm_scale * q[t,i,:] . (c_s || kR_s)        (576 dims)
//     out[t,i,:] = sum_s softmax_s(z[i,:]) c_s              (512 dims)
//
// Work unit: (row t, key split).  A cluster of two CTAs takes one unit and
// splits the 576 dims between them: CTA r holds latent dims [256r, 256r+256)
// and RoPE dims [32r, 32r+32) of Q (128 heads) and of every gathered key.
//   * S_r = Q_r . KV_r^T (M=128 heads, N=64 keys, K=288) on the tensor cores.
//   * Each CTA sends its partial logit tile to the peer through distributed
//     shared memory, as a per-row max plus 16-bit fixed-point distances to it
//     (16.5 KB per 64 keys, one bulk copy).  Each CTA then forms
//     z = S_own (exact fp32) + S_peer (decoded) and runs its own online
//     softmax; the two sums differ only by the transport rounding, and each
//     CTA's (max, sum) state normalises its own half of the value dims.
//   * O_r += P . V_r with V_r = latent dims [256r, 256r+256) of the same
//     gathered rows (M=128, N=256, K=64), P read from tensor memory.
// No FLOP is done twice, every gathered byte is read once, and the 128 heads
// share each gathered row.  The softmax runs in the log2 domain with a lazy
// rescale: the running max is only moved (and O rescaled) when a block's max
// exceeds it by more than 8, so P stays <= 256.
//
// Roles per CTA (896 threads, seven warpgroups):
//   warp 0       TMEM allocation and single-thread MMA issue
//   warps 1-15   gather: 16-byte cp.async pieces of the selected rows into a
//                swizzled 3-stage ring.  A random 576-byte half row is a few
//                sectors from each of many DRAM pages, so the gather is bound
//                by the loads each warp keeps in flight: fifteen issuing warps
//                keep ~3x more bytes in flight than four.
//   warps 16-19  exchange: partial logits of block j to the peer while the
//                softmax works on block j-1 (thread = head = TMEM lane)
//   warps 20-27  softmax and epilogue: two warps per TMEM lane quarter, each
//                taking 32 of the block's 64 keys of its 32 heads, so the
//                per-block chain is half as long; the two halves agree on the
//                row max through shared memory
// The gather and MMA warpgroups give registers to the exchange and softmax
// warpgroups (setmaxnreg): 4 x 128 x 48 + 3 x 128 x 104 = 64,512 registers,
// the 896 threads x 72 the kernel is launched with (checked before launch).
// TMEM: S double buffer (2 x 64 cols), P double buffer (2 x 32 cols of bf16x2),
// O (256 cols).
#include <cuda_bf16.h>

#include "dsa_kernels.cuh"

namespace dsa {
namespace {

constexpr int kH = 128, kDC = 512, kDR = 64, kD = kDC + kDR;
constexpr int kBlk = 64;
constexpr int kNS = 3;
constexpr int kMaxKeys = 2048;
constexpr int kMaxSplits = 8;                 // key splits of a decode row, a power of 2
constexpr int kGatherWarp0 = 1, kGatherWarps = 15;
constexpr int kGatherThreads = 32 * kGatherWarps;       // 480
constexpr int kExWarp0 = 16;                            // warps 16-19
constexpr int kSmWarp0 = 20;                            // warps 20-27
constexpr int kThreads = 32 * 28;                       // 896: seven warpgroups
constexpr int kRegsLaunch = 72, kRegsLow = 48, kRegsHigh = 104;
static_assert(4 * 128 * kRegsLow + 3 * 128 * kRegsHigh <= kThreads * kRegsLaunch,
              "register split exceeds the launch's registers");
static_assert(kThreads * kRegsLaunch <= 65536, "launch registers exceed the SM's");
static_assert(kThreads % 32 == 0 && (kMaxSplits & (kMaxSplits - 1)) == 0, "layout");
constexpr int kPieces = 36;                 // 16-byte pieces of one key's 288 dims per CTA
constexpr uint32_t kColS = 0, kColP = 128, kColO = 256, kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;
// One exchanged tile of partial logits of 128 heads x 64 keys in the transport
// format below (row max + 16-bit fixed-point distance to it).
struct __align__(16) XTile {
  uint4 d[kH * 8];                          // 8 x 16-byte pieces per head, swizzled
  float m[kH];
};
constexpr uint32_t kXBytes = sizeof(XTile);

struct __align__(1024) MlaSmem {
  uint8_t q[4][kH * 128];                   // Q latent dims of this CTA: 4 SW128 chunks of 64 dims
  uint8_t kv[kNS][4][kBlk * 128];           // gathered latent dims: 4 SW128 chunks x 64 keys
  uint8_t kv_rope[kNS][kBlk * 64];          // gathered RoPE dims (32), SW64
  uint8_t q_rope[kH * 64];                  // Q RoPE dims (32), SW64
  XTile xbuf;                               // the peer's partial logits of the current block
  XTile sbuf;                               // this CTA's partial logits, bulk-copied to the peer
  int32_t rows[kMaxKeys];                   // physical cache row per selected key, -1 = none
  uint32_t valid[2 * kMaxKeys / kBlk];      // per 32 keys: bit i set = key i has a cache row
  float red_m[2][2][kH];                    // softmax halves: block max, [block parity][half][head]
  float red_l[2][kH];                       // softmax halves: final sums
  uint64_t q_full, x_full, x_free;
  uint64_t m_ready, m_full;                 // split merge in a 4-CTA cluster
  uint64_t kv_full[kNS], kv_empty[kNS];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint32_t tmem_base;
  int last_flag;                            // this CTA merges the row's splits
};

__device__ __forceinline__ uint8_t* smem_base(MlaSmem& S) { return reinterpret_cast<uint8_t*>(&S); }
// The split merge inside a 4-CTA cluster: each CTA of a pair keeps 128 of its
// 256 value dims and receives the other split's partial O of them (64 KB fp32,
// into Q's space) and its (max, sum) per head; it sends the other 128 from
// the first two gather stages.  The finished bf16 rows are staged in the third.
constexpr size_t kRecvO = 0, kSendO = 64 * 1024, kStage4 = 128 * 1024;
constexpr size_t kSendMl = 160 * 1024, kRecvMl = 161 * 1024;
constexpr uint32_t kMergeO = 64 * 1024, kMergeMl = kH * 8, kMergeTx = kMergeO + kMergeMl;
static_assert(offsetof(MlaSmem, kv) == kSendO && offsetof(MlaSmem, kv) + 2 * sizeof(MlaSmem::kv[0]) == kStage4 &&
                  offsetof(MlaSmem, kv_rope) == kSendMl && kRecvMl + kMergeMl <= kSendMl + sizeof(MlaSmem::kv_rope),
              "cluster merge layout");

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^x with the hardware approximation (ex2.approx.ftz.f32; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Transport format of a partial logit row (log2 domain) between the two CTAs:
// the row max m (fp32) and, per key, u = round(1024 * (m - z)) as a 16-bit
// integer saturated at 65535 (a key 64 below the row max carries a weight under
// 2^-64).  Error <= 2^-11 in the exponent (0.034% in the weight).  Encoding and
// decoding use a float magic-number add, so no conversion instruction is needed.
constexpr float kFix = 1024.f, kFixInv = 1.f / 1024.f, kMagic = 12582912.f;   // 1.5 * 2^23
// Encodes row h of a partial logit tile (z, scaled here by c) into `x`: the
// row max and eight swizzled 16-byte pieces of packed distances.
__device__ __forceinline__ void encode_partial(float (&z)[64], float c, XTile& x, int h) {
  float pm[8];
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    z[i] *= c;
    pm[i & 7] = (i < 8) ? z[i] : fmaxf(pm[i & 7], z[i]);
  }
  const float m = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                        fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = 4 * q + e;
      const uint32_t u0 = __float_as_uint(fminf((m - z[2 * i]) * kFix, 65535.f) + kMagic);
      const uint32_t u1 = __float_as_uint(fminf((m - z[2 * i + 1]) * kFix, 65535.f) + kMagic);
      w[e] = __byte_perm(u0, u1, 0x5410);         // low 16 bits of each
    }
    x.d[h * 8 + (q ^ (h & 7))] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  x.m[h] = m;
}
// z of the two keys packed in w, given the row max m.
__device__ __forceinline__ float2 decode_partial(uint32_t w, float m) {
  const float u0 = __uint_as_float(0x4B000000u | (w & 0xFFFFu)) - 8388608.f;
  const float u1 = __uint_as_float(0x4B000000u | (w >> 16)) - 8388608.f;
  return make_float2(fmaf(-u0, kFixInv, m), fmaf(-u1, kFixInv, m));
}

// 32 value dims of the O accumulator from tensor memory (zeros when the split
// saw no key, whose accumulator was never written).
__device__ __forceinline__ void load_o(uint32_t taddr, bool empty, float (&o)[32]) {
  if (empty) {
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = 0.f;
    return;
  }
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
  tmem_wait_ld();
}
// f[0..8) * inv as eight bf16 (round to nearest even) in one 16-byte piece.
__device__ __forceinline__ uint4 pack8(const float* f, float inv) {
  return make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                    pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
}
// Row h of the CTA's finished output tile in shared memory: 256 bf16 dims as
// 32 pieces of 16 bytes, piece c stored at c ^ (h % 32) so that a warp's 32
// rows hit distinct banks; o * inv are dims [8 c0, 8 c0 + 32).
__device__ __forceinline__ void stage_bf16(uint8_t* stg, int h, int c0, const float (&o)[32], float inv) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(stg + h * 512 + (((c0 + q) ^ (h & 31)) << 4)) = pack8(&o[8 * q], inv);
}
// Arrival ticket of one of a row's key splits: the slot holds (launch id << 32 |
// arrivals); a slot tagged with another launch (an earlier one, or never
// written) counts as empty, and the last arrival resets the count, so the
// slots need no clearing between launches.
// Returns the arrivals of this launch, this one included (0 if the CAS loop,
// which only ever competes with the row's other splits, were to run away).
__device__ __forceinline__ uint32_t take_ticket(unsigned long long* slot, uint32_t id, DeviceStatus* st) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(slot);
  for (int it = 0; it < 1 << 16; ++it) {
    const unsigned long long nv =
        (uint32_t)(cur >> 32) == id ? cur + 1ull : ((unsigned long long)id << 32) | 1ull;
    const unsigned long long got = atomicCAS(slot, cur, nv);
    if (got == cur) return (uint32_t)nv;
    cur = got;
  }
  set_status(st, DSA_ERR_TIMEOUT, 29);
  return 0u;
}

__device__ __forceinline__ void tstamp(long long* tr, uint32_t rank, int ev, int j) {
  if (tr != nullptr && blockIdx.x < 2 && j < kTraceBlocks)
    tr[((int)rank * kTraceEvents + ev) * kTraceBlocks + j] = clock64();
}

__device__ __forceinline__ void setmaxnreg_inc_high() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
}
__device__ __forceinline__ void setmaxnreg_dec_low() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
}

// ------------------------------------------------------------ MMA issuer (warp 0, lane 0)
__device__ __forceinline__ void mma_role(MlaSmem& S, const MlaArgs& a, uint32_t tmem, int nblk,
                                         uint32_t rank) {
  const int lane = threadIdx.x & 31;
  if (lane == 0 && nblk > 0) {
    constexpr uint32_t idesc_s = idesc_bf16(kBlk, false);
    constexpr uint32_t idesc_pv = idesc_bf16(256, true);
    bool ok = mbar_wait(&S.q_full, 0, a.status, 31);
    fence_proxy_async_smem();
    const uint32_t qa = smem_u32(S.q[0]), qra = smem_u32(S.q_rope);
    for (int j = 0; ok && j <= nblk; ++j) {
      if (j < nblk) {
        const int st = j % kNS, b = j & 1;
        if (!(ok = mbar_wait(&S.kv_full[st], (j / kNS) & 1, a.status, 32))) break;
        fence_proxy_async_smem();           // gathered (generic-proxy) writes -> tensor cores
        if (!(ok = mbar_wait(&S.s_free[b], ((j >> 1) & 1) ^ 1, a.status, 33))) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(S.kv[st][0]), kra = smem_u32(S.kv_rope[st]);
        const uint32_t d = tmem + kColS + b * 64;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(d, sdesc_sw128(qa + ch * kH * 128 + 32 * kk, 16, 1024),
                     sdesc_sw128(ka + ch * kBlk * 128 + 32 * kk, 16, 1024), idesc_s,
                     (ch | kk) != 0);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_bf16(d, sdesc_sw64(qra + 32 * kk, 512), sdesc_sw64(kra + 32 * kk, 512), idesc_s, 1);
        mma_commit(&S.s_full[b]);
        tstamp(a.trace, rank, 2, j);
      }
      if (j >= 1) {
        const int jj = j - 1, st = jj % kNS, b = jj & 1;
        if (!(ok = mbar_wait(&S.p_full[b], (jj >> 1) & 1, a.status, 34))) break;
        tc_fence_after();
        const uint32_t va = smem_u32(S.kv[st][0]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + kColO, tmem + kColP + b * 32 + kk * 8,
                      sdesc_sw128(va + kk * 16 * 128, kBlk * 128, 1024), idesc_pv,
                      (jj > 0 || kk > 0));
        mma_commit(&S.kv_empty[st]);
        mma_commit(&S.pv_done[b]);
        tstamp(a.trace, rank, 3, jj);
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) mla_tc_kernel(MlaArgs a, int keys_per_split) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  MlaSmem& S = *reinterpret_cast<MlaSmem*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                           ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  // CTA rank r of the pair holds dims half r; with the split merge in the
  // cluster, ranks 2 and 3 are the second split's pair
  const uint32_t crank = cluster_ctarank(), rank = crank & 1u, peer = crank ^ 1u;
  const int unit = blockIdx.x >> 1;
  const int t = unit / a.splits, sp = unit % a.splits;
  pdl_launch_dependents();

  // Setup that reads no input memory overlaps the predecessor's tail: barrier
  // init and the TMEM allocation.  Every read of an input (row lengths, Q, the
  // selection, the caches) comes after pdl_wait(), so a predecessor that
  // writes any of them (and triggers its dependents early) is complete and
  // visible first.
  if (threadIdx.x == 0) {
    mbar_init(&S.q_full, kGatherThreads);
    mbar_init(&S.x_full, 1);                 // armed by this CTA, completed by the peer's copy
    mbar_init(&S.x_free, 1);                 // the peer's receive buffer is free
    mbar_init(&S.m_ready, 1);                // the other split's CTA can take its half
    mbar_init(&S.m_full, 1);                 // this CTA's half of the other split landed
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&S.kv_full[i], kGatherThreads);
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_free[i], 128 + 256);   // exchange + softmax warpgroups
      mbar_init(&S.p_full[i], 256);         // softmax warpgroups
      mbar_init(&S.pv_done[i], 1);
    }
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  trace_kernel(a.status, DSA_KERNEL_MLA_TC);
  const int klen = a.row_klen[t];
  const int nsel = min(klen, a.topk);
  const int k0 = sp * keys_per_split;
  const int nvalid = max(0, min(nsel - k0, keys_per_split));
  const int nblk = (nvalid + kBlk - 1) / kBlk;
  const int seq = a.row_seq[t];
  if (threadIdx.x == 0 && nblk > 0) mbar_expect_tx(&S.x_full, kXBytes);   // arm the first transfer
  if (threadIdx.x == 0 && a.merge_in_cluster) mbar_expect_tx(&S.m_full, kMergeTx);
  const bool gather_warp = warp >= kGatherWarp0 && warp < kGatherWarp0 + kGatherWarps;
  const int g = threadIdx.x - 32 * kGatherWarp0;          // gather thread index (0..479)
  // physical rows of the selected keys of this split (entries past nvalid are
  // none): the index loads go out first (they gate the first gather), then the
  // Q pieces, then the block-table loads
  {
    constexpr int kPer = (kMaxKeys + kThreads - 1) / kThreads;
    const int32_t* idx = a.idx + (int64_t)t * a.topk + k0;
    const int nk = nblk * kBlk;
    int sv[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = threadIdx.x + u * kThreads;
      sv[u] = i < nvalid ? __ldg(idx + i) : -1;
    }
    // then Q: its pieces land while the selection is resolved below (the
    // gather warps arrive on q_full for them once the barrier init is visible)
    if (gather_warp && nblk > 0) {
      const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(a.q) + (int64_t)t * kH * kD;
      for (int qi = g; qi < kH * kPieces; qi += kGatherThreads) {
        const int h = qi / kPieces, c = qi - h * kPieces;
        if (c < 32) {
          cp_async_16(S.q[c >> 3] + sw128_off(h, c & 7), qrow + h * kD + 256 * rank + 8 * c);
        } else {
          cp_async_16(S.q_rope + sw64_off(h, c - 32), qrow + h * kD + kDC + 32 * rank + 8 * (c - 32));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = threadIdx.x + u * kThreads;
      int row = -1;
      if (i < nk) {
        const int sk = sv[u];
        if (sk >= 0 && sk < klen) {
          bool ok = true;
          const int64_t r = a.map.row(seq, sk, a.status, &ok);
          row = ok ? (int32_t)r : -1;
        }
        S.rows[i] = row;
      }
      // a warp holds 32 consecutive keys (kThreads is a multiple of 32): their
      // validity bits in one ballot
      const uint32_t bits = __ballot_sync(0xffffffffu, row >= 0);
      if ((threadIdx.x & 31) == 0 && (i >> 5) < 2 * nblk) S.valid[i >> 5] = bits;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every CTA of the cluster has initialised its barriers: the exchange and
  // softmax warpgroups, which touch other CTAs' shared memory, wait for that;
  // the gather and MMA warpgroups, which touch only their own, start at once.
  cluster_arrive();
  const uint32_t tmem = S.tmem_base;
  // Registers: the gather / MMA warpgroups (0-3) give theirs to the exchange
  // and softmax warpgroups (4-6).  Each warpgroup executes one setmaxnreg, at
  // the head of its role's branch.
  if (warp < kExWarp0) {
    setmaxnreg_dec_low();
    if (warp == 0) {
      mma_role(S, a, tmem, nblk, rank);
    } else if (nblk > 0) {
    // ------------------------------------------------------------ gather (480 threads)
      cp_async_mbar_arrive(&S.q_full);        // arrives when this thread's Q pieces land
      const __nv_bfloat16* lat = static_cast<const __nv_bfloat16*>(a.latent);
      for (int j = 0; j < nblk; ++j) {
        const int st = j % kNS;
        if (!mbar_wait(&S.kv_empty[st], ((j / kNS) & 1) ^ 1, a.status, 21)) break;
        for (int qi = g; qi < kBlk * kPieces; qi += kGatherThreads) {
          const int key = qi / kPieces, c = qi - key * kPieces;
          const int row = S.rows[j * kBlk + key];
          const __nv_bfloat16* src = lat + (int64_t)(row < 0 ? 0 : row) * kD +
                                     (c < 32 ? 256 * rank + 8 * c : kDC + 32 * rank + 8 * (c - 32));
          uint8_t* dst = c < 32 ? S.kv[st][c >> 3] + sw128_off(key, c & 7)
                                : S.kv_rope[st] + sw64_off(key, c - 32);
          cp_async_16_zfill(dst, src, row >= 0);
        }
        // arrives when this thread's pieces of block j land; the MMA thread makes
        // them visible to the tensor cores (proxy fence) after its wait
        cp_async_mbar_arrive(&S.kv_full[st]);
      }
      cp_async_wait_all();
    }
    cluster_wait();
  } else if (warp < kSmWarp0) {
    setmaxnreg_inc_high();
    cluster_wait();
    // ------------------------------------------------------------ exchange (128 threads)
    // Copies this CTA's partial logits of block j to the peer with one bulk copy
    // while the softmax warpgroups are still working on block j-1.  A wait that
    // times out only marks the warpgroup dead: the named barriers stay uniform.
    const int h = threadIdx.x - 32 * kExWarp0;                // head = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float c = a.sm_scale * kLog2e;
    bool dead = false;
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      float z[64];
      if (h == 0 && j > 0) bulk_wait_read0();               // the previous copy has left sbuf
      named_bar_sync(2, 128);
      dead = dead || !mbar_wait(&S.s_full[b], (j >> 1) & 1, a.status, 22);
      if (!dead) {
        tc_fence_after();
        tmem_ld32(tmem + lane_off + kColS + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&z[0]));
        tmem_ld32(tmem + lane_off + kColS + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&z[32]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&S.s_free[b]);
        encode_partial(z, c, S.sbuf, h);
      }
      fence_proxy_async_smem();                              // sbuf writes -> async copy engine
      named_bar_sync(2, 128);
      if (h == 0 && !dead) {
        if (mbar_wait_cluster(&S.x_free, (j & 1) ^ 1, a.status, 23)) {
          bulk_copy_to_peer(&S.xbuf, &S.sbuf, kXBytes, &S.x_full, peer);
          bulk_commit();
        }
      }
    }
    if (h == 0) bulk_wait_read0();
  } else {
    setmaxnreg_inc_high();
    cluster_wait();
    // ------------------------------------------------------------ softmax / output (256 threads)
    // Thread (half, h): head h (= TMEM lane), keys [32 half, 32 half + 32) of
    // every block, value dims [128 half, 128 half + 128) of this CTA's 256 in
    // the epilogue.  Both halves take the same rescale decisions: they use the
    // same block max (exchanged through red_m) and the same running max.
    const int sidx = threadIdx.x - 32 * kSmWarp0;             // 0..255
    const int half = sidx >> 7, h = sidx & 127;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float c = a.sm_scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    // A wait that times out marks the thread dead; the loop is left together
    // at the named barrier, and warp-collective tcgen05 ops stay uniform.
    bool dead = false;
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      dead = dead || !mbar_wait(&S.s_full[b], (j >> 1) & 1, a.status, 28);
      tc_fence_after();
      if (sidx == 0) tstamp(a.trace, rank, 4, j);
      float s[32];
      tmem_ld32(tmem + lane_off + kColS + b * 64 + 32 * half, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&S.s_free[b]);
      // z = c * S_own (exact) + the peer's partial (decoded).  The two CTAs see
      // the same sum up to that rounding; each keeps its own softmax state
      // (m, l), used for its own half of the value dims.
      dead = dead || !mbar_wait_cluster(&S.x_full, j & 1, a.status, 24);
      if (sidx == 0) tstamp(a.trace, rank, 5, j);
      {
        const float m_peer = S.xbuf.m[h];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w4 = S.xbuf.d[h * 8 + ((4 * half + q) ^ (h & 7))];
          const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = decode_partial(w[e], m_peer);
            s[8 * q + 2 * e] = fmaf(s[8 * q + 2 * e], c, f.x);
            s[8 * q + 2 * e + 1] = fmaf(s[8 * q + 2 * e + 1], c, f.y);
          }
        }
      }
      if (sidx == 0) tstamp(a.trace, rank, 0, j);
      // masked (only partial blocks) logits in the log2 domain; this half's max
      const uint32_t mask = S.valid[2 * j + half];
      if (mask != 0xFFFFFFFFu) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (!((mask >> i) & 1u)) s[i] = -INFINITY;
      }
      float pm[8];
#pragma unroll
      for (int i = 0; i < 32; ++i) pm[i & 7] = (i < 8) ? s[i] : fmaxf(pm[i & 7], s[i]);
      const float mh = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                             fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      S.red_m[b][half][h] = mh;
      // every softmax thread has read xbuf and published its half's max; all alive
      if (named_bar_or(3, 256, dead)) { dead = true; break; }
      if (sidx == 0) {
        if (j + 1 < nblk) mbar_expect_tx(&S.x_full, kXBytes);   // arm the next transfer first
        // then free the buffer: every thread's reads of it were consumed before
        // the barrier above, so the arrive needs no release ordering
        mbar_arrive_cluster_relaxed(&S.x_free, peer);
      }
      if (sidx == 0) tstamp(a.trace, rank, 1, j);
      const float mb = fmaxf(mh, S.red_m[b][half ^ 1][h]);
      // lazy rescale (warp-uniform because tcgen05.ld/st are warp-collective;
      // both halves of a lane quarter decide alike)
      const bool need = mb > m_used + kRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mb : m_used;
        const float alpha = need ? (m_used == -INFINITY ? 0.f : exp2f(m_used - m_new)) : 1.f;
        if (j > 0) {
          dead = dead || !mbar_wait(&S.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.status, 25);
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            const uint32_t col = tmem + lane_off + kColO + 128 * half + 32 * cc;
            tmem_ld32(col, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(col, o);
          }
          tmem_wait_st();
        }
        l *= alpha;
        m_used = m_new;
      }
      // p = 2^(s - m); a masked key (s = -inf) gives 0.  While no key of the row
      // has been visible, every s is -inf and m is taken as 0.
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t p2[16];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float p0 = ex2_approx(s[2 * i] - mu);
        const float p1 = ex2_approx(s[2 * i + 1] - mu);
        ls[i & 3] += p0 + p1;
        p2[i] = pack_bf16x2(p0, p1);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (sidx == 0) tstamp(a.trace, rank, 7, j);
      // P buffer b is free once the PV of block j-2 is done
      dead = dead || !mbar_wait(&S.pv_done[b], ((j >> 1) & 1) ^ 1, a.status, 26);
      tc_fence_after();
      tmem_st16(tmem + lane_off + kColP + b * 32 + 16 * half, p2);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&S.p_full[b]);
      if (sidx == 0) tstamp(a.trace, rank, 6, j);
    }
    // ---- output: this CTA's value dims [128 half, 128 half + 128) of head h
    const int64_t ro = ((int64_t)t * kH + h);
    if (!dead && nblk > 0) {
      dead = !mbar_wait(&S.pv_done[(nblk - 1) & 1], ((nblk - 1) >> 1) & 1, a.status, 27);
      tc_fence_after();
    }
    // the row's sum over both key halves; a timed-out wait anywhere fails the CTA
    S.red_l[half][h] = l;
    const bool fail = named_bar_or(4, 256, dead);
    const float lt = S.red_l[0][h] + S.red_l[1][h];
    const bool empty = nblk == 0;        // no visible key in this split: O = 0, l = 0
    const int col0 = 128 * half;         // this thread's value dims within the CTA's 256
    if (a.merge_in_cluster) {
      // Two key splits in one 4-CTA cluster: the CTA of split s keeps value dims
      // [128 s, 128 s + 128) of its rank's 256, receives the other split's
      // partial O of them and (max, sum) through shared memory, and sends that
      // split's CTA of the same rank (cluster rank crank ^ 2) the other 128.
      // Every CTA takes part in the exchange, also after a timed-out wait, so
      // that its partner's waits end.
      const uint32_t partner = crank ^ 2u;
      uint8_t* base = smem_base(S);
      const int keep0 = 128 * sp, send0 = 128 * (sp ^ 1);
      // this CTA's receive area (Q's space) is free: its last products are done
      if (sidx == 0) mbar_arrive_cluster(&S.m_ready, partner);
      float4* send = reinterpret_cast<float4*>(base + kSendO);
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        float o[32];
        load_o(tmem + lane_off + kColO + send0 + 64 * half + 32 * cc, empty || fail, o);
        const int d0 = (64 * half + 32 * cc) / 4;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          send[(d0 + i) * kH + h] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
      if (half == 0) reinterpret_cast<float2*>(base + kSendMl)[h] = make_float2(m_used, lt);
      fence_proxy_async_smem();            // generic writes -> bulk copy engine
      named_bar_sync(4, 256);
      if (sidx == 0 && mbar_wait_cluster(&S.m_ready, 0, a.status, 30)) {
        bulk_copy_to_peer(base + kRecvO, base + kSendO, kMergeO, &S.m_full, partner);
        bulk_copy_to_peer(base + kRecvMl, base + kSendMl, kMergeMl, &S.m_full, partner);
        bulk_commit();
        bulk_wait_read0();
      }
      const bool got = mbar_wait_cluster(&S.m_full, 0, a.status, 31);
      const bool bad = named_bar_or(4, 256, fail || !got);
      if (!bad) {
        // out = (w0 O_0 + w1 O_1) / (w0 l_0 + w1 l_1), w_s = 2^(m_s - M), split 0 first
        const float2 mine = make_float2(m_used, lt);
        const float2 theirs = reinterpret_cast<const float2*>(base + kRecvMl)[h];
        const float2 s0 = sp == 0 ? mine : theirs, s1 = sp == 0 ? theirs : mine;
        const float M = fmaxf(s0.x, s1.x);
        const float w0 = s0.x == -INFINITY ? 0.f : exp2f(s0.x - M);
        const float w1 = s1.x == -INFINITY ? 0.f : exp2f(s1.x - M);
        const float L = fmaf(w1, s1.y, w0 * s0.y);
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const float4* recv = reinterpret_cast<const float4*>(base + kRecvO);
        uint8_t* stg4 = base + kStage4;     // 128 rows x 256 bytes, pieces swizzled by row
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          float own[32], acc[32];
          load_o(tmem + lane_off + kColO + keep0 + 64 * half + 32 * cc, empty, own);
          const int d0 = (64 * half + 32 * cc) / 4;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = recv[(d0 + i) * kH + h];
            const float r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = sp == 0 ? own[4 * i + e] : r[e];
              const float x1 = sp == 0 ? r[e] : own[4 * i + e];
              acc[4 * i + e] = fmaf(w1, x1, w0 * x0);
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = (64 * half + 32 * cc) / 8 + q;
            *reinterpret_cast<uint4*>(stg4 + h * 256 + ((c ^ (h & 15)) << 4)) = pack8(&acc[8 * q], inv);
          }
        }
        if (half == 0 && rank == 0 && sp == 0 && a.lse)
          a.lse[ro] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        named_bar_sync(4, 256);
        // 128 rows x 16 pieces of 16 bytes; a half warp writes one row's 256 bytes
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + (int64_t)t * kH * kDC + 256 * rank + keep0;
#pragma unroll 4
        for (int k = 0; k < 8; ++k) {
          const int i = sidx + 256 * k, row = i >> 4, ch = i & 15;
          const uint4 v = *reinterpret_cast<const uint4*>(stg4 + row * 256 + ((ch ^ (row & 15)) << 4));
          reinterpret_cast<uint4*>(out + (int64_t)row * kDC)[ch] = v;
        }
      } else {
        // a bounded wait ran out (recorded in the status word): zeros
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + ro * kDC + 256 * rank +
                                              keep0 + 64 * half);
#pragma unroll 1
        for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    } else if (!fail) {
      // The finished rows go through shared memory (the gather ring, idle once the
      // last PV is done) so that global writes are whole 512-byte row segments.
      uint8_t* stg = &S.kv[0][0][0];
      bool write_out = true;
      if (a.splits == 1) {
        const float inv = (lt > 0.f) ? 1.f / lt : 0.f;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          load_o(tmem + lane_off + kColO + col0 + 32 * cc, empty, o);
          stage_bf16(stg, h, (col0 + 32 * cc) / 8, o, inv);
        }
        if (half == 0 && rank == 0 && a.lse)
          a.lse[ro] = lt > 0.f ? (m_used + log2f(lt)) * kLn2 : -INFINITY;
      } else {
        // Split-K: publish this split's unnormalised O and (max, sum); the last of
        // the row's splits to arrive (per CTA rank) merges them in split order:
        //   out = sum_s w_s O_s / sum_s w_s l_s,  w_s = 2^(m_s - M),  M = max_s m_s.
        float4* po = reinterpret_cast<float4*>(a.part_o);
        float2* pml = reinterpret_cast<float2*>(a.part_ml);
        const int64_t per_unit = (256 / 4) * kH;           // float4s of one (row, split, rank)
        const int64_t mine = (((int64_t)t * a.splits + sp) * 2 + rank) * per_unit;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          load_o(tmem + lane_off + kColO + col0 + 32 * cc, empty, o);
          const int d0 = (col0 + 32 * cc) / 4;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            po[mine + (int64_t)(d0 + i) * kH + h] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
        if (half == 0) pml[(((int64_t)t * a.splits + sp) * 2 + rank) * kH + h] = make_float2(m_used, lt);
        // release this CTA's partial (the barrier orders every thread's stores
        // before thread 0's fence), then take the ticket
        named_bar_sync(4, 256);
        if (sidx == 0) {
          __threadfence();
          unsigned long long* slot = &a.part_cnt[(int64_t)t * 2 + rank];
          const bool last = take_ticket(slot, a.launch_id, a.status) == (uint32_t)a.splits;
          // every split has arrived: reset the count, so that a replay of the same
          // launch (a captured graph keeps its launch id) counts from zero again
          if (last) *slot = (unsigned long long)a.launch_id << 32;
          S.last_flag = last;
          __threadfence();
        }
        named_bar_sync(4, 256);
        write_out = S.last_flag != 0;
        if (write_out) {
          if (sidx == 0 && a.status != nullptr) atomicOr(&a.status->ran, DSA_KERNEL_MLA_COMBINE);
          float ws[kMaxSplits];
          float M = -INFINITY, L = 0.f;
#pragma unroll
          for (int s2 = 0; s2 < kMaxSplits; ++s2) {
            ws[s2] = s2 < a.splits ? __ldcg(&pml[(((int64_t)t * a.splits + s2) * 2 + rank) * kH + h]).x
                                   : -INFINITY;
            M = fmaxf(M, ws[s2]);
          }
#pragma unroll
          for (int s2 = 0; s2 < kMaxSplits; ++s2) {
            if (s2 < a.splits) {
              const float2 v = __ldcg(&pml[(((int64_t)t * a.splits + s2) * 2 + rank) * kH + h]);
              ws[s2] = (v.x == -INFINITY) ? 0.f : exp2f(v.x - M);
              L += ws[s2] * v.y;
            } else {
              ws[s2] = 0.f;
            }
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            const int d0 = (col0 + 32 * cc) / 4;
            float acc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) {
              if (s2 < a.splits) {
                const float w = ws[s2];
                if (s2 == sp) {
                  float o[32];
                  load_o(tmem + lane_off + kColO + col0 + 32 * cc, empty, o);
#pragma unroll
                  for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, o[i], acc[i]);
                } else {
                  const int64_t u = (((int64_t)t * a.splits + s2) * 2 + rank) * per_unit;
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const float4 v = __ldcg(po + u + (int64_t)(d0 + i) * kH + h);
                    acc[4 * i] = fmaf(w, v.x, acc[4 * i]);
                    acc[4 * i + 1] = fmaf(w, v.y, acc[4 * i + 1]);
                    acc[4 * i + 2] = fmaf(w, v.z, acc[4 * i + 2]);
                    acc[4 * i + 3] = fmaf(w, v.w, acc[4 * i + 3]);
                  }
                }
              }
            }
            stage_bf16(stg, h, (col0 + 32 * cc) / 8, acc, inv);
          }
          if (half == 0 && rank == 0 && a.lse)
            a.lse[ro] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        }
      }
      if (write_out) {
        named_bar_sync(4, 256);
        // 128 rows x 32 pieces of 16 bytes; a warp writes one row's 512 bytes
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + (int64_t)t * kH * kDC + 256 * rank;
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
          const int i = sidx + 256 * k, row = i >> 5, ch = i & 31;
          const uint4 v = *reinterpret_cast<const uint4*>(stg + row * 512 + ((ch ^ (row & 31)) << 4));
          reinterpret_cast<uint4*>(out + (int64_t)row * kDC)[ch] = v;
        }
      }
    } else {
      // a bounded wait ran out (recorded in the status word): zeros
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + ro * kDC + 256 * rank + col0);
#pragma unroll 1
      for (int i = 0; i < 16; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no remote access to this CTA's shared memory is still pending
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool mla_tc_supported(const MlaArgs& a) {
  return a.mla_dtype == DSA_BF16 && a.n_heads == kH && a.d_c == kDC && a.d_r == kDR &&
         a.topk <= kMaxKeys && a.topk >= 1;
}

// Key splits of a decode batch: enough (row, split) CTA pairs to cover the SMs once.
int mla_tc_splits(int num_rows) {
  if (num_rows <= 0) return 1;
  const int pairs = device_sm_count() / 2;
  int s = 1;
  while (s < kMaxSplits && (int64_t)num_rows * s * 2 <= pairs) s <<= 1;
  return s;
}

// Split-K scratch: partial O (fp32) and (max, sum) per (row, split, head), then
// one 8-byte arrival ticket per (row, CTA rank).
size_t mla_ws_bytes(int num_rows, int n_heads, int d_c, int splits) {
  if (splits <= 1) return 0;
  return (size_t)num_rows * splits * n_heads * (d_c * sizeof(float) + 4 * sizeof(float)) +
         (size_t)num_rows * 2 * sizeof(unsigned long long);
}

static_assert(sizeof(MlaSmem) + 1024 <= 227 * 1024, "shared memory of the attention kernel");

// The kernel moves registers between warpgroups (setmaxnreg): the increases
// wait until the decreases have returned enough registers, which needs the
// launch to hold exactly the register budget the split was sized for.  A
// build whose register count differs is refused instead of launched.
dsa_status check_register_split() {
  static std::atomic<int> ok[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_error("no current CUDA device");
    return DSA_ERR_CUDA;
  }
  if (dev >= 0 && dev < kMaxDevices && ok[dev].load(std::memory_order_acquire) == 1) return DSA_OK;
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, mla_tc_kernel) != cudaSuccess) {
    set_error("cudaFuncGetAttributes(mla_tc_kernel) failed");
    return DSA_ERR_CUDA;
  }
  if (fa.numRegs != kRegsLaunch) {
    set_error("mla_tc_kernel built with %d registers per thread; its warpgroup register split "
              "needs exactly %d", fa.numRegs, kRegsLaunch);
    return DSA_ERR_UNSUPPORTED;
  }
  if (dev >= 0 && dev < kMaxDevices) ok[dev].store(1, std::memory_order_release);
  return DSA_OK;
}

// Clusters of four attention CTAs that can be resident at once on this device
// (0 if the query fails), looked up once per device.
int max_merge_clusters(size_t smem) {
  static std::atomic<int> cached[kMaxDevices];
  static std::atomic<bool> have[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (have[dev].load()) return cached[dev].load();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 4;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, mla_tc_kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cached[dev].store(n);
  have[dev].store(true);
  return n;
}

dsa_status launch_mla_tc(const MlaArgs& a, cudaStream_t stream) {
  if (a.num_rows == 0) return DSA_OK;
  const size_t smem = sizeof(MlaSmem) + 1024;
  static std::atomic<bool> attr[kMaxDevices] = {};
  if (dsa_status st = set_smem_limit_once(reinterpret_cast<const void*>(mla_tc_kernel), smem, attr))
    return st;
  if (dsa_status st = check_register_split()) return st;
  const int keys_per_split = (int)(ceil_div64(ceil_div64(a.topk, a.splits), kBlk) * kBlk);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.num_rows * a.splits * 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // Two key splits of a row run as one 4-CTA cluster and merge through shared
  // memory when every cluster of the grid can be resident at once.
  MlaArgs la = a;
  la.merge_in_cluster = a.splits == 2 && a.num_rows <= max_merge_clusters(smem) ? 1 : 0;
  cudaLaunchAttribute attr2[2];
  attr2[0].id = cudaLaunchAttributeClusterDimension;
  attr2[0].val.clusterDim.x = la.merge_in_cluster ? 4 : 2;
  attr2[0].val.clusterDim.y = 1;
  attr2[0].val.clusterDim.z = 1;
  attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr2;
  cfg.numAttrs = 2;
  // a launch id for the split arrival tickets: distinct for consecutive launches, never 0
  static std::atomic<uint32_t> launch_seq{0};
  do la.launch_id = launch_seq.fetch_add(1u) + 1u; while (la.launch_id == 0u);
  cudaError_t e = cudaLaunchKernelEx(&cfg, mla_tc_kernel, la, keys_per_split);
  if (e != cudaSuccess) {
    set_error("mla_tc launch: %s", cudaGetErrorString(e));
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
