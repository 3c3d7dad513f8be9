// IBCS, the intra-block clustering selector, for sm_100a.
//
// AB-Attention page ("AB-Attention: Video Difüzyon Transformer'larını
// Hızlandırmak İçin Doğru Blok Dikkat Mekanizması"), section "AB-Attention ve
// Üç Temel Yeniliği", IBCS item: the queries of each query block are clustered
// in place (no token permutation) and the clusters estimate each KV block's
// importance cheaply.  Three kernels:
//
//  ksum_kernel    kbar_j = mean of the valid keys of KV block j (bf16 out).
//                 One warp per KV block; HBM-bound.
//  kmeans_kernel  Lloyd k-means of one query block.  Distances come from
//                 |mu_c|^2 - 2 q.mu_c with q.mu_c on the tensor cores (the
//                 fp32 centroid split into bf16 hi + lo parts, two
//                 accumulating MMAs, so the dot products keep ~16 bits);
//                 argmin per query, then the per-cluster sums as a second
//                 product Q^T x onehot(assignment) with fp32 accumulation.
//  score_kernel   S = mu kbar^T / sqrt(d) on the tensor cores for 128/C query
//                 blocks at once (M = 128 centroid rows, N = 128 KV blocks per
//                 chunk), per-centroid softmax over j in two passes (max and
//                 sum, then normalised values), then the cluster-share mixture
//                 P_ij = sum_c (n_c / n_i) p_cj reduced across the C lanes of
//                 each query block with warp shuffles.
#pragma once

#include "ab_ptx.cuh"
#include "ab_sample.cuh"

namespace ab {

// ------------------------------------------------------------------- ksum
template <int D>
__global__ void __launch_bounds__(256) ksum_kernel(const __nv_bfloat16* __restrict__ K,
                                                   __nv_bfloat16* __restrict__ Ksum, int BH, int L,
                                                   int Nkv, int kv_block) {
  constexpr int kPer = D / 32;  // dims per lane
  const int warp_global = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (warp_global >= BH * Nkv) return;
  const int bh = warp_global / Nkv;
  const int j = warp_global - bh * Nkv;
  const int n = min(kv_block, L - j * kv_block);
  const __nv_bfloat16* src = K + (int64_t(bh) * L + int64_t(j) * kv_block) * D + lane * kPer;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  for (int t = 0; t < n; ++t) {
    if constexpr (kPer == 4) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src + int64_t(t) * D));
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
      acc[0] += __low2float(a);
      acc[1] += __high2float(a);
      acc[2] += __low2float(b);
      acc[3] += __high2float(b);
    } else {
      const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(src + int64_t(t) * D));
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw);
      acc[0] += __low2float(a);
      acc[1] += __high2float(a);
    }
  }
  const float inv = 1.f / float(n);
  __nv_bfloat16* dst = Ksum + (int64_t(bh) * Nkv + j) * D + lane * kPer;
  if constexpr (kPer == 4) {
    uint2 out;
    out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = out;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
}

// ----------------------------------------------------------------- k-means
// Shared memory of one k-means CTA.  With C <= 8 the hi tile holds the hi
// parts in rows 0 .. C-1 and the lo parts in rows C .. 2C-1, and the second
// tile is the one-hot assignment tile alone; with C = 16 the one-hot tile
// aliases the lo-part tile: the distance product that reads the lo part has
// completed before the one-hot is written, and the sum product that reads the
// one-hot has completed before the next lo part is written.  Rows no part or
// cluster uses stay zero.
template <int D>
struct KmSmem {
  static constexpr int kOffQ = 0;                      // 128 x 128 bf16, SW128 slabs of 16 KB (slab 1 unused if D = 64)
  static constexpr int kOffBhi = kOffQ + 2 * 16384;    // 16 x D bf16, SW128 slabs of 2 KB
  static constexpr int kOffBlo = kOffBhi + 2 * 2048;   // 16 x D bf16 / one-hot 16 x 128 queries
  static constexpr int kOffMusq = kOffBlo + 2 * 2048;  // float [16][4 warps], partial |mu_c|^2
  static constexpr int kOffWcnt = kOffMusq + 256;      // int [16][4 warps], partial cluster sizes
  static constexpr int kOffBar = kOffWcnt + 256;
  static constexpr int kOffMisc = kOffBar + 16;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

// Element (row, e) of a 128B-swizzled K-major bf16 tile with `slab_bytes`
// slabs of 64 columns: byte offset.
__device__ __forceinline__ uint32_t sw_tile_off(int slab_bytes, int row, int e) {
  const int slab = e >> 6, col = e & 63;
  return uint32_t(slab * slab_bytes) + sw128_offset(uint32_t(row), uint32_t(col >> 3)) + uint32_t((col & 7) * 2);
}

// Warp sum of N values per lane (N a power of two <= 32) by recursive halving:
// lane l returns the total of value (l >> (5 - log2 N)).
template <int N>
__device__ __forceinline__ float warp_sum_scatter(const float (&in)[N]) {
  static_assert(N >= 1 && N <= 32 && (N & (N - 1)) == 0, "N must be a power of two <= 32");
  const int lane = threadIdx.x & 31;
  float v[N];
#pragma unroll
  for (int k = 0; k < N; ++k) v[k] = in[k];
  int off = 16;
#pragma unroll
  for (int n = N; n > 1; n >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < n / 2; ++k) {
      const float send = upper ? v[k] : v[k + n / 2];
      const float keep = upper ? v[k + n / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  return r;
}

// One CTA (128 threads) per query block.  Thread e < D keeps dimension e of
// every centroid in registers.  Per Lloyd iteration, two small tensor-core
// products:
//   distances  q . mu_c = Q (128 x d) x [mu_hi; mu_lo]^T: for C <= 8 one
//              product with N = 16 (hi parts in columns c, lo parts in C + c,
//              added by the thread; half the MMAs to issue), for C = 16 two
//              products accumulating in the same 16 columns; thread q reads
//              its columns and takes argmin |mu_c|^2 - 2 q . mu_c;
//   sums       sum_{q in c} q = Q^T (d x 128) x onehot (128 x 16): Q is read
//              as an MN-major operand (d contiguous), so thread e receives the
//              sums of dimension e for every cluster in 16 TMEM columns.
// Outputs: centroids (fp32, optional), counts (optional), and for the scorer
// the bf16 centroids and int counts.
template <int D, int C>
__global__ void __launch_bounds__(128, C <= 8 ? 5 : 3) kmeans_kernel(const __grid_constant__ CUtensorMap tmQ, int L, int Nq,
                                                     int q_block, int iters, float* __restrict__ cent_out,
                                                     int32_t* __restrict__ counts_out,
                                                     __nv_bfloat16* __restrict__ cent_ws,
                                                     int32_t* __restrict__ counts_ws) {
  using SM = KmSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* musq_part = reinterpret_cast<float*>(smem + SM::kOffMusq);  // [16][4]
  int* wcnt = reinterpret_cast<int*>(smem + SM::kOffWcnt);           // [16][4]
  const uint32_t bar_q = sbase + SM::kOffBar, bar_mma = sbase + SM::kOffBar + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / Nq;
  const int qi = blockIdx.x - bh * Nq;
  const int n_i = min(q_block, L - qi * q_block);
  const bool own_dim = tid < D;  // thread e = tid holds dimension e of every centroid

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(bar_q, (D / 64) * 16384);
    for (int s = 0; s < D / 64; ++s)
      tma_load_3d(sbase + SM::kOffQ + s * 16384, &tmQ, bar_q, s * 64, qi * q_block, bh);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 32);  // columns 0-15 distances, 16-31 sums
    tmem_relinquish();
  }
  // centroid tiles start zero (rows >= C stay zero)
  for (int k = tid; k < 2 * 2 * 2048 / 16; k += 128)
    reinterpret_cast<uint4*>(smem + SM::kOffBhi)[k] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tlane = uint32_t(warp * 32) << 16;

  bool ok = mbar_wait(bar_q, 0, abort_flag);
  ok = __syncthreads_and(ok);

  const uint8_t* qtile = smem + SM::kOffQ;
  // initial centroids: the query at offset floor((c + 1/2) n_i / C)
  float mu[C];
  int cnt[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int src = ((2 * c + 1) * n_i) / (2 * C);
    mu[c] = own_dim ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qtile + sw_tile_off(16384, src, tid)))
                    : 0.f;
    cnt[c] = 0;
  }

  const uint32_t id_dist = idesc_bf16_f32(128, 16, 0, 0);  // Q (K-major) x mu parts (K-major)
  const uint32_t id_sum = idesc_bf16_f32(128, 16, 1, 0);   // Q^T (MN-major) x onehot (K-major)
  // With C <= 8 the lo parts sit in rows C .. 2C-1 of the hi tile, so one
  // N = 16 product gives both (columns c and C + c); with C = 16 they take
  // a tile and a product of their own.
  constexpr bool kPacked = 2 * C <= 16;
  // operand descriptors, built once; each MMA adds its byte offset
  const SmemDesc dq = smem_desc_base(sbase + SM::kOffQ, 16, 1024);        // Q, K-major
  const SmemDesc dqt = smem_desc_base(sbase + SM::kOffQ, 16384, 1024);    // Q read MN-major
  const SmemDesc dhi = smem_desc_base(sbase + SM::kOffBhi, 16, 1024);
  const SmemDesc dlo = smem_desc_base(sbase + SM::kOffBlo, 16, 1024);     // lo parts / one-hot
  uint32_t phase = 0;
  for (int it = 0; it < iters && ok; ++it) {
    // centroid tiles: bf16 hi and lo parts of mu (row c, column e); partial |mu_c|^2
    float m2[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
      m2[c] = mu[c] * mu[c];
      if (own_dim) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(mu[c]);
        const __nv_bfloat16 lo = __float2bfloat16_rn(mu[c] - __bfloat162float(hi));
        *reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffBhi + sw_tile_off(2048, c, tid)) = hi;
        if constexpr (kPacked) {
          *reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffBhi + sw_tile_off(2048, C + c, tid)) = lo;
        } else {
          *reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffBlo + sw_tile_off(2048, c, tid)) = lo;
        }
      }
    }
    {
      const float part = warp_sum_scatter<C>(m2);
      constexpr int kLanesPer = 32 / C;
      if ((lane & (kLanesPer - 1)) == 0) musq_part[(lane / kLanesPer) * 4 + warp] = part;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * 2048 + (kk & 3) * 32;
        mma_bf16_ss(tmem, desc_at(dq, aoff), desc_at(dhi, boff), id_dist, kk > 0 ? 1u : 0u);
        if constexpr (!kPacked) mma_bf16_ss(tmem, desc_at(dq, aoff), desc_at(dlo, boff), id_dist, 1u);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, phase & 1, abort_flag);
    ++phase;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    // dot products of this thread's query with the 16 centroid rows
    uint32_t dv[16];
    tmem_ld16(tmem + tlane, dv);
    tmem_wait_ld();
    int best = C;  // C marks "no query" (rows beyond the block)
    if (tid < n_i) {
      float bd = INFINITY;
      best = 0;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const float4 p4 = *reinterpret_cast<const float4*>(musq_part + 4 * c);
        const float musq = (p4.x + p4.y) + (p4.z + p4.w);
        const float dot = kPacked ? __uint_as_float(dv[c]) + __uint_as_float(dv[C + c]) : __uint_as_float(dv[c]);
        const float dist = fmaf(-2.f, dot, musq);
        if (dist < bd) {  // strict: ties go to the lower c
          bd = dist;
          best = c;
        }
      }
    }
    // cluster sizes (ballots) and this query's one-hot column (over the lo tile)
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const uint32_t bal = __ballot_sync(0xffffffffu, best == c);
      if (lane == 0) wcnt[4 * c + warp] = __popc(bal);
      const uint32_t off = uint32_t((tid >> 6) * 2048) + sw128_offset(uint32_t(c), uint32_t((tid & 63) >> 3)) +
                           uint32_t((tid & 7) * 2);
      *reinterpret_cast<__nv_bfloat16*>(smem + SM::kOffBlo + off) = __float2bfloat16_rn(best == c ? 1.f : 0.f);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // K = 128 queries, 16 per step
        mma_bf16_ss(tmem + 16u, desc_at(dqt, kk * 2048), desc_at(dlo, (kk >> 2) * 2048 + (kk & 3) * 32), id_sum,
                    kk > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, phase & 1, abort_flag);
    ++phase;
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    // new centroid = sum of members / count (thread e holds dimension e); an
    // empty cluster keeps its centroid
    uint32_t sv[16];
    tmem_ld16(tmem + tlane + 16u, sv);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int4 w4 = *reinterpret_cast<const int4*>(wcnt + 4 * c);
      cnt[c] = (w4.x + w4.y) + (w4.z + w4.w);
      // the sum is exact (bf16 values times a 0/1 one-hot, accumulated in
      // fp32); dividing by the count with the reciprocal instruction (2 ulp)
      // instead of an IEEE division takes a fifth of the update's time
      if (own_dim && cnt[c] > 0) mu[c] = __fdividef(__uint_as_float(sv[c]), float(cnt[c]));
    }
  }

  {
    // A wait that gave up (AB_ERR_TIMEOUT recorded) leaves markers instead
    // of results: NaN centroids and count -1, so that the scores built from
    // them are NaN rather than values left in the workspace by an earlier call.
    const int64_t row0 = (int64_t(bh) * Nq + qi) * C;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      if (own_dim) {
        const float m = ok ? mu[c] : __uint_as_float(0x7fc00000u);
        if (cent_out) cent_out[(row0 + c) * D + tid] = m;
        cent_ws[(row0 + c) * D + tid] = __float2bfloat16_rn(m);
      }
      if (tid == c) {
        if (counts_out) counts_out[row0 + c] = ok ? cnt[c] : -1;
        counts_ws[row0 + c] = ok ? cnt[c] : -1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

// Maximum of v[0 .. N) as a balanced tree of 3-input max operations.
template <int N>
__device__ __forceinline__ float max_tree(const float* v) {
  if constexpr (N == 1) {
    return v[0];
  } else if constexpr (N == 2) {
    return fmaxf(v[0], v[1]);
  } else if constexpr (N == 3) {
    return fmax3(v[0], v[1], v[2]);
  } else {
    constexpr int kA = N / 3, kB = (N - kA) / 2;
    return fmax3(max_tree<kA>(v), max_tree<kB>(v + kA), max_tree<N - kA - kB>(v + kA + kB));
  }
}

// ------------------------------------------------------------------ scores
template <int D, bool kSample = false>
struct ScSmem {
  static constexpr int kSlabs = D / 64;
  static constexpr int kSampleRows = 9 * 16 * 512;  // kSample: nine warps' quantised rows, over A and B
  static constexpr int kA = kSlabs * 16384;          // 128 centroid rows x D bf16
  static constexpr int kB = kSlabs * 16384;          // 128 K summaries x D bf16 (one chunk)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kA;           // 2 stages
  static constexpr int kEndB = kOffB + 2 * kB;
  static constexpr int kOffW = kSample && kSampleRows > kEndB ? kSampleRows : kEndB;  // float [128] row weights
  static constexpr int kOffX = kOffW + 512;          // float [2 halves][2][128] max/sum exchange
  static constexpr int kOffBar = kOffX + 2048;       // a_full, b_full[2], b_empty[2], s_full[2], t_free[2], drain, xch
  static constexpr int kOffMisc = kOffBar + 12 * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(!kSample || kSampleRows <= kOffW, "the sampling rows end before the row weights");
};

struct ScoreArgs {
  int L, Nq, Nkv, q_block, kv_block;
  const int32_t* counts_ws;  // [BH, Nq, C]
  float* P;                  // [BH, Nq, Nkv]
  float scale_log2;          // log2(e) / sqrt(d)
  float last_bias;           // log2(n_last / kv_block) of the last KV block
  SipArgs sip;               // kSample: SIP of the CTA's rows right after their P (P = sip.P rows)
};

// Reduce 32 per-lane values over aligned groups of C lanes and scatter the
// sums: after the call lane g (g = lane % C) of a group holds, in v[0 ..
// 32/C), the group sums of columns [g * 32/C, (g + 1) * 32/C).
template <int C>
__device__ __forceinline__ void group_reduce_scatter(float (&v)[32], int lane) {
#pragma unroll
  for (int m = C / 2; m >= 1; m >>= 1) {
    const bool upper = (lane & m) != 0;
    const int half = 32 * m / C;  // values still held per lane, halved by this stage
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < half) {
        const float send = upper ? v[k] : v[k + half];
        const float keep = upper ? v[k + half] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
  }
}

// Warps 0-7 read the scores (warp w: TMEM lanes 32 (w % 4).., columns
// [64 (w / 4), +64) of every 128-column chunk), warp 8 loads and issues the
// MMAs.  Two CTAs share an SM (96 KB of shared memory, 256 TMEM columns each).  The two column halves of a row keep separate running max / sum in
// the first pass and merge them before the second.
// kSample (rows of at most 2048 blocks): once the CTA's rows of P are written,
// its nine warps run SIP on them (sip_warp_row, one warp per row, each row's
// weights in 8 KB of the shared memory the scoring no longer uses), so the
// sampling of these rows starts as soon as their estimate exists, next to the
// scoring of the other CTAs, without a second launch or a DRAM round trip of
// P (it is read back from L2).
template <int D, int C, bool kSample = false>
__global__ void __launch_bounds__(288, 2)
    score_kernel(const __grid_constant__ CUtensorMap tmCent, const __grid_constant__ CUtensorMap tmKsum,
                 const ScoreArgs a) {
  using SM = ScSmem<D, kSample>;
  constexpr int G = 128 / C;  // query blocks per CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SM::kOffBar;
  auto bar = [&](int k) { return bar0 + 8u * uint32_t(k); };
  enum { kA = 0, kBFull = 1, kBEmpty = 3, kSFull = 5, kTFree = 7, kDrain = 9, kXch = 10 };
  float* roww = reinterpret_cast<float*>(smem + SM::kOffW);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int groups_per_head = (a.Nq + G - 1) / G;
  const int bh = blockIdx.x / groups_per_head;
  const int i0 = (blockIdx.x - bh * groups_per_head) * G;
  const int nchunks = (a.Nkv + 127) / 128;

  if (tid == 0) {
    mbar_init(bar(kA), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBFull + s), 1);
      mbar_init(bar(kBEmpty + s), 1);
      mbar_init(bar(kSFull + s), 1);
      mbar_init(bar(kTFree + s), 8);  // one arrival per reader warp
    }
    mbar_init(bar(kDrain), 1);
    mbar_init(bar(kXch), 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 128) {
    // row r = (query block i0 + r / C, centroid r % C): weight n_c / n_i (0 if none)
    const int i = i0 + tid / C;
    float w = 0.f;
    if (tid < G * C && i < a.Nq) {
      const int n_i = min(a.q_block, a.L - i * a.q_block);
      w = float(a.counts_ws[(int64_t(bh) * a.Nq + i) * C + (tid % C)]) / float(n_i);
    }
    roww[tid] = w;
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = 2 * nchunks;  // pass 0: max and sum; pass 1: values

  if (warp == 8) {
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(bar(kA), SM::kA);
      for (int s = 0; s < SM::kSlabs; ++s)
        tma_load_3d(sbase + SM::kOffA + s * 16384, &tmCent, bar(kA), s * 64, (bh * a.Nq + i0) * C, 0);
      auto load_b = [&](int g) {
        const int st = g & 1;
        const int chunk = g % nchunks;
        mbar_arrive_expect_tx(bar(kBFull + st), SM::kB);
        for (int s = 0; s < SM::kSlabs; ++s)
          tma_load_3d(sbase + SM::kOffB + st * SM::kB + s * 16384, &tmKsum, bar(kBFull + st), s * 64,
                      chunk * 128, bh);
      };
      load_b(0);
      if (total > 1) load_b(1);
      ok = mbar_wait(bar(kA), 0, abort_flag);
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      for (int g = 0; g < total && ok; ++g) {
        const int st = g & 1;
        if (!mbar_wait(bar(kBFull + st), (g >> 1) & 1, abort_flag)) { ok = false; break; }
        if (g >= 2 && !mbar_wait(bar(kTFree + st), ((g - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + uint32_t(st * 128), smem_desc_sw128(sbase + SM::kOffA + aoff, 16, 1024),
                      smem_desc_sw128(sbase + SM::kOffB + st * SM::kB + boff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kSFull + st));
        mma_commit(bar(kBEmpty + st));
        if (g + 2 < total) {
          if (!mbar_wait(bar(kBEmpty + st), (g >> 1) & 1, abort_flag)) { ok = false; break; }
          load_b(g + 2);
        }
      }
      mma_commit(bar(kDrain));
      mbar_wait_drain(bar(kDrain), 0);
    }
  } else {
    const int r = tid & 127;   // centroid row == TMEM lane
    const int ch = warp >> 2;  // column half of every chunk
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float w = roww[r];
    const float sc = a.scale_log2;
    float* xm = reinterpret_cast<float*>(smem + SM::kOffX);  // [2][2][128]: max, sum per half
    // Scores are kept in raw units s (x = s * sc); the running max M is in
    // the x (log2) domain.  Columns past Nkv read as -inf; the last block's
    // log2(n_last / kv_block) is added to its raw score as bias / sc.
    const float last_raw = a.last_bias / sc;
    float M = -INFINITY, Z = 0.f;
    bool ok = true;
    for (int g = 0; g < total && ok; ++g) {
      const int st = g & 1;
      const int chunk = g % nchunks;
      const bool pass2 = g >= nchunks;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(kSFull + st), (g >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // all 64 columns of this half at once, then release the TMEM buffer
      float v[64];
#pragma unroll
      for (int piece = 0; piece < 2; ++piece)
        tmem_ld32_nowait(tmem + lane_base + uint32_t(st * 128 + ch * 64 + piece * 32),
                         reinterpret_cast<uint32_t*>(v) + piece * 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kTFree + st));
      const int j0 = chunk * 128 + ch * 64;
      if (j0 + 64 > a.Nkv - 1) {  // this half holds the last block or columns past Nkv
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const int j = j0 + k;
          v[k] = j < a.Nkv - 1 ? v[k] : (j == a.Nkv - 1 ? v[k] + last_raw : -INFINITY);
        }
      }
      if (g == nchunks) {
        // merge the two halves' running max and sum before the second pass
        xm[(0 * 2 + ch) * 128 + r] = M;
        xm[(1 * 2 + ch) * 128 + r] = Z;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kXch));
        ok = __all_sync(0xffffffffu, mbar_wait(bar(kXch), 0, abort_flag));
        if (!ok) break;
        const float M2 = xm[(0 * 2 + (ch ^ 1)) * 128 + r], Z2 = xm[(1 * 2 + (ch ^ 1)) * 128 + r];
        const float Mx = fmaxf(M, M2);  // at least one half has a valid column
        Z = (M == -INFINITY ? 0.f : Z * ex2_approx(M - Mx)) + (M2 == -INFINITY ? 0.f : Z2 * ex2_approx(M2 - Mx));
        M = Mx;
      }
      if (!pass2) {
        const float pm = fmaxf(M, max_tree<64>(v) * sc);
        if (pm != -INFINITY) {  // a half entirely past Nkv changes nothing
          const float nm = -pm;
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < 64; ++k) s4[k & 3] += ex2_approx(fmaf(v[k], sc, nm));
          Z = (M == -INFINITY ? 0.f : Z * ex2_approx(M - pm)) + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
          M = pm;
        }
      } else {
        // p_cj n_c / n_i = exp2(x - M + log2(w / Z)): the row weight rides in the exponent
        const float nm = w > 0.f ? __log2f(w / Z) - M : -INFINITY;
        constexpr int kPer = 32 / C;
        const int gl = lane % C;
        const int i = i0 + r / C;
        const bool store = i < a.Nq && (r / C) < G;
        float* prow = a.P + (int64_t(bh) * a.Nq + (store ? i : 0)) * a.Nkv;
#pragma unroll
        for (int piece = 0; piece < 2; ++piece) {
          float u[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) u[k] = ex2_approx(fmaf(v[piece * 32 + k], sc, nm));
          group_reduce_scatter<C>(u, lane);
          if (store) {
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
              const int j = j0 + piece * 32 + gl * kPer + k;
              if (j < a.Nkv) prow[j] = u[k];
            }
          }
        }
      }
    }
  }
  if constexpr (kSample) __threadfence();  // P visible in L2 to the sampling warps below
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if constexpr (kSample) {
    if (!*abort_flag) {
      for (int r = warp; r < G; r += 9) {
        const int i = i0 + r;
        if (i < a.Nq) sip_warp_row<16, false, true>(a.sip, bh * a.Nq + i, reinterpret_cast<uint4*>(smem) + warp * 32 * 16);
      }
    }
  }
}

}  // namespace ab
