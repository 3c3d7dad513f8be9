// SIP, sampling with inclusion-probability weighting, for sm_100a.
//
// AB-Attention page ("AB-Attention: Video Difüzyon Transformer'larını
// Hızlandırmak İçin Doğru Blok Dikkat Mekanizması"), section "AB-Attention ve
// Üç Temel Yeniliği", SIP item: KV blocks are sampled in proportion to the
// IBCS estimate and the kept ones carry their inverse inclusion probability,
// so that the sparse pass estimates dense attention instead of truncating it.
//
// One CTA (256 threads) per query block, all integer arithmetic:
//   W_j = max(1, floor(P_j 2^24));
//   capping: the capped set is always {j : W_j >= theta} (capping is monotone
//   in W), so the fixed point is found by iterating a threshold: with
//   R = Kb - #{W >= theta} and S = sum of W_j below theta, every j with
//   R W_j >= S joins, i.e. theta <- min(theta, ceil(S / R)), until stable;
//   Pi_j = 2^32 above theta, else max(1, floor(R W_j 2^32 / S));
//   keep j iff u_j < Pi_j, with u_j word (j mod 4) of
//   Philox4x32-10((j div 4, i, h, b), (seed lo, seed hi)).  For a free block
//   this is tested without dividing: u < max(1, floor(X/S)) with X = R W 2^32
//   holds iff u == 0 or (u + 1) S <= X.
// Each thread owns 4 consecutive j per 1024-wide chunk (one Philox call per
// thread and chunk).  Phases: (1) the quantised row is cached in shared memory
// (rows up to kSipSmemCap entries; longer rows re-read P); (2) capping rounds,
// one barrier each; (3) draws, with the kept j compacted in ascending order
// by a block-wide scan; (4) Pi of the kept entries, one output position per
// thread, so the exact division runs without divergence.
#pragma once

#include "ab_ptx.cuh"

namespace ab {

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplications of counter
// words 0 and 2, the high halves XORed into words 1 and 3 with the round key,
// the key advanced by the Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t lo0 = 0xD2511F53u * c.x;
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

struct SipArgs {
  const float* P;  // [rows, Nkv]
  int32_t* idx;
  uint32_t* pi_q32;
  int32_t* count;
  int H, Nq, Nkv, Kb;
  uint32_t seed_lo, seed_hi;
  int64_t row0;  // global index of the first row (for the draws' counters): rows are (b, h, i) in order
};

__host__ __device__ __forceinline__ uint32_t quantise_w(float p) {
  const float s = floorf(p * 16777216.0f);
  return s < 1.0f ? 1u : uint32_t(s);  // p <= 1, so s <= 2^24
}

// a S <= X 2^32 for a < 2^32 + 1, S = S_hi 2^32 + S_lo < 2^64, X < 2^64:
// a S = (a S_hi) 2^32 + a S_lo, compared without 128-bit products.
// `a` is passed as a_minus_1 (so that a = 2^32 fits) .
__host__ __device__ __forceinline__ bool mul_le_shift32(uint32_t a_minus_1, uint32_t S_hi, uint32_t S_lo, uint64_t X) {
  const uint64_t t = uint64_t(a_minus_1) * S_lo + S_lo;  // a S_lo < 2^64
  const uint64_t h = uint64_t(a_minus_1) * S_hi + S_hi;  // a S_hi
  if (h > X) return false;
  const uint64_t r = X - h;
  return r >= (1ull << 32) || t <= (r << 32);
}

// Pi = max(1, floor(X 2^32 / S)) < 2^32 for a free block (X = R W < S): a
// double estimate (error below one unit), then the exact test a S <= X 2^32
// moves it to the largest such a.
__host__ __device__ __forceinline__ uint32_t pi_free(uint64_t X, uint32_t S_hi, uint32_t S_lo, double inv_s32) {
  uint64_t est = uint64_t(double(X) * inv_s32);
  if (est > 0xFFFFFFFFull) est = 0xFFFFFFFFull;
  while (est > 0 && !mul_le_shift32(uint32_t(est - 1), S_hi, S_lo, X)) --est;
  while (est < 0xFFFFFFFFull && mul_le_shift32(uint32_t(est), S_hi, S_lo, X)) ++est;
  return est < 1 ? 1u : uint32_t(est);
}

constexpr int kSipThreads = 256;
constexpr int kSipSmemCap = 16384;  // entries of W cached in shared memory (64 KB)

// Systematic sampling with the same inclusion probabilities (the sampling
// design is left open by the pages; SIP item of the AB-Attention page): one
// offset U per row, word 0 of Philox4x32-10 at counter (0xFFFFFFFF, i, h, b);
// with C_j the cumulative Pi in block order, block j is kept iff a point
// U + m 2^32 (m >= 0) lies in [C_j, C_j + Pi_j).  Each block is kept with
// probability Pi_j / 2^32; the sample size is floor or ceil of sum Pi / 2^32.
// A block-wide scan of the 64-bit Pi gives C_j; a second scan places the kept
// blocks in ascending order.
template <typename Load4>
__device__ __forceinline__ void systematic_pass(const SipArgs& a, uint32_t theta, uint64_t R, uint64_t S, int b,
                                                int h, int i, Load4 load4, uint64_t* scan64, int* scan) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int Nkv = a.Nkv;
  const uint32_t S_hi = uint32_t(S >> 32), S_lo = uint32_t(S);
  const uint32_t R32 = uint32_t(R);
  const double inv_s32 = S ? 4294967296.0 / double(S) : 0.0;
  const uint64_t U = philox4x32_10(make_uint4(0xFFFFFFFFu, uint32_t(i), uint32_t(h), uint32_t(b)), a.seed_lo,
                                   a.seed_hi).x;
  auto points_below = [&](uint64_t x) -> uint64_t { return x > U ? ((x - U - 1) >> 32) + 1 : 0; };
  int32_t* out_idx = a.idx + int64_t(row) * Nkv;
  uint32_t* out_pi = a.pi_q32 + int64_t(row) * Nkv;
  uint64_t base_c = 0;
  int base = 0;
  for (int c0 = 0; c0 < Nkv; c0 += 4 * kSipThreads) {
    const int j0 = c0 + 4 * tid;
    uint64_t pis[4] = {0, 0, 0, 0};
    if (j0 < Nkv) {
      uint32_t w[4];
      load4(j0, w);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (j0 + q < Nkv) pis[q] = w[q] >= theta ? (1ull << 32) : uint64_t(pi_free(uint64_t(R32) * w[q], S_hi, S_lo, inv_s32));
    }
    // exclusive block scan of the per-thread Pi sums
    const uint64_t mine = (pis[0] + pis[1]) + (pis[2] + pis[3]);
    uint64_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) scan64[warp] = incl;
    __syncthreads();
    uint64_t woff = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const uint64_t v = scan64[w];
      if (w < warp) woff += v;
      total += v;
    }
    uint64_t C = base_c + woff + incl - mine;
    uint32_t keep_mask = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint64_t next = C + pis[q];
      if (j0 + q < Nkv && points_below(next) - points_below(C) == 1) keep_mask |= 1u << q;
      C = next;
    }
    // ordered positions of the kept blocks
    const int kept = __popc(keep_mask);
    int kincl = kept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, kincl, o);
      if (lane >= o) kincl += y;
    }
    if (lane == 31) scan[warp] = kincl;
    __syncthreads();
    int kwoff = 0, ktotal = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int v = scan[w];
      if (w < warp) kwoff += v;
      ktotal += v;
    }
    int pos = base + kwoff + kincl - kept;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (keep_mask & (1u << q)) {
        out_idx[pos] = j0 + q;
        out_pi[pos] = uint32_t(pis[q] & 0xFFFFFFFFull);
        ++pos;
      }
    }
    base_c += total;
    base += ktotal;
    __syncthreads();  // scan64[] and scan[] are reused by the next chunk
  }
  if (tid == 0) a.count[row] = base;
}

template <bool kCached, bool kSystematic>
__global__ void __launch_bounds__(kSipThreads) sip_kernel(const SipArgs a) {
  __shared__ uint64_t red_sum[2][8];
  __shared__ uint64_t scan64[8];
  __shared__ uint32_t red_cnt[2][8];
  __shared__ int scan[8];
  extern __shared__ uint4 wcache4[];  // [ceil(Nkv / 4)] when cached; entries >= Nkv hold 0
  uint32_t* wcache = reinterpret_cast<uint32_t*>(wcache4);
  const int row = blockIdx.x;
  const int64_t grow = a.row0 + row;
  const int b = int(grow / (int64_t(a.H) * a.Nq));
  const int h = int((grow / a.Nq) % a.H);
  const int i = int(grow % a.Nq);
  const float* P = a.P + int64_t(row) * a.Nkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Nkv = a.Nkv;

  // W of j0 .. j0 + 3 (j0 a multiple of 4, j0 < Nkv); entries >= Nkv read 0
  auto load4 = [&](int j0, uint32_t (&w)[4]) {
    if constexpr (kCached) {
      const uint4 v = wcache4[j0 >> 2];
      w[0] = v.x;
      w[1] = v.y;
      w[2] = v.z;
      w[3] = v.w;
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = j0 + q < Nkv ? quantise_w(__ldg(P + j0 + q)) : 0u;
    }
  };
  if constexpr (kCached) {
    const int n4 = (Nkv + 3) >> 2;
    for (int k = tid; k < 4 * n4; k += kSipThreads) wcache[k] = k < Nkv ? quantise_w(__ldg(P + k)) : 0u;
    __syncthreads();
  }

  // ---- capping threshold (fixed point; at most Nkv + 1 rounds)
  uint32_t theta = 0xFFFFFFFFu;  // above every W: nothing capped
  uint64_t R = 0, S = 0;
  for (int round = 0; round <= Nkv + 1; ++round) {
    uint32_t ncap = 0;
    uint64_t sum = 0;
    for (int j0 = 4 * tid; j0 < Nkv; j0 += 4 * kSipThreads) {
      uint32_t w[4];
      load4(j0, w);
      uint32_t part = 0;  // <= 4 * 2^24
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool cap = w[q] >= theta;
        ncap += cap ? 1u : 0u;
        part += cap ? 0u : w[q];
      }
      sum += part;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ncap += __shfl_xor_sync(0xffffffffu, ncap, o);
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    const int buf = round & 1;  // double buffer: one barrier per round
    if (lane == 0) {
      red_cnt[buf][warp] = ncap;
      red_sum[buf][warp] = sum;
    }
    __syncthreads();
    uint64_t nc = 0;
    S = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      nc += red_cnt[buf][w];
      S += red_sum[buf][w];
    }
    R = uint64_t(a.Kb) - nc;
    if (R == 0 || S == 0) break;
    // ceil(S / R): double quotient, then exact integer correction
    uint64_t q = uint64_t(double(S) / double(R));
    while (q * R > S) --q;
    while ((q + 1) * R <= S) ++q;
    const uint64_t t_new = q + (q * R != S ? 1u : 0u);  // R W >= S  <=>  W >= ceil(S / R)
    if (t_new >= theta) break;
    theta = uint32_t(t_new);  // t_new < theta <= 2^32 - 1
  }

  if constexpr (kSystematic) {
    systematic_pass(a, theta, R, S, b, h, i, load4, scan64, scan);
    return;
  }
  // ---- draws and ordered compaction, 4 consecutive j per thread per chunk
  const uint32_t k0 = a.seed_lo, k1 = a.seed_hi;
  const uint32_t S_hi = uint32_t(S >> 32), S_lo = uint32_t(S);
  const uint32_t R32 = uint32_t(R);  // R <= Kb < 2^31
  int32_t* out_idx = a.idx + int64_t(row) * Nkv;
  uint32_t* out_pi = a.pi_q32 + int64_t(row) * Nkv;
  int base = 0;
  for (int c0 = 0; c0 < Nkv; c0 += 4 * kSipThreads) {
    const int j0 = c0 + 4 * tid;
    uint32_t keep_mask = 0;
    if (j0 < Nkv) {
      const uint4 u4 = philox4x32_10(make_uint4(uint32_t(j0 >> 2), uint32_t(i), uint32_t(h), uint32_t(b)), k0, k1);
      const uint32_t us[4] = {u4.x, u4.y, u4.z, u4.w};
      uint32_t w[4];
      load4(j0, w);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        bool keep;
        if (w[q] >= theta) {
          keep = true;  // capped: pi = 1
        } else {
          const uint64_t X = uint64_t(R32) * w[q];
          keep = us[q] == 0u || mul_le_shift32(us[q], S_hi, S_lo, X);  // (u + 1) S <= X 2^32
        }
        if (keep && j0 + q < Nkv) keep_mask |= 1u << q;
      }
    }
    // exclusive scan of the per-thread kept counts, in thread (= j) order
    const int mine = __popc(keep_mask);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) scan[warp] = incl;
    __syncthreads();
    int warp_off = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int v = scan[w];
      if (w < warp) warp_off += v;
      total += v;
    }
    int pos = base + warp_off + incl - mine;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (keep_mask & (1u << q)) out_idx[pos++] = j0 + q;
    }
    base += total;
    __syncthreads();  // scan[] is reused by the next chunk; out_idx is read below
  }

  // ---- inclusion probabilities of the kept entries
  // Pi = max(1, floor(X 2^32 / S)) < 2^32 for a free entry: a double estimate
  // (error below one unit), then the exact test a S <= X 2^32 moves it to the
  // largest such a.
  const double inv_s32 = S ? 4294967296.0 / double(S) : 0.0;
  for (int k = tid; k < base; k += kSipThreads) {
    const int j = out_idx[k];
    const uint32_t w = kCached ? wcache[j] : quantise_w(__ldg(P + j));
    out_pi[k] = w < theta ? pi_free(uint64_t(R32) * w, S_hi, S_lo, inv_s32) : 0u;  // capped: Pi = 2^32
  }
  if (tid == 0) a.count[row] = base;
}

// One warp per row, for rows of at most 32 * 4 * KMAX blocks: the same
// arithmetic as sip_kernel (results are identical integers), with the
// quantised row in the warp's own slice of shared memory and warp shuffles
// instead of block barriers.
// Lane l owns blocks j = 128 k + 4 l + q (k < KMAX, q < 4), i.e. the same 4
// consecutive blocks per Philox call.  kSystematic: systematic sampling with
// the same Pi (as systematic_pass: one offset U per row, block j kept iff a
// point U + m 2^32 lies in [C_j, C_j + Pi_j), C_j the running sum of Pi in
// ascending j, here a warp scan per 128-block chunk).
// One warp samples row `row` of a.P (Nkv <= 128 KMAX), the whole row's
// quantised weights in this warp's KMAX x 512 bytes of shared memory at
// `wsm` (16-byte aligned; lane l keeps its four weights of chunk k at uint4
// index 32 k + l, so a warp's loads are contiguous).  Holding the row in
// registers instead (64 per lane at KMAX = 16) left 16 warps per SM and
// took 9 % longer.  kCoherent: P was written earlier by the calling kernel
// itself, so it is read through L2 (__ldcg) rather than the read-only path,
// which is only valid for data the kernel does not write.
template <int KMAX, bool kSystematic, bool kCoherent>
__device__ __forceinline__ void sip_warp_row(const SipArgs& a, int row, uint4* wsm) {
  static_assert(KMAX * 4 * 16777216ull < 4294967296ull, "per-lane partial sums must fit 32 bits");
  const int lane = threadIdx.x & 31;
  auto loadP = [](const float* p) { return kCoherent ? __ldcg(p) : __ldg(p); };
  const int64_t grow = a.row0 + row;
  const int b = int(grow / (int64_t(a.H) * a.Nq));
  const int h = int((grow / a.Nq) % a.H);
  const int i = int(grow % a.Nq);
  const int Nkv = a.Nkv;
  const float* P = a.P + int64_t(row) * Nkv;
  // the four weights of chunk k of this lane
  auto wk = [&](int k) -> uint4 { return wsm[32 * k + lane]; };
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    uint32_t v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = 128 * k + 4 * lane + q;
      v[q] = j < Nkv ? quantise_w(loadP(P + j)) : 0u;  // entries >= Nkv: 0, never capped
    }
    wsm[32 * k + lane] = make_uint4(v[0], v[1], v[2], v[3]);
  }

  // ---- capping threshold (fixed point)
  uint32_t theta = 0xFFFFFFFFu;
  uint64_t R = 0, S = 0;
  for (int round = 0; round <= Nkv + 1; ++round) {
    uint32_t ncap = 0, part = 0;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      const uint4 v4 = wk(k);
      const uint32_t v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool cap = v[q] >= theta;
        ncap += cap ? 1u : 0u;
        part += cap ? 0u : v[q];
      }
    }
    uint64_t sum = part;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ncap += __shfl_xor_sync(0xffffffffu, ncap, o);
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    R = uint64_t(a.Kb) - ncap;
    S = sum;
    if (R == 0 || S == 0) break;
    uint64_t qt = uint64_t(double(S) / double(R));
    while (qt * R > S) --qt;
    while ((qt + 1) * R <= S) ++qt;
    const uint64_t t_new = qt + (qt * R != S ? 1u : 0u);  // ceil(S / R)
    if (t_new >= theta) break;
    theta = uint32_t(t_new);
  }

  // ---- draws and ordered compaction
  const uint32_t S_hi = uint32_t(S >> 32), S_lo = uint32_t(S);
  const uint32_t R32 = uint32_t(R);
  int32_t* out_idx = a.idx + int64_t(row) * Nkv;
  uint32_t* out_pi = a.pi_q32 + int64_t(row) * Nkv;
  const double inv_s32 = S ? 4294967296.0 / double(S) : 0.0;
  int base = 0;
  if constexpr (kSystematic) {
    const uint64_t U = philox4x32_10(make_uint4(0xFFFFFFFFu, uint32_t(i), uint32_t(h), uint32_t(b)), a.seed_lo,
                                     a.seed_hi).x;
    auto points_below = [&](uint64_t x) -> uint64_t { return x > U ? ((x - U - 1) >> 32) + 1 : 0; };
    uint64_t base_c = 0;  // sum of Pi over the earlier chunks
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (128 * k >= Nkv) break;  // warp-uniform
      const int j0 = 128 * k + 4 * lane;
      const uint4 v4 = wk(k);
      const uint32_t v[4] = {v4.x, v4.y, v4.z, v4.w};
      uint64_t pis[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        pis[q] = j0 + q >= Nkv ? 0ull
                 : v[q] >= theta ? (1ull << 32)
                                 : uint64_t(pi_free(uint64_t(R32) * v[q], S_hi, S_lo, inv_s32));
      const uint64_t mine = (pis[0] + pis[1]) + (pis[2] + pis[3]);
      uint64_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint64_t C = base_c + incl - mine;
      uint32_t keep_mask = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint64_t next = C + pis[q];
        if (j0 + q < Nkv && points_below(next) - points_below(C) == 1) keep_mask |= 1u << q;
        C = next;
      }
      const int kept = __popc(keep_mask);
      int kincl = kept;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, kincl, o);
        if (lane >= o) kincl += y;
      }
      int pos = base + kincl - kept;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (keep_mask & (1u << q)) {
          out_idx[pos] = j0 + q;
          out_pi[pos] = uint32_t(pis[q] & 0xFFFFFFFFull);
          ++pos;
        }
      }
      base += __shfl_sync(0xffffffffu, kincl, 31);
      base_c += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) a.count[row] = base;
  } else {
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (128 * k >= Nkv) break;  // warp-uniform
      const int j0 = 128 * k + 4 * lane;
      uint32_t keep_mask = 0;
      if (j0 < Nkv) {
        const uint4 u4 = philox4x32_10(make_uint4(uint32_t(j0 >> 2), uint32_t(i), uint32_t(h), uint32_t(b)),
                                       a.seed_lo, a.seed_hi);
        const uint32_t us[4] = {u4.x, u4.y, u4.z, u4.w};
        const uint4 v4 = wk(k);
        const uint32_t v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          bool keep;
          if (v[q] >= theta) {
            keep = true;
          } else {
            const uint64_t X = uint64_t(R32) * v[q];
            keep = us[q] == 0u || mul_le_shift32(us[q], S_hi, S_lo, X);
          }
          if (keep && j0 + q < Nkv) keep_mask |= 1u << q;
        }
      }
      const int mine = __popc(keep_mask);
      int incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - mine;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (keep_mask & (1u << q)) out_idx[pos++] = j0 + q;
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();  // out_idx written by the other lanes is read below

    // ---- inclusion probabilities of the kept entries (as in sip_kernel)
    for (int e = lane; e < base; e += 32) {
      const int j = out_idx[e];
      const uint32_t wj = quantise_w(loadP(P + j));
      out_pi[e] = wj < theta ? pi_free(uint64_t(R32) * wj, S_hi, S_lo, inv_s32) : 0u;
    }
    if (lane == 0) a.count[row] = base;
  }
}

// One warp per row for rows of at most 128 KMAX blocks, 8 warps per CTA,
// each with its row in KMAX x 512 bytes of dynamic shared memory.
template <int KMAX, bool kSystematic>
__global__ void __launch_bounds__(256, 3) sip_warp_kernel(const SipArgs a, int rows) {
  extern __shared__ uint4 sip_rows[];  // [8 warps][32 KMAX]
  const int warp = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;  // whole warp: no block-level synchronisation below
  sip_warp_row<KMAX, kSystematic, false>(a, row, sip_rows + warp * 32 * KMAX);
}

// Truncation, the selection SIP is contrasted with (AB-Attention page,
// section "Video Difüzyon Modellerinde Dikkat (Attention) Darboğazı": pruned
// blocks drop out of the softmax; SIP item: SIP estimates dense attention
// rather than truncating it).  One CTA (256 threads) per row keeps the Kb
// blocks with the largest P, ties to the lower j, in ascending order, with
// pi = 1 (pi_q32 = 0).  P >= 0, so the order of the values is the order of
// their bit patterns as unsigned integers: a 4-pass, 8-bit radix select finds
// the Kb-th largest key T and how many keys equal to T are kept; one ordered
// pass then writes every key > T and the first of the keys == T.
__global__ void __launch_bounds__(256) topk_kernel(const SipArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel[2];
  __shared__ uint32_t scan[8];
  const int row = blockIdx.x;
  const float* P = a.P + int64_t(row) * a.Nkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Nkv = a.Nkv;
  uint32_t prefix = 0, pmask = 0, need = uint32_t(a.Kb);  // rank of T among the keys matching prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[tid] = 0;
    __syncthreads();
    for (int j = tid; j < Nkv; j += 256) {
      const uint32_t key = __float_as_uint(__ldg(P + j));
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255 - 8 l - t (t = 0..7), i.e. the bins in descending order
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        c[t] = hist[255 - 8 * lane - t];
        tot += c[t];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t above = incl - tot;  // keys in higher bins
      if (above < need && need <= incl) {  // exactly one lane: T's digit is in its bins
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (above < need && need <= above + c[t]) {
            sel[0] = uint32_t(255 - 8 * lane - t);
            sel[1] = need - above;
          }
          above += c[t];
        }
      }
    }
    __syncthreads();
    prefix |= sel[0] << shift;
    pmask |= 0xFFu << shift;
    need = sel[1];
    __syncthreads();  // hist and sel are rewritten by the next pass
  }
  const uint32_t T = prefix;
  const uint32_t take_eq = need;  // keys equal to T that are kept (the lowest j)

  // ordered pass: 4 consecutive j per thread per 1024-wide chunk
  int32_t* out_idx = a.idx + int64_t(row) * Nkv;
  uint32_t* out_pi = a.pi_q32 + int64_t(row) * Nkv;
  uint32_t base_gt = 0, base_eq = 0;
  for (int c0 = 0; c0 < Nkv; c0 += 1024) {
    const int j0 = c0 + 4 * tid;
    uint32_t gt = 0, eq = 0;  // 4-bit masks
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j0 + q < Nkv) {
        const uint32_t key = __float_as_uint(__ldg(P + j0 + q));
        gt |= (key > T ? 1u : 0u) << q;
        eq |= (key == T ? 1u : 0u) << q;
      }
    }
    // exclusive scan of packed (gt count, eq count), 16 bits each (<= 1024 per chunk)
    const uint32_t mine = uint32_t(__popc(gt)) | (uint32_t(__popc(eq)) << 16);
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) scan[warp] = incl;
    __syncthreads();
    uint32_t woff = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const uint32_t v = scan[w];
      if (w < warp) woff += v;
      total += v;
    }
    const uint32_t excl = woff + incl - mine;
    uint32_t n_gt = base_gt + (excl & 0xFFFFu), n_eq = base_eq + (excl >> 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool is_gt = (gt >> q) & 1u, is_eq = (eq >> q) & 1u;
      if (is_gt || (is_eq && n_eq < take_eq)) {
        const uint32_t pos = n_gt + (n_eq < take_eq ? n_eq : take_eq);
        out_idx[pos] = j0 + q;
        out_pi[pos] = 0u;
      }
      n_gt += is_gt ? 1u : 0u;
      n_eq += is_eq ? 1u : 0u;
    }
    base_gt += total & 0xFFFFu;
    base_eq += total >> 16;
    __syncthreads();  // scan[] is reused by the next chunk
  }
  if (tid == 0) a.count[row] = a.Kb;
}

}  // namespace ab
