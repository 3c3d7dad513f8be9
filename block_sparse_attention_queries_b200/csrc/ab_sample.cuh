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
// Kept blocks are compacted in ascending j with a block-wide scan; each thread
// owns 4 consecutive j per 1024-wide chunk (one Philox call per thread).  The
// quantised row W is read from global memory once and kept in shared memory
// (rows up to kSipSmemCap entries; longer rows re-read P instead).
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
};

__device__ __forceinline__ uint64_t quantise_w(float p) {
  const float s = floorf(p * 16777216.0f);
  return s < 1.0f ? 1ull : uint64_t(s);
}

// Block-wide sum of (count, sum) pairs over 256 threads.
__device__ __forceinline__ void block_sum2(uint64_t& a, uint64_t& b, uint64_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  __syncthreads();
  if (lane == 0) {
    red[warp] = a;
    red[8 + warp] = b;
  }
  __syncthreads();
  a = 0;
  b = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    a += red[w];
    b += red[8 + w];
  }
}

constexpr int kSipSmemCap = 16384;  // entries of W cached in shared memory (64 KB)

__global__ void __launch_bounds__(256) sip_kernel(const SipArgs a) {
  __shared__ uint64_t red[16];
  __shared__ int scan[8];
  extern __shared__ uint32_t wcache[];  // [Nkv] when Nkv <= kSipSmemCap
  const int row = blockIdx.x;
  const int b = row / (a.H * a.Nq);
  const int h = (row / a.Nq) % a.H;
  const int i = row % a.Nq;
  const float* P = a.P + int64_t(row) * a.Nkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Nkv = a.Nkv;
  const bool cached = Nkv <= kSipSmemCap;
  if (cached) {
    for (int j = tid; j < Nkv; j += 256) wcache[j] = uint32_t(quantise_w(__ldg(P + j)));
    __syncthreads();
  }
  auto W = [&](int j) -> uint64_t { return cached ? uint64_t(wcache[j]) : quantise_w(__ldg(P + j)); };

  // ---- capping threshold (fixed point; at most Nkv + 1 rounds)
  uint64_t theta = ~0ull;  // nothing capped
  uint64_t R = 0, S = 0;
  for (int round = 0; round <= Nkv + 1; ++round) {
    uint64_t ncap = 0, sum = 0;
    for (int j = tid; j < Nkv; j += 256) {
      const uint64_t w = W(j);
      if (w >= theta) ncap += 1;
      else sum += w;
    }
    block_sum2(ncap, sum, red);
    R = uint64_t(a.Kb) - ncap;
    S = sum;
    if (R == 0 || S == 0) break;
    const uint64_t t_new = (S + R - 1) / R;  // R W >= S  <=>  W >= ceil(S / R)
    if (t_new >= theta) break;
    theta = t_new;
  }

  // ---- draws and ordered compaction, 4 consecutive j per thread per chunk
  const uint32_t k0 = a.seed_lo, k1 = a.seed_hi;
  int32_t* out_idx = a.idx + int64_t(row) * Nkv;
  uint32_t* out_pi = a.pi_q32 + int64_t(row) * Nkv;
  int base = 0;
  for (int c0 = 0; c0 < Nkv; c0 += 1024) {
    const int j0 = c0 + 4 * tid;
    uint32_t keep_mask = 0;
    uint32_t pis[4] = {0, 0, 0, 0};
    if (j0 < Nkv) {
      const uint4 u4 = philox4x32_10(make_uint4(uint32_t(j0 >> 2), uint32_t(i), uint32_t(h), uint32_t(b)), k0, k1);
      const uint32_t us[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = j0 + q;
        if (j >= Nkv) break;
        const uint64_t w = W(j);
        bool keep;
        uint32_t pq;
        if (w >= theta) {
          keep = true;  // capped: pi = 1
          pq = 0;
        } else {
          const unsigned __int128 X = (unsigned __int128)(R * w) << 32;
          const unsigned __int128 lhs = (unsigned __int128)(uint64_t(us[q]) + 1ull) * S;
          keep = (us[q] == 0u) || (lhs <= X);
          pq = 0;
          if (keep) {
            // Pi = max(1, floor(X / S)) < 2^32: double estimate, exact integer fix-up
            uint64_t est = uint64_t(double(R * w) * 4294967296.0 / double(S));
            while ((unsigned __int128)est * S > X) --est;
            while ((unsigned __int128)(est + 1) * S <= X) ++est;
            pq = est < 1 ? 1u : uint32_t(est);
          }
        }
        if (keep) keep_mask |= 1u << q;
        pis[q] = pq;
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
      if (keep_mask & (1u << q)) {
        out_idx[pos] = j0 + q;
        out_pi[pos] = pis[q];
        ++pos;
      }
    }
    base += total;
    __syncthreads();  // scan[] is reused by the next chunk
  }
  if (tid == 0) a.count[row] = base;
}

}  // namespace ab
