// Fused 1/pi-weighted block-sparse attention (and its dense special case) for
// sm_100a.
//
// AB-Attention page ("AB-Attention: Video Difüzyon Transformer'larını
// Hızlandırmak İçin Doğru Blok Dikkat Mekanizması"), section "AB-Attention ve
// Üç Temel Yeniliği": the kernel packs KV blocks much smaller than a tile into
// full tensor-core tiles (the "Donanım Dostu Çekirdek" item) and the kept
// blocks are reweighted by their inverse inclusion probability (SIP item).
// The softmax is the online (running max and sum) form of the FlashAttention
// tiling mentioned on the Cross-Attention glossary page ("Sıkça Sorulan
// Sorular").
//
// One CTA computes one query block of one (b, h): a 128-row query tile Q (rows
// beyond the block are computed and discarded).  Its list of kept KV blocks is
// consumed in tiles of 128 keys: 128 / kvb list entries per tile, each gathered
// by TMA into consecutive rows of the K and V tiles.  Per tile:
//   S = Q K^T            tcgen05, M=128 N=128 K=d, fp32 accumulator in TMEM
//   x = S log2(e)/sqrt(d) + log2(1/pi_slot)   (masked keys -> -inf)
//   P = exp2(x - m)      bf16, written to shared memory (128B swizzle)
//   O += P V             tcgen05, M=128 N=d K=128, fp32 accumulator in TMEM
// Weighting every term of block j by 1/pi_j is the additive bias log2(1/pi_j)
// inside the exponent, so the weights enter the running max and sum for free.
// The reference max m is only moved when a row max exceeds it by more than 8
// (factor 256), so O is rescaled in TMEM only on those rare tiles; the final
// O / l is unchanged by the choice of m.
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue (warp w owns TMEM
// lanes 32w..32w+31, thread = query row), warp 4 TMA producer, warp 5 MMA
// issuer and TMEM owner.  K tiles use a 3-deep ring (released when S is done),
// V tiles a 2-deep ring (released when P V is done), S is double-buffered in
// TMEM so that S(t+1) is computed while the softmax of tile t runs.
#pragma once

#include "ab_ptx.cuh"

namespace ab {

struct AttnArgs {
  int BH, H, L, Nq, Nkv;
  int q_block;   // 64 or 128
  const int32_t* idx;
  const uint32_t* pi_q32;
  const int32_t* count;
  __nv_bfloat16* O;
  float scale_log2;  // log2(e) / sqrt(d)
};

template <int D>
struct AttnSmem {
  static constexpr int kSlabs = D / 64;
  static constexpr int kSlab = 128 * 128;            // one 128-row x 128-byte slab
  static constexpr int kTile = kSlabs * kSlab;       // 128 rows x D bf16
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTile;
  static constexpr int kOffV = kOffK + kKStages * kTile;
  static constexpr int kOffP = kOffV + kVStages * kTile;
  static constexpr int kOffMeta = kOffP + 2 * kSlab;  // P: 128 x 128 bf16
  // per V stage: 8 slot biases (log2 1/pi) and 8 valid-key counts
  static constexpr int kMetaBytes = kVStages * 64;
  static constexpr int kOffBar = kOffMeta + kMetaBytes;
  static constexpr int kNumBars = 16;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// barrier indices
enum : int {
  kBarQ = 0,
  kBarKFull = 1,   // 3
  kBarKEmpty = 4,  // 3
  kBarVFull = 7,   // 2
  kBarVEmpty = 9,  // 2
  kBarSFull = 11,  // 2
  kBarPFull = 13,
  kBarODone = 14,
  kBarDrain = 15,
};

// Warp-uniform bounded wait: every lane of the calling warp gets the same answer.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Lane 0 waits, the rest of the warp learns the outcome.
__device__ __forceinline__ bool lane0_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// D: head dim (64 or 128).  KVB: keys per list slot (16, 32, 64), or 128 for
// dense attention (tile t = keys [128t, 128t+128), no list, no weights).
template <int D, int KVB>
__global__ void __launch_bounds__(192, 1)
    ab_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using SM = AttnSmem<D>;
  constexpr bool kDense = (KVB == 128);
  constexpr int kSlots = 128 / KVB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SM::kOffBar;
  auto bar = [&](int k) { return bar0 + 8u * uint32_t(k); };
  float* meta_bias = reinterpret_cast<float*>(smem + SM::kOffMeta);    // [2 stages] x 16, first 8 used
  int* meta_valid = reinterpret_cast<int*>(smem + SM::kOffMeta + 32);  // same stride, offset by 8 words
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.Nq;
  const int qi = blockIdx.x - bh * a.Nq;

  // list length and number of 128-key tiles of this query block
  int cnt;
  if (kDense) {
    cnt = (a.L + 127) / 128;
  } else {
    cnt = a.count[blockIdx.x];
    if (cnt < 0 || cnt > a.Nkv) {
      if (threadIdx.x == 0) raise_error(AB_ERR_CAPACITY);
      cnt = cnt < 0 ? 0 : a.Nkv;
    }
  }
  const int T = kDense ? cnt : (cnt + kSlots - 1) / kSlots;
  const int64_t list_base = int64_t(blockIdx.x) * a.Nkv;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
    }
    mbar_init(bar(kBarPFull), 128);
    mbar_init(bar(kBarODone), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // Lane s < kSlots owns list slot s of every tile: it reads the list entry,
    // issues the TMA copies of that KV block's rows into the K (and one step
    // later the V) tile, and hands the slot's weight and valid-key count to
    // lane 0, which publishes them with the V tile.
    constexpr uint32_t kTileBytes = uint32_t(SM::kTile);
    int issued_k[3] = {0, 0, 0}, issued_v[2] = {0, 0};
    if (T > 0 && lane == 0) {
      mbar_arrive_expect_tx(bar(kBarQ), kTileBytes);
      for (int s = 0; s < SM::kSlabs; ++s)
        tma_load_3d(sbase + SM::kOffQ + s * SM::kSlab, &tmQ, bar(kBarQ), s * 64, qi * a.q_block, bh);
    }
    int prev_row = 0, row = 0, prev_valid = 0, valid = 0;
    float prev_bias = 0.f, bias = 0.f;
    bool ok = true;
    for (int u = 0; u <= T && ok; ++u) {
      if (u < T) {
        if (lane < kSlots) {
          if (kDense) {
            row = u * 128;
            valid = min(128, a.L - row);
            bias = 0.f;
          } else {
            const int e = u * kSlots + lane;
            int j = -1;
            uint32_t pq = 0;
            if (e < cnt) {
              j = a.idx[list_base + e];
              pq = a.pi_q32[list_base + e];
              if (j < 0 || j >= a.Nkv) {
                raise_error(AB_ERR_CAPACITY);
                j = -1;
              }
            }
            if (j >= 0) {
              row = j * KVB;
              valid = min(KVB, a.L - row);
              bias = pq == 0u ? 0.f : 32.f - log2f(float(pq));  // log2(1/pi), Pi = pq or 2^32
            } else {
              row = 0;  // empty slot: any in-range rows (finite data), fully masked
              valid = 0;
              bias = 0.f;
            }
          }
        }
        const int ks = u % 3;
        if (!lane0_wait(bar(kBarKEmpty + ks), ((u / 3) & 1) ^ 1, abort_flag)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(bar(kBarKFull + ks), kTileBytes);
        __syncwarp();
        if (lane < kSlots) {
          for (int s = 0; s < SM::kSlabs; ++s)
            tma_load_3d(sbase + SM::kOffK + ks * SM::kTile + s * SM::kSlab + lane * KVB * 128, &tmK,
                        bar(kBarKFull + ks), s * 64, row, bh);
        }
        issued_k[ks] += 1;
      }
      if (u >= 1) {
        const int t = u - 1;
        const int vs = t & 1;
        if (!lane0_wait(bar(kBarVEmpty + vs), ((t >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        float b_all[kSlots];
        int v_all[kSlots];
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
          b_all[s] = __shfl_sync(0xffffffffu, prev_bias, s);
          v_all[s] = __shfl_sync(0xffffffffu, prev_valid, s);
        }
        if (lane == 0) {
#pragma unroll
          for (int s = 0; s < kSlots; ++s) {
            meta_bias[vs * 16 + s] = b_all[s];
            meta_valid[vs * 16 + s] = v_all[s];
          }
          mbar_arrive_expect_tx(bar(kBarVFull + vs), kTileBytes);
        }
        __syncwarp();
        if (lane < kSlots) {
          for (int s = 0; s < SM::kSlabs; ++s)
            tma_load_3d(sbase + SM::kOffV + vs * SM::kTile + s * SM::kSlab + lane * KVB * 128, &tmV,
                        bar(kBarVFull + vs), s * 64, prev_row, bh);
        }
        issued_v[vs] += 1;
      }
      prev_row = row;
      prev_bias = bias;
      prev_valid = valid;
    }
    if (!ok && lane == 0) {
      // let the copies already issued land before shared memory is released
      for (int s = 0; s < 3; ++s)
        if (issued_k[s]) mbar_wait_drain(bar(kBarKFull + s), (issued_k[s] - 1) & 1);
      for (int s = 0; s < 2; ++s)
        if (issued_v[s]) mbar_wait_drain(bar(kBarVFull + s), (issued_v[s] - 1) & 1);
      if (T > 0) mbar_wait_drain(bar(kBarQ), 0);
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA
    if (T > 0 && lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);  // Q (K-major) x K tile (K-major)
      const uint32_t idO = idesc_bf16_f32(128, D, 0, 1);    // P (K-major) x V tile (MN-major)
      const uint32_t tO = tmem + 256u;
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag);
      auto issue_S = [&](int t) -> bool {
        const int ks = t % 3;
        if (!mbar_wait(bar(kBarKFull + ks), (t / 3) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t qa = sbase + SM::kOffQ;
        const uint32_t kb = sbase + SM::kOffK + ks * SM::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * SM::kSlab + (kk & 3) * 32;
          mma_bf16_ss(tmem + uint32_t(t & 1) * 128u, smem_desc_sw128(qa + off, 16, 1024),
                      smem_desc_sw128(kb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBarSFull + (t & 1)));
        mma_commit(bar(kBarKEmpty + ks));
        return true;
      };
      if (ok) ok = issue_S(0);
      if (ok && T > 1) ok = issue_S(1);
      for (int t = 0; t < T && ok; ++t) {
        if (!mbar_wait(bar(kBarPFull), t & 1, abort_flag)) { ok = false; break; }
        if (!mbar_wait(bar(kBarVFull + (t & 1)), (t >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pa = sbase + SM::kOffP;
        const uint32_t vb = sbase + SM::kOffV + (t & 1) * SM::kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * SM::kSlab + (kk & 3) * 32;
          mma_bf16_ss(tO, smem_desc_sw128(pa + aoff, 16, 1024), smem_desc_sw128(vb + kk * 2048, SM::kSlab, 1024),
                      idO, (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(kBarODone));
        mma_commit(bar(kBarVEmpty + (t & 1)));
        if (t + 2 < T) ok = issue_S(t + 2);
      }
      // every MMA issued above completes before TMEM and shared memory go away
      mma_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0);
    }
  } else {
    // ------------------------------------------------------ softmax warps
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + 256u + lane_base;
    float m_use = -INFINITY;  // reference max (log2 domain)
    float l = 0.f;            // running sum of exp2(x - m_use)
    bool ok = true;
    uint8_t* pbase = smem + SM::kOffP;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1;
      if (!warp_wait(bar(kBarSFull + sb), (t >> 1) & 1, abort_flag)) { ok = false; break; }
      if (!warp_wait(bar(kBarVFull + sb), (t >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + uint32_t(sb * 128 + c * 32) + lane_base, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) x[c * 32 + k] = __uint_as_float(v[k]);
      }
      float s_bias[kSlots];
      int s_valid[kSlots];
#pragma unroll
      for (int s = 0; s < kSlots; ++s) {
        s_bias[s] = meta_bias[sb * 16 + s];
        s_valid[s] = meta_valid[sb * 16 + s];
      }
      float rmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < 128; ++k) {
        constexpr int kb = KVB;
        const int s = k / kb;
        const int w = k % kb;
        const float xv = (w < s_valid[s]) ? fmaf(x[k], a.scale_log2, s_bias[s]) : -INFINITY;
        x[k] = xv;
        rmax = fmaxf(rmax, xv);
      }
      // lazy reference max: move it only when the row max passes it by > 8
      const bool need = rmax > m_use + 8.f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_use - rmax);  // 0 on the first tile
        m_use = rmax;
        l *= alpha;
      }
      const float mref = (m_use == -INFINITY) ? 0.f : m_use;
      if (t > 0) {
        // P V of the previous tile is done: P smem is free and O is stable
        if (!warp_wait(bar(kBarODone), (t - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + uint32_t(c * 32), v);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
            tmem_st32(tO + uint32_t(c * 32), v);
          }
          tmem_wait_st();
        }
      }
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float p0 = ex2_approx(x[c * 8 + 2 * h] - mref);
          const float p1 = ex2_approx(x[c * 8 + 2 * h + 1] - mref);
          lsum += p0 + p1;
          pk[h] = pack_bf16x2(p0, p1);
        }
        const uint32_t off = uint32_t(c >> 3) * SM::kSlab + sw128_offset(uint32_t(r), uint32_t(c & 7));
        *reinterpret_cast<uint4*>(pbase + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull));
    }
    // ---------------------------------------------------------- epilogue
    const int n_i = min(a.q_block, a.L - qi * a.q_block);
    __nv_bfloat16* orow = a.O + (int64_t(bh) * a.L + int64_t(qi) * a.q_block + r) * D;
    if (T > 0 && ok) ok = warp_wait(bar(kBarODone), (T - 1) & 1, abort_flag);
    if (T > 0 && ok) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + uint32_t(c * 32), v);
        tmem_wait_ld();
        if (r < n_i) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv);
            o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv);
            o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv);
            o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = o;
          }
        }
      }
    } else if (T == 0 && r < n_i) {
      for (int c = 0; c < D / 8; ++c) *reinterpret_cast<uint4*>(orow + c * 8) = make_uint4(0, 0, 0, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ab
