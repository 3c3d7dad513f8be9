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
// One CTA computes two query blocks ("streams" 0 and 1, query blocks 2k and
// 2k+1 of one (b, h)), each a 128-row query tile (rows beyond the block are
// computed and discarded).  A stream's list of kept KV blocks is consumed in
// tiles of 128 keys: 128 / KVB list entries per tile, each gathered by TMA
// into consecutive rows of the K and V tiles.  Per tile of stream s:
//   S_s = Q_s K^T        tcgen05 (A, B in shared memory), M=128 N=128 K=d
//   x = S log2(e)/sqrt(d) + log2(1/pi_slot)   (masked keys -> -inf)
//   P_s = exp2(x - m)    bf16, stored back into TMEM over S_s
//   O_s += P_s V         tcgen05 (A = P_s in TMEM, B = V in shared memory)
// Weighting every term of block j by 1/pi_j is the additive bias log2(1/pi_j)
// inside the exponent, so the weights enter the running max and sum for free.
// The reference max m moves only when a row max passes it by more than
// kLazyMax (a factor 2^16: the bf16 weights stay far from overflow, and the
// 1/pi biases, up to 32 in log2, move the max less often than with a tighter
// bound); O_s is then rescaled in TMEM by the softmax warps themselves.
//
// The two streams ping-pong: while the softmax warps of one stream work, the
// tensor core runs the other stream's MMAs.  The MMA warp issues, per tile of
// stream s, O_s += P_s V and then S_s(t+1) = Q_s K(t+1)^T into the same TMEM
// columns; MMAs issued by one thread execute in order, so the next S never
// overwrites P before the P V product has read it, and a commit after S_s(t+1)
// also guarantees that O_s(t) is complete when the softmax reads S_s(t+1).
//
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d),
// O_1 [256+d, 256+2d); P_s (bf16 pairs) occupies the first 64 columns of S_s.
// P is stored in two halves of 64 keys, each announced on its own barrier,
// so that the P V product starts on the first half.
// Warps (384 threads, three warpgroups): 0-3 softmax + epilogue of stream 0,
// 4-7 of stream 1 (warp w owns TMEM lanes 32(w%4)..+31, thread = query row),
// 8 TMA producer of Q and K, 9 MMA issuer and TMEM owner, 10 TMA producer of
// V, 11 idle.  The third warpgroup hands registers to the two softmax
// warpgroups (setmaxnreg): 384 x 168 at launch = 128 x kRegsCtl + 256 x
// kRegsSoftmax.  Tiles of the two streams are interleaved in one order
// ("merged order": 0,1,0,1,... then the longer stream alone) that the
// producers, the MMA warp and the K / V rings share.
#pragma once

#include "ab_ptx.cuh"

namespace ab {

struct AttnArgs {
  int BH, H, L, Lk, Nq, Nkv;  // L queries, Lk keys per (b, h)
  int q_block;  // 64 or 128
  const int32_t* idx;
  const uint32_t* pi_q32;
  const int32_t* count;
  __nv_bfloat16* O;
  float scale_log2;  // log2(e) / sqrt(d)
};

constexpr int kAttnThreads = 384;
constexpr float kLazyMax = 16.f;  // log2 slack of the lazily moved reference max
constexpr int kRegsLaunch = 168;   // registers per thread the kernel is launched with
constexpr int kRegsCtl = 56;       // producer / MMA warpgroup after re-balancing
constexpr int kRegsSoftmax = 224;  // softmax warpgroups after re-balancing
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kAttnThreads * kRegsLaunch, "register split exceeds the launch");

// Stages of the K and V tile rings.
constexpr int kKRing = 3;
constexpr int kVRing = 2;
constexpr int kAttnBars = 13 + 2 * (kKRing + kVRing);  // mbarriers (listed below)

template <int D>
struct AttnSmem {
  static constexpr int kSlabs = D / 64;
  static constexpr int kSlab = 128 * 128;       // one 128-row x 128-byte slab
  static constexpr int kTile = kSlabs * kSlab;  // 128 rows x D bf16
  static constexpr int kKStages = kKRing;
  static constexpr int kVStages = kVRing;
  static constexpr int kOffQ = 0;  // two Q tiles
  static constexpr int kOffK = kOffQ + 2 * kTile;
  static constexpr int kOffV = kOffK + kKStages * kTile;
  static constexpr int kOffMeta = kOffV + kVStages * kTile;  // per K stage: 8 biases, 8 valid counts
  static constexpr int kMetaStride = 64;
  static constexpr int kOffBar = kOffMeta + kKStages * kMetaStride;
  static constexpr int kNumBars = kAttnBars;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "more shared memory than a CTA may have");
};

// barrier indices
enum : int {
  kBarQ = 0,                          // 2 (per stream)
  kBarKFull = 2,                      // kKRing
  kBarKEmpty = kBarKFull + kKRing,    // kKRing (128 arrivals: the softmax warps of the tile's stream)
  kBarVFull = kBarKEmpty + kKRing,    // kVRing
  kBarVEmpty = kBarVFull + kVRing,    // kVRing
  kBarSFull = kBarVEmpty + kVRing,    // 2 (per stream)
  kBarPFull = kBarSFull + 2,          // 2 (per stream, 128 arrivals)
  kBarOFinal = kBarPFull + 2,         // 2 (per stream)
  kBarDrain = kBarOFinal + 2,
  kBarPHalf = kBarDrain + 1,          // 2 (per stream, 128 arrivals): keys [0, 64) of P are in TMEM
  kBarOStaged = kBarPHalf + 2,        // 2 (per stream, one arrival per warp): the output tile is in shared memory
  kBarCount = kBarOStaged + 2,
};
static_assert(kBarCount == kAttnBars, "barrier count");

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

// Merged tile order of two streams with T0 and T1 tiles.
struct Merge {
  int T0, T1, m, longer;
  __host__ __device__ Merge(int a, int b) : T0(a), T1(b), m(a < b ? a : b), longer(a >= b ? 0 : 1) {}
  __host__ __device__ int total() const { return T0 + T1; }
  __host__ __device__ void tile(int g, int& s, int& t) const {
    if (g < 2 * m) {
      s = g & 1;
      t = g >> 1;
    } else {
      s = longer;
      t = g - m;
    }
  }
  __host__ __device__ int index(int s, int t) const { return t < m ? 2 * t + s : m + t; }
};

// D: head dim (64 or 128).  KVB: keys per list slot (16, 32, 64), or 128 for
// dense attention (tile t = keys [128t, 128t+128), no list, no weights).
// kGrouped: K and V are read through a 5-D view {64 columns, 8 rows, d/64
// halves, L/8 row groups, B*H} (needs L % 8 == 0), so that one TMA box
// brings a whole KV block (both 64-column halves) into a K/V tile laid out as
// [row group][half][8 rows][128 B]; otherwise one 3-D box per 64-column half,
// into [half][128 rows][128 B].  Both are 128B-swizzled MMA operands; only the
// strides in the descriptors differ.
template <int D, int KVB, bool kGrouped>
__global__ void __launch_bounds__(kAttnThreads, 1)
    ab_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                        const AttnArgs a) {
  using SM = AttnSmem<D>;
  constexpr bool kDense = (KVB == 128);
  constexpr int kSlots = 128 / KVB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SM::kOffBar;
  auto bar = [&](int k) { return bar0 + 8u * uint32_t(k); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pairs = (a.Nq + 1) / 2;
  const int bh = blockIdx.x / pairs;
  const int qi0 = (blockIdx.x - bh * pairs) * 2;

  // list length and number of 128-key tiles of each stream
  int cnt[2], T[2];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int qi = qi0 + s;
    if (qi >= a.Nq) {
      cnt[s] = 0;
    } else if (kDense) {
      cnt[s] = (a.Lk + 127) / 128;
    } else {
      int c = a.count[int64_t(bh) * a.Nq + qi];
      if (c < 0 || c > a.Nkv) {
        if (threadIdx.x == 0) raise_error(AB_ERR_CAPACITY);
        c = c < 0 ? 0 : a.Nkv;
      }
      cnt[s] = c;
    }
    T[s] = kDense ? cnt[s] : (cnt[s] + kSlots - 1) / kSlots;
  }
  const Merge mg(T[0], T[1]);
  const int G = mg.total();
  // Dense attention with two query blocks: both streams read the same K and V
  // tiles (keys [128t, 128t+128)), so each is loaded once, into K stage t % kKRing
  // and V stage t % 2, for merged tiles 2t and 2t+1; otherwise every merged
  // tile g has stages of its own (g % kKRing, g % kVRing).
  const bool share = kDense && T[0] == T[1];

  if (threadIdx.x == 0) {
    for (int k = 0; k < kVRing; ++k) {
      mbar_init(bar(kBarVFull + k), 1);
      mbar_init(bar(kBarVEmpty + k), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarQ + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), 128);
      mbar_init(bar(kBarPHalf + s), 128);
      mbar_init(bar(kBarOFinal + s), 1);
      mbar_init(bar(kBarOStaged + s), 4);
    }
    for (int k = 0; k < kKRing; ++k) {
      mbar_init(bar(kBarKFull + k), 1);
      mbar_init(bar(kBarKEmpty + k), share ? 256 : 128);  // the softmax warps of every stream that reads it
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    regs_dec<kRegsCtl>();
  if (warp == 8 || warp == 10) {
    // ----------------------------------------------------------- producers
    // Warp 8 loads the Q tiles and the K tiles, warp 10 the V tiles: each
    // walks the merged tile order on its own, so the two TMA streams are
    // issued independently.  Lane e < kSlots owns list slot e of every tile:
    // it reads the list entry and issues the TMA copy of that KV block's rows
    // into rows [e*KVB, (e+1)*KVB) of the tile.  Warp 8's lane 0 publishes the
    // slots' weights and valid-key counts with the K tile.
    const bool is_k = warp == 8;
    constexpr uint32_t kTileBytes = uint32_t(SM::kTile);
    int loads = 0;  // tiles loaded into this ring
    if (is_k && lane == 0) {
      for (int s = 0; s < 2; ++s) {
        if (T[s] == 0) continue;
        mbar_arrive_expect_tx(bar(kBarQ + s), kTileBytes);
        for (int sl = 0; sl < SM::kSlabs; ++sl)
          tma_load_3d(sbase + SM::kOffQ + s * SM::kTile + sl * SM::kSlab, &tmQ, bar(kBarQ + s), sl * 64,
                      (qi0 + s) * a.q_block, bh);
      }
    }
    // List entries are fetched two tiles ahead of their use, so that the
    // latency of the global loads overlaps the waits and copies of the
    // tiles before.
    auto fetch = [&](int u, int& j, uint32_t& pq) {
      j = -1;
      pq = 0;
      if (!kDense && u < G && lane < kSlots) {
        int s, t;
        mg.tile(u, s, t);
        const int e = t * kSlots + lane;
        if (e < cnt[s]) {
          const int64_t at = (int64_t(bh) * a.Nq + qi0 + s) * a.Nkv + e;
          j = __ldg(a.idx + at);
          pq = __ldg(a.pi_q32 + at);
          if (j < 0 || j >= a.Nkv) {
            if (is_k) raise_error(AB_ERR_CAPACITY);
            j = -1;
          }
        }
      }
    };
    int j_cur, j_next, j_far;
    uint32_t pq_cur, pq_next, pq_far;
    fetch(0, j_cur, pq_cur);
    fetch(1, j_next, pq_next);
    const int nstage = is_k ? kKRing : kVRing;
    const uint32_t full0 = bar(is_k ? kBarKFull : kBarVFull), empty0 = bar(is_k ? kBarKEmpty : kBarVEmpty);
    const uint32_t dst0 = sbase + (is_k ? SM::kOffK : SM::kOffV);
    const CUtensorMap* tm = is_k ? &tmK : &tmV;
    bool ok = true;
    for (int u = 0; u < G; ++u) {
      fetch(u + 2, j_far, pq_far);
      int s, t;
      mg.tile(u, s, t);
      if (share && s == 1) continue;  // stream 1 reads the tile stream 0 loaded
      float bias = 0.f;
      int valid = 0, row = 0;  // an empty slot reads any in-range rows (finite data), fully masked
      if (lane < kSlots) {
        if (kDense) {
          row = t * 128;
          valid = min(128, a.Lk - row);
        } else if (j_cur >= 0) {
          row = j_cur * KVB;
          valid = min(KVB, a.Lk - row);
          bias = pq_cur == 0u ? 0.f : 32.f - log2f(float(pq_cur));  // log2(1/pi), Pi = pq or 2^32
        }
      }
      const int si = share ? t : u;  // position in this ring's sequence of loads
      const int st = si % nstage, use = si / nstage;
      const uint32_t full = full0 + 8u * uint32_t(st), empty = empty0 + 8u * uint32_t(st);
      if (!lane0_wait(empty, (use & 1) ^ 1, abort_flag)) { ok = false; break; }
      if (is_k && lane < kSlots) {
        // this slot's weight and valid-key count, published with the K tile
        reinterpret_cast<float*>(smem + SM::kOffMeta + st * SM::kMetaStride)[lane] = bias;
        reinterpret_cast<int*>(smem + SM::kOffMeta + st * SM::kMetaStride + 32)[lane] = valid;
      }
      if (lane == 0) mbar_arrive_expect_tx(full, kTileBytes);
      __syncwarp();
      if (lane < kSlots) {
        const uint32_t dst = dst0 + uint32_t(st * SM::kTile);
        if constexpr (kGrouped) {
          tma_load_5d(dst + lane * KVB * SM::kSlabs * 128, tm, full, 0, 0, 0, row / 8, bh);
        } else {
          for (int sl = 0; sl < SM::kSlabs; ++sl)
            tma_load_3d(dst + sl * SM::kSlab + lane * KVB * 128, tm, full, sl * 64, row, bh);
        }
      }
      ++loads;
      j_cur = j_next;
      pq_cur = pq_next;
      j_next = j_far;
      pq_next = pq_far;
    }
    if (!ok && lane == 0) {
      // let the copies already issued land before shared memory is released
      // (the last load into stage k is the largest i < loads with i % nstage == k)
      for (int k = 0; k < nstage && k < loads; ++k) {
        const int last = loads - 1 - ((loads - 1 - k) % nstage);
        mbar_wait_drain(full0 + 8u * uint32_t(k), (last / nstage) & 1);
      }
      if (is_k)
        for (int s = 0; s < 2; ++s)
          if (T[s] > 0) mbar_wait_drain(bar(kBarQ + s), 0);
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA
    if (G > 0 && lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);  // Q (K-major) x K tile (K-major)
      const uint32_t idO = idesc_bf16_f32(128, D, 0, 1);    // P (TMEM) x V tile (MN-major)
      // descriptor bases, computed once; each MMA only adds its K offset
      constexpr uint32_t kSboK = kGrouped ? uint32_t(SM::kSlabs) * 1024u : 1024u;
      constexpr uint32_t kLboV = kGrouped ? 1024u : uint32_t(SM::kSlab);
      constexpr uint32_t kSboV = kGrouped ? uint32_t(SM::kSlabs) * 1024u : 1024u;
      const SmemDesc qdesc[2] = {smem_desc_base(sbase + SM::kOffQ, 16, 1024),
                                 smem_desc_base(sbase + SM::kOffQ + SM::kTile, 16, 1024)};
      const SmemDesc kdesc0 = smem_desc_base(sbase + SM::kOffK, 16, kSboK);
      const SmemDesc vdesc0 = smem_desc_base(sbase + SM::kOffV, kLboV, kSboV);
      bool ok = true;
      for (int s = 0; s < 2 && ok; ++s)
        if (T[s] > 0) ok = mbar_wait(bar(kBarQ + s), 0, abort_flag);
      auto issue_S = [&](int s, int t) -> bool {
        const int ki = share ? t : mg.index(s, t);
        const int ks = ki % kKRing;
        if (!mbar_wait(bar(kBarKFull + ks), (ki / kKRing) & 1, abort_flag)) return false;
        tc_fence_after();
        // K tile: next 64 columns at kHalfK, 8-row groups kSboK apart
        constexpr uint32_t kHalfK = kGrouped ? 1024u : uint32_t(SM::kSlab);
        const SmemDesc qd = qdesc[s];
        SmemDesc kd = kdesc0;
        kd.lo += uint32_t(ks) * uint32_t(SM::kTile >> 4);
        const uint32_t tSs = tmem + uint32_t(s) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_bf16_ss(tSs, desc_at(qd, (kk >> 2) * SM::kSlab + (kk & 3) * 32),
                      desc_at(kd, (kk >> 2) * kHalfK + (kk & 3) * 32), idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(kBarSFull + s));
        return true;
      };
      // first tile of each stream, in merged order
      for (int g = 0; g < min(G, 2) && ok; ++g) {
        int s, t;
        mg.tile(g, s, t);
        if (t == 0) ok = issue_S(s, 0);
      }
      for (int g = 0; g < G && ok; ++g) {
        int s, t;
        mg.tile(g, s, t);
        // P V in two halves of 64 keys: the first starts as soon as the
        // softmax warps have stored keys [0, 64) of P
        if (!mbar_wait(bar(kBarPHalf + s), t & 1, abort_flag)) { ok = false; break; }
        const int vi = share ? t : g;  // V tile's position in the V ring's loads
        if (!mbar_wait(bar(kBarVFull + vi % kVRing), (vi / kVRing) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tO = tmem + 256u + uint32_t(s * D);
        const uint32_t tP = tmem + uint32_t(s) * 128u;
        // V tile (MN-major): 16 keys per k-step, next 64 columns at kLboV, next 8 keys at kSboV
        constexpr uint32_t kStepV = kGrouped ? 16u * uint32_t(SM::kSlabs) * 128u : 2048u;
        SmemDesc vd = vdesc0;
        vd.lo += uint32_t(vi % kVRing) * uint32_t(SM::kTile >> 4);
        mma_bf16_ts(tO, tP, desc_at(vd, 0), idO, t > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 4; ++kk) mma_bf16_ts(tO, tP + uint32_t(kk * 8), desc_at(vd, kk * kStepV), idO, 1u);
        if (!mbar_wait(bar(kBarPFull + s), t & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 4; kk < 8; ++kk) mma_bf16_ts(tO, tP + uint32_t(kk * 8), desc_at(vd, kk * kStepV), idO, 1u);
        if (!share || s == 1) mma_commit(bar(kBarVEmpty + vi % kVRing));  // shared: after both streams' P V
        if (t + 1 < T[s]) {
          ok = issue_S(s, t + 1);
        } else {
          mma_commit(bar(kBarOFinal + s));
        }
      }
      // every MMA issued above completes before TMEM and shared memory go away
      mma_commit(bar(kBarDrain));
      mbar_wait_drain(bar(kBarDrain), 0);
    }
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------ softmax warps
    const int s = warp >> 2;       // stream
    const int r = threadIdx.x & 127;  // query row within the tile == TMEM lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + uint32_t(s) * 128u + lane_base;
    const uint32_t tO = tmem + 256u + uint32_t(s * D) + lane_base;
    const int qi = qi0 + s;
    float m_use = -INFINITY;  // reference max (log2 domain)
    // Running sum of the weights exp2(x - m_use) as the P V product sees them,
    // i.e. rounded to bfloat16: O / l is then a weighted mean whose weights
    // are exactly the bf16 P.  (With the lazy reference max the largest weight
    // of a row is not 1 and its rounding would otherwise bias O toward 0.)
    float l = 0.f;
    bool ok = true;
    // Keys [64h, 64h + 64) of P are stored: let the MMA warp use them.
    auto publish = [&](int h) {
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar((h == 0 ? kBarPHalf : kBarPFull) + s));
    };
    for (int t = 0; t < T[s] && ok; ++t) {
      // O_s is complete up to tile t-1 when S_s(t) is (the commit behind S_s(t)
      // covers it); a moved reference max rescales it before this tile's P V
      // product accumulates into it.
      auto rescale_O = [&](bool need, float alpha) {
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          // 8 columns at a time: the scores of this tile are live in registers
#pragma unroll 1
          for (int c = 0; c < D / 8; ++c) {
            uint32_t o[8];
            tmem_ld8(tO + uint32_t(c * 8), o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st8(tO + uint32_t(c * 8), o);
          }
        }
      };
      const int ki = share ? t : mg.index(s, t);  // K tile's position in the K ring's loads
      const int ks = ki % kKRing;
      if (!warp_wait(bar(kBarSFull + s), t & 1, abort_flag)) { ok = false; break; }
      if (!warp_wait(bar(kBarKFull + ks), (ki / kKRing) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32_nowait(tS + uint32_t(c * 32), reinterpret_cast<uint32_t*>(x) + c * 32);
      // slot metadata of this tile (published with the K tile), then release the K stage
      const float* mb = reinterpret_cast<const float*>(smem + SM::kOffMeta + ks * SM::kMetaStride);
      const int* mv = reinterpret_cast<const int*>(smem + SM::kOffMeta + ks * SM::kMetaStride + 32);
      float s_bias[kSlots];
      int s_valid[kSlots];
      bool full = true;
#pragma unroll
      for (int e = 0; e < kSlots; ++e) {
        s_bias[e] = mb[e];
        s_valid[e] = mv[e];
        full = full && (s_valid[e] == KVB);
      }
      mbar_arrive(bar(kBarKEmpty + ks));
      tmem_wait_ld();
      float l_lo = 0.f, l_hi = 0.f;  // this tile's sum of the bf16 weights (even, odd columns)
      bool need;
      float alpha = 1.f;
      if (full) {
        // Row max from per-slot maxima of the raw scores (scale > 0 commutes
        // with max), then p = exp2(s * scale + (bias_slot - m)) with one packed
        // FMA per pair of columns.
        float rmax = -INFINITY;
#pragma unroll
        for (int e = 0; e < kSlots; ++e) {
          float mx = x[e * KVB];
#pragma unroll
          for (int k = 1; k + 1 < KVB; k += 2) mx = fmax3(mx, x[e * KVB + k], x[e * KVB + k + 1]);
          mx = fmaxf(mx, x[e * KVB + KVB - 1]);
          rmax = fmaxf(rmax, fmaf(mx, a.scale_log2, s_bias[e]));
        }
        need = rmax > m_use + kLazyMax;
        if (need) {
          alpha = ex2_approx(m_use - rmax);  // 0 on the first tile
          m_use = rmax;
          l *= alpha;
        }
        rescale_O(need, alpha);
        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int c = 64 * h + 2 * k;
            const float off = s_bias[c / KVB] - m_use;
            float p0, p1;
            f2_unpack(f2_fma(f2_pack(x[c], x[c + 1]), sc2, f2_pack(off, off)), p0, p1);
            p0 = ex2_approx(p0);
            p1 = ex2_approx(p1);
            pk[k] = pack_bf16x2(p0, p1);
            add_bf16x2_f32(pk[k], l_lo, l_hi);
          }
          tmem_st32_ptr(tS + uint32_t(32 * h), pk);
          publish(h);
        }
      } else {
        float rmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < 128; ++k) {
          const int e = k / KVB, w = k % KVB;
          x[k] = (w < s_valid[e]) ? fmaf(x[k], a.scale_log2, s_bias[e]) : -INFINITY;
          rmax = fmaxf(rmax, x[k]);
        }
        // lazy reference max: move it only when the row max passes it by > kLazyMax
        need = rmax > m_use + kLazyMax;
        if (need) {
          alpha = ex2_approx(m_use - rmax);  // 0 on the first tile
          m_use = rmax;
          l *= alpha;
        }
        rescale_O(need, alpha);
        const float mref = (m_use == -INFINITY) ? 0.f : m_use;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float p0 = ex2_approx(x[64 * h + 2 * k] - mref);
            const float p1 = ex2_approx(x[64 * h + 2 * k + 1] - mref);
            pk[k] = pack_bf16x2(p0, p1);
            add_bf16x2_f32(pk[k], l_lo, l_hi);
          }
          tmem_st32_ptr(tS + uint32_t(32 * h), pk);
          publish(h);
        }
      }
      l += l_lo + l_hi;
    }
    // ---------------------------------------------------------- epilogue
    // O / l rounded to bf16 is staged in this stream's Q buffer (no MMA reads
    // it any more once O is final) in the 128B-swizzled [half][row][128 B]
    // layout, then written by TMA stores of {64 columns, q_block rows}: whole
    // 128-byte lines, rows past the sequence clipped by the tensor map.  A
    // stream without tiles writes zeros (O = 0 for an empty list).
    if (qi < a.Nq) {
      if (T[s] > 0 && ok) ok = warp_wait(bar(kBarOFinal + s), 0, abort_flag);
      uint8_t* stage = smem + SM::kOffQ + s * SM::kTile;
      if (ok) {
        const float inv = l > 0.f ? 1.f / l : 0.f;  // a row whose keys were all masked gets 0
        if (T[s] > 0) tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (T[s] > 0) {
            tmem_ld32(tO + uint32_t(c * 32), o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0u;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            const int col = c * 32 + q * 8;  // first of the 8 columns
            *reinterpret_cast<uint4*>(stage + (col / 64) * SM::kSlab + sw128_offset(uint32_t(r), uint32_t((col % 64) / 8))) = v;
          }
        }
        fence_proxy_async_smem();  // the TMA store reads what the generic proxy wrote
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarOStaged + s));
      if ((warp & 3) == 0 && lane == 0 && ok && mbar_wait(bar(kBarOStaged + s), 0, abort_flag)) {
        for (int sl = 0; sl < SM::kSlabs; ++sl)
          tma_store_3d(&tmO, smem_u32(stage) + uint32_t(sl * SM::kSlab), sl * 64, qi * a.q_block, bh);
        bulk_commit_group();
        bulk_wait_read_all();  // shared memory stays valid until the stores have read it
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ab
