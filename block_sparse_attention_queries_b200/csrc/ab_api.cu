// C ABI of the AB-Attention hot path (declared in include/ab.h): argument
// checks, workspace layout, TMA descriptors and kernel launches.  The library
// allocates no memory; every buffer belongs to the caller.
#include <cmath>
#include <vector>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "ab_attention.cuh"
#include "ab_sample.cuh"
#include "ab_select.cuh"

namespace {

using namespace ab;

struct Dims {
  int B, H, L, Lk, d, q_block, kv_block, C, iters;  // L queries, Lk keys per (b, h)
  int BH, Nq, Nkv, Kb;
  float keep;
  uint64_t seed;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NVTX range around one entry point (host side: argument checks and launches);
// free unless a profiler is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

int budget_of(int Nkv, double keep) {
  double kb = std::floor(keep * double(Nkv) + 0.5);
  if (kb < 1.0) kb = 1.0;
  if (kb > double(Nkv)) kb = double(Nkv);
  return int(kb);
}

// Host-side validation shared by every entry point.  `need_method` also checks
// the fields only the sparse path uses.
ab_status check_params(const ab_params* p, bool need_method, Dims* out) {
  if (!p) return AB_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->L < 1 || p->L > (1 << 24)) return AB_ERR_INVALID_ARG;
  if (p->L_kv < 0 || p->L_kv > (1 << 24)) return AB_ERR_INVALID_ARG;
  if (int64_t(p->B) * p->H > (int64_t(1) << 20)) return AB_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return p->d > 0 ? AB_ERR_UNSUPPORTED : AB_ERR_INVALID_ARG;
  if (p->q_block != 64 && p->q_block != 128) return p->q_block > 0 ? AB_ERR_UNSUPPORTED : AB_ERR_INVALID_ARG;
  if (need_method) {
    if (p->kv_block != 16 && p->kv_block != 32 && p->kv_block != 64)
      return p->kv_block > 0 ? AB_ERR_UNSUPPORTED : AB_ERR_INVALID_ARG;
    if (p->C != 1 && p->C != 2 && p->C != 4 && p->C != 8 && p->C != 16)
      return (p->C >= 1 && p->C <= 16) ? AB_ERR_UNSUPPORTED : AB_ERR_INVALID_ARG;
    if (p->kmeans_iters < 1 || p->kmeans_iters > 16) return AB_ERR_INVALID_ARG;
    if (!(p->keep_ratio > 0.f) || !(p->keep_ratio <= 1.f)) return AB_ERR_INVALID_ARG;
  }
  Dims d{};
  d.B = p->B; d.H = p->H; d.L = p->L; d.Lk = p->L_kv > 0 ? p->L_kv : p->L; d.d = p->d; d.q_block = p->q_block;
  d.kv_block = need_method ? p->kv_block : 16;
  d.C = p->C; d.iters = p->kmeans_iters; d.keep = p->keep_ratio; d.seed = p->seed;
  d.BH = p->B * p->H;
  d.Nq = (p->L + d.q_block - 1) / d.q_block;
  d.Nkv = (d.Lk + d.kv_block - 1) / d.kv_block;
  d.Kb = need_method ? budget_of(d.Nkv, double(p->keep_ratio)) : 0;
  if (int64_t(d.BH) * d.Nq > 0x7fffffff || int64_t(d.BH) * d.Nq * d.Nkv > (int64_t(1) << 40))
    return AB_ERR_INVALID_ARG;
  *out = d;
  return AB_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Workspace {
  size_t off_ksum, off_cent, off_cnt, total;
};

Workspace workspace_layout(const Dims& d) {
  Workspace w{};
  w.off_ksum = 0;
  w.off_cent = align256(w.off_ksum + size_t(d.BH) * d.Nkv * d.d * 2);
  w.off_cnt = align256(w.off_cent + size_t(d.BH) * d.Nq * d.C * d.d * 2);
  w.total = align256(w.off_cnt + size_t(d.BH) * d.Nq * d.C * 4);
  return w;
}

// ---------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor viewed as {inner, rows, outer}, 128B swizzle, box {64, box_rows, 1};
// reads outside the tensor return zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, rows, outer};
  const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// K or V ([B*H, L, d] bf16, L % 8 == 0) viewed as {64, 8 rows, d/64 halves,
// L/8 row groups, B*H}: one box of {64, 8, d/64, box_groups, 1} holds
// 8*box_groups whole rows, laid out [group][half][row][128 B].
bool make_map_grouped(CUtensorMap* m, const void* base, uint64_t d, uint64_t L, uint64_t BH, uint32_t box_groups) {
  auto fn = encode_fn();
  if (!fn || L % 8 != 0) return false;
  const cuuint64_t dims[5] = {64, 8, d / 64, L / 8, BH};
  const cuuint64_t strides[4] = {d * 2, 128, 8 * d * 2, L * d * 2};
  const cuuint32_t box[5] = {64, 8, uint32_t(d / 64), box_groups, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

ab_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? AB_OK : AB_ERR_CUDA;
}

// ---------------------------------------------------------------- launches
PFN_cuCtxGetCurrent_v4000 ctx_current_fn();

// The selector's second stream, one per CUDA context, created on first use
// and kept (like the host pipeline's copy streams): the K-block summaries,
// which only read K, run on it beside the k-means launch, which only reads
// Q; the scoring launch waits for both.  A call holds the lock from the fork
// to the join so that calls from several host threads take turns.
struct SideStream {
  CUcontext ctx = nullptr;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;
};
std::mutex g_side_mutex;
std::vector<SideStream*> g_sides;  // never freed

SideStream* side_stream_current_context() {
  auto get_ctx = ctx_current_fn();
  if (!get_ctx) return nullptr;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  std::lock_guard<std::mutex> lock(g_side_mutex);
  for (SideStream* x : g_sides)
    if (x->ctx == ctx) return x;
  SideStream* x = new SideStream;
  x->ctx = ctx;
  if (cudaStreamCreateWithFlags(&x->s, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&x->fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&x->join, cudaEventDisableTiming) != cudaSuccess) {
    if (x->fork) cudaEventDestroy(x->fork);
    if (x->s) cudaStreamDestroy(x->s);
    delete x;
    return nullptr;
  }
  g_sides.push_back(x);
  return x;
}

// sip != nullptr: the scoring kernel also runs SIP on its rows (rows of at
// most kFusedSampleMaxNkv blocks).  overlap: the K-block summaries run on the
// context's second stream beside k-means (false: everything on `st`).
template <int D>
ab_status run_select(const Dims& d, const void* Q, const void* K, float* P, float* cent, int32_t* counts,
                     uint8_t* ws, cudaStream_t st, const SipArgs* sip = nullptr, bool overlap = true) {
  const Workspace w = workspace_layout(d);
  auto* ksum = reinterpret_cast<__nv_bfloat16*>(ws + w.off_ksum);
  auto* cent_ws = reinterpret_cast<__nv_bfloat16*>(ws + w.off_cent);
  auto* cnt_ws = reinterpret_cast<int32_t*>(ws + w.off_cnt);

  // K-block summaries, on the second stream when there is one
  SideStream* side = overlap ? side_stream_current_context() : nullptr;
  std::unique_lock<std::mutex> side_lock;
  if (side) {
    side_lock = std::unique_lock<std::mutex>(side->mu);
    if (cudaEventRecord(side->fork, st) != cudaSuccess || cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
      return AB_ERR_CUDA;
  }
  {
    const int64_t warps = int64_t(d.BH) * d.Nkv;
    ksum_kernel<D><<<unsigned((warps + 7) / 8), 256, 0, side ? side->s : st>>>(
        reinterpret_cast<const __nv_bfloat16*>(K), ksum, d.BH, d.Lk, d.Nkv, d.kv_block);
    if (launch_status() != AB_OK) return AB_ERR_CUDA;
    if (side && cudaEventRecord(side->join, side->s) != cudaSuccess) return AB_ERR_CUDA;
  }
  // k-means per query block
  {
    CUtensorMap tmQ;
    if (!make_map(&tmQ, Q, D, d.L, d.BH, 128)) return AB_ERR_CUDA;
    const int smem = KmSmem<D>::kAlloc;
    auto launch = [&](auto kern) -> ab_status {
      if (set_smem(kern, smem) != cudaSuccess) return AB_ERR_CUDA;
      kern<<<unsigned(d.BH * d.Nq), 128, smem, st>>>(tmQ, d.L, d.Nq, d.q_block, d.iters, cent, counts, cent_ws,
                                                     cnt_ws);
      return launch_status();
    };
    ab_status s;
    switch (d.C) {
      case 1: s = launch(kmeans_kernel<D, 1>); break;
      case 2: s = launch(kmeans_kernel<D, 2>); break;
      case 4: s = launch(kmeans_kernel<D, 4>); break;
      case 8: s = launch(kmeans_kernel<D, 8>); break;
      default: s = launch(kmeans_kernel<D, 16>); break;
    }
    if (s != AB_OK) return s;
  }
  if (side && cudaStreamWaitEvent(st, side->join, 0) != cudaSuccess) return AB_ERR_CUDA;
  // scores and block mass
  {
    CUtensorMap tmCent, tmKsum;
    if (!make_map(&tmCent, cent_ws, D, uint64_t(d.BH) * d.Nq * d.C, 1, 128)) return AB_ERR_CUDA;
    if (!make_map(&tmKsum, ksum, D, d.Nkv, d.BH, 128)) return AB_ERR_CUDA;
    ScoreArgs a{};
    a.L = d.L; a.Nq = d.Nq; a.Nkv = d.Nkv; a.q_block = d.q_block; a.kv_block = d.kv_block;
    a.counts_ws = cnt_ws;
    a.P = P;
    a.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
    const int n_last = d.Lk - (d.Nkv - 1) * d.kv_block;
    a.last_bias = float(std::log2(double(n_last) / double(d.kv_block)));
    if (sip) a.sip = *sip;
    const int G = 128 / d.C;
    const unsigned grid = unsigned(d.BH * ((d.Nq + G - 1) / G));
    const int smem = sip ? ScSmem<D, true>::kAlloc : ScSmem<D>::kAlloc;
    auto launch = [&](auto kern) -> ab_status {
      if (set_smem(kern, smem) != cudaSuccess) return AB_ERR_CUDA;
      kern<<<grid, 288, smem, st>>>(tmCent, tmKsum, a);
      return launch_status();
    };
    if (sip) {
      switch (d.C) {
        case 1: return launch(score_kernel<D, 1, true>);
        case 2: return launch(score_kernel<D, 2, true>);
        case 4: return launch(score_kernel<D, 4, true>);
        case 8: return launch(score_kernel<D, 8, true>);
        default: return launch(score_kernel<D, 16, true>);
      }
    }
    switch (d.C) {
      case 1: return launch(score_kernel<D, 1>);
      case 2: return launch(score_kernel<D, 2>);
      case 4: return launch(score_kernel<D, 4>);
      case 8: return launch(score_kernel<D, 8>);
      default: return launch(score_kernel<D, 16>);
    }
  }
}

template <int D>
ab_status run_attention(const Dims& d, const void* Q, const void* K, const void* V, const int32_t* idx,
                        const uint32_t* pi_q32, const int32_t* count, void* O, bool dense, cudaStream_t st) {
  const int kvb = dense ? 128 : d.kv_block;
  const bool grouped = (d.Lk % 8) == 0;
  CUtensorMap tmQ, tmK, tmV, tmO;
  if (!make_map(&tmQ, Q, D, d.L, d.BH, 128)) return AB_ERR_CUDA;
  // output tiles are stored q_block rows at a time (a 128-row tile holds two
  // query blocks when q_block is 64)
  if (!make_map(&tmO, O, D, d.L, d.BH, uint32_t(d.q_block))) return AB_ERR_CUDA;
  if (grouped) {
    if (!make_map_grouped(&tmK, K, D, d.Lk, d.BH, uint32_t(kvb / 8))) return AB_ERR_CUDA;
    if (!make_map_grouped(&tmV, V, D, d.Lk, d.BH, uint32_t(kvb / 8))) return AB_ERR_CUDA;
  } else {
    if (!make_map(&tmK, K, D, d.Lk, d.BH, uint32_t(kvb))) return AB_ERR_CUDA;
    if (!make_map(&tmV, V, D, d.Lk, d.BH, uint32_t(kvb))) return AB_ERR_CUDA;
  }
  AttnArgs a{};
  a.BH = d.BH; a.H = d.H; a.L = d.L; a.Lk = d.Lk; a.Nq = d.Nq; a.Nkv = dense ? (d.Lk + 127) / 128 : d.Nkv;
  a.q_block = d.q_block;
  a.idx = idx; a.pi_q32 = pi_q32; a.count = count;
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.scale_log2 = float(1.4426950408889634 / std::sqrt(double(D)));
  const int smem = AttnSmem<D>::kAlloc;
  auto launch = [&](auto kern) -> ab_status {
    if (set_smem(kern, smem) != cudaSuccess) return AB_ERR_CUDA;
    // The kernel re-balances registers between its warpgroups; that only
    // works if it is launched with the register count the split assumes.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return AB_ERR_CUDA;
    if (fa.numRegs < kRegsLaunch) return AB_ERR_UNSUPPORTED;
    // one CTA per pair of query blocks (2k, 2k+1) of a (b, h)
    kern<<<unsigned(d.BH * ((d.Nq + 1) / 2)), kAttnThreads, smem, st>>>(tmQ, tmK, tmV, tmO, a);
    return launch_status();
  };
  if (grouped) {
    switch (kvb) {
      case 16: return launch(ab_attention_kernel<D, 16, true>);
      case 32: return launch(ab_attention_kernel<D, 32, true>);
      case 64: return launch(ab_attention_kernel<D, 64, true>);
      default: return launch(ab_attention_kernel<D, 128, true>);
    }
  }
  switch (kvb) {
    case 16: return launch(ab_attention_kernel<D, 16, false>);
    case 32: return launch(ab_attention_kernel<D, 32, false>);
    case 64: return launch(ab_attention_kernel<D, 64, false>);
    default: return launch(ab_attention_kernel<D, 128, false>);
  }
}

ab_status do_select(const Dims& d, const void* Q, const void* K, float* P, float* cent, int32_t* counts, void* ws,
                    size_t ws_bytes, cudaStream_t st, bool overlap = true) {
  if (!Q || !K || !P || !ws) return AB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(P) || !aligned16(ws)) return AB_ERR_INVALID_ARG;
  if ((cent && !aligned16(cent)) || (counts && !aligned16(counts))) return AB_ERR_INVALID_ARG;
  if (ws_bytes < workspace_layout(d).total) return AB_ERR_WORKSPACE;
  auto* w = reinterpret_cast<uint8_t*>(ws);
  return d.d == 128 ? run_select<128>(d, Q, K, P, cent, counts, w, st, nullptr, overlap)
                    : run_select<64>(d, Q, K, P, cent, counts, w, st, nullptr, overlap);
}

// One warp per row (the row's quantised weights in shared memory), for rows
// of at most 2048 blocks: the smallest chunk count that holds the row.
template <bool kSystematic>
ab_status launch_sip_warp(const SipArgs& a, int rows, int Nkv, cudaStream_t st) {
  auto go = [&](auto kmax) -> ab_status {
    constexpr int KMAX = decltype(kmax)::value;
    constexpr int smem = 8 * 32 * KMAX * 16;
    if (smem > 48 * 1024 && set_smem(sip_warp_kernel<KMAX, kSystematic>, smem) != cudaSuccess)
      return AB_ERR_CUDA;
    sip_warp_kernel<KMAX, kSystematic><<<unsigned((rows + 7) / 8), 256, smem, st>>>(a, rows);
    return launch_status();
  };
  if (Nkv <= 512) return go(std::integral_constant<int, 4>{});
  if (Nkv <= 1024) return go(std::integral_constant<int, 8>{});
  return go(std::integral_constant<int, 16>{});
}

// rows: the rows of this call (d.BH * d.Nq unless a caller processes a range of
// heads); H and row0 place them in the full problem for the draws' counters.
ab_status do_sample(const Dims& d, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count, cudaStream_t st,
                    int H = -1, int64_t row0 = 0) {
  if (!P || !idx || !pi_q32 || !count) return AB_ERR_INVALID_ARG;
  if (!aligned16(P) || !aligned16(idx) || !aligned16(pi_q32) || !aligned16(count)) return AB_ERR_INVALID_ARG;
  SipArgs a{};
  a.P = P; a.idx = idx; a.pi_q32 = pi_q32; a.count = count;
  a.H = H > 0 ? H : d.H; a.Nq = d.Nq; a.Nkv = d.Nkv; a.Kb = d.Kb;
  a.seed_lo = uint32_t(d.seed); a.seed_hi = uint32_t(d.seed >> 32);
  a.row0 = row0;
  const int rows = d.BH * d.Nq;
  if (d.Nkv <= 2048) {  // one warp per row
    return launch_sip_warp<false>(a, rows, d.Nkv, st);
  } else if (d.Nkv <= kSipSmemCap) {
    const int smem = 16 * ((d.Nkv + 3) / 4);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(sip_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return AB_ERR_CUDA;
    sip_kernel<true, false><<<unsigned(d.BH * d.Nq), kSipThreads, smem, st>>>(a);
  } else {
    sip_kernel<false, false><<<unsigned(d.BH * d.Nq), kSipThreads, 0, st>>>(a);
  }
  return launch_status();
}

constexpr int kFusedSampleMaxNkv = 2048;  // rows the scoring kernel's warps sample (8 KB of shared memory each)

// ab_select then ab_sample; for rows of at most kFusedSampleMaxNkv blocks in
// one launch less (the scoring kernel samples the rows it has just scored).
// H and row0 as for do_sample.
ab_status do_select_sample(const Dims& d, const void* Q, const void* K, float* P, int32_t* idx, uint32_t* pi_q32,
                           int32_t* count, void* ws, size_t ws_bytes, cudaStream_t st, int H = -1,
                           int64_t row0 = 0) {
  // every argument is checked before anything is enqueued, on both paths
  if (!Q || !K || !P || !ws || !idx || !pi_q32 || !count) return AB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(P) || !aligned16(ws)) return AB_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(pi_q32) || !aligned16(count)) return AB_ERR_INVALID_ARG;
  if (ws_bytes < workspace_layout(d).total) return AB_ERR_WORKSPACE;
  if (d.Nkv > kFusedSampleMaxNkv) {
    const ab_status s = do_select(d, Q, K, P, nullptr, nullptr, ws, ws_bytes, st);
    return s != AB_OK ? s : do_sample(d, P, idx, pi_q32, count, st, H, row0);
  }
  SipArgs a{};
  a.P = P; a.idx = idx; a.pi_q32 = pi_q32; a.count = count;
  a.H = H > 0 ? H : d.H; a.Nq = d.Nq; a.Nkv = d.Nkv; a.Kb = d.Kb;
  a.seed_lo = uint32_t(d.seed); a.seed_hi = uint32_t(d.seed >> 32);
  a.row0 = row0;
  auto* w = reinterpret_cast<uint8_t*>(ws);
  return d.d == 128 ? run_select<128>(d, Q, K, P, nullptr, nullptr, w, st, &a)
                    : run_select<64>(d, Q, K, P, nullptr, nullptr, w, st, &a);
}

// Every device argument of a whole-path call (select, sample, attention),
// checked before anything is enqueued: non-null, 16-byte aligned, and a
// workspace of at least ws_need bytes.
ab_status check_path_args(const void* Q, const void* K, const void* V, const float* P, const int32_t* idx,
                          const uint32_t* pi_q32, const int32_t* count, const void* O, const void* ws,
                          size_t ws_bytes, size_t ws_need) {
  const void* ptrs[] = {Q, K, V, P, idx, pi_q32, count, O, ws};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return AB_ERR_INVALID_ARG;
  return ws_bytes < ws_need ? AB_ERR_WORKSPACE : AB_OK;
}

ab_status do_attention(const Dims& d, const void* Q, const void* K, const void* V, const int32_t* idx,
                       const uint32_t* pi_q32, const int32_t* count, void* O, bool dense, cudaStream_t st) {
  if (!Q || !K || !V || !O) return AB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return AB_ERR_INVALID_ARG;
  if (!dense) {
    if (!idx || !pi_q32 || !count) return AB_ERR_INVALID_ARG;
    if (!aligned16(idx) || !aligned16(pi_q32) || !aligned16(count)) return AB_ERR_INVALID_ARG;
  }
  return d.d == 128 ? run_attention<128>(d, Q, K, V, idx, pi_q32, count, O, dense, st)
                    : run_attention<64>(d, Q, K, V, idx, pi_q32, count, O, dense, st);
}

// ------------------------------------------- scratch for ab_select_static
// One file-scope device array serves every ab_select_static call on a device.
// Host code cannot use the symbol itself as a device address; its address is
// looked up with cudaGetSymbolAddress, with the device current.  The address
// belongs to the CUDA context it was looked up in, so it is cached per device
// together with that context and looked up again when the calling thread's
// current context is another one (a context made current by a host
// framework, or a new primary context after a device reset).
static __device__ __align__(256) uint8_t g_select_scratch[AB_SELECT_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchAddr {
  CUcontext ctx;
  void* ptr;
};
ScratchAddr g_scratch_addr[kMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 ctx_current_fn() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &ptr, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
  });
  return fn;
}

// Device address of g_select_scratch in the calling thread's current context
// (nullptr on failure).
void* static_scratch_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  auto get_ctx = ctx_current_fn();
  if (!get_ctx) return nullptr;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;  // null before the thread's first runtime call
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchAddr& e = g_scratch_addr[dev];
  if (ctx && e.ptr && e.ctx == ctx) return e.ptr;
  void* ptr = nullptr;  // the lookup also makes the device's context current if none was
  if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || !ptr) return nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  e.ctx = ctx;
  e.ptr = ptr;
  return ptr;
}

}  // namespace

extern "C" {

int32_t ab_budget(const ab_params* p) {
  Dims d;
  if (check_params(p, true, &d) != AB_OK) return -1;
  return d.Kb;
}

ab_status ab_workspace_size(const ab_params* p, size_t* bytes) {
  Dims d;
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  if (!bytes) return AB_ERR_INVALID_ARG;
  *bytes = workspace_layout(d).total;
  return AB_OK;
}

ab_status ab_select(const ab_params* p, const void* Q, const void* K, float* P, float* centroids, int32_t* counts,
                    void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  NvtxRange nvtx("ab_select");
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  return do_select(d, Q, K, P, centroids, counts, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

ab_status ab_select_sample(const ab_params* p, const void* Q, const void* K, float* P, int32_t* idx,
                           uint32_t* pi_q32, int32_t* count, void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  NvtxRange nvtx("ab_select_sample");
  return do_select_sample(d, Q, K, P, idx, pi_q32, count, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

ab_status ab_sample(const ab_params* p, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count,
                    void* stream) {
  Dims d;
  NvtxRange nvtx("ab_sample");
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  return do_sample(d, P, idx, pi_q32, count, static_cast<cudaStream_t>(stream));
}

ab_status ab_sample_systematic(const ab_params* p, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count,
                               void* stream) {
  Dims d;
  NvtxRange nvtx("ab_sample_systematic");
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  if (!P || !idx || !pi_q32 || !count) return AB_ERR_INVALID_ARG;
  if (!aligned16(P) || !aligned16(idx) || !aligned16(pi_q32) || !aligned16(count)) return AB_ERR_INVALID_ARG;
  SipArgs a{};
  a.P = P; a.idx = idx; a.pi_q32 = pi_q32; a.count = count;
  a.H = d.H; a.Nq = d.Nq; a.Nkv = d.Nkv; a.Kb = d.Kb;
  a.seed_lo = uint32_t(d.seed); a.seed_hi = uint32_t(d.seed >> 32);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = d.BH * d.Nq;
  if (d.Nkv <= 2048) {  // one warp per row
    return launch_sip_warp<true>(a, rows, d.Nkv, st);
  } else if (d.Nkv <= kSipSmemCap) {
    const int smem = 16 * ((d.Nkv + 3) / 4);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(sip_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return AB_ERR_CUDA;
    sip_kernel<true, true><<<unsigned(d.BH * d.Nq), kSipThreads, smem, st>>>(a);
  } else {
    sip_kernel<false, true><<<unsigned(d.BH * d.Nq), kSipThreads, 0, st>>>(a);
  }
  return launch_status();
}

ab_status ab_sample_topk(const ab_params* p, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count,
                         void* stream) {
  Dims d;
  NvtxRange nvtx("ab_sample_topk");
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  if (!P || !idx || !pi_q32 || !count) return AB_ERR_INVALID_ARG;
  if (!aligned16(P) || !aligned16(idx) || !aligned16(pi_q32) || !aligned16(count)) return AB_ERR_INVALID_ARG;
  SipArgs a{};
  a.P = P; a.idx = idx; a.pi_q32 = pi_q32; a.count = count;
  a.H = d.H; a.Nq = d.Nq; a.Nkv = d.Nkv; a.Kb = d.Kb;
  topk_kernel<<<unsigned(d.BH * d.Nq), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

ab_status ab_attention(const ab_params* p, const void* Q, const void* K, const void* V, const int32_t* idx,
                       const uint32_t* pi_q32, const int32_t* count, void* O, void* stream) {
  Dims d;
  NvtxRange nvtx("ab_attention");
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  return do_attention(d, Q, K, V, idx, pi_q32, count, O, false, static_cast<cudaStream_t>(stream));
}

ab_status ab_attention_dense(const ab_params* p, const void* Q, const void* K, const void* V, void* O,
                             void* stream) {
  Dims d;
  NvtxRange nvtx("ab_attention_dense");
  const ab_status s = check_params(p, false, &d);
  if (s != AB_OK) return s;
  return do_attention(d, Q, K, V, nullptr, nullptr, nullptr, O, true, static_cast<cudaStream_t>(stream));
}

ab_status ab_forward(const ab_params* p, const void* Q, const void* K, const void* V, float* P, int32_t* idx,
                     uint32_t* pi_q32, int32_t* count, void* O, void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  NvtxRange nvtx("ab_forward");
  ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  s = check_path_args(Q, K, V, P, idx, pi_q32, count, O, workspace, ws_bytes, workspace_layout(d).total);
  if (s != AB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = do_select(d, Q, K, P, nullptr, nullptr, workspace, ws_bytes, st);
  if (s != AB_OK) return s;
  s = do_sample(d, P, idx, pi_q32, count, st);
  if (s != AB_OK) return s;
  return do_attention(d, Q, K, V, idx, pi_q32, count, O, false, st);
}

ab_status ab_forward_slice(const ab_params* p, int32_t bh0, int32_t nbh, const void* Q, const void* K,
                           const void* V, float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count, void* O,
                           void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  NvtxRange nvtx("ab_forward_slice");
  ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  if (nbh < 1 || bh0 < 0 || int64_t(bh0) + nbh > int64_t(d.BH)) return AB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the slice as a problem of its own (B = 1, H = nbh); the draws keep the
  // whole problem's counters (its H and the slice's first row)
  Dims dc = d;
  dc.B = 1; dc.H = nbh; dc.BH = nbh;
  s = check_path_args(Q, K, V, P, idx, pi_q32, count, O, workspace, ws_bytes, workspace_layout(dc).total);
  if (s != AB_OK) return s;
  s = do_select(dc, Q, K, P, nullptr, nullptr, workspace, ws_bytes, st);
  if (s != AB_OK) return s;
  s = do_sample(dc, P, idx, pi_q32, count, st, d.H, int64_t(bh0) * d.Nq);
  if (s != AB_OK) return s;
  return do_attention(dc, Q, K, V, idx, pi_q32, count, O, false, st);
}

namespace {

// Copy streams and events of the pipelined host call, created on a
// context's first call and kept for the library's lifetime (one set per
// CUDA context, like the static scratch address).  A call holds the set's
// lock while it enqueues, so calls from several host threads take turns;
// re-recording an event after a stream has waited on it is safe (the wait
// captured the earlier record).
struct HostPipe {
  CUcontext ctx = nullptr;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr, in_done = nullptr, comp_done = nullptr;
  std::mutex mu;
};
std::mutex g_pipes_mutex;
std::vector<HostPipe*> g_pipes;  // never freed: streams outlive every call

HostPipe* host_pipe_current_context() {
  auto get_ctx = ctx_current_fn();
  if (!get_ctx) return nullptr;
  CUcontext ctx = nullptr;
  int dev = -1;  // setting the current device makes its primary context current if none was
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  std::lock_guard<std::mutex> lock(g_pipes_mutex);
  for (HostPipe* h : g_pipes)
    if (h->ctx == ctx) return h;
  HostPipe* h = new HostPipe;
  h->ctx = ctx;
  cudaEvent_t* evs[4] = {&h->start, &h->done, &h->in_done, &h->comp_done};
  bool ok = cudaStreamCreateWithFlags(&h->in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&h->out, cudaStreamNonBlocking) == cudaSuccess;
  for (cudaEvent_t* e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    for (cudaEvent_t* e : evs)
      if (*e) cudaEventDestroy(*e);
    if (h->in) cudaStreamDestroy(h->in);
    if (h->out) cudaStreamDestroy(h->out);
    delete h;
    return nullptr;
  }
  g_pipes.push_back(h);
  return h;
}

}  // namespace

ab_status ab_forward_host(const ab_params* p, const void* Q_host, const void* K_host, const void* V_host,
                          void* O_host, void* Q, void* K, void* V, float* P, int32_t* idx, uint32_t* pi_q32,
                          int32_t* count, void* O, void* workspace, size_t ws_bytes, void* stream) {
  Dims d;
  NvtxRange nvtx("ab_forward_host");
  ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  if (!Q_host || !K_host || !V_host || !O_host) return AB_ERR_INVALID_ARG;
  s = check_path_args(Q, K, V, P, idx, pi_q32, count, O, workspace, ws_bytes, workspace_layout(d).total);
  if (s != AB_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t q_head = size_t(d.L) * d.d * 2, kv_head = size_t(d.Lk) * d.d * 2;  // bytes per (b, h)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return AB_ERR_CUDA;
  // groups of up to ceil(BH / 10) heads, a multiple of 4 so that every group's
  // row offset keeps the per-row buffers 16-byte aligned
  const int per = (((d.BH + 9) / 10) + 3) / 4 * 4;
  if (cap != cudaStreamCaptureStatusNone || per >= d.BH) {  // one stream: copies, path, copy back
    const size_t qb = size_t(d.BH) * q_head, kvb = size_t(d.BH) * kv_head;
    if (cudaMemcpyAsync(Q, Q_host, qb, cudaMemcpyHostToDevice, st) != cudaSuccess) return AB_ERR_CUDA;
    if (cudaMemcpyAsync(K, K_host, kvb, cudaMemcpyHostToDevice, st) != cudaSuccess) return AB_ERR_CUDA;
    if (cudaMemcpyAsync(V, V_host, kvb, cudaMemcpyHostToDevice, st) != cudaSuccess) return AB_ERR_CUDA;
    s = ab_forward(p, Q, K, V, P, idx, pi_q32, count, O, workspace, ws_bytes, stream);
    if (s != AB_OK) return s;
    if (cudaMemcpyAsync(O_host, O, qb, cudaMemcpyDeviceToHost, st) != cudaSuccess) return AB_ERR_CUDA;
    return AB_OK;
  }
  // Pipelined over groups of heads (every (b, h) is independent): the inputs
  // of group c + 1 cross PCIe while group c computes on the caller's stream
  // and group c - 1's output crosses back, on the context's two copy streams.
  HostPipe* hp = host_pipe_current_context();
  if (!hp) return AB_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hp->mu);
  HostPipe& pipe = *hp;
  const cudaEvent_t start = pipe.start, done = pipe.done, in_done = pipe.in_done, comp_done = pipe.comp_done;
  if (cudaEventRecord(start, st) != cudaSuccess) return AB_ERR_CUDA;  // after the caller's earlier work
  if (cudaStreamWaitEvent(pipe.in, start, 0) != cudaSuccess) return AB_ERR_CUDA;
  if (cudaStreamWaitEvent(pipe.out, start, 0) != cudaSuccess) return AB_ERR_CUDA;
  auto bf = [](const void* base, size_t off) { return static_cast<const uint8_t*>(base) + off; };
  auto bw = [](void* base, size_t off) { return static_cast<uint8_t*>(base) + off; };
  for (int bh0 = 0; bh0 < d.BH; bh0 += per) {
    const int nbh = per < d.BH - bh0 ? per : d.BH - bh0;
    const size_t off = size_t(bh0) * q_head, bytes = size_t(nbh) * q_head;           // Q, O
    const size_t koff = size_t(bh0) * kv_head, kbytes = size_t(nbh) * kv_head;       // K, V
    if (cudaMemcpyAsync(bw(Q, off), bf(Q_host, off), bytes, cudaMemcpyHostToDevice, pipe.in) != cudaSuccess ||
        cudaMemcpyAsync(bw(K, koff), bf(K_host, koff), kbytes, cudaMemcpyHostToDevice, pipe.in) != cudaSuccess ||
        cudaMemcpyAsync(bw(V, koff), bf(V_host, koff), kbytes, cudaMemcpyHostToDevice, pipe.in) != cudaSuccess)
      return AB_ERR_CUDA;
    if (cudaEventRecord(in_done, pipe.in) != cudaSuccess) return AB_ERR_CUDA;
    if (cudaStreamWaitEvent(st, in_done, 0) != cudaSuccess) return AB_ERR_CUDA;
    // the group as a problem of its own (B = 1, H = nbh); the draws keep the
    // counters of the full problem (H, first row)
    Dims dc = d;
    dc.B = 1; dc.H = nbh; dc.BH = nbh;
    const size_t rows0 = size_t(bh0) * d.Nq;
    float* Pc = P + rows0 * d.Nkv;
    int32_t* idxc = idx + rows0 * d.Nkv;
    uint32_t* pic = pi_q32 + rows0 * d.Nkv;
    int32_t* cntc = count + rows0;
    s = do_select(dc, bf(Q, off), bf(K, koff), Pc, nullptr, nullptr, workspace, ws_bytes, st);
    if (s != AB_OK) return s;
    s = do_sample(dc, Pc, idxc, pic, cntc, st, d.H, int64_t(rows0));
    if (s != AB_OK) return s;
    s = do_attention(dc, bf(Q, off), bf(K, koff), bf(V, koff), idxc, pic, cntc, bw(O, off), false, st);
    if (s != AB_OK) return s;
    if (cudaEventRecord(comp_done, st) != cudaSuccess) return AB_ERR_CUDA;
    if (cudaStreamWaitEvent(pipe.out, comp_done, 0) != cudaSuccess) return AB_ERR_CUDA;
    if (cudaMemcpyAsync(bw(O_host, off), bf(O, off), bytes, cudaMemcpyDeviceToHost, pipe.out) != cudaSuccess)
      return AB_ERR_CUDA;
  }
  if (cudaEventRecord(done, pipe.out) != cudaSuccess) return AB_ERR_CUDA;
  if (cudaStreamWaitEvent(st, done, 0) != cudaSuccess) return AB_ERR_CUDA;  // the caller's stream covers it all
  return AB_OK;
}

ab_status ab_select_static(const ab_params* p, const void* Q, const void* K, float* P, float* centroids,
                           int32_t* counts, void* stream) {
  Dims d;
  NvtxRange nvtx("ab_select_static");
  const ab_status s = check_params(p, true, &d);
  if (s != AB_OK) return s;
  if (workspace_layout(d).total > size_t(AB_SELECT_STATIC_SCRATCH_BYTES)) return AB_ERR_WORKSPACE;
  void* scratch = static_scratch_current_device();
  if (!scratch) return AB_ERR_CUDA;
  return do_select(d, Q, K, P, centroids, counts, scratch, size_t(AB_SELECT_STATIC_SCRATCH_BYTES),
                   static_cast<cudaStream_t>(stream), /*overlap=*/false);
}

ab_status ab_get_device_error(void* stream, int32_t* code) {
  if (!code) return AB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyFromSymbolAsync(&host, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return AB_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return AB_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return AB_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return AB_ERR_CUDA;
  *code = host;
  return AB_OK;
}

const char* ab_status_string(ab_status s) {
  switch (s) {
    case AB_OK: return "ok";
    case AB_ERR_INVALID_ARG: return "invalid argument";
    case AB_ERR_UNSUPPORTED: return "unsupported size";
    case AB_ERR_CUDA: return "CUDA error";
    case AB_ERR_CAPACITY: return "list entry or count out of range";
    case AB_ERR_TIMEOUT: return "device pipeline wait timed out";
    case AB_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

}  // extern "C"
