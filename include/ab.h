/*
 * ab.h -- C ABI of the AB-Attention (Accurate Block Attention) hot path for
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one summarised on the page "AB-Attention: Video Difüzyon
 * Transformer'larını Hızlandırmak İçin Doğru Blok Dikkat Mekanizması"
 * (Edumints summary of Hugging Face Papers entry 2610.39663), called "the
 * AB-Attention page" below.  Its section "AB-Attention ve Üç Temel Yeniliği"
 * names three parts, each behind one call here:
 *
 *   ab_select     IBCS, the intra-block clustering selector: cluster the queries
 *                 inside each query block (no token permutation) and estimate
 *                 every KV block's share of the block's attention mass.
 *   ab_sample     SIP, sampling with inclusion-probability weighting: draw KV
 *                 blocks in proportion to that estimate and keep each kept
 *                 block's inverse inclusion probability.  (ab_sample_systematic
 *                 draws a fixed-size sample with the same probabilities;
 *                 ab_sample_topk is the truncation SIP replaces.)
 *   ab_attention  the kernel that packs the small kept KV blocks into full
 *                 tensor-core tiles and computes the 1/pi-weighted softmax, an
 *                 estimate of softmax(Q K^T / sqrt(d)) V (the formula of the
 *                 "Cross-Attention (Çapraz Dikkat Mekanizması)" glossary page,
 *                 "Cross-Attention Nasıl Çalışır?").
 *
 * ab_attention_dense computes exact dense attention with the same kernel
 * family (the reference point for speed), ab_forward runs the three steps on
 * device buffers, ab_forward_host runs them on host buffers.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors Q and O are [B, H, L, d], K and V are [B, H, Lk, d], all
 *    bfloat16, contiguous, d fastest, tokens in raster order of the (t, y, x)
 *    grid.  Lk = ab_params.L_kv, or L when L_kv is 0 (self-attention); under
 *    cross-attention the keys and values come from a sequence of their own
 *    length (Cross-Attention glossary page, "Cross-Attention Nasıl
 *    Çalışır?").  Query blocks are the contiguous runs of q_block queries
 *    (Nq = ceil(L / q_block)); KV blocks the runs of kv_block keys
 *    (Nkv = ceil(Lk / kv_block)); the last block of each kind may be
 *    partial.
 *  - Memory: the caller allocates and owns every buffer (device memory unless a
 *    call says "host"); the library allocates and frees no memory (it creates
 *    streams and events once per CUDA context and keeps them: two copy
 *    streams and four events for the pipelined ab_forward_host, one stream
 *    and two events on which the selecting calls run the K-block summaries
 *    beside k-means).
 *    Every device pointer must be 16-byte aligned.
 *  - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *    Every call only enqueues work on it and returns; results are ready when
 *    the stream reaches them (work on the library's own streams is joined
 *    back to `stream` by events, which also works under stream capture).
 *    The library keeps no state between calls other than the device error
 *    word, the fixed scratch array behind ab_select_static and those
 *    streams and events.
 *  - Errors: arguments are checked on the host before anything is launched;
 *    a bad argument returns AB_ERR_INVALID_ARG (or AB_ERR_UNSUPPORTED for a
 *    valid but unimplemented size) and enqueues nothing.  AB_ERR_CUDA reports
 *    a failed launch.  Problems found on the device (a list entry out of range,
 *    a count above capacity, a pipeline wait that timed out) never trap: the
 *    kernel records the first one in the device error word and skips the bad
 *    work; read it with ab_get_device_error.
 *  - Randomness: the only random numbers are SIP's draws, from
 *    Philox4x32-10 (Salmon et al., SC'11) keyed by ab_params.seed, so a call
 *    is deterministic for fixed inputs and seed.
 */
#ifndef AB_ATTENTION_AB_H_
#define AB_ATTENTION_AB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AB_OK = 0,
  AB_ERR_INVALID_ARG = 1, /* null/misaligned pointer, size out of range */
  AB_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d = 96) */
  AB_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  AB_ERR_CAPACITY = 4,    /* device: count > Nkv or a list index >= Nkv */
  AB_ERR_TIMEOUT = 5,     /* device: a pipeline wait gave up (kernel ended early) */
  AB_ERR_WORKSPACE = 6,   /* workspace too small */
} ab_status;

/* Problem description shared by every call. */
typedef struct {
  int32_t B, H, L, d;        /* batch, heads, query tokens, head dim; d in {64, 128}; 1 <= L <= 2^24 */
  int32_t q_block;           /* query block size, 64 or 128 */
  int32_t kv_block;          /* KV block size, 16, 32 or 64 */
  int32_t C;                 /* clusters per query block: 1, 2, 4, 8 or 16 */
  int32_t kmeans_iters;      /* Lloyd iterations, 1..16 (3 in the workloads) */
  float keep_ratio;          /* target kept fraction of KV blocks, in (0, 1] */
  int32_t L_kv;              /* key/value tokens Lk, 0 <= L_kv <= 2^24; 0 means Lk = L */
  uint64_t seed;             /* Philox key of the SIP draws */
} ab_params;

/*
 * Kept KV blocks per query block in expectation:
 *   Kb = clamp(floor(keep_ratio * Nkv + 1/2), 1, Nkv)   (computed in double).
 * Returns -1 if p is invalid.
 */
int32_t ab_budget(const ab_params* p);

/* Bytes of device workspace ab_select (and ab_forward) need for *p. */
ab_status ab_workspace_size(const ab_params* p, size_t* bytes);

/*
 * IBCS (AB-Attention page, "AB-Attention ve Üç Temel Yeniliği", IBCS item).
 * For every (b, h) and query block i:
 *   kbar_j  = mean of the valid keys of KV block j;
 *   mu, n_c = Lloyd k-means of the block's n_i queries with C clusters and
 *             kmeans_iters iterations (initial centroid c is the query at
 *             offset floor((c + 1/2) n_i / C); an empty cluster keeps its
 *             centroid; n_c are the sizes of the last assignment);
 *   S_cj    = mu_c . kbar_j / sqrt(d) + ln n_j   (n_j = valid keys in block j);
 *   P[i,j]  = sum_c (n_c / n_i) softmax_j(S_cj).
 * The centroid-summary product runs on the tensor cores in bfloat16 with fp32
 * accumulation, so P matches an exact evaluation to a few 1e-3 relative.
 *
 *   Q          device, [B, H, L, d] bf16.
 *   K          device, [B, H, Lk, d] bf16.
 *   P          device, out, [B, H, Nq, Nkv] fp32; each row sums to 1.
 *   centroids  device, out, optional (NULL), [B, H, Nq, C, d] fp32.
 *   counts     device, out, optional (NULL), [B, H, Nq, C] int32.
 *   workspace  device scratch of at least ab_workspace_size bytes
 *              (AB_ERR_WORKSPACE otherwise); contents need no initialisation.
 */
ab_status ab_select(const ab_params* p, const void* Q, const void* K, float* P, float* centroids,
                    int32_t* counts, void* workspace, size_t ws_bytes, void* stream);

/*
 * SIP (AB-Attention page, "AB-Attention ve Üç Temel Yeniliği", SIP item).
 * For every row (b, h, i) of P, entirely in integer arithmetic:
 *   W_j  = max(1, floor(P[i,j] * 2^24));
 *   inclusion probabilities proportional to W, capped at 1, summing to Kb: the
 *   capped set A grows until stable by adding every j not in A with
 *   R W_j >= S (R = Kb - |A|, S = sum of W_j over j not in A); then
 *   Pi_j = 2^32 for j in A, else max(1, floor(R W_j 2^32 / S)); pi_j = Pi_j / 2^32;
 *   u_j  = word (j mod 4) of Philox4x32-10(counter (j div 4, i, h, b),
 *          key (seed mod 2^32, seed div 2^32)); block j is kept iff u_j < Pi_j.
 * Kept blocks are written in ascending j order.
 *
 *   P       device, [B, H, Nq, Nkv] fp32 (any source).
 *   idx     device, out, [B, H, Nq, Nkv] int32: row r's first count[r]
 *           entries are the kept j; the rest are left untouched.
 *   pi_q32  device, out, [B, H, Nq, Nkv] uint32: Pi_j mod 2^32 of each kept
 *           block (0 encodes pi = 1), aligned with idx.
 *   count   device, out, [B, H, Nq] int32.
 * Results are bit-identical to the integer specification above.
 */
ab_status ab_sample(const ab_params* p, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count,
                    void* stream);

/*
 * Systematic sampling with SIP's inclusion probabilities: a fixed-size
 * alternative to ab_sample's independent draws (AB-Attention page, SIP item:
 * blocks are sampled in proportion to the IBCS estimate and reweighted by the
 * inverse inclusion probability; the sampling design is left open).  Pi_j as
 * for ab_sample; one offset U per row, word 0 of Philox4x32-10 at counter
 * (0xFFFFFFFF, i, h, b) with key (seed lo, seed hi); with C_j the sum of Pi_k
 * over k < j, block j is kept iff some point U + m 2^32 (m >= 0) lies in
 * [C_j, C_j + Pi_j).  Every block is kept with probability Pi_j / 2^32 (the
 * same weights make numerator and denominator unbiased) and count is floor or
 * ceil of sum_j Pi_j / 2^32 (Kb or Kb - 1).  Same arguments, layout,
 * ownership and errors as ab_sample; results are bit-identical to this
 * integer specification.
 */
ab_status ab_sample_systematic(const ab_params* p, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count,
                               void* stream);

/*
 * Truncation, the selection SIP replaces (AB-Attention page, section "Video
 * Difüzyon Modellerinde Dikkat (Attention) Darboğazı": pruned blocks vanish
 * from the softmax; SIP item: SIP estimates dense attention rather than
 * truncating it).  For every row of P, keep the Kb blocks with the largest
 * P (Kb as for ab_sample; ties to the lower block index), in ascending order,
 * with weight 1 (pi_q32 = 0); count = Kb.  Same arguments, layout, ownership
 * and errors as ab_sample; P must be >= 0 (as ab_select writes it).  With
 * ab_attention this is block-sparse attention without reweighting, at the same
 * budget as SIP.
 */
ab_status ab_sample_topk(const ab_params* p, const float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count,
                         void* stream);

/*
 * 1/pi-weighted block-sparse attention (AB-Attention page, SIP item: one pass
 * estimates dense attention instead of truncating it; "Donanım Dostu Çekirdek"
 * item: KV blocks much smaller than a tile are packed into full tensor-core
 * tiles).  For query q of block i, with s_k = q . k / sqrt(d) and
 * w_j = 2^32 / Pi_j (1 when pi_q32 = 0):
 *   O_q = sum_{j in list(i)} w_j sum_{k in j, k < Lk} e^{s_k} v_k
 *       / sum_{j in list(i)} w_j sum_{k in j, k < Lk} e^{s_k};
 * a query block with count 0 gets O = 0.  The lists may come from ab_sample
 * (ab_sample_systematic, ab_sample_topk) or from any other source, in any
 * order; each entry must
 * satisfy 0 <= idx < Nkv and count <= Nkv (violations raise AB_ERR_CAPACITY on
 * the device and the offending entries or rows are skipped).
 *
 *   Q        device, [B, H, L, d] bf16.
 *   K, V     device, [B, H, Lk, d] bf16.
 *   idx, pi_q32, count  device, as written by ab_sample.
 *   O        device, out, [B, H, L, d] bf16 (round to nearest even).
 */
ab_status ab_attention(const ab_params* p, const void* Q, const void* K, const void* V, const int32_t* idx,
                       const uint32_t* pi_q32, const int32_t* count, void* O, void* stream);

/*
 * Dense attention O = softmax(Q K^T / sqrt(d)) V, bidirectional, no mask
 * (Cross-Attention glossary page, "Cross-Attention Nasıl Çalışır?"; the
 * AB-Attention page's "3D tam dikkat").  Uses q_block (64 or 128), B, H, L,
 * L_kv, d from *p; the other fields are ignored.  Same layout rules as
 * ab_attention.
 */
ab_status ab_attention_dense(const ab_params* p, const void* Q, const void* K, const void* V, void* O,
                             void* stream);

/*
 * ab_select followed by ab_sample, with the same outputs (P and the lists,
 * bit-identical to the two calls in a row), in one launch less: for rows of
 * at most 2048 KV blocks the scoring kernel runs SIP on the rows of P it has
 * just computed (AB-Attention page, "AB-Attention ve Üç Temel Yeniliği": the
 * IBCS estimate is what SIP samples from), so P is read back from L2 rather
 * than after a DRAM round trip.  Longer rows run the two steps as separate
 * launches.  Arguments as for ab_select (P is still written) and ab_sample;
 * errors as for those two calls, all found before either step is enqueued.
 * On a B200 the fused launch measured slower
 * than the two launches (its nine warps per scoring CTA sample with fewer
 * rows in flight than the sampler's own grid), so ab_forward keeps the two.
 */
ab_status ab_select_sample(const ab_params* p, const void* Q, const void* K, float* P, int32_t* idx,
                           uint32_t* pi_q32, int32_t* count, void* workspace, size_t ws_bytes, void* stream);

/*
 * The three steps in order on device buffers: ab_select (into P, with
 * centroids/counts not kept), ab_sample, ab_attention.  `workspace` as for
 * ab_select.  Every buffer is checked (non-null, 16-byte aligned, workspace
 * size) before the first step is enqueued.
 */
ab_status ab_forward(const ab_params* p, const void* Q, const void* K, const void* V, float* P,
                     int32_t* idx, uint32_t* pi_q32, int32_t* count, void* O, void* workspace,
                     size_t ws_bytes, void* stream);

/*
 * ab_forward on a slice of the problem's heads: the (b, h) pairs whose
 * flattened index b * H + h lies in [bh0, bh0 + nbh), for instance one GPU's
 * share when a layer's heads are divided among GPUs.  Every (b, h) is
 * independent on the whole path (selection, sampling and attention of a head
 * read only that head's Q, K and V), so the slices need no exchange of data.
 * *p describes the WHOLE problem (B, H and the rest); Q, O ([nbh, L, d]), K,
 * V ([nbh, Lk, d]), P, idx, pi_q32 ([nbh, Nq, Nkv]) and count ([nbh, Nq])
 * hold the slice only, in the layouts of the full tensors.  SIP's draws take
 * the whole problem's counters (b, h, i, j), so the slice's lists and output
 * are bit-identical to the same heads of ab_forward on the whole problem.
 * `workspace` as for ab_select, sized for the slice (ab_workspace_size of
 * the problem with B = 1, H = nbh).  AB_ERR_INVALID_ARG if the range is
 * empty or leaves [0, B * H); buffers are checked as for ab_forward, before
 * anything is enqueued.
 */
ab_status ab_forward_slice(const ab_params* p, int32_t bh0, int32_t nbh, const void* Q, const void* K,
                           const void* V, float* P, int32_t* idx, uint32_t* pi_q32, int32_t* count, void* O,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * ab_forward from HOST buffers: copies Q_host (host, [B, H, L, d] bf16),
 * K_host and V_host (host, [B, H, Lk, d] bf16; page-locked memory gives
 * asynchronous copies) to the device buffers Q, K, V, runs the path, and
 * copies O back to O_host (host, [B, H, L, d] bf16).  Results are bit-identical to ab_forward on the same inputs.  When
 * B * H > 4 and `stream` is not being captured, the call pipelines groups of
 * heads (every (b, h) is independent): the inputs of one group cross PCIe on
 * an internal stream while the previous group computes on `stream` and the
 * one before it copies back on a second internal stream; the two streams and
 * their events are created on the context's first pipelined call and reused
 * (calls from several host threads take turns enqueueing), and `stream`
 * waits for all of it.  Otherwise everything is enqueued on
 * `stream`.  O_host is valid once `stream` has been synchronised.  The device
 * buffers are owned by the caller.
 */
ab_status ab_forward_host(const ab_params* p, const void* Q_host, const void* K_host, const void* V_host,
                          void* O_host, void* Q, void* K, void* V, float* P, int32_t* idx,
                          uint32_t* pi_q32, int32_t* count, void* O, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * Size of the device array behind ab_select_static, in bytes (48 MiB).
 */
#define AB_SELECT_STATIC_SCRATCH_BYTES (48u * 1024u * 1024u)

/*
 * ab_select without a caller-supplied workspace, for callers that cannot
 * allocate device memory: code running inside a host framework that owns
 * every device allocation (a plugin under an inference engine's memory
 * planner), or code that must not block, since cudaMalloc and cudaFree can
 * synchronise the device.  The paper has no counterpart: this is an
 * interface choice of this library, not part of the method.
 *
 * Same arguments, outputs and results as ab_select, minus the workspace.  The
 * scratch is one array of AB_SELECT_STATIC_SCRATCH_BYTES in device memory,
 * defined at file scope in the library, so every GPU that loads the library
 * holds it until the process exits.  A problem whose ab_workspace_size
 * exceeds that limit is rejected with AB_ERR_WORKSPACE before anything is
 * enqueued (the Wan2.1-480p layer, 42 MB, fits; the HunyuanVideo-720p layer,
 * 91 MB, does not).  Nothing is allocated or freed, by this call or by the
 * library on its behalf.
 *
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * Every call on a device shares the one array and leaves its contents behind;
 * nothing in it needs to start at zero, because each call writes every byte
 * it reads, the failure path included (a k-means wait that gives up writes
 * NaN centroids and count -1, so that call's P is NaN and AB_ERR_TIMEOUT is
 * in the device error word).  Calls whose work overlaps on the GPU (other
 * streams, other host threads) race on the array: order them on one stream or
 * synchronise.  The array's address belongs to a CUDA context: it is looked
 * up again whenever the calling thread's current context differs from the one
 * it was looked up in.
 */
ab_status ab_select_static(const ab_params* p, const void* Q, const void* K, float* P, float* centroids,
                           int32_t* counts, void* stream);

/*
 * Reads and clears the device error word of the current device, after
 * synchronising `stream`.  *code receives AB_OK or the first ab_status raised
 * on the device since the last read.  Returns AB_ERR_CUDA if the read failed.
 */
ab_status ab_get_device_error(void* stream, int32_t* code);

/* Static description of a status code. */
const char* ab_status_string(ab_status s);

#ifdef __cplusplus
}
#endif

#endif /* AB_ATTENTION_AB_H_ */
