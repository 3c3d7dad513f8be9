// AB-Attention CPU oracle.
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
// statement of what the block-sparse attention path computes.  Only the
// tests, the package smoke check and the benchmark's CPU-baseline leg may
// load it.  It shares no code, header, table or constant with the CUDA
// library; the two meet only in the seeded inputs.
//
// Source pages (cited by title and section):
//  * "AB-Attention: Video Difüzyon Transformer'larını Hızlandırmak İçin Doğru
//    Blok Dikkat Mekanizması" (Edumints summary of Hugging Face Papers entry
//    2610.39663) -- called "the AB-Attention page" below.  Its section
//    "AB-Attention ve Üç Temel Yeniliği" defines the three parts: IBCS
//    (cluster the queries inside each query block, no token permutation),
//    SIP (sample blocks in proportion to the IBCS estimates and reweight by
//    the inverse inclusion probability, so one pass estimates dense attention
//    instead of truncating it) and the kernel (small KV blocks packed into
//    full tensor-core tiles).  Section "Video Difüzyon Modellerinde Dikkat
//    (Attention) Darboğazı" states the problem: 3D full attention over the
//    current activations, block-sparse over selected KV blocks.
//  * "Cross-Attention (Çapraz Dikkat Mekanizması)" glossary page, sections
//    "Cross-Attention Nasıl Çalışır?" and "Self-Attention ile Karşılaştırma":
//    Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V, Q, K, V from the same
//    sequence for self-attention.
//
// The pages give no equations, constants or tie-breaks for IBCS or SIP.  Every
// such choice below is marked "reading:" and is the plainest reading that the
// pages support.  Every floating-point sum is in double; inputs are the fp32
// values of bfloat16 tensors (exact).
//
// Parity status: every function here is pinned by the CPU tests (closed
// forms, invariants, a library Philox, exact subset enumeration, Monte Carlo);
// none is "parity unpinned".

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Philox4x32-10, from its published definition: J. K. Salmon, M. A. Moraes,
// R. O. Dror, D. E. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11), section 3.4 (the Philox S-box, N = 4, W = 32).  Each round takes the
// two 32x32->64 products of counter words 0 and 2 with the multipliers, XORs
// the high halves with the other two words and the round key, and permutes;
// the key is bumped by the Weyl constants between rounds.
// ---------------------------------------------------------------------------
const uint32_t kMul0 = 0xD2511F53u;
const uint32_t kMul1 = 0xCD9E8D57u;
const uint32_t kWeyl0 = 0x9E3779B9u;  // golden ratio
const uint32_t kWeyl1 = 0xBB67AE85u;  // sqrt(3) - 1

void philox_10(const uint32_t in_ctr[4], const uint32_t in_key[2], uint32_t out[4]) {
  uint32_t x0 = in_ctr[0], x1 = in_ctr[1], x2 = in_ctr[2], x3 = in_ctr[3];
  uint32_t k0 = in_key[0], k1 = in_key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += kWeyl0;
      k1 += kWeyl1;
    }
    const uint64_t p0 = (uint64_t)kMul0 * (uint64_t)x0;
    const uint64_t p1 = (uint64_t)kMul1 * (uint64_t)x2;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t y0 = hi1 ^ x1 ^ k0;
    const uint32_t y1 = lo1;
    const uint32_t y2 = hi0 ^ x3 ^ k1;
    const uint32_t y3 = lo0;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Number of valid tokens in block `j` of size `bs` over a sequence of length L.
inline int block_len(int j, int bs, int L) { return std::min(bs, L - j * bs); }

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// RNG entry point (for the tests): out = Philox4x32-10(ctr, key).
// ---------------------------------------------------------------------------
void orc_philox4x32_10(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
  philox_10(ctr, key, out);
}

// ---------------------------------------------------------------------------
// Dense attention, the ground truth.  Cross-Attention glossary page,
// "Cross-Attention Nasıl Çalışır?": softmax(Q K^T / sqrt(d)) V; self-attention
// ("Self-Attention ile Karşılaştırma") takes Q, K, V from one sequence.  The
// AB-Attention page's "3D tam dikkat" is bidirectional: no mask.
// One (b, h) slice: K, V are [L, d] fp32 (L keys), Q holds at least
// row0 + nrows query rows of d (a sequence of its own length under
// cross-attention); rows [row0, row0 + nrows) of the output go to O [nrows, d].
// ---------------------------------------------------------------------------
void orc_dense_rows(const float* Q, const float* K, const float* V, int L, int d,
                    int row0, int nrows, double* O) {
  const double scale = 1.0 / std::sqrt((double)d);
  std::vector<double> s(L);
  for (int r = 0; r < nrows; ++r) {
    const float* q = Q + (size_t)(row0 + r) * d;
    double m = -INFINITY;
    for (int k = 0; k < L; ++k) {
      double acc = 0.0;
      const float* kk = K + (size_t)k * d;
      for (int e = 0; e < d; ++e) acc += (double)q[e] * (double)kk[e];
      s[k] = acc * scale;
      m = std::max(m, s[k]);
    }
    double den = 0.0;
    double* o = O + (size_t)r * d;
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int k = 0; k < L; ++k) {
      const double p = std::exp(s[k] - m);
      den += p;
      const float* v = V + (size_t)k * d;
      for (int e = 0; e < d; ++e) o[e] += p * (double)v[e];
    }
    for (int e = 0; e < d; ++e) o[e] /= den;
  }
}

// ---------------------------------------------------------------------------
// IBCS, step 1: KV-block summaries.  AB-Attention page, "AB-Attention ve Üç
// Temel Yeniliği", IBCS item (block importance estimated cheaply); reading:
// the summary of a KV block is the mean of its valid keys (padding beyond L is
// never averaged).  K is one (b, h) slice [L, d]; Ksum is [Nkv, d].
// ---------------------------------------------------------------------------
void orc_ksum(const float* K, int L, int d, int kv_block, double* Ksum) {
  const int Nkv = ceil_div(L, kv_block);
  for (int j = 0; j < Nkv; ++j) {
    const int n = block_len(j, kv_block, L);
    double* out = Ksum + (size_t)j * d;
    for (int e = 0; e < d; ++e) out[e] = 0.0;
    for (int t = 0; t < n; ++t) {
      const float* k = K + (size_t)(j * kv_block + t) * d;
      for (int e = 0; e < d; ++e) out[e] += (double)k[e];
    }
    for (int e = 0; e < d; ++e) out[e] /= (double)n;
  }
}

// ---------------------------------------------------------------------------
// IBCS, step 2: cluster the queries of one query block, in place, with no
// token permutation (AB-Attention page, IBCS item).  Reading: Lloyd's
// k-means with C clusters and `iters` iterations on the n queries Qb [n, d];
//  * init: centroid c is the query at offset floor((c + 1/2) n / C);
//  * each iteration assigns every query to the centroid at least squared
//    Euclidean distance (ties go to the lowest c), then moves every centroid to
//    the mean of its members; a cluster left empty keeps its centroid;
//  * counts[c] is the size of cluster c in the last assignment.
// Outputs mu [C, d] and counts [C].  `assign` [n] (may be null) receives the
// last assignment.  Returns the number of iterations run.
// ---------------------------------------------------------------------------
int orc_kmeans(const float* Qb, int n, int d, int C, int iters, double* mu,
               int32_t* counts, int32_t* assign) {
  for (int c = 0; c < C; ++c) {
    const int src = (int)std::floor((c + 0.5) * (double)n / (double)C);
    for (int e = 0; e < d; ++e) mu[(size_t)c * d + e] = (double)Qb[(size_t)src * d + e];
  }
  std::vector<int> a(n, 0);
  std::vector<double> sum((size_t)C * d);
  for (int it = 0; it < iters; ++it) {
    for (int q = 0; q < n; ++q) {
      int best = 0;
      double best_d = INFINITY;
      for (int c = 0; c < C; ++c) {
        double dist = 0.0;
        for (int e = 0; e < d; ++e) {
          const double diff = (double)Qb[(size_t)q * d + e] - mu[(size_t)c * d + e];
          dist += diff * diff;
        }
        if (dist < best_d) {  // strict: a tie keeps the lower c
          best_d = dist;
          best = c;
        }
      }
      a[q] = best;
    }
    std::fill(sum.begin(), sum.end(), 0.0);
    for (int c = 0; c < C; ++c) counts[c] = 0;
    for (int q = 0; q < n; ++q) {
      counts[a[q]] += 1;
      for (int e = 0; e < d; ++e) sum[(size_t)a[q] * d + e] += (double)Qb[(size_t)q * d + e];
    }
    for (int c = 0; c < C; ++c) {
      if (counts[c] == 0) continue;  // empty cluster keeps its centroid
      for (int e = 0; e < d; ++e) mu[(size_t)c * d + e] = sum[(size_t)c * d + e] / counts[c];
    }
  }
  if (assign)
    for (int q = 0; q < n; ++q) assign[q] = a[q];
  return iters;
}

// ---------------------------------------------------------------------------
// IBCS, step 3: block-mass estimate of one query block (AB-Attention page,
// IBCS item: an estimate of each block's importance; SIP item: sampling
// proportional to that estimate).  Reading: a KV block's attention mass
// for centroid c is approximated by n_j exp(mu_c . kbar_j / sqrt(d)), i.e.
// score S_cj = mu_c . kbar_j / sqrt(d) + ln n_j, normalised over j with a
// softmax; the query block's estimate mixes the per-centroid distributions by
// cluster share:  P_j = sum_c (n_c / n_i) softmax_j(S_cj).
// mu [C, d], counts [C], Ksum [Nkv, d]; P [Nkv].
// ---------------------------------------------------------------------------
void orc_block_mass(const double* mu, const int32_t* counts, int C, int n_i,
                    const double* Ksum, int Nkv, int L, int kv_block, int d, double* P) {
  const double scale = 1.0 / std::sqrt((double)d);
  std::vector<double> s(Nkv);
  for (int j = 0; j < Nkv; ++j) P[j] = 0.0;
  for (int c = 0; c < C; ++c) {
    if (counts[c] == 0) continue;
    double m = -INFINITY;
    for (int j = 0; j < Nkv; ++j) {
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += mu[(size_t)c * d + e] * Ksum[(size_t)j * d + e];
      s[j] = dot * scale + std::log((double)block_len(j, kv_block, L));
      m = std::max(m, s[j]);
    }
    double z = 0.0;
    for (int j = 0; j < Nkv; ++j) {
      s[j] = std::exp(s[j] - m);
      z += s[j];
    }
    const double w = (double)counts[c] / (double)n_i;
    for (int j = 0; j < Nkv; ++j) P[j] += w * s[j] / z;
  }
}

// ---------------------------------------------------------------------------
// IBCS for one (b, h) slice: summaries, then k-means and block mass for the
// query blocks listed in `rows` (nrows of them; rows == null means all Nq).
// Q [L, d] (queries), K [Lk, d] (keys): Lk = L for self-attention; under
// cross-attention (Cross-Attention page, "Cross-Attention Nasıl Çalışır?")
// the keys come from another sequence, so the query blocks follow L and the
// KV blocks Lk.  P [nrows, Nkv]; mu [nrows, C, d] and counts [nrows, C] may
// be null.
// ---------------------------------------------------------------------------
void orc_select_head(const float* Q, const float* K, int L, int Lk, int d, int q_block, int kv_block,
                     int C, int iters, const int32_t* rows, int nrows, double* P, double* mu,
                     int32_t* counts) {
  const int Nq = ceil_div(L, q_block);
  const int Nkv = ceil_div(Lk, kv_block);
  if (!rows) nrows = Nq;
  std::vector<double> ksum((size_t)Nkv * d);
  orc_ksum(K, Lk, d, kv_block, ksum.data());
  std::vector<double> m((size_t)C * d);
  std::vector<int32_t> cnt(C);
  for (int r = 0; r < nrows; ++r) {
    const int i = rows ? rows[r] : r;
    const int n_i = block_len(i, q_block, L);
    orc_kmeans(Q + (size_t)i * q_block * d, n_i, d, C, iters, m.data(), cnt.data(), nullptr);
    orc_block_mass(m.data(), cnt.data(), C, n_i, ksum.data(), Nkv, Lk, kv_block, d,
                   P + (size_t)r * Nkv);
    if (mu) std::memcpy(mu + (size_t)r * C * d, m.data(), sizeof(double) * C * d);
    if (counts) std::memcpy(counts + (size_t)r * C, cnt.data(), sizeof(int32_t) * C);
  }
}

// ---------------------------------------------------------------------------
// SIP budget.  Reading: the expected number of kept KV blocks per query block
// is Kb = clamp(floor(keep_ratio * Nkv + 1/2), 1, Nkv).
// ---------------------------------------------------------------------------
int orc_budget(int Nkv, double keep_ratio) {
  double kb = std::floor(keep_ratio * (double)Nkv + 0.5);
  if (kb < 1.0) kb = 1.0;
  if (kb > (double)Nkv) kb = (double)Nkv;
  return (int)kb;
}

// ---------------------------------------------------------------------------
// Truncation for one query block: the selection that SIP is contrasted with.
// AB-Attention page, section "Video Difüzyon Modellerinde Dikkat (Attention)
// Darboğazı" (pruned blocks drop out of the softmax entirely) and section
// "AB-Attention ve Üç Temel Yeniliği", SIP item (SIP estimates dense attention
// rather than truncating it).  Readings: the same IBCS estimate P and the
// same budget Kb; keep the Kb blocks with the largest P, ties to the lower j;
// no reweighting (pi = 1, stored as pi_q32 = 0); kept j in ascending order.
// Returns count = Kb.
// ---------------------------------------------------------------------------
int orc_topk_row(const float* P, int Nkv, int Kb, int32_t* idx, uint32_t* pi_q32, int32_t* count) {
  std::vector<int> order(Nkv);
  for (int j = 0; j < Nkv; ++j) order[j] = j;
  // larger P first; equal P: lower j first
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return P[x] > P[y]; });
  std::vector<int> kept(order.begin(), order.begin() + Kb);
  std::sort(kept.begin(), kept.end());
  for (int e = 0; e < Kb; ++e) {
    idx[e] = kept[e];
    pi_q32[e] = 0u;
  }
  *count = Kb;
  return Kb;
}

// ---------------------------------------------------------------------------
// SIP for one query block (AB-Attention page, "AB-Attention ve Üç Temel
// Yeniliği", SIP item: blocks are sampled in proportion to the IBCS estimate
// and the kept ones are reweighted by the inverse inclusion probability).
// Readings, in order:
//  1. quantise: W_j = max(1, floor(P_j * 2^24)) (P_j is the fp32 estimate);
//  2. inclusion probabilities proportional to W with capping at 1, summing to
//     Kb (probability proportional to size): the capped set A grows until
//     it is stable; with R = Kb - |A| and S = sum of W over j not in A, every
//     j not in A with R W_j >= S joins A.  Then Pi_j = 2^32 for j in A and
//     Pi_j = max(1, floor(R W_j 2^32 / S)) otherwise (pi_j = Pi_j / 2^32);
//  3. independent Bernoulli draws: u_j = word (j mod 4) of
//     Philox4x32-10(counter = (j div 4, i, h, b), key = (seed lo, seed hi));
//     block j is kept iff u_j < Pi_j;
//  4. the kept j in ascending order go to idx[0..count), with
//     pi_q32 = Pi_j mod 2^32 (0 encodes pi = 1).
// P is one fp32 row [Nkv]; idx and pi_q32 hold up to Nkv entries.  Pi (may be
// null) receives every Pi_j as a 64-bit integer.  Returns count.
// ---------------------------------------------------------------------------
// Steps 1-2 of SIP: the Q32 inclusion probabilities Pi_j of one row.
static void sip_probabilities(const float* P, int Nkv, int Kb, uint64_t* Pi) {
  std::vector<uint64_t> W(Nkv);
  for (int j = 0; j < Nkv; ++j) {
    const double scaled = std::floor((double)P[j] * 16777216.0);
    W[j] = scaled < 1.0 ? 1u : (uint64_t)scaled;
  }
  std::vector<char> capped(Nkv, 0);
  uint64_t R = 0, S = 0;
  for (;;) {
    uint64_t ncap = 0;
    S = 0;
    for (int j = 0; j < Nkv; ++j) {
      if (capped[j]) ncap += 1;
      else S += W[j];
    }
    R = (uint64_t)Kb - ncap;
    bool grew = false;
    for (int j = 0; j < Nkv; ++j) {
      if (!capped[j] && (unsigned __int128)R * W[j] >= (unsigned __int128)S) {
        capped[j] = 1;
        grew = true;
      }
    }
    if (!grew) break;
  }
  for (int j = 0; j < Nkv; ++j) {
    if (capped[j]) {
      Pi[j] = 1ull << 32;
    } else {
      const unsigned __int128 num = ((unsigned __int128)R * W[j]) << 32;
      uint64_t pij = (uint64_t)(num / S);
      Pi[j] = pij < 1 ? 1 : pij;
    }
  }
}

int orc_sip_row(const float* P, int Nkv, int Kb, uint64_t seed, int b, int h, int i,
                int32_t* idx, uint32_t* pi_q32, int32_t* count, uint64_t* Pi) {
  std::vector<uint64_t> pis(Nkv);
  sip_probabilities(P, Nkv, Kb, pis.data());
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  int n = 0;
  for (int j = 0; j < Nkv; ++j) {
    const uint64_t pij = pis[j];
    if (Pi) Pi[j] = pij;
    const uint32_t ctr[4] = {(uint32_t)(j >> 2), (uint32_t)i, (uint32_t)h, (uint32_t)b};
    uint32_t u4[4];
    philox_10(ctr, key, u4);
    const uint64_t u = u4[j & 3];
    if (u < pij) {
      idx[n] = j;
      pi_q32[n] = (uint32_t)(pij & 0xffffffffull);
      n += 1;
    }
  }
  *count = n;
  return n;
}

// ---------------------------------------------------------------------------
// Systematic sampling with the same inclusion probabilities: the sampling
// design is not fixed by the pages (AB-Attention page, SIP item: blocks are
// sampled in proportion to the IBCS estimate and reweighted by the inverse
// inclusion probability).  Reading: one uniform offset U per row, word 0 of
// Philox4x32-10 with counter (0xFFFFFFFF, i, h, b) (outside the per-block
// counters j div 4 of SIP), key (seed lo, seed hi); with C_j = sum_{k<j} Pi_k,
// block j is kept iff one of the points U + m 2^32 (m = 0, 1, ...) lies in
// [C_j, C_j + Pi_j).  Each block is kept with probability Pi_j / 2^32 (so
// the same 1/pi weights make numerator and denominator unbiased) and the
// sample size is fixed up to one: the number of points below sum_j Pi_j.
// Lists as for SIP (ascending, pi_q32 = Pi mod 2^32).  Returns count.
// ---------------------------------------------------------------------------
// The selection for a given offset U in [0, 2^32) (U is a parameter so that
// tests can sweep it).
int orc_systematic_row_u(const float* P, int Nkv, int Kb, uint64_t U, int32_t* idx, uint32_t* pi_q32,
                         int32_t* count) {
  std::vector<uint64_t> pis(Nkv);
  sip_probabilities(P, Nkv, Kb, pis.data());
  // points strictly below x: U + m 2^32 < x for m >= 0
  auto points_below = [&](uint64_t x) -> uint64_t { return x > U ? ((x - U - 1) >> 32) + 1 : 0; };
  uint64_t C = 0;
  int n = 0;
  for (int j = 0; j < Nkv; ++j) {
    const uint64_t next = C + pis[j];
    if (points_below(next) - points_below(C) == 1) {
      idx[n] = j;
      pi_q32[n] = (uint32_t)(pis[j] & 0xffffffffull);
      n += 1;
    }
    C = next;
  }
  *count = n;
  return n;
}

int orc_systematic_row(const float* P, int Nkv, int Kb, uint64_t seed, int b, int h, int i,
                       int32_t* idx, uint32_t* pi_q32, int32_t* count) {
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  const uint32_t ctr[4] = {0xFFFFFFFFu, (uint32_t)i, (uint32_t)h, (uint32_t)b};
  uint32_t u4[4];
  philox_10(ctr, key, u4);
  return orc_systematic_row_u(P, Nkv, Kb, (uint64_t)u4[0], idx, pi_q32, count);
}

// ---------------------------------------------------------------------------
// Reweighted sums for one query (AB-Attention page, SIP item: "one pass
// statistically estimates dense attention instead of truncating it").
// Reading: numerator and denominator of the softmax are each a
// Horvitz-Thompson sum over the kept KV blocks, every term of block j weighted
// by 1/pi_j:
//   num = sum_{j kept} (1/pi_j) sum_{k in j, k < L} exp(s_k - shift) v_k,
//   den = sum_{j kept} (1/pi_j) sum_{k in j, k < L} exp(s_k - shift),
// with s_k = q . k / sqrt(d).  The shift only scales both sums.
// q [d]; K, V [L, d] of the same (b, h); num [d].
// ---------------------------------------------------------------------------
void orc_ht_sums(const float* q, const float* K, const float* V, int L, int d, int kv_block,
                 const int32_t* idx, const uint32_t* pi_q32, int count, double shift,
                 double* num, double* den) {
  const double scale = 1.0 / std::sqrt((double)d);
  for (int e = 0; e < d; ++e) num[e] = 0.0;
  *den = 0.0;
  for (int t = 0; t < count; ++t) {
    const int j = idx[t];
    const double pij = pi_q32[t] == 0 ? 4294967296.0 : (double)pi_q32[t];
    const double w = 4294967296.0 / pij;
    const int n = block_len(j, kv_block, L);
    for (int r = 0; r < n; ++r) {
      const int k = j * kv_block + r;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += (double)q[e] * (double)K[(size_t)k * d + e];
      const double p = w * std::exp(dot * scale - shift);
      *den += p;
      for (int e = 0; e < d; ++e) num[e] += p * (double)V[(size_t)k * d + e];
    }
  }
}

// ---------------------------------------------------------------------------
// Reweighted block-sparse attention for the queries of query block i of one
// (b, h) slice: O_q = num_q / den_q from orc_ht_sums with the shift set to the
// largest weighted logit max_{j kept, k in j} (s_k + ln(1/pi_j)).  Reading: an
// empty list (count = 0) gives O = 0.  All queries of the block share its
// list (block-sparse attention, AB-Attention page, "Darboğazı" section).
// Q [L, d]; K, V [Lk, d] (Lk = L for self-attention, another sequence's
// length under cross-attention); O [n_i, d].
// ---------------------------------------------------------------------------
void orc_ht_attention_block(const float* Q, const float* K, const float* V, int L, int Lk, int d,
                            int q_block, int kv_block, int i, const int32_t* idx,
                            const uint32_t* pi_q32, int count, double* O) {
  const int n_i = block_len(i, q_block, L);
  const double scale = 1.0 / std::sqrt((double)d);
  std::vector<double> num(d);
  for (int r = 0; r < n_i; ++r) {
    const float* q = Q + (size_t)(i * q_block + r) * d;
    double* o = O + (size_t)r * d;
    if (count == 0) {
      for (int e = 0; e < d; ++e) o[e] = 0.0;
      continue;
    }
    double m = -INFINITY;
    for (int t = 0; t < count; ++t) {
      const int j = idx[t];
      const double pij = pi_q32[t] == 0 ? 4294967296.0 : (double)pi_q32[t];
      const double bias = std::log(4294967296.0 / pij);
      const int n = block_len(j, kv_block, Lk);
      for (int rr = 0; rr < n; ++rr) {
        const int k = j * kv_block + rr;
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += (double)q[e] * (double)K[(size_t)k * d + e];
        m = std::max(m, dot * scale + bias);
      }
    }
    double den = 0.0;
    orc_ht_sums(q, K, V, Lk, d, kv_block, idx, pi_q32, count, m, num.data(), &den);
    for (int e = 0; e < d; ++e) o[e] = num[e] / den;
  }
}

}  // extern "C"
