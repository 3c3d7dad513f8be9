// Host-side check of the CUDA sampler's integer arithmetic (the functions of
// ab_sample.cuh that are host-callable) against exact 128-bit integer
// arithmetic, over random and edge-case inputs far beyond the ranges real P
// rows reach:
//   mul_le_shift32(a - 1, S, X)  ==  (a S <= X 2^32)                a in [1, 2^32]
//   pi_free(X, S)                ==  max(1, floor(X 2^32 / S))       0 <= X < S
//   quantise_w(p)                ==  max(1, floor(p 2^24))           p in [0, 1]
// Prints the number of cases and of mismatches; exits 1 on any mismatch.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <random>

#include "ab_sample.cuh"

using u128 = unsigned __int128;

static bool ref_le(uint64_t a, uint64_t S, uint64_t X) { return u128(a) * S <= (u128(X) << 32); }

static uint32_t ref_pi(uint64_t X, uint64_t S) {
  const u128 q = (u128(X) << 32) / S;
  return q < 1 ? 1u : uint32_t(q);
}

int main() {
  std::mt19937_64 rng(20261202);
  long cases = 0, bad = 0;
  auto rnd_bits = [&](int bits) -> uint64_t {
    if (bits <= 0) return 0;
    const uint64_t v = rng();
    return bits >= 64 ? v : (v & ((uint64_t(1) << bits) - 1));
  };

  // mul_le_shift32
  for (int it = 0; it < 4000000; ++it) {
    const uint64_t a = 1 + (it % 7 == 0 ? (uint64_t(1) << 32) - 1 - rnd_bits(3) : rnd_bits(1 + int(rng() % 32)));
    const uint64_t S = rnd_bits(1 + int(rng() % 64));
    uint64_t X;
    if (it % 3 == 0) {  // X near a S / 2^32, where the comparison is tight
      const u128 p = u128(a) * S;
      X = uint64_t(p >> 32) + (rng() % 3) - 1;
    } else {
      X = rnd_bits(1 + int(rng() % 64));
    }
    const bool got = ab::mul_le_shift32(uint32_t(a - 1), uint32_t(S >> 32), uint32_t(S), X);
    ++cases;
    if (got != ref_le(a, S, X)) {
      if (bad < 10) std::printf("mul_le_shift32 a=%llu S=%llu X=%llu\n", (unsigned long long)a,
                                (unsigned long long)S, (unsigned long long)X);
      ++bad;
    }
  }

  // pi_free on free blocks: 0 <= X < S
  auto check_pi = [&](uint64_t X, uint64_t S) {
    const double inv = 4294967296.0 / double(S);
    const uint32_t got = ab::pi_free(X, uint32_t(S >> 32), uint32_t(S), inv);
    ++cases;
    if (got != ref_pi(X, S)) {
      if (bad < 10) std::printf("pi_free X=%llu S=%llu got=%u want=%u\n", (unsigned long long)X,
                                (unsigned long long)S, got, ref_pi(X, S));
      ++bad;
    }
  };
  for (int it = 0; it < 4000000; ++it) {
    const uint64_t S = 1 + rnd_bits(1 + int(rng() % 63));
    uint64_t X;
    switch (it % 5) {
      case 0: X = S - 1; break;
      case 1: X = 0; break;
      case 2: {  // X at a multiple of S / 2^32 (exact quotients) and one below
        const uint64_t q = rnd_bits(32);
        const u128 num = u128(q) * S;
        X = uint64_t(num >> 32) - (rng() & 1);
        if (X >= S) X = S - 1;
        break;
      }
      default: X = rng() % S;
    }
    check_pi(X, S);
  }
  // realistic rows: S = sum of up to 2^14 weights of at most 2^24, X = R W with R <= 2^14
  for (int it = 0; it < 2000000; ++it) {
    const uint64_t S = 1 + rnd_bits(1 + int(rng() % 38));
    const uint64_t W = 1 + rnd_bits(1 + int(rng() % 24));
    const uint64_t R = 1 + rnd_bits(1 + int(rng() % 14));
    const uint64_t X = R * W;
    if (X < S) check_pi(X, S);
  }

  // quantise_w: every float in [0, 1] with a random mantissa, every exponent
  for (int e = 0; e <= 127; ++e) {
    for (int it = 0; it < 20000; ++it) {
      uint32_t bits = (uint32_t(e) << 23) | uint32_t(rng() & 0x7FFFFFu);
      if (e == 127) bits = 0x3F800000u;  // 1.0 is the only value with this exponent in [0, 1]
      float p;
      std::memcpy(&p, &bits, 4);
      const double f = std::floor(double(p) * 16777216.0);
      const uint32_t want = f < 1.0 ? 1u : uint32_t(f);
      ++cases;
      if (ab::quantise_w(p) != want) {
        if (bad < 10) std::printf("quantise_w p=%.9g got=%u want=%u\n", p, ab::quantise_w(p), want);
        ++bad;
      }
    }
  }
  std::printf("cases %ld mismatches %ld\n", cases, bad);
  return bad ? 1 : 0;
}
