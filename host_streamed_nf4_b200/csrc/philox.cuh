// philox.cuh -- the counter-based generator behind LoRA dropout:
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC 2011).  Ten rounds of: multiply counter words 0 and 2
// by the two round multipliers (64-bit products, split into halves), then
// new = {hi(w2*M1) ^ w1 ^ k0, lo(w2*M1), hi(w0*M0) ^ w3 ^ k1, lo(w0*M0)};
// the key advances by the two Weyl increments between rounds.
//
// Dropout mask of element e of a row-major [T, K] input under (seed,
// offset): word e % 4 of Philox({lo(e/4), hi(e/4), lo(offset),
// hi(offset)}, {lo(seed), hi(seed)}); the element is kept when the word's
// top 24 bits are >= floor(p * 2^24) (the product formed in fp32), and a
// kept value becomes bf16_rne(fp32(x) * fp32(1 / fp32(1 - p))).
#pragma once

#include <stdint.h>

namespace hsnf4 {

struct Philox4 {
  uint32_t w[4];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    // one 32 x 32 -> 64-bit multiply each gives both halves
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t lo0 = static_cast<uint32_t>(p0), hi0 = static_cast<uint32_t>(p0 >> 32);
    const uint32_t lo1 = static_cast<uint32_t>(p1), hi1 = static_cast<uint32_t>(p1 >> 32);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  Philox4 r;
  r.w[0] = c0;
  r.w[1] = c1;
  r.w[2] = c2;
  r.w[3] = c3;
  return r;
}

// The four dropout words of element group q (elements 4q .. 4q+3).
__device__ __forceinline__ Philox4 dropout_words(uint64_t q, uint64_t seed, uint64_t offset) {
  return philox4x32_10(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32),
                       static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32),
                       static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
}

// Host side: the integer threshold and the fp32 scale, formed the same way
// everywhere (fp32 product / difference / quotient, each rounded once).
struct DropoutParams {
  uint64_t seed, offset;
  uint32_t thr;  // keep <=> (word >> 8) >= thr
  float scale;   // 1 / (1 - p)
};

inline DropoutParams make_dropout(float p, uint64_t seed, uint64_t offset) {
  DropoutParams d;
  d.seed = seed;
  d.offset = offset;
  volatile float q = p * 16777216.0f;
  d.thr = static_cast<uint32_t>(q);
  volatile float one_minus = 1.0f - p;
  d.scale = 1.0f / one_minus;
  return d;
}

}  // namespace hsnf4
