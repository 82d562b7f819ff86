// philox.cuh -- Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC'11), device side.
//
// The verification walk draws its uniforms from a counter, so any thread can produce
// the uniform of any (sequence, node, token) without state:
//   key     = (seed_lo, seed_hi)
//   counter = (v >> 2, b << 16 | purpose << 8 | node, offset_lo, offset_hi)
//   u       = (2 * (word[v & 3] >> 9) + 1) * 2^-24        (exact in fp32, inside (0,1))
// purpose 0: accept test of candidate `node` (v = 0); purpose 1: final sample at `node`.
#pragma once

#include <stdint.h>

namespace eagle {

// b fills 16 bits of the counter word, purpose and node 8 bits each: callers keep
// node, purpose <= kPhiloxMaxField and b <= 65535 (checked on the host).
constexpr int kPhiloxMaxField = 255;

struct Philox4 {
  uint32_t w[4];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {  // Weyl sequence key schedule between rounds
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0;
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  Philox4 r;
  r.w[0] = c0;
  r.w[1] = c1;
  r.w[2] = c2;
  r.w[3] = c3;
  return r;
}

__device__ __forceinline__ float word_to_uniform(uint32_t x) {
  return (2.0f * static_cast<float>(x >> 9) + 1.0f) * 5.9604644775390625e-8f;  // 2^-24
}

// The four uniforms of vocabulary group g (tokens 4g .. 4g+3).
__device__ __forceinline__ Philox4 philox_group(uint64_t seed, uint64_t offset, uint32_t b,
                                                uint32_t node, uint32_t purpose, uint32_t group) {
  return philox4x32_10(group, (b << 16) | (purpose << 8) | node, static_cast<uint32_t>(offset),
                       static_cast<uint32_t>(offset >> 32), static_cast<uint32_t>(seed),
                       static_cast<uint32_t>(seed >> 32));
}

__device__ __forceinline__ float uniform_at(uint64_t seed, uint64_t offset, uint32_t b, uint32_t node,
                                            uint32_t v, uint32_t purpose) {
  const Philox4 r = philox_group(seed, offset, b, node, purpose, v >> 2);
  return word_to_uniform(r.w[v & 3]);
}

}  // namespace eagle
