// Counter-based random draws for the verification chain.
//
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC'11): ten rounds of a 4x32-bit S-box built from two 32x32->64
// multiplications, with a Weyl sequence bumping the 2x32-bit key between
// rounds.  Written here for the device; the CPU oracle carries its own copy.
#pragma once
#include <cstdint>

namespace sv {

struct Philox4 {
  uint32_t w[4];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kMulA = 0xD2511F53u;
  constexpr uint32_t kMulB = 0xCD9E8D57u;
  constexpr uint32_t kWeylA = 0x9E3779B9u;
  constexpr uint32_t kWeylB = 0xBB67AE85u;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t hiA = __umulhi(kMulA, c0), loA = kMulA * c0;
    const uint32_t hiB = __umulhi(kMulB, c2), loB = kMulB * c2;
    const uint32_t n0 = hiB ^ c1 ^ k0;
    const uint32_t n2 = hiA ^ c3 ^ k1;
    c0 = n0;
    c1 = loB;
    c2 = n2;
    c3 = loA;
    k0 += kWeylA;
    k1 += kWeylB;
  }
  Philox4 r;
  r.w[0] = c0;
  r.w[1] = c1;
  r.w[2] = c2;
  r.w[3] = c3;
  return r;
}

// Draw `draw` (0 = accept test, 1 = residual/bonus sample) of drafted position
// `position` of global request `request`: a 53-bit uniform on [0, 1) from the
// top 27 bits of word 0 and the top 26 bits of word 1 of
// Philox(counter = (2*position + draw, request, step, 0), key = seed).
__device__ __forceinline__ double draw_uniform(uint64_t seed, uint32_t request, uint32_t position,
                                               uint32_t draw, uint32_t step) {
  const Philox4 r = philox4x32_10(2u * position + draw, request, step, 0u,
                                  static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  const uint64_t bits = (static_cast<uint64_t>(r.w[0] >> 5) << 26) | (r.w[1] >> 6);
  return static_cast<double>(bits) * 0x1p-53;
}

}  // namespace sv
