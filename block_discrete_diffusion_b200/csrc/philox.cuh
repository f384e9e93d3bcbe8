// philox.cuh -- Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC'11) and the sampler's draws built on it.
//
// Stream layout (the pages name no generator; this is the build's stated reading): key = the 64-bit
// seed as (low word, high word); counter = (element index / 4, absolute position, step, tag), word
// = element index mod 4.  Tags: 0 Gumbel noise, 1 re-randomisation, 2 canvas initialisation.
#pragma once
#include <stdint.h>

namespace dg {

enum : uint32_t { RNG_TAG_GUMBEL = 0, RNG_TAG_RERAND = 1, RNG_TAG_INIT = 2 };

__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    // one 32 x 32 -> 64-bit product per multiplier gives both halves
    const uint64_t pa = (uint64_t)ctr.x * 0xD2511F53u;
    const uint64_t pc = (uint64_t)ctr.z * 0xCD9E8D57u;
    ctr = make_uint4((uint32_t)(pc >> 32) ^ ctr.y ^ k0, (uint32_t)pc, (uint32_t)(pa >> 32) ^ ctr.w ^ k1, (uint32_t)pa);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return ctr;
}

__device__ __forceinline__ uint4 rng_block(uint64_t seed, uint32_t c0, uint32_t pos, uint32_t step, uint32_t tag) {
  return philox4x32_10(make_uint4(c0, pos, step, tag), (uint32_t)seed, (uint32_t)(seed >> 32));
}

// Open-interval uniform (2*(x>>9)+1) * 2^-24, exact in fp32.
__device__ __forceinline__ float u01_open(uint32_t x) {
  return __uint2float_rn(((x >> 9) << 1) | 1u) * 5.9604644775390625e-08f;
}

// Standard Gumbel draw -log(-log u) with full-precision logf (u is within 2^-24 of 1 at the top).
__device__ __forceinline__ float gumbel_from_word(uint32_t x) {
  return -logf(-logf(u01_open(x)));
}

// Prefilter for the Gumbel-max: -__logf(-__logf(u)) with the hardware logarithm.  Below u = 0.999
// the documented __logf error bounds (absolute 2^-21.41 on [0.5, 2], 3 ulp elsewhere) keep it within
// 4e-4 of gumbel_from_word; kGumbelFastSlack covers that, so an element whose prefiltered score is
// more than the slack below the running best cannot reach it.  From u = 0.999 upwards (the largest
// draws) the accurate value is always taken.
constexpr float kGumbelFastSlack = 1e-3f;
constexpr float kGumbelFastMaxU = 0.999f;
__device__ __forceinline__ float gumbel_fast_from_u(float u) { return -__logf(-__logf(u)); }

// Largest Gumbel value any word can give, rounded up: -log(-log(1 - 2^-24)) = 16.6355...
constexpr float kGumbelMax = 16.6400f;

// Uniform id in [0, vocab): high 32 bits of x * vocab.
__device__ __forceinline__ int32_t token_from_word(uint32_t x, uint32_t vocab) {
  return (int32_t)__umulhi(x, vocab);
}

}  // namespace dg
