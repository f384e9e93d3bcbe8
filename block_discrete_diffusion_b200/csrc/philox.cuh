// philox.cuh -- Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC'11) and the sampler's draws built on it.
//
// Stream layout (the pages name no generator; this is the build's stated reading): key = the 64-bit
// seed as (low word, high word); counter = (element index / 4, absolute position, step, tag), word
// = element index mod 4.  Tags: 0 Gumbel noise, 1 re-randomisation, 2 canvas initialisation.
#pragma once
#include <stdint.h>

#include "dg_device.cuh"

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

// Open-interval uniform (2*(x>>9)+1) * 2^-24, exact in fp32: the float 1 + (x>>9) * 2^-23 built
// from its bits, minus 1 - 2^-24 (the two operands are within a factor of two, so the difference is
// exact).
__device__ __forceinline__ float u01_open(uint32_t x) {
  return __fsub_rn(__uint_as_float(0x3F800000u | (x >> 9)), __uint_as_float(0x3F7FFFFFu));
}

// Standard Gumbel draw -log(-log u) with full-precision logf (u is within 2^-24 of 1 at the top).
__device__ __forceinline__ float gumbel_from_word(uint32_t x) {
  return -logf(-logf(u01_open(x)));
}

// Screen for the Gumbel-max.  -ln(-ln u) = -ln(ln 2) - ln 2 * log2(-log2 u); with both base-2
// logarithms from lg2.approx (documented error: absolute 2^-22 on [0.5, 2], relative 2^-22
// elsewhere) and u < 0.999, the inner value is at least 1.44e-3, so it carries a relative error
// below 1.7e-4 and the screened draw is within 1.7e-4 + 2e-6 of gumbel_from_word.  Scores of
// tempered logits up to kScreenMaxZ in magnitude add at most three roundings of 6.2e-5 each, so
// the screened score plus kGumbelFastSlack is above the accurate score and less than two slacks
// below it.  Draws with u >= kGumbelFastMaxU and larger logits always take the accurate value.
constexpr float kGumbelFastSlack = 1e-3f;
constexpr float kGumbelFastMaxU = 0.999f;
constexpr float kScreenMaxZ = 1024.f;
constexpr float kNegLnLn2 = 0.36651292058166435f;   // -ln(ln 2)

// Screened score z + g + kGumbelFastSlack of an element with tempered logit l * inv_temp.
__device__ __forceinline__ float gumbel_screen_score(float l, float inv_temp, float u) {
  const float L = fast_log2(-fast_log2(u));
  return __fmaf_rn(-0.6931471805599453f, L, __fmaf_rn(l, inv_temp, kNegLnLn2 + kGumbelFastSlack));
}

// Largest Gumbel value any word can give, rounded up: -log(-log(1 - 2^-24)) = 16.6355...
constexpr float kGumbelMax = 16.6400f;

// Uniform id in [0, vocab): high 32 bits of x * vocab.
__device__ __forceinline__ int32_t token_from_word(uint32_t x, uint32_t vocab) {
  return (int32_t)__umulhi(x, vocab);
}

}  // namespace dg
