// expert_fp8.cu -- grouped expert GEMMs with both operands in e4m3 on the tensor cores
// (tcgen05.mma kind::f8f6f4): expert_f8_kernel for chunks of up to 32 tokens per expert (one or a few
// canvases), expert_f8_pair_kernel on CTA pairs for 256-token chunks (many canvases; further below).
//
// The FP8 form of the per-layer matrices stores e4m3 bytes q with one fp32 scale s_w per 128 x 128
// tile (w = q * s_w).  Here the activations are e4m3 too, with one fp32 scale per token and per
// block of channels: the gathered rows (gate|up input) per 128 channels, the SwiGLU rows (down input)
// per 64 features, s = amax / 448.  A tile's MMAs over one scale block give sum q_w q_a; that partial
// sum is scaled by s_w * s_a and added to an fp32 accumulator.  So the K loop is split into slices
// (128 deep for gate|up, 64 for down): the MMA warp multiplies each slice into one of sixteen TMEM
// buffers and the epilogue warps promote it into registers (thread = weight row, 32 token columns),
// while the next slices run.  Against the bf16 path this halves the weight bytes streamed from HBM
// (the bound at these token counts) and needs no expansion of the weights to bf16.
//
// Roles (320 threads): warp 0 TMA producer (e4m3 weight tile 128 rows x 128 bytes and the chunk's
// 32 token rows x 128 bytes per stage, 128-byte swizzle), warp 1 MMA issuer, warps 2-9 promotion and
// epilogue (two warps per TMEM lane quadrant, 16 token columns each; per chunk one table of the
// combined scales s_w * s_a, so a slice costs a TMEM load and one FMA per column).  MODE 1: gate|up rows of one expert (64 + 64 rows) times its tokens, SwiGLU in the
// epilogue, the result quantized per (token, 64 features) to e4m3 for the down GEMM; MODE 2: down
// rows (128) times the tokens' SwiGLU rows, fp32 outputs for the combine.
//
// The activation quantization is this kernel's reading of the FP8 form: the pages' H100 numbers are
// FP8 at batch 1 ("Numbers: speed vs accuracy" in the technical-report summary), and the weights'
// per-tile scales are fp32 (not the power-of-two block scales the hardware's block-scaled MMA takes),
// so the scales are applied in the epilogue per slice.
#include <cuda_fp8.h>
#include <stdio.h>

#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int kF8Threads = 320;                    // warps 0 (TMA), 1 (MMA), 2-9 (promotion + epilogue)
constexpr int kF8EpiThreads = 256;
constexpr int kF8BN = 32;                          // token columns per chunk
constexpr uint32_t kF8WTile = 128 * 128;           // 128 weight rows x 128 bytes of K
constexpr uint32_t kF8XTile = kF8BN * 128;         // 32 token rows x 128 bytes of K
constexpr uint32_t kF8Stage = kF8WTile + kF8XTile;
constexpr int kF8Stages = 8;
constexpr int kF8Slices = 16;                      // TMEM slice buffers of 32 columns (all 512 columns): the
                                                   // MMAs run up to 16 slices ahead of the promotion
constexpr int kF8MaxSl = 64;                       // scale blocks per token row (d / 128 or F / 64)
constexpr int kF8EpiStride = kF8BN + 1;
constexpr size_t kF8Smem = 1024 + (size_t)kF8Stages * kF8Stage + 128 * kF8EpiStride * 4 +
                           2 * (size_t)kF8BN * kF8MaxSl * 4 + 512;
static_assert(kF8Smem <= 232448, "shared memory budget");

struct F8Barriers {
  uint64_t full[kF8Stages];
  uint64_t empty[kF8Stages];
  uint64_t sfull[kF8Slices];
  uint64_t sempty[kF8Slices];
  uint32_t tmem_slot;
};

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format 0), fp32 D, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B^T with e4m3 operands (32 K per instruction), fp32 accumulation; one thread issues.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void f8_epi_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// 32 lanes x 16 consecutive fp32 columns of TMEM (thread `lane` of warp w: lane 32 (w % 4) + lane).
__device__ __forceinline__ void tmem_ld_16cols(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 columns of TMEM into registers without waiting (tmem_wait_ld16 completes the loads).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld16() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Two floats to two e4m3 bytes (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

template <int MODE>
__global__ void __launch_bounds__(kF8Threads, 1)
    expert_f8_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     ExpertParams p, int n_exp, int* err) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* stage_out = reinterpret_cast<float*>(tiles + (size_t)kF8Stages * kF8Stage);
  // [2][kF8MaxSl][32 tokens] combined scales s_w * s_a per (weight-row half, slice, token) of a chunk
  float* cs_s = stage_out + 128 * kF8EpiStride;
  F8Barriers* bars = reinterpret_cast<F8Barriers*>(cs_s + 2 * kF8BN * kF8MaxSl);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = MODE == 1 ? p.d : p.F;
  const int nkb = (K + 127) / 128;                              // 128-byte K stages
  const int nsl = MODE == 1 ? K / 128 : (K + 63) / 64;          // promotion slices (= activation scale blocks)
  const int MT = MODE == 1 ? p.F / 64 : p.d / 128;              // weight tiles per expert
  const int n_items = n_exp * MT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kF8Stages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < kF8Slices; ++s) {
      mbar_init(&bars->sfull[s], 1);
      mbar_init(&bars->sempty[s], 8);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_slot, kF8Slices * kF8BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  pdl_wait();   // routing, the quantized activation rows and their scales come from the preceding kernels

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();   // every weight tile is read once
      uint32_t it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int e = item / MT, mt = item % MT;
        const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
        for (int c0 = 0; c0 < n_e && ok; c0 += kF8BN) {
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % kF8Stages;
            if (!mbar_wait(&bars->empty[s], ((it / kF8Stages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) {
              ok = false;
              break;
            }
            uint8_t* a = tiles + (size_t)s * kF8Stage;
            mbar_arrive_expect_tx(&bars->full[s], kF8Stage);
            if (MODE == 1) {
              const int r0 = e * 2 * p.F + mt * 64;
              tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 128, r0, pol_w);                  // gate rows
              tma_load_2d_hint(&tmW, &bars->full[s], a + kF8WTile / 2, kb * 128, r0 + p.F, pol_w);  // up rows
            } else {
              tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 128, e * p.d + mt * 128, pol_w);
            }
            tma_load_2d(&tmX, &bars->full[s], a + kF8WTile, kb * 128, off + c0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      uint32_t it = 0, g = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int e = item / MT;
        const int n_e = p.offsets[e + 1] - p.offsets[e];
        for (int c0 = 0; c0 < n_e && ok; c0 += kF8BN) {
          const int nmma = (min(kF8BN, n_e - c0) + 15) & ~15;
          const uint32_t idesc = idesc_e4m3_f32(128, nmma);
          for (int kb = 0; kb < nkb && ok; ++kb, ++it) {
            const int s = it % kF8Stages;
            if (!mbar_wait(&bars->full[s], (it / kF8Stages) & 1, err, DEV_ERR_TIMEOUT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* a = tiles + (size_t)s * kF8Stage;
            const uint64_t ad = smem_desc_sw128(smem_u32(a));
            const uint64_t bd = smem_desc_sw128(smem_u32(a + kF8WTile));
            // MODE 1: one 128-deep slice per stage; MODE 2: two 64-deep slices (the second of the last
            // stage lies past F when F % 128 == 64: no slice)
            const int per = MODE == 1 ? 1 : 2;
            for (int h = 0; h < per; ++h) {
              if (kb * per + h >= nsl) break;
              const uint32_t b = g % kF8Slices;
              if (!mbar_wait(&bars->sempty[b], ((g / kF8Slices) & 1) ^ 1, err, DEV_ERR_TIMEOUT_MMA)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t acc = tmem + b * kF8BN;
              constexpr int kSteps = MODE == 1 ? 4 : 2;        // 32 K per instruction
#pragma unroll
              for (int k = 0; k < kSteps; ++k)
                umma_e4m3(acc, desc_advance(ad, (h * kSteps + k) * 32), desc_advance(bd, (h * kSteps + k) * 32), idesc,
                          k != 0);
              umma_commit(&bars->sfull[b]);
              ++g;
            }
            umma_commit(&bars->empty[s]);
          }
        }
      }
    }
  } else {
    // ------------------------------ promotion + epilogue (warps 2-9) ------------------------------
    // Warps w and w + 4 read the same TMEM lanes (weight rows 32 (w % 4) ..) and split the chunk's 32
    // token columns: columns 16 ch .. 16 ch + 15 with ch = (w - 2) / 4.
    const int quarter = warp & 3;                 // TMEM lanes [32 quarter, 32 quarter + 32)
    const int ch = (warp - 2) >> 2;               // token-column half
    const int r = quarter * 32 + lane;            // weight row of the tile
    const int et = threadIdx.x - 64;              // 0..255 among the epilogue threads
    const int half_row = MODE == 1 && r >= 64 ? 1 : 0;   // gate (0) or up (1) rows in MODE 1
    uint32_t g = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int e = item / MT, mt = item % MT;
      const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
      const int nwb = p.w_scale_cols;
      for (int c0 = 0; c0 < n_e; c0 += kF8BN) {
        const int nc = min(kF8BN, n_e - c0);
        f8_epi_sync();                            // the previous chunk is done with cs_s and stage_out
        // combined scale s_w(half, K block of the slice) * s_a(token, slice), once per chunk, off the
        // per-slice path
        const int halves = MODE == 1 ? 2 : 1;
        for (int i = et; i < halves * nsl * kF8BN; i += kF8EpiThreads) {
          const int n = i % kF8BN, sl = (i / kF8BN) % nsl, hf = i / (kF8BN * nsl);
          const int srow = MODE == 1 ? (e * 2 * p.F + hf * p.F + mt * 64) / 128 : (e * p.d + mt * 128) / 128;
          const int kb = MODE == 1 ? sl : sl >> 1;
          const float sw = kb < nwb ? __ldg(p.w_scale + (size_t)srow * nwb + kb) : 0.f;
          const float sa = n < nc ? __ldg(p.a_scale + (size_t)(off + c0 + n) * p.a_scale_cols + sl) : 0.f;
          cs_s[(hf * kF8MaxSl + sl) * kF8BN + n] = sw * sa;
        }
        f8_epi_sync();
        const float* cs_row = cs_s + (size_t)half_row * kF8MaxSl * kF8BN + ch * 16;
        float acc[16];
#pragma unroll
        for (int n = 0; n < 16; ++n) acc[n] = 0.f;
        for (int sl = 0; sl < nsl; ++sl, ++g) {
          const uint32_t b = g % kF8Slices;
          ok = ok && mbar_wait(&bars->sfull[b], (g / kF8Slices) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
          tc_fence_after();
          float v[16];
          tmem_ld_16cols(tmem + ((uint32_t)(quarter * 32) << 16) + b * kF8BN + ch * 16, v);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sempty[b]);
          const float4* c4 = reinterpret_cast<const float4*>(cs_row + sl * kF8BN);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 c = c4[q4];
            acc[4 * q4 + 0] = __fmaf_rn(v[4 * q4 + 0], c.x, acc[4 * q4 + 0]);
            acc[4 * q4 + 1] = __fmaf_rn(v[4 * q4 + 1], c.y, acc[4 * q4 + 1]);
            acc[4 * q4 + 2] = __fmaf_rn(v[4 * q4 + 2], c.z, acc[4 * q4 + 2]);
            acc[4 * q4 + 3] = __fmaf_rn(v[4 * q4 + 3], c.w, acc[4 * q4 + 3]);
          }
        }
        if (MODE == 2) {
          if (ok) {
            const int m = mt * 128 + r;           // output feature of the down projection
#pragma unroll
            for (int n = 0; n < 16; ++n)
              if (ch * 16 + n < nc) p.y_out[(size_t)(off + c0 + ch * 16 + n) * p.d + m] = acc[n];
          }
        } else {
          // gate rows 0-63, up rows 64-127: SwiGLU of (row f, row 64 + f) through shared memory
#pragma unroll
          for (int n = 0; n < 16; ++n) stage_out[r * kF8EpiStride + ch * 16 + n] = acc[n];
          f8_epi_sync();
          // thread -> token n = et / 8, features fq .. fq + 7 with fq = 8 (et % 8); the 8 threads of a
          // token (adjacent lanes) share the amax of its 64 features
          const int n = et >> 3, fq = (et & 7) * 8;
          float h[8];
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float gg = stage_out[(fq + i) * kF8EpiStride + n], uu = stage_out[(64 + fq + i) * kF8EpiStride + n];
            h[i] = gg / (1.f + __expf(-gg)) * uu;
            amax = fmaxf(amax, fabsf(h[i]));
          }
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
          const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
          if (ok && n < nc) {
            const uint32_t q0 = e4m3x2(h[0] * inv, h[1] * inv) | (e4m3x2(h[2] * inv, h[3] * inv) << 16);
            const uint32_t q1 = e4m3x2(h[4] * inv, h[5] * inv) | (e4m3x2(h[6] * inv, h[7] * inv) << 16);
            const size_t row = (size_t)(off + c0 + n);
            *reinterpret_cast<uint2*>(p.hq_out + row * p.F + mt * 64 + fq) = make_uint2(q0, q1);
            if ((et & 7) == 0) p.hs_out[row * (p.F / 64) + mt] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kF8Slices * kF8BN);
}

// xq[slot[t*k + r]] = e4m3(xn[t] / s), xs[slot[t*k + r]][b] = s = amax / 448 of channel block b (128
// channels) of the row: one warp per (token, block) -- many independent warps, so the loads of all
// blocks are in flight at once -- writes the block's k copies.
// The normed row's 4 values at column c of row t: read from xn, or formed as bf16(x * r * g) (the
// FFN RMSNorm folded into the gather, the product order of the RMSNorm kernel).
template <bool FROM_X>
__global__ void gather_rows_q8_kernel(const __nv_bfloat16* __restrict__ xn, const float* __restrict__ x,
                                      const float* __restrict__ rr, const float* __restrict__ g,
                                      const int32_t* __restrict__ slot, int n_rows, int top_k, int d,
                                      uint8_t* __restrict__ xq, float* __restrict__ xs) {
  pdl_trigger();
  pdl_wait();
  const int nblk = d / 128;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= n_rows * nblk) return;
  const int t = wid / nblk, b = wid % nblk;
  const int my_slot = lane < top_k ? slot[(size_t)t * top_k + lane] : 0;
  const int c = b * 128 + lane * 4;
  float v0, v1, v2, v3;
  if constexpr (FROM_X) {
    const float r = rr[t];
    const float4 xv = *reinterpret_cast<const float4*>(x + (size_t)t * d + c);
    const float4 gv = __ldg(reinterpret_cast<const float4*>(g + c));
    v0 = __bfloat162float(__float2bfloat16_rn(xv.x * r * gv.x));
    v1 = __bfloat162float(__float2bfloat16_rn(xv.y * r * gv.y));
    v2 = __bfloat162float(__float2bfloat16_rn(xv.z * r * gv.z));
    v3 = __bfloat162float(__float2bfloat16_rn(xv.w * r * gv.w));
  } else {
    const uint2 raw = *reinterpret_cast<const uint2*>(xn + (size_t)t * d + c);
    const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    v0 = __low2float(p0); v1 = __high2float(p0); v2 = __low2float(p1); v3 = __high2float(p1);
  }
  const float amax = warp_max(fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3))));
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const uint32_t q = e4m3x2(v0 * inv, v1 * inv) | (e4m3x2(v2 * inv, v3 * inv) << 16);
  for (int rr = 0; rr < top_k; ++rr) {
    const int row = __shfl_sync(0xffffffffu, my_slot, rr);
    *reinterpret_cast<uint32_t*>(xq + (size_t)row * d + b * 128 + lane * 4) = q;
    if (lane == 0) xs[(size_t)row * nblk + b] = sc;
  }
}

// ---------------------------------------------------------------------------------------------
// Many tokens per expert (several canvases): CTA pairs
// ---------------------------------------------------------------------------------------------
// With hundreds of tokens per expert the product is bound by the tensor cores, so the tile grows to
// 256 tokens x 256 weight rows on a CTA pair (tcgen05 cta_group::2, M = 256): the tokens are the M
// side (128 rows in each CTA), the weight rows the N side, half in each CTA -- MODE 1: the gate rows of
// 128 features in the leader and the up rows of the same features in the peer, so that one
// accumulator row holds both halves of every SwiGLU feature; MODE 2: 128 output features in each.
// Thread = token row, so a slice's activation scale is one number per thread and its weight scale one
// number per block of columns: the promotion is one FMA per accumulator element, and the
// accumulators (128 per thread) stay in registers.  Two TMEM slice buffers of 256 columns: the MMAs
// of one slice overlap the promotion of the other.  Work items are (expert, weight tile, 256-token
// chunk), chunks innermost, so that the chunks of one weight tile run at the same time on
// neighbouring pairs and share its HBM read through L2.
constexpr int kFpThreads = 320;                // warp 0 TMA (both CTAs), warp 1 MMA (leader), warps 2-9 promotion
constexpr int kFpStages = 6;
constexpr uint32_t kFpATile = 128 * 128;       // 128 token rows x 128 bytes of K
constexpr uint32_t kFpBTile = 128 * 128;       // up to 128 weight rows x 128 bytes of K
constexpr uint32_t kFpStage = kFpATile + kFpBTile;
constexpr int kFpMaxExp = 256;
constexpr int kFpCumInts = (kFpMaxExp + 1 + 3) / 4 * 4;   // the barriers after them stay 16-byte aligned
constexpr size_t kFpSmem = 1024 + (size_t)kFpStages * kFpStage + 2 * 128 * 4 + kFpCumInts * 4 + 256;
static_assert(kFpSmem <= 232448, "shared memory budget");

struct FpBarriers {
  uint64_t full[kFpStages];
  uint64_t empty[kFpStages];
  uint64_t sfull[2];
  uint64_t sempty[2];
  uint32_t tmem_slot;
};

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFpThreads, 1)
    expert_f8_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                          ExpertParams p, int n_exp, int* err) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* amx = reinterpret_cast<float*>(tiles + (size_t)kFpStages * kFpStage);   // [2][128]: half-block amax
  int* s_cum = reinterpret_cast<int*>(amx + 256);                                // first item of each expert
  FpBarriers* bars = reinterpret_cast<FpBarriers*>(s_cum + kFpCumInts);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();       // 0: leader, 1: peer
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int K = MODE == 1 ? p.d : p.F;
  const int nkb = (K + 127) / 128;                              // 128-byte K stages
  const int nsl = MODE == 1 ? K / 128 : (K + 63) / 64;          // promotion slices (= activation scale blocks)
  const int NT = MODE == 1 ? (p.F + 127) / 128 : p.d / 256;     // weight tiles per expert

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFpStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->sfull[b], 1);
      mbar_init(&bars->sempty[b], 16);          // the promotion warps of both CTAs
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(&bars->tmem_slot, 512);
  tc_fence_before();
  cluster_sync();                               // both CTAs' barriers and tensor memory exist
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  const uint32_t lead_full0 = dsmem_map(smem_u32(&bars->full[0]), 0);
  const uint32_t lead_sempty0 = dsmem_map(smem_u32(&bars->sempty[0]), 0);
  pdl_wait();   // routing, the quantized activation rows and their scales come from the preceding kernels

  // items per expert: NT weight tiles x ceil(n_e / 256) chunks; s_cum = exclusive prefix over experts
  if (warp == 2) {
    int run = 0;
    for (int e0 = 0; e0 < n_exp; e0 += 32) {
      const int e = e0 + lane;
      const int v = e < n_exp ? NT * ((p.offsets[e + 1] - p.offsets[e] + 255) / 256) : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < n_exp) s_cum[e] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_cum[n_exp] = run;
  }
  __syncthreads();
  const int n_items = s_cum[n_exp];
  int ecur = 0;
  // item -> expert e, weight tile t, chunk c (items increase along every role's walk)
  auto decode = [&](int item, int& e, int& t, int& c) {
    while (s_cum[ecur + 1] <= item) ++ecur;
    e = ecur;
    const int nch = (p.offsets[e + 1] - p.offsets[e] + 255) / 256;
    t = (item - s_cum[e]) / nch;
    c = (item - s_cum[e]) % nch;
  };

  if (warp == 0) {
    // ------------------------------ TMA producer (both CTAs) ------------------------------
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();   // token rows and weight tiles are each read by several items
      uint32_t it = 0;
      bool ok = true;
      for (int item = pair; item < n_items && ok; item += n_pairs) {
        int e, t, c;
        decode(item, e, t, c);
        const int nf = MODE == 1 ? min(128, p.F - t * 128) : 128;   // weight rows this CTA holds
        const int tok0 = p.offsets[e] + c * 256 + (int)rank * 128;
        const int wrow = MODE == 1 ? e * 2 * p.F + (int)rank * p.F + t * 128 : e * p.d + t * 256 + (int)rank * 128;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kFpStages;
          if (!mbar_wait(&bars->empty[s], ((it / kFpStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* a = tiles + (size_t)s * kFpStage;
          if (rank == 0) mbar_arrive_expect_tx(&bars->full[s], 2 * (kFpATile + (uint32_t)nf * 128));
          const uint32_t bar = lead_full0 + (uint32_t)(s * sizeof(uint64_t));
#pragma unroll
          for (int q = 0; q < 4; ++q) tma_load_2d_pair(&tmX, bar, a + q * 4096, kb * 128, tok0 + q * 32, pol);
          if (MODE == 1) {
            for (int h = 0; h < nf / 64; ++h)
              tma_load_2d_pair(&tmW, bar, a + kFpATile + h * 8192, kb * 128, wrow + h * 64, pol);
          } else {
            tma_load_2d_pair(&tmW, bar, a + kFpATile, kb * 128, wrow, pol);
          }
        }
      }
      // tail: every stage released once more, i.e. the leader's last commits (multicast to this CTA)
      // have arrived here before the CTA may leave
      for (int i = 0; i < kFpStages && ok; ++i, ++it)
        ok = mbar_wait(&bars->empty[it % kFpStages], ((it / kFpStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader) ------------------------------
    if (rank == 0 && lane == 0) {
      uint32_t it = 0, g = 0;
      bool ok = true;
      for (int item = pair; item < n_items && ok; item += n_pairs) {
        int e, t, c;
        decode(item, e, t, c);
        const int nf = MODE == 1 ? min(128, p.F - t * 128) : 128;
        const uint32_t idesc = idesc_e4m3_f32(256, 2 * nf);
        for (int kb = 0; kb < nkb && ok; ++kb, ++it) {
          const int s = it % kFpStages;
          if (!mbar_wait(&bars->full[s], (it / kFpStages) & 1, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* a = tiles + (size_t)s * kFpStage;
          const uint64_t ad = smem_desc_sw128(smem_u32(a));
          const uint64_t bd = smem_desc_sw128(smem_u32(a + kFpATile));
          // MODE 1: one 128-deep slice per stage; MODE 2: two 64-deep slices (none past F)
          const int per = MODE == 1 ? 1 : 2;
          for (int h = 0; h < per; ++h) {
            if (kb * per + h >= nsl) break;
            const uint32_t b = g & 1;
            if (!mbar_wait(&bars->sempty[b], ((g >> 1) & 1) ^ 1, err, DEV_ERR_TIMEOUT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            constexpr int kSteps = MODE == 1 ? 4 : 2;        // 32 K per instruction
#pragma unroll
            for (int k = 0; k < kSteps; ++k)
              umma_e4m3_pair(tmem + b * 256, desc_advance(ad, (h * kSteps + k) * 32), desc_advance(bd, (h * kSteps + k) * 32),
                             idesc, k != 0);
            umma_commit_pair(&bars->sfull[b]);
            ++g;
          }
          umma_commit_pair(&bars->empty[s]);
        }
      }
    }
  } else {
    // ------------------------------ promotion + epilogue (warps 2-9 of both CTAs) ------------------------------
    // Warps w and w + 4 read TMEM lanes 32 (w % 4) .. (token rows of this CTA) and split the columns:
    // MODE 1 the gate columns [ch nf/2, (ch + 1) nf/2) and the matching up columns nf + ..., MODE 2
    // the output columns [128 ch, 128 ch + 128).
    const int q = warp & 3, ch = (warp - 2) >> 2;
    const int lrow = q * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    const int nwb = p.w_scale_cols;
    uint32_t g = 0;
    bool ok = true;
    for (int item = pair; item < n_items; item += n_pairs) {
      int e, t, c;
      decode(item, e, t, c);
      const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
      const int nf = MODE == 1 ? min(128, p.F - t * 128) : 128;
      const int half = nf / 2;                   // MODE 1: SwiGLU features of this thread
      const int tl = c * 256 + (int)rank * 128 + lrow;
      const bool valid = tl < n_e;
      const size_t token = (size_t)(off + (valid ? tl : 0));
      // scale rows (128-row tiles of the weight matrix) of this thread's column blocks
      const int r0 = MODE == 1 ? (e * 2 * p.F + t * 128 + ch * half) / 128 : (e * p.d + t * 256 + ch * 128) / 128;
      const int r1 = MODE == 1 ? (e * 2 * p.F + p.F + t * 128 + ch * half) / 128 : r0;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      // the scales of slice sl + 1 are loaded while slice sl is promoted
      const float* pa = p.a_scale + token * p.a_scale_cols;
      const float* pw0 = p.w_scale + (size_t)r0 * nwb;
      const float* pw1 = p.w_scale + (size_t)r1 * nwb;
      float sa_n = valid ? __ldg(pa) : 0.f, sw0_n = __ldg(pw0), sw1_n = MODE == 1 ? __ldg(pw1) : 0.f;
      for (int sl = 0; sl < nsl; ++sl, ++g) {
        const float sa = sa_n, sw0 = sw0_n, sw1 = sw1_n;
        if (sl + 1 < nsl) {
          const int kb1 = MODE == 1 ? sl + 1 : (sl + 1) >> 1;
          sa_n = valid ? __ldg(pa + sl + 1) : 0.f;
          sw0_n = __ldg(pw0 + kb1);
          if (MODE == 1) sw1_n = __ldg(pw1 + kb1);
        }
        const float c0s = sw0 * sa;
        const float c1s = MODE == 1 ? sw1 * sa : 0.f;
        const uint32_t b = g & 1;
        ok = ok && mbar_wait(&bars->sfull[b], (g >> 1) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
        tc_fence_after();
        const uint32_t ta = tq + b * 256;
        // two 16-column TMEM loads in flight per wait: the 128 accumulators and 32 loaded values fit the
        // registers, and a slice takes four load round trips
        if (MODE == 1) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j * 16 < half) {
              uint32_t v[2][16];
              tmem_ld16_nowait(ta + ch * half + j * 16, v[0]);
              tmem_ld16_nowait(ta + nf + ch * half + j * 16, v[1]);
              tmem_wait_ld16();
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                acc[j * 16 + i] = __fmaf_rn(__uint_as_float(v[0][i]), c0s, acc[j * 16 + i]);
                acc[64 + j * 16 + i] = __fmaf_rn(__uint_as_float(v[1][i]), c1s, acc[64 + j * 16 + i]);
              }
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            uint32_t v[2][16];
            tmem_ld16_nowait(ta + ch * 128 + j * 16, v[0]);
            tmem_ld16_nowait(ta + ch * 128 + j * 16 + 16, v[1]);
            tmem_wait_ld16();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              acc[j * 16 + i] = __fmaf_rn(__uint_as_float(v[0][i]), c0s, acc[j * 16 + i]);
              acc[j * 16 + 16 + i] = __fmaf_rn(__uint_as_float(v[1][i]), c0s, acc[j * 16 + 16 + i]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(lead_sempty0 + b * (uint32_t)sizeof(uint64_t));
      }
      if (MODE == 2) {
        if (ok && valid) {
          float4* dst = reinterpret_cast<float4*>(p.y_out + token * p.d + t * 256 + ch * 128);
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        }
      } else {
        // SwiGLU of this thread's features (gate acc[i], up acc[64 + i]), e4m3 per (token, 64 features)
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          if (i < half) {
            const float gg = acc[i], uu = acc[64 + i];
            acc[i] = gg / (1.f + __expf(-gg)) * uu;
            amax = fmaxf(amax, fabsf(acc[i]));
          }
        }
        if (half < 64) {
          // the 64-feature block is shared with warp w ^ 4 (same token rows, the other half): exchange
          amx[ch * 128 + lrow] = amax;
          f8_epi_sync();
          amax = fmaxf(amax, amx[(ch ^ 1) * 128 + lrow]);
          f8_epi_sync();
        }
        const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
        if (ok && valid) {
          const int f0 = t * 128 + ch * half;      // first feature of this thread
          uint8_t* dst = p.hq_out + token * p.F + f0;
#pragma unroll
          for (int i = 0; i < 64; i += 16) {
            if (i < half) {
              uint4 w;
              w.x = e4m3x2(acc[i] * inv, acc[i + 1] * inv) | (e4m3x2(acc[i + 2] * inv, acc[i + 3] * inv) << 16);
              w.y = e4m3x2(acc[i + 4] * inv, acc[i + 5] * inv) | (e4m3x2(acc[i + 6] * inv, acc[i + 7] * inv) << 16);
              w.z = e4m3x2(acc[i + 8] * inv, acc[i + 9] * inv) | (e4m3x2(acc[i + 10] * inv, acc[i + 11] * inv) << 16);
              w.w = e4m3x2(acc[i + 12] * inv, acc[i + 13] * inv) | (e4m3x2(acc[i + 14] * inv, acc[i + 15] * inv) << 16);
              *reinterpret_cast<uint4*>(dst + i) = w;
            }
          }
          if (half == 64 || ch == 0) p.hs_out[token * (p.F / 64) + f0 / 64] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync();                               // no CTA leaves while the pair's MMAs or arrivals may touch it
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

template <int MODE>
cudaError_t launch_f8_pair(const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp, int n_ctas,
                           int* err, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(expert_f8_pair_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kFpSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(expert_f8_pair_kernel<MODE>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_ctas & ~1);
  cfg.blockDim = dim3(kFpThreads);
  cfg.dynamicSmemBytes = kFpSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, expert_f8_pair_kernel<MODE>, w, x, p, n_exp, err);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    // say which resource the launch exceeded
    cudaFuncAttributes fa{};
    cudaGetLastError();
    if (cudaFuncGetAttributes(&fa, expert_f8_pair_kernel<MODE>) == cudaSuccess) {
      fprintf(stderr, "expert_f8_pair_kernel<%d>: %s (registers %d, max threads %d, static smem %zu, dynamic %zu)\n",
              MODE, cudaGetErrorString(e), fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes, kFpSmem);
    }
  }
  return e;
}

template <int MODE>
cudaError_t launch_f8(const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp, int n_ctas,
                      int* err, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(expert_f8_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kF8Smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(expert_f8_kernel<MODE>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int items = n_exp * (MODE == 1 ? p.F / 64 : p.d / 128);
  return launch_k(expert_f8_kernel<MODE>, dim3(n_ctas < items ? n_ctas : items), dim3(kF8Threads), kF8Smem, st, 1, w,
                  x, p, n_exp, err);
}

}  // namespace

cudaError_t gather_rows_q8(const GatherSrc& src, const int32_t* slot, int n_rows, int top_k, int d, uint8_t* xq,
                           float* xs, cudaStream_t st) {
  if (d % 128 || top_k > 32 || (!src.xn && (!src.x || !src.r || !src.g))) return cudaErrorInvalidValue;
  const int warps = n_rows * (d / 128);
  if (src.xn)
    return launch_k(gather_rows_q8_kernel<false>, dim3((warps + 7) / 8), dim3(256), 0, st, 1, src.xn, src.x, src.r,
                    src.g, slot, n_rows, top_k, d, xq, xs);
  return launch_k(gather_rows_q8_kernel<true>, dim3((warps + 7) / 8), dim3(256), 0, st, 1, src.xn, src.x, src.r, src.g,
                  slot, n_rows, top_k, d, xq, xs);
}

cudaError_t gemm_expert_f8_pair(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p,
                                int n_exp, int n_ctas, int* err, cudaStream_t st) {
  if (!p.w_scale || !p.a_scale || !p.offsets || n_exp <= 0 || n_exp > kFpMaxExp || n_ctas < 2) return cudaErrorInvalidValue;
  if (mode == 1 && (p.d % 128 || p.F % 64 || p.a_scale_cols != p.d / 128 || !p.hq_out || !p.hs_out))
    return cudaErrorInvalidValue;
  if (mode == 2 && (p.d % 256 || p.F % 64 || p.a_scale_cols != p.F / 64 || !p.y_out)) return cudaErrorInvalidValue;
  return mode == 1 ? launch_f8_pair<1>(w, x, p, n_exp, n_ctas, err, st) : launch_f8_pair<2>(w, x, p, n_exp, n_ctas, err, st);
}

cudaError_t gemm_expert_f8(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                           int n_ctas, int* err, cudaStream_t st) {
  if (!p.w_scale || !p.a_scale) return cudaErrorInvalidValue;
  if (mode == 1 && (p.d % 128 || p.d / 128 > kF8MaxSl || p.F % 64 || !p.hq_out || !p.hs_out))
    return cudaErrorInvalidValue;
  if (mode == 2 && (p.F % 64 || (p.F + 63) / 64 > kF8MaxSl || p.d % 128 || !p.y_out)) return cudaErrorInvalidValue;
  return mode == 1 ? launch_f8<1>(w, x, p, n_exp, n_ctas, err, st) : launch_f8<2>(w, x, p, n_exp, n_ctas, err, st);
}

}  // namespace dg
