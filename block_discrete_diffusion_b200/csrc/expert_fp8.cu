// expert_fp8.cu -- grouped expert GEMMs with both operands in e4m3 on the tensor cores
// (tcgen05.mma kind::f8f6f4), for chunks of up to 32 tokens per expert (one or a few canvases).
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
// Roles (192 threads): warp 0 TMA producer (e4m3 weight tile 128 rows x 128 bytes and the chunk's
// 32 token rows x 128 bytes per stage, 128-byte swizzle), warp 1 MMA issuer, warps 2-5 promotion and
// epilogue.  MODE 1: gate|up rows of one expert (64 + 64 rows) times its tokens, SwiGLU in the
// epilogue, the result quantized per (token, 64 features) to e4m3 for the down GEMM; MODE 2: down
// rows (128) times the tokens' SwiGLU rows, fp32 outputs for the combine.
//
// The activation quantization is this kernel's reading of the FP8 form: the pages' H100 numbers are
// FP8 at batch 1 ("Numbers: speed vs accuracy" in the technical-report summary), and the weights'
// per-tile scales are fp32 (not the power-of-two block scales the hardware's block-scaled MMA takes),
// so the scales are applied in the epilogue per slice.
#include <cuda_fp8.h>

#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int kF8Threads = 192;
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
                           (size_t)kF8BN * kF8MaxSl * 4 + 2 * 32 * 4 + 512;
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

__device__ __forceinline__ void f8_epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

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
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* stage_out = reinterpret_cast<float*>(tiles + (size_t)kF8Stages * kF8Stage);
  float* sa_s = stage_out + 128 * kF8EpiStride;                 // [32 tokens][kF8MaxSl] activation scales
  float* sw_s = sa_s + kF8BN * kF8MaxSl;                        // [2][32] the item's weight scales per K block
  F8Barriers* bars = reinterpret_cast<F8Barriers*>(sw_s + 2 * 32);
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
      mbar_init(&bars->sempty[s], 4);
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
    // ------------------------------ promotion + epilogue (warps 2-5) ------------------------------
    const int quarter = warp & 3;                 // TMEM lanes [32 quarter, 32 quarter + 32)
    const int r = quarter * 32 + lane;            // weight row of the tile
    const int et = threadIdx.x - 64;              // 0..127 among the epilogue threads
    uint32_t g = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int e = item / MT, mt = item % MT;
      const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
      // weight scales of the item per K block (MODE 1: the gate half [0] and the up half [1] sit in
      // different 128-row tiles) and the chunk's activation scales go to shared memory once, off the
      // per-slice path
      const int nwb = p.w_scale_cols;
      for (int c0 = 0; c0 < n_e; c0 += kF8BN) {
        const int nc = min(kF8BN, n_e - c0);
        f8_epi_sync();                            // the previous chunk is done with sa_s, sw_s and stage_out
        for (int i = et; i < kF8BN * nsl; i += 128) {
          const int n = i / nsl, b = i % nsl;
          sa_s[n * kF8MaxSl + b] = n < nc ? __ldg(p.a_scale + (size_t)(off + c0 + n) * p.a_scale_cols + b) : 0.f;
        }
        if (et < 2 * 32) {
          const int half = et >> 5, b = et & 31;
          const int srow = MODE == 1 ? (e * 2 * p.F + half * p.F + mt * 64) / 128 : (e * p.d + mt * 128) / 128;
          sw_s[et] = b < nwb ? __ldg(p.w_scale + (size_t)srow * nwb + b) : 0.f;
        }
        f8_epi_sync();
        const float* sw_row = sw_s + (MODE == 1 && r >= 64 ? 32 : 0);
        float acc[kF8BN];
#pragma unroll
        for (int n = 0; n < kF8BN; ++n) acc[n] = 0.f;
        for (int sl = 0; sl < nsl; ++sl, ++g) {
          const uint32_t b = g % kF8Slices;
          ok = ok && mbar_wait(&bars->sfull[b], (g / kF8Slices) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
          tc_fence_after();
          float v[32];
          tmem_ld_32cols(tmem + ((uint32_t)(quarter * 32) << 16) + b * kF8BN, v);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->sempty[b]);
          const float sw = sw_row[MODE == 1 ? sl : sl >> 1];
#pragma unroll
          for (int n = 0; n < kF8BN; ++n) acc[n] = __fmaf_rn(v[n], sw * sa_s[n * kF8MaxSl + sl], acc[n]);
        }
        if (MODE == 2) {
          if (ok) {
            const int m = mt * 128 + r;           // output feature of the down projection
#pragma unroll
            for (int n = 0; n < kF8BN; ++n)
              if (n < nc) p.y_out[(size_t)(off + c0 + n) * p.d + m] = acc[n];
          }
        } else {
          // gate rows 0-63, up rows 64-127: SwiGLU of (row f, row 64 + f) through shared memory
#pragma unroll
          for (int n = 0; n < kF8BN; ++n) stage_out[r * kF8EpiStride + n] = acc[n];
          f8_epi_sync();
          // thread -> token n = et / 4, features fq .. fq + 15 with fq = 16 (et % 4); the 4 threads of a
          // token (adjacent lanes) share the amax of its 64 features
          const int n = et >> 2, fq = (et & 3) * 16;
          float h[16];
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float gg = stage_out[(fq + i) * kF8EpiStride + n], uu = stage_out[(64 + fq + i) * kF8EpiStride + n];
            h[i] = gg / (1.f + __expf(-gg)) * uu;
            amax = fmaxf(amax, fabsf(h[i]));
          }
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
          const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
          if (ok && n < nc) {
            uint32_t q[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              q[i] = e4m3x2(h[4 * i] * inv, h[4 * i + 1] * inv) | (e4m3x2(h[4 * i + 2] * inv, h[4 * i + 3] * inv) << 16);
            const size_t row = (size_t)(off + c0 + n);
            *reinterpret_cast<uint4*>(p.hq_out + row * p.F + mt * 64 + fq) = make_uint4(q[0], q[1], q[2], q[3]);
            if ((et & 3) == 0) p.hs_out[row * (p.F / 64) + mt] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
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
__global__ void gather_rows_q8_kernel(const __nv_bfloat16* __restrict__ xn, const int32_t* __restrict__ slot,
                                      int n_rows, int top_k, int d, uint8_t* __restrict__ xq, float* __restrict__ xs) {
  pdl_trigger();
  pdl_wait();
  const int nblk = d / 128;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= n_rows * nblk) return;
  const int t = wid / nblk, b = wid % nblk;
  const int my_slot = lane < top_k ? slot[(size_t)t * top_k + lane] : 0;
  const uint2 raw = *reinterpret_cast<const uint2*>(xn + (size_t)t * d + b * 128 + lane * 4);
  const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  const float v0 = __low2float(p0), v1 = __high2float(p0), v2 = __low2float(p1), v3 = __high2float(p1);
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

cudaError_t gather_rows_q8(const __nv_bfloat16* xn, const int32_t* slot, int n_rows, int top_k, int d, uint8_t* xq,
                           float* xs, cudaStream_t st) {
  if (d % 128 || top_k > 32) return cudaErrorInvalidValue;
  const int warps = n_rows * (d / 128);
  return launch_k(gather_rows_q8_kernel, dim3((warps + 7) / 8), dim3(256), 0, st, 1, xn, slot, n_rows, top_k, d, xq,
                  xs);
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
