// gemm.cu -- tcgen05 GEMMs of the canvas step.
//
// All products are D = A * B^T with A [M][K] and B [N][K] bf16, K-major (row-major with K
// contiguous), fp32 accumulation in tensor memory.  Operand tiles are TMA-loaded with 128-byte
// swizzle into a ring of shared-memory stages; one thread issues the loads, one thread issues the
// MMAs, and the four warps of the CTA drain TMEM in the epilogue.
//
//   dense_gemm_kernel<BN, EPI>   one 128 x BN tile per CTA (A = activations, B = weights):
//     EPI_QKV    the fused Q|K|V projection; rotary embedding (NeoX half split, positions P+j)
//                applied in registers; Q to the head-major query buffer, K to the cache rows,
//                V to the transposed value cache (decoder layer "attention block": pre-norm
//                Gemma-style layer, read from "same architecture as Gemma 4 26B A4B").
//     EPI_RESID  x += D (attention output projection + residual).
//     EPI_F32    out = D (router logits, vocabulary logits).
//   expert_gemm_kernel<MODE>     grouped, swap-AB (weights are the 128-row M side, the few tokens
//                routed to one expert are the N side):
//     MODE 1     [gate | up] rows of expert e times its gathered tokens; SwiGLU in the epilogue.
//     MODE 2     down-projection rows of expert e times its SwiGLU rows, scaled by each
//                assignment's gate weight (top-k routed MoE of the 26B-A4B model, 3.8B active).
#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int kGemmThreads = 128;
constexpr uint32_t kATileBytes = 128 * 64 * 2;   // 128 rows x 64 bf16

template <int BN>
struct DenseCfg {
  static constexpr uint32_t kBTileBytes = BN * 64 * 2;
  static constexpr uint32_t kStageBytes = kATileBytes + kBTileBytes;
  static constexpr int kStages = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;
};

struct GemmBarriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t accum;
  uint32_t tmem_slot;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ---------------------------------------------------------------------------------------------
// dense GEMM
// ---------------------------------------------------------------------------------------------
template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    dense_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                      int K, EpiParams ep, int* err) {
  using C = DenseCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = align1024(smem_raw);
  GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(tiles + (size_t)C::kStages * C::kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN;
  const int nk = K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->accum, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&bars->tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0 && lane == 0) {
    const uint64_t pol_w = l2_policy_evict_first();
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % C::kStages;
      const uint32_t ph = (kb / C::kStages) & 1;
      if (!mbar_wait(&bars->empty[s], ph ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      uint8_t* a = tiles + (size_t)s * C::kStageBytes;
      mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
      tma_load_2d(&tmA, &bars->full[s], a, kb * 64, m0);
      tma_load_2d_hint(&tmB, &bars->full[s], a + kATileBytes, kb * 64, n0, pol_w);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % C::kStages;
      const uint32_t ph = (kb / C::kStages) & 1;
      if (!mbar_wait(&bars->full[s], ph, err, DEV_ERR_TIMEOUT_MMA)) break;
      tc_fence_after();
      uint8_t* a = tiles + (size_t)s * C::kStageBytes;
      const uint64_t ad = smem_desc_sw128(smem_u32(a));
      const uint64_t bd = smem_desc_sw128(smem_u32(a + kATileBytes));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_bf16(tmem, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0);
      umma_commit(&bars->empty[s]);
    }
    umma_commit(&bars->accum);
  }
  __syncwarp();

  // ---------------- epilogue: thread owns accumulator row m0 + 32*warp + lane ----------------
  const bool ok = mbar_wait(&bars->accum, 0, err, DEV_ERR_TIMEOUT_EPILOGUE);
  tc_fence_after();
  const int row = m0 + warp * 32 + lane;
  const bool row_ok = ok && row < M;
  const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);

  if constexpr (EPI == EPI_QKV) {
    // Feature tile [n0, n0+BN) lies inside one of the Q / K / V regions (BN divides the region sizes).
    const int dh = ep.dh, half = dh >> 1;
    const int q_end = ep.n_q * dh, k_end = q_end + ep.n_kv * dh;
    const int seq = row / ep.rows_per_seq, j = row % ep.rows_per_seq;
    const int cseq = ep.seq_base + seq;
    const int pos = row_ok ? ep.seq_P[cseq] + j : 0;
    for (int h0 = 0; h0 < BN; h0 += dh) {
      const int f0 = n0 + h0;
      if (f0 >= N) break;
      if (f0 < k_end) {
        // rotate pairs (i, i+half) of this head, 32 pairs at a time
        for (int c = 0; c < half; c += 32) {
          float a[32], b[32];
          tmem_ld_32cols(tbase + h0 + c, a);
          tmem_ld_32cols(tbase + h0 + half + c, b);
          if (!row_ok) continue;
          const float2* cs = ep.rope + (size_t)pos * half + c;
          uint32_t lo[16], hi[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 c0 = cs[i], c1 = cs[i + 1];
            lo[i / 2] = pack_bf16x2(a[i] * c0.x - b[i] * c0.y, a[i + 1] * c1.x - b[i + 1] * c1.y);
            hi[i / 2] = pack_bf16x2(b[i] * c0.x + a[i] * c0.y, b[i + 1] * c1.x + a[i + 1] * c1.y);
          }
          __nv_bfloat16* dst;
          if (f0 < q_end) {
            const int h = f0 / dh;
            dst = ep.q + (((size_t)seq * ep.n_q + h) * ep.rows_per_seq + j) * dh;
          } else {
            const int h = (f0 - q_end) / dh;
            dst = ep.kc + (((size_t)cseq * ep.n_kv + h) * ep.max_ctx + pos) * dh;
          }
          uint4* d0 = reinterpret_cast<uint4*>(dst + c);
          uint4* d1 = reinterpret_cast<uint4*>(dst + half + c);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            d0[v] = make_uint4(lo[4 * v], lo[4 * v + 1], lo[4 * v + 2], lo[4 * v + 3]);
            d1[v] = make_uint4(hi[4 * v], hi[4 * v + 1], hi[4 * v + 2], hi[4 * v + 3]);
          }
        }
      } else {
        // V: written transposed, vt[cseq][h][i][pos]; lanes hold consecutive positions
        const int h = (f0 - k_end) / dh;
        __nv_bfloat16* dst = ep.vt + (((size_t)cseq * ep.n_kv + h) * dh) * ep.max_ctx + pos;
        for (int c = 0; c < dh; c += 32) {
          float a[32];
          tmem_ld_32cols(tbase + h0 + c, a);
          if (!row_ok) continue;
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[(size_t)(c + i) * ep.max_ctx] = __float2bfloat16_rn(a[i]);
        }
      }
    }
  } else {
    for (int c = 0; c < BN; c += 32) {
      float a[32];
      tmem_ld_32cols(tbase + c, a);
      if (!row_ok) continue;
      const int col = n0 + c;
      float* dst = (EPI == EPI_RESID ? ep.x : ep.out) + (size_t)row * ep.ldo + col;
      if (col + 32 <= N) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          float4 o = make_float4(a[4 * v], a[4 * v + 1], a[4 * v + 2], a[4 * v + 3]);
          if constexpr (EPI == EPI_RESID) {
            const float4 x = d4[v];
            o.x += x.x; o.y += x.y; o.z += x.z; o.w += x.w;
          }
          d4[v] = o;
        }
      } else {
        for (int i = 0; i < 32 && col + i < N; ++i) dst[i] = (EPI == EPI_RESID ? dst[i] : 0.f) + a[i];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

// ---------------------------------------------------------------------------------------------
// grouped expert GEMMs (swap-AB)
// ---------------------------------------------------------------------------------------------
constexpr int kExpBN = 64;                         // tokens per accumulator chunk
constexpr int kExpStages = 3;
constexpr uint32_t kExpBTile = kExpBN * 64 * 2;    // 8 KB: two 32-row boxes
constexpr uint32_t kExpStageBytes = kATileBytes + kExpBTile;
constexpr int kEpiStride = kExpBN + 1;             // padded fp32 staging rows
constexpr size_t kExpSmemBytes = 1024 + (size_t)kExpStages * kExpStageBytes + 128 * kEpiStride * 4 + 256;

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 2)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       ExpertParams p, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const int e = blockIdx.y, mt = blockIdx.x;
  const int n_e = p.counts[e];
  if (n_e <= 0) return;
  const int off = p.offsets[e];
  uint8_t* tiles = align1024(smem_raw);
  float* stage_out = reinterpret_cast<float*>(tiles + (size_t)kExpStages * kExpStageBytes);
  GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(stage_out + 128 * kEpiStride);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = MODE == 1 ? p.d : p.F;
  const int nk = K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kExpStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->accum, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&bars->tmem_slot, kExpBN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);

  uint32_t it = 0;   // ring position shared by producer and MMA issuer (both walk the same sequence)
  int chunk = 0;
  for (int c0 = 0; c0 < n_e; c0 += kExpBN, ++chunk) {
    const int nc = min(kExpBN, n_e - c0);
    const int nmma = (nc + 15) & ~15;
    const int nb = (nc + 31) >> 5;
    const uint32_t tx = kATileBytes + (uint32_t)nb * 4096u;
    if (warp == 0 && lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t i = it + kb;
        const int s = i % kExpStages;
        const uint32_t ph = (i / kExpStages) & 1;
        if (!mbar_wait(&bars->empty[s], ph ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
        uint8_t* a = tiles + (size_t)s * kExpStageBytes;
        mbar_arrive_expect_tx(&bars->full[s], tx);
        if (MODE == 1) {
          const int r0 = e * 2 * p.F + mt * 64;
          tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 64, r0, pol_w);               // gate rows
          tma_load_2d_hint(&tmW, &bars->full[s], a + 8192, kb * 64, r0 + p.F, pol_w);  // up rows
        } else {
          tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 64, e * p.d + mt * 128, pol_w);
        }
        for (int b = 0; b < nb; ++b)
          tma_load_2d(&tmX, &bars->full[s], a + kATileBytes + b * 4096, kb * 64, off + c0 + 32 * b);
      }
    } else if (warp == 1 && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, nmma);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t i = it + kb;
        const int s = i % kExpStages;
        const uint32_t ph = (i / kExpStages) & 1;
        if (!mbar_wait(&bars->full[s], ph, err, DEV_ERR_TIMEOUT_MMA)) break;
        tc_fence_after();
        uint8_t* a = tiles + (size_t)s * kExpStageBytes;
        const uint64_t ad = smem_desc_sw128(smem_u32(a));
        const uint64_t bd = smem_desc_sw128(smem_u32(a + kATileBytes));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16(tmem, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0);
        umma_commit(&bars->empty[s]);
      }
      umma_commit(&bars->accum);
    }
    it += nk;
    __syncwarp();

    const bool ok = mbar_wait(&bars->accum, chunk & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
    tc_fence_after();
    if (MODE == 1) {
      // stage the whole 128 x nmma accumulator (64 gate rows, then 64 up rows) in shared memory
      const int r = warp * 32 + lane;
      for (int cb = 0; cb < nmma; cb += 32) {
        float v[32];
        tmem_ld_32cols(tbase + cb, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) stage_out[r * kEpiStride + cb + i] = v[i];
      }
      __syncthreads();
      if (ok) {
        // thread -> (token n = tid/4 + 32*pass, features f = (tid%4)*16 .. +16)
        const int fq = (threadIdx.x & 3) * 16;
        for (int n = threadIdx.x >> 2; n < nc; n += 32) {
          uint32_t packed[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float g0 = stage_out[(fq + i) * kEpiStride + n], u0 = stage_out[(64 + fq + i) * kEpiStride + n];
            const float g1 = stage_out[(fq + i + 1) * kEpiStride + n],
                        u1 = stage_out[(64 + fq + i + 1) * kEpiStride + n];
            const float h0 = g0 / (1.f + __expf(-g0)) * u0;
            const float h1 = g1 / (1.f + __expf(-g1)) * u1;
            packed[i / 2] = pack_bf16x2(h0, h1);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.h_out + (size_t)(off + c0 + n) * p.F + mt * 64 + fq);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
      }
    } else {
      const int m = mt * 128 + warp * 32 + lane;   // output feature of the down projection
      for (int cb = 0; cb < nmma; cb += 32) {
        float v[32];
        tmem_ld_32cols(tbase + cb, v);
        if (!ok) continue;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int n = cb + i;
          if (n < nc) {
            const int rowa = off + c0 + n;
            p.y_out[(size_t)rowa * p.d + m] = v[i] * p.perm_gate[rowa];
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kExpBN);
}

// ---------------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------------
template <int BN, int EPI>
static cudaError_t launch_dense(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, const EpiParams& ep,
                                int* err, cudaStream_t st) {
  using C = DenseCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(dense_gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((M + 127) / 128, (N + BN - 1) / BN);
  dense_gemm_kernel<BN, EPI><<<grid, kGemmThreads, C::kSmemBytes, st>>>(a, b, M, N, K, ep, err);
  return cudaGetLastError();
}

cudaError_t gemm_dense(int bn, int epi, const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const EpiParams& ep, int* err, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (K % 64 != 0) return cudaErrorInvalidValue;
#define DG_DENSE_CASE(BN_, EPI_) \
  if (bn == BN_ && epi == EPI_) return launch_dense<BN_, EPI_>(a, b, M, N, K, ep, err, st);
  DG_DENSE_CASE(128, EPI_QKV)
  DG_DENSE_CASE(64, EPI_RESID)
  DG_DENSE_CASE(128, EPI_RESID)
  DG_DENSE_CASE(128, EPI_F32)
  DG_DENSE_CASE(256, EPI_F32)
  DG_DENSE_CASE(64, EPI_F32)
#undef DG_DENSE_CASE
  return cudaErrorInvalidValue;
}

template <int MODE>
static cudaError_t launch_expert(const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                                 int* err, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kExpSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(MODE == 1 ? p.F / 64 : p.d / 128, n_exp);
  expert_gemm_kernel<MODE><<<grid, kGemmThreads, kExpSmemBytes, st>>>(w, x, p, err);
  return cudaGetLastError();
}

cudaError_t gemm_expert(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                        int* err, cudaStream_t st) {
  return mode == 1 ? launch_expert<1>(w, x, p, n_exp, err, st) : launch_expert<2>(w, x, p, n_exp, err, st);
}

}  // namespace dg
