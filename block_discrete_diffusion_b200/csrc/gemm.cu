// gemm.cu -- tcgen05 GEMMs of the canvas step.
//
// All products are D = A * B^T with A [M][K] and B [N][K] bf16, K-major (row-major with K
// contiguous), fp32 accumulation in tensor memory.  Operand tiles are TMA-loaded with 128-byte
// swizzle into a ring of shared-memory stages; one thread issues the loads, one thread issues the
// MMAs, and the epilogue warps drain TMEM.
//
//   dense_gemm_kernel<BN, EPI, Z>  one 128 x BN tile per cluster of Z CTAs (split-K over the
//                cluster when there are few tiles; A = activations, B = weights), epilogue from
//                shared memory with coalesced stores:
//     EPI_QKV    the fused Q|K|V projection; rotary embedding (NeoX half split, positions P+j);
//                Q to the head-major query buffer, K to the cache rows, V to the transposed value
//                cache (decoder layer "attention block": pre-norm Gemma-style layer, read from
//                "same architecture as Gemma 4 26B A4B").
//     EPI_RESID  x += D (attention output projection + residual).
//     EPI_F32    out = D (router logits; vocabulary logits of several canvases).
//   expert_gemm_kernel<MODE, BN, FP8>  persistent, warp-specialised, swap-AB (weights are the
//                128-row M side, the tokens routed to one expert the N side, BN tokens per chunk):
//     MODE 1     [gate | up] rows of expert e times its gathered tokens; SwiGLU in the epilogue.
//     MODE 2     down-projection rows of expert e times its SwiGLU rows (the combine applies the
//                gate weights; top-k routed MoE of the 26B-A4B model, 3.8B active); also the
//                vocabulary head of one canvas (one "expert" holding all 256 rows).
//     FP8        weights as e4m3 bytes, expanded to bf16(q * s) in shared memory by converter warps.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

constexpr int kGemmThreads = 128;
constexpr uint32_t kATileBytes = 128 * 64 * 2;   // 128 rows x 64 bf16

// BN <= 128: two CTAs per SM (up to 96 KB of stages each); BN = 256: one CTA per SM.
template <int BN>
struct DenseCfg {
  static constexpr uint32_t kBTileBytes = BN * 64 * 2;
  static constexpr uint32_t kStageBytes = kATileBytes + kBTileBytes;
  static constexpr int kStages = BN >= 256 ? 4 : (BN >= 128 ? 3 : 4);
  static constexpr int kMinBlocks = BN >= 256 ? 1 : 2;
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
// Epilogue of RPC finished rows held in shared memory (t[r * rs + c], rows row0.., columns n0..),
// laid out so that global stores are coalesced: F32 / RESID rows by one warp each (lane = 4
// columns); Q and K heads rotated pairwise by one warp per row (lane = rotary pair), stored
// head-major; V heads by one warp per channel (lane = row, positions contiguous in the
// transposed value cache).
// With ep.rw (EPI_RESID, BN = 128): the updated rows x' also go back into the shared tile, and the
// tile's per-row sums of squares to ep.ssq (the FFN RMSNorm's statistics, folded in here).
template <int BN, int EPI, int RPC>
__device__ __forceinline__ void epilogue_from_smem(const EpiParams& ep, float* t, int rs, int row0, int n0,
                                                   int M, int N) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = kGemmThreads / 32;
  constexpr int RPW = (RPC + NW - 1) / NW;   // rows per warp
  constexpr int RB = RPW < 8 ? RPW : 8;      // rows whose loads are issued together
  // A 128-row tile lies inside one sequence's rows_per_seq rows: one committed length for all rows.
  // Global loads (length, rotary table, residual) are all issued before the stores that follow them.
  const int seq = row0 / ep.rows_per_seq, j0 = row0 % ep.rows_per_seq;
  if constexpr (EPI == EPI_QKV) {
    const int dh = ep.dh, half = dh >> 1;
    const int q_end = ep.n_q * dh, k_end = q_end + ep.n_kv * dh;
    const int cseq = ep.seq_base + seq;
    const int P = __ldg(ep.seq_P + cseq);
    for (int h0 = 0; h0 < BN; h0 += dh) {
      const int f_head = n0 + h0;
      if (f_head >= N) break;
      if (f_head < k_end) {
        for (int kb = 0; kb < RPW; kb += RB) {
          float2 cs[RB][2];
#pragma unroll
          for (int k = 0; k < RB; ++k) {
            const int r = warp + NW * (kb + k);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int i = lane + 32 * u;
              cs[k][u] = (kb + k < RPW && r < RPC && row0 + r < M && i < half)
                             ? __ldg(ep.rope + (size_t)(P + j0 + r) * half + i)
                             : make_float2(0.f, 0.f);
            }
          }
#pragma unroll
          for (int k = 0; k < RB; ++k) {
            const int r = warp + NW * (kb + k);
            if (kb + k >= RPW || r >= RPC || row0 + r >= M) break;
            const int j = j0 + r;
            __nv_bfloat16* dst =
                f_head < q_end ? ep.q + (((size_t)seq * ep.n_q + f_head / dh) * ep.rows_per_seq + j) * dh
                               : ep.kc + (((size_t)cseq * ep.n_kv + (f_head - q_end) / dh) * ep.max_ctx + P + j) * dh;
            const float* tr = t + r * rs + h0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int i = lane + 32 * u;
              if (i < half) {
                const float a = tr[i], b = tr[half + i];
                dst[i] = __float2bfloat16_rn(a * cs[k][u].x - b * cs[k][u].y);
                dst[half + i] = __float2bfloat16_rn(b * cs[k][u].x + a * cs[k][u].y);
              }
            }
          }
        }
      } else {
        // transposed value cache: one warp per channel, lanes along positions (contiguous)
        __nv_bfloat16* vbase = ep.vt + (((size_t)cseq * ep.n_kv + (f_head - k_end) / dh) * dh) * ep.max_ctx + P + j0;
        for (int c = warp; c < dh; c += NW)
          for (int r = lane; r < RPC && row0 + r < M; r += 32)
            vbase[(size_t)c * ep.max_ctx + r] = __float2bfloat16_rn(t[r * rs + h0 + c]);
      }
    }
  } else {
    constexpr int CG = BN / 128;             // 128-column groups (lane = 4 columns of each)
    for (int kb = 0; kb < RPW; kb += RB) {
      float4 xv[RB][CG];
      if constexpr (EPI == EPI_RESID) {
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          const int r = warp + NW * (kb + k);
#pragma unroll
          for (int g = 0; g < CG; ++g) {
            const int c = g * 128 + lane * 4;
            xv[k][g] = (kb + k < RPW && r < RPC && row0 + r < M && n0 + c + 4 <= N)
                           ? *reinterpret_cast<const float4*>(ep.x + (size_t)(row0 + r) * ep.ldo + n0 + c)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        const int r = warp + NW * (kb + k);
        if (kb + k >= RPW || r >= RPC || row0 + r >= M) break;
        float* dst = (EPI == EPI_RESID ? ep.x : ep.out) + (size_t)(row0 + r) * ep.ldo + n0;
        float* tr = t + r * rs;
        float ss = 0.f;
#pragma unroll
        for (int g = 0; g < CG; ++g) {
          const int c = g * 128 + lane * 4;
          if (n0 + c + 4 <= N) {
            float4 v = *reinterpret_cast<const float4*>(tr + c);
            if (EPI == EPI_RESID) {
              v.x += xv[k][g].x; v.y += xv[k][g].y; v.z += xv[k][g].z; v.w += xv[k][g].w;
              if (ep.rw) {
                *reinterpret_cast<float4*>(tr + c) = v;
                ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
              }
            }
            *reinterpret_cast<float4*>(dst + c) = v;
          } else {
            for (int q = 0; q < 4 && n0 + c + q < N; ++q)
              dst[c + q] = (EPI == EPI_RESID ? dst[c + q] : 0.f) + tr[c + q];
          }
        }
        if (EPI == EPI_RESID && ep.rw) {
          ss = warp_sum(ss);
          if (lane == 0) ep.ssq[(size_t)(n0 / 128) * M + row0 + r] = ss;
        }
      }
    }
  }
}

__device__ __forceinline__ void mma_bf16_m16n8k16(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The folded router's operands of a 128-column tile: the router weights W[e][n0 + c] of this warp's
// 8-expert groups (w, w + 4, w + 8, w + 12) as mma.sync B fragments, and the gains g[n0 + c] of this
// lane's columns.  Loaded once the accumulator is complete, so that their latency hides under the
// drain, the split-K reduction and the residual epilogue.
struct RouterFrags {
  uint32_t b[4][8][2];
  float2 g[8][2];
};
template <bool WITH_B>
__device__ __forceinline__ void router_frags_load(const EpiParams& ep, int n0, RouterFrags& f) {
  constexpr int NW = kGemmThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;   // fragment row group / column pair
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    f.g[ks][0] = __ldg(reinterpret_cast<const float2*>(ep.rg + n0 + 16 * ks + 2 * tig));
    f.g[ks][1] = __ldg(reinterpret_cast<const float2*>(ep.rg + n0 + 16 * ks + 8 + 2 * tig));
  }
  if constexpr (!WITH_B) return;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int nt = warp + NW * j;
    if (nt < ep.n_exp / 8) {
      const __nv_bfloat16* wr = ep.rw + (size_t)(nt * 8 + gid) * ep.ldo + n0 + 2 * tig;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        f.b[j][ks][0] = __ldg(reinterpret_cast<const unsigned int*>(wr + 16 * ks));
        f.b[j][ks][1] = __ldg(reinterpret_cast<const unsigned int*>(wr + 16 * ks + 8));
      }
    }
  }
}

// The tile's 128 columns of the router weights W[e][n0 + c] into shared memory with asynchronous copies
// (rows of kRwPitch bytes: 256 + 16, so that the eight rows an ldmatrix reads fall in different banks).
constexpr int kRwPitch = 272;
__device__ __forceinline__ void router_w_to_smem(const EpiParams& ep, int n0, uint8_t* wr_s) {
  for (int i = threadIdx.x; i < ep.n_exp * 16; i += kGemmThreads) {
    const int e = i >> 4, c16 = i & 15;
    const __nv_bfloat16* src = ep.rw + (size_t)e * ep.ldo + n0 + c16 * 8;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(wr_s + e * kRwPitch + c16 * 16)),
                 "l"(src)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// The router's share of the tile (ep.rw): rpart[n0/128][row][e] = sum over the tile's 128 columns c of
// bf16(x'[row][c] g[c]) * W[e][c], for the RPC updated rows held in shared memory.  A small product
// (RPC x n_exp x 128), so it runs on warp-level mma.sync (16 rows x 8 experts x 16 columns per
// instruction, fp32 accumulation) inside the epilogue; warp w takes the 8-expert groups w, w + 4, ...
template <int RPC, bool B_SMEM>
__device__ __forceinline__ void router_partial_from_smem(const EpiParams& ep, const RouterFrags& f, const float* t,
                                                         int rs, int row0, int n0, int M, const uint8_t* wr_s) {
  static_assert(RPC % 16 == 0, "16-row blocks");
  constexpr int NW = kGemmThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  float* out = ep.rpart + (size_t)(n0 / 128) * M * ep.n_exp;
#pragma unroll 1
  for (int mt = 0; mt < RPC / 16; ++mt) {
    // A fragments of this 16-row block (bf16(x' g)), shared by the warp's expert groups
    uint32_t a[8][4];
    const float* r0 = t + (mt * 16 + gid) * rs + 2 * tig;
    const float* r1 = r0 + 8 * rs;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const float2 x00 = *reinterpret_cast<const float2*>(r0 + 16 * ks);
      const float2 x10 = *reinterpret_cast<const float2*>(r1 + 16 * ks);
      const float2 x01 = *reinterpret_cast<const float2*>(r0 + 16 * ks + 8);
      const float2 x11 = *reinterpret_cast<const float2*>(r1 + 16 * ks + 8);
      a[ks][0] = pack_bf16x2(x00.x * f.g[ks][0].x, x00.y * f.g[ks][0].y);
      a[ks][1] = pack_bf16x2(x10.x * f.g[ks][0].x, x10.y * f.g[ks][0].y);
      a[ks][2] = pack_bf16x2(x01.x * f.g[ks][1].x, x01.y * f.g[ks][1].y);
      a[ks][3] = pack_bf16x2(x11.x * f.g[ks][1].x, x11.y * f.g[ks][1].y);
    }
    const int ra = row0 + mt * 16 + gid;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int nt = warp + NW * j;
      if (nt < ep.n_exp / 8) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (B_SMEM) {
          // B fragments of two column steps per ldmatrix.x4: lanes 8 m .. 8 m + 7 address the group's rows at
          // columns 16 (ks + m / 2) + 8 (m % 2)
          const int mi = lane >> 3;
          const uint32_t rowa = smem_u32(wr_s + (nt * 8 + (lane & 7)) * kRwPitch) + (uint32_t)(((mi >> 1) * 16 + (mi & 1) * 8) * 2);
#pragma unroll
          for (int ks = 0; ks < 8; ks += 2) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(rowa + ks * 32, b0, b1, b2, b3);
            mma_bf16_m16n8k16(c, a[ks], b0, b1);
            mma_bf16_m16n8k16(c, a[ks + 1], b2, b3);
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) mma_bf16_m16n8k16(c, a[ks], f.b[j][ks][0], f.b[j][ks][1]);
        }
        const int e = nt * 8 + 2 * tig;
        if (ra < M) *reinterpret_cast<float2*>(out + (size_t)ra * ep.n_exp + e) = make_float2(c[0], c[1]);
        if (ra + 8 < M) *reinterpret_cast<float2*>(out + (size_t)(ra + 8) * ep.n_exp + e) = make_float2(c[2], c[3]);
      }
    }
  }
}

// One 128 x BN output tile per cluster of Z CTAs; CTA z of the cluster multiplies k-blocks
// [z nk/Z, (z+1) nk/Z).  Z = 1: the accumulator goes from TMEM (thread = row) to shared memory and
// the epilogue runs from there.
// Z > 1: every CTA writes its fp32 partial to its slot of an L2-resident scratch (coalesced); after
// a cluster barrier CTA z sums rows [z 128/Z, (z+1) 128/Z) over the Z slots in rank order (so the
// result does not depend on timing) and runs the epilogue on those rows from shared memory.
template <int BN, int EPI, int Z>
__global__ void __launch_bounds__(kGemmThreads, DenseCfg<BN>::kMinBlocks)
    dense_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                      int K, EpiParams ep, int* err) {
  using C = DenseCfg<BN>;
  static_assert(Z == 1 || (Z > 1 && 128 % Z == 0 && (BN / (2 * Z)) % 4 == 0), "bad split");
  static_assert((size_t)128 * (BN + 4) * 4 <= (size_t)C::kStages * C::kStageBytes, "parked tile too big");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = align1024(smem_raw);
  GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(tiles + (size_t)C::kStages * C::kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN;
  const int nk_all = K / 64;
  const int zz = Z > 1 ? (int)blockIdx.z : 0;
  const int kb0 = zz * nk_all / Z;
  const int nk = (zz + 1) * nk_all / Z - kb0;
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }

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
    // The weights (B) of the first stages do not depend on the previous kernel (unless a preceding
    // kernel writes them): load them before waiting for it; the activation tiles (A) follow the wait.
    const int npre = nk < C::kStages ? nk : C::kStages;
    if (ep.late_weights) pdl_wait();
    for (int kb = 0; kb < npre; ++kb) {
      uint8_t* a = tiles + (size_t)kb * C::kStageBytes;
      mbar_expect_tx(&bars->full[kb], C::kBTileBytes);
      tma_load_2d_hint(&tmB, &bars->full[kb], a + kATileBytes, (kb0 + kb) * 64, n0, pol_w);
    }
    if (!ep.late_weights) pdl_wait();
    for (int kb = 0; kb < npre; ++kb) {
      uint8_t* a = tiles + (size_t)kb * C::kStageBytes;
      mbar_arrive_expect_tx(&bars->full[kb], kATileBytes);
      tma_load_2d(&tmA, &bars->full[kb], a, (kb0 + kb) * 64, m0);
    }
    for (int kb = npre; kb < nk; ++kb) {
      const int s = kb % C::kStages;
      const uint32_t ph = (kb / C::kStages) & 1;
      if (!mbar_wait(&bars->empty[s], ph ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
      uint8_t* a = tiles + (size_t)s * C::kStageBytes;
      mbar_arrive_expect_tx(&bars->full[s], C::kStageBytes);
      tma_load_2d(&tmA, &bars->full[s], a, (kb0 + kb) * 64, m0);
      tma_load_2d_hint(&tmB, &bars->full[s], a + kATileBytes, (kb0 + kb) * 64, n0, pol_w);
    }
  } else {
    pdl_wait();
  }
  if (warp == 1 && lane == 0) {
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

  const bool ok = mbar_wait(&bars->accum, 0, err, DEV_ERR_TIMEOUT_EPILOGUE);
  tc_fence_after();
  RouterFrags rf;
  if constexpr (EPI == EPI_RESID && BN == 128) {
    if (ep.rw) router_frags_load<Z == 1>(ep, n0, rf);   // Z > 1: the weights go to shared memory below
  }
  const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);

  if constexpr (Z == 1) {
    // ---------------- accumulator -> shared memory (thread = row) -> coalesced epilogue ----------------
    constexpr int RS = BN + 4;
    float* red = reinterpret_cast<float*>(tiles);
    {
      const int r = warp * 32 + lane;
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld_32cols(tbase + c, v);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(red + r * RS + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    }
    if (__syncthreads_and(ok)) {
      epilogue_from_smem<BN, EPI, 128>(ep, red, RS, m0, n0, M, N);
      if constexpr (EPI == EPI_RESID && BN == 128) {
        if (ep.rw) {
          __syncthreads();
          router_partial_from_smem<128, false>(ep, rf, red, RS, m0, n0, M, nullptr);
        }
      }
    }
  } else {
    // ---------------- split-K: partials through an L2-resident scratch, summed in rank order ----------------
    constexpr int RS = BN + 4;                 // padded row stride of the shared-memory tiles
    constexpr int F4 = BN / 4;                 // float4 per row
    constexpr int RPC = 128 / Z;               // rows finished by this CTA
    float* red = reinterpret_cast<float*>(tiles);
    {
      const int r = warp * 32 + lane;
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld_32cols(tbase + c, v);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(red + r * RS + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    }
    __syncthreads();
    // slot zz of this tile: [128][BN], written with coalesced stores.  The projections whose outputs are
    // bf16 (Q/K/V) or small next to the fp32 residual they are added to (O) keep their partials in bf16
    // (half the bytes through L2; one more rounding of 2^-9 relative per partial); the fp32 router
    // logits keep fp32 partials.
    constexpr bool kBfPart = EPI != EPI_F32;
    float* slots = ep.part + (size_t)(blockIdx.y * gridDim.x + blockIdx.x) * Z * 128 * BN;
    if constexpr (kBfPart) {
      uint2* dst = reinterpret_cast<uint2*>(slots) + (size_t)zz * 128 * F4;
      for (int i = threadIdx.x; i < 128 * F4; i += kGemmThreads) {
        const float4 v = *reinterpret_cast<const float4*>(red + (i / F4) * RS + 4 * (i % F4));
        __stcg(dst + i, make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w)));
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(slots + (size_t)zz * 128 * BN);
      for (int i = threadIdx.x; i < 128 * F4; i += kGemmThreads)
        __stcg(dst + i, *reinterpret_cast<const float4*>(red + (i / F4) * RS + 4 * (i % F4)));
    }
    // every slot of the tile is written (the barrier's release / acquire at cluster scope makes the
    // peers' global stores visible), and this CTA's shared tile is free again
    cluster_sync();
    // the folded router's weight columns into the shared memory past the reduced rows (in flight during the
    // reduction and the residual epilogue)
    uint8_t* wr_s = reinterpret_cast<uint8_t*>(red + RPC * RS);
    if constexpr (EPI == EPI_RESID && BN == 128) {
      static_assert((size_t)RPC * RS * 4 + 128 * kRwPitch <= (size_t)C::kStages * C::kStageBytes, "router staging");
      if (ep.rw) router_w_to_smem(ep, n0, wr_s);
    }
    {
      constexpr int IT = RPC * F4 / kGemmThreads;           // float4 per thread
      constexpr int B = IT < 16 / Z ? IT : 16 / Z;          // iterations whose Z loads are in flight together
      static_assert((RPC * F4) % kGemmThreads == 0 && IT % B == 0, "reduction split");
      for (int i0 = 0; i0 < IT; i0 += B) {
        float4 v[B][Z];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int i = threadIdx.x + (i0 + b) * kGemmThreads;
          const size_t off = (size_t)(zz * RPC + i / F4) * BN + 4 * (i % F4);
#pragma unroll
          for (int z = 0; z < Z; ++z) {
            if constexpr (kBfPart) {
              const uint2 q = __ldcg(reinterpret_cast<const uint2*>(slots) + ((size_t)z * 128 * BN + off) / 4);
              v[b][z] = make_float4(bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y));
            } else {
              v[b][z] = __ldcg(reinterpret_cast<const float4*>(slots + (size_t)z * 128 * BN + off));
            }
          }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int i = threadIdx.x + (i0 + b) * kGemmThreads;
          float4 acc = v[b][0];
#pragma unroll
          for (int z = 1; z < Z; ++z) {
            acc.x += v[b][z].x; acc.y += v[b][z].y; acc.z += v[b][z].z; acc.w += v[b][z].w;
          }
          *reinterpret_cast<float4*>(red + (i / F4) * RS + 4 * (i % F4)) = acc;
        }
      }
    }
    if (__syncthreads_and(ok)) {
      epilogue_from_smem<BN, EPI, RPC>(ep, red, RS, m0 + zz * RPC, n0, M, N);
      if constexpr (EPI == EPI_RESID && BN == 128) {
        if (ep.rw) {
          asm volatile("cp.async.wait_all;" ::: "memory");
          __syncthreads();
          router_partial_from_smem<RPC, true>(ep, rf, red, RS, m0 + zz * RPC, n0, M, wr_s);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

// ---------------------------------------------------------------------------------------------
// grouped expert GEMMs (swap-AB), persistent and warp-specialised
// ---------------------------------------------------------------------------------------------
// Work items are (expert, 128-row weight tile) pairs, dealt round-robin to one CTA per SM; an item
// with n tokens is n/64 accumulator chunks.  Warp 0 streams weight tiles and the chunk's activation
// rows through a ring of shared-memory stages that runs on across items; warp 1 issues the MMAs
// into one of two TMEM accumulators; warps 2-5 drain the other accumulator, so the epilogue of one
// chunk overlaps the MMAs of the next.
// BN = tokens per accumulator chunk: 64 when a few tokens reach each expert (batch 1), 256 when
// hundreds do (several canvases), so that a weight tile is streamed once per 256 tokens.
// bf16 weights: a ring of kStages (weight tile 16 KB + token tile) stages.
// FP8 weights: a ring of kStages load slots (e4m3 weight tile 8 KB + token tile) and, apart from
// it, kConv bf16 weight tiles that the converter warps fill; the deeper load ring keeps about as
// many weight bytes in flight from HBM as the bf16 ring does.
template <int BN, bool FP8>
struct ExpCfg {
  static constexpr uint32_t kBTile = BN * 64 * 2;            // BN token rows x 64 k (32-row boxes)
  static constexpr uint32_t kAOff = FP8 ? kATileBytes / 2 : kATileBytes;   // token tile offset in a slot
  static constexpr uint32_t kStageBytes = kAOff + kBTile;
  static constexpr int kStages = FP8 ? (BN >= 256 ? 4 : 13) : (BN >= 256 ? 4 : 7);
  static constexpr int kConv = FP8 ? (BN >= 256 ? 2 : 3) : 0;
  static constexpr int kEpiCols = BN < 64 ? BN : 64;         // MODE 1 epilogue slice (accumulator columns)
  static constexpr int kEpiStride = kEpiCols + 1;            // padded fp32 staging rows
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + (size_t)kConv * kATileBytes +
                                       128 * kEpiStride * 4 + 512;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kStages <= 16 && kConv <= 4, "barrier arrays");
};
constexpr int kExpThreads = 192;                   // 6 warps (bf16 weights)
constexpr int kConvWarps = 4;                      // FP8: converter warps
constexpr int kExpThreadsFp8 = kExpThreads + 32 * kConvWarps;

struct ExpBarriers {
  uint64_t full[16];
  uint64_t empty[16];
  uint64_t cfull[4];   // FP8: a bf16 weight tile has been expanded
  uint64_t cempty[4];  // FP8: the MMAs reading a bf16 weight tile have completed
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_slot;
};

__device__ __forceinline__ void epi_bar_sync() {   // the 128 epilogue threads only (named barrier 1)
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// 4 e4m3 bytes times a scale -> 4 bf16: hardware e4m3x2 -> f16x2, fp32 multiply (the product's fp32
// rounding), one round-to-nearest-even to bf16.
__device__ __forceinline__ uint32_t e4m3x2_scaled(uint32_t two, float sc) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x * sc, f.y * sc);
}
__device__ __forceinline__ uint2 e4m3x4_scaled(uint32_t w, float sc) {
  return make_uint2(e4m3x2_scaled(w, sc), e4m3x2_scaled(w >> 16, sc));
}

// FP8: the weight operand arrives as e4m3 bytes (TMA into a load slot); kConvWarps converter warps
// expand it to bf16(q * s) in one of two bf16 tiles, in the 128-byte-swizzled layout the MMA reads.
template <int MODE, int BN, bool FP8>
__global__ void __launch_bounds__(FP8 ? kExpThreadsFp8 : kExpThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       ExpertParams p, int n_exp, int* err) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  uint8_t* tiles = align1024(smem_raw);
  using C = ExpCfg<BN, FP8>;
  constexpr int kExpStages = C::kStages;
  constexpr uint32_t kExpStageBytes = C::kStageBytes;
  constexpr int kExpBN = BN;
  uint8_t* conv_tiles = tiles + (size_t)kExpStages * kExpStageBytes;   // FP8: kConv bf16 weight tiles
  float* stage_out = reinterpret_cast<float*>(conv_tiles + (size_t)C::kConv * kATileBytes);
  constexpr int kEpiCols = C::kEpiCols, kEpiStride = C::kEpiStride, kConv = C::kConv > 0 ? C::kConv : 1;
  ExpBarriers* bars = reinterpret_cast<ExpBarriers*>(stage_out + 128 * kEpiStride);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = MODE == 1 ? p.d : p.F;
  const int nk = K / 64;
  const int MT = MODE == 1 ? p.F / 64 : p.d / 128;   // weight tiles per expert
  const int n_items = n_exp * MT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kExpStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int c = 0; c < kConv; ++c) {
      mbar_init(&bars->cfull[c], kConvWarps);
      mbar_init(&bars->cempty[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_slot, 2 * kExpBN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  if (!FP8 && p.pre_bytes > 0 && (int)blockIdx.x < n_items) {
    // While the preceding (light) kernels still run, the HBM is idle: bring the first columns of
    // this CTA's first weight tile into L2 (weights are never written by this step).  One range
    // per weight row (rows are K-contiguous); TMA reads them after the wait.
    const int e = blockIdx.x / MT, mt = blockIdx.x % MT;
    const uint8_t* wbase = static_cast<const uint8_t*>(p.w_base);
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
      const int row = MODE == 1 ? (i < 64 ? e * 2 * p.F + mt * 64 + i : e * 2 * p.F + p.F + mt * 64 + (i - 64))
                                : e * p.d + mt * 128 + i;
      l2_prefetch_bulk(wbase + (size_t)row * K * 2, (uint32_t)p.pre_bytes);
    }
  }
  pdl_wait();   // the routing (offsets) and the activation rows come from the preceding kernels

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      // 64-token bf16 chunks read every weight tile once: evict first; wide chunks (and the 32-token
      // FP8 chunks) may read it again a few microseconds later: normal policy, the re-read hits L2
      const uint64_t pol_w = (BN >= 256 || FP8) ? l2_policy_evict_normal() : l2_policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int e = item / MT, mt = item % MT;
        const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
        for (int c0 = 0; c0 < n_e && ok; c0 += kExpBN) {
          const int nb = (min(kExpBN, n_e - c0) + 31) >> 5;
          const uint32_t tx = (FP8 ? kATileBytes / 2 : kATileBytes) + (uint32_t)nb * 4096u;
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % kExpStages;
            if (!mbar_wait(&bars->empty[s], ((it / kExpStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) {
              ok = false;
              break;
            }
            uint8_t* a = tiles + (size_t)s * kExpStageBytes;
            mbar_arrive_expect_tx(&bars->full[s], tx);
            if (FP8) {   // e4m3 rows of 64 bytes at the start of the slot
              if (MODE == 1) {
                const int r0 = e * 2 * p.F + mt * 64;
                tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 64, r0, pol_w);
                tma_load_2d_hint(&tmW, &bars->full[s], a + 4096, kb * 64, r0 + p.F, pol_w);
              } else {
                tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 64, e * p.d + mt * 128, pol_w);
              }
            } else if (MODE == 1) {
              const int r0 = e * 2 * p.F + mt * 64;
              tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 64, r0, pol_w);               // gate rows
              tma_load_2d_hint(&tmW, &bars->full[s], a + 8192, kb * 64, r0 + p.F, pol_w);  // up rows
            } else {
              tma_load_2d_hint(&tmW, &bars->full[s], a, kb * 64, e * p.d + mt * 128, pol_w);
            }
            for (int b = 0; b < nb; ++b)
              tma_load_2d(&tmX, &bars->full[s], a + C::kAOff + b * 4096, kb * 64, off + c0 + 32 * b);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      uint32_t it = 0, j = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int e = item / MT;
        const int n_e = p.offsets[e + 1] - p.offsets[e];
        for (int c0 = 0; c0 < n_e && ok; c0 += kExpBN, ++j) {
          const int nmma = (min(kExpBN, n_e - c0) + 15) & ~15;
          const uint32_t idesc = idesc_bf16_f32(128, nmma);
          const uint32_t b = j & 1;
          if (!mbar_wait(&bars->acc_empty[b], ((j >> 1) & 1) ^ 1, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem + b * kExpBN;
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % kExpStages;
            const int cv = it % kConv;
            if (!mbar_wait(&bars->full[s], (it / kExpStages) & 1, err, DEV_ERR_TIMEOUT_MMA) ||
                (FP8 && !mbar_wait(&bars->cfull[cv], (it / kConv) & 1, err, DEV_ERR_TIMEOUT_MMA))) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* a = tiles + (size_t)s * kExpStageBytes;
            const uint64_t ad = smem_desc_sw128(smem_u32(FP8 ? conv_tiles + cv * kATileBytes : a));
            const uint64_t bd = smem_desc_sw128(smem_u32(a + C::kAOff));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(acc, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0);
            umma_commit(&bars->empty[s]);
            if (FP8) umma_commit(&bars->cempty[cv]);
          }
          umma_commit(&bars->acc_full[b]);
        }
      }
    }
  } else if (FP8 && warp >= 6) {
    // ------------------------------ FP8 converters (warps 6 ..) ------------------------------
    // Lane l keeps the scales of 128-column block l of the item's two 64-row halves (MODE 1: gate,
    // up) or of its 128-row tile (MODE 2); the next item's are loaded while this one is converted.
    // Waits are made warp-uniform so that the shuffles always see all 32 lanes.
    const int ct = threadIdx.x - kExpThreads;     // 0 .. 32 kConvWarps - 1
    auto load_scales = [&](int item, float& s0, float& s1) {
      const int e = item / MT, mt = item % MT;
      const int sr0 = MODE == 1 ? (e * 2 * p.F + mt * 64) / 128 : (e * p.d + mt * 128) / 128;
      const int sr1 = MODE == 1 ? (e * 2 * p.F + p.F + mt * 64) / 128 : sr0;
      s0 = lane < p.w_scale_cols ? __ldg(p.w_scale + (size_t)sr0 * p.w_scale_cols + lane) : 0.f;
      s1 = lane < p.w_scale_cols ? __ldg(p.w_scale + (size_t)sr1 * p.w_scale_cols + lane) : 0.f;
    };
    uint32_t it = 0;
    bool ok = true;
    float cur0 = 0.f, cur1 = 0.f;
    if ((int)blockIdx.x < n_items) load_scales(blockIdx.x, cur0, cur1);
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int e = item / MT;
      const int n_e = p.offsets[e + 1] - p.offsets[e];
      float nxt0 = 0.f, nxt1 = 0.f;
      if (item + (int)gridDim.x < n_items) load_scales(item + gridDim.x, nxt0, nxt1);
      for (int c0 = 0; c0 < n_e && ok; c0 += kExpBN) {
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kExpStages;
          const int cv = it % kConv;
          const bool got = mbar_wait(&bars->full[s], (it / kExpStages) & 1, err, DEV_ERR_TIMEOUT_PRODUCER) &&
                           mbar_wait(&bars->cempty[cv], ((it / kConv) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          const uint8_t* a8 = tiles + (size_t)s * kExpStageBytes;     // e4m3 rows of 64 bytes
          uint8_t* a = conv_tiles + cv * kATileBytes;                 // bf16, 128-byte swizzle
          const float sc0 = __shfl_sync(0xffffffffu, cur0, kb >> 1);
          const float sc1 = __shfl_sync(0xffffffffu, cur1, kb >> 1);
          // 16-byte chunk g = ct + 32 kConvWarps i of the e4m3 tile: row g / 4, bytes 16 (g % 4) ..
#pragma unroll
          for (int i = 0; i < 512 / (32 * kConvWarps); ++i) {
            const int g = ct + 32 * kConvWarps * i, row = g >> 2, qc = g & 3;
            const uint4 q = *reinterpret_cast<const uint4*>(a8 + g * 16);
            const float sc = row < 64 ? sc0 : sc1;
            uint8_t* dst = a + row * 128;
            const uint2 p0 = e4m3x4_scaled(q.x, sc), p1 = e4m3x4_scaled(q.y, sc);
            const uint2 p2 = e4m3x4_scaled(q.z, sc), p3 = e4m3x4_scaled(q.w, sc);
            *reinterpret_cast<uint4*>(dst + (((2 * qc) ^ (row & 7)) << 4)) = make_uint4(p0.x, p0.y, p1.x, p1.y);
            *reinterpret_cast<uint4*>(dst + (((2 * qc + 1) ^ (row & 7)) << 4)) = make_uint4(p2.x, p2.y, p3.x, p3.y);
          }
          fence_proxy_async_smem();                 // generic-proxy writes -> tensor-core reads
          __syncwarp();
          if ((threadIdx.x & 31) == 0) mbar_arrive(&bars->cfull[cv]);
        }
      }
      cur0 = nxt0;
      cur1 = nxt1;
    }
  } else {
    // ------------------------------ epilogue (warps 2-5) ------------------------------
    const int quarter = warp & 3;                 // TMEM lanes [32 quarter, 32 quarter + 32)
    const int r = quarter * 32 + lane;            // accumulator row = weight row of the tile
    const int et = threadIdx.x - 64;              // 0..127 among the epilogue threads
    uint32_t j = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int e = item / MT, mt = item % MT;
      const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
      for (int c0 = 0; c0 < n_e; c0 += kExpBN, ++j) {
        const int nc = min(kExpBN, n_e - c0);
        const int nmma = (nc + 15) & ~15;
        const uint32_t b = j & 1;
        const bool ok = mbar_wait(&bars->acc_full[b], (j >> 1) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
        tc_fence_after();
        const uint32_t acc = tmem + ((uint32_t)(quarter * 32) << 16) + b * kExpBN;
        if (MODE == 1) {
          // slices of kEpiCols tokens: accumulator -> staging rows -> SwiGLU of (gate row f, up row 64 + f)
          for (int cs = 0; cs < nmma; cs += kEpiCols) {
            const int ncs = min(kEpiCols, nmma - cs);
            for (int cb = 0; cb < ncs; cb += 32) {
              float v[32];
              tmem_ld_32cols(acc + cs + cb, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) stage_out[r * kEpiStride + cb + i] = v[i];
            }
            if (cs + kEpiCols >= nmma) {          // last TMEM read of this accumulator: release it
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->acc_empty[b]);
            }
            epi_bar_sync();
            if (ok) {
              // thread -> (token n = et/4 + 32*pass, features f = (et%4)*16 .. +16); gate rows 0-63, up rows 64-127
              const int fq = (et & 3) * 16;
              const int ncv = min(ncs, nc - cs);
              for (int n = et >> 2; n < ncv; n += 32) {
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                  const float g0 = stage_out[(fq + i) * kEpiStride + n], u0 = stage_out[(64 + fq + i) * kEpiStride + n];
                  const float g1 = stage_out[(fq + i + 1) * kEpiStride + n],
                              u1 = stage_out[(64 + fq + i + 1) * kEpiStride + n];
                  packed[i / 2] = pack_bf16x2(g0 / (1.f + __expf(-g0)) * u0, g1 / (1.f + __expf(-g1)) * u1);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.h_out + (size_t)(off + c0 + cs + n) * p.F + mt * 64 + fq);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
              }
            }
            epi_bar_sync();   // the staging buffer is rewritten by the next slice
          }
        } else {
          const int m = mt * 128 + r;             // output feature of the down projection
          for (int cb = 0; cb < nmma; cb += 32) {
            float v[32];
            tmem_ld_32cols(acc + cb, v);
            if (cb + 32 >= nmma) {                // last TMEM read of this accumulator: release it
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->acc_empty[b]);
            }
            if (!ok) continue;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int n = cb + i;
              if (n < nc) {
                const int rowa = off + c0 + n;
                p.y_out[(size_t)rowa * p.d + m] = v[i];
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 2 * kExpBN);
}

// ---------------------------------------------------------------------------------------------
// gate|up and down in one persistent launch (bf16 weights, 64-token chunks)
// ---------------------------------------------------------------------------------------------
// The work list is every (expert, 64 gate + 64 up rows) item, then every (expert, 128 down rows)
// item, dealt round-robin to one CTA per SM.  A CTA's down items come after its own gate|up items
// in its order, and a down item of expert e reads the SwiGLU rows of all of e's gate|up items: its
// producer waits (bounded) until done[e] counts them, after which the TMA reads rows other CTAs
// wrote.  Against two launches this fills the half-empty last round of the gate|up items with down
// items and removes the launch in between.  done[] is zeroed by the gather that precedes the launch.
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// generic-proxy writes of other threads (already acquired) -> this thread's later async-proxy (TMA) reads
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

template <int BN>
__global__ void __launch_bounds__(kExpThreads, 1)
    expert_updown_kernel(const __grid_constant__ CUtensorMap tmWu, const __grid_constant__ CUtensorMap tmX,
                         const __grid_constant__ CUtensorMap tmWd, const __grid_constant__ CUtensorMap tmH,
                         ExpertParams p, int n_exp, int* done, int* err) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmWu);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmWd);
    tma_prefetch_desc(&tmH);
  }
  uint8_t* tiles = align1024(smem_raw);
  using C = ExpCfg<BN, false>;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kStageBytes = C::kStageBytes;
  float* stage_out = reinterpret_cast<float*>(tiles + (size_t)kStages * kStageBytes);
  constexpr int kEpiCols = C::kEpiCols, kEpiStride = C::kEpiStride;
  ExpBarriers* bars = reinterpret_cast<ExpBarriers*>(stage_out + 128 * kEpiStride);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MTu = p.F / 64, MTd = p.d / 128;             // weight tiles per expert: gate|up, down
  const int n_up = n_exp * MTu, n_items = n_up + n_exp * MTd;
  // item -> (gate|up?, expert, tile)
  auto decode = [&](int item, bool& up, int& e, int& mt) {
    up = item < n_up;
    const int j = up ? item : item - n_up;
    const int MT = up ? MTu : MTd;
    e = j / MT;
    mt = j % MT;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_slot, 2 * BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  if (p.pre_bytes > 0 && (int)blockIdx.x < n_up) {
    // the first gate|up tile into L2 while the preceding (light) kernels still run
    const int e = blockIdx.x / MTu, mt = blockIdx.x % MTu;
    const uint8_t* wbase = static_cast<const uint8_t*>(p.w_base);
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
      const int row = i < 64 ? e * 2 * p.F + mt * 64 + i : e * 2 * p.F + p.F + mt * 64 + (i - 64);
      l2_prefetch_bulk(wbase + (size_t)row * p.d * 2, (uint32_t)p.pre_bytes);
    }
  }
  pdl_wait();   // routing, the gathered rows and done[] (zeroed) come from the preceding kernels

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      uint32_t it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        bool up;
        int e, mt;
        decode(item, up, e, mt);
        const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
        if (!up && n_e > 0) {
          // every gate|up tile of expert e has written its SwiGLU rows (bounded wait)
          if (ld_acquire_gpu(done + e) < MTu) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t i = 1; ld_acquire_gpu(done + e) < MTu; ++i) {
              if ((i & 63) == 0) {
                if (*reinterpret_cast<volatile int*>(err) != 0) { ok = false; break; }
                if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
                  report_error(err, DEV_ERR_TIMEOUT_PRODUCER);
                  ok = false;
                  break;
                }
              }
            }
            if (!ok) break;
          }
          fence_proxy_async_global();
        }
        const int K = up ? p.d : p.F;
        const int nk = K / 64;
        for (int c0 = 0; c0 < n_e && ok; c0 += BN) {
          const int nb = (min(BN, n_e - c0) + 31) >> 5;
          const uint32_t tx = kATileBytes + (uint32_t)nb * 4096u;
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % kStages;
            if (!mbar_wait(&bars->empty[s], ((it / kStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) {
              ok = false;
              break;
            }
            uint8_t* a = tiles + (size_t)s * kStageBytes;
            mbar_arrive_expect_tx(&bars->full[s], tx);
            if (up) {
              const int r0 = e * 2 * p.F + mt * 64;
              tma_load_2d_hint(&tmWu, &bars->full[s], a, kb * 64, r0, pol_w);               // gate rows
              tma_load_2d_hint(&tmWu, &bars->full[s], a + 8192, kb * 64, r0 + p.F, pol_w);  // up rows
              for (int b = 0; b < nb; ++b)
                tma_load_2d(&tmX, &bars->full[s], a + C::kAOff + b * 4096, kb * 64, off + c0 + 32 * b);
            } else {
              tma_load_2d_hint(&tmWd, &bars->full[s], a, kb * 64, e * p.d + mt * 128, pol_w);
              for (int b = 0; b < nb; ++b)
                tma_load_2d(&tmH, &bars->full[s], a + C::kAOff + b * 4096, kb * 64, off + c0 + 32 * b);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      uint32_t it = 0, j = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        bool up;
        int e, mt;
        decode(item, up, e, mt);
        const int n_e = p.offsets[e + 1] - p.offsets[e];
        const int nk = (up ? p.d : p.F) / 64;
        for (int c0 = 0; c0 < n_e && ok; c0 += BN, ++j) {
          const int nmma = (min(BN, n_e - c0) + 15) & ~15;
          const uint32_t idesc = idesc_bf16_f32(128, nmma);
          const uint32_t b = j & 1;
          if (!mbar_wait(&bars->acc_empty[b], ((j >> 1) & 1) ^ 1, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem + b * BN;
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % kStages;
            if (!mbar_wait(&bars->full[s], (it / kStages) & 1, err, DEV_ERR_TIMEOUT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* a = tiles + (size_t)s * kStageBytes;
            const uint64_t ad = smem_desc_sw128(smem_u32(a));
            const uint64_t bd = smem_desc_sw128(smem_u32(a + C::kAOff));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(acc, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0);
            umma_commit(&bars->empty[s]);
          }
          umma_commit(&bars->acc_full[b]);
        }
      }
    }
  } else {
    // ------------------------------ epilogue (warps 2-5) ------------------------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int et = threadIdx.x - 64;
    uint32_t j = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      bool up;
      int e, mt;
      decode(item, up, e, mt);
      const int off = p.offsets[e], n_e = p.offsets[e + 1] - off;
      bool item_ok = true;
      for (int c0 = 0; c0 < n_e; c0 += BN, ++j) {
        const int nc = min(BN, n_e - c0);
        const int nmma = (nc + 15) & ~15;
        const uint32_t b = j & 1;
        const bool ok = mbar_wait(&bars->acc_full[b], (j >> 1) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
        item_ok = item_ok && ok;
        tc_fence_after();
        const uint32_t acc = tmem + ((uint32_t)(quarter * 32) << 16) + b * BN;
        if (up) {
          for (int cs = 0; cs < nmma; cs += kEpiCols) {
            const int ncs = min(kEpiCols, nmma - cs);
            for (int cb = 0; cb < ncs; cb += 32) {
              float v[32];
              tmem_ld_32cols(acc + cs + cb, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) stage_out[r * kEpiStride + cb + i] = v[i];
            }
            if (cs + kEpiCols >= nmma) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->acc_empty[b]);
            }
            epi_bar_sync();
            if (ok) {
              const int fq = (et & 3) * 16;
              const int ncv = min(ncs, nc - cs);
              for (int n = et >> 2; n < ncv; n += 32) {
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                  const float g0 = stage_out[(fq + i) * kEpiStride + n], u0 = stage_out[(64 + fq + i) * kEpiStride + n];
                  const float g1 = stage_out[(fq + i + 1) * kEpiStride + n],
                              u1 = stage_out[(64 + fq + i + 1) * kEpiStride + n];
                  packed[i / 2] = pack_bf16x2(g0 / (1.f + __expf(-g0)) * u0, g1 / (1.f + __expf(-g1)) * u1);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.h_out + (size_t)(off + c0 + cs + n) * p.F + mt * 64 + fq);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
              }
            }
            epi_bar_sync();
          }
        } else {
          const int m = mt * 128 + r;
          for (int cb = 0; cb < nmma; cb += 32) {
            float v[32];
            tmem_ld_32cols(acc + cb, v);
            if (cb + 32 >= nmma) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->acc_empty[b]);
            }
            if (!ok) continue;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int n = cb + i;
              if (n < nc) p.y_out[(size_t)(off + c0 + n) * p.d + m] = v[i];
            }
          }
        }
      }
      if (up) {
        // this tile's SwiGLU rows of expert e are written: count them for e's down items
        __threadfence();
        epi_bar_sync();
        if (et == 0 && item_ok) red_release_gpu_add(done + e, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 2 * BN);
}

// ---------------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------------
template <int BN, int EPI, int Z>
static cudaError_t launch_dense(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, const EpiParams& ep,
                                int* err, cudaStream_t st) {
  using C = DenseCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(dense_gemm_kernel<BN, EPI, Z>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // all of the unified L1/shared storage as shared memory, so kMinBlocks CTAs fit on an SM
    e = cudaFuncSetAttribute(dense_gemm_kernel<BN, EPI, Z>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_k(dense_gemm_kernel<BN, EPI, Z>, dim3((M + 127) / 128, (N + BN - 1) / BN, Z), dim3(kGemmThreads),
                  C::kSmemBytes, st, Z, a, b, M, N, K, ep, err);
}

cudaError_t gemm_dense(int bn, int epi, const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const EpiParams& ep, int* err, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (K % 64 != 0) return cudaErrorInvalidValue;
  const int z = ep.k_splits > 1 ? ep.k_splits : 1;
  if (z > K / 64) return cudaErrorInvalidValue;
  if (z > 1 && (!ep.part || (long long)((M + 127) / 128) * ((N + bn - 1) / bn) * z > ep.part_slots || bn != 128))
    return cudaErrorInvalidValue;   // the split-K scratch holds part_slots [128][128] tiles
  if (ep.rw && (epi != EPI_RESID || bn != 128 || N % 128 || ep.ldo != N || ep.n_exp <= 0 || ep.n_exp % 8 ||
                ep.n_exp > 128 || !ep.rg || !ep.rpart || !ep.ssq))
    return cudaErrorInvalidValue;   // the folded router: whole 128-column tiles, 8-expert groups
#define DG_DENSE_CASE(BN_, EPI_, Z_) \
  if (bn == BN_ && epi == EPI_ && z == Z_) return launch_dense<BN_, EPI_, Z_>(a, b, M, N, K, ep, err, st);
  DG_DENSE_CASE(128, EPI_QKV, 1)
  DG_DENSE_CASE(128, EPI_QKV, 2)
  DG_DENSE_CASE(128, EPI_QKV, 4)
  DG_DENSE_CASE(128, EPI_QKV, 8)
  DG_DENSE_CASE(128, EPI_RESID, 1)
  DG_DENSE_CASE(128, EPI_RESID, 2)
  DG_DENSE_CASE(128, EPI_RESID, 4)
  DG_DENSE_CASE(128, EPI_RESID, 8)
  DG_DENSE_CASE(128, EPI_F32, 1)
  DG_DENSE_CASE(128, EPI_F32, 2)
  DG_DENSE_CASE(128, EPI_F32, 4)
  DG_DENSE_CASE(128, EPI_F32, 8)
  DG_DENSE_CASE(256, EPI_F32, 1)
#undef DG_DENSE_CASE
  return cudaErrorInvalidValue;
}

template <int MODE, int BN, bool FP8>
static cudaError_t launch_expert(const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                                 int n_ctas, int* err, cudaStream_t st) {
  using C = ExpCfg<BN, FP8>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<MODE, BN, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(expert_gemm_kernel<MODE, BN, FP8>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int items = n_exp * (MODE == 1 ? p.F / 64 : p.d / 128);
  return launch_k(expert_gemm_kernel<MODE, BN, FP8>, dim3(n_ctas < items ? n_ctas : items),
                  dim3(FP8 ? kExpThreadsFp8 : kExpThreads), C::kSmemBytes, st, 1, w, x, p, n_exp, err);
}

cudaError_t gemm_expert_updown(const CUtensorMap& wu, const CUtensorMap& x, const CUtensorMap& wd, const CUtensorMap& h,
                               const ExpertParams& p, int n_exp, int n_ctas, int* done, int* err, cudaStream_t st) {
  if (p.w_scale || !done || p.d % 128 || p.F % 64) return cudaErrorInvalidValue;
  using C = ExpCfg<64, false>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(expert_updown_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(expert_updown_kernel<64>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int items = n_exp * (p.F / 64 + p.d / 128);
  return launch_k(expert_updown_kernel<64>, dim3(n_ctas < items ? n_ctas : items), dim3(kExpThreads), C::kSmemBytes,
                  st, 1, wu, x, wd, h, p, n_exp, done, err);
}

// wide = 1: 256-token accumulator chunks (many tokens per expert); 0: 64-token chunks.  p.w_scale
// != nullptr: the weights are e4m3 with one fp32 scale per 128 x 128 tile (w is a byte map).
cudaError_t gemm_expert(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                        int n_ctas, int wide, int* err, cudaStream_t st) {
  const bool f8 = p.w_scale != nullptr;
  // chunk width: 256 (wide), else 64 tokens for bf16 weights and 32 for FP8 (smaller slots, so the
  // e4m3 ring keeps enough weight bytes in flight)
  const int bn = wide ? 256 : (f8 ? 32 : 64);
#define DG_EXPERT_CASE(M_, BN_, F8_) \
  if (mode == M_ && bn == BN_ && f8 == F8_) return launch_expert<M_, BN_, F8_>(w, x, p, n_exp, n_ctas, err, st);
  DG_EXPERT_CASE(1, 64, false)
  DG_EXPERT_CASE(2, 64, false)
  DG_EXPERT_CASE(1, 256, false)
  DG_EXPERT_CASE(2, 256, false)
  DG_EXPERT_CASE(1, 32, true)
  DG_EXPERT_CASE(2, 32, true)
  DG_EXPERT_CASE(1, 256, true)
  DG_EXPERT_CASE(2, 256, true)
#undef DG_EXPERT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dg
