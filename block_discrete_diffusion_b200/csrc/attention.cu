// attention.cu -- canvas attention on tcgen05.
//
// Every canvas row attends to all committed-prefix keys [0, P) and to all canvas keys (no mask
// inside the canvas): bidirectional attention inside the current block with the prompt and the
// committed blocks held as cache ("Dual attention of prefill and denoising" in the diffusion-gemma
// developer guide; the block-diagonal training mask in "Composition of DiffusionGemma" of the
// technical-report summary).  Prompt prefill uses the same kernel with a causal mask.
//
// Grid: (query tile, key split, sequence x KV head).  A CTA owns 128 query rows of one GQA group
// (the n_q/n_kv query heads that share a KV head are adjacent in the head-major query buffer, so a
// 128-row tile is one TMA box) and a contiguous run of 128-key tiles.  Per key tile:
//   S = Q K^T            (tcgen05, M=128 queries, N=128 keys, K=dh) -> TMEM
//   online softmax       (one thread per query row, exp2 domain, fp32) -> P bf16 in swizzled smem
//   O_t = P V            (tcgen05, M=128, N=dh, K=128 keys; V is cached transposed so both
//                         operands are K-major) -> TMEM, folded into fp32 registers with the
//                         running rescale.
// Splits write un-normalised (O, m, l) partials; attn_merge_kernel combines them.
#include <math.h>

#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

template <int DH>
struct AttnCfg {
  static constexpr uint32_t kQBytes = 128u * DH * 2u;
  static constexpr uint32_t kKBytes = 128u * DH * 2u;
  static constexpr uint32_t kVBytes = (uint32_t)DH * 128u * 2u;
  static constexpr uint32_t kPBytes = 128u * 128u * 2u;
  static constexpr int kStages = 2;
  static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
  static constexpr uint32_t kTmemCols = 256;   // S in [0,128), O in [128, 128+DH)
  static constexpr size_t kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kPBytes + 256;
};

struct AttnBarriers {
  uint64_t qfull;
  uint64_t kvfull[2];
  uint64_t s_done;
  uint64_t o_done;
  uint32_t tmem_slot;
};

template <int DH>
__device__ __forceinline__ void attn_issue_kv(const CUtensorMap* tk, const CUtensorMap* tv, AttnBarriers* b,
                                              uint8_t* stage, int s, int tile, int z) {
  using C = AttnCfg<DH>;
  mbar_arrive_expect_tx(&b->kvfull[s], C::kStageBytes);
#pragma unroll
  for (int h = 0; h < DH / 64; ++h) tma_load_3d(tk, &b->kvfull[s], stage + h * 16384, h * 64, tile * 128, z);
#pragma unroll
  for (int hk = 0; hk < 2; ++hk)
    tma_load_3d(tv, &b->kvfull[s], stage + C::kKBytes + hk * (DH * 128), tile * 128 + hk * 64, 0, z);
}

template <int DH>
__global__ void __launch_bounds__(128, 1)
    attn_partial_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, AttnParams p, int n_seq, int* err) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = base;
  uint8_t* kv_s = q_s + C::kQBytes;
  uint8_t* p_s = kv_s + C::kStages * C::kStageBytes;
  AttnBarriers* bars = reinterpret_cast<AttnBarriers*>(p_s + C::kPBytes);

  const int warp = threadIdx.x >> 5;
  const int qt = blockIdx.x, split = blockIdx.y;
  const int seq = blockIdx.z / p.n_kv, kvh = blockIdx.z % p.n_kv;
  const int G = p.n_q / p.n_kv;
  const int cseq = p.seq_base + seq;
  pdl_trigger();

  if (threadIdx.x == 0) {
    mbar_init(&bars->qfull, 1);
    mbar_init(&bars->kvfull[0], 1);
    mbar_init(&bars->kvfull[1], 1);
    mbar_init(&bars->s_done, 1);
    mbar_init(&bars->o_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&bars->tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  pdl_wait();   // queries, keys, values and P come from the preceding kernels

  const int P = p.seq_P[cseq];
  const int nkeys = P + p.Tq;
  const int ntiles = (nkeys + 127) >> 7;
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(ntiles, t0 + p.tiles_per_split);

  // this thread's query row
  const int rr = qt * 128 + threadIdx.x;
  const int g = rr / p.rows_per_seq, j = rr % p.rows_per_seq;
  const int h = kvh * G + g;
  const bool row_valid = (g < G) && (j < p.Tq);
  const int qpos = P + j;
  const size_t prow = ((size_t)(split * n_seq + seq) * p.n_q + h) * p.rows_per_seq + j;

  if (t0 >= t1) {   // empty split: neutral partial
    if (row_valid) {
      p.ml[prow * 2 + 0] = -INFINITY;
      p.ml[prow * 2 + 1] = 0.f;
      float4* o4 = reinterpret_cast<float4*>(p.opart + prow * DH);
      for (int c = 0; c < DH / 4; ++c) o4[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
    return;
  }

  const int qrow0 = (seq * p.n_q + kvh * G) * p.rows_per_seq + qt * 128;
  const int z = p.layer * p.cache_seq_stride + cseq * p.n_kv + kvh;
  const uint32_t t_s = tmem + ((uint32_t)(warp * 32) << 16);
  const uint32_t t_o = t_s + 128;

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars->qfull, C::kQBytes);
#pragma unroll
    for (int hh = 0; hh < DH / 64; ++hh) tma_load_2d(&tq, &bars->qfull, q_s + hh * 16384, hh * 64, qrow0);
    for (int t = t0; t < min(t1, t0 + C::kStages); ++t)
      attn_issue_kv<DH>(&tk, &tv, bars, kv_s + (size_t)((t - t0) % C::kStages) * C::kStageBytes,
                        (t - t0) % C::kStages, t, z);
  }

  const float sl2 = 1.4426950408889634f * rsqrtf((float)DH);
  float o[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  bool ok = true;

  for (int t = t0; t < t1; ++t) {
    const int it = t - t0;
    const int s = it % C::kStages;
    uint8_t* stage = kv_s + (size_t)s * C::kStageBytes;
    if (threadIdx.x == 0 && ok) {
      if (it == 0) ok = mbar_wait(&bars->qfull, 0, err, DEV_ERR_TIMEOUT_ATTN);
      if (ok) ok = mbar_wait(&bars->kvfull[s], (it / C::kStages) & 1, err, DEV_ERR_TIMEOUT_ATTN);
      tc_fence_after();
      if (ok) {
        const uint32_t idesc = idesc_bf16_f32(128, 128);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint64_t ad = desc_advance(smem_desc_sw128(smem_u32(q_s + (kk / 4) * 16384)), (kk % 4) * 32);
          const uint64_t bd = desc_advance(smem_desc_sw128(smem_u32(stage + (kk / 4) * 16384)), (kk % 4) * 32);
          umma_bf16(tmem, ad, bd, idesc, kk != 0);
        }
      }
      umma_commit(&bars->s_done);
    }
    __syncwarp();
    ok = mbar_wait(&bars->s_done, it & 1, err, DEV_ERR_TIMEOUT_ATTN) && ok;
    tc_fence_after();

    // ---- online softmax of this thread's row over the 128 keys of tile t ----
    const int key0 = t * 128;
    int kmax = nkeys - key0;                       // keys [key0, key0 + kmax) exist
    if (p.causal) kmax = min(kmax, qpos - key0 + 1);
    float tmax = -INFINITY;
#pragma unroll
    for (int cb = 0; cb < 128; cb += 32) {
      float v[32];
      tmem_ld_32cols(t_s + cb, v);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (cb + i < kmax) tmax = fmaxf(tmax, v[i] * sl2);
    }
    const float m_new = fmaxf(m, tmax);
    const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m - m_new);
    float lt = 0.f;
#pragma unroll
    for (int cb = 0; cb < 128; cb += 32) {
      float v[32];
      tmem_ld_32cols(t_s + cb, v);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float p0 = (cb + i < kmax) ? fast_exp2(v[i] * sl2 - m_new) : 0.f;
        float p1 = (cb + i + 1 < kmax) ? fast_exp2(v[i + 1] * sl2 - m_new) : 0.f;
        __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
        lt += __low2float(b2) + __high2float(b2);
        pk[i / 2] = *reinterpret_cast<uint32_t*>(&b2);
      }
      // keys [cb, cb+32) of row threadIdx.x -> 4 swizzled 16-byte chunks
      const int r = threadIdx.x;
      uint8_t* prow_s = p_s + (cb / 64) * 16384 + r * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int chunk = ((cb % 64) / 8) + ch;
        *reinterpret_cast<uint4*>(prow_s + ((chunk ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
    }
    l = l * alpha + lt;
    m = m_new;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    if (threadIdx.x == 0) {
      tc_fence_after();
      if (ok) {
        const uint32_t idesc = idesc_bf16_f32(128, DH);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = desc_advance(smem_desc_sw128(smem_u32(p_s + (kk / 4) * 16384)), (kk % 4) * 32);
          const uint64_t bd =
              desc_advance(smem_desc_sw128(smem_u32(stage + C::kKBytes + (kk / 4) * (DH * 128))), (kk % 4) * 32);
          umma_bf16(tmem + 128, ad, bd, idesc, kk != 0);
        }
      }
      umma_commit(&bars->o_done);
    }
    __syncwarp();
    ok = mbar_wait(&bars->o_done, it & 1, err, DEV_ERR_TIMEOUT_ATTN) && ok;
    tc_fence_after();
#pragma unroll
    for (int cb = 0; cb < DH; cb += 32) {
      float v[32];
      tmem_ld_32cols(t_o + cb, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[cb + i] = o[cb + i] * alpha + v[i];
    }
    tc_fence_before();
    __syncthreads();
    // stage s is free again (both MMAs that read it have completed): prefetch tile t + kStages
    if (threadIdx.x == 0 && ok && t + C::kStages < t1) attn_issue_kv<DH>(&tk, &tv, bars, stage, s, t + C::kStages, z);
  }

  if (row_valid && ok) {
    p.ml[prow * 2 + 0] = m;
    p.ml[prow * 2 + 1] = l;
    float4* o4 = reinterpret_cast<float4*>(p.opart + prow * DH);
#pragma unroll
    for (int c = 0; c < DH / 4; ++c) o4[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

// One warp per (sequence, query head, row): combine the split partials (lane s < n_splits holds
// split s's (m, l)) and write the row of the token-major attention output
// [seq*rows_per_seq + j][h*dh + c] in bf16; each lane owns dh/32 consecutive columns.
template <int DH>
__global__ void attn_merge_kernel(AttnParams p, int n_seq, __nv_bfloat16* out) {
  pdl_trigger();
  pdl_wait();
  const int warp = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (warp >= n_seq * p.n_q * p.Tq) return;
  const int j = warp % p.Tq;
  const int sh = warp / p.Tq;          // seq * n_q + h
  const int seq = sh / p.n_q, h = sh % p.n_q;
  const size_t stride = (size_t)n_seq * p.n_q * p.rows_per_seq;
  const size_t r0 = (size_t)sh * p.rows_per_seq + j;
  float ms = -INFINITY, ls = 0.f;
  if (lane < p.n_splits) {
    const float2 v = *reinterpret_cast<const float2*>(p.ml + (lane * stride + r0) * 2);
    ms = v.x;
    ls = v.y;
  }
  const float M = warp_max(ms);
  const float wgt = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
  const float den = warp_sum(wgt * ls);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  constexpr int kPer = DH / 32;
  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
  for (int s = 0; s < p.n_splits; ++s) {
    const float ws = __shfl_sync(0xffffffffu, wgt, s);
    if (ws == 0.f) continue;
    const float* src = p.opart + (s * stride + r0) * DH + lane * kPer;
    if constexpr (kPer == 4) {
      const float4 v = *reinterpret_cast<const float4*>(src);
      acc[0] += ws * v.x; acc[1] += ws * v.y; acc[2] += ws * v.z; acc[3] += ws * v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(src);
      acc[0] += ws * v.x; acc[1] += ws * v.y;
    }
  }
  __nv_bfloat16* dst = out + ((size_t)seq * p.rows_per_seq + j) * (p.n_q * DH) + h * DH + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
}

template <int DH>
static cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const AttnParams& p, int n_seq, int* err, cudaStream_t st) {
  using C = AttnCfg<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_partial_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int G = p.n_q / p.n_kv;
  dim3 grid((G * p.rows_per_seq + 127) / 128, p.n_splits, n_seq * p.n_kv);
  return launch_k(attn_partial_kernel<DH>, grid, dim3(128), C::kSmemBytes, st, 1, tq, tk, tv, p, n_seq, err);
}

cudaError_t attention_partial(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const AttnParams& p, int n_seq, int* err, cudaStream_t st) {
  if (p.dh == 128) return launch_attn<128>(tq, tk, tv, p, n_seq, err, st);
  if (p.dh == 64) return launch_attn<64>(tq, tk, tv, p, n_seq, err, st);
  return cudaErrorInvalidValue;
}

cudaError_t attention_merge(const AttnParams& p, int n_seq, __nv_bfloat16* out, cudaStream_t st) {
  if (p.n_splits > 32) return cudaErrorInvalidValue;
  const int rows = n_seq * p.n_q * p.Tq;
  const int blocks = (rows + 7) / 8;
  if (p.dh == 128) return launch_k(attn_merge_kernel<128>, dim3(blocks), dim3(256), 0, st, 1, p, n_seq, out);
  if (p.dh == 64) return launch_k(attn_merge_kernel<64>, dim3(blocks), dim3(256), 0, st, 1, p, n_seq, out);
  return cudaErrorInvalidValue;
}

}  // namespace dg
