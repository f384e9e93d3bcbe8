// head_sampler.cu -- the vocabulary head fused with the sampler's per-row reductions (one canvas).
//
// One denoising step ends with the final RMSNorm, the vocabulary projection and the sampler: the
// tempered softmax's entropy, the Gumbel-max draw and the step rule ("Composition of DiffusionGemma",
// sampler settings, in the technical-report summary; the entropy_bound sampler of "Serving with
// vLLM" in the diffusion-gemma developer guide).  The sampler only needs, per canvas row, the
// softmax statistics (max m, S = sum 2^(z2 - m), A = sum 2^(z2 - m)(z2 - m) in the exp2 domain)
// and the best perturbed score with its index; those reduce over any split of the vocabulary.
// This kernel computes the logits of one canvas tile by tile in tensor memory and folds every tile
// straight into those per-row reductions, so the [256][vocab] fp32 logits are never written to
// (or read back from) HBM.
//
// Layout: the 256 canvas rows are the MMA's M side (two 128-row tiles, A = the normed hidden state,
// re-read from L2 for every item), a tile of NV vocabulary rows of the head is the N side (B,
// streamed from HBM once).  Items are vocabulary tiles, dealt round-robin to one CTA per SM.
// Warp 0 loads (TMA, 128-byte swizzle, one ring of stages that runs across items), warp 1 issues
// tcgen05.mma into TMEM, warps 2-9 are the sampler: warp w reads TMEM lanes 32 (w % 4) .. of token
// tile (w - 2) / 4, so each thread owns one canvas row and walks its vocabulary columns in increasing
// order, 32 per tcgen05.ld, keeping that row's running statistics and best draw in registers over
// every item of the CTA.  At the end each thread writes one partial record of its row; the
// sampler's finalize kernel merges the records of all CTAs and applies the step rule.
//   NV = 128: two accumulators of 2 x 128 columns, the sampler on one item overlaps the MMAs of the
//             next (the token tiles are read from L2 once per 128 vocabulary rows);
//   NV = 256: one accumulator of 2 x 256 columns (all of TMEM): the token tiles are read once per
//             256 vocabulary rows, the loads of the next item run ahead while the sampler drains.
// The Gumbel draws follow the stream layout of philox.cuh and the exact pruning of the standalone
// sampler (sampler.cu), with a per-row bound instead of a warp-wide one.
#include <math.h>

#include "dg_device.cuh"
#include "dg_kernels.h"
#include "philox.cuh"

namespace dg {

namespace {

constexpr int kHsThreads = 320;                    // 10 warps: producer, MMA, 8 sampler warps
constexpr uint32_t kHsATile = 128 * 64 * 2;        // 128 canvas rows x 64 k (bf16)
constexpr float kLog2eH = 1.4426950408889634f;

template <int NV>
struct HsCfg {
  static constexpr uint32_t kBTile = NV * 64 * 2;
  static constexpr uint32_t kStage = 2 * kHsATile + kBTile;
  static constexpr int kStages = NV == 128 ? 4 : 3;
  static constexpr int kAcc = NV == 128 ? 2 : 1;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStage + 256;
  static_assert(2 * NV * kAcc == 512, "the accumulators fill TMEM exactly");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct HsBarriers {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_slot;
};

// Running sampler state of one canvas row (thread-local).
struct RowState {
  float m;        // running max of z * log2(e)
  uint64_t S2;    // two lanes of sum 2^(z2 - m)
  uint64_t A2;    // two lanes of sum 2^(z2 - m) (z2 - m)
  float best;     // best accurate perturbed score z + g seen so far
  int bidx;       // its vocabulary index
  float lim;      // a score some element of this row reaches (pruning bound)
};

// Fold 16 consecutive logits v[0..16) of columns v0 .. v0 + 15 (v0 % 4 == 0) into the row state.
__device__ __forceinline__ void absorb16(RowState& st, const float* v, int v0, float inv_temp, float s2,
                                         uint32_t pos, uint32_t step, uint32_t k0, uint32_t k1) {
  float gmax[4], gabs[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    gmax[g] = fmaxf(fmaxf(v[4 * g], v[4 * g + 1]), fmaxf(v[4 * g + 2], v[4 * g + 3]));
    gabs[g] = fmaxf(fmaxf(fabsf(v[4 * g]), fabsf(v[4 * g + 1])), fmaxf(fabsf(v[4 * g + 2]), fabsf(v[4 * g + 3])));
  }
  // softmax statistics: one rescale per 16 values
  const float bm = fmaxf(fmaxf(gmax[0], gmax[1]), fmaxf(gmax[2], gmax[3])) * s2;
  if (bm > st.m) {
    if (st.m != -INFINITY) {
      const float f = fast_exp2(st.m - bm);
      st.A2 = fmul_f32x2(ffma_f32x2(st.S2, pack_f32x2(st.m - bm, st.m - bm), st.A2), pack_f32x2(f, f));
      st.S2 = fmul_f32x2(st.S2, pack_f32x2(f, f));
    }
    st.m = bm;
  }
  const uint64_t s2p = pack_f32x2(s2, s2), negm = pack_f32x2(-st.m, -st.m);
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    const uint64_t t01 = ffma_f32x2(pack_f32x2(v[i], v[i + 1]), s2p, negm);
    const uint64_t t23 = ffma_f32x2(pack_f32x2(v[i + 2], v[i + 3]), s2p, negm);
    const uint64_t e01 = pack_f32x2(fast_exp2(lo_f32(t01)), fast_exp2(hi_f32(t01)));
    const uint64_t e23 = pack_f32x2(fast_exp2(lo_f32(t23)), fast_exp2(hi_f32(t23)));
    st.S2 = fadd_f32x2(st.S2, fadd_f32x2(e01, e23));
    st.A2 = ffma_f32x2(e23, t23, ffma_f32x2(e01, t01, st.A2));
  }
  // Gumbel draws screened with hardware logarithms.  The four Philox blocks are computed without a
  // branch (straight-line code, so their rounds overlap: one thread per row leaves little else to hide
  // their latency); a group that cannot reach the bound even with the largest draw is masked out after.
  const float kSkip = __int_as_float(0x7fffffff);   // NaN: compares false, marks draws not taken
  uint4 w4[4];
#pragma unroll
  for (int g = 0; g < 4; ++g)
    w4[g] = philox4x32_10(make_uint4((uint32_t)((v0 >> 2) + g), pos, step, RNG_TAG_GUMBEL), k0, k1);
  float fs[4][4];
  float fmax_ = -INFINITY;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const bool take = __fmaf_rn(gmax[g], inv_temp, kGumbelMax) >= st.lim;
    const bool screen = gabs[g] * inv_temp <= kScreenMaxZ;
    const uint32_t ww[4] = {w4[g].x, w4[g].y, w4[g].z, w4[g].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float uu = u01_open(ww[i]);
      const float f = gumbel_screen_score(v[4 * g + i], inv_temp, uu);
      const bool exact_only = !screen || uu >= kGumbelFastMaxU;
      fs[g][i] = !take ? kSkip : (exact_only ? INFINITY : f);
      fmax_ = fmaxf(fmax_, (take && !exact_only) ? f : -INFINITY);
    }
  }
  // every screened score minus two slacks is below that element's accurate score
  st.lim = fmaxf(st.lim, fmax_ - 2.f * kGumbelFastSlack);
  // accurate scores only where the screened score reaches the bound, in increasing index order (the
  // strict comparison keeps the lowest index among equal scores)
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    if (fs[g][0] >= st.lim || fs[g][1] >= st.lim || fs[g][2] >= st.lim || fs[g][3] >= st.lim) {
      const uint32_t ww[4] = {w4[g].x, w4[g].y, w4[g].z, w4[g].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (fs[g][i] >= st.lim) {
          const float sc = __fmaf_rn(v[4 * g + i], inv_temp, gumbel_from_word(ww[i]));
          if (sc > st.best) {
            st.best = sc;
            st.bidx = v0 + 4 * g + i;
          }
        }
      }
    }
  }
  st.lim = fmaxf(st.lim, st.best);
}

template <int NV>
__global__ void __launch_bounds__(kHsThreads, 1)
    head_sampler_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        HeadSamplerArgs p, int* err) {
  using C = HsCfg<NV>;
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  HsBarriers* bars = reinterpret_cast<HsBarriers*>(tiles + (size_t)C::kStages * C::kStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.d / 64;
  const int n_items = p.vocab / NV;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < C::kAcc; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 8);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();   // head rows are read once per step
      // the head does not depend on the preceding kernels: its first stages load before the wait
      const int first = blockIdx.x;
      const int npre = first < n_items ? (nk < C::kStages ? nk : C::kStages) : 0;
      for (int kb = 0; kb < npre; ++kb) {
        uint8_t* a = tiles + (size_t)kb * C::kStage;
        mbar_expect_tx(&bars->full[kb], C::kBTile);
        tma_load_2d_hint(&tmB, &bars->full[kb], a + 2 * kHsATile, kb * 64, first * NV, pol_w);
      }
      pdl_wait();   // the normed hidden state comes from the preceding kernel
      for (int kb = 0; kb < npre; ++kb) {
        uint8_t* a = tiles + (size_t)kb * C::kStage;
        mbar_arrive_expect_tx(&bars->full[kb], 2 * kHsATile);
        tma_load_2d(&tmA, &bars->full[kb], a, kb * 64, p.row0);
        tma_load_2d(&tmA, &bars->full[kb], a + kHsATile, kb * 64, p.row0 + 128);
      }
      uint32_t it = 0;
      bool ok = true;
      for (int item = first; item < n_items && ok; item += gridDim.x) {
        for (int kb = 0; kb < nk; ++kb, ++it) {
          if (it < (uint32_t)npre) continue;
          const int s = it % C::kStages;
          if (!mbar_wait(&bars->empty[s], ((it / C::kStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* a = tiles + (size_t)s * C::kStage;
          mbar_arrive_expect_tx(&bars->full[s], C::kStage);
          tma_load_2d(&tmA, &bars->full[s], a, kb * 64, p.row0);
          tma_load_2d(&tmA, &bars->full[s], a + kHsATile, kb * 64, p.row0 + 128);
          tma_load_2d_hint(&tmB, &bars->full[s], a + 2 * kHsATile, kb * 64, item * NV, pol_w);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    pdl_wait();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NV);
      uint32_t it = 0, j = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++j) {
        const uint32_t b = j % C::kAcc;
        if (!mbar_wait(&bars->acc_empty[b], ((j / C::kAcc) & 1) ^ 1, err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&bars->full[s], (it / C::kStages) & 1, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* a = tiles + (size_t)s * C::kStage;
          const uint64_t bd = smem_desc_sw128(smem_u32(a + 2 * kHsATile));
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t ad = smem_desc_sw128(smem_u32(a + h * kHsATile));
            const uint32_t acc = tmem + b * (2 * NV) + h * NV;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(acc, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0);
          }
          umma_commit(&bars->empty[s]);
        }
        if (ok) umma_commit(&bars->acc_full[b]);
      }
    }
  } else {
    // ------------------------------ sampler (warps 2-9) ------------------------------
    pdl_wait();   // commit mask and committed lengths come from the preceding kernels
    const int q = warp & 3;                     // TMEM lane quadrant this warp may read
    const int h = (warp - 2) >> 2;              // token tile
    const int row = h * 128 + q * 32 + lane;    // canvas row of this thread
    const bool active = !p.commit_in[row];
    const uint32_t pos = (uint32_t)((p.seq_P ? p.seq_P[0] : 0) + row);
    const uint32_t k0 = (uint32_t)p.seed, k1 = (uint32_t)(p.seed >> 32);
    int step = p.step;
    float inv_temp = p.inv_temp;
    if (p.d_step) {   // step index kept on the device: this step's index and temperature
      step = *p.d_step;
      inv_temp = __fdiv_rn(1.0f, schedule_temperature(p.t_start, p.t_end, p.max_steps, step));
    }
    const float s2 = inv_temp * kLog2eH;
    RowState st{-INFINITY, 0ull, 0ull, -INFINITY, 0x7fffffff, -INFINITY};
    uint32_t j = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
      const uint32_t b = j % C::kAcc;
      ok = ok && mbar_wait(&bars->acc_full[b], (j / C::kAcc) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
      tc_fence_after();
      const uint32_t acc = tmem + ((uint32_t)(q * 32) << 16) + b * (2 * NV) + h * NV;
      // one copy of the chunk body (kept rolled: the unrolled chunks overflow the instruction cache)
#pragma unroll 1
      for (int c = 0; c < NV; c += 32) {
        float v[32];
        tmem_ld_32cols(acc + c, v);
        if (c + 32 >= NV) {                     // last TMEM read of this accumulator: release it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->acc_empty[b]);
        }
        if (!ok) continue;
        const int v0 = item * NV + c;
        if (p.logits_out) {
          float4* dst = reinterpret_cast<float4*>(p.logits_out + (size_t)row * p.vocab + v0);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        if (active) {
          absorb16(st, v, v0, inv_temp, s2, pos, (uint32_t)step, k0, k1);
          absorb16(st, v + 16, v0 + 16, inv_temp, s2, pos, (uint32_t)step, k0, k1);
        }
      }
    }
    if (ok && active) {
      float* out = p.partial + ((size_t)row * gridDim.x + blockIdx.x) * 8;
      out[0] = st.m;
      out[1] = lo_f32(st.S2) + hi_f32(st.S2);
      out[2] = lo_f32(st.A2) + hi_f32(st.A2);
      out[3] = st.best;
      out[4] = __int_as_float(st.bidx);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------------------------
// CTA-pair form (tcgen05 cta_group::2): a pair of CTAs on two SMs computes 256 canvas rows x 256
// vocabulary rows per item with M = 256 MMAs.  Each CTA holds its own 128 canvas rows (A) and half of
// the item's head rows (B); the leader CTA (rank 0 of the cluster) issues the MMAs, which read both
// CTAs' shared memory and write each CTA's 128 rows into that CTA's tensor memory.  Per SM this halves
// the stage (32 KB: 16 KB of canvas rows, 16 KB of head rows) and the canvas rows re-read from L2 per
// vocabulary row, so more weight bytes are in flight; two 256-column accumulators per CTA keep the
// sampler of one item overlapping the MMAs of the next.  Loads of both CTAs complete on the leader's
// barriers; the leader's commits arrive in both CTAs; the peer's sampler warps release accumulators
// on the leader's barrier.  Every wait is bounded.
// ---------------------------------------------------------------------------------------------
constexpr int kHpStages = 6;
constexpr uint32_t kHpStage = 2 * kHsATile;                   // 128 canvas rows + 128 head rows, 64 k
constexpr size_t kHpSmem = 1024 + (size_t)kHpStages * kHpStage + 256;
static_assert(kHpSmem <= 232448, "shared memory budget");

struct HpBarriers {
  uint64_t full[kHpStages];
  uint64_t empty[kHpStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_slot;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kHsThreads, 1)
    head_sampler_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             HeadSamplerArgs p, int* err) {
  constexpr int NV = 256;                       // vocabulary rows per item (128 per CTA)
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  HpBarriers* bars = reinterpret_cast<HpBarriers*>(tiles + (size_t)kHpStages * kHpStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();      // 0: leader, 1: peer
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int nk = p.d / 64;
  const int n_items = p.vocab / NV;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kHpStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 16);       // the sampler warps of both CTAs
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(&bars->tmem_slot, 512);
  tc_fence_before();
  cluster_sync();                               // both CTAs' barriers and tensor memory exist
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  const uint32_t lead_full0 = dsmem_map(smem_u32(&bars->full[0]), 0);
  const uint32_t lead_acc_empty0 = dsmem_map(smem_u32(&bars->acc_empty[0]), 0);

  if (warp == 0) {
    // ------------------------------ TMA producer (both CTAs) ------------------------------
    if (lane == 0) {
      pdl_wait();                               // the normed hidden state comes from the preceding kernel
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_a = l2_policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int item = pair; item < n_items && ok; item += n_pairs) {
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kHpStages;
          if (!mbar_wait(&bars->empty[s], ((it / kHpStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* a = tiles + (size_t)s * kHpStage;
          if (rank == 0) mbar_arrive_expect_tx(&bars->full[s], 2 * kHpStage);   // both CTAs' bytes
          const uint32_t bar = lead_full0 + (uint32_t)(s * sizeof(uint64_t));
          tma_load_2d_pair(&tmA, bar, a, kb * 64, p.row0 + (int)rank * 128, pol_a);                       // canvas rows
          tma_load_2d_pair(&tmB, bar, a + kHsATile, kb * 64, item * NV + (int)rank * 128, pol_w);  // head rows
        }
      }
      // tail: every stage released once more, i.e. the leader's last commits (multicast to this CTA)
      // have arrived here before the CTA may leave
      for (int i = 0; i < kHpStages && ok; ++i, ++it)
        ok = mbar_wait(&bars->empty[it % kHpStages], ((it / kHpStages) & 1) ^ 1, err, DEV_ERR_TIMEOUT_PRODUCER);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader) ------------------------------
    if (rank == 0 && lane == 0) {
      pdl_wait();
      constexpr uint32_t idesc = idesc_bf16_f32(256, NV);
      uint32_t it = 0, j = 0;
      bool ok = true;
      for (int item = pair; item < n_items && ok; item += n_pairs, ++j) {
        const uint32_t b = j & 1;
        if (!mbar_wait(&bars->acc_empty[b], ((j >> 1) & 1) ^ 1, err, DEV_ERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kHpStages;
          if (!mbar_wait(&bars->full[s], (it / kHpStages) & 1, err, DEV_ERR_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* a = tiles + (size_t)s * kHpStage;
          const uint64_t ad = smem_desc_sw128(smem_u32(a));
          const uint64_t bd = smem_desc_sw128(smem_u32(a + kHsATile));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_pair(tmem + b * NV, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0);
          umma_commit_pair(&bars->empty[s]);
        }
        if (ok) umma_commit_pair(&bars->acc_full[b]);
      }
    }
  } else {
    // ------------------------------ sampler (warps 2-9 of both CTAs) ------------------------------
    pdl_wait();
    const int q = warp & 3;                     // TMEM lane quadrant this warp may read
    const int ch = (warp - 2) >> 2;             // column half of the 256-column accumulator
    const int row = (int)rank * 128 + q * 32 + lane;
    const bool active = !p.commit_in[row];
    const uint32_t pos = (uint32_t)((p.seq_P ? p.seq_P[0] : 0) + row);
    const uint32_t k0 = (uint32_t)p.seed, k1 = (uint32_t)(p.seed >> 32);
    int step = p.step;
    float inv_temp = p.inv_temp;
    if (p.d_step) {
      step = *p.d_step;
      inv_temp = __fdiv_rn(1.0f, schedule_temperature(p.t_start, p.t_end, p.max_steps, step));
    }
    const float s2 = inv_temp * kLog2eH;
    RowState st{-INFINITY, 0ull, 0ull, -INFINITY, 0x7fffffff, -INFINITY};
    uint32_t j = 0;
    bool ok = true;
    for (int item = pair; item < n_items; item += n_pairs, ++j) {
      const uint32_t b = j & 1;
      ok = ok && mbar_wait(&bars->acc_full[b], (j >> 1) & 1, err, DEV_ERR_TIMEOUT_EPILOGUE);
      tc_fence_after();
      const uint32_t acc = tmem + ((uint32_t)(q * 32) << 16) + b * NV + ch * 128;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        float v[32];
        tmem_ld_32cols(acc + c, v);
        if (c + 32 >= 128) {                    // last TMEM read of this accumulator: release it (leader's barrier)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead_acc_empty0 + b * (uint32_t)sizeof(uint64_t));
        }
        if (!ok) continue;
        const int v0 = item * NV + ch * 128 + c;
        if (p.logits_out) {
          float4* dst = reinterpret_cast<float4*>(p.logits_out + (size_t)row * p.vocab + v0);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        if (active) {
          absorb16(st, v, v0, inv_temp, s2, pos, (uint32_t)step, k0, k1);
          absorb16(st, v + 16, v0 + 16, inv_temp, s2, pos, (uint32_t)step, k0, k1);
        }
      }
    }
    if (ok && active) {
      float* out = p.partial + ((size_t)row * (2 * n_pairs) + 2 * pair + ch) * 8;
      out[0] = st.m;
      out[1] = lo_f32(st.S2) + hi_f32(st.S2);
      out[2] = lo_f32(st.A2) + hi_f32(st.A2);
      out[3] = st.best;
      out[4] = __int_as_float(st.bidx);
    }
  }

  tc_fence_before();
  cluster_sync();                               // no CTA leaves while the pair's MMAs or arrivals may touch it
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

cudaError_t launch_head_sampler_pair(const CUtensorMap& a, const CUtensorMap& b, const HeadSamplerArgs& p, int n_ctas,
                                     int* err, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(head_sampler_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kHpSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(head_sampler_pair_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_ctas);
  cfg.blockDim = dim3(kHsThreads);
  cfg.dynamicSmemBytes = kHpSmem;
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, head_sampler_pair_kernel, a, b, p, err);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int NV>
cudaError_t launch_head_sampler(const CUtensorMap& a, const CUtensorMap& b, const HeadSamplerArgs& p, int n_ctas,
                                int* err, cudaStream_t st) {
  using C = HsCfg<NV>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(head_sampler_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(head_sampler_kernel<NV>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_k(head_sampler_kernel<NV>, dim3(n_ctas), dim3(kHsThreads), C::kSmem, st, 1, a, b, p, err);
}

}  // namespace

int head_sampler_ctas(int vocab, int nv, int n_sms) {
  if (nv == kHeadSamplerPair) {                 // pairs of CTAs, 256 vocabulary rows per pair item
    const int items = vocab / 256;
    const int pairs = (items < n_sms / 2 ? items : n_sms / 2);
    return 2 * pairs;
  }
  const int items = vocab / nv;
  return items < n_sms ? items : n_sms;
}

cudaError_t head_sampler_run(const CUtensorMap& xn_map, const CUtensorMap& head_map, int nv, const HeadSamplerArgs& p,
                             int n_ctas, const SamplerArgs& fin, int* err, cudaStream_t st) {
  if (p.d % 64 || n_ctas <= 0) return cudaErrorInvalidValue;
  cudaError_t e;
  if (nv == kHeadSamplerPair) {
    if (p.vocab % 256 || n_ctas % 2) return cudaErrorInvalidValue;
    e = launch_head_sampler_pair(xn_map, head_map, p, n_ctas, err, st);
  } else {
    if ((nv != 128 && nv != 256) || p.vocab % nv) return cudaErrorInvalidValue;
    e = nv == 128 ? launch_head_sampler<128>(xn_map, head_map, p, n_ctas, err, st)
                  : launch_head_sampler<256>(xn_map, head_map, p, n_ctas, err, st);
  }
  if (e != cudaSuccess) return e;
  // one record per row and CTA: merged one warp per row, then the step rule
  return sampler_premerge_finalize_run(fin, p.partial + (size_t)256 * n_ctas * 8, st);
}

}  // namespace dg
