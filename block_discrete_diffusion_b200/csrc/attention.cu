// attention.cu -- canvas attention on tcgen05.
//
// Every canvas row attends to all committed-prefix keys [0, P) and to all canvas keys (no mask
// inside the canvas): bidirectional attention inside the current block with the prompt and the
// committed blocks held as cache ("Dual attention of prefill and denoising" in the diffusion-gemma
// developer guide; the block-diagonal training mask in "Composition of DiffusionGemma" of the
// technical-report summary).  Prompt prefill uses the same kernel with a causal mask.
//
// Grid: (query-tile pair, key split, sequence x KV head).  A CTA owns two 128-row query tiles of
// one GQA group (the n_q/n_kv query heads that share a KV head are adjacent in the head-major query
// buffer) and a contiguous run of 128-key tiles, so every K/V tile it loads serves 256 query rows.
// Warp roles (320 threads):
//   warp 8      TMA producer: both Q tiles once, then K(t), V(t), K(t+1), ... through a 3-buffer ring
//   warp 9      MMA issuer:   S_x = Q_x K^T into TMEM, O_x += P_x V into TMEM, in the order
//               S_0(0) S_1(0) | PV_0(t) S_0(t+1) PV_1(t) S_1(t+1) ..., so the tensor core works on
//               one tile's products while the other tile's softmax runs
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1 (thread = query row): S from TMEM,
//               row max, P = exp2(S - m) in bf16 to swizzled shared memory, running sum
// The running max is updated lazily: O (in TMEM) and the sum are rescaled only when a row's max
// grows by more than 2^8, so P stays below 256 and most tiles need no rescale; the final O / l is
// the same.  With one key split the normalised row is written straight to the attention output;
// otherwise un-normalised (O, m, l) partials go to attn_merge_kernel.
#include <math.h>

#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

template <int DH>
struct AttnCfg {
  static constexpr uint32_t kTileBytes = 128u * DH * 2u;   // a Q tile, a K tile or a V tile (DH x 128 keys)
  static constexpr uint32_t kPBytes = 128u * 128u * 2u;    // P: 128 rows x 128 keys, bf16
  static constexpr int kBufs = 3;                          // K / V ring
  static constexpr uint32_t kTmemCols = 512;               // S0 [0,128) S1 [128,256) O0 [256,..) O1 [384,..)
  static constexpr size_t kSmemBytes = 1024 + 2 * kTileBytes + kBufs * kTileBytes + 2 * kPBytes + 256;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};
constexpr int kAttnThreads = 320;
constexpr float kLazyRescale = 8.f;   // log2 units: rescale O only when the max grows by more than this

struct AttnBarriers {
  uint64_t q_full;
  uint64_t kv_full[3], kv_empty[3];
  uint64_t s_full[2], s_free[2], p_ready[2], pv_done[2];
  uint32_t tmem_slot;
};

__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int DH, bool CG>
__device__ __forceinline__ void merge_row(const AttnParams& p, int n_seq, int seq, int h, int j, __nv_bfloat16* out,
                                          int lane);

template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, AttnParams p, int n_seq, __nv_bfloat16* out, int* err) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = base;                                  // 2 tiles
  uint8_t* kv_s = q_s + 2 * C::kTileBytes;              // kBufs tiles
  uint8_t* p_s = kv_s + C::kBufs * C::kTileBytes;       // 2 P tiles
  AttnBarriers* bars = reinterpret_cast<AttnBarriers*>(p_s + 2 * C::kPBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, split = blockIdx.y;
  const int seq = blockIdx.z / p.n_kv, kvh = blockIdx.z % p.n_kv;
  const int G = p.n_q / p.n_kv;
  const int cseq = p.seq_base + seq;
  pdl_trigger();
  if (threadIdx.x == 0) {   // descriptors into the TMA unit's cache while the previous kernel still runs
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int b = 0; b < C::kBufs; ++b) {
      mbar_init(&bars->kv_full[b], 1);
      mbar_init(&bars->kv_empty[b], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->s_free[x], 4);
      mbar_init(&bars->p_ready[x], 4);
      mbar_init(&bars->pv_done[x], 1);
    }
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(&bars->tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;
  pdl_wait();   // queries and the canvas keys / values come from the preceding kernels

  const int P = p.seq_P[cseq];
  const int nkeys = P + p.Tq;
  const int ntiles = (nkeys + 127) >> 7;
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(ntiles, t0 + p.tiles_per_split);
  const int T = t1 > t0 ? t1 - t0 : 0;
  const int z = p.layer * p.cache_seq_stride + cseq * p.n_kv + kvh;
  const int qrow0 = (seq * p.n_q + kvh * G) * p.rows_per_seq + pair * 256;

  if (warp == 8) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0 && T > 0) {
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::kTileBytes);
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int hh = 0; hh < DH / 64; ++hh)
          tma_load_2d(&tq, &bars->q_full, q_s + x * C::kTileBytes + hh * 16384, hh * 64, qrow0 + x * 128);
      for (int i = 0; i < 2 * T; ++i) {
        const int b = i % C::kBufs;
        if (!mbar_wait(&bars->kv_empty[b], ((i / C::kBufs) & 1) ^ 1, err, DEV_ERR_TIMEOUT_ATTN)) break;
        uint8_t* dst = kv_s + (size_t)b * C::kTileBytes;
        const int t = t0 + (i >> 1);
        mbar_arrive_expect_tx(&bars->kv_full[b], C::kTileBytes);
        if ((i & 1) == 0) {
#pragma unroll
          for (int h = 0; h < DH / 64; ++h) tma_load_3d(&tk, &bars->kv_full[b], dst + h * 16384, h * 64, t * 128, z);
        } else {
#pragma unroll
          for (int hk = 0; hk < 2; ++hk)
            tma_load_3d(&tv, &bars->kv_full[b], dst + hk * (DH * 128), t * 128 + hk * 64, 0, z);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, DH);
      bool ok = mbar_wait(&bars->q_full, 0, err, DEV_ERR_TIMEOUT_ATTN);
      auto issue_s = [&](int x, int tt) {
        const int i = 2 * tt, b = i % C::kBufs;
        ok = ok && mbar_wait(&bars->kv_full[b], (i / C::kBufs) & 1, err, DEV_ERR_TIMEOUT_ATTN);
        ok = ok && mbar_wait(&bars->s_free[x], (tt & 1) ^ 1, err, DEV_ERR_TIMEOUT_ATTN);
        tc_fence_after();
        if (ok) {
          const uint8_t* kb = kv_s + (size_t)b * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint64_t ad =
                desc_advance(smem_desc_sw128(smem_u32(q_s + x * C::kTileBytes + (kk / 4) * 16384)), (kk % 4) * 32);
            const uint64_t bd = desc_advance(smem_desc_sw128(smem_u32(kb + (kk / 4) * 16384)), (kk % 4) * 32);
            umma_bf16(tmem + x * 128, ad, bd, idesc_s, kk != 0);
          }
        }
        umma_commit(&bars->s_full[x]);
        if (x == 1) umma_commit(&bars->kv_empty[b]);   // both S products of K(t) issued
      };
      auto issue_pv = [&](int x, int tt) {
        const int i = 2 * tt + 1, b = i % C::kBufs;
        ok = ok && mbar_wait(&bars->kv_full[b], (i / C::kBufs) & 1, err, DEV_ERR_TIMEOUT_ATTN);
        ok = ok && mbar_wait(&bars->p_ready[x], tt & 1, err, DEV_ERR_TIMEOUT_ATTN);
        tc_fence_after();
        if (ok) {
          const uint8_t* vb = kv_s + (size_t)b * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad =
                desc_advance(smem_desc_sw128(smem_u32(p_s + x * C::kPBytes + (kk / 4) * 16384)), (kk % 4) * 32);
            const uint64_t bd = desc_advance(smem_desc_sw128(smem_u32(vb + (kk / 4) * (DH * 128))), (kk % 4) * 32);
            umma_bf16(tmem + 256 + x * 128, ad, bd, idesc_o, (tt | kk) != 0);
          }
        }
        umma_commit(&bars->pv_done[x]);
        if (x == 1) umma_commit(&bars->kv_empty[b]);   // both PV products of V(t) issued
      };
      issue_s(0, 0);
      issue_s(1, 0);
      for (int tt = 0; tt < T; ++tt) {
        issue_pv(0, tt);
        if (tt + 1 < T) issue_s(0, tt + 1);
        issue_pv(1, tt);
        if (tt + 1 < T) issue_s(1, tt + 1);
      }
    }
  } else {
    // ------------------------------ softmax (warps 0-3: tile 0, warps 4-7: tile 1) ------------------------------
    const int x = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + x * 128;
    const uint32_t t_o = tmem + lane_off + 256 + x * 128;
    const int rr = pair * 256 + x * 128 + r;       // query row inside the GQA group
    const int g = rr / p.rows_per_seq, j = rr % p.rows_per_seq;
    const int h = kvh * G + g;
    const bool row_valid = (g < G) && (j < p.Tq);
    const int qpos = P + j;
    const float sl2 = 1.4426950408889634f * rsqrtf((float)DH);
    uint8_t* prow = p_s + x * C::kPBytes + r * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int tt = 0; tt < T; ++tt) {
      ok = ok && mbar_wait(&bars->s_full[x], tt & 1, err, DEV_ERR_TIMEOUT_ATTN);
      tc_fence_after();
      const int key0 = (t0 + tt) * 128;
      int kmax = nkeys - key0;                        // keys [key0, key0 + kmax) exist (and are visible)
      if (p.causal) kmax = min(kmax, qpos - key0 + 1);
      const bool full = kmax >= 128;                  // no masked key in this tile for this row
      // P pass: P = exp2(S scale - m_ref) in bf16 to this tile's swizzled P buffer (4 x 16-byte chunks
      // per 32 keys); returns the fp32 sum and the raw max of the visible scores
      auto p_pass = [&](float m_ref, float& rmax) {
        uint64_t lt2 = 0;                               // two fp32 partial sums (packed)
        const uint64_t sl2x2 = pack_f32x2(sl2, sl2), negm2 = pack_f32x2(-m_ref, -m_ref);
        rmax = -INFINITY;
#pragma unroll
        for (int cb = 0; cb < 128; cb += 64) {
          float s[64];
          tmem_ld32_nowait(t_s + cb, s);
          tmem_ld32_nowait(t_s + cb + 32, s + 32);
          tmem_wait_ld();
          uint32_t pk[32];
          if (full) {
            // packed fp32 pairs: one FMA and one add per two keys
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              rmax = fmaxf(rmax, fmaxf(s[i], s[i + 1]));
              const uint64_t x = ffma_f32x2(pack_f32x2(s[i], s[i + 1]), sl2x2, negm2);
              const float p0 = fast_exp2(lo_f32(x)), p1 = fast_exp2(hi_f32(x));
              lt2 = fadd_f32x2(lt2, pack_f32x2(p0, p1));
              pk[i / 2] = pack_bf16x2(p0, p1);
            }
          } else {
            float lt = 0.f;
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              const bool v0 = cb + i < kmax, v1 = cb + i + 1 < kmax;   // masked keys: p = 0
              if (v0) rmax = fmaxf(rmax, s[i]);
              if (v1) rmax = fmaxf(rmax, s[i + 1]);
              const float p0 = v0 ? fast_exp2(fmaf(s[i], sl2, -m_ref)) : 0.f;
              const float p1 = v1 ? fast_exp2(fmaf(s[i + 1], sl2, -m_ref)) : 0.f;
              lt += p0 + p1;
              pk[i / 2] = pack_bf16x2(p0, p1);
            }
            lt2 = fadd_f32x2(lt2, pack_f32x2(lt, 0.f));
          }
          uint8_t* prow_c = prow + (cb / 64) * 16384;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(prow_c + ((ch ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        return lo_f32(lt2) + hi_f32(lt2);
      };
      // PV(tt-1) of this tile completed before S(tt) (tensor-core operations complete in order), so O
      // and this tile's P buffer are free here.  Optimistic single pass against the running max; a
      // warp redoes the tile when one of its rows' max grew by more than kLazyRescale (or has none yet).
      float rmax = -INFINITY, lt = 0.f;
      bool redo = m_used == -INFINITY;
      if (!__any_sync(0xffffffffu, redo)) {
        lt = p_pass(m_used, rmax);
        redo = rmax * sl2 > m_used + kLazyRescale;
      }
      if (__any_sync(0xffffffffu, redo)) {
        // the row max of this tile (raw scores; the scale is positive); every lane of the warp takes
        // part in the collective TMEM loads, also lanes whose row needs no redo
        rmax = -INFINITY;
#pragma unroll
        for (int cb = 0; cb < 128; cb += 64) {
          float s[64];
          tmem_ld32_nowait(t_s + cb, s);
          tmem_ld32_nowait(t_s + cb + 32, s + 32);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (cb + i < kmax) rmax = fmaxf(rmax, s[i]);
        }
        // lazy max: O and l are rescaled only when this row's max grows by more than kLazyRescale
        const float tmax = rmax * sl2;
        const bool grow = redo && tmax > m_used + kLazyRescale;
        const float m_new = grow ? tmax : m_used;
        const float alpha = (grow && m_used != -INFINITY) ? fast_exp2(m_used - m_new) : 1.f;
        l *= alpha;
        m_used = m_new;
        if (tt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int cb = 0; cb < DH; cb += 32) {
            float o[32];
            tmem_ld32_nowait(t_o + cb, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(t_o + cb, o);
          }
          tmem_wait_st();
        }
        lt = p_pass(m_used, rmax);   // rows without a redo recompute the values they already wrote
      }
      l += lt;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->s_free[x]);    // S(tt) is read: S(tt+1) may overwrite it
        mbar_arrive(&bars->p_ready[x]);
      }
    }
    // ---- output ----
    if (T > 0) {
      ok = ok && mbar_wait(&bars->pv_done[x], (T - 1) & 1, err, DEV_ERR_TIMEOUT_ATTN);
      tc_fence_after();
    }
    const size_t prw = ((size_t)(split * n_seq + seq) * p.n_q + h) * p.rows_per_seq + j;
    if (p.n_splits == 1) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = out + ((size_t)seq * p.rows_per_seq + j) * (p.n_q * DH) + h * DH;
#pragma unroll
      for (int cb = 0; cb < DH; cb += 32) {
        float o[32];
        tmem_ld32_nowait(t_o + cb, o);
        tmem_wait_ld();
        if (row_valid && ok && T > 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4*>(dst + cb + i) =
                make_uint4(pack_bf16x2(o[i] * inv, o[i + 1] * inv), pack_bf16x2(o[i + 2] * inv, o[i + 3] * inv),
                           pack_bf16x2(o[i + 4] * inv, o[i + 5] * inv), pack_bf16x2(o[i + 6] * inv, o[i + 7] * inv));
        }
      }
    } else if (T == 0) {   // empty split: neutral partial
      if (row_valid) {
        p.ml[prw * 2 + 0] = -INFINITY;
        p.ml[prw * 2 + 1] = 0.f;
        uint4* o8 = reinterpret_cast<uint4*>(p.opart + prw * DH);
        for (int c = 0; c < DH / 8; ++c) o8[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    } else {
      // the partial row in bf16 (un-normalised, values up to l times the largest |v|): half the bytes of
      // fp32 for the store here and the merge's loads, one more rounding of 2^-9 relative
      uint4* o8 = reinterpret_cast<uint4*>(p.opart + prw * DH);
#pragma unroll
      for (int cb = 0; cb < DH; cb += 32) {
        float o[32];
        tmem_ld32_nowait(t_o + cb, o);
        tmem_wait_ld();
        if (row_valid && ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            o8[(cb + i) / 8] = make_uint4(pack_bf16x2(o[i], o[i + 1]), pack_bf16x2(o[i + 2], o[i + 3]),
                                          pack_bf16x2(o[i + 4], o[i + 5]), pack_bf16x2(o[i + 6], o[i + 7]));
        }
      }
      if (row_valid && ok) {
        p.ml[prw * 2 + 0] = m_used;
        p.ml[prw * 2 + 1] = l;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) tmem_dealloc(tmem, C::kTmemCols);
  if (p.n_splits > 1 && p.merge_in_cluster) {
    // the pair's splits are the CTAs of this cluster (cluster dims (1, n_splits, 1)): once every split's
    // partials are written (the barrier's release / acquire at cluster scope makes them visible), CTA
    // `split` merges its share of the pair's 256 rows, one warp per row
    cluster_sync();
    const int per = (256 + p.n_splits - 1) / p.n_splits;
    const int q1 = min(256, (split + 1) * per);
    for (int q = split * per + warp; q < q1; q += kAttnThreads / 32) {
      const int rr = pair * 256 + q;
      const int g = rr / p.rows_per_seq, j = rr % p.rows_per_seq;
      if (g < G && j < p.Tq) merge_row<DH, true>(p, n_seq, seq, kvh * G + g, j, out, lane);
    }
  }
}

// One warp per (sequence, query head, row): combine the split partials (lane s < n_splits holds
// split s's (m, l)) and write the row of the token-major attention output
// [seq*rows_per_seq + j][h*dh + c] in bf16; each lane owns dh/32 consecutive columns.  Loads bypass
// L1 when CG (in the in-cluster merge the partials come from other CTAs of the same launch).
template <typename T>
__device__ __forceinline__ T ld_partial(const T* p, bool cg) {
  return cg ? __ldcg(p) : *p;
}
template <int DH, bool CG>
__device__ __forceinline__ void merge_row(const AttnParams& p, int n_seq, int seq, int h, int j, __nv_bfloat16* out,
                                          int lane) {
  const int sh = seq * p.n_q + h;
  const size_t stride = (size_t)n_seq * p.n_q * p.rows_per_seq;
  const size_t r0 = (size_t)sh * p.rows_per_seq + j;
  constexpr int kPer = DH / 32;
  // splits in groups of 8: a group's loads are all issued before they are summed (in split order); the
  // first group's loads are issued together with the (m, l) loads, before the weights are reduced
  float v[8][kPer];
  auto load_group = [&](int s0) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int s = s0 + u;
      const __nv_bfloat16* src = p.opart + ((size_t)s * stride + r0) * DH + lane * kPer;
#pragma unroll
      for (int c = 0; c < kPer; ++c) v[u][c] = 0.f;
      if (s < p.n_splits) {
        if constexpr (kPer == 4) {
          const uint2 q = ld_partial(reinterpret_cast<const uint2*>(src), CG);
          v[u][0] = bf16_lo(q.x); v[u][1] = bf16_hi(q.x); v[u][2] = bf16_lo(q.y); v[u][3] = bf16_hi(q.y);
        } else {
          const uint32_t q = ld_partial(reinterpret_cast<const uint32_t*>(src), CG);
          v[u][0] = bf16_lo(q); v[u][1] = bf16_hi(q);
        }
      }
    }
  };
  float ms = -INFINITY, ls = 0.f;
  if (lane < p.n_splits) {
    const float2 q = ld_partial(reinterpret_cast<const float2*>(p.ml + (lane * stride + r0) * 2), CG);
    ms = q.x;
    ls = q.y;
  }
  load_group(0);
  const float M = warp_max(ms);
  const float wgt = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
  const float den = warp_sum(wgt * ls);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
  for (int s0 = 0;;) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float ws = __shfl_sync(0xffffffffu, wgt, (s0 + u) & 31);
      if (s0 + u < p.n_splits && ws != 0.f) {
#pragma unroll
        for (int c = 0; c < kPer; ++c) acc[c] += ws * v[u][c];
      }
    }
    s0 += 8;
    if (s0 >= p.n_splits) break;
    load_group(s0);
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
__global__ void attn_merge_kernel(AttnParams p, int n_seq, __nv_bfloat16* out) {
  pdl_trigger();
  pdl_wait();
  const int warp = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (warp >= n_seq * p.n_q * p.Tq) return;
  const int j = warp % p.Tq;
  const int sh = warp / p.Tq;          // seq * n_q + h
  merge_row<DH, false>(p, n_seq, sh / p.n_q, sh % p.n_q, j, out, lane);
}

template <int DH>
static cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const AttnParams& p, int n_seq, __nv_bfloat16* out, int* err, cudaStream_t st) {
  using C = AttnCfg<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int G = p.n_q / p.n_kv;
  dim3 grid((G * p.rows_per_seq + 255) / 256, p.n_splits, n_seq * p.n_kv);
  if (!(p.n_splits > 1 && p.merge_in_cluster))
    return launch_k(attn_fwd_kernel<DH>, grid, dim3(kAttnThreads), C::kSmemBytes, st, 1, tq, tk, tv, p, n_seq, out,
                    err);
  // the splits of a query-tile pair as one cluster (1, n_splits, 1)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  attr[n].id = cudaLaunchAttributeClusterDimension;
  attr[n].val.clusterDim.x = 1;
  attr[n].val.clusterDim.y = p.n_splits;
  attr[n].val.clusterDim.z = 1;
  ++n;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_fwd_kernel<DH>, tq, tk, tv, p, n_seq, out, err);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// n_splits == 1: the attention output is written directly to `out`; otherwise the partials are
// merged inside the launch (merge_in_cluster, n_splits <= 8) or left for attention_merge.
cudaError_t attention_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const AttnParams& p, int n_seq, __nv_bfloat16* out, int* err, cudaStream_t st) {
  if (p.merge_in_cluster && p.n_splits > 8) return cudaErrorInvalidValue;   // portable cluster size
  if (p.dh == 128) return launch_attn<128>(tq, tk, tv, p, n_seq, out, err, st);
  if (p.dh == 64) return launch_attn<64>(tq, tk, tv, p, n_seq, out, err, st);
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
