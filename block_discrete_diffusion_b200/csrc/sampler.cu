// sampler.cu -- the uniform-state canvas sampler (entropy-bound commit, self-correcting
// re-randomisation, adaptive stop) over fp32 vocabulary logits.
//
// Constants and rules from the pages: canvas of 256, at most 48 steps, temperature linear 0.8 ->
// 0.4, adaptive-stop threshold 0.005 ("Composition of DiffusionGemma", sampler settings, in the
// technical-report summary); the entropy_bound sampler with bound 0.1 ("Serving with vLLM" in the
// diffusion-gemma developer guide); random placeholder start and re-randomisation of positions
// whose confidence dropped ("Uniform State Diffusion", same guide).  The precise rule (which
// entropy, which threshold re-randomises, what ends a block) is the build's written reading:
//   H = entropy (nats) of softmax(l / T);  y = argmax_v (l_v / T + Gumbel_v);
//   commit iff H <= entropy_bound (or, with commit_rule 1, iff the entropies of the uncommitted
//   positions at or before it in ascending (H, position) order sum to <= entropy_bound);
//   else re-randomise iff H > rerand_entropy, else take y;
//   stop iff all committed, or mean H over the canvas (committed = 0) <= stop_mean_entropy, or the
//   step budget is reached (fixed_steps > 0: exactly fixed_steps steps); on stop the remaining
//   positions take y and commit.
//
// sampler_partial_kernel: grid (vocab chunk, row).  One pass over the chunk with 16-byte loads, 16
// logits per thread per batch; each thread keeps (m, S, A) of the tempered softmax in the exp2
// domain (packed fp32 pairs, one rescale per batch) and its best perturbed score.  Gumbel-max with a
// warp-wide lower bound `lim` on the chunk's best score: a group of four logits whose largest
// tempered value cannot reach it even with the largest possible Gumbel draw skips the Philox call;
// the other draws get a screened score from hardware logarithms, the warp's largest screened score
// (minus the screen's error) raises the bound, and only draws whose screened score still reaches it
// take the accurate logarithms.  Both tests only drop elements whose accurate score is below a
// score that some element reaches, so the result is the exact Gumbel-max of the accurate scores.
// sampler_finalize_kernel: one CTA per sequence, one thread per canvas position.
#include <math.h>

#include "dg_device.cuh"
#include "dg_kernels.h"
#include "philox.cuh"

namespace dg {

constexpr int kSampThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct SoftStats {
  float m;   // running max of z * log2(e)
  float S;   // sum 2^(z2 - m)
  float A;   // sum 2^(z2 - m) * (z2 - m)
};

__device__ __forceinline__ SoftStats stats_merge(SoftStats a, SoftStats b) {
  if (a.m == -INFINITY) return b;
  if (b.m == -INFINITY) return a;
  const float M = fmaxf(a.m, b.m);
  const float fa = fast_exp2(a.m - M), fb = fast_exp2(b.m - M);
  SoftStats r;
  r.m = M;
  r.S = fa * a.S + fb * b.S;
  r.A = fa * (a.A + a.S * (a.m - M)) + fb * (b.A + b.S * (b.m - M));
  return r;
}

__device__ __forceinline__ void best_merge(float& bs, int& bi, float os, int oi) {
  if (os > bs || (os == bs && oi < bi)) {
    bs = os;
    bi = oi;
  }
}

__global__ void __launch_bounds__(kSampThreads)
    sampler_partial_kernel(const float* __restrict__ logits, int canvas, int vocab, int n_chunks,
                           const int* __restrict__ seq_P, const uint8_t* __restrict__ commit_in, float inv_temp,
                           uint64_t seed, int step, float* __restrict__ partial, const int* __restrict__ d_step,
                           float t_start, float t_end, int max_steps) {
  pdl_trigger();
  pdl_wait();
  if (d_step) {   // step index kept on the device: this step's index and temperature
    step = *d_step;
    inv_temp = __fdiv_rn(1.0f, schedule_temperature(t_start, t_end, max_steps, step));
  }
  const int row = blockIdx.y, chunk = blockIdx.x;
  if (commit_in[row]) return;
  const int seq = row / canvas, j = row % canvas;
  const uint32_t pos = (uint32_t)((seq_P ? seq_P[seq] : 0) + j);
  const uint64_t sd = seed + (uint64_t)seq;
  const uint32_t k0 = (uint32_t)sd, k1 = (uint32_t)(sd >> 32);
  const int vchunk = vocab / n_chunks;
  const int g0 = (chunk * vchunk) >> 2, g1 = ((chunk + 1) * vchunk) >> 2;   // float4 groups
  const float4* lr = reinterpret_cast<const float4*>(logits + (size_t)row * vocab);
  const float s2 = inv_temp * kLog2e;

  // softmax statistics: running max m (exp2 domain) and (S, A) as two packed lanes each
  float m = -INFINITY;
  uint64_t S2 = 0, A2 = 0;
  float best = -INFINITY;   // this thread's best accurate score and its element
  int bidx = 0x7fffffff;
  float lim = -INFINITY;    // a score some element of the chunk reaches or exceeds (pruning bound)
  const float kSkip = __int_as_float(0x7fffffff);   // NaN: compares false, marks draws not taken

  // the trip count is the same for every thread (the warp-wide maximum below needs all lanes)
  for (int base = g0; base < g1; base += 4 * kSampThreads) {
    const int gb = base + threadIdx.x;
    // the next batch's 16 KB move into L2 while this one is processed
    const int nb = base + 4 * kSampThreads;
    if (threadIdx.x == 0 && nb < g1) l2_prefetch_bulk(lr + nb, (uint32_t)min(4 * kSampThreads, g1 - nb) * 16u);
    float4 q[4];
    bool have[4];
    float gmax[4], gabs[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int g = gb + u * kSampThreads;
      have[u] = g < g1;
      q[u] = have[u] ? __ldcs(lr + g) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      gmax[u] = fmaxf(fmaxf(q[u].x, q[u].y), fmaxf(q[u].z, q[u].w));
      gabs[u] = fmaxf(fmaxf(fabsf(q[u].x), fabsf(q[u].y)), fmaxf(fabsf(q[u].z), fabsf(q[u].w)));
    }
    // batch max in the exp2 domain, then one rescale of (S, A)
    const float bm = fmaxf(fmaxf(gmax[0], gmax[1]), fmaxf(gmax[2], gmax[3])) * s2;
    if (bm > m) {
      if (m != -INFINITY) {
        const float f = fast_exp2(m - bm);
        A2 = fmul_f32x2(ffma_f32x2(S2, pack_f32x2(m - bm, m - bm), A2), pack_f32x2(f, f));
        S2 = fmul_f32x2(S2, pack_f32x2(f, f));
      }
      m = bm;
    }
    const uint64_t s2p = pack_f32x2(s2, s2), negm = pack_f32x2(-m, -m);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!have[u]) continue;
      const uint64_t t01 = ffma_f32x2(pack_f32x2(q[u].x, q[u].y), s2p, negm);
      const uint64_t t23 = ffma_f32x2(pack_f32x2(q[u].z, q[u].w), s2p, negm);
      const uint64_t e01 = pack_f32x2(fast_exp2(lo_f32(t01)), fast_exp2(hi_f32(t01)));
      const uint64_t e23 = pack_f32x2(fast_exp2(lo_f32(t23)), fast_exp2(hi_f32(t23)));
      S2 = fadd_f32x2(S2, fadd_f32x2(e01, e23));
      A2 = ffma_f32x2(e23, t23, ffma_f32x2(e01, t01, A2));
    }

    // Gumbel draws of the groups that can reach the bound, screened with hardware logarithms
    float fs[4][4];
    float fmax_ = -INFINITY;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll
      for (int i = 0; i < 4; ++i) fs[u][i] = kSkip;
      if (have[u] && __fmaf_rn(gmax[u], inv_temp, kGumbelMax) >= lim) {
        const uint4 w = philox4x32_10(make_uint4((uint32_t)(gb + u * kSampThreads), pos, (uint32_t)step,
                                                 RNG_TAG_GUMBEL), k0, k1);
        const bool screen = gabs[u] * inv_temp <= kScreenMaxZ;
        const float zz[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float uu = u01_open(ww[i]);
          const float f = gumbel_screen_score(zz[i], inv_temp, uu);
          const bool exact_only = !screen || uu >= kGumbelFastMaxU;
          fs[u][i] = exact_only ? INFINITY : f;
          fmax_ = fmaxf(fmax_, exact_only ? -INFINITY : f);
        }
      }
    }
    // every screened score minus two slacks is below that element's accurate score
    lim = fmaxf(lim, warp_max(fmax_) - 2.f * kGumbelFastSlack);
    // accurate scores only where the screened score reaches the bound (elements in increasing
    // index order, so the strict comparison keeps the lowest index among equal scores); the few
    // groups holding such a draw generate their Philox block again rather than keep 16 words live
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (fs[u][0] >= lim || fs[u][1] >= lim || fs[u][2] >= lim || fs[u][3] >= lim) {
        const int g = gb + u * kSampThreads;
        const uint4 w = philox4x32_10(make_uint4((uint32_t)g, pos, (uint32_t)step, RNG_TAG_GUMBEL), k0, k1);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        const float zz[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (fs[u][i] >= lim) {
            const float sc = __fmaf_rn(zz[i], inv_temp, gumbel_from_word(ww[i]));
            if (sc > best) {
              best = sc;
              bidx = 4 * g + i;
            }
          }
        }
      }
    }
    lim = fmaxf(lim, best);
  }
  SoftStats st = {m, lo_f32(S2) + hi_f32(S2), lo_f32(A2) + hi_f32(A2)};

  // block reduction: warp shuffles, then the 8 warp results through shared memory
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftStats other = {__shfl_xor_sync(0xffffffffu, st.m, o), __shfl_xor_sync(0xffffffffu, st.S, o),
                       __shfl_xor_sync(0xffffffffu, st.A, o)};
    st = stats_merge(st, other);
    best_merge(best, bidx, __shfl_xor_sync(0xffffffffu, best, o), __shfl_xor_sync(0xffffffffu, bidx, o));
  }
  __shared__ float red[kSampThreads / 32][5];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[w][0] = st.m;
    red[w][1] = st.S;
    red[w][2] = st.A;
    red[w][3] = best;
    red[w][4] = __int_as_float(bidx);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    SoftStats t = {red[0][0], red[0][1], red[0][2]};
    float bb = red[0][3];
    int bi = __float_as_int(red[0][4]);
    for (int i = 1; i < kSampThreads / 32; ++i) {
      t = stats_merge(t, SoftStats{red[i][0], red[i][1], red[i][2]});
      best_merge(bb, bi, red[i][3], __float_as_int(red[i][4]));
    }
    float* out = partial + ((size_t)row * n_chunks + chunk) * 8;
    out[0] = t.m;
    out[1] = t.S;
    out[2] = t.A;
    out[3] = bb;
    out[4] = __int_as_float(bi);
  }
}

__global__ void sampler_finalize_kernel(SamplerArgs a) {
  pdl_trigger();
  pdl_wait();
  if (a.d_step) a.step = *a.d_step;
  __shared__ float red_h[32];
  __shared__ int red_c[32];
  const int seq = blockIdx.x;
  float Hsum_part = 0.f;
  int all_part = 1;
  // positions are strided over the block so any canvas length works with 256 threads
  const int n_iter = (a.canvas + blockDim.x - 1) / blockDim.x;
  // first pass: per-position decision without the stop override; remember (id, y, commit) locally
  __shared__ float s_H[1024];   // cumulative rule: entropies of the uncommitted positions (canvas <= 1024)
  int my_id[4], my_y[4], my_rr[4];
  uint8_t my_c[4], my_unc[4];
  float my_H[4];
  for (int it = 0; it < n_iter && it < 4; ++it) {
    const int jj = threadIdx.x + it * blockDim.x;
    my_id[it] = 0; my_y[it] = 0; my_rr[it] = 0; my_c[it] = 1; my_unc[it] = 0; my_H[it] = 0.f;
    if (jj >= a.canvas) continue;
    const int row = seq * a.canvas + jj;
    if (a.commit_in[row]) {
      my_id[it] = a.ids_in[row];
      my_y[it] = my_id[it];
      my_c[it] = 1;
      my_H[it] = 0.f;
      continue;
    }
    SoftStats st = {-INFINITY, 0.f, 0.f};
    float best = -INFINITY;
    int bidx = 0x7fffffff;
    for (int c = 0; c < a.n_chunks; ++c) {
      const float* pr = a.partial + ((size_t)row * a.n_chunks + c) * 8;
      st = stats_merge(st, SoftStats{pr[0], pr[1], pr[2]});
      best_merge(best, bidx, pr[3], __float_as_int(pr[4]));
    }
    const float H = logf(st.S) - kLn2 * st.A / st.S;
    const uint32_t pos = (uint32_t)((a.seq_P ? a.seq_P[seq] : 0) + jj);
    const uint4 w = rng_block(a.seed + (uint64_t)seq, 0u, pos, (uint32_t)a.step, RNG_TAG_RERAND);
    const int rr = token_from_word(w.x, (uint32_t)a.vocab);
    my_H[it] = H;
    my_y[it] = bidx;
    my_rr[it] = rr;
    my_unc[it] = 1;
    Hsum_part += H;
  }
  // commit decisions: per position (H <= bound), or cumulative (ascending (H, position) order while
  // the running entropy sum stays <= bound: position i commits iff the entropies of the uncommitted
  // positions ordered at or before it sum to <= bound)
  if (a.commit_rule == 1) {
    for (int jj = threadIdx.x; jj < a.canvas; jj += blockDim.x) s_H[jj] = INFINITY;   // committed: excluded
    __syncthreads();
    for (int it = 0; it < n_iter && it < 4; ++it)
      if (my_unc[it]) s_H[threadIdx.x + it * blockDim.x] = my_H[it];
    __syncthreads();
  }
  for (int it = 0; it < n_iter && it < 4; ++it) {
    if (!my_unc[it]) continue;
    const int jj = threadIdx.x + it * blockDim.x;
    bool commits;
    if (a.commit_rule == 1) {
      const float hi = my_H[it];
      float run = 0.f;
      for (int k = 0; k < a.canvas; ++k) {
        const float hk = s_H[k];
        if (hk < hi || (hk == hi && k <= jj)) run += hk;
      }
      commits = run <= a.entropy_bound;
    } else {
      commits = my_H[it] <= a.entropy_bound;
    }
    if (commits) {
      my_id[it] = my_y[it];
      my_c[it] = 1;
    } else {
      my_id[it] = my_H[it] > a.rerand_entropy ? my_rr[it] : my_y[it];
      my_c[it] = 0;
      all_part = 0;
    }
  }
  // canvas-mean entropy and the all-committed test
  float hs = warp_sum(Hsum_part);
  int al = __all_sync(0xffffffffu, all_part);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red_h[w] = hs;
    red_c[w] = al;
  }
  __syncthreads();
  float Hsum = 0.f;
  int all = 1;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
    Hsum += red_h[i];
    all &= red_c[i];
  }
  const float mean = Hsum / (float)a.canvas;
  int stop;
  if (a.fixed_steps > 0)
    stop = (a.step + 1 >= a.fixed_steps);
  else
    stop = all || (mean <= a.stop_mean_entropy) || (a.step + 1 >= a.max_steps);
  for (int it = 0; it < n_iter && it < 4; ++it) {
    const int jj = threadIdx.x + it * blockDim.x;
    if (jj >= a.canvas) continue;
    const int row = seq * a.canvas + jj;
    int id = my_id[it];
    uint8_t c = my_c[it];
    if (stop && !c) {
      id = my_y[it];
      c = 1;
    }
    a.ids_out[row] = id;
    a.commit_out[row] = c;
    a.entropy[row] = my_H[it];
  }
  if (threadIdx.x == 0) a.stop[seq] = stop;
}

// Many partial records per row (one per CTA of the fused head): one warp per row merges them -- lane
// l takes records l, l + 32, ... in order, then the lanes combine by shuffles -- into a single record
// per row (the same (m, S, A, best, index) merge as the finalize; ties of the best score go to the
// lower index in both).  Rows committed before the step are skipped, as the finalize skips them.
__global__ void sampler_premerge_kernel(const float* __restrict__ partial, int n_rows, int n_chunks,
                                        const uint8_t* __restrict__ commit_in, float* __restrict__ merged) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= n_rows || commit_in[row]) return;
  SoftStats st = {-INFINITY, 0.f, 0.f};
  float best = -INFINITY;
  int bidx = 0x7fffffff;
  for (int c = lane; c < n_chunks; c += 32) {
    const float* pr = partial + ((size_t)row * n_chunks + c) * 8;
    const float4 a = *reinterpret_cast<const float4*>(pr);
    const float b = pr[4];
    st = stats_merge(st, SoftStats{a.x, a.y, a.z});
    best_merge(best, bidx, a.w, __float_as_int(b));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftStats other = {__shfl_xor_sync(0xffffffffu, st.m, o), __shfl_xor_sync(0xffffffffu, st.S, o),
                       __shfl_xor_sync(0xffffffffu, st.A, o)};
    st = stats_merge(st, other);
    best_merge(best, bidx, __shfl_xor_sync(0xffffffffu, best, o), __shfl_xor_sync(0xffffffffu, bidx, o));
  }
  if (lane == 0) {
    float* out = merged + (size_t)row * 8;
    *reinterpret_cast<float4*>(out) = make_float4(st.m, st.S, st.A, best);
    out[4] = __int_as_float(bidx);
  }
}

cudaError_t sampler_premerge_finalize_run(const SamplerArgs& a, float* merged, cudaStream_t st) {
  if (a.canvas > 4 * 256 || a.n_chunks <= 0) return cudaErrorInvalidValue;
  const int rows = a.n_seq * a.canvas;
  cudaError_t e = launch_k(sampler_premerge_kernel, dim3((rows + 7) / 8), dim3(256), 0, st, 1, a.partial, rows,
                           a.n_chunks, a.commit_in, merged);
  if (e != cudaSuccess) return e;
  SamplerArgs f = a;
  f.partial = merged;
  f.n_chunks = 1;
  return sampler_finalize_run(f, st);
}

int sampler_chunks(int vocab) {
  int c = vocab / 32768;
  if (c < 1) c = 1;
  while (c > 1 && (vocab % (c * 4) != 0)) --c;
  return c;
}

cudaError_t sampler_run(const SamplerArgs& a, cudaStream_t st) {
  if (a.canvas > 4 * 256 || a.vocab % (4 * a.n_chunks) != 0) return cudaErrorInvalidValue;
  dim3 grid(a.n_chunks, a.n_seq * a.canvas);
  cudaError_t e = launch_k(sampler_partial_kernel, grid, dim3(kSampThreads), 0, st, 1, a.logits, a.canvas, a.vocab,
                           a.n_chunks, a.seq_P, a.commit_in, a.inv_temp, a.seed, a.step, a.partial, a.d_step,
                           a.t_start, a.t_end, a.max_steps);
  if (e != cudaSuccess) return e;
  return sampler_finalize_run(a, st);
}

cudaError_t sampler_finalize_run(const SamplerArgs& a, cudaStream_t st) {
  if (a.canvas > 4 * 256 || a.n_chunks <= 0) return cudaErrorInvalidValue;
  return launch_k(sampler_finalize_kernel, dim3(a.n_seq), dim3(256), 0, st, 1, a);
}

}  // namespace dg
