// misc.cu -- bandwidth/latency kernels around the GEMMs: embedding gather, RMSNorm, the rotary
// table, the top-k router (with the expert bucketing in its last CTA for one canvas), the
// multi-CTA bucketing for many canvases, the activation gather, the MoE combine, canvas
// initialisation and cache loading.
#include <math.h>

#include "dg_device.cuh"
#include "dg_kernels.h"
#include "philox.cuh"

namespace dg {

__device__ __forceinline__ float block_sum_256(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  t = red[0];
  __syncthreads();
  return t;
}

// x[r][:] = emb[ids[r]][:] (bf16 -> fp32).  Out-of-range ids read row 0 and raise DEV_ERR_BAD_INDEX.
__global__ void embed_kernel(const __nv_bfloat16* __restrict__ emb, const int32_t* __restrict__ ids, int d, int vocab,
                             float* __restrict__ x, int* err, const float* __restrict__ g, float eps,
                             __nv_bfloat16* __restrict__ xn) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int r = blockIdx.x;
  int id = ids[r];
  if (id < 0 || id >= vocab) {
    if (threadIdx.x == 0) report_error(err, DEV_ERR_BAD_INDEX);
    id = 0;
  }
  const uint4* src = reinterpret_cast<const uint4*>(emb + (size_t)id * d);
  float4* dst = reinterpret_cast<float4*>(x + (size_t)r * d);
  for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
    const uint4 u = src[c];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
    const float2 f0 = __bfloat1622float2(b[0]), f1 = __bfloat1622float2(b[1]);
    const float2 f2 = __bfloat1622float2(b[2]), f3 = __bfloat1622float2(b[3]);
    dst[2 * c] = make_float4(f0.x, f0.y, f1.x, f1.y);
    dst[2 * c + 1] = make_float4(f2.x, f2.y, f3.x, f3.y);
  }
  if (!g) return;
  // the first layer's RMSNorm of the embedded row (the row was written by other threads of the block)
  __syncthreads();
  float ss = 0.f;
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = dst[c];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum_256(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  uint2* o2 = reinterpret_cast<uint2*>(xn + (size_t)r * d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = dst[c], w = g4[c];
    o2[c] = make_uint2(pack_bf16x2(v.x * inv * w.x, v.y * inv * w.y), pack_bf16x2(v.z * inv * w.z, v.w * inv * w.w));
  }
}

// out[r] = bf16( x[r] / sqrt(mean(x[r]^2) + eps) * g )
__global__ void rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ g, int d, float eps,
                               __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int r = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)r * d);
  float ss = 0.f;
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = xr[c];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum_256(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  uint2* o = reinterpret_cast<uint2*>(out + (size_t)r * d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = xr[c], w = g4[c];
    o[c] = make_uint2(pack_bf16x2(v.x * inv * w.x, v.y * inv * w.y), pack_bf16x2(v.z * inv * w.z, v.w * inv * w.w));
  }
}

// (cos, sin) of pos * theta^(-2i/dh) for i < dh/2, computed in double and rounded to fp32.
__global__ void rope_table_kernel(float2* table, int dh, double theta) {
  pdl_trigger();
  pdl_wait();
  const int pos = blockIdx.x, i = threadIdx.x;
  const double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)dh);
  double s, c;
  sincos(ang, &s, &c);
  table[(size_t)pos * (dh / 2) + i] = make_float2((float)c, (float)s);
}

// One warp per row: the top_k largest router logits (ties -> lower expert id), gates = softmax over
// the selected logits; per-expert counts accumulate with integer atomics (order-free, exact).
// The router logits arrive as n_parts split-K partial planes (part_stride apart), summed here in
// plane order.  Lane l owns experts [l*V, l*V + V), V = ceil(E/32) <= 8.
struct RouterNorm {    // the FFN RMSNorm folded into the router (ssq == nullptr: the logits are final)
  const float* ssq;
  int n_ssq, d;
  float eps;
  float* r_out;
  float* logits_out;
};

template <int V>
__device__ __forceinline__ void router_topk_row(const float* __restrict__ logits, int n_parts, size_t part_stride,
                                                int row, int n_rows, int n_exp, int top_k, int32_t* __restrict__ sel,
                                                float* __restrict__ gate, int32_t* __restrict__ counts,
                                                const RouterNorm& rn, int lane);
__device__ void assign_rows_block(const int32_t* sel, const float* gate, int32_t* counts, int n_assign, int top_k,
                                  int n_exp, int32_t* __restrict__ offsets, int32_t* __restrict__ slot);

struct FusedAssign {   // the last CTA of the top-k launch also buckets the assignments (done != nullptr)
  int32_t* done;       // launch counter, reset to 0 by that CTA
  int32_t* offsets;
  int32_t* slot;
};

struct TopkGatherArgs {   // router_topk_gather_kernel: the gather's source and destination, the bucketing state
  GatherSrc src;
  __nv_bfloat16* xp;
  int d;
  int32_t* sync;          // [3] zero-initialised: arrivals, offsets ready, leavers
  int32_t* offsets;       // [n_exp + 1]
  int32_t* cursor;        // [n_exp]
  int32_t* slot;          // [n_rows * top_k]
  int32_t* zero;          // nullable: n_zero ints cleared (the merged expert launch's counters)
  int n_zero;
  int* err;
};

struct ExpertPrefetch {   // w == nullptr: none
  const uint8_t* w;
  int n_ctas, F, d, row_bytes;
};

template <int V>
__global__ void router_topk_kernel(const float* __restrict__ logits, int n_parts, size_t part_stride, int n_rows,
                                   int n_exp, int top_k, int32_t* __restrict__ sel, float* __restrict__ gate,
                                   int32_t* __restrict__ counts, FusedAssign fa, RouterNorm rn, ExpertPrefetch pf) {
  pdl_trigger();
  pdl_wait();
  if (pf.w) {
    // the expert launch's first weight tiles into L2 (HBM is otherwise idle until that launch): whole
    // rows as one request per 64-row block (gate or up half of a tile, contiguous), else per row
    const int MTu = pf.F / 64;
    const bool blocks = pf.row_bytes == 2 * pf.d;
    const int n = pf.n_ctas * (blocks ? 2 : 128);
    for (int i = threadIdx.x * gridDim.x + blockIdx.x; i < n; i += gridDim.x * blockDim.x) {   // spread over CTAs
      const int c = blocks ? i >> 1 : i >> 7, k = blocks ? (i & 1) * 64 : i & 127;
      const int e = c / MTu, mt = c % MTu;
      const int row = e * 2 * pf.F + (k < 64 ? mt * 64 + k : pf.F + mt * 64 + (k - 64));
      l2_prefetch_bulk(pf.w + (size_t)row * pf.d * 2, (uint32_t)(blocks ? 64 * pf.row_bytes : pf.row_bytes));
    }
  }
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row < n_rows)
    router_topk_row<V>(logits, n_parts, part_stride, row, n_rows, n_exp, top_k, sel, gate, counts, rn, lane);
  if (fa.done) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(fa.done, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      assign_rows_block(sel, gate, counts, n_rows * top_k, top_k, n_exp, fa.offsets, fa.slot);
      if (threadIdx.x == 0) *fa.done = 0;
    }
  }
}

template <int V>
__device__ __forceinline__ void router_topk_row(const float* __restrict__ logits, int n_parts, size_t part_stride,
                                                int row, int n_rows, int n_exp, int top_k, int32_t* __restrict__ sel,
                                                float* __restrict__ gate, int32_t* __restrict__ counts,
                                                const RouterNorm& rn, int lane) {
  float v[V];
  const float* lr = logits + (size_t)row * n_exp + lane * V;
#pragma unroll
  for (int i = 0; i < V; ++i) v[i] = 0.f;
  bool done = false;
  // the row's sums of squares are loaded first, so that their latency overlaps the planes'
  float ss = 0.f;
  if (rn.ssq)
    for (int t = lane; t < rn.n_ssq; t += 32) ss += __ldcg(rn.ssq + (size_t)t * n_rows + row);
  // planes in batches (24 with float4 lanes, 8 otherwise) whose loads are all in flight together,
  // summed in plane order (a missing plane adds an exact 0)
  if constexpr (V == 4) {
    if ((n_exp % 4) == 0 && lane * V < n_exp) {
      for (int z0 = 0; z0 < n_parts; z0 += 24) {
        float4 q[24];
#pragma unroll
        for (int u = 0; u < 24; ++u)
          q[u] = z0 + u < n_parts ? __ldcg(reinterpret_cast<const float4*>(lr + (z0 + u) * part_stride))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 24; ++u) {
          v[0] += q[u].x; v[1] += q[u].y; v[2] += q[u].z; v[3] += q[u].w;
        }
      }
      done = true;
    }
  }
  if (!done) {
    for (int z0 = 0; z0 < n_parts; z0 += 8) {
      float q[8][V];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int i = 0; i < V; ++i)
          q[u][i] = (z0 + u < n_parts && lane * V + i < n_exp) ? __ldcg(lr + (z0 + u) * part_stride + i) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int i = 0; i < V; ++i) v[i] += q[u][i];
    }
  }
  if (rn.ssq) {
    // 1/rms of the row from the residual epilogue's per-tile sums of squares (fixed summation order)
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)rn.d + rn.eps);
    if (lane == 0) rn.r_out[row] = r;
    float* lo = rn.logits_out + (size_t)row * n_exp + lane * V;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      v[i] *= r;
      if (lane * V + i < n_exp) lo[i] = v[i];
    }
  }
#pragma unroll
  for (int i = 0; i < V; ++i)
    if (lane * V + i >= n_exp) v[i] = -INFINITY;
  uint32_t taken = 0;
  float first = 0.f, denom = 0.f, my_v = 0.f;
  int my_e = 0;
  for (int k = 0; k < top_k; ++k) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int e = lane * V + i;
      if (e < n_exp && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be / V == lane) taken |= 1u << (be % V);
    if (k == 0) first = bv;
    if (k == lane) {
      my_v = bv;
      my_e = be;
    }
    denom += __expf(bv - first);
  }
  if (lane < top_k) {
    sel[(size_t)row * top_k + lane] = my_e;
    gate[(size_t)row * top_k + lane] = __expf(my_v - first) / denom;
    atomicAdd(&counts[my_e], 1);
  }
}

// One CTA: expert offsets (exclusive prefix sum of the counts) and a row of the bucketed layout for
// every (token, rank) assignment.  Rows inside an expert are handed out with shared-memory atomics,
// so their order varies between runs; no result depends on it (each expert-GEMM column reads only
// its own row, and the combine sums a token's rows in rank order).
// Offsets (exclusive prefix sum of the counts, by the first 256 threads) and the bucketed row of
// every assignment; counts cleared for the next layer.  Needs blockDim.x >= 256.  Loads bypass L1
// (sel, gate and counts may come from other CTAs of the same launch).
__device__ void assign_rows_block(const int32_t* sel, const float* gate, int32_t* counts, int n_assign, int top_k,
                                  int n_exp, int32_t* __restrict__ offsets, int32_t* __restrict__ slot) {
  __shared__ int s_off[257];
  __shared__ int s_cur[256];
  __shared__ int s_wsum[8];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (threadIdx.x < 256) {
    const int c = threadIdx.x < n_exp ? __ldcg(counts + threadIdx.x) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[w] = incl;
    s_off[threadIdx.x] = incl - c;
    s_cur[threadIdx.x] = 0;
  }
  __syncthreads();
  // the counts are consumed: clear them for the next layer's router (no separate memset)
  if (threadIdx.x < n_exp) counts[threadIdx.x] = 0;
  if (threadIdx.x < 256) {
    int base = 0;
    for (int i = 0; i < w; ++i) base += s_wsum[i];
    s_off[threadIdx.x] += base;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int i = 0; i < 8; ++i) tot += s_wsum[i];
    s_off[n_exp] = tot;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= n_exp; e += blockDim.x) offsets[e] = s_off[e];
  // 8 assignments per thread per pass, their expert ids loaded together
  for (int a0 = threadIdx.x; a0 < n_assign; a0 += 8 * blockDim.x) {
    int e[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int a = a0 + u * blockDim.x;
      e[u] = a < n_assign ? __ldcg(sel + a) : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (e[u] >= 0) slot[a0 + u * blockDim.x] = s_off[e[u]] + atomicAdd(&s_cur[e[u]], 1);
  }
}

__global__ void assign_rows_kernel(const int32_t* __restrict__ sel, const float* __restrict__ gate,
                                   int32_t* __restrict__ counts, int n_assign, int top_k, int n_exp,
                                   int32_t* __restrict__ offsets, int32_t* __restrict__ slot) {
  pdl_trigger();
  pdl_wait();
  assign_rows_block(sel, gate, counts, n_assign, top_k, n_exp, offsets, slot);
}

// Many assignments (several canvases): the offsets come from one small CTA (prefix sum; per-expert
// cursors start at the offsets; counts cleared), then every assignment takes a row with a global
// atomic on its expert's cursor (row order inside an expert is free, as above).
__global__ void expert_offsets_kernel(int32_t* __restrict__ counts, int n_exp, int32_t* __restrict__ offsets,
                                      int32_t* __restrict__ cursor) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_wsum[8];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = threadIdx.x < n_exp ? counts[threadIdx.x] : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_wsum[w] = incl;
  __syncthreads();
  int base = 0;
  for (int i = 0; i < w; ++i) base += s_wsum[i];
  if (threadIdx.x < n_exp) {
    offsets[threadIdx.x] = base + incl - c;
    cursor[threadIdx.x] = base + incl - c;
    counts[threadIdx.x] = 0;
  }
  if (threadIdx.x == n_exp - 1) offsets[n_exp] = base + incl;
}

__global__ void scatter_rows_kernel(const int32_t* __restrict__ sel, int n_assign, int32_t* __restrict__ cursor,
                                    int32_t* __restrict__ slot) {
  pdl_trigger();
  pdl_wait();
  const int a = blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= n_assign) return;
  slot[a] = atomicAdd(&cursor[sel[a]], 1);
}

// 8 elements of a normed row: bf16(x * r * g), the product order of rmsnorm_kernel.
__device__ __forceinline__ uint4 norm8(const float4 (&x)[2], const float4 (&g)[2], float r) {
  const float4 a = x[0], b = x[1], ga = g[0], gb = g[1];
  return make_uint4(pack_bf16x2(a.x * r * ga.x, a.y * r * ga.y), pack_bf16x2(a.z * r * ga.z, a.w * r * ga.w),
                    pack_bf16x2(b.x * r * gb.x, b.y * r * gb.y), pack_bf16x2(b.z * r * gb.z, b.w * r * gb.w));
}

// Row t into its k bucketed rows (lane r < top_k holds rank r's row `my_slot`), one warp: the row is
// read once (xn[t], or with FROM_X the FFN RMSNorm formed here, bf16(x[t] * rr[t] * g)).
template <bool FROM_X>
__device__ __forceinline__ void gather_row(const __nv_bfloat16* __restrict__ xn, const float* __restrict__ x,
                                           const float* __restrict__ rr, const float* __restrict__ g, int t,
                                           int my_slot, int top_k, int d, __nv_bfloat16* __restrict__ xp, int lane) {
  const uint4* src = reinterpret_cast<const uint4*>(xn + (size_t)t * d);
  const float* xr = x + (size_t)t * d;
  const float r = FROM_X ? rr[t] : 0.f;
  const int n16 = d / 8;   // 16-byte chunks (8 elements) per bf16 row
  for (int c0 = 0; c0 < n16; c0 += 32 * 4) {
    uint4 v[4];
    if constexpr (FROM_X) {
      // all 16 loads of the 4 chunks in flight before any product
      float4 xa[4][2], ga[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < n16) {
          xa[u][0] = *reinterpret_cast<const float4*>(xr + 8 * c);
          xa[u][1] = *reinterpret_cast<const float4*>(xr + 8 * c + 4);
          ga[u][0] = __ldg(reinterpret_cast<const float4*>(g + 8 * c));
          ga[u][1] = __ldg(reinterpret_cast<const float4*>(g + 8 * c + 4));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = norm8(xa[u], ga[u], r);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < n16) v[u] = src[c];
      }
    }
    for (int r = 0; r < top_k; ++r) {
      uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)__shfl_sync(0xffffffffu, my_slot, r) * d);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < n16) dst[c] = v[u];
      }
    }
  }
}

// xp[slot[t*k + r]] = row t for every rank r: one warp per token.
template <bool FROM_X>
__global__ void gather_rows_kernel(const __nv_bfloat16* __restrict__ xn, const float* __restrict__ x,
                                   const float* __restrict__ rr, const float* __restrict__ g,
                                   const int32_t* __restrict__ slot, int n_rows, int top_k, int d,
                                   __nv_bfloat16* __restrict__ xp, int32_t* __restrict__ zero, int n_zero) {
  pdl_trigger();
  pdl_wait();
  if (zero && blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= n_rows) return;
  const int my_slot = lane < top_k ? slot[(size_t)t * top_k + lane] : 0;   // rank `lane`'s row, loaded once
  gather_row<FROM_X>(xn, x, rr, g, t, my_slot, top_k, d, xp, lane);
}

// One canvas, the gather folded into the top-k launch: one warp per row, two rows per CTA, every CTA
// resident at once (the grid fits the SMs).  Each warp takes its row's top-k (as router_topk_kernel);
// the last CTA to finish publishes the expert offsets (exclusive prefix of the counts) as cursors and
// raises a flag; every warp, once the flag is up (bounded wait), takes a bucketed row per rank with an
// atomic on its expert's cursor (row order inside an expert is free: each expert-GEMM column reads its
// own row, the combine sums a token's rows in rank order) and copies its normed row there.  The last
// CTA to leave lowers the flags for the next launch.  sync: [0] arrivals, [1] offsets ready, [2] leavers.
template <int V, bool FROM_X>
__global__ void router_topk_gather_kernel(const float* __restrict__ logits, int n_parts, size_t part_stride,
                                          int n_rows, int n_exp, int top_k, int32_t* __restrict__ sel,
                                          float* __restrict__ gate, int32_t* __restrict__ counts, RouterNorm rn,
                                          TopkGatherArgs ga) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row < n_rows)
    router_topk_row<V>(logits, n_parts, part_stride, row, n_rows, n_exp, top_k, sel, gate, counts, rn, lane);
  __shared__ int s_last;
  __shared__ int s_wsum[2];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ga.sync + 0, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (s_last) {
    __threadfence();
    // offsets: exclusive prefix of the counts (n_exp <= 256; 64 threads, 4 experts each)
    int c[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = threadIdx.x * 4 + i;
      c[i] = e < n_exp ? __ldcg(counts + e) : 0;
      tot += c[i];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_wsum[threadIdx.x >> 5] = incl;
    __syncthreads();
    int run = incl - tot + ((threadIdx.x >> 5) ? s_wsum[0] : 0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = threadIdx.x * 4 + i;
      if (e < n_exp) {
        ga.offsets[e] = run;
        ga.cursor[e] = run;
        counts[e] = 0;      // consumed: cleared for the next layer's router
      }
      run += c[i];
    }
    if (threadIdx.x == 0) ga.offsets[n_exp] = s_wsum[0] + s_wsum[1];
    for (int i = threadIdx.x; i < ga.n_zero; i += blockDim.x) ga.zero[i] = 0;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) atomicExch(ga.sync + 1, 1);
  }
  __shared__ int s_ready;
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    int ready = atomicAdd(ga.sync + 1, 0);
    for (uint32_t i = 1; ready == 0; ++i) {
      if ((i & 63) == 0 && globaltimer_ns() - t0 > kWaitTimeoutNs) {
        report_error(ga.err, DEV_ERR_TIMEOUT_ROUTE);
        break;
      }
      ready = atomicAdd(ga.sync + 1, 0);
    }
    s_ready = ready;
  }
  __syncthreads();
  __threadfence();
  // without the offsets (the wait ran out) the cursors are not valid: no row is taken or written
  if (s_ready && row < n_rows) {
    int my_slot = 0;
    if (lane < top_k) {
      const int e = sel[(size_t)row * top_k + lane];   // written by this lane above
      my_slot = atomicAdd(ga.cursor + e, 1);
      ga.slot[(size_t)row * top_k + lane] = my_slot;
    }
    gather_row<FROM_X>(ga.src.xn, ga.src.x, ga.src.r, ga.src.g, row, my_slot, top_k, ga.d, ga.xp, lane);
  }
  __syncthreads();
  if (threadIdx.x == 0 && atomicAdd(ga.sync + 2, 1) == (int)gridDim.x - 1) {
    ga.sync[0] = 0;
    ga.sync[1] = 0;
    ga.sync[2] = 0;
  }
}

// x[t] += sum over ranks r (in rank order) of gate[t][r] * y[slot[t*k + r]]; with g != nullptr also the next
// RMSNorm of the updated row: xn[t] = bf16(x[t] / sqrt(mean(x[t]^2) + eps) * g).
__global__ void moe_combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ slot,
                                   const float* __restrict__ gate, int top_k, int d, float* __restrict__ x,
                                   const float* __restrict__ g, float eps, __nv_bfloat16* __restrict__ xn) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  __shared__ int rows[32];
  __shared__ float gw[32];
  __shared__ float red[32];
  if (threadIdx.x < top_k) {
    rows[threadIdx.x] = slot[(size_t)t * top_k + threadIdx.x];
    gw[threadIdx.x] = gate[(size_t)t * top_k + threadIdx.x];
  }
  __syncthreads();
  float4* xr = reinterpret_cast<float4*>(x + (size_t)t * d);
  float ss = 0.f;
#pragma unroll 1
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 xo = xr[c];
    // ranks in batches of 8: the batch's loads are all in flight before its products are summed (rank order)
    for (int r0 = 0; r0 < top_k; r0 += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (r0 + u < top_k) v[u] = __ldcs(reinterpret_cast<const float4*>(y + (size_t)rows[r0 + u] * d) + c);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (r0 + u < top_k) {
          const float w = gw[r0 + u];
          acc.x += w * v[u].x; acc.y += w * v[u].y; acc.z += w * v[u].z; acc.w += w * v[u].w;
        }
    }
    float4 o = xo;
    o.x += acc.x; o.y += acc.y; o.z += acc.z; o.w += acc.w;
    xr[c] = o;
    ss += o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
  }
  if (!g) return;
  ss = block_sum_256(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  uint2* o2 = reinterpret_cast<uint2*>(xn + (size_t)t * d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = xr[c], w = g4[c];
    o2[c] = make_uint2(pack_bf16x2(v.x * inv * w.x, v.y * inv * w.y), pack_bf16x2(v.z * inv * w.z, v.w * inv * w.w));
  }
}

// out[i] = sum over planes z (in order) of in[z * stride + i]
__global__ void sum_planes_kernel(float* __restrict__ out, const float* __restrict__ in, int n_planes, size_t stride,
                                  size_t n) {
  pdl_trigger();
  pdl_wait();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = 0.f;
  for (int z = 0; z < n_planes; ++z) acc += in[z * stride + i];
  out[i] = acc;
}

__global__ void add_to_P_kernel(int* seq_P, int first, int count, int delta) {
  pdl_trigger();
  pdl_wait();
  const int i = threadIdx.x + blockIdx.x * blockDim.x;
  if (i < count) seq_P[first + i] += delta;
}

// Token-major prefix K/V [P][n_kv][dh] -> key cache [n_kv][max_ctx][dh] and transposed value cache
// [n_kv][dh][max_ctx] of one (layer, sequence).
__global__ void load_prefix_kernel(const __nv_bfloat16* __restrict__ k_in, const __nv_bfloat16* __restrict__ v_in,
                                   int n_kv, int dh, int max_ctx, __nv_bfloat16* __restrict__ kc,
                                   __nv_bfloat16* __restrict__ vt) {
  pdl_trigger();
  pdl_wait();
  const int pos = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
  const size_t src = ((size_t)pos * n_kv + h) * dh + c;
  kc[((size_t)h * max_ctx + pos) * dh + c] = k_in[src];
  vt[((size_t)h * dh + c) * max_ctx + pos] = v_in[src];
}

// Uniform random placeholder ids (uniform-state start of a canvas), commit mask cleared.
__global__ void canvas_init_kernel(const int* __restrict__ seq_P, int canvas, uint64_t seed, int vocab,
                                   int32_t* __restrict__ ids, uint8_t* __restrict__ commit) {
  pdl_trigger();
  pdl_wait();
  const int seq = blockIdx.x;
  const int P = seq_P ? seq_P[seq] : 0;
  for (int j = threadIdx.x; j < canvas; j += blockDim.x) {
    const uint4 w = rng_block(seed + (uint64_t)seq, 0u, (uint32_t)(P + j), 0u, RNG_TAG_INIT);
    ids[(size_t)seq * canvas + j] = token_from_word(w.x, (uint32_t)vocab);
    commit[(size_t)seq * canvas + j] = 0;
  }
}

// ---------------------------------------------------------------------------------------------
cudaError_t embed_rows(const __nv_bfloat16* emb, const int32_t* ids, int n_rows, int d, int vocab, float* x, int* err,
                       const float* g, float eps, __nv_bfloat16* xn, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  return launch_k(embed_kernel, dim3(n_rows), dim3(256), 0, st, 1, emb, ids, d, vocab, x, err, g, eps, xn);
}
cudaError_t rmsnorm_rows(const float* x, const float* g, int n_rows, int d, float eps, __nv_bfloat16* out,
                         cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  return launch_k(rmsnorm_kernel, dim3(n_rows), dim3(256), 0, st, 1, x, g, d, eps, out);
}
cudaError_t rope_table(float2* table, int max_ctx, int dh, float theta, cudaStream_t st) {
  return launch_k(rope_table_kernel, dim3(max_ctx), dim3(dh / 2), 0, st, 1, table, dh, (double)theta);
}
cudaError_t router_topk(const float* logits, int n_parts, size_t part_stride, int n_rows, int n_exp, int top_k,
                        int32_t* sel, float* gate, int32_t* counts, const FusedAssignArgs* fused,
                        const RouterNormArgs* norm, const ExpertPrefetchArgs* prefetch, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  const int V = (n_exp + 31) / 32;
  const dim3 grid((n_rows + 7) / 8);
  FusedAssign fa{};
  if (fused) fa = FusedAssign{fused->done, fused->offsets, fused->slot};
  RouterNorm rn{};
  if (norm) {
    if (!norm->ssq || !norm->r_out || !norm->logits_out || norm->n_ssq <= 0 || norm->d <= 0) return cudaErrorInvalidValue;
    rn = RouterNorm{norm->ssq, norm->n_ssq, norm->d, norm->eps, norm->r_out, norm->logits_out};
  }
  ExpertPrefetch pf{};
  if (prefetch && prefetch->w_gate_up) {
    if (prefetch->F % 64 || prefetch->row_bytes <= 0 || prefetch->row_bytes % 16 || prefetch->row_bytes > 2 * prefetch->d ||
        prefetch->n_ctas > n_exp * (prefetch->F / 64))
      return cudaErrorInvalidValue;
    pf = ExpertPrefetch{static_cast<const uint8_t*>(prefetch->w_gate_up), prefetch->n_ctas, prefetch->F, prefetch->d,
                        prefetch->row_bytes};
  }
#define DG_TOPK_CASE(V_) \
  if (V == V_) return launch_k(router_topk_kernel<V_>, grid, dim3(256), 0, st, 1, logits, n_parts, part_stride, n_rows, n_exp, top_k, sel, gate, counts, fa, rn, pf);
  DG_TOPK_CASE(1)
  DG_TOPK_CASE(2)
  DG_TOPK_CASE(4)
  DG_TOPK_CASE(8)
#undef DG_TOPK_CASE
  return cudaErrorInvalidValue;
}
cudaError_t router_topk_gather(const float* logits, int n_parts, size_t part_stride, int n_rows, int n_exp, int top_k,
                               int32_t* sel, float* gate, int32_t* counts, const RouterNormArgs* norm,
                               const TopkGatherLaunch& g, int n_sms, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  const int V = (n_exp + 31) / 32;
  const int blocks = (n_rows + 1) / 2;
  if (n_exp > 256 || top_k > 32 || g.d % 8 || blocks > n_sms || !g.sync || !g.offsets || !g.cursor || !g.slot || !g.xp ||
      (!g.src.xn && (!g.src.x || !g.src.r || !g.src.g)))
    return cudaErrorInvalidValue;   // every CTA must be resident at once: the grid fits the SMs
  RouterNorm rn{};
  if (norm) {
    if (!norm->ssq || !norm->r_out || !norm->logits_out || norm->n_ssq <= 0 || norm->d <= 0) return cudaErrorInvalidValue;
    rn = RouterNorm{norm->ssq, norm->n_ssq, norm->d, norm->eps, norm->r_out, norm->logits_out};
  }
  const TopkGatherArgs ga{g.src, g.xp, g.d, g.sync, g.offsets, g.cursor, g.slot, g.zero, g.n_zero, g.err};
  const bool fx = g.src.xn == nullptr;
#define DG_TG_CASE(V_)                                                                                              \
  if (V == V_)                                                                                                      \
    return fx ? launch_k(router_topk_gather_kernel<V_, true>, dim3(blocks), dim3(64), 0, st, 1, logits, n_parts,     \
                         part_stride, n_rows, n_exp, top_k, sel, gate, counts, rn, ga)                              \
              : launch_k(router_topk_gather_kernel<V_, false>, dim3(blocks), dim3(64), 0, st, 1, logits, n_parts,    \
                         part_stride, n_rows, n_exp, top_k, sel, gate, counts, rn, ga);
  DG_TG_CASE(1)
  DG_TG_CASE(2)
  DG_TG_CASE(4)
  DG_TG_CASE(8)
#undef DG_TG_CASE
  return cudaErrorInvalidValue;
}
cudaError_t assign_rows(const int32_t* sel, const float* gate, int32_t* counts, int n_rows, int top_k, int n_exp,
                        int32_t* offsets, int32_t* cursor, int32_t* slot, int* n_launched, cudaStream_t st) {
  if (n_exp > 256) return cudaErrorInvalidValue;
  const int n_assign = n_rows * top_k;
  if (n_assign <= 8192) {   // one canvas: a single CTA does both (one launch)
    *n_launched = 1;
    return launch_k(assign_rows_kernel, dim3(1), dim3(1024), 0, st, 1, sel, gate, counts, n_assign, top_k, n_exp,
                    offsets, slot);
  }
  *n_launched = 2;
  cudaError_t e = launch_k(expert_offsets_kernel, dim3(1), dim3(256), 0, st, 1, counts, n_exp, offsets, cursor);
  if (e != cudaSuccess) return e;
  return launch_k(scatter_rows_kernel, dim3((n_assign + 255) / 256), dim3(256), 0, st, 1, sel, n_assign, cursor, slot);
}
cudaError_t gather_rows(const GatherSrc& src, const int32_t* slot, int n_rows, int top_k, int d, __nv_bfloat16* xp,
                        cudaStream_t st, int32_t* zero, int n_zero) {
  if (n_rows <= 0) return cudaSuccess;
  if (d % 8 || (!src.xn && (!src.x || !src.r || !src.g))) return cudaErrorInvalidValue;
  // two tokens (warps) per CTA: the copy of 256 tokens spreads over 128 SMs
  if (src.xn)
    return launch_k(gather_rows_kernel<false>, dim3((n_rows + 1) / 2), dim3(64), 0, st, 1, src.xn, src.x, src.r, src.g,
                    slot, n_rows, top_k, d, xp, zero, n_zero);
  return launch_k(gather_rows_kernel<true>, dim3((n_rows + 1) / 2), dim3(64), 0, st, 1, src.xn, src.x, src.r, src.g,
                  slot, n_rows, top_k, d, xp, zero, n_zero);
}
cudaError_t moe_combine(const float* y, const int32_t* slot, const float* gate, int n_rows, int top_k, int d, float* x,
                        const float* g, float eps, __nv_bfloat16* xn, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  return launch_k(moe_combine_kernel, dim3(n_rows), dim3(256), 0, st, 1, y, slot, gate, top_k, d, x, g, eps, xn);
}
cudaError_t sum_planes(float* out, const float* in, int n_planes, size_t stride, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  return launch_k(sum_planes_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, 1, out, in, n_planes, stride, n);
}
cudaError_t add_to_P(int* seq_P, int first, int count, int delta, cudaStream_t st) {
  return launch_k(add_to_P_kernel, dim3((count + 127) / 128), dim3(128), 0, st, 1, seq_P, first, count, delta);
}
cudaError_t load_prefix(const __nv_bfloat16* k_in, const __nv_bfloat16* v_in, int P, int n_kv, int dh, int max_ctx,
                        __nv_bfloat16* kc, __nv_bfloat16* vt, cudaStream_t st) {
  if (P <= 0) return cudaSuccess;
  return launch_k(load_prefix_kernel, dim3(P, n_kv), dim3(dh), 0, st, 1, k_in, v_in, n_kv, dh, max_ctx, kc, vt);
}
cudaError_t canvas_init_ids(const int* seq_P, int n_seq, int canvas, uint64_t seed, int vocab, int32_t* ids,
                            uint8_t* commit, cudaStream_t st) {
  return launch_k(canvas_init_kernel, dim3(n_seq), dim3(256), 0, st, 1, seq_P, canvas, seed, vocab, ids, commit);
}

// The adaptive-stop test of the block loop ("Composition of DiffusionGemma" flowchart: refine, check
// the stop condition, refine again) on the device: after a step, advance the step index and let the
// graph's while-node run the body again unless every sequence has stopped or the budget is spent.
__global__ void decode_loop_control_kernel(const int32_t* __restrict__ stop, int n_seq, int* step, int budget,
                                           cudaGraphConditionalHandle handle) {
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x != 0) return;
  int all = 1;
  for (int i = 0; i < n_seq; ++i) all &= stop[i] != 0;
  const int s = *step + 1;
  *step = s;
  cudaGraphSetConditional(handle, (!all && s < budget) ? 1u : 0u);
}

cudaError_t decode_loop_control(const int32_t* stop, int n_seq, int* step, int budget,
                                cudaGraphConditionalHandle handle, cudaStream_t st) {
  return launch_k(decode_loop_control_kernel, dim3(1), dim3(32), 0, st, 1, stop, n_seq, step, budget, handle);
}

}  // namespace dg
