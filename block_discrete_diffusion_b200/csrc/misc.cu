// misc.cu -- bandwidth/latency kernels around the GEMMs: embedding gather, RMSNorm, the rotary
// table, the top-k router, expert bucketing with the activation gather, the MoE combine, canvas
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
                             float* __restrict__ x, int* err) {
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
}

// out[r] = bf16( x[r] / sqrt(mean(x[r]^2) + eps) * g )
__global__ void rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ g, int d, float eps,
                               __nv_bfloat16* __restrict__ out) {
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
  const int pos = blockIdx.x, i = threadIdx.x;
  const double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)dh);
  double s, c;
  sincos(ang, &s, &c);
  table[(size_t)pos * (dh / 2) + i] = make_float2((float)c, (float)s);
}

// One warp per row: the top_k largest router logits (ties -> lower expert id), gates = softmax over
// the selected logits; per-expert counts accumulate with integer atomics (order-free, exact).
__global__ void router_topk_kernel(const float* __restrict__ logits, int n_rows, int n_exp, int top_k,
                                   int32_t* __restrict__ sel, float* __restrict__ gate, int32_t* __restrict__ counts) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  constexpr int kPer = 8;   // up to 256 experts
  float v[kPer];
  const float* lr = logits + (size_t)row * n_exp;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = i * 32 + lane;
    v[i] = e < n_exp ? lr[e] : -INFINITY;
  }
  uint32_t taken = 0;
  float first = 0.f, denom = 0.f, my_v = 0.f;
  int my_e = 0;
  for (int k = 0; k < top_k; ++k) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = i * 32 + lane;
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
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
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

// One CTA per expert: stable bucketing of the (token, rank) assignments routed to expert e (token
// order kept), then the gather of their normalised activation rows into the bucketed buffer.
__global__ void bucket_gather_kernel(const int32_t* __restrict__ sel, const float* __restrict__ gate,
                                     const int32_t* __restrict__ counts, int n_assign, int top_k, int n_exp,
                                     const __nv_bfloat16* __restrict__ xn, int d, int32_t* __restrict__ offsets,
                                     float* __restrict__ perm_gate, int32_t* __restrict__ perm_tok,
                                     int32_t* __restrict__ slot, __nv_bfloat16* __restrict__ xp) {
  __shared__ int warp_cnt[32];
  __shared__ int s_off;
  const int e = blockIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) {
    int o = 0;
    for (int i = 0; i < e; ++i) o += counts[i];
    s_off = o;
    offsets[e] = o;
    if (e == n_exp - 1) offsets[n_exp] = o + counts[e];
  }
  __syncthreads();
  const int off = s_off;
  int running = 0;
  for (int base = 0; base < n_assign; base += blockDim.x) {
    const int a = base + threadIdx.x;
    const bool flag = a < n_assign && sel[a] == e;
    const uint32_t mask = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_cnt[w] = __popc(mask);
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < nw; ++i) {
      before += i < w ? warp_cnt[i] : 0;
      total += warp_cnt[i];
    }
    if (flag) {
      const int row = off + running + before + __popc(mask & ((1u << lane) - 1u));
      perm_gate[row] = gate[a];
      perm_tok[row] = a / top_k;
      slot[a] = row;
    }
    running += total;
    __syncthreads();
  }
  const int cnt = counts[e];
  for (int r = off + w; r < off + cnt; r += nw) {
    const uint4* src = reinterpret_cast<const uint4*>(xn + (size_t)perm_tok[r] * d);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * d);
    for (int c = lane; c < d / 8; c += 32) dst[c] = src[c];
  }
}

// x[t] += sum over ranks r (in rank order) of y[slot[t*k + r]]
__global__ void moe_combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ slot, int top_k, int d,
                                   float* __restrict__ x) {
  const int t = blockIdx.x;
  __shared__ int rows[32];
  if (threadIdx.x < top_k) rows[threadIdx.x] = slot[(size_t)t * top_k + threadIdx.x];
  __syncthreads();
  float4* xr = reinterpret_cast<float4*>(x + (size_t)t * d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < top_k; ++r) {
      const float4 v = reinterpret_cast<const float4*>(y + (size_t)rows[r] * d)[c];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    float4 o = xr[c];
    o.x += acc.x; o.y += acc.y; o.z += acc.z; o.w += acc.w;
    xr[c] = o;
  }
}

__global__ void add_to_P_kernel(int* seq_P, int first, int count, int delta) {
  const int i = threadIdx.x + blockIdx.x * blockDim.x;
  if (i < count) seq_P[first + i] += delta;
}

// Token-major prefix K/V [P][n_kv][dh] -> key cache [n_kv][max_ctx][dh] and transposed value cache
// [n_kv][dh][max_ctx] of one (layer, sequence).
__global__ void load_prefix_kernel(const __nv_bfloat16* __restrict__ k_in, const __nv_bfloat16* __restrict__ v_in,
                                   int n_kv, int dh, int max_ctx, __nv_bfloat16* __restrict__ kc,
                                   __nv_bfloat16* __restrict__ vt) {
  const int pos = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
  const size_t src = ((size_t)pos * n_kv + h) * dh + c;
  kc[((size_t)h * max_ctx + pos) * dh + c] = k_in[src];
  vt[((size_t)h * dh + c) * max_ctx + pos] = v_in[src];
}

// Uniform random placeholder ids (uniform-state start of a canvas), commit mask cleared.
__global__ void canvas_init_kernel(const int* __restrict__ seq_P, int canvas, uint64_t seed, int vocab,
                                   int32_t* __restrict__ ids, uint8_t* __restrict__ commit) {
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
                       cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  embed_kernel<<<n_rows, 256, 0, st>>>(emb, ids, d, vocab, x, err);
  return cudaGetLastError();
}
cudaError_t rmsnorm_rows(const float* x, const float* g, int n_rows, int d, float eps, __nv_bfloat16* out,
                         cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  rmsnorm_kernel<<<n_rows, 256, 0, st>>>(x, g, d, eps, out);
  return cudaGetLastError();
}
cudaError_t rope_table(float2* table, int max_ctx, int dh, float theta, cudaStream_t st) {
  rope_table_kernel<<<max_ctx, dh / 2, 0, st>>>(table, dh, (double)theta);
  return cudaGetLastError();
}
cudaError_t router_topk(const float* logits, int n_rows, int n_exp, int top_k, int32_t* sel, float* gate,
                        int32_t* counts, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  router_topk_kernel<<<(n_rows + 7) / 8, 256, 0, st>>>(logits, n_rows, n_exp, top_k, sel, gate, counts);
  return cudaGetLastError();
}
cudaError_t bucket_gather(const int32_t* sel, const float* gate, const int32_t* counts, int n_rows, int top_k,
                          int n_exp, const __nv_bfloat16* xn, int d, int32_t* offsets, float* perm_gate,
                          int32_t* perm_tok, int32_t* slot, __nv_bfloat16* xp, cudaStream_t st) {
  bucket_gather_kernel<<<n_exp, 256, 0, st>>>(sel, gate, counts, n_rows * top_k, top_k, n_exp, xn, d, offsets,
                                              perm_gate, perm_tok, slot, xp);
  return cudaGetLastError();
}
cudaError_t moe_combine(const float* y, const int32_t* slot, int n_rows, int top_k, int d, float* x,
                        cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  moe_combine_kernel<<<n_rows, 256, 0, st>>>(y, slot, top_k, d, x);
  return cudaGetLastError();
}
cudaError_t add_to_P(int* seq_P, int first, int count, int delta, cudaStream_t st) {
  add_to_P_kernel<<<(count + 127) / 128, 128, 0, st>>>(seq_P, first, count, delta);
  return cudaGetLastError();
}
cudaError_t load_prefix(const __nv_bfloat16* k_in, const __nv_bfloat16* v_in, int P, int n_kv, int dh, int max_ctx,
                        __nv_bfloat16* kc, __nv_bfloat16* vt, cudaStream_t st) {
  if (P <= 0) return cudaSuccess;
  load_prefix_kernel<<<dim3(P, n_kv), dh, 0, st>>>(k_in, v_in, n_kv, dh, max_ctx, kc, vt);
  return cudaGetLastError();
}
cudaError_t canvas_init_ids(const int* seq_P, int n_seq, int canvas, uint64_t seed, int vocab, int32_t* ids,
                            uint8_t* commit, cudaStream_t st) {
  canvas_init_kernel<<<n_seq, 256, 0, st>>>(seq_P, canvas, seed, vocab, ids, commit);
  return cudaGetLastError();
}

}  // namespace dg
