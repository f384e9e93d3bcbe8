// dg_api.cu -- the C ABI (include/dg.h): handles, workspace layout, TMA descriptors and the launch
// sequences of prefill, canvas step, block commit and the decode loop.  Host code only; every step
// of the method runs in the kernels of gemm.cu, attention.cu, misc.cu and sampler.cu.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "dg.h"
#include "dg_kernels.h"

#define DG_API extern "C" __attribute__((visibility("default")))

using namespace dg;

bool dg::pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("DG_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

namespace {

thread_local char g_err[512] = "";

dg_status fail(dg_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

#define CK(call)                                                                                     \
  do {                                                                                               \
    cudaError_t e_ = (call);                                                                         \
    if (e_ != cudaSuccess) return fail(DG_ERR_CUDA, "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                                       __FILE__, __LINE__);                                          \
  } while (0)

// NVTX range for the lifetime of one API call (profilers filter kernels by it).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

constexpr int kCanvas = 256;
constexpr int kAttnTargetCtas = 148;    // attention CTAs hold a whole SM (all of TMEM)
constexpr int kMaxSplits = 16;
constexpr int kRouterSplits = 8;        // cluster size of the router GEMM's split-K
constexpr int kGemmTargetCtas = 296;    // two CTAs per SM for the 128-wide dense GEMM tiles
constexpr int kSplitKSlots = kGemmTargetCtas;   // split-K partial tiles: tiles x splits <= this (dense_splits)
constexpr int kHeadSamplerMaxCtas = 256;        // CTAs of the fused head + sampler (one per SM)
constexpr int kRouteRows = 1024;                // rows up to which the router folds into the O epilogue

// Cluster size (power of two, <= 8) of the split-K dense GEMMs for `tiles` output tiles over nk
// 64-deep k-blocks: enough CTAs for about two per SM, at least 4 k-blocks per CTA.
int dense_splits(int tiles, int nk) {
  int z = 1;
  while (z < 8 && tiles * z * 2 <= kGemmTargetCtas && nk / (z * 2) >= 4) z *= 2;
  return z;
}

// ---------------------------------------------------------------------------------------------
// TMA descriptor creation through the driver entry point (no libcuda link dependency)
// ---------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 [rows][cols] (cols contiguous), box box_rows x 64, 128-byte swizzle.
dg_status map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (cols * 2) % 16)
    return fail(DG_ERR_INVALID_ARG, "TMA operand not 16-byte aligned (ptr %p, row bytes %llu)", ptr,
                (unsigned long long)(cols * 2));
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (2d, %llux%llu box %u) failed: %d",
                                     (unsigned long long)rows, (unsigned long long)cols, box_rows, (int)r);
  return DG_OK;
}

// 2-D bytes [rows][cols] (e4m3 weights), box box_rows x 64 bytes, no swizzle (rows land 64 bytes
// apart; the expert kernel's converter warps lay them out for the tensor cores).
dg_status map_2d_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || cols % 16)
    return fail(DG_ERR_INVALID_ARG, "FP8 TMA operand not 16-byte aligned (ptr %p, row bytes %llu)", ptr,
                (unsigned long long)cols);
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (2d u8, %llux%llu box %u) failed: %d",
                                     (unsigned long long)rows, (unsigned long long)cols, box_rows, (int)r);
  return DG_OK;
}

// 2-D bytes [rows][cols] (e4m3 operands of the tensor cores), box box_rows x 128 bytes, 128-byte swizzle
// (the K-major layout kind::f8f6f4 reads: 128 K elements per 128-byte row).
dg_status map_2d_u8_sw128(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || cols % 16)
    return fail(DG_ERR_INVALID_ARG, "FP8 TMA operand not 16-byte aligned (ptr %p, row bytes %llu)", ptr,
                (unsigned long long)cols);
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (2d u8 sw128, %llux%llu box %u) failed: %d",
                                     (unsigned long long)rows, (unsigned long long)cols, box_rows, (int)r);
  return DG_OK;
}

// 3-D bf16 [d2][d1][d0] (d0 contiguous), box {64, box1, 1}, 128-byte swizzle.
dg_status map_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1) {
  EncodeTiledFn f = encode_fn();
  if (!f) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (3d) failed: %d", (int)r);
  return DG_OK;
}

// ---------------------------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------------------------
struct WsLayout {
  int R, A, split_cap, chunks;
  size_t err, seqP, x, xn, q, opart, ml, attn, rlog, sel, gate, counts, offsets, slot, xp, hb,
      y, logits, samp, hsamp, rope, cids, ccommit, cH, cstop, splitk, head_off, cursor, topk_done, dstep, bsteps,
      xq, xs, hq, hs, xdone, rpart, ssq, rr, total;
  int route_rows;   // rows up to which the FFN RMSNorm and router fold into the O epilogue (0: never)
  bool f8mma;     // FP8 form: e4m3 activations for the e4m3 x e4m3 expert GEMMs
  size_t wq[5];   // FP8 form only: one layer's matrices in bf16 (qkv, o, router, gate_up, down)
};

// Elements of the five per-layer matrices, in the order qkv, o, router, gate_up, down.
void layer_matrix_shapes(const dg_model_config& c, uint64_t rows[5], uint64_t cols[5]) {
  const uint64_t d = c.d_model;
  rows[0] = (uint64_t)(c.n_q + 2 * c.n_kv) * c.d_head; cols[0] = d;
  rows[1] = d;                                       cols[1] = (uint64_t)c.n_q * c.d_head;
  rows[2] = c.n_exp;                                 cols[2] = d;
  rows[3] = (uint64_t)c.n_exp * 2 * c.d_ff;          cols[3] = d;
  rows[4] = (uint64_t)c.n_exp * d;                   cols[4] = c.d_ff;
}

// Key splits of the attention.  A CTA (a pair of 128-row query tiles) holds a whole SM.  Few
// CTAs: split the keys until about one wave is busy.  Many CTAs: at most 4 splits, the count that
// wastes the least of the last wave (a split costs one merge pass, so 1 wins near-ties).
int attn_split_cap(const dg_model_config& c, int n_seq) {
  const int G = c.n_q / c.n_kv;
  const int pairs = (G * kCanvas + 255) / 256;
  const int base = pairs * n_seq * c.n_kv;
  if (base < kAttnTargetCtas) return std::max(1, std::min(kMaxSplits, kAttnTargetCtas / base));   // one wave
  int best = 1;
  double best_eff = 0.0;
  for (int sp = 1; sp <= 4; ++sp) {
    const int ctas = base * sp;
    const int waves = (ctas + kAttnTargetCtas - 1) / kAttnTargetCtas;
    const double eff = (double)ctas / ((double)waves * kAttnTargetCtas) - 0.02 * (sp > 1);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = sp;
    }
  }
  return best;
}

// Many tokens per expert on average (several canvases): 256-token accumulator chunks.  DG_EXPERT_WIDE
// = 0 / 1 forces the narrow (32 or 64-token) / wide chunks for every row count (read once).
bool expert_chunks_wide(const dg_model_config& c, int rows) {
  static const int force = [] {
    const char* v = getenv("DG_EXPERT_WIDE");
    return v ? (atoi(v) != 0 ? 1 : 0) : -1;
  }();
  if (force >= 0) return force == 1;
  return rows * c.top_k >= 128 * c.n_exp;
}

WsLayout ws_layout(const dg_model_config& c, int n_seq, int max_ctx) {
  WsLayout L{};
  L.R = n_seq * kCanvas;
  L.A = L.R * c.top_k;
  L.split_cap = attn_split_cap(c, n_seq);
  L.chunks = sampler_chunks(c.vocab);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 1023) & ~size_t(1023);
    return o;
  };
  const size_t d = c.d_model, R = L.R, A = L.A, dh = c.d_head, nq = c.n_q;
  L.err = take(64);
  L.seqP = take(sizeof(int) * n_seq);
  L.x = take(4 * R * d);
  L.xn = take(2 * R * d);
  L.q = take(2 * (size_t)n_seq * nq * kCanvas * dh);
  L.opart = take(2 * (size_t)L.split_cap * n_seq * nq * kCanvas * dh);
  L.ml = take(8 * (size_t)L.split_cap * n_seq * nq * kCanvas);
  L.attn = take(2 * R * nq * dh);
  L.rlog = take(4 * R * c.n_exp);
  L.sel = take(4 * A);
  L.gate = take(4 * A);
  L.counts = take(4 * (size_t)c.n_exp);
  L.offsets = take(4 * (size_t)(c.n_exp + 1));
  L.slot = take(4 * A);
  L.xp = take(2 * A * d);
  L.hb = take(2 * A * (size_t)c.d_ff);
  L.y = take(4 * A * d);
  L.logits = take(4 * R * (size_t)c.vocab);
  L.samp = take(4 * 8 * R * (size_t)L.chunks);
  L.hsamp = take(4 * 8 * (size_t)kCanvas * (kHeadSamplerMaxCtas + 1));   // one canvas: the fused head's records
  L.rope = take(8 * (size_t)max_ctx * (dh / 2));
  L.cids = take(4 * R);
  L.ccommit = take(R);
  L.cH = take(4 * R);
  L.cstop = take(4 * (size_t)n_seq);
  L.splitk = take(4 * (size_t)kSplitKSlots * 128 * 128);
  L.head_off = take(8);
  L.cursor = take(4 * 256);
  L.topk_done = take(64);
  L.dstep = take(64);
  L.xdone = take(4 * (size_t)c.n_exp);
  // the FFN RMSNorm + router folded into the O-projection epilogue (up to kRouteRows rows: the
  // per-tile partial planes stay small): router partials [d/128][rows][E], sums of squares, 1/rms
  L.route_rows = (c.n_exp % 8 == 0 && c.n_exp <= 128) ? std::min(L.R, kRouteRows) : 0;
  if (L.route_rows) {
    L.rpart = take(4 * (d / 128) * (size_t)L.route_rows * c.n_exp);
    L.ssq = take(4 * (d / 128) * (size_t)L.route_rows);
    L.rr = take(4 * (size_t)L.route_rows);
  }
  L.bsteps = take(4 * ((size_t)max_ctx / kCanvas + 1));
  if (c.wdtype == DG_WDTYPE_FP8_BLOCK128) {
    uint64_t rows[5], cols[5];
    layer_matrix_shapes(c, rows, cols);
    for (int i = 0; i < 3; ++i) L.wq[i] = take(2 * rows[i] * cols[i]);   // the expert GEMMs read e4m3 directly
    // the expert GEMMs multiply e4m3 by e4m3 (quantized activations + scales): few tokens per expert
    // on single CTAs, many on CTA pairs
    L.f8mma = c.d_model % 128 == 0 && c.d_ff % 64 == 0;
    if (L.f8mma) {
      L.xq = take(A * d);
      L.xs = take(4 * A * (d / 128));
      L.hq = take(A * (size_t)c.d_ff);
      L.hs = take(4 * A * (size_t)(c.d_ff / 64));
    }
  }

  L.total = off + 1024;   // slack for base alignment
  return L;
}

bool shape_ok(const dg_model_config* c, const char** why) {
  if (!c) return (*why = "null config", false);
  if (c->d_head != 64 && c->d_head != 128) return (*why = "d_head must be 64 or 128", false);
  if (c->d_model <= 0 || c->d_model % 128) return (*why = "d_model must be a positive multiple of 128", false);
  if (c->d_ff <= 0 || c->d_ff % 64) return (*why = "d_ff must be a positive multiple of 64", false);
  if (c->n_q <= 0 || c->n_kv <= 0 || c->n_q % c->n_kv) return (*why = "n_q must be a multiple of n_kv", false);
  if ((c->n_q * c->d_head) % 128 || (c->n_kv * c->d_head) % 128)
    return (*why = "n_q*d_head and n_kv*d_head must be multiples of 128", false);
  if (c->n_exp <= 0 || c->n_exp > 256) return (*why = "n_exp must be in [1, 256]", false);
  if (c->top_k <= 0 || c->top_k > 32 || c->top_k > c->n_exp) return (*why = "top_k must be in [1, min(32, n_exp)]", false);
  if (c->n_layers <= 0) return (*why = "n_layers must be positive", false);
  if (c->vocab <= 0 || c->vocab % 1024) return (*why = "vocab must be a positive multiple of 1024", false);
  if (c->wdtype != DG_WDTYPE_BF16 && c->wdtype != DG_WDTYPE_FP8_BLOCK128) return (*why = "unknown wdtype", false);
  if (c->wdtype == DG_WDTYPE_FP8_BLOCK128 && (2 * c->d_ff) % 128)
    return (*why = "FP8 weights need 2 d_ff % 128 == 0", false);
  if (c->wdtype == DG_WDTYPE_FP8_BLOCK128 && (c->d_model > 32 * 128 || c->d_ff > 32 * 128))
    return (*why = "FP8 weights need d_model, d_ff <= 4096 (32 scale blocks per row)", false);
  return true;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

dg_status dg::record_error(dg_status st, const char* msg) {
  snprintf(g_err, sizeof g_err, "%s", msg);
  return st;
}

// The sampler settings every entry point shares.  The temperature schedule is only defined on
// steps 0 .. max_steps - 1 (it reaches t_end at the last one and would extrapolate past it), so a
// fixed budget above max_steps and a step outside the schedule are rejected.
dg_status dg::check_sampler_params(const dg_sampler_params* p, int step, const char* fn) {
  if (!p) return fail(DG_ERR_INVALID_ARG, "%ssampler params are null", fn);
  if (p->canvas_len != kCanvas) return fail(DG_ERR_UNSUPPORTED, "%scanvas_len must be 256", fn);
  if (p->max_steps <= 0 || p->fixed_steps < 0) return fail(DG_ERR_INVALID_ARG, "%sbad step budget", fn);
  if (p->fixed_steps > p->max_steps)
    return fail(DG_ERR_INVALID_ARG, "%sfixed_steps %d exceeds max_steps %d (the temperature schedule's length)", fn,
                p->fixed_steps, p->max_steps);
  if (!(p->t_start > 0.f) || !(p->t_end > 0.f)) return fail(DG_ERR_INVALID_ARG, "%stemperatures must be > 0", fn);
  if (p->commit_mode != 0 && p->commit_mode != 1) return fail(DG_ERR_INVALID_ARG, "%scommit_mode must be 0 or 1", fn);
  if (p->commit_rule != 0 && p->commit_rule != 1) return fail(DG_ERR_INVALID_ARG, "%scommit_rule must be 0 or 1", fn);
  if (step >= p->max_steps)
    return fail(DG_ERR_INVALID_ARG, "%sstep %d is outside the %d-step temperature schedule", fn, step, p->max_steps);
  return DG_OK;
}

// ---------------------------------------------------------------------------------------------
// handles
// ---------------------------------------------------------------------------------------------
struct LayerMaps {
  CUtensorMap wqkv, wo, wrouter, wgu, wdown;
  CUtensorMap wgu8, wdown8;   // FP8 form: the expert matrices with 128-byte swizzled boxes (e4m3 MMA)
};

struct dg_model {
  dg_model_config cfg;
  int n_sms;   // streaming multiprocessors of the current device (persistent grids)
  const __nv_bfloat16 *emb, *head;
  const float* final_norm;
  std::vector<dg_layer_weights> layers;
  std::vector<LayerMaps> maps;
  CUtensorMap head_map;      // 256-row boxes (dense head GEMM)
  CUtensorMap head_map128;   // 128-row boxes (persistent swap-AB head GEMM)
  bool fp8;   // per-layer matrices in the FP8 block-scaled form (expanded per layer into the workspace)
};

struct dg_seqs {
  dg_model* m;
  int n_seq, max_ctx;
  cudaStream_t st;
  __nv_bfloat16 *kc, *vt;
  WsLayout L;
  uint8_t* ws;
  // typed workspace views
  int *err, *seqP;
  float *x, *ml, *rlog, *gate, *y, *logits, *samp, *hsamp, *splitk;
  __nv_bfloat16* opart;   // attention key-split partial outputs
  __nv_bfloat16 *xn, *q, *attn, *xp, *hb;
  int32_t *sel, *counts, *offsets, *slot, *cids, *cstop;
  uint8_t* ccommit;
  float* cH;

  float2* rope;
  CUtensorMap xn_map, xp_map, attn_map, hb_map, q_map, k_map, v_map;
  LayerMaps wmaps;              // FP8 form: descriptors of the bf16 scratch matrices
  CUtensorMap xn32_map;         // xn in 32-row boxes (token operand of the persistent head GEMM)
  CUtensorMap xq_map, hq_map;   // FP8 form, few tokens per expert: e4m3 token operands (32-row boxes)
  uint8_t *xq, *hq;             // ... the gathered rows and the SwiGLU rows in e4m3
  float *xs, *hs;               // ... and their scales
  bool fp8_native;              // use the e4m3 x e4m3 expert GEMMs where available (DG_FP8_NATIVE, default on)
  bool fp8_pair;                // many tokens per expert: the CTA-pair e4m3 kernels (DG_FP8_PAIR=1; off by
                                // default), else the kernels that expand e4m3 weights to bf16
  int32_t* xdone;               // per-expert count of finished gate|up tiles (merged expert launch)
  float* rpart;                 // folded router: per-tile router partials, sums of squares, 1/rms per row
  float* ssq;
  float* rr;
  bool route_fused;             // fold the FFN RMSNorm + router into the O epilogue (DG_ROUTE_FUSED, default on)
  bool expert_merged;           // bf16, narrow chunks: gate|up and down in one launch (DG_EXPERT_MERGED, default on)
  bool head_fused_batch;        // several canvases: the fused head + sampler once per canvas (DG_HEAD_FUSED_BATCH,
                                // default on), else the dense head GEMM + the sampler over all logits
  int32_t* head_off;            // {0, R}: all rows as one "expert" for the persistent head GEMM
  int32_t* cursor;              // per-expert row cursors of the multi-CTA bucketing
  int32_t* topk_done;           // launch counter of the top-k kernel that also buckets
  int* dstep;                   // the device-resident block loop: step index of the current block
  int* bsteps;                  // ... and the step count of each block of a dg_decode call
  int attn_plan_P;              // >= 0: plan the attention key splits for this committed length (a captured
                                // step body serves every block of a decode call); -1: the current lengths
  cudaStream_t cap_stream;      // private stream the decode loop's step body is captured on (lazily created)
  int decode_graph;             // dg_decode runs each block's steps as a CUDA graph while-loop (DG_DECODE_GRAPH)
  cudaGraphExec_t loop_exec;    // that graph, kept for later dg_decode calls with the same sampler settings
  dg_sampler_params loop_prm;   // (its attention splits are planned for the largest committed length,
                                // max_ctx - 256, so it serves every block of every call)
  __nv_bfloat16* wq[5];         // FP8 form: the scratch matrices (qkv, o, router, gate_up, down)
  std::vector<int> P;   // host mirror of the committed lengths
  int step;
  bool block_open;
  int max_splits;   // upper bound on attention key splits (DG_ATTN_MAX_SPLITS, default: no extra bound)
  bool attn_cluster_merge;   // key splits merged inside the attention launch (DG_ATTN_CLUSTER_MERGE=1; off by default)
  int pre_bytes;    // bytes per weight row the gate|up GEMM brings into L2 before its wait (DG_EXPERT_PREFETCH)
  bool prefetch_early;   // merged expert launch: the top-k launch issues that prefetch too (DG_PREFETCH_EARLY=1)
  bool topk_gather;      // one canvas, merged experts: bucketing + gather inside the top-k launch (DG_TOPK_GATHER=1)
  int head_nv;      // one canvas: tiling of the fused head + sampler (kHeadSamplerPair: CTA pairs; 128 or 256
                    // vocabulary rows per single-SM tile; 0: the head GEMM writes the logits and the
                    // standalone sampler reads them; DG_HEAD_SAMPLER)
  // statistics: launches per kernel class; optional event timing
  long long launches[DG_K_COUNT];
  double ms[DG_K_COUNT];
  bool timing;
  std::vector<cudaEvent_t> events;            // pairs (start, end)
  std::vector<std::pair<int, int>> pending;   // (class, pair index) not yet folded into ms
  int next_pair;
  ~dg_seqs() {
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    if (loop_exec) {
      cudaStreamSynchronize(st);
      cudaGraphExecDestroy(loop_exec);
    }
    if (cap_stream) cudaStreamDestroy(cap_stream);
  }
};

namespace {

constexpr int kEventPairs = 4096;

cudaError_t stats_fold(dg_seqs* s) {
  if (s->pending.empty()) return cudaSuccess;
  cudaError_t e = cudaStreamSynchronize(s->st);
  if (e != cudaSuccess) return e;
  for (auto& pr : s->pending) {
    float t = 0.f;
    e = cudaEventElapsedTime(&t, s->events[2 * pr.second], s->events[2 * pr.second + 1]);
    if (e != cudaSuccess) return e;
    s->ms[pr.first] += t;
  }
  s->pending.clear();
  s->next_pair = 0;
  return cudaSuccess;
}

int stats_begin(dg_seqs* s) {
  if (!s->timing) return -1;
  if (s->next_pair >= kEventPairs && stats_fold(s) != cudaSuccess) return -1;
  const int i = s->next_pair++;
  cudaEventRecord(s->events[2 * i], s->st);
  return i;
}

void stats_end(dg_seqs* s, int cls, int n_kernels, int pair) {
  s->launches[cls] += n_kernels;
  if (pair >= 0) {
    cudaEventRecord(s->events[2 * pair + 1], s->st);
    s->pending.emplace_back(cls, pair);
  }
}

}  // namespace

// launch `call` (n_kernels kernels of class cls) on the handle's stream, counted and optionally timed
#define LAUNCH(s, cls, n_kernels, call)     \
  do {                                      \
    const int pair_ = stats_begin(s);       \
    CK(call);                               \
    stats_end(s, cls, n_kernels, pair_);    \
  } while (0)

DG_API const char* dg_last_error(void) { return g_err; }

DG_API dg_status dg_model_create(const dg_model_config* cfg, const dg_weights* w, dg_model** out) {
  const char* why = "";
  if (!out) return fail(DG_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  if (!shape_ok(cfg, &why)) return fail(DG_ERR_INVALID_ARG, "model config: %s", why);
  if (!w || !w->layers || !aligned16(w->emb) || !aligned16(w->head) || !aligned16(w->final_norm))
    return fail(DG_ERR_INVALID_ARG, "weights: null or unaligned emb/head/final_norm/layers");
  const bool fp8 = cfg->wdtype == DG_WDTYPE_FP8_BLOCK128;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const dg_layer_weights& L = w->layers[l];
    if (!aligned16(L.attn_norm) || !aligned16(L.w_qkv) || !aligned16(L.w_o) || !aligned16(L.ffn_norm) ||
        !aligned16(L.w_router) || !aligned16(L.w_gate_up) || !aligned16(L.w_down))
      return fail(DG_ERR_INVALID_ARG, "layer %d: null or unaligned weight pointer", l);
    if (fp8 && (!L.s_qkv || !L.s_o || !L.s_router || !L.s_gate_up || !L.s_down ||
                ((reinterpret_cast<uintptr_t>(L.s_qkv) | reinterpret_cast<uintptr_t>(L.s_o) |
                  reinterpret_cast<uintptr_t>(L.s_router) | reinterpret_cast<uintptr_t>(L.s_gate_up) |
                  reinterpret_cast<uintptr_t>(L.s_down)) & 3)))
      return fail(DG_ERR_INVALID_ARG, "layer %d: null or unaligned FP8 scale pointer", l);
  }
  dg_model* m = new (std::nothrow) dg_model();
  if (!m) return fail(DG_ERR_INVALID_ARG, "host allocation failed");
  m->cfg = *cfg;
  m->fp8 = fp8;
  {
    int dev = 0;
    m->n_sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&m->n_sms, cudaDevAttrMultiProcessorCount, dev);
  }
  m->emb = static_cast<const __nv_bfloat16*>(w->emb);
  m->head = static_cast<const __nv_bfloat16*>(w->head);
  m->final_norm = static_cast<const float*>(w->final_norm);
  m->layers.assign(w->layers, w->layers + cfg->n_layers);
  m->maps.resize(cfg->n_layers);
  const dg_model_config& c = *cfg;
  const uint64_t d = c.d_model, qkv = (uint64_t)(c.n_q + 2 * c.n_kv) * c.d_head;
  dg_status st = DG_OK;
  for (int l = 0; l < c.n_layers && st == DG_OK && fp8; ++l) {
    // FP8: the expert GEMMs read e4m3 bytes directly (64-row boxes for gate|up halves, 128 for down)
    const dg_layer_weights& L = m->layers[l];
    LayerMaps& M = m->maps[l];
    if ((st = map_2d_u8(&M.wgu, L.w_gate_up, (uint64_t)c.n_exp * 2 * c.d_ff, d, 64)) != DG_OK) break;
    if ((st = map_2d_u8(&M.wdown, L.w_down, (uint64_t)c.n_exp * d, c.d_ff, 128)) != DG_OK) break;
    if ((st = map_2d_u8_sw128(&M.wgu8, L.w_gate_up, (uint64_t)c.n_exp * 2 * c.d_ff, d, 64)) != DG_OK) break;
    if ((st = map_2d_u8_sw128(&M.wdown8, L.w_down, (uint64_t)c.n_exp * d, c.d_ff, 128)) != DG_OK) break;
  }
  for (int l = 0; l < c.n_layers && st == DG_OK && !fp8; ++l) {
    const dg_layer_weights& L = m->layers[l];
    LayerMaps& M = m->maps[l];
    if ((st = map_2d(&M.wqkv, L.w_qkv, qkv, d, 128)) != DG_OK) break;
    if ((st = map_2d(&M.wo, L.w_o, d, (uint64_t)c.n_q * c.d_head, 128)) != DG_OK) break;
    if ((st = map_2d(&M.wrouter, L.w_router, c.n_exp, d, 128)) != DG_OK) break;
    if ((st = map_2d(&M.wgu, L.w_gate_up, (uint64_t)c.n_exp * 2 * c.d_ff, d, 64)) != DG_OK) break;
    if ((st = map_2d(&M.wdown, L.w_down, (uint64_t)c.n_exp * d, c.d_ff, 128)) != DG_OK) break;
  }
  if (st == DG_OK) st = map_2d(&m->head_map, w->head, c.vocab, d, 256);
  if (st == DG_OK) st = map_2d(&m->head_map128, w->head, c.vocab, d, 128);
  if (st != DG_OK) {
    delete m;
    return st;
  }
  *out = m;
  return DG_OK;
}

DG_API void dg_model_destroy(dg_model* m) { delete m; }

DG_API size_t dg_kv_bytes(const dg_model_config* cfg, int n_seq, int max_ctx) {
  const char* why;
  if (!shape_ok(cfg, &why) || n_seq <= 0 || max_ctx <= 0 || max_ctx % kCanvas) return 0;
  return 2ull * cfg->n_layers * n_seq * cfg->n_kv * (size_t)max_ctx * cfg->d_head * 2ull;
}

DG_API size_t dg_workspace_bytes(const dg_model_config* cfg, int n_seq, int max_ctx) {
  const char* why;
  if (!shape_ok(cfg, &why) || n_seq <= 0 || max_ctx <= 0 || max_ctx % kCanvas) return 0;
  return ws_layout(*cfg, n_seq, max_ctx).total;
}

DG_API dg_status dg_seqs_create(dg_model* m, int n_seq, int max_ctx, void* kv, size_t kv_bytes, void* ws,
                                size_t ws_bytes, void* stream, dg_seqs** out) {
  if (!out) return fail(DG_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  if (!m) return fail(DG_ERR_INVALID_ARG, "model is null");
  if (n_seq <= 0 || max_ctx <= 0 || max_ctx % kCanvas)
    return fail(DG_ERR_INVALID_ARG, "n_seq must be > 0 and max_ctx a positive multiple of 256");
  const dg_model_config& c = m->cfg;
  const size_t need_kv = dg_kv_bytes(&c, n_seq, max_ctx);
  const size_t need_ws = dg_workspace_bytes(&c, n_seq, max_ctx);
  if (!kv || !ws) return fail(DG_ERR_INVALID_ARG, "kv and ws must be device buffers");
  if (kv_bytes < need_kv) return fail(DG_ERR_CAPACITY, "kv buffer %zu bytes < %zu needed", kv_bytes, need_kv);
  if (ws_bytes < need_ws) return fail(DG_ERR_CAPACITY, "workspace %zu bytes < %zu needed", ws_bytes, need_ws);
  if (!aligned16(kv)) return fail(DG_ERR_INVALID_ARG, "kv buffer must be 16-byte aligned");

  dg_seqs* s = new (std::nothrow) dg_seqs();
  if (!s) return fail(DG_ERR_INVALID_ARG, "host allocation failed");
  s->m = m;
  s->n_seq = n_seq;
  s->max_ctx = max_ctx;
  s->st = static_cast<cudaStream_t>(stream);
  s->L = ws_layout(c, n_seq, max_ctx);
  s->ws = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 1023) & ~uintptr_t(1023));
  const size_t half_kv = need_kv / 2;
  s->kc = static_cast<__nv_bfloat16*>(kv);
  s->vt = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(kv) + half_kv);
  uint8_t* b = s->ws;
  const WsLayout& L = s->L;
  s->err = reinterpret_cast<int*>(b + L.err);
  s->seqP = reinterpret_cast<int*>(b + L.seqP);
  s->x = reinterpret_cast<float*>(b + L.x);
  s->xn = reinterpret_cast<__nv_bfloat16*>(b + L.xn);
  s->q = reinterpret_cast<__nv_bfloat16*>(b + L.q);
  s->opart = reinterpret_cast<__nv_bfloat16*>(b + L.opart);
  s->ml = reinterpret_cast<float*>(b + L.ml);
  s->attn = reinterpret_cast<__nv_bfloat16*>(b + L.attn);
  s->rlog = reinterpret_cast<float*>(b + L.rlog);
  s->sel = reinterpret_cast<int32_t*>(b + L.sel);
  s->gate = reinterpret_cast<float*>(b + L.gate);
  s->counts = reinterpret_cast<int32_t*>(b + L.counts);
  s->offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  s->slot = reinterpret_cast<int32_t*>(b + L.slot);
  s->xp = reinterpret_cast<__nv_bfloat16*>(b + L.xp);
  s->hb = reinterpret_cast<__nv_bfloat16*>(b + L.hb);
  s->y = reinterpret_cast<float*>(b + L.y);
  s->logits = reinterpret_cast<float*>(b + L.logits);
  s->samp = reinterpret_cast<float*>(b + L.samp);
  s->hsamp = reinterpret_cast<float*>(b + L.hsamp);
  s->rope = reinterpret_cast<float2*>(b + L.rope);
  s->cids = reinterpret_cast<int32_t*>(b + L.cids);
  s->ccommit = b + L.ccommit;
  s->cH = reinterpret_cast<float*>(b + L.cH);
  s->cstop = reinterpret_cast<int32_t*>(b + L.cstop);
  s->splitk = reinterpret_cast<float*>(b + L.splitk);
  s->head_off = reinterpret_cast<int32_t*>(b + L.head_off);
  s->cursor = reinterpret_cast<int32_t*>(b + L.cursor);
  s->topk_done = reinterpret_cast<int32_t*>(b + L.topk_done);
  s->xq = L.f8mma ? b + L.xq : nullptr;
  s->hq = L.f8mma ? b + L.hq : nullptr;
  s->xs = L.f8mma ? reinterpret_cast<float*>(b + L.xs) : nullptr;
  s->hs = L.f8mma ? reinterpret_cast<float*>(b + L.hs) : nullptr;
  s->fp8_native = true;
  if (const char* v = getenv("DG_FP8_NATIVE")) s->fp8_native = atoi(v) != 0;
  s->fp8_pair = false;
  if (const char* v = getenv("DG_FP8_PAIR")) s->fp8_pair = atoi(v) != 0;
  s->xdone = reinterpret_cast<int32_t*>(b + L.xdone);
  s->rpart = L.route_rows ? reinterpret_cast<float*>(b + L.rpart) : nullptr;
  s->ssq = L.route_rows ? reinterpret_cast<float*>(b + L.ssq) : nullptr;
  s->rr = L.route_rows ? reinterpret_cast<float*>(b + L.rr) : nullptr;
  s->route_fused = true;
  if (const char* v = getenv("DG_ROUTE_FUSED")) s->route_fused = atoi(v) != 0;
  s->expert_merged = true;
  if (const char* v = getenv("DG_EXPERT_MERGED")) s->expert_merged = atoi(v) != 0;
  s->head_fused_batch = true;
  if (const char* v = getenv("DG_HEAD_FUSED_BATCH")) s->head_fused_batch = atoi(v) != 0;
  s->dstep = reinterpret_cast<int*>(b + L.dstep);
  s->bsteps = reinterpret_cast<int*>(b + L.bsteps);
  s->attn_plan_P = -1;
  s->cap_stream = nullptr;
  s->loop_exec = nullptr;
  memset(&s->loop_prm, 0, sizeof s->loop_prm);
  s->decode_graph = 1;
  if (const char* v = getenv("DG_DECODE_GRAPH")) s->decode_graph = atoi(v) != 0;
  for (int i = 0; i < 5; ++i) s->wq[i] = m->fp8 && i < 3 ? reinterpret_cast<__nv_bfloat16*>(b + L.wq[i]) : nullptr;

  s->P.assign(n_seq, 0);
  s->step = 0;
  s->block_open = false;
  for (int k = 0; k < DG_K_COUNT; ++k) {
    s->launches[k] = 0;
    s->ms[k] = 0.0;
  }
  s->timing = false;
  s->next_pair = 0;
  s->max_splits = kMaxSplits;
  if (const char* v = getenv("DG_ATTN_MAX_SPLITS")) s->max_splits = std::max(1, atoi(v));
  s->attn_cluster_merge = false;
  if (const char* v = getenv("DG_ATTN_CLUSTER_MERGE")) s->attn_cluster_merge = atoi(v) != 0;
  s->pre_bytes = 1 << 20;   // capped at the row length: the whole first tile
  s->head_nv = kHeadSamplerPair;   // CTA pairs: the fastest form measured on B200 (0.44 vs 0.47 ms at V 262144)
  if (const char* v = getenv("DG_HEAD_SAMPLER")) {
    const int nv = atoi(v);
    s->head_nv = (nv == 0 || nv == 128 || nv == 256 || nv == kHeadSamplerPair) ? nv : kHeadSamplerPair;
  }
  if (c.vocab % 256 || (s->head_nv && head_sampler_ctas(c.vocab, s->head_nv, m->n_sms) > kHeadSamplerMaxCtas))
    s->head_nv = 0;
  if (const char* v = getenv("DG_EXPERT_PREFETCH")) s->pre_bytes = std::max(0, atoi(v));
  s->prefetch_early = false;
  if (const char* v = getenv("DG_PREFETCH_EARLY")) s->prefetch_early = atoi(v) != 0;
  s->topk_gather = false;
  if (const char* v = getenv("DG_TOPK_GATHER")) s->topk_gather = atoi(v) != 0;

  const uint64_t d = c.d_model, R = L.R, A = L.A;
  const uint64_t zdim = (uint64_t)c.n_layers * n_seq * c.n_kv;
  dg_status st = DG_OK;
  if (st == DG_OK) st = map_2d(&s->xn_map, s->xn, R, d, 128);
  if (st == DG_OK) st = map_2d(&s->attn_map, s->attn, R, (uint64_t)c.n_q * c.d_head, 128);
  if (st == DG_OK) st = map_2d(&s->xp_map, s->xp, A, d, 32);
  if (st == DG_OK) st = map_2d(&s->hb_map, s->hb, A, c.d_ff, 32);
  if (st == DG_OK) st = map_2d(&s->xn32_map, s->xn, R, d, 32);
  if (st == DG_OK) st = map_2d(&s->q_map, s->q, (uint64_t)n_seq * c.n_q * kCanvas, c.d_head, 128);
  if (st == DG_OK) st = map_3d(&s->k_map, s->kc, c.d_head, max_ctx, zdim, 128);
  if (st == DG_OK) st = map_3d(&s->v_map, s->vt, max_ctx, c.d_head, zdim, c.d_head);
  if (st == DG_OK && L.f8mma) {
    st = map_2d_u8_sw128(&s->xq_map, s->xq, A, d, 32);
    if (st == DG_OK) st = map_2d_u8_sw128(&s->hq_map, s->hq, A, c.d_ff, 32);
  }
  if (st == DG_OK && m->fp8) {
    uint64_t rows[5], cols[5];
    layer_matrix_shapes(c, rows, cols);
    LayerMaps& W = s->wmaps;
    st = map_2d(&W.wqkv, s->wq[0], rows[0], cols[0], 128);
    if (st == DG_OK) st = map_2d(&W.wo, s->wq[1], rows[1], cols[1], 128);
    if (st == DG_OK) st = map_2d(&W.wrouter, s->wq[2], rows[2], cols[2], 128);
  }
  if (st != DG_OK) {
    delete s;
    return st;
  }
  // clear the cache and the buffers whose stale contents a masked lane may read, build the table
  cudaError_t e = cudaMemsetAsync(kv, 0, need_kv, s->st);
  if (e == cudaSuccess) e = cudaMemsetAsync(s->ws, 0, L.rope, s->st);
  if (e == cudaSuccess) e = cudaMemsetAsync(s->topk_done, 0, 64, s->st);   // launch counter starts at 0

  if (e == cudaSuccess) e = rope_table(s->rope, max_ctx, c.d_head, c.rope_theta, s->st);
  if (e == cudaSuccess) {
    const int32_t h_off[2] = {0, (int32_t)L.R};
    e = cudaMemcpyAsync(s->head_off, h_off, sizeof h_off, cudaMemcpyHostToDevice, s->st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s->st);   // h_off is on this stack frame
  }
  if (e != cudaSuccess) {
    delete s;
    return fail(DG_ERR_CUDA, "seqs init: %s", cudaGetErrorString(e));
  }
  *out = s;
  return DG_OK;
}

DG_API void dg_seqs_destroy(dg_seqs* s) { delete s; }

DG_API dg_status dg_seqs_get_state(const dg_seqs* s, int* h_P, int* h_step) {
  if (!s) return fail(DG_ERR_INVALID_ARG, "seqs is null");
  if (h_P)
    for (int i = 0; i < s->n_seq; ++i) h_P[i] = s->P[i];
  if (h_step) *h_step = s->step;
  return DG_OK;
}

DG_API float dg_temperature(const dg_sampler_params* p, int step) {
  if (!p) return 0.f;
  return schedule_temperature(p->t_start, p->t_end, p->max_steps, step);
}

// ---------------------------------------------------------------------------------------------
// layer stack
// ---------------------------------------------------------------------------------------------
namespace {

size_t layer_kv_elems(const dg_seqs* s) {
  return (size_t)s->n_seq * s->m->cfg.n_kv * s->max_ctx * s->m->cfg.d_head;
}

// One decoder layer on `rows` rows of x.  n_local sequences starting at cache sequence seq_base,
// Tq rows per sequence (rows == n_local * 256 for a canvas, rows == Tq for a prefill chunk).
// xn_ready: xn already holds RMSNorm_attn(x) of this layer (written by the previous combine or the
// embedding); next_gain != nullptr: the combine also writes RMSNorm(x) with that gain into xn.
dg_status run_layer(dg_seqs* s, int l, float* x, int rows, int n_local, int seq_base, int Tq, bool causal,
                    float* x_mid, float* rlog_out, bool xn_ready = false, const float* next_gain = nullptr) {
  const dg_model_config& c = s->m->cfg;
  const dg_layer_weights& W = s->m->layers[l];
  const bool fp8 = s->m->fp8;
  const LayerMaps& M = fp8 ? s->wmaps : s->m->maps[l];
  cudaStream_t st = s->st;
  const int d = c.d_model, dh = c.d_head;

  if (fp8) {
    // expand this layer's FP8 matrices into the bf16 scratch the GEMM descriptors point at
    uint64_t mr[5], mc[5];
    layer_matrix_shapes(c, mr, mc);
    const void* q[5] = {W.w_qkv, W.w_o, W.w_router, W.w_gate_up, W.w_down};
    const float* sc[5] = {W.s_qkv, W.s_o, W.s_router, W.s_gate_up, W.s_down};
    DequantArgs da{};
    da.n = 3;   // qkv, o, router; the expert GEMMs expand their e4m3 tiles on the fly
    for (int i = 0; i < 3; ++i)
      da.mat[i] = DequantMat{static_cast<const uint8_t*>(q[i]), sc[i], s->wq[i], (long long)mr[i], (int)mc[i]};
    LAUNCH(s, DG_K_DEQUANT, 1, dequant_fp8(da, s->m->n_sms, st));
  }

  if (!xn_ready)
    LAUNCH(s, DG_K_RMSNORM, 1, rmsnorm_rows(x, static_cast<const float*>(W.attn_norm), rows, d, c.rms_eps, s->xn, st));
  EpiParams ep{};
  ep.q = s->q;
  ep.kc = s->kc + (size_t)l * layer_kv_elems(s);
  ep.vt = s->vt + (size_t)l * layer_kv_elems(s);
  ep.rope = s->rope;
  ep.seq_P = s->seqP;
  ep.n_q = c.n_q;
  ep.n_kv = c.n_kv;
  ep.dh = dh;
  ep.rows_per_seq = kCanvas;
  ep.max_ctx = s->max_ctx;
  ep.seq_base = seq_base;
  ep.late_weights = fp8;
  ep.part = s->splitk;
  ep.part_slots = kSplitKSlots;
  const int n_qkv = (c.n_q + 2 * c.n_kv) * dh;
  ep.k_splits = dense_splits(((rows + 127) / 128) * (n_qkv / 128), d / 64);
  LAUNCH(s, DG_K_QKV, 1, gemm_dense(128, EPI_QKV, s->xn_map, M.wqkv, rows, n_qkv, d, ep, s->err, st));

  // attention over cache [0, P) + the Tq new rows
  int Pmax = 0;
  for (int i = 0; i < n_local; ++i) Pmax = std::max(Pmax, s->P[seq_base + i]);
  if (s->attn_plan_P >= 0) Pmax = std::max(Pmax, s->attn_plan_P);   // splits beyond the keys stay empty
  const int ntiles = (Pmax + Tq + 127) / 128;
  AttnParams ap{};
  ap.n_q = c.n_q;
  ap.n_kv = c.n_kv;
  ap.dh = dh;
  ap.rows_per_seq = kCanvas;
  ap.Tq = Tq;
  ap.max_ctx = s->max_ctx;
  ap.causal = causal ? 1 : 0;
  ap.seq_base = seq_base;
  ap.cache_seq_stride = s->n_seq * c.n_kv;
  ap.layer = l;
  int sp = std::min(std::min(s->L.split_cap, s->max_splits), ntiles);
  // With DG_ATTN_CLUSTER_MERGE=1, the splits of a query-tile pair merged inside the attention launch over a
  // cluster of at most 8 CTAs, for direct calls whose launch is one wave (with several waves the merging
  // CTAs hold their SMs from the next wave, and inside the device-resident loop's graph the step got slower).
  // Off by default: at batch 1 it saved 0.08 ms per step behind a 2048-token prompt but cost 22 us per layer
  // behind 4096 positions.
  const int units = ((c.n_q / c.n_kv) * kCanvas + 255) / 256 * n_local * c.n_kv;
  const bool cmerge = s->attn_cluster_merge && s->attn_plan_P < 0 && sp > 1 && units * std::min(sp, 8) <= s->m->n_sms;
  if (cmerge) sp = std::min(sp, 8);
  ap.tiles_per_split = (ntiles + sp - 1) / sp;
  ap.n_splits = (ntiles + ap.tiles_per_split - 1) / ap.tiles_per_split;
  ap.seq_P = s->seqP;
  ap.opart = s->opart;
  ap.ml = s->ml;
  ap.merge_in_cluster = cmerge ? 1 : 0;
  LAUNCH(s, DG_K_ATTN, 1, attention_fwd(s->q_map, s->k_map, s->v_map, ap, n_local, s->attn, s->err, st));
  if (ap.n_splits > 1 && !ap.merge_in_cluster) LAUNCH(s, DG_K_ATTN_MERGE, 1, attention_merge(ap, n_local, s->attn, st));

  // Few rows: the FFN RMSNorm and the router fold into the O epilogue (the router is linear and the
  // RMSNorm scales a row by one factor: logits = (x' g) W^T / rms(x')), and the gather forms the
  // normed rows; no RMSNorm or router launch.
  const float* ffn_g = static_cast<const float*>(W.ffn_norm);
  const bool route = s->route_fused && rows <= s->L.route_rows;
  EpiParams eo{};
  eo.x = x;
  eo.ldo = d;
  eo.late_weights = fp8;
  eo.part = s->splitk;
  eo.part_slots = kSplitKSlots;
  eo.k_splits = dense_splits(((rows + 127) / 128) * (d / 128), c.n_q * dh / 64);
  if (route) {
    eo.rw = fp8 ? s->wq[2] : static_cast<const __nv_bfloat16*>(W.w_router);
    eo.rg = ffn_g;
    eo.rpart = s->rpart;
    eo.ssq = s->ssq;
    eo.n_exp = c.n_exp;
  }
  LAUNCH(s, DG_K_OPROJ, 1, gemm_dense(128, EPI_RESID, s->attn_map, M.wo, rows, d, c.n_q * dh, eo, s->err, st));
  if (x_mid) CK(cudaMemcpyAsync(x_mid, x, sizeof(float) * (size_t)rows * d, cudaMemcpyDeviceToDevice, st));

  // mixture of experts
  if (!route) {
    LAUNCH(s, DG_K_RMSNORM, 1, rmsnorm_rows(x, ffn_g, rows, d, c.rms_eps, s->xn, st));
    EpiParams er{};
    er.out = s->rlog;
    er.ldo = c.n_exp;
    er.late_weights = fp8;
    er.part = s->splitk;
    er.part_slots = kSplitKSlots;
    er.k_splits = std::min(kRouterSplits, dense_splits((rows + 127) / 128, d / 64));
    LAUNCH(s, DG_K_ROUTER, 1, gemm_dense(128, EPI_F32, s->xn_map, M.wrouter, rows, c.n_exp, d, er, s->err, st));
  }
  // one canvas: the last CTA of the top-k launch also does the bucketing (one launch fewer)
  const bool fuse_assign = rows * c.top_k <= 8192 && c.n_exp <= 256;
  FusedAssignArgs fa{s->topk_done, s->offsets, s->slot};
  const RouterNormArgs rn{s->ssq, d / 128, d, c.rms_eps, s->rr, s->rlog};
  const GatherSrc gsrc = route ? GatherSrc{nullptr, x, s->rr, ffn_g} : GatherSrc{s->xn, nullptr, nullptr, nullptr};
  // the merged bf16 expert launch's first weight tiles go into L2 from the top-k launch (two kernels early)
  const int wide = expert_chunks_wide(c, rows) ? 1 : 0;
  const bool merged = !fp8 && !wide && s->expert_merged;
  const bool early = merged && s->pre_bytes > 0 && s->prefetch_early;
  const int n_exp_ctas = std::min(s->m->n_sms, c.n_exp * (c.d_ff / 64));
  const ExpertPrefetchArgs pfa{W.w_gate_up, n_exp_ctas, c.d_ff, d, std::min(s->pre_bytes, d * 2) & ~15};
  // One canvas, merged bf16 experts, DG_TOPK_GATHER=1: the bucketing and the gather run in the top-k launch
  // itself.  Off by default: the step got 0.05 ms slower (the separate gather overlaps the expert launch's
  // prologue better than the fused launch's serial offsets phase).
  const bool topk_gather = fuse_assign && merged && !early && s->topk_gather && (rows + 1) / 2 <= s->m->n_sms;
  if (topk_gather) {
    const TopkGatherLaunch tg{gsrc, s->xp, d, s->topk_done, s->offsets, s->cursor, s->slot, s->xdone, c.n_exp, s->err};
    if (route)
      LAUNCH(s, DG_K_TOPK, 1,
             router_topk_gather(s->rpart, d / 128, (size_t)rows * c.n_exp, rows, c.n_exp, c.top_k, s->sel, s->gate,
                                s->counts, &rn, tg, s->m->n_sms, st));
    else
      LAUNCH(s, DG_K_TOPK, 1,
             router_topk_gather(s->rlog, 1, 0, rows, c.n_exp, c.top_k, s->sel, s->gate, s->counts, nullptr, tg,
                                s->m->n_sms, st));
  } else if (route) {
    LAUNCH(s, DG_K_TOPK, 1,
           router_topk(s->rpart, d / 128, (size_t)rows * c.n_exp, rows, c.n_exp, c.top_k, s->sel, s->gate, s->counts,
                       fuse_assign ? &fa : nullptr, &rn, early ? &pfa : nullptr, st));
  } else {
    LAUNCH(s, DG_K_TOPK, 1,
           router_topk(s->rlog, 1, 0, rows, c.n_exp, c.top_k, s->sel, s->gate, s->counts, fuse_assign ? &fa : nullptr,
                       nullptr, early ? &pfa : nullptr, st));
  }
  if (rlog_out)
    CK(cudaMemcpyAsync(rlog_out, s->rlog, sizeof(float) * (size_t)rows * c.n_exp, cudaMemcpyDeviceToDevice, st));
  if (!fuse_assign) {
    int n_assign_k = 1;
    LAUNCH(s, DG_K_BUCKET, n_assign_k,
           assign_rows(s->sel, s->gate, s->counts, rows, c.top_k, c.n_exp, s->offsets, s->cursor, s->slot,
                       &n_assign_k, st));
  }
  const bool wide_rows = expert_chunks_wide(c, rows);
  const bool f8pair = wide_rows && s->fp8_pair && d % 256 == 0;
  const bool f8mma = fp8 && s->L.f8mma && s->fp8_native && (!wide_rows || f8pair);
  if (f8mma) {
    // e4m3 x e4m3: the gathered rows quantized per 128 channels, the SwiGLU rows per 64 features
    LAUNCH(s, DG_K_BUCKET, 1, gather_rows_q8(gsrc, s->slot, rows, c.top_k, d, s->xq, s->xs, st));
    ExpertParams q{};
    q.offsets = s->offsets;
    q.d = d;
    q.F = c.d_ff;
    const LayerMaps& ME = s->m->maps[l];
    ExpertParams qu = q, qd = q;
    qu.w_scale = W.s_gate_up;
    qu.w_scale_cols = (d + 127) / 128;
    qu.a_scale = s->xs;
    qu.a_scale_cols = d / 128;
    qu.hq_out = s->hq;
    qu.hs_out = s->hs;
    qd.w_scale = W.s_down;
    qd.w_scale_cols = (c.d_ff + 127) / 128;
    qd.a_scale = s->hs;
    qd.a_scale_cols = c.d_ff / 64;
    qd.y_out = s->y;
    if (f8pair) {
      LAUNCH(s, DG_K_EXPERT_UP, 1, gemm_expert_f8_pair(1, ME.wgu8, s->xq_map, qu, c.n_exp, s->m->n_sms, s->err, st));
      LAUNCH(s, DG_K_EXPERT_DOWN, 1, gemm_expert_f8_pair(2, ME.wdown8, s->hq_map, qd, c.n_exp, s->m->n_sms, s->err, st));
    } else {
      LAUNCH(s, DG_K_EXPERT_UP, 1, gemm_expert_f8(1, ME.wgu8, s->xq_map, qu, c.n_exp, s->m->n_sms, s->err, st));
      LAUNCH(s, DG_K_EXPERT_DOWN, 1, gemm_expert_f8(2, ME.wdown8, s->hq_map, qd, c.n_exp, s->m->n_sms, s->err, st));
    }
    LAUNCH(s, DG_K_COMBINE, 1,
           moe_combine(s->y, s->slot, s->gate, rows, c.top_k, d, x, next_gain, c.rms_eps, s->xn, st));
    return DG_OK;
  }
  // many tokens per expert on average (several canvases): 256-token accumulator chunks (wide)
  if (!topk_gather)
    LAUNCH(s, DG_K_BUCKET, 1,
           gather_rows(gsrc, s->slot, rows, c.top_k, d, s->xp, st, merged ? s->xdone : nullptr, c.n_exp));
  ExpertParams xp{};
  xp.offsets = s->offsets;
  xp.h_out = s->hb;
  xp.y_out = s->y;
  xp.d = d;
  xp.F = c.d_ff;
  const LayerMaps& ME = s->m->maps[l];   // expert weight descriptors: bf16, or e4m3 bytes in the FP8 form
  ExpertParams xu = xp, xd = xp;
  if (!fp8 && !wide && s->pre_bytes > 0) {
    xu.w_base = W.w_gate_up;
    xu.pre_bytes = std::min(s->pre_bytes, d * 2) & ~15;
  }
  if (fp8) {
    xu.w_scale = W.s_gate_up;
    xu.w_scale_cols = (d + 127) / 128;
    xd.w_scale = W.s_down;
    xd.w_scale_cols = (c.d_ff + 127) / 128;
  }
  if (merged) {
    // gate|up, then down, in one persistent launch (counted as the gate|up class)
    ExpertParams xm = xp;
    xm.w_base = xu.w_base;
    xm.pre_bytes = xu.pre_bytes;
    LAUNCH(s, DG_K_EXPERT_UP, 1,
           gemm_expert_updown(ME.wgu, s->xp_map, ME.wdown, s->hb_map, xm, c.n_exp, s->m->n_sms, s->xdone, s->err, st));
  } else {
    LAUNCH(s, DG_K_EXPERT_UP, 1, gemm_expert(1, ME.wgu, s->xp_map, xu, c.n_exp, s->m->n_sms, wide, s->err, st));
    LAUNCH(s, DG_K_EXPERT_DOWN, 1, gemm_expert(2, ME.wdown, s->hb_map, xd, c.n_exp, s->m->n_sms, wide, s->err, st));
  }
  LAUNCH(s, DG_K_COMBINE, 1, moe_combine(s->y, s->slot, s->gate, rows, c.top_k, d, x, next_gain, c.rms_eps, s->xn, st));
  return DG_OK;
}

// Embedding + all layers on the n_seq canvases (rows n_seq*256).  hidden: nullable debug dump.
dg_status run_canvas_stack(dg_seqs* s, const int32_t* d_ids, float* hidden) {
  const dg_model_config& c = s->m->cfg;
  const int R = s->L.R;
  const size_t plane = (size_t)R * c.d_model;
  LAUNCH(s, DG_K_EMBED, 1,
         embed_rows(s->m->emb, d_ids, R, c.d_model, c.vocab, s->x, s->err,
                    static_cast<const float*>(s->m->layers[0].attn_norm), c.rms_eps, s->xn, s->st));
  if (hidden) CK(cudaMemcpyAsync(hidden, s->x, sizeof(float) * plane, cudaMemcpyDeviceToDevice, s->st));
  for (int l = 0; l < c.n_layers; ++l) {
    // the combine of layer l writes the next layer's normed operand (the head's after the last layer)
    const float* next = l + 1 < c.n_layers ? static_cast<const float*>(s->m->layers[l + 1].attn_norm) : s->m->final_norm;
    dg_status r = run_layer(s, l, s->x, R, s->n_seq, 0, kCanvas, false, nullptr, nullptr, true, next);
    if (r != DG_OK) return r;
    if (hidden)
      CK(cudaMemcpyAsync(hidden + (size_t)(l + 1) * plane, s->x, sizeof(float) * plane, cudaMemcpyDeviceToDevice,
                         s->st));
  }
  return DG_OK;
}

dg_status check_params(const dg_seqs* s, const dg_sampler_params* p) {
  (void)s;
  return check_sampler_params(p, -1, "");
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// public calls
// ---------------------------------------------------------------------------------------------
DG_API dg_status dg_load_prefix(dg_seqs* s, int seq, int P, const void* const* h_k, const void* const* h_v) {
  NvtxRange nvtx_range("dg_load_prefix");
  if (!s || !h_k || !h_v) return fail(DG_ERR_INVALID_ARG, "null argument");
  if (seq < 0 || seq >= s->n_seq) return fail(DG_ERR_INVALID_ARG, "seq %d out of range", seq);
  if (P < 0 || P + kCanvas > s->max_ctx) return fail(DG_ERR_CAPACITY, "prefix %d + canvas exceeds max_ctx", P);
  const dg_model_config& c = s->m->cfg;
  const size_t per_seq = (size_t)c.n_kv * s->max_ctx * c.d_head;
  for (int l = 0; l < c.n_layers; ++l) {
    if (!h_k[l] || !h_v[l]) return fail(DG_ERR_INVALID_ARG, "layer %d prefix pointer is null", l);
    __nv_bfloat16* kc = s->kc + (size_t)l * layer_kv_elems(s) + (size_t)seq * per_seq;
    __nv_bfloat16* vt = s->vt + (size_t)l * layer_kv_elems(s) + (size_t)seq * per_seq;
    CK(load_prefix(static_cast<const __nv_bfloat16*>(h_k[l]), static_cast<const __nv_bfloat16*>(h_v[l]), P, c.n_kv,
                   c.d_head, s->max_ctx, kc, vt, s->st));
  }
  CK(add_to_P(s->seqP, seq, 1, P - s->P[seq], s->st));
  s->P[seq] = P;
  return DG_OK;
}

DG_API dg_status dg_prefill(dg_seqs* s, const int32_t* d_ids, const int32_t* h_lens) {
  NvtxRange nvtx_range("dg_prefill");
  if (!s || !d_ids || !h_lens) return fail(DG_ERR_INVALID_ARG, "null argument");
  const dg_model_config& c = s->m->cfg;
  for (int i = 0; i < s->n_seq; ++i)
    if (h_lens[i] < 0 || s->P[i] + h_lens[i] + kCanvas > s->max_ctx)
      return fail(DG_ERR_CAPACITY, "sequence %d: prompt of %d tokens does not fit (P=%d, max_ctx=%d)", i, h_lens[i],
                  s->P[i], s->max_ctx);
  size_t off = 0;
  for (int i = 0; i < s->n_seq; ++i) {
    for (int c0 = 0; c0 < h_lens[i]; c0 += kCanvas) {
      const int n = std::min(kCanvas, h_lens[i] - c0);
      LAUNCH(s, DG_K_EMBED, 1,
             embed_rows(s->m->emb, d_ids + off + c0, n, c.d_model, c.vocab, s->x, s->err,
                        static_cast<const float*>(s->m->layers[0].attn_norm), c.rms_eps, s->xn, s->st));
      for (int l = 0; l < c.n_layers; ++l) {
        const float* next = l + 1 < c.n_layers ? static_cast<const float*>(s->m->layers[l + 1].attn_norm) : nullptr;
        dg_status r = run_layer(s, l, s->x, n, 1, i, n, true, nullptr, nullptr, true, next);
        if (r != DG_OK) return r;
      }
      LAUNCH(s, DG_K_MISC, 1, add_to_P(s->seqP, i, 1, n, s->st));
      s->P[i] += n;
    }
    off += h_lens[i];
  }
  s->block_open = false;
  return DG_OK;
}

DG_API dg_status dg_canvas_init(dg_seqs* s, const dg_sampler_params* p, int32_t* d_ids, uint8_t* d_commit) {
  NvtxRange nvtx_range("dg_canvas_init");
  if (!s || !d_ids || !d_commit) return fail(DG_ERR_INVALID_ARG, "null argument");
  dg_status r = check_params(s, p);
  if (r != DG_OK) return r;
  for (int i = 0; i < s->n_seq; ++i)
    if (s->P[i] + kCanvas > s->max_ctx) return fail(DG_ERR_CAPACITY, "sequence %d: no room for a canvas", i);
  LAUNCH(s, DG_K_MISC, 1, canvas_init_ids(s->seqP, s->n_seq, kCanvas, p->seed, s->m->cfg.vocab, d_ids, d_commit, s->st));
  s->step = 0;
  s->block_open = true;
  return DG_OK;
}

namespace {

// The launches of one canvas step (layer stack, head, sampler).  d_step == nullptr: the step index and
// temperature are host values (s->step); otherwise the kernels read the step index from *d_step (the
// body of the device-resident block loop, which advances it on the device).
dg_status issue_step(dg_seqs* s, const dg_sampler_params* p, int32_t* d_ids, uint8_t* d_commit, float* d_entropy,
                     int32_t* d_stop, float* d_hidden, float* d_logits_out, const int* d_step) {
  const dg_model_config& c = s->m->cfg;
  dg_status r = run_canvas_stack(s, d_ids, d_hidden);   // leaves RMSNorm_final(x) in xn
  if (r != DG_OK) return r;
  SamplerArgs a{};
  a.logits = s->logits;
  a.n_seq = s->n_seq;
  a.canvas = kCanvas;
  a.vocab = c.vocab;
  a.n_chunks = s->L.chunks;
  a.seq_P = s->seqP;
  a.ids_in = d_ids;
  a.commit_in = d_commit;
  a.ids_out = d_ids;
  a.commit_out = d_commit;
  a.entropy = d_entropy;
  a.stop = d_stop;
  a.partial = s->samp;
  a.inv_temp = 1.0f / dg_temperature(p, s->step);
  a.seed = p->seed;
  a.step = s->step;
  a.max_steps = p->max_steps;
  a.fixed_steps = p->fixed_steps;
  a.entropy_bound = p->entropy_bound;
  a.stop_mean_entropy = p->stop_mean_entropy;
  a.rerand_entropy = p->rerand_entropy;
  a.commit_rule = p->commit_rule;
  a.d_step = d_step;
  a.t_start = p->t_start;
  a.t_end = p->t_end;
  if (s->head_nv > 0 && (s->L.R == kCanvas || s->head_fused_batch)) {
    // the head's logits folded into the sampler's per-row reductions tile by tile in TMEM (the logits
    // reach HBM only as the optional debug copy), then the step rule; one canvas per pass (each pass
    // streams the head once: at 32 canvases 32 passes of 0.37 ms against a dense head GEMM of 11.7 ms that
    // writes 8.6 GB of logits and a sampler pass of 4.8 ms that reads them)
    const int n_ctas = head_sampler_ctas(c.vocab, s->head_nv, s->m->n_sms);
    for (int i = 0; i < s->n_seq; ++i) {
      HeadSamplerArgs hs{};
      hs.d = c.d_model;
      hs.vocab = c.vocab;
      hs.row0 = i * kCanvas;
      hs.seq_P = s->seqP + i;
      hs.commit_in = d_commit + (size_t)i * kCanvas;
      hs.inv_temp = a.inv_temp;
      hs.seed = p->seed + (uint64_t)i;       // sequence i's stream
      hs.step = s->step;
      hs.partial = s->hsamp;
      hs.logits_out = d_logits_out ? d_logits_out + (size_t)i * kCanvas * c.vocab : nullptr;
      hs.d_step = d_step;
      hs.t_start = p->t_start;
      hs.t_end = p->t_end;
      hs.max_steps = p->max_steps;
      SamplerArgs ai = a;
      ai.n_seq = 1;
      ai.seq_P = s->seqP + i;
      ai.ids_in = d_ids + (size_t)i * kCanvas;
      ai.commit_in = d_commit + (size_t)i * kCanvas;
      ai.ids_out = d_ids + (size_t)i * kCanvas;
      ai.commit_out = d_commit + (size_t)i * kCanvas;
      ai.entropy = d_entropy + (size_t)i * kCanvas;
      ai.stop = d_stop + i;
      ai.seed = p->seed + (uint64_t)i;
      ai.partial = s->hsamp;
      ai.n_chunks = n_ctas;
      LAUNCH(s, DG_K_HEAD, 3,
             head_sampler_run(s->xn_map, s->head_nv == 256 ? s->m->head_map : s->m->head_map128, s->head_nv, hs,
                              n_ctas, ai, s->err, s->st));
    }
    return DG_OK;
  }
  if (s->L.R <= kCanvas) {
    // one canvas: the head as a persistent swap-AB GEMM (vocabulary rows are the 128-row side, the
    // 256 canvas rows one 256-wide chunk), one CTA per SM, epilogues overlapping the weight stream
    ExpertParams hp{};
    hp.offsets = s->head_off;
    hp.y_out = s->logits;
    hp.d = c.vocab;        // output rows of the weight (logit columns)
    hp.F = c.d_model;      // reduction length
    LAUNCH(s, DG_K_HEAD, 1,
           gemm_expert(2, s->m->head_map128, s->xn32_map, hp, 1, s->m->n_sms, 1, s->err, s->st));
  } else {
    EpiParams eh{};
    eh.out = s->logits;
    eh.ldo = c.vocab;
    LAUNCH(s, DG_K_HEAD, 1,
           gemm_dense(256, EPI_F32, s->xn_map, s->m->head_map, s->L.R, c.vocab, c.d_model, eh, s->err, s->st));
  }
  if (d_logits_out)
    CK(cudaMemcpyAsync(d_logits_out, s->logits, sizeof(float) * (size_t)s->L.R * c.vocab, cudaMemcpyDeviceToDevice,
                       s->st));
  LAUNCH(s, DG_K_SAMPLER, 2, sampler_run(a, s->st));
  return DG_OK;
}

}  // namespace

DG_API dg_status dg_canvas_step(dg_seqs* s, const dg_sampler_params* p, int32_t* d_ids, uint8_t* d_commit,
                                float* d_entropy, int32_t* d_stop, float* d_hidden, float* d_logits_out) {
  NvtxRange nvtx_range("dg_canvas_step");
  if (!s || !d_ids || !d_commit || !d_entropy || !d_stop) return fail(DG_ERR_INVALID_ARG, "null argument");
  dg_status r = check_params(s, p);
  if (r != DG_OK) return r;
  if (!s->block_open) return fail(DG_ERR_STATE, "no open canvas: call dg_canvas_init first");
  const int budget = p->fixed_steps > 0 ? p->fixed_steps : p->max_steps;
  if (s->step >= budget) return fail(DG_ERR_STATE, "step budget of %d already used", budget);
  r = issue_step(s, p, d_ids, d_commit, d_entropy, d_stop, d_hidden, d_logits_out, nullptr);
  if (r != DG_OK) return r;
  s->step += 1;
  return DG_OK;
}

DG_API dg_status dg_block_commit(dg_seqs* s, const int32_t* d_ids) {
  NvtxRange nvtx_range("dg_block_commit");
  if (!s || !d_ids) return fail(DG_ERR_INVALID_ARG, "null argument");
  for (int i = 0; i < s->n_seq; ++i)
    if (s->P[i] + kCanvas > s->max_ctx) return fail(DG_ERR_CAPACITY, "sequence %d: cache full", i);
  dg_status r = run_canvas_stack(s, d_ids, nullptr);
  if (r != DG_OK) return r;
  LAUNCH(s, DG_K_MISC, 1, add_to_P(s->seqP, 0, s->n_seq, kCanvas, s->st));
  for (int i = 0; i < s->n_seq; ++i) s->P[i] += kCanvas;
  s->block_open = false;
  return DG_OK;
}

DG_API dg_status dg_block_commit_last_kv(dg_seqs* s) {
  NvtxRange nvtx_range("dg_block_commit_last_kv");
  if (!s) return fail(DG_ERR_INVALID_ARG, "null argument");
  if (!s->block_open || s->step == 0) return fail(DG_ERR_STATE, "no canvas step since dg_canvas_init");
  for (int i = 0; i < s->n_seq; ++i)
    if (s->P[i] + kCanvas > s->max_ctx) return fail(DG_ERR_CAPACITY, "sequence %d: cache full", i);
  LAUNCH(s, DG_K_MISC, 1, add_to_P(s->seqP, 0, s->n_seq, kCanvas, s->st));
  for (int i = 0; i < s->n_seq; ++i) s->P[i] += kCanvas;
  s->block_open = false;
  return DG_OK;
}

DG_API dg_status dg_layer_forward(dg_seqs* s, int layer, int n_rows, int causal, float* d_x, float* d_x_mid,
                                  float* d_router_logits) {
  NvtxRange nvtx_range("dg_layer_forward");
  if (!s || !d_x) return fail(DG_ERR_INVALID_ARG, "null argument");
  if (layer < 0 || layer >= s->m->cfg.n_layers) return fail(DG_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (n_rows <= 0 || n_rows > kCanvas) return fail(DG_ERR_INVALID_ARG, "n_rows must be in [1, 256]");
  const bool canvas = (n_rows == kCanvas && !causal);
  if (!canvas && s->n_seq != 1) return fail(DG_ERR_UNSUPPORTED, "partial or causal rows need n_seq == 1");
  for (int i = 0; i < s->n_seq; ++i)
    if (s->P[i] + kCanvas > s->max_ctx) return fail(DG_ERR_CAPACITY, "sequence %d: no room for a canvas", i);
  if (canvas) return run_layer(s, layer, d_x, s->L.R, s->n_seq, 0, kCanvas, false, d_x_mid, d_router_logits);
  return run_layer(s, layer, d_x, n_rows, 1, 0, n_rows, causal != 0, d_x_mid, d_router_logits);
}

namespace {

// One block's step loop as a CUDA graph: a while-node whose body is one canvas step (every kernel reads
// the step index from s->dstep) followed by the loop control, which advances the index and sets the
// node's condition from the stop flags.  The graph runs the loop without the host: no read of the
// stop flags and no launch per step.  The body is captured on a private stream (capture needs a
// stream other than the legacy default) with the attention splits planned for plan_P, the largest
// committed length the loop will see, so one graph serves every block of a decode call.
dg_status build_step_loop(dg_seqs* s, const dg_sampler_params* p, int plan_P, cudaGraphExec_t* out) {
  *out = nullptr;
  const int budget = p->fixed_steps > 0 ? p->fixed_steps : p->max_steps;
  if (!s->cap_stream) CK(cudaStreamCreateWithFlags(&s->cap_stream, cudaStreamNonBlocking));
  cudaGraph_t g = nullptr;
  CK(cudaGraphCreate(&g, 0));
  cudaGraphConditionalHandle h;
  cudaError_t e = cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault);   // the body runs once
  cudaGraphNodeParams np = {};
  cudaGraphNode_t node;
  if (e == cudaSuccess) {
    np.type = cudaGraphNodeTypeConditional;
    np.conditional.handle = h;
    np.conditional.type = cudaGraphCondTypeWhile;
    np.conditional.size = 1;
    e = cudaGraphAddNode(&node, g, nullptr, 0, &np);
  }
  if (e != cudaSuccess) {
    cudaGraphDestroy(g);
    return fail(DG_ERR_CUDA, "decode loop graph: %s", cudaGetErrorString(e));
  }
  cudaGraph_t body = np.conditional.phGraph_out[0];
  // capture the body: the launches go to the private stream, uncounted and untimed
  cudaStream_t saved_st = s->st;
  const bool saved_timing = s->timing;
  long long saved_launches[DG_K_COUNT];
  for (int k = 0; k < DG_K_COUNT; ++k) saved_launches[k] = s->launches[k];
  s->st = s->cap_stream;
  s->timing = false;
  s->attn_plan_P = plan_P;
  dg_status r = DG_OK;
  e = cudaStreamBeginCaptureToGraph(s->st, body, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal);
  if (e == cudaSuccess) {
    r = issue_step(s, p, s->cids, s->ccommit, s->cH, s->cstop, nullptr, nullptr, s->dstep);
    if (r == DG_OK) {
      const cudaError_t le = decode_loop_control(s->cstop, s->n_seq, s->dstep, budget, h, s->st);
      if (le != cudaSuccess) r = fail(DG_ERR_CUDA, "decode loop control: %s", cudaGetErrorString(le));
    }
    cudaGraph_t captured = nullptr;
    const cudaError_t ee = cudaStreamEndCapture(s->st, &captured);
    if (r == DG_OK && ee != cudaSuccess) r = fail(DG_ERR_CUDA, "decode loop capture: %s", cudaGetErrorString(ee));
  } else {
    r = fail(DG_ERR_CUDA, "decode loop capture: %s", cudaGetErrorString(e));
  }
  s->st = saved_st;
  s->timing = saved_timing;
  s->attn_plan_P = -1;
  for (int k = 0; k < DG_K_COUNT; ++k) s->launches[k] = saved_launches[k];
  if (r == DG_OK) {
    e = cudaGraphInstantiate(out, g, 0);
    if (e != cudaSuccess) r = fail(DG_ERR_CUDA, "decode loop instantiate: %s", cudaGetErrorString(e));
  }
  cudaGraphDestroy(g);
  return r;
}

// Conditional nodes need a driver of CUDA 12.4 or later.
bool graph_loop_supported() {
  static const int ok = [] {
    int v = 0;
    return cudaDriverGetVersion(&v) == cudaSuccess && v >= 12040 ? 1 : 0;
  }();
  return ok != 0;
}

}  // namespace

DG_API dg_status dg_decode(dg_seqs* s, const dg_sampler_params* p, int max_blocks, int32_t* d_out, int32_t* h_n_out,
                           int32_t* h_steps) {
  NvtxRange nvtx_range("dg_decode");
  if (!s || !d_out || !h_n_out || max_blocks <= 0) return fail(DG_ERR_INVALID_ARG, "bad argument");
  dg_status r = check_params(s, p);
  if (r != DG_OK) return r;
  const int n = s->n_seq;
  const int budget = p->fixed_steps > 0 ? p->fixed_steps : p->max_steps;
  const size_t out_stride = (size_t)max_blocks * kCanvas;
  int Pmax = 0;
  for (int i = 0; i < n; ++i) {
    if (s->P[i] + max_blocks * kCanvas > s->max_ctx)
      return fail(DG_ERR_CAPACITY, "sequence %d: %d blocks do not fit (P=%d, max_ctx=%d)", i, max_blocks, s->P[i],
                  s->max_ctx);
    Pmax = std::max(Pmax, s->P[i]);
  }
  (void)Pmax;
  // device-resident step loop: one graph per sequence set and sampler settings, kept across calls
  cudaGraphExec_t loop = nullptr;
  if (s->decode_graph && graph_loop_supported()) {
    if (s->loop_exec && memcmp(&s->loop_prm, p, sizeof *p) != 0) {
      CK(cudaStreamSynchronize(s->st));
      cudaGraphExecDestroy(s->loop_exec);
      s->loop_exec = nullptr;
    }
    if (!s->loop_exec) {
      r = build_step_loop(s, p, s->max_ctx - kCanvas, &s->loop_exec);
      if (r != DG_OK) return r;
      s->loop_prm = *p;
    }
    loop = s->loop_exec;
  }
  std::vector<int32_t> h_stop(n), h_ids((size_t)n * kCanvas);
  std::vector<int> done(n, 0);
  for (int i = 0; i < n; ++i) h_n_out[i] = 0;
  int blocks_run = 0;
  for (int b = 0; b < max_blocks; ++b) {
    r = dg_canvas_init(s, p, s->cids, s->ccommit);
    if (r != DG_OK) break;
    int steps = 0;
    if (loop) {
      cudaError_t e = cudaMemsetAsync(s->dstep, 0, sizeof(int), s->st);
      if (e == cudaSuccess) e = cudaGraphLaunch(loop, s->st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(s->bsteps + b, s->dstep, sizeof(int), cudaMemcpyDeviceToDevice, s->st);
      if (e != cudaSuccess) {
        r = fail(DG_ERR_CUDA, "decode loop launch: %s", cudaGetErrorString(e));
        break;
      }
    } else {
      for (;;) {
        r = dg_canvas_step(s, p, s->cids, s->ccommit, s->cH, s->cstop, nullptr, nullptr);
        if (r != DG_OK) break;
        ++steps;
        cudaError_t e = cudaMemcpyAsync(h_stop.data(), s->cstop, sizeof(int32_t) * n, cudaMemcpyDeviceToHost, s->st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s->st);
        if (e != cudaSuccess) {
          r = fail(DG_ERR_CUDA, "stop flags: %s", cudaGetErrorString(e));
          break;
        }
        bool all = true;
        for (int i = 0; i < n; ++i) all = all && h_stop[i] != 0;
        if (all || steps >= budget) break;
      }
      if (r != DG_OK) break;
      if (h_steps) h_steps[b] = steps;
    }
    ++blocks_run;
    if (loop) s->step = budget;   // the graph ran the block's steps (their count is on the device)
    r = p->commit_mode == 1 ? dg_block_commit_last_kv(s) : dg_block_commit(s, s->cids);
    if (r != DG_OK) break;
    cudaError_t e = cudaMemcpy2DAsync(d_out + (size_t)b * kCanvas, out_stride * sizeof(int32_t), s->cids,
                                      kCanvas * sizeof(int32_t), kCanvas * sizeof(int32_t), n, cudaMemcpyDeviceToDevice,
                                      s->st);
    if (e == cudaSuccess && p->eos_id >= 0) {
      e = cudaMemcpyAsync(h_ids.data(), s->cids, sizeof(int32_t) * h_ids.size(), cudaMemcpyDeviceToHost, s->st);
      if (e == cudaSuccess) e = cudaStreamSynchronize(s->st);
    }
    if (e != cudaSuccess) {
      r = fail(DG_ERR_CUDA, "decode output: %s", cudaGetErrorString(e));
      break;
    }
    bool all_done = true;
    for (int i = 0; i < n; ++i) {
      if (done[i]) continue;
      int take = kCanvas;
      if (p->eos_id >= 0)
        for (int j = 0; j < kCanvas; ++j)
          if (h_ids[(size_t)i * kCanvas + j] == p->eos_id) {
            take = j + 1;
            done[i] = 1;
            break;
          }
      h_n_out[i] += take;
      all_done = all_done && done[i];
    }
    if (all_done) break;
  }
  if (loop) {
    if (r == DG_OK && h_steps && blocks_run > 0) {
      const cudaError_t e = cudaMemcpyAsync(h_steps, s->bsteps, sizeof(int32_t) * blocks_run, cudaMemcpyDeviceToHost,
                                            s->st);
      if (e != cudaSuccess) r = fail(DG_ERR_CUDA, "block step counts: %s", cudaGetErrorString(e));
    }
    const cudaError_t e = cudaStreamSynchronize(s->st);
    if (r == DG_OK && e != cudaSuccess) r = fail(DG_ERR_CUDA, "decode: %s", cudaGetErrorString(e));
    return r;
  }
  if (r != DG_OK) return r;
  CK(cudaStreamSynchronize(s->st));
  return DG_OK;
}

DG_API size_t dg_sample_workspace_bytes(int n_rows, int vocab) {
  if (n_rows <= 0 || vocab <= 0) return 0;
  return (size_t)4 * 8 * n_rows * sampler_chunks(vocab) + 1024;
}

DG_API dg_status dg_sample(const float* d_logits, int n_seq, int vocab, const dg_sampler_params* p, int step,
                           const int32_t* d_seq_P, int32_t* d_ids, uint8_t* d_commit, float* d_entropy, int32_t* d_stop,
                           void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("dg_sample");
  if (!d_logits || !p || !d_ids || !d_commit || !d_entropy || !d_stop || !ws)
    return fail(DG_ERR_INVALID_ARG, "null argument");
  if (n_seq <= 0 || vocab <= 0 || vocab % 1024 || n_seq > (1 << 20))
    return fail(DG_ERR_INVALID_ARG, "bad n_seq / vocab");
  if (step < 0) return fail(DG_ERR_INVALID_ARG, "bad step");
  const dg_status ps = check_sampler_params(p, step, "dg_sample: ");
  if (ps != DG_OK) return ps;
  const int rows = n_seq * kCanvas;
  if (ws_bytes < dg_sample_workspace_bytes(rows, vocab)) return fail(DG_ERR_CAPACITY, "sampler workspace too small");
  SamplerArgs a{};
  a.logits = d_logits;
  a.n_seq = n_seq;
  a.canvas = kCanvas;
  a.vocab = vocab;
  a.n_chunks = sampler_chunks(vocab);
  a.seq_P = d_seq_P;
  a.ids_in = d_ids;
  a.commit_in = d_commit;
  a.ids_out = d_ids;
  a.commit_out = d_commit;
  a.entropy = d_entropy;
  a.stop = d_stop;
  a.partial = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  a.inv_temp = 1.0f / dg_temperature(p, step);
  a.seed = p->seed;
  a.step = step;
  a.max_steps = p->max_steps;
  a.fixed_steps = p->fixed_steps;
  a.entropy_bound = p->entropy_bound;
  a.stop_mean_entropy = p->stop_mean_entropy;
  a.rerand_entropy = p->rerand_entropy;
  a.commit_rule = p->commit_rule;
  CK(sampler_run(a, static_cast<cudaStream_t>(stream)));
  return DG_OK;
}

DG_API size_t dg_head_sample_workspace_bytes(int vocab) {
  if (vocab <= 0 || vocab % 1024) return 0;
  return (size_t)4 * 8 * kCanvas * (kHeadSamplerMaxCtas + 1) + 4 + 1024;   // partial + merged records, error word
}

DG_API dg_status dg_head_sample(const void* d_xn, const void* d_head, int d_model, int vocab, int nv,
                                const dg_sampler_params* p, int step, const int32_t* d_seq_P, int32_t* d_ids,
                                uint8_t* d_commit, float* d_entropy, int32_t* d_stop, float* d_logits_out, void* ws,
                                size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("dg_head_sample");
  if (!d_xn || !d_head || !d_ids || !d_commit || !d_entropy || !d_stop || !ws)
    return fail(DG_ERR_INVALID_ARG, "dg_head_sample: null argument");
  if (d_model <= 0 || d_model % 64 || vocab <= 0 || vocab % 1024)
    return fail(DG_ERR_INVALID_ARG, "dg_head_sample: d_model %% 64 == 0 and vocab %% 1024 == 0 needed");
  if (nv != 128 && nv != 256 && nv != kHeadSamplerPair)
    return fail(DG_ERR_INVALID_ARG, "dg_head_sample: nv must be 128, 256 or 2 (CTA pairs)");
  if (step < 0) return fail(DG_ERR_INVALID_ARG, "dg_head_sample: bad step");
  const dg_status ps = check_sampler_params(p, step, "dg_head_sample: ");
  if (ps != DG_OK) return ps;
  if (ws_bytes < dg_head_sample_workspace_bytes(vocab)) return fail(DG_ERR_CAPACITY, "dg_head_sample: workspace too small");
  int dev = 0, n_sms = 148;
  CK(cudaGetDevice(&dev));
  CK(cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev));
  CUtensorMap xn_map, head_map;
  dg_status st = map_2d(&xn_map, d_xn, kCanvas, d_model, 128);
  if (st == DG_OK) st = map_2d(&head_map, d_head, vocab, d_model, nv == kHeadSamplerPair ? 128 : nv);
  if (st != DG_OK) return st;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  float* partial = reinterpret_cast<float*>(base);
  int* err = reinterpret_cast<int*>(base + (size_t)4 * 8 * kCanvas * (kHeadSamplerMaxCtas + 1));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  CK(cudaMemsetAsync(err, 0, sizeof(int), cs));
  const int n_ctas = std::min(head_sampler_ctas(vocab, nv, n_sms), kHeadSamplerMaxCtas);
  HeadSamplerArgs hs{};
  hs.d = d_model;
  hs.vocab = vocab;
  hs.seq_P = d_seq_P;
  hs.commit_in = d_commit;
  hs.inv_temp = 1.0f / dg_temperature(p, step);
  hs.seed = p->seed;
  hs.step = step;
  hs.partial = partial;
  hs.logits_out = d_logits_out;
  SamplerArgs a{};
  a.n_seq = 1;
  a.canvas = kCanvas;
  a.vocab = vocab;
  a.n_chunks = n_ctas;
  a.seq_P = d_seq_P;
  a.ids_in = d_ids;
  a.commit_in = d_commit;
  a.ids_out = d_ids;
  a.commit_out = d_commit;
  a.entropy = d_entropy;
  a.stop = d_stop;
  a.partial = partial;
  a.inv_temp = hs.inv_temp;
  a.seed = p->seed;
  a.step = step;
  a.max_steps = p->max_steps;
  a.fixed_steps = p->fixed_steps;
  a.entropy_bound = p->entropy_bound;
  a.stop_mean_entropy = p->stop_mean_entropy;
  a.rerand_entropy = p->rerand_entropy;
  a.commit_rule = p->commit_rule;
  CK(head_sampler_run(xn_map, head_map, nv, hs, n_ctas, a, err, cs));
  return DG_OK;
}

DG_API dg_status dg_head_sample_error(void* ws, void* stream, int* h_code) {
  if (!ws || !h_code) return fail(DG_ERR_INVALID_ARG, "null argument");
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  int* err = reinterpret_cast<int*>(base + (size_t)4 * 8 * kCanvas * (kHeadSamplerMaxCtas + 1));
  CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  CK(cudaMemcpy(h_code, err, sizeof(int), cudaMemcpyDeviceToHost));
  if (*h_code) return fail(DG_ERR_DEVICE, "device-side error code %d", *h_code);
  return DG_OK;
}

DG_API dg_status dg_device_error(dg_seqs* s, int* h_code) {
  if (!s || !h_code) return fail(DG_ERR_INVALID_ARG, "null argument");
  CK(cudaStreamSynchronize(s->st));
  int code = 0;
  CK(cudaMemcpy(&code, s->err, sizeof(int), cudaMemcpyDeviceToHost));
  CK(cudaMemset(s->err, 0, sizeof(int)));
  *h_code = code;
  if (code) return fail(DG_ERR_DEVICE, "device-side error code %d", code);
  return DG_OK;
}

DG_API dg_status dg_stats_reset(dg_seqs* s, int timing) {
  if (!s) return fail(DG_ERR_INVALID_ARG, "seqs is null");
  CK(stats_fold(s));
  for (int k = 0; k < DG_K_COUNT; ++k) {
    s->launches[k] = 0;
    s->ms[k] = 0.0;
  }
  if (timing && s->events.empty()) {
    s->events.resize(2 * kEventPairs);
    for (auto& e : s->events) CK(cudaEventCreate(&e));
  }
  s->timing = timing != 0;
  s->next_pair = 0;
  return DG_OK;
}

DG_API dg_status dg_stats_read(dg_seqs* s, long long* h_launches, double* h_ms) {
  if (!s || !h_launches) return fail(DG_ERR_INVALID_ARG, "null argument");
  CK(stats_fold(s));
  for (int k = 0; k < DG_K_COUNT; ++k) {
    h_launches[k] = s->launches[k];
    if (h_ms) h_ms[k] = s->ms[k];
  }
  return DG_OK;
}
