// dg_kernels.h -- internal launch interface between the C ABI runtime (dg_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "dg.h"

namespace dg {

// Set the calling thread's dg_last_error() message; returns st.
dg_status record_error(dg_status st, const char* msg);

// Host-side checks of the sampler settings shared by every entry point (fn prefixes the message).
// step >= 0: also that the step lies inside the max_steps-step temperature schedule.
dg_status check_sampler_params(const dg_sampler_params* p, int step, const char* fn);

// Programmatic dependent launch on/off for every kernel of the library (on unless DG_PDL=0).
bool pdl_enabled();

// Launch with programmatic stream serialization (the kernel's prologue may overlap the previous
// kernel's tail; the kernel orders itself with griddepcontrol.wait) and an optional cluster of
// (1, 1, cluster_z) CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_z,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = cluster_z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

enum { EPI_QKV = 0, EPI_RESID = 1, EPI_F32 = 2 };

struct EpiParams {
  float* out;            // EPI_F32: out[row * ldo + col]
  int k_splits;          // 1, 2, 4 or 8: K split over a cluster of this many CTAs (DSMEM reduction)
  float* x;              // EPI_RESID: x[row * ldo + col] += acc
  int ldo;
  __nv_bfloat16* q;      // EPI_QKV: query buffer [seq][n_q][rows_per_seq][dh]
  __nv_bfloat16* kc;     // key cache of this layer [seq][n_kv][max_ctx][dh] (post-rotary)
  __nv_bfloat16* vt;     // value cache of this layer, transposed [seq][n_kv][dh][max_ctx]
  const float2* rope;    // (cos, sin) table [max_ctx][dh/2]
  const int* seq_P;      // committed length of each sequence (device)
  int n_q, n_kv, dh, rows_per_seq, max_ctx, seq_base;
  int late_weights;      // 1: the weights are written by a preceding kernel (FP8 scratch): load them
                         // only after the grid-dependency wait
  float* part;           // k_splits > 1: fp32 scratch of part_slots [128][BN] partial tiles
  int part_slots;
  // EPI_RESID with rw != nullptr (BN = 128, ldo % 128 == 0, n_exp % 8 == 0, n_exp <= 128): the FFN
  // RMSNorm and the router folded into the residual epilogue.  For the updated rows x' and the
  // tile's 128 columns (tile t = n0 / 128): ssq[t][row] = sum of x'^2, and rpart[t][row][e] = sum over
  // the columns c of bf16(x'[c] rg[c]) * rw[e][c] (fp32 sums).  The router logit of a row is
  // (sum over t of rpart[t][row][e]) / sqrt(sum over t of ssq[t][row] / ldo + eps), formed by the
  // top-k kernel, because RMSNorm scales a whole row by one factor and the router is linear.
  const __nv_bfloat16* rw;   // router weights [n_exp][ldo]
  const float* rg;           // FFN RMSNorm gain [ldo]
  float* rpart;              // [ldo / 128][M][n_exp]
  float* ssq;                // [ldo / 128][M]
  int n_exp;
};

// One FP8 block-scaled matrix to expand: e4m3 q [rows][cols], scales s [ceil(rows/128)][ceil(cols/128)].
struct DequantMat {
  const uint8_t* q;
  const float* s;
  __nv_bfloat16* out;
  long long rows;
  int cols;              // multiple of 16
};
struct DequantArgs {
  DequantMat mat[5];
  int n;
};

struct ExpertParams {
  const int* offsets;    // [E+1] first bucketed row of each expert (expert e owns rows [off[e], off[e+1]))
  __nv_bfloat16* h_out;  // MODE 1: SwiGLU rows [A][F]
  float* y_out;          // MODE 2: expert outputs [A][d] (the combine applies the gates)
  int d, F;
  const float* w_scale;  // FP8 weights: fp32 scale per 128 x 128 tile of the weight matrix viewed as
  int w_scale_cols;      // 2-D, w_scale_cols tiles per row; nullptr for bf16 weights
  const void* w_base;    // bf16 weights [rows][K], and the bytes of each row of the CTA's first tile to
  int pre_bytes;         // bring into L2 before the grid-dependency wait (0: none; % 16 == 0)
  // e4m3 activations (gemm_expert_f8): the token operand's scales [A][a_scale_cols] (MODE 1: per 128
  // channels of the gathered rows; MODE 2: per 64 features of the SwiGLU rows), and MODE 1's output:
  // SwiGLU rows in e4m3 [A][F] with one scale per (row, 64 features) [A][F/64]
  const float* a_scale;
  int a_scale_cols;
  uint8_t* hq_out;
  float* hs_out;
};

struct AttnParams {
  int n_q, n_kv, dh;
  int rows_per_seq;      // query-buffer rows per head (256)
  int Tq;                // query rows present per head (256 for a canvas, n for a prefill chunk)
  int max_ctx;
  int causal;            // 0: canvas (all keys visible), 1: prefill (key <= own position)
  int seq_base;          // cache sequence index of local sequence 0
  int cache_seq_stride;  // layer offset inside the 3-D cache maps, in (seq, head) units
  int layer;
  int n_splits, tiles_per_split;
  const int* seq_P;
  __nv_bfloat16* opart;  // [split][seq][n_q][rows_per_seq][dh] un-normalised partial outputs (bf16)
  float* ml;             // [split][seq][n_q][rows_per_seq][2] (running max in log2 units, sum)
  int merge_in_cluster;  // n_splits > 1: the splits of a query-tile pair form a thread-block cluster and
                         // merge their partials after a cluster barrier (no attention_merge launch)
};

cudaError_t gemm_dense(int bn, int epi, const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const EpiParams& ep, int* err, cudaStream_t st);
// persistent: n_ctas CTAs (one per SM) loop over the (expert, weight tile) items; wide selects
// 256-token (else 64-token) accumulator chunks
cudaError_t gemm_expert(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                        int n_ctas, int wide, int* err, cudaStream_t st);
// gate|up (MODE 1 items, then) down (MODE 2 items) in one persistent launch, bf16 weights, 64-token
// chunks: wu/x as gemm_expert mode 1, wd/h as mode 2; done[n_exp] zeroed before the launch (a down item
// of expert e waits until done[e] counts e's F/64 gate|up tiles); one CTA per SM, all resident
cudaError_t gemm_expert_updown(const CUtensorMap& wu, const CUtensorMap& x, const CUtensorMap& wd, const CUtensorMap& h,
                               const ExpertParams& p, int n_exp, int n_ctas, int* done, int* err, cudaStream_t st);
// e4m3 x e4m3 grouped expert GEMMs (expert_fp8.cu): chunks of 32 tokens, per-slice scale promotion;
// w: e4m3 weights with 128-byte boxes (64 rows for MODE 1, 128 for MODE 2), x: e4m3 token rows, 32-row
// boxes of 128 bytes, both 128-byte swizzled
cudaError_t gemm_expert_f8(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p, int n_exp,
                           int n_ctas, int* err, cudaStream_t st);
// e4m3 x e4m3 grouped expert GEMMs on CTA pairs for many tokens per expert (256-token chunks, 256
// weight rows per tile): w as gemm_expert_f8 (64-row boxes for MODE 1, 128-row for MODE 2), x 32-row
// boxes; n_ctas even (pairs)
cudaError_t gemm_expert_f8_pair(int mode, const CUtensorMap& w, const CUtensorMap& x, const ExpertParams& p,
                                int n_exp, int n_ctas, int* err, cudaStream_t st);
// The rows a gather copies: bf16 normed rows xn, or (xn == nullptr) formed from the residual stream,
// bf16(x[t] * r[t] * g) with r[t] = 1/rms of row t (the FFN RMSNorm folded into the gather).
struct GatherSrc {
  const __nv_bfloat16* xn;
  const float* x;
  const float* r;
  const float* g;
};
// gather the normed rows into the bucketed order as e4m3 with one scale per (row, 128 channels)
cudaError_t gather_rows_q8(const GatherSrc& src, const int32_t* slot, int n_rows, int top_k, int d, uint8_t* xq,
                           float* xs, cudaStream_t st);
cudaError_t attention_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const AttnParams& p, int n_seq, __nv_bfloat16* out, int* err, cudaStream_t st);
cudaError_t attention_merge(const AttnParams& p, int n_seq, __nv_bfloat16* out, cudaStream_t st);

// elementwise / routing kernels (misc.cu)
// g != nullptr: also the RMSNorm of each embedded row into xn (bf16), gain g
cudaError_t embed_rows(const __nv_bfloat16* emb, const int32_t* ids, int n_rows, int d, int vocab, float* x,
                       int* err, const float* g, float eps, __nv_bfloat16* xn, cudaStream_t st);
cudaError_t rmsnorm_rows(const float* x, const float* g, int n_rows, int d, float eps, __nv_bfloat16* out,
                         cudaStream_t st);
cudaError_t dequant_fp8(const DequantArgs& a, int n_sms, cudaStream_t st);
cudaError_t rope_table(float2* table, int max_ctx, int dh, float theta, cudaStream_t st);
// Bucketing done by the last CTA of the top-k launch (one canvas: n_rows * top_k <= 8192).
struct FusedAssignArgs {
  int32_t* done;         // zero-initialised launch counter (reset by that CTA)
  int32_t* offsets;
  int32_t* slot;
};
// The FFN RMSNorm folded into the router (EpiParams::rw): the top-k kernel scales the summed logit
// planes of each row by r = 1/sqrt(sum of the n_ssq partial sums of squares / d + eps), writes r and
// the scaled logits.
struct RouterNormArgs {
  const float* ssq;      // [n_ssq][n_rows]
  int n_ssq, d;
  float eps;
  float* r_out;          // [n_rows]
  float* logits_out;     // [n_rows][n_exp]
};
// The first gate|up weight tile of each of n_ctas persistent expert CTAs (CTA c starts with item c:
// expert c / (F/64), 64 gate rows and 64 up rows at tile c % (F/64)), brought into L2 by the top-k
// launch, so that the weight stream of the expert launch two kernels later starts in L2.
struct ExpertPrefetchArgs {
  const void* w_gate_up;   // bf16 [n_exp][2F][d]
  int n_ctas, F, d;
  int row_bytes;           // bytes of each weight row to prefetch (multiple of 16, <= 2 d)
};
// norm, prefetch: nullable (the logits are final; no prefetch)
cudaError_t router_topk(const float* logits, int n_parts, size_t part_stride, int n_rows, int n_exp, int top_k,
                        int32_t* sel, float* gate, int32_t* counts, const FusedAssignArgs* fused,
                        const RouterNormArgs* norm, const ExpertPrefetchArgs* prefetch, cudaStream_t st);
// One canvas: top-k, bucketing and the gather in one launch (router_topk_gather_kernel; two rows per CTA,
// all CTAs resident, so (n_rows + 1) / 2 <= n_sms).  sync: 3 zero-initialised ints (left zero on exit).
struct TopkGatherLaunch {
  GatherSrc src;
  __nv_bfloat16* xp;
  int d;
  int32_t* sync;
  int32_t* offsets;
  int32_t* cursor;
  int32_t* slot;
  int32_t* zero;
  int n_zero;
  int* err;
};
cudaError_t router_topk_gather(const float* logits, int n_parts, size_t part_stride, int n_rows, int n_exp, int top_k,
                               int32_t* sel, float* gate, int32_t* counts, const RouterNormArgs* norm,
                               const TopkGatherLaunch& g, int n_sms, cudaStream_t st);
// expert offsets and the bucketed row of every (token, rank) assignment; *n_launched = kernels used
cudaError_t assign_rows(const int32_t* sel, const float* gate, int32_t* counts, int n_rows, int top_k, int n_exp,
                        int32_t* offsets, int32_t* cursor, int32_t* slot, int* n_launched, cudaStream_t st);
// zero (nullable): n_zero ints set to 0 by the launch (the expert kernels' per-launch counters)
cudaError_t gather_rows(const GatherSrc& src, const int32_t* slot, int n_rows, int top_k, int d, __nv_bfloat16* xp,
                        cudaStream_t st, int32_t* zero = nullptr, int n_zero = 0);
// g != nullptr: also the RMSNorm of each updated row into xn (bf16), gain g
cudaError_t moe_combine(const float* y, const int32_t* slot, const float* gate, int n_rows, int top_k, int d, float* x, const float* g,
                        float eps, __nv_bfloat16* xn, cudaStream_t st);
cudaError_t sum_planes(float* out, const float* in, int n_planes, size_t stride, size_t n, cudaStream_t st);
cudaError_t add_to_P(int* seq_P, int first, int count, int delta, cudaStream_t st);
cudaError_t load_prefix(const __nv_bfloat16* k_in, const __nv_bfloat16* v_in, int P, int n_kv, int dh, int max_ctx,
                        __nv_bfloat16* kc, __nv_bfloat16* vt, cudaStream_t st);
cudaError_t canvas_init_ids(const int* seq_P, int n_seq, int canvas, uint64_t seed, int vocab, int32_t* ids,
                            uint8_t* commit, cudaStream_t st);
// body end of the device-resident block loop: *step += 1; the while-node condition = not all stopped and
// *step < budget
cudaError_t decode_loop_control(const int32_t* stop, int n_seq, int* step, int budget,
                                cudaGraphConditionalHandle handle, cudaStream_t st);

// sampler (sampler.cu)
struct SamplerArgs {
  const float* logits;   // [n_seq * canvas][vocab]
  int n_seq, canvas, vocab, n_chunks;
  const int* seq_P;      // absolute position of row 0 of each sequence (nullptr -> 0)
  const int32_t* ids_in;
  const uint8_t* commit_in;
  int32_t* ids_out;
  uint8_t* commit_out;
  float* entropy;        // [n_seq * canvas]
  int32_t* stop;         // [n_seq]
  float* partial;        // [n_seq * canvas][n_chunks][8]
  float inv_temp;
  uint64_t seed;
  int step, max_steps, fixed_steps;
  float entropy_bound, stop_mean_entropy, rerand_entropy;
  int commit_rule;       // 0 per-position entropy bound, 1 cumulative entropy bound
  const int* d_step;     // nullable: the step index lives on the device (a step loop that runs without the
  float t_start, t_end;  // host); step and inv_temp are then derived from *d_step on the schedule
};
cudaError_t sampler_run(const SamplerArgs& a, cudaStream_t st);
// the finalize kernel alone (a.partial holds a.n_chunks records per row)
cudaError_t sampler_finalize_run(const SamplerArgs& a, cudaStream_t st);
// many records per row: one warp per row merges a.partial's a.n_chunks records into merged [rows][8], then
// the finalize runs on the merged records
cudaError_t sampler_premerge_finalize_run(const SamplerArgs& a, float* merged, cudaStream_t st);
int sampler_chunks(int vocab);

// vocabulary head fused with the sampler's reductions, one canvas (head_sampler.cu)
struct HeadSamplerArgs {
  int d, vocab;
  int row0;                // first row of this canvas in the normed-row map (canvas c of a batch: 256 c)
  const int* seq_P;        // committed length of the sequence (device; nullptr -> 0)
  const uint8_t* commit_in;
  float inv_temp;
  uint64_t seed;
  int step;
  float* partial;          // [256][n_ctas][8] per-row partial records (one per CTA), then [256][8] merged ones
  float* logits_out;       // nullable: [256][vocab] fp32 copy of the logits
  const int* d_step;       // nullable: step index on the device (see SamplerArgs)
  float t_start, t_end;
  int max_steps;
};

// Temperature of step s on the linear schedule, computed as the host's dg_temperature does (double
// arithmetic, one rounding to fp32), and the sampler's 1 / T.
__host__ __device__ inline float schedule_temperature(float t_start, float t_end, int max_steps, int s) {
  const double frac = max_steps > 1 ? (double)s / (double)(max_steps - 1) : 0.0;
  return (float)((double)t_start - ((double)t_start - (double)t_end) * frac);
}
// nv value selecting the CTA-pair form (tcgen05 cta_group::2, 256 vocabulary rows per pair item)
constexpr int kHeadSamplerPair = 2;
// CTAs of the fused head for nv vocabulary rows per item (one per SM, at most one per item; the pair
// form: an even count, one pair per two SMs)
int head_sampler_ctas(int vocab, int nv, int n_sms);
// the fused head (xn_map: 128-row boxes of the normed rows; head_map: nv-row boxes of the head),
// then the sampler's finalize with fin.partial = p.partial and fin.n_chunks = n_ctas
cudaError_t head_sampler_run(const CUtensorMap& xn_map, const CUtensorMap& head_map, int nv, const HeadSamplerArgs& p,
                             int n_ctas, const SamplerArgs& fin, int* err, cudaStream_t st);

}  // namespace dg
