/*
 * dg.h -- C ABI of the B200 (sm_100a) block-diffusion canvas decoder.
 *
 * The decoder is block-autoregressive, uniform-state text diffusion over a Gemma-4-26B-A4B-shaped
 * mixture-of-experts model.  Sources, cited by page title and section:
 *   [guide]  "diffusion-gemma developer guide" (aisparkup.com wiki)
 *   [report] "DiffusionGemma: a diffusion LLM that refines 256-token blocks in parallel"
 *            (42jerrykim.github.io, summary of the technical report)
 * The report's flowchart ("Composition of DiffusionGemma") is the call sequence of this ABI:
 *   prompt -> KV cache            dg_prefill
 *   256-token canvas of noise     dg_canvas_init
 *   one bidirectional refinement  dg_canvas_step   (repeated until the adaptive-stop test passes)
 *   block -> KV cache             dg_block_commit
 *   loop until EOS                dg_decode
 *
 * Conventions
 *  - Ownership: the caller owns every device buffer (weights, KV cache, workspace, inputs,
 *    outputs), typically allocated through PyTorch.  The library allocates no device memory; its
 *    handles are small host structures.  Every pointer named d_* is device memory; h_* is host.
 *  - Asynchrony: every call is enqueued on the stream given to dg_seqs_create and returns without
 *    waiting, except dg_decode (synchronises once at the end, and once per block to find an EOS)
 *    and dg_device_error (synchronises the stream).
 *  - Errors: arguments and state are checked on the host before any launch; nothing traps on the
 *    device.  A kernel that sees a bad index or whose pipeline wait runs out records a code that
 *    dg_device_error returns (DG_ERR_DEVICE).  dg_last_error() gives a message for the last non-OK
 *    status of the calling thread.
 *  - Devices: one process drives one GPU (launched one process per GPU).  The kernels' shared-memory
 *    attributes are set once per process, on the device current at the first launch.
 *  - Determinism: outputs depend only on (weights, inputs, params, seed).
 *  - Layouts are row-major; bf16 is IEEE bfloat16, fp32 is IEEE binary32.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,  /* a null pointer, a bad size, a shape the kernels do not support */
  DG_ERR_CAPACITY = 2,     /* the KV cache or the workspace is too small */
  DG_ERR_STATE = 3,        /* call out of order (e.g. a step after the block stopped) */
  DG_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  DG_ERR_UNSUPPORTED = 5,  /* valid request this build does not implement */
  DG_ERR_DEVICE = 6        /* a kernel recorded a device-side error (wait timeout, bad index) */
} dg_status;

typedef struct dg_model dg_model; /* opaque: config + borrowed weight pointers + TMA descriptors */
typedef struct dg_seqs dg_seqs;   /* opaque: n sequences sharing one KV cache and one workspace */

/* Storage form of the per-layer matrices (w_qkv, w_o, w_router, w_gate_up, w_down). */
#define DG_WDTYPE_BF16 0          /* bf16 */
#define DG_WDTYPE_FP8_BLOCK128 1  /* OCP FP8 E4M3 bytes, one fp32 scale per 128 x 128 tile (w = q * s) */

/* Model shape.  Requirements of this build: d_head in {64, 128}; d_model % 128 == 0;
 * d_ff % 64 == 0; n_q % n_kv == 0; n_exp <= 256; top_k <= 32; vocab % 1024 == 0; with
 * DG_WDTYPE_FP8_BLOCK128 also 2 d_ff % 128 == 0 (128-row tiles never straddle two experts). */
typedef struct {
  int d_model, n_q, n_kv, d_head, n_exp, top_k, d_ff, n_layers, vocab;
  float rms_eps;    /* RMSNorm epsilon (1e-6) */
  float rope_theta; /* rotary base (10000) */
  int wdtype;       /* DG_WDTYPE_BF16 or DG_WDTYPE_FP8_BLOCK128 */
} dg_model_config;

/* One decoder layer's weights, device pointers, layouts [out_features][in_features]:
 *   attn_norm  fp32 [d]                   RMSNorm gain before attention
 *   w_qkv      [(n_q+2 n_kv) dh][d]       Q rows, then K rows, then V rows
 *   w_o        [d][n_q dh]
 *   ffn_norm   fp32 [d]                   RMSNorm gain before the MoE
 *   w_router   [n_exp][d]
 *   w_gate_up  [n_exp][2 d_ff][d]         per expert: d_ff gate rows, then d_ff up rows
 *   w_down     [n_exp][d][d_ff]
 * The five matrices are bf16 (DG_WDTYPE_BF16) or e4m3 bytes (DG_WDTYPE_FP8_BLOCK128).  In the FP8
 * form s_* are their fp32 scales, one per 128 x 128 tile of the matrix viewed as 2-D
 * ([n_exp 2 d_ff][d] for w_gate_up, [n_exp d][d_ff] for w_down), row-major over
 * [ceil(rows/128)][ceil(cols/128)] tiles; the weight is q * s exactly.  The GEMMs compute with the
 * weights rounded to bf16 (one rounding of q * s), activations in bf16, accumulation in fp32.
 * s_* are ignored in the bf16 form.  Buffers must be 16-byte aligned and stay valid while the model
 * exists. */
typedef struct {
  const void *attn_norm, *w_qkv, *w_o, *ffn_norm, *w_router, *w_gate_up, *w_down;
  const float *s_qkv, *s_o, *s_router, *s_gate_up, *s_down;
} dg_layer_weights;

typedef struct {
  const void *emb;                /* bf16 [vocab][d]  embedding table */
  const void *final_norm;         /* fp32 [d]         final RMSNorm gain */
  const void *head;               /* bf16 [vocab][d]  vocabulary projection (untied) */
  const dg_layer_weights *layers; /* host array of n_layers entries, copied by dg_model_create */
} dg_weights;

/* Sampler settings.  Defaults from the pages: canvas 256, at most 48 steps, temperature linear
 * 0.8 -> 0.4, adaptive stop at canvas-mean entropy 0.005 ([report] "Composition", sampler
 * settings); entropy bound 0.1 ([guide] "Serving with vLLM").  rerand_entropy (re-randomise a
 * non-committing position whose entropy exceeds it) has no value on the pages; 0.5 ln(vocab) is
 * this build's default. */
typedef struct {
  int canvas_len;          /* must be 256 */
  int max_steps;           /* step budget of the temperature schedule (48) */
  int fixed_steps;         /* > 0: exactly this many steps per block (<= max_steps), adaptive stop
                              off; 0: adaptive */
  float t_start, t_end;    /* 0.8, 0.4 */
  float entropy_bound;     /* 0.1 */
  float stop_mean_entropy; /* 0.005 */
  float rerand_entropy;    /* 0.5 ln(vocab) */
  uint64_t seed;           /* sequence i uses seed + i */
  int eos_id;              /* -1: no EOS */
  int commit_mode;         /* dg_decode's block commit: 0 dg_block_commit (recompute, default),
                              1 dg_block_commit_last_kv (keep the last step's K/V) */
  int commit_rule;         /* 0: an uncommitted position commits iff H <= entropy_bound (default);
                              1: cumulative: the uncommitted positions in ascending (H, position)
                              order commit while their running entropy sum stays <= entropy_bound */
} dg_sampler_params;

/* Message for the last non-OK status returned on this thread ("" if none). */
const char *dg_last_error(void);

/* Model handle.  Checks the shape, copies the config and the per-layer pointer table, builds the
 * weight TMA descriptors.  Weights are borrowed, not copied. */
dg_status dg_model_create(const dg_model_config *cfg, const dg_weights *w, dg_model **out);
void dg_model_destroy(dg_model *m);

/* Bytes the caller must provide for the KV cache (all layers, n_seq sequences of max_ctx
 * positions; max_ctx % 256 == 0) and for the workspace.  0 on invalid arguments.
 * KV cache layout (bf16): the key half first, then the value half, each
 * L * n_seq * n_kv * max_ctx * d_head elements:
 *   K[l][seq][h][pos][c]   keys after rotary embedding, head-major
 *   Vt[l][seq][h][c][pos]  values, transposed (positions contiguous) */
size_t dg_kv_bytes(const dg_model_config *cfg, int n_seq, int max_ctx);
/* With DG_WDTYPE_FP8_BLOCK128 the workspace also holds one layer's QKV, O and router matrices in
 * bf16 (expanded there just before the layer runs; the expert GEMMs read the e4m3 bytes directly). */
size_t dg_workspace_bytes(const dg_model_config *cfg, int n_seq, int max_ctx);

/* Sequence set: n_seq independent sequences (1 = batch 1) with max_ctx positions each.  kv and ws
 * are caller device buffers of at least dg_kv_bytes / dg_workspace_bytes; both belong to this
 * handle until dg_seqs_destroy.  The cache is cleared and every sequence starts empty (P = 0).
 * stream is a cudaStream_t (NULL = legacy default stream). */
dg_status dg_seqs_create(dg_model *m, int n_seq, int max_ctx, void *kv, size_t kv_bytes, void *ws,
                         size_t ws_bytes, void *stream, dg_seqs **out);
void dg_seqs_destroy(dg_seqs *s);

/* Committed length P of every sequence (h_P[n_seq]) and the canvas step index of the current block. */
dg_status dg_seqs_get_state(const dg_seqs *s, int *h_P, int *h_step);

/* Install a ready-made committed prefix for sequence `seq` (replacing its cache content): per
 * layer l, d_k[l] and d_v[l] are bf16 [P][n_kv][d_head] (K already rotated).  Sets that sequence's
 * P.  h_k / h_v are host arrays of n_layers device pointers. */
dg_status dg_load_prefix(dg_seqs *s, int seq, int P, const void *const *h_k, const void *const *h_v);

/* Prompt -> KV cache ([report] flowchart, first box; causal attention over the prompt).
 * d_ids: the prompts packed back to back (int32), h_lens[n_seq] their lengths.  Each sequence's
 * tokens are appended at its current P, in chunks of 256 positions. */
dg_status dg_prefill(dg_seqs *s, const int32_t *d_ids, const int32_t *h_lens);

/* New canvas for every sequence: uniform random placeholder ids (Philox stream tag 2 at the
 * absolute positions P..P+255), commit mask cleared, step index reset.  d_ids int32
 * [n_seq][256], d_commit uint8 [n_seq][256]. */
dg_status dg_canvas_init(dg_seqs *s, const dg_sampler_params *p, int32_t *d_ids, uint8_t *d_commit);

/* One denoising step over all canvases: the full layer stack on the n_seq*256 canvas rows
 * (bidirectional inside the canvas, full view of the committed prefix), vocabulary logits, and the
 * sampler.  In/out: d_ids, d_commit.  Out: d_entropy fp32 [n_seq][256] (0 for positions committed
 * before this step), d_stop int32 [n_seq].  d_hidden (nullable): fp32 [n_layers+1][n_seq*256][d],
 * the residual stream before the first layer and after each layer.  d_logits_out (nullable): fp32
 * [n_seq*256][vocab] copy of the logits.  The committed prefix [0, P) of the cache is not modified;
 * the block's own cache rows [P, P+256) are used as scratch.  DG_ERR_STATE after the block has
 * stopped (call dg_block_commit and dg_canvas_init first). */
dg_status dg_canvas_step(dg_seqs *s, const dg_sampler_params *p, int32_t *d_ids, uint8_t *d_commit,
                         float *d_entropy, int32_t *d_stop, float *d_hidden, float *d_logits_out);

/* Append the finished canvases to the KV cache ([guide] "Block Autoregressive Diffusion", step 2):
 * one pass of the layer stack over the final ids with the canvas mask writes every layer's K/V to
 * cache rows [P, P+256), then P += 256.  DG_ERR_CAPACITY if P + 256 > max_ctx. */
dg_status dg_block_commit(dg_seqs *s, const int32_t *d_ids);

/* Append the finished canvases keeping the K/V that the block's last dg_canvas_step computed in
 * cache rows [P, P+256): P += 256 without another pass of the layer stack.  The kept K/V are those
 * of the ids that step read (one sampling older than the final ids).  The pages only say that the
 * finished block is committed to the cache; dg_block_commit (recompute from the final ids) is this
 * library's default reading and this call the cheaper alternative.  DG_ERR_STATE if no canvas step
 * ran since dg_canvas_init; DG_ERR_CAPACITY if P + 256 > max_ctx. */
dg_status dg_block_commit_last_kv(dg_seqs *s);

/* The whole block loop ([report] flowchart): for each of up to max_blocks blocks: dg_canvas_init,
 * dg_canvas_step until every sequence's stop flag is set (sequences that stopped keep their ids),
 * dg_block_commit; a sequence ends after the block that contains eos_id (its output cut after the
 * first EOS).  d_out int32 [n_seq][max_blocks*256] receives the committed tokens, h_n_out[n_seq]
 * their counts.  h_steps (nullable) [max_blocks] receives the step count of each block.
 * The steps of a block run on the device without the host: a CUDA graph whose while-node repeats
 * one canvas step (step index and temperature kept on the device) until every stop flag is set or
 * the budget is spent (the adaptive-stop test of the flowchart).  The graph is built on the first
 * call (driver 12.4+; captured on a private stream) and kept in the handle for later calls with
 * the same sampler settings.  The host reads the ids once per block only when eos_id >= 0, and
 * synchronises once at the end. */
dg_status dg_decode(dg_seqs *s, const dg_sampler_params *p, int max_blocks, int32_t *d_out, int32_t *h_n_out,
                    int32_t *h_steps);

/* One decoder layer on caller hidden states (the attention block and the MoE block of a canvas
 * step, without embedding, head or sampler).  n_rows = 256 with causal = 0: every sequence's canvas
 * (d_x fp32 [n_seq*256][d] in/out) at positions P..P+255, bidirectional; n_rows < 256 or causal = 1
 * (n_seq must be 1): n_rows rows at positions P..P+n_rows-1 attending to the cache and, causally
 * or not, to each other (the mask of one prefill chunk).  The rows' K/V are written to cache rows
 * [P, P+n_rows) (scratch; P is not advanced).  d_x_mid (nullable) receives x after the attention
 * residual, d_router_logits (nullable) fp32 [rows][n_exp]. */
dg_status dg_layer_forward(dg_seqs *s, int layer, int n_rows, int causal, float *d_x, float *d_x_mid,
                           float *d_router_logits);

/* Sampler alone over caller logits (finite fp32 [n_seq*canvas_len][vocab]): the entropy / Gumbel-argmax /
 * commit / re-randomise / stop rule of step `step` (0 <= step < max_steps, the temperature
 * schedule's range; DG_ERR_INVALID_ARG otherwise).  d_seq_P (nullable, int32 [n_seq]): absolute
 * position of each sequence's first canvas row (0 if NULL).  d_ids, d_commit in/out as in
 * dg_canvas_step.  ws: device scratch of dg_sample_workspace_bytes(n_seq*canvas_len, vocab). */
size_t dg_sample_workspace_bytes(int n_rows, int vocab);
dg_status dg_sample(const float *d_logits, int n_seq, int vocab, const dg_sampler_params *p, int step,
                    const int32_t *d_seq_P, int32_t *d_ids, uint8_t *d_commit, float *d_entropy, int32_t *d_stop,
                    void *ws, size_t ws_bytes, void *stream);

/* dg_sample without a workspace argument.  The method's description has no counterpart of this entry point: it is
 * an interface of this library only.  For callers that cannot allocate device memory -- a server whose pool owns all
 * free HBM, a real-time loop that must not allocate, a C component with no CUDA allocator -- the
 * sampler's per-(row, vocabulary chunk) partial results live in a static device array of the
 * library (1 MiB, held on every GPU that loads the library until the process exits).  Limit:
 * n_seq * 256 * chunks <= 32768 records, where chunks is the sampler's split of the vocabulary:
 * the largest c <= max(1, vocab / 32768) with vocab % (4 c) == 0 (8 chunks, so 16 canvases, at
 * vocab 262144); larger requests return DG_ERR_CAPACITY.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current) and keeps it for the
 * life of the process: make that call before any stream capture, and do not call cudaDeviceReset
 * after it.  It allocates nothing (no cudaMalloc / cudaFree).  All calls on a device share
 * the array and it keeps the last call's contents (nothing in it needs to start at zero); calls
 * that may overlap on the GPU race and must not be issued.  Arguments and outputs as dg_sample. */
dg_status dg_sample_noalloc(const float *d_logits, int n_seq, int vocab, const dg_sampler_params *p, int step,
                            const int32_t *d_seq_P, int32_t *d_ids, uint8_t *d_commit, float *d_entropy,
                            int32_t *d_stop, void *stream);
/* Largest n_seq * 256 that dg_sample_noalloc accepts for this vocabulary size (0 for a vocabulary
 * the sampler rejects: vocab <= 0 or vocab % 1024 != 0). */
size_t dg_sample_noalloc_max_rows(int vocab);

/* The vocabulary head fused with the sampler, on caller inputs, for one canvas: logits
 * l = xn head^T (d_xn bf16 [256][d_model], the final-normed canvas rows; d_head bf16
 * [vocab][d_model]) computed tile by tile in tensor memory and folded into the sampler's per-row
 * reductions without being written to memory, then the step rule of `step` as in dg_sample
 * (d_seq_P nullable: the sequence's committed length, 0 if NULL; ids / commit in/out, entropy and
 * stop out).  This is the head + sampler of dg_canvas_step at one canvas ([guide] "Serving with
 * vLLM": the entropy_bound sampler runs on the head's output every step).  nv: the tiling -- 128 or
 * 256 vocabulary rows per tile on one SM, or 2: pairs of SMs (256 vocabulary rows per pair tile, the
 * pair's tensor cores multiplying all 256 canvas rows at once).  d_logits_out (nullable): fp32
 * [256][vocab] copy of the logits.  ws: device
 * scratch of dg_head_sample_workspace_bytes(vocab) bytes; a device-side error (a pipeline wait
 * that ran out) is recorded there and returned by dg_head_sample_error, which synchronises the
 * stream.  Buffers 16-byte aligned; d_model % 64 == 0, vocab % 1024 == 0. */
size_t dg_head_sample_workspace_bytes(int vocab);
dg_status dg_head_sample(const void *d_xn, const void *d_head, int d_model, int vocab, int nv,
                         const dg_sampler_params *p, int step, const int32_t *d_seq_P, int32_t *d_ids,
                         uint8_t *d_commit, float *d_entropy, int32_t *d_stop, float *d_logits_out, void *ws,
                         size_t ws_bytes, void *stream);
dg_status dg_head_sample_error(void *ws, void *stream, int *h_code);

/* Synchronise the handle's stream and return the first device-side error code recorded since the
 * last call (0 = none) in *h_code; the record is cleared.  Returns DG_ERR_DEVICE if non-zero. */
dg_status dg_device_error(dg_seqs *s, int *h_code);

/* Kernel classes counted by the statistics below (one class may launch more than one kernel). */
typedef enum {
  DG_K_EMBED = 0,     /* embedding gather */
  DG_K_RMSNORM,       /* RMSNorm -> bf16 GEMM operand */
  DG_K_QKV,           /* fused Q|K|V projection + rotary (tcgen05) */
  DG_K_ATTN,          /* canvas attention partials (tcgen05) */
  DG_K_ATTN_MERGE,    /* split-KV merge */
  DG_K_OPROJ,         /* output projection + residual (tcgen05) */
  DG_K_ROUTER,        /* router logits (tcgen05) */
  DG_K_TOPK,          /* top-k selection, gates, expert counts */
  DG_K_BUCKET,        /* expert bucketing + activation gather */
  DG_K_EXPERT_UP,     /* grouped gate|up GEMM + SwiGLU (tcgen05) */
  DG_K_EXPERT_DOWN,   /* grouped down GEMM x gate (tcgen05) */
  DG_K_COMBINE,       /* top-k combine + residual */
  DG_K_HEAD,          /* vocabulary logits (tcgen05) */
  DG_K_SAMPLER,       /* sampler partial + finalize */
  DG_K_MISC,          /* canvas init, cache bookkeeping */
  DG_K_DEQUANT,       /* FP8 block-scaled weights -> bf16 (DG_WDTYPE_FP8_BLOCK128 only) */
  DG_K_COUNT
} dg_kernel_class;

/* Reset the per-class counters of this handle.  timing != 0 also brackets every launch with CUDA
 * events on the handle's stream (adds a small overhead per launch). */
dg_status dg_stats_reset(dg_seqs *s, int timing);

/* Synchronise the stream and read, per class, the kernels launched (h_launches[DG_K_COUNT]) and,
 * when timing is on, the summed device milliseconds (h_ms[DG_K_COUNT], nullable). */
dg_status dg_stats_read(dg_seqs *s, long long *h_launches, double *h_ms);

/* Temperature of step s: fp32(t_start - (t_start - t_end) * s / (max_steps - 1)). */
float dg_temperature(const dg_sampler_params *p, int step);

#ifdef __cplusplus
}
#endif

#endif /* DG_H */
