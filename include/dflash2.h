/*
 * dflash2.h — C ABI of the DFlash 2 drafter block step on one NVIDIA B200 (sm_100a).
 *
 * The step (FastFlowLM model card for Qwen3.8-27B-DFlash2, "Draft", "Weights",
 * "Taps" and "How it is used" rows; MLX sidecar card, "Contents"): the target's
 * residual features at five tapped layers are fused by an fc layer into
 * context rows; a block of 8 positions (the last emitted token and 7 mask
 * positions) runs through 5 Qwen3-style layers (RMSNorm, two-tap dynamic
 * convolution, GQA attention with a 2048-token sliding window over the paged
 * KV cache, SwiGLU MLP); the shared output head scores the 7 drafted positions,
 * the 16 best tokens per position are kept, and a rank-256 selector picks one
 * path through them; greedy acceptance then keeps the longest prefix that
 * agrees with the target's tokens, plus one target token.
 *
 * Conventions for every call:
 *  - Pointers named in the structs below are DEVICE pointers unless a comment
 *    says host.  All memory is owned by the caller; the library allocates
 *    nothing (no cudaMalloc, no host heap) and frees nothing.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous on it unless stated otherwise.
 *  - bf16 tensors are uint16_t bit patterns; row-major; no padding.
 *  - Return value: DFLASH2_OK (0) or a negative DFLASH2_ERR_* code.  Host-side
 *    validation failures launch nothing.  Conditions only the GPU can see
 *    (token id out of range, an unmapped KV page inside the window, non-finite
 *    logits, an expired bounded wait) set bits in a device error word at the
 *    start of the workspace; read it with dflash2_device_error().
 */
#ifndef DFLASH2_H
#define DFLASH2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DFLASH2_MAX_LAYERS 8

#define DFLASH2_OK 0
#define DFLASH2_ERR_ARG (-1)       /* null pointer or bad scalar argument */
#define DFLASH2_ERR_SHAPE (-2)     /* configuration outside what the kernels support */
#define DFLASH2_ERR_ALIGN (-3)     /* a device pointer is not 16-byte aligned */
#define DFLASH2_ERR_WORKSPACE (-4) /* workspace or prepared-weight buffer too small */
#define DFLASH2_ERR_CUDA (-5)      /* a CUDA launch or copy failed */
#define DFLASH2_ERR_LAYOUT (-6)    /* Q4_K weights passed without dflash2_prepare_weights */
#define DFLASH2_ERR_STATIC_LIMIT (-7) /* request larger than the built-in scratch of dflash2_draft_step_static */

/* device error bits (dflash2_device_error) */
#define DFLASH2_DEV_TOKEN 1     /* a block token id is outside [0, vocab) */
#define DFLASH2_DEV_PAGE 2      /* a KV page needed by the window or an append is unmapped (-1) */
#define DFLASH2_DEV_NONFINITE 4 /* a candidate logit is NaN or infinite */
#define DFLASH2_DEV_TIMEOUT 8   /* a bounded wait on a bulk copy expired */

/* Model dimensions.  The full drafter (FastFlowLM card, "Draft" row; aiqre.com
 * model page, vocabulary): layers 5, hidden 5120, ffn 17408, n_q 32, n_kv 8,
 * head_dim 128, window 2048, vocab 248320, n_taps 5, block 8, topk 16, rank 256.
 * Supported: head_dim 128, page_size 16, topk 16, 2 <= block <= 16,
 * n_q % n_kv == 0, (n_q / n_kv) * block <= 64, hidden, ffn, n_q*head_dim and
 * n_taps*hidden multiples of 256, vocab and rank multiples of 16, rank <= 256.
 * rope_theta: RoPE base (1e6); rms_eps: RMSNorm epsilon (1e-6).
 * wfmt: storage of fc and the layer matrices: 0 = Q4_K; 1 = bf16; 2 = MLX-style 4-bit group-64
 * (MLX sidecar card, "Contents"): per row, per group of 64 inputs, 32 bytes of 4-bit codes (low
 * nibble first) then the group's bf16 scale and bias, weight = scale*q + bias (36 bytes per 64
 * weights); 3 = Q8_0 (Mindket listing, "Good to know"): per block of 32 inputs an fp16 d then 32
 * signed 8-bit codes, weight = d*q (34 bytes per 32).  The W_dc generators are bf16 in every
 * format.  Q4_K and MLX weights are decoded inside the products; Q8_0 is decoded when the weights
 * are prepared (each weight rounded once to bf16) and then streamed as bf16. */
typedef struct dflash2_config {
  int32_t layers, hidden, ffn, n_q, n_kv, head_dim, window, vocab, n_taps, block, topk, rank,
      page_size;
  float rope_theta, rms_eps;
  int32_t wfmt;
} dflash2_config;

/* One layer.  Matrices are [out, in] row-major: bf16, or Q4_K as 144-byte
 * super-blocks of 256 consecutive inputs (d fp16, dmin fp16, eight 6-bit
 * scales and eight 6-bit mins each packed little-endian into 6 bytes, 128
 * bytes of 4-bit codes, low nibble first; weight = d*sc*q - dmin*m).  After
 * dflash2_prepare_weights the Q4_K pointers refer to the prepared layout.
 *   wq [n_q*hd, H], wk/wv [n_kv*hd, H], wo [H, n_q*hd], wg/wu [F, H], wd [H, F]
 *   ln1, ln2 [H]: attention / MLP pre-norm weights; qn, kn [hd]: per-head q/k norms
 *   dc_w [2*(H/4), H]: dynamic-convolution gate generator; dc_s0, dc_s1 [H]:
 *   static taps.  y_t = (s0 + tanh g_t[c/4]) x_t + (s1 + tanh g_t[H/4 + c/4]) x_{t-1},
 *   g_t = dc_w x_t, x = RMSNorm(h; ln1), causal along the block (x_{-1} = 0). */
typedef struct dflash2_layer_weights {
  const void *wq, *wk, *wv, *wo, *wg, *wu, *wd;
  const uint16_t *ln1, *ln2, *qn, *kn, *dc_w, *dc_s0, *dc_s1;
} dflash2_layer_weights;

/* fc [H, n_taps*H] (wfmt), fc_norm [H]; final_norm [H]; embed and lm_head
 * [vocab, H] bf16 (the target's shared embedding table and output head);
 * sel_proj [rank, H]; cb_a, cb_b [vocab, rank] (the selector's projection and
 * its two codebooks, FastFlowLM card, "Weights" row).  prepared: 0 for the
 * canonical Q4_K layout, 1 once dflash2_prepare_weights has filled the struct. */
typedef struct dflash2_weights {
  const void *fc;
  const uint16_t *fc_norm;
  dflash2_layer_weights layer[DFLASH2_MAX_LAYERS];
  const uint16_t *final_norm, *embed, *lm_head, *sel_proj, *cb_a, *cb_b;
  int32_t prepared;
} dflash2_weights;

/* Paged KV cache of the context tokens (aiqre.com model page, "Memory": 20 KiB
 * per token at 16-bit = 5 layers x 8 heads x 128 x {K,V} x 2 bytes).
 * k[l], v[l]: bf16 [num_pages][n_kv][page_size][head_dim] per layer.
 * page_table: int32 [batch][max_pages]; logical page i of a request holds its
 * tokens page_size*i .. page_size*i + page_size-1; -1 = not backed (allowed for
 * pages the window can no longer reach).  seq_len: int32 [batch], cached
 * tokens before the step; the step appends n_new rows and advances it. */
typedef struct dflash2_kv {
  uint16_t *k[DFLASH2_MAX_LAYERS];
  uint16_t *v[DFLASH2_MAX_LAYERS];
  const int32_t *page_table;
  int32_t max_pages, num_pages;
  int32_t *seq_len;
} dflash2_kv;

/* Per-step inputs (device).
 * taps: bf16 [batch][block][n_taps*hidden], row t of request b holds the target's
 *   features at layers 5, 19, 33, 47, 61 (in that order) for its t-th new token;
 *   rows t >= n_new[b] are ignored.
 * n_new: int32 [batch], 0..block new context tokens per request.
 * block_tokens: int32 [batch][block]: position 0 = last emitted token, 1..block-1 =
 *   the caller's mask id. */
typedef struct dflash2_inputs {
  const uint16_t *taps;
  const int32_t *n_new;
  const int32_t *block_tokens;
} dflash2_inputs;

/* Optional device outputs for checking and profiling; any field may be NULL.
 * hidden: fp32 [layers+1][batch*block][hidden] residual stream after the
 *   embedding and after each layer; ctx: bf16 [batch*block][hidden] fused
 *   context rows; final_h: bf16 [batch*(block-1)][hidden] final-normed rows (the
 *   LM head's operand); cand: int32 and cand_logit: fp32 [batch*(block-1)][16];
 *   z: fp32 [batch*(block-1)][rank] selector projection.
 * ev_lm_begin / ev_lm_end: cudaEvent_t (as void*) recorded on `stream` around
 *   the LM-head + top-16 kernel. */
typedef struct dflash2_debug {
  float *hidden;
  uint16_t *ctx;
  uint16_t *final_h;
  int32_t *cand;
  float *cand_logit;
  float *z;
  void *ev_lm_begin, *ev_lm_end;
} dflash2_debug;

/* Bytes of device workspace dflash2_draft_step needs for `batch` requests on
 * the current device (depends on its SM count).  0 on an invalid config. */
size_t dflash2_workspace_size(const dflash2_config *cfg, int32_t batch);

/* Bytes of the prepared weight copy: every streamed matrix (fc, the layer matrices, the
 * dynamic-convolution generators, the output head with the selector projection; the head twice:
 * in the streaming records and in the tensor cores' operand layout used for many drafted rows). */
size_t dflash2_prepared_size(const dflash2_config *cfg);

/* Repack the streamed matrices of `src` (canonical layouts, device) into `dst`
 * (device, 16-byte aligned, dst_bytes >= dflash2_prepared_size): the 8 tiles of 16 rows
 * of each column group interleaved per K unit (Q4_K: 256-wide super-blocks, codes in
 * mma fragment order; bf16: 64-wide steps), gate and up interleaved 4 + 4 tiles per
 * group, and the output head followed by the selector projection as one matrix in
 * records of 16 tiles per 64-wide step (32 KB), padded to whole records.  Values are not
 * changed: the prepared copy holds the same bits, reordered.  Fills `out` (host struct)
 * with `src`'s pointers except the streamed matrices, which point into dst (wu aliases
 * wg; lm_head and sel_proj both point at the combined head, whose tensor-core operand copy follows
 * it: records of 256 features x 64-wide K steps, 32 KB each, 128-byte swizzled); out->prepared = 1.  The embedding
 * table, norms, static taps and codebooks stay where they are.  Asynchronous on `stream`. */
int dflash2_prepare_weights(const dflash2_config *cfg, const dflash2_weights *src, void *dst,
                            size_t dst_bytes, dflash2_weights *out, void *stream);

/* One block step for `batch` requests (the section comment at the top of this
 * file).  out_path: int32 [batch][block-1] drafted token ids; out_scores: fp32
 * [batch][block-1], the selector's cumulative path score at each position.
 * Appends n_new context rows per request to every layer's cache and advances
 * kv->seq_len.  workspace: device, >= dflash2_workspace_size bytes, 256-byte
 * aligned; its first word is the device error word, cleared at the start of
 * the step.  dbg may be NULL. */
int dflash2_draft_step(const dflash2_config *cfg, const dflash2_weights *w, const dflash2_inputs *in,
                       const dflash2_kv *kv, int32_t batch, int32_t *out_path, float *out_scores,
                       void *workspace, size_t ws_bytes, const dflash2_debug *dbg, void *stream);

/* Allocation-free variant of dflash2_draft_step.  (This entry point has no
 * counterpart in the drafter's description; it exists for callers, not for the
 * method.)  Some callers cannot hand the library a workspace: code embedded in a
 * host framework whose device memory is owned by its own pool and that forbids
 * direct cudaMalloc, or a latency-critical path where an allocation (which may
 * synchronise the device) is not acceptable.  This call needs no workspace: its
 * scratch is a 16 MiB array compiled into the library (DFLASH2_STATIC_SCRATCH_BYTES),
 * which every GPU that loads the library keeps until the process exits.  It
 * allocates nothing itself.
 *  - Enough for the full drafter at batch 1 (about 8 MiB); requests whose step
 *    workspace (dflash2_workspace_size minus its host-copy staging) exceeds the
 *    array are rejected with DFLASH2_ERR_STATIC_LIMIT before any launch.
 *  - The first call on a device looks up the array's device address (with that
 *    device current); make that first call before any stream capture.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents; the step clears what must start at zero.  Calls that overlap on
 *    the GPU (different streams, or threads without ordering) race on it: order
 *    them on one stream.
 *  - dev_err: optional DEVICE pointer to one int32 that receives the step's device
 *    error bits (DFLASH2_DEV_*), copied on `stream` after the step; NULL to skip.
 * Other arguments, outputs and errors as dflash2_draft_step. */
#define DFLASH2_STATIC_SCRATCH_BYTES (16u << 20)
int dflash2_draft_step_static(const dflash2_config *cfg, const dflash2_weights *w, const dflash2_inputs *in,
                              const dflash2_kv *kv, int32_t batch, int32_t *out_path, float *out_scores,
                              int32_t *dev_err, const dflash2_debug *dbg, void *stream);

/* Greedy acceptance (FastFlowLM card, "How it is used"): draft int32
 * [batch][block-1], target int32 [batch][block] (the target's most likely token
 * for block positions 1..block).  accepted[b] = longest n <= block-1 with
 * draft[b][i] == target[b][i] for i < n; emitted[b] = draft[b][0..n-1], then
 * target[b][n], then -1 padding to `block`.  Device pointers. */
int dflash2_accept(const int32_t *draft, const int32_t *target, int32_t batch, int32_t block,
                   int32_t *accepted, int32_t *emitted, void *stream);

/* The output head sharded by vocabulary across GPUs (one process per GPU), for the latency of a
 * single request: the head is 69 % of a step's bytes and, like the NPU's separate 8-row head
 * (FastFlowLM card, "How it is used"), can run apart from the layers.  Every rank holds the
 * layers; rank r holds head rows [v0, v0 + rows) (and the selector projection).  Each rank runs
 * dflash2_draft_step_head_shard: the layers, its shard of the head, and its local top-16 per drafted
 * row (global vocabulary ids, logit descending, smaller id first) into out_cand_val /
 * out_cand_id [batch*(block-1)][16], the selector projection into out_z
 * [batch*(block-1)][rank]; it appends the context rows and advances seq_len like
 * dflash2_draft_step.  The caller exchanges the candidates (an all-gather of [G][rows][16] values
 * and ids: bytes, not megabytes) and one rank runs dflash2_select on the G gathered lists with the
 * codebooks, which produces the path and scores exactly as the unsharded step would from the same
 * candidates.  The codebooks are not sharded: only the 2 x 16 x 7 gathered rows are read per step,
 * so they cost no bandwidth.
 *  - dflash2_head_shard_size / dflash2_prepare_head_shard: bytes and preparation of a shard from
 *    its canonical bf16 rows lm_head_rows [rows][hidden] and sel_proj [rank][hidden] (rows a
 *    multiple of 16); the prepared shard is what head_shard points to.
 *  - dflash2_draft_step_head_shard: w's lm_head and sel_proj are not used, its codebooks may be
 *    NULL; workspace as dflash2_draft_step; 0 <= v0, v0 + rows <= vocab.
 *  - dflash2_select: nparts (1..256) lists cand_val/cand_id [nparts][batch*(block-1)][16], z from
 *    any shard, block_tokens [batch][block]; writes out_path / out_scores; does not touch seq_len.
 * Device pointers; asynchronous on `stream`. */
size_t dflash2_head_shard_size(const dflash2_config *cfg, int32_t rows);
int dflash2_prepare_head_shard(const dflash2_config *cfg, const uint16_t *lm_head_rows, int32_t rows,
                               const uint16_t *sel_proj, void *dst, size_t dst_bytes, void *stream);
int dflash2_draft_step_head_shard(const dflash2_config *cfg, const dflash2_weights *w, const void *head_shard,
                                  int32_t v0, int32_t rows, const dflash2_inputs *in, const dflash2_kv *kv,
                                  int32_t batch, float *out_cand_val, int32_t *out_cand_id, float *out_z,
                                  void *workspace, size_t ws_bytes, void *stream);
int dflash2_select(const dflash2_config *cfg, const dflash2_weights *w, int32_t batch, int32_t nparts,
                   const float *cand_val, const int32_t *cand_id, const float *z, const int32_t *block_tokens,
                   int32_t *out_path, float *out_scores, void *workspace, size_t ws_bytes, void *stream);

/* Acceptance for sampled decoding by exact rejection sampling (MLX sidecar card, "Contents";
 * Mindket listing, "For newcomers and experts": the target's distribution is preserved).  For
 * each request, in block order: accept drafted token d_i with probability min(1, p_i(d_i) /
 * q_i(d_i)); at the first rejection emit a token drawn from max(0, p_i - q_i) (normalised), or, when
 * all block-1 drafted tokens are accepted, one drawn from p_{block-1}.  The decisions are exact:
 * accept iff u_accept[b][i] * q_i(d_i) < p_i(d_i) with the product formed exactly; the residual
 * is taken in 32-bit fixed point, floor(max(0, p - q) * 2^32) per token (fp32 subtraction), and
 * the emitted token is the first whose running sum exceeds floor(u_sample[b] * T / 2^32), T the
 * total; an empty residual samples p itself.  fp32 values below the normal range count as 0.
 *   draft int32 [batch][block-1]; p_target fp32 [batch][block][vocab], row i = the target's
 *   probabilities for block position i+1; q_draft fp32 [batch][block-1][vocab], or NULL for the
 *   point mass on the drafted token (the selector's path is deterministic); u_accept fp32
 *   [batch][block-1] uniforms in [0,1); u_sample uint32 [batch] uniform 32-bit integers (the
 *   caller's random numbers: the call draws none).  A drafted id outside [0, vocab) is rejected
 *   (probability 0) and never used as an index.  accepted int32 [batch]; emitted int32
 *   [batch][block]: the accepted tokens, the sampled token, then -1.  Device pointers;
 *   asynchronous on `stream`. */
int dflash2_accept_sampled(const int32_t *draft, const float *p_target, const float *q_draft, const float *u_accept,
                           const uint32_t *u_sample, int32_t batch, int32_t block, int32_t vocab, int32_t *accepted,
                           int32_t *emitted, void *stream);

/* Greedy acceptance that also prepares the next round's draft inputs on the device, so
 * consecutive rounds need no host work between the acceptance and the next draft (FastFlowLM
 * card, "How it is used": the target keeps the longest agreeing prefix plus one token of its
 * own, and drafting continues from there).  accepted and emitted as dflash2_accept; then
 *   n_new_next[b] = accepted[b] + 1 (the accepted drafted tokens and the target's token are the
 *     tokens whose target features the next round fuses as context rows), and
 *   block_tokens_next[b] = {target[b][accepted[b]], mask_id, ..., mask_id} (block entries).
 * n_new_next and block_tokens_next may be the very buffers the step just read (its n_new and
 * block_tokens): the acceptance runs after the step on the same stream.  The caller supplies the
 * next round's taps rows 0..accepted[b] (the target's features of those tokens).  Device
 * pointers; mask_id >= 0; asynchronous on `stream`. */
int dflash2_accept_chain(const int32_t *draft, const int32_t *target, int32_t batch, int32_t block, int32_t mask_id,
                         int32_t *accepted, int32_t *emitted, int32_t *n_new_next, int32_t *block_tokens_next,
                         void *stream);

/* Per-step inputs that a speculative round updates in place (device): same meaning as
 * dflash2_inputs; n_new and block_tokens are overwritten with the next round's values. */
typedef struct dflash2_inputs_mut {
  const uint16_t *taps;
  int32_t *n_new;
  int32_t *block_tokens;
} dflash2_inputs_mut;

/* One speculative round on device buffers, after the target has scored the previous draft:
 * dflash2_accept_chain of prev_path (int32 [batch][block-1], the previous round's drafted path)
 * against `target` (int32 [batch][block], the target's most likely tokens for that block's
 * positions 1..block), which writes the next round's n_new and block tokens into `in`, then
 * dflash2_draft_step of the next block (taps: the target's features of the accepted tokens and
 * its own token, rows 0..accepted[b], supplied by the caller) into out_path / out_scores.  The
 * KV cache and seq_len advance as in dflash2_draft_step.  out_path may be prev_path (the step
 * writes it only after the acceptance has read it).  Asynchronous, no host synchronisation and
 * no host reads of device data: a serving loop issues the target's pass and this call per round,
 * or replays one captured CUDA graph of both (after an uncaptured step has set the kernels'
 * attributes on the device).  0 <= mask_id < vocab.  Everything the step validates is validated
 * before anything is queued. */
int dflash2_spec_round(const dflash2_config *cfg, const dflash2_weights *w, dflash2_inputs_mut *in,
                       const dflash2_kv *kv, int32_t batch, const int32_t *prev_path, const int32_t *target,
                       int32_t mask_id, int32_t *accepted, int32_t *emitted, int32_t *out_path, float *out_scores,
                       void *workspace, size_t ws_bytes, void *stream);

/* A whole speculative draft round with HOST buffers: copies taps, n_new,
 * block_tokens and target (host, same layouts as above) into the workspace,
 * runs dflash2_draft_step and dflash2_accept, copies path, scores, accepted and
 * emitted back to host memory and synchronizes `stream`.  Weights and the KV
 * cache stay on the device.  When n_new, block_tokens, target, the four
 * outputs and dev_err (if given) are all page-locked and 4-byte aligned, the
 * library's kernels read and write them in place (the device-mapped view of
 * page-locked memory) instead of issuing eight small copies; otherwise they are
 * copied.  taps is always copied (asynchronously when page-locked).  Returns
 * the first error; device error bits are returned in *dev_err (host) when
 * dev_err is not NULL. */
int dflash2_spec_step_host(const dflash2_config *cfg, const dflash2_weights *w, const dflash2_kv *kv,
                           int32_t batch, const uint16_t *taps_h, const int32_t *n_new_h,
                           const int32_t *block_tokens_h, const int32_t *target_h, int32_t *path_h,
                           float *scores_h, int32_t *accepted_h, int32_t *emitted_h,
                           int32_t *dev_err, void *workspace, size_t ws_bytes, void *stream);

/* Copy the device error word of `workspace` to *out_bits (host) and
 * synchronize `stream`. */
int dflash2_device_error(const void *workspace, int32_t *out_bits, void *stream);

/* Kernels one dflash2_draft_step call launches for `batch` requests on the
 * current device (memsets not counted): embedding, fc product, fc norm, six per
 * layer (seven when the attention chunks are merged by a kernel of their own,
 * which the plan picks for more than 32 query vectors per kv head or when
 * window + block size exceeds 3058 keys), final norm, output head, selector.
 * 0 on an invalid config or batch. */
int32_t dflash2_step_kernels(const dflash2_config *cfg, int32_t batch);

/* Static description of an error code. */
const char *dflash2_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH2_H */
