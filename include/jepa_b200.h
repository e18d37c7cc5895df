/*
 * jepa_b200.h -- C ABI of the B200 (sm_100a) JEPA ViT encoder forward.
 *
 * The operation: the forward pass of a JEPA ViT image/video encoder --
 * tubelet patch-embed with an additive positional table and an optional CLS
 * token, pre-LN transformer blocks (LayerNorm, QKV, bidirectional or
 * block-causal multi-head attention, out-projection, GELU MLP of ratio 4,
 * residuals), a final LayerNorm, then mean / CLS / full-map output or an
 * attentive-pool classifier.  Sources, by page:
 *   - "LeVJEPA ViT-L/16 (VideoMix) -- GGUF for jepa.cpp" (intro: tubelet 1,
 *     block-causal mask, CLS a read-only sink; "Run it": --pool mean|cls|none);
 *   - "V-JEPA 2 ViT-L/16 SSv2 classifier -- GGUF for jepa.cpp" (intro:
 *     tubelet 2, 256x256, attentive-pooler head with 174 classes);
 *   - "LeWorldModel Push-T -- GGUF for jepa.cpp" (intro: ViT-Ti/14, D=192);
 *   - "Quantization" (jepa.cpp docs; "The rule": tensor names and which
 *     matrices are stored as q8_0 / q4_0; "File sizes": 8.5 / 4.5 bits per
 *     weight);
 *   - "jepa.cpp -- measured benchmarks" ("Attentive-pool head": 3 self-
 *     attention blocks + one cross-attention query + MLP + linear; "What the
 *     milliseconds are": timing of the compute graph alone).
 *
 * Conventions for every call:
 *   - Every function returning int returns a jepa_b200_status (0 = OK, < 0 =
 *     error).  No exception or abort crosses the ABI; invalid arguments are
 *     rejected on the host before any work is enqueued.
 *   - Pointers documented as "device" are CUDA device memory owned by the
 *     caller and must stay valid until the work enqueued on `stream` is done.
 *     `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Compute calls are asynchronous; errors that only the device
 *     can see (a bounded wait that ran out) are reported by the next
 *     jepa_b200_sync_status / jepa_b200_op_sync_status.
 *   - Row-major layouts; "[a, b]" means b is the contiguous axis.
 */
#ifndef JEPA_B200_H
#define JEPA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JEPA_B200_API __attribute__((visibility("default")))
#else
#define JEPA_B200_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JEPA_B200_OK = 0,
  JEPA_B200_ERR_ARG = -1,            /* null pointer, bad enum, size out of range, misaligned pointer */
  JEPA_B200_ERR_MISSING_TENSOR = -2, /* a tensor the config needs is absent from the table */
  JEPA_B200_ERR_SHAPE = -3,          /* a tensor or buffer has the wrong shape / size */
  JEPA_B200_ERR_DTYPE = -4,          /* dtype not allowed for that tensor */
  JEPA_B200_ERR_CUDA = -5,           /* a CUDA runtime/driver call failed */
  JEPA_B200_ERR_TIMEOUT = -6,        /* a bounded device-side wait ran out; the kernel unwound */
  JEPA_B200_ERR_UNSUPPORTED = -7     /* valid request the library does not implement */
} jepa_b200_status;

/* Tensor dtypes use ggml's type ids (0 f32, 1 f16, 2 q4_0, 8 q8_0), the
 * numbering of the GGUF files the pages describe. */
typedef enum {
  JEPA_B200_F32 = 0,
  JEPA_B200_F16 = 1,
  JEPA_B200_Q4_0 = 2, /* 32-element blocks: fp16 scale d + 16 bytes; byte j = q[j] | q[j+16] << 4; value (q-8)*d */
  JEPA_B200_Q8_0 = 8  /* 32-element blocks: fp16 scale d + 32 x int8 q; value q*d */
} jepa_b200_dtype;

typedef enum {
  JEPA_B200_POOL_NONE = 0,     /* full token map, f32 [B, N, D] */
  JEPA_B200_POOL_MEAN = 1,     /* mean over the patch tokens (CLS excluded), f32 [B, D] */
  JEPA_B200_POOL_CLS = 2,      /* the CLS row, f32 [B, D] */
  JEPA_B200_POOL_ATTENTIVE = 3, /* attentive-pool classifier logits, f32 [B, n_classes] */
  JEPA_B200_POOL_LEWM = 4       /* the LeWM projector on the final-normed CLS row: world-model states,
                                   f32 [B, D] (a model loaded with wm_depth > 0) */
} jepa_b200_pool;

typedef enum {
  JEPA_B200_MASK_BIDIR = 0,       /* every token reads every token */
  JEPA_B200_MASK_BLOCK_CAUSAL = 1 /* bidirectional inside a time slot, causal across slots; CLS reads
                                     every token and no patch reads CLS */
} jepa_b200_mask;

/* Model shape.  N = (frames/tubelet) * (img_h/patch) * (img_w/patch) + has_cls.
 * Requirements (JEPA_B200_ERR_SHAPE otherwise): dim = 64 * heads, at most
 * 4096; dim and mlp multiples of 64, mlp at most 16384; img_h, img_w
 * multiples of patch; frames a multiple of tubelet; N at most 524288 (one
 * clip within a call's row limit); 3 * tubelet * patch^2 at most 32768. */
typedef struct {
  int dim, depth, heads, mlp;
  int patch, tubelet, img_h, img_w, frames;
  int has_cls;        /* 1: a CLS row 0 is prepended (enc.cls_token) */
  int mask;           /* jepa_b200_mask */
  int head_sa_blocks; /* attentive head: self-attention blocks before the cross-attention (0 = no head) */
  int n_classes;      /* attentive head: logits (0 = no head) */
  float ln_eps;       /* LayerNorm epsilon */
  int rope;           /* 1: 3-D rotary positions in the encoder's attention instead of an additive
                       * enc.pos_embed (the V-JEPA 2 encoders); needs has_cls = 0, at most 64
                       * slots, patch rows and patch columns.  The head dims form three groups
                       * of 20 (slot, patch row, patch column); in group a the pair
                       * (20a + 2i, 20a + 2i + 1) of q and k turns by pos_a * 10000^(-2i/20),
                       * i < 10; dims 60..63 stay as they are. */
  int quant_f16_copy; /* 1: also keep an f16 copy of every q8_0 / q4_0 matrix (dequantised once at
                       * load) and run the GEMMs of 256 rows or more on it; 0 (default): keep the
                       * blocks only, every GEMM unpacks them in its loader. */
  /* Masked predictor (pred_depth 0: none), run by jepa_b200_predict: width, blocks,
   * heads (pred_dim / pred_heads = 32 or 64) and MLP width of the V-JEPA 2 predictor
   * ("jepa.cpp -- measured benchmarks", "Masked predictor": 12 blocks, width 384,
   * head dim 32). */
  int pred_depth, pred_dim, pred_heads, pred_mlp;
  int act_bf16;       /* 1: every 16-bit activation and MMA operand (LayerNorm outputs, Q, K, V, P,
                       * the attention output, the MLP's hidden values, the weights' 16-bit form)
                       * is bf16 instead of f16; the residual stream, LayerNorm statistics,
                       * softmax and every accumulation stay f32. */
  /* LeWM world model (wm_depth 0: none), run by jepa_b200_lewm_predict / _rollout and
   * POOL_LEWM ("LeWorldModel Push-T" card, intro: the CLS row projected to a state,
   * six AdaLN-zero causal blocks conditioned on a 10-d action; benchmarks page, "LeWM
   * world model": a 3-frame window of 192-d states).  The state width is dim (at most
   * 256, heads of 64: dim = 64 * wm_heads); wm_mlp and wm_pred_hidden (the hidden width
   * of pred.proj) at most 1024, multiples of 64; wm_proj_hidden (enc.proj's hidden
   * width) a multiple of 64; wm_action_dim at most 64; wm_window (frames a predictor
   * call reads, the rows of pred.pos_embed) at most 32.  Needs has_cls; excludes
   * pred_depth > 0 (both name their tensors pred.*). */
  int wm_depth, wm_heads, wm_mlp, wm_action_dim, wm_window, wm_proj_hidden, wm_pred_hidden;
} jepa_b200_config;

/* One entry of the tensor table.  Host memory, owned by the caller; it is
 * copied to the device by jepa_b200_load_weights and may be freed afterwards.
 * shape is PyTorch order ([out, in] for matrices; patch_embed [D, 3, kt, p, p]).
 * data holds float32 / float16 values, or the raw q8_0 / q4_0 blocks with the
 * blocks running along the last (input) axis. */
typedef struct {
  const char *name;
  int dtype; /* jepa_b200_dtype */
  int ndim;
  int64_t shape[5];
  const void *data;
  size_t nbytes;
} jepa_b200_tensor;

typedef struct jepa_b200_model jepa_b200_model;

/* Validate the table against cfg and upload it to `device`.  Names follow the
 * "Quantization" page's scheme: enc.patch_embed.{weight,bias}, enc.pos_embed
 * [N, D] (not with rope), enc.cls_token [D] (has_cls), enc.blk.<i>.{ln1,attn_qkv,attn_out,ln2,
 * ffn_up,ffn_down}.{weight,bias}, enc.norm.{weight,bias}; with a head also
 * head.blk.<i>.*, head.query [D], head.ln_kv.*, head.xattn.{q,k,v,out,
 * ffn_up,ffn_down}.{weight,bias}, head.xattn.ln2.*, head.cls.{weight,bias};
 * with a predictor pred.embed.{weight [Dp, D], bias}, pred.mask_tokens
 * [1, Dp], pred.pos_embed [N, Dp], pred.blk.<i>.* (the encoder block's
 * tensors at width Dp = pred_dim), pred.norm.*, pred.proj.{weight [D, Dp],
 * bias [D]}; with a world model enc.proj.{0,2}.{weight [Hp, D] / [D, Hp], bias},
 * pred.action_embed.{0,2}.{weight [D, A] / [D, D], bias [D]}, pred.pos_embed
 * [wm_window, D], pred.blk.<i>.{adaln.weight [6D, D], adaln.bias [6D], attn_qkv,
 * attn_out, ffn_up, ffn_down}.{weight,bias} (no LayerNorm tensors: the blocks'
 * LayerNorms have no affine parameters), pred.norm.*, pred.proj.{0,2}.{weight
 * [Hq, D] / [D, Hq], bias}.  The world model's matrices are unpacked once to
 * 16-bit arenas that its kernel streams (q8_0 / q4_0 sources keep their blocks
 * as well); pred.action_embed.0.weight stays f32.
 * q8_0 / q4_0 are accepted only for the matrices that page re-types and only
 * when the input dimension is a multiple of 64.  f32 matrices are rounded to
 * f16 once here; 1-D tensors and pos_embed are kept in f32.  A q8_0 / q4_0
 * matrix is kept as its blocks, which every GEMM's loader and the head's
 * few-row kernels unpack (each q*d or (q-8)*d rounded once to f16); with
 * cfg->quant_f16_copy it is also dequantised once, on the device, to an f16
 * copy holding those same values, which the GEMMs of 256 or more rows then
 * read instead.
 * Names the model does not use (a predictor's, say) are ignored; a name given
 * twice is ERR_ARG.
 * On success *out_model owns its device memory until jepa_b200_free.
 * Errors: ERR_ARG, ERR_MISSING_TENSOR, ERR_SHAPE, ERR_DTYPE, ERR_CUDA. */
JEPA_B200_API int jepa_b200_load_weights(const jepa_b200_config *cfg, const jepa_b200_tensor *table, int n_tensors, int device,
                           jepa_b200_model **out_model);

/* Forward pass of B clips.
 * pixels: device, f32 [B, frames, 3, img_h, img_w], already normalised.
 * pool:   jepa_b200_pool; ATTENTIVE needs a model loaded with a head.
 * out:    device, f32, shape given by jepa_b200_out_shape; out_bytes its size.
 * Enqueued on `stream`; the model's workspace grows to the largest B seen
 * (that growth allocates and synchronises the device).  A model must not be
 * used by two calls that overlap in time.
 * Errors: ERR_ARG (null, B < 1, bad pool, CLS pool on a model without CLS,
 * pixels or out not 16-byte aligned), ERR_SHAPE (out_bytes too small, or
 * B * N above 524288 rows), ERR_MISSING_TENSOR (ATTENTIVE without a head),
 * ERR_CUDA. */
JEPA_B200_API int jepa_b200_encode(jepa_b200_model *m, const float *pixels, int B, int pool, float *out, size_t out_bytes,
                     void *stream);

/* The masked predictor of a model loaded with pred_depth > 0 ("jepa.cpp --
 * measured benchmarks", "Masked predictor"): each clip's context tokens are
 * projected to the predictor's width (pred.embed), the learned mask token
 * stands at every target position, both add the pred.pos_embed row of their
 * token index, the sequence [context | targets] runs through the predictor's
 * pre-LN blocks with bidirectional attention, and the target rows leave
 * through pred.norm and pred.proj.
 * tokens: device, f32 [B, N, dim] (the encoder's last_hidden_state, e.g. from
 *         jepa_b200_encode with POOL_NONE);
 * ctx_idx, tgt_idx: HOST int arrays of n_ctx / n_tgt token indices in
 *         [0, N), the same for every clip (copied to the device by the call);
 * out:    device, f32 [B, n_tgt, dim]; out_bytes its size.
 * Enqueued on `stream`; the predictor's workspace grows to the largest
 * B * (n_ctx + n_tgt) seen.  Errors: ERR_ARG (null pointers, B or counts
 * < 1, an index out of range, no predictor), ERR_SHAPE (out_bytes too small,
 * B * (n_ctx + n_tgt) above 524288 rows), ERR_CUDA. */
JEPA_B200_API int jepa_b200_predict(jepa_b200_model *m, const float *tokens, int B, const int *ctx_idx, int n_ctx,
                                    const int *tgt_idx, int n_tgt, float *out, size_t out_bytes, void *stream);

/* The LeWM predictor ("LeWorldModel Push-T" card, intro; benchmarks page,
 * "LeWM world model"), one predictor call over T <= wm_window frames of C
 * independent candidates.  For frame t: x = state + pred.pos_embed[t];
 * c = action_embed.2(SiLU(action_embed.0(action))); six AdaLN-zero blocks
 * ([shift1 scale1 gate1 shift2 scale2 gate2] = adaln(SiLU(c)); x += gate1 *
 * attn_out(attention(LN(x)(1 + scale1) + shift1)) with frame t reading frames
 * <= t; x += gate2 * ffn_down(GELU(ffn_up(LN(x)(1 + scale2) + shift2)))),
 * then pred.proj.2(GELU(pred.proj.0(pred.norm(x)))): row t is the predicted
 * state of frame t + 1.  Row t depends on frames <= t only, bit for bit.
 * states:  device, f32 [C, T, D];  actions: device, f32 [C, T, wm_action_dim];
 * out:     device, f32 [C, T, D]; out_bytes its size.
 * One kernel launch on `stream`.  Errors: ERR_ARG (null, C or T
 * < 1, no world model), ERR_SHAPE (T > wm_window, out_bytes too small),
 * ERR_CUDA. */
JEPA_B200_API int jepa_b200_lewm_predict(jepa_b200_model *m, const float *states, const float *actions, int C, int T,
                                         float *out, size_t out_bytes, void *stream);

/* Rollout of the LeWM predictor: from T0 observed states per candidate, `steps`
 * predictor calls, each over the last min(wm_window, frames so far) frames,
 * each appending the prediction of its last row as the next frame.
 * states:  device, f32 [C, T0, D];
 * actions: device, f32 [C, T0 + steps - 1, wm_action_dim] (action f of frame f);
 * out:     device, f32 [C, steps, D]: the states of frames T0 .. T0 + steps - 1.
 * The whole rollout is one kernel launch on `stream`.  Errors: ERR_ARG (null,
 * C, T0 or steps < 1, no world model), ERR_SHAPE (out_bytes too small), ERR_CUDA. */
JEPA_B200_API int jepa_b200_lewm_rollout(jepa_b200_model *m, const float *states, int T0, const float *actions, int C,
                                         int steps, float *out, size_t out_bytes, void *stream);

/* End-to-end variant with HOST buffers: copies pixels (host, f32 [B, frames,
 * 3, H, W]; pinned memory makes the copy asynchronous) to model-owned device
 * staging, runs jepa_b200_encode, copies the result back to out (host) and
 * synchronises `stream`.  Returns the device status of the whole call
 * (including ERR_TIMEOUT). */
JEPA_B200_API int jepa_b200_encode_host(jepa_b200_model *m, const float *pixels, int B, int pool, float *out, size_t out_bytes,
                          void *stream);

/* Output shape of encode: [B, D] (mean, cls), [B, N, D] (none), [B, n_classes]
 * (attentive).  Writes shape[0..2] (unused trailing entries 0) and returns the
 * number of dimensions (2 or 3), or a negative status. */
JEPA_B200_API int jepa_b200_out_shape(const jepa_b200_model *m, int B, int pool, int64_t shape[3]);

/* Debug stage dump for parity checks: runs patch-embed and the first `layer`
 * blocks (0 <= layer <= depth) of the encoder on pixels (device) and writes
 * the f32 residual stream [B, N, D] to out (device).  stage must be 0.
 * Same kernels and launch configuration as jepa_b200_encode. */
JEPA_B200_API int jepa_b200_debug_stage(jepa_b200_model *m, const float *pixels, int B, int layer, int stage, float *out,
                          size_t out_bytes, void *stream);

/* Synchronise `stream` and return the device status of the model's last
 * calls: OK, ERR_TIMEOUT (a bounded wait ran out) or ERR_CUDA.  Clears it. */
JEPA_B200_API int jepa_b200_sync_status(jepa_b200_model *m, void *stream);

/* Device milliseconds of the kernel sequence of the last encode (between two
 * events around it; excludes host work and workspace growth).  Blocks until
 * that encode finished.  Returns a negative value if there is none. */
JEPA_B200_API double jepa_b200_last_ms(jepa_b200_model *m);

/* Bytes of weights resident on the device after the load (repacked blocks
 * plus, for quantised matrices, their f16 copies). */
JEPA_B200_API size_t jepa_b200_model_n_bytes(const jepa_b200_model *m);

/* Replay the forward as a CUDA graph (default on): when two consecutive
 * encodes have the same (pixels, out, B, pool, wait bound), the second
 * captures its kernel sequence on a stream of the model's own and it and
 * later calls with those inputs launch that graph on `stream`.  Other calls,
 * and every call while this is off or profiling is on, launch the kernels
 * one by one.  Errors: ERR_ARG. */
JEPA_B200_API int jepa_b200_set_graph(jepa_b200_model *m, int enable);

/* Bound, in nanoseconds, of every device-side wait of the model's kernels
 * (default 4e9).  0 makes the first wait that does not succeed at once give
 * up: used to test the timeout path.  Returns OK or ERR_ARG. */
JEPA_B200_API int jepa_b200_set_timeout_ns(jepa_b200_model *m, unsigned long long ns);

/* Number of kernel launches the last encode enqueued. */
JEPA_B200_API int jepa_b200_last_launch_count(const jepa_b200_model *m);

/* Kernel classes of the per-kernel timing below. */
typedef enum {
  JEPA_B200_KC_PATCH_EMBED = 0, /* patch matrix + patch-embed GEMM + CLS rows */
  JEPA_B200_KC_LAYERNORM = 1,   /* LN1, LN2 and the final norm */
  JEPA_B200_KC_GEMM_QKV = 2,
  JEPA_B200_KC_ATTENTION = 3,
  JEPA_B200_KC_GEMM_OUT = 4,
  JEPA_B200_KC_GEMM_UP = 5,     /* ffn_up + GELU */
  JEPA_B200_KC_GEMM_DOWN = 6,
  JEPA_B200_KC_POOL_HEAD = 7,   /* mean pooling and the attentive head */
  JEPA_B200_KC_COUNT = 8
} jepa_b200_kernel_class;

/* Per-kernel device timing: while enabled, encode records a CUDA event pair
 * on `stream` around every launch (adds event records between kernels;
 * leave it off for throughput runs).  Returns OK or ERR_ARG. */
JEPA_B200_API int jepa_b200_set_profiling(jepa_b200_model *m, int enable);

/* Synchronise on the recorded events and return, per kernel class, the summed
 * device milliseconds (ms[c]) and the number of launches (launches[c]) since
 * the last read; n is the length of both arrays (>= JEPA_B200_KC_COUNT).
 * Clears the record.  Returns OK, ERR_ARG or ERR_CUDA. */
JEPA_B200_API int jepa_b200_profile_read(jepa_b200_model *m, double *ms, int *launches, int n);

JEPA_B200_API const char *jepa_b200_status_str(int status);

/* Release the model's device memory.  Safe on NULL. */
JEPA_B200_API void jepa_b200_free(jepa_b200_model *m);

/* ------------------------------------------------------------------------
 * Single-kernel entry points.  Same kernels the forward uses, exposed for
 * parity tests and for callers that build their own sequence.  All pointers
 * are device memory; all are asynchronous on `stream`; device-side errors
 * are reported by jepa_b200_op_sync_status.
 * ---------------------------------------------------------------------- */

/* Fused LayerNorm over rows of D floats (pre-LN block norms and the final
 * norm).  Output row r = LN(x row r * in_row_stride).  out_dtype F16 or F32.
 * Requires D % 4 == 0, D <= 4096; x, out 16-byte aligned. */
JEPA_B200_API int jepa_b200_op_layernorm(const float *x, int rows, int D, int in_row_stride, const float *gamma,
                           const float *beta, float eps, void *out, int out_dtype, void *stream);

/* Split q8_0 / q4_0 blocks [N rows, K/32 blocks] into the GEMM's layout:
 * qs = int8 [N, K] (q8_0) or nibble bytes [N, K/2] in block order (q4_0),
 * scales = fp16 [N, K/32].  Byte moves only (bit-exact).  K % 32 == 0. */
JEPA_B200_API int jepa_b200_op_repack(int dtype, const void *blocks, int N, int K, void *qs, void *scales, void *stream);

/* f16 [N, K] from repacked quants and scales (the layout jepa_b200_op_repack
 * writes): element (n, k) = q * d (q8_0) or (q - 8) * d (q4_0), d the fp16
 * scale of its 32-element block, the exact product rounded once to f16 --
 * the values the GEMM's loader unpack produces, made once for GEMMs with many
 * rows (ggml's q8_0 / q4_0 block formats; which matrices carry them:
 * "Quantization" page, "The rule").
 * K % 32 == 0; out 16-byte aligned.  Errors: ERR_ARG, ERR_DTYPE, ERR_SHAPE. */
JEPA_B200_API int jepa_b200_op_dequant_f16(int dtype, const void *qs, const void *scales, int N, int K, void *out,
                                           void *stream);

/* Epilogues of jepa_b200_op_linear. */
typedef enum {
  JEPA_B200_EPI_F16 = 0,      /* out f16 [M, ldo] = A W^T + bias */
  JEPA_B200_EPI_GELU_F16 = 1, /* out f16 = GELU(A W^T + bias), exact erf form */
  JEPA_B200_EPI_RESID_F32 = 2,/* out f32 += A W^T + bias (residual add) */
  JEPA_B200_EPI_F32 = 3       /* out f32 = A W^T + bias */
} jepa_b200_epilogue;

/* tcgen05 GEMM out = epilogue(A W^T + bias).  A: f16 [M, K]; W: f16 [N, K]
 * (w_scales NULL) or the repacked q8_0 / q4_0 form (w = qs, w_scales =
 * scales).  bias f32 [N] or NULL.  Requires K % 64 == 0, N a multiple of
 * 128 or 192, ldo >= N.  A, W, out 16-byte aligned. */
JEPA_B200_API int jepa_b200_op_linear(const void *A, int M, int K, const void *w, const void *w_scales, int w_dtype, int N,
                        const float *bias, int epilogue, void *out, int ldo, void *stream);

/* The QKV projection with its scatter epilogue: columns [0, N) of A W^T +
 * bias are the parts first_part, first_part+1, ... of (q, k, v), each D =
 * 64 * heads wide.  q, k: f16 [B*heads, ntok, 64]; vt: f16 [B*heads, 64,
 * npad] (V transposed, npad >= ntok a multiple of 128; columns >= ntok are
 * left untouched).  Rows of A are tokens b*ntok + t.  Pass NULL for a part
 * that is not produced. */
JEPA_B200_API int jepa_b200_op_linear_qkv(const void *A, int M, int K, const void *w, const void *w_scales, int w_dtype, int N,
                            const float *bias, int ntok, int heads, int npad, int first_part, void *q, void *k,
                            void *vt, void *stream);

/* Flash attention O = softmax(q k^T / 8 + mask) v per (clip, head), d_h = 64.
 * q, k: f16 [B*heads, ntok, 64]; vt: f16 [B*heads, 64, npad] (zero beyond
 * ntok); out: f16 [B*ntok, heads*64] (token-major, head h in columns
 * 64h..64h+63).  mask: jepa_b200_mask; has_cls and patches_per_slot define
 * the block-causal rule (ntok = has_cls + slots * patches_per_slot). */
JEPA_B200_API int jepa_b200_op_attention(const void *q, const void *k, const void *vt, int B, int heads, int ntok, int npad,
                           int mask, int has_cls, int patches_per_slot, void *out, void *stream);

/* Tubelet patch-embed, plus pos_embed and the CLS row: the pixels unfolded
 * into the patch matrix (f16, in a per-device scratch buffer of the library
 * that grows on demand: calls on several streams must not overlap), then the
 * tensor-core GEMM whose epilogue adds the bias and the positional rows.
 * pixels f32 [B, T, 3, H, W]; w_pe f16 [D, kpad] (kpad = 3*kt*p*p rounded up
 * to 64, zero padded); bias f32 [D]; pos f32 [ntok, D]; cls f32 [D] (has_cls);
 * x out f32 [B, ntok, D] with ntok = has_cls + (T/kt)(H/p)(W/p).  The shape
 * limits are the model's: D <= 4096, 3*kt*p*p <= 32768, B * ntok <= 524288
 * (JEPA_B200_ERR_SHAPE otherwise). */
JEPA_B200_API int jepa_b200_op_patch_embed(const float *pixels, int B, int T, int H, int W, int patch, int tubelet,
                             const void *w_pe, int D, const float *bias, const float *pos, const float *cls,
                             int has_cls, float *x, void *stream);

/* Small-M matrix-vector product y = epi(x W^T + bias) for M <= 64 rows
 * (attentive head).  x f32 [M, K]; W as in op_linear (K % 32 == 0 for
 * quantised, K % 8 == 0 for f16); epi 0 = store, 1 = GELU, 2 = residual:
 * y = resid[row * resid_row_stride] + x W^T + bias (resid may alias y when
 * resid_row_stride = N).  y f32 [M, N]. */
JEPA_B200_API int jepa_b200_op_gemv(const float *x, int M, int K, const void *w, const void *w_scales, int w_dtype, int N,
                      const float *bias, int epi, const float *resid, int resid_row_stride, float *y, void *stream);

/* One-query cross-attention per (clip, head): q f32 [heads*64] shared by
 * every clip; k f16 [B*heads, ntok, 64]; vt f16 [B*heads, 64, npad];
 * out f32 [B, heads*64].  ntok <= 16384. */
JEPA_B200_API int jepa_b200_op_xattn_1q(const float *q, const void *k, const void *vt, int B, int heads, int ntok, int npad,
                          float *out, void *stream);

/* Mean over rows first..ntok-1 of each clip of y f32 [B, ntok, D] -> out f32 [B, D]. */
JEPA_B200_API int jepa_b200_op_mean_pool(const float *y, int B, int ntok, int D, int first, float *out, void *stream);

/* Mean pooling that allocates nothing, for callers that cannot call
 * cudaMalloc (serving loops under a fixed device-memory budget, code that
 * must not stall the device, which cudaMalloc may synchronise, hosts whose
 * allocator belongs to another framework).  There is no counterpart on the
 * pages: it is jepa_b200_op_mean_pool with its partial sums kept in a fixed
 * file-scope device array (4 MiB on every GPU that loads the library, held
 * until exit) instead of a buffer grown with cudaMalloc.
 * y f32 [B, ntok, D] -> out f32 [B, D] (mean over rows first..ntok-1), device
 * pointers.  Limit: B * D <= 32768; larger sizes return ERR_SHAPE before any
 * device work.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current and keeps it for
 * the later calls on that device.  Every call shares the array and overwrites
 * the partial sums it reads, so its previous contents never matter, but calls
 * that overlap on the GPU (two streams, two host threads) race on it.
 * Returns OK, ERR_ARG, ERR_SHAPE or ERR_CUDA. */
JEPA_B200_API int jepa_b200_op_mean_pool_noalloc(const float *y, int B, int ntok, int D, int first, float *out,
                                                 void *stream);

/* Synchronise `stream`, return and clear the device status of the op calls
 * (OK, ERR_TIMEOUT, ERR_CUDA). */
JEPA_B200_API int jepa_b200_op_sync_status(void *stream);

/* Bound in nanoseconds of device-side waits for the op entry points
 * (default 4e9; 0 exercises the timeout path). */
JEPA_B200_API void jepa_b200_op_set_timeout_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif
#endif /* JEPA_B200_H */
