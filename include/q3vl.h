/*
 * q3vl.h -- C ABI of libq3vl: the full-sequence causal prefill of a
 * Qwen3-VL text decoder layer and layer stack on an NVIDIA B200 (sm_100a),
 * a KV cache written by the prefill with one-token decode against it, and
 * the steps either side of the layers (embedding gather, LM head).
 *
 * Sources of the operations (web pages, cited by title and item):
 *   [P] inferencelayer 0.2.3 src/vision.rs, `mrope_positions` -- positions
 *       from runs of image placeholders and a grid list.
 *   [C] cortiq-engine 0.8.21 src/cortiq_engine/qwen3te.rs -- the layer:
 *       `rms_norm_into`, `silu`, `Qwen3Encoder::norm_rope`,
 *       `Qwen3Encoder::mrope_positions`, `Qwen3Encoder::attention_gemm`,
 *       `Qwen3Encoder::encode_with_images`.
 *   [H] hf2q 0.1.1 src/inference/models/qwen3vl_text/forward.rs -- module
 *       doc (per-layer order, bias before the q/k norm; "Why no KV cache
 *       yet"), and `forward_text_prefill_logits_last`: its DeepStack
 *       validation, step 1 (embedding lookup and soft-token splice) and
 *       step 4 (final norm and LM head).
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers on the current
 *     device; "host" pointers are ordinary host memory.
 *   - The caller owns every buffer. The library allocates no device memory
 *     in any call; scratch space is the caller's workspace `ws`.
 *   - Device work is enqueued on `stream` (NULL = the legacy default
 *     stream) and never synchronised inside a call. A return of Q3VL_OK
 *     means the work was validated and launched.
 *   - Errors that can only be seen on the device (a grid/run mismatch, a
 *     DeepStack row out of range, a device wait that hit its time limit)
 *     are recorded in a per-device error word; read and clear it with
 *     q3vl_device_status().
 *   - Matrices are row-major. Weight matrices use the torch-Linear
 *     [out_features, in_features] layout.
 *   - dtype BF16: weights and activations bf16, accumulation fp32.
 *     dtype FP32: everything fp32 (CUDA-core FMA, no TF32).
 *   - No C++ exception crosses this boundary; the message of the last
 *     non-zero status of the calling thread is q3vl_last_error().
 */
#ifndef Q3VL_H
#define Q3VL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* q3vl_stream; /* same type as cudaStream_t */

enum q3vl_status_code {
  Q3VL_OK = 0,
  Q3VL_EINVAL = -1,       /* null pointer, bad size or shape */
  Q3VL_ERANGE = -2,       /* an image/DeepStack row outside [0, S) or repeated */
  Q3VL_EGRID = -3,        /* image placeholders and grids disagree [P] */
  Q3VL_EDEEPSTACK = -4,   /* DeepStack slabs and image rows disagree [H] */
  Q3VL_EWORKSPACE = -5,   /* workspace or packed buffer too small */
  Q3VL_ECUDA = -6,        /* a CUDA runtime call failed */
  Q3VL_ETIMEOUT = -7,     /* a device-side wait hit its time limit */
  Q3VL_EUNSUPPORTED = -8  /* head_dim != 128, a decode shape outside its limits, ... */
};

enum q3vl_dtype { Q3VL_DTYPE_FP32 = 0, Q3VL_DTYPE_BF16 = 1 };

/* Shape and constants of one decoder layer ([C] `Qwen3Encoder` fields). */
typedef struct q3vl_config {
  int32_t hidden;           /* H; multiple of 64 */
  int32_t n_heads;          /* nh; a multiple of n_kv_heads */
  int32_t n_kv_heads;       /* nkv */
  int32_t head_dim;         /* hd; must be 128 */
  int32_t intermediate;     /* I; multiple of 128 */
  int32_t dtype;            /* enum q3vl_dtype */
  int32_t has_qkv_bias;     /* 0 or 1 */
  int32_t mrope_section[3]; /* (t, h, w) slot counts, (24, 20, 20) */
  double rope_theta;        /* 5e6 */
  double rms_eps;           /* 1e-6 */
} q3vl_config;

/* A layer's weights as a checkpoint holds them (device, dtype of cfg). */
typedef struct q3vl_raw_weights {
  const void* attn_norm;  /* [H] input RMSNorm gain (plain gain, not 1+w) */
  const void* wq;         /* [nh*hd, H] */
  const void* wk;         /* [nkv*hd, H] */
  const void* wv;         /* [nkv*hd, H] */
  const void* bq;         /* [nh*hd] or NULL (required iff has_qkv_bias) */
  const void* bk;         /* [nkv*hd] or NULL */
  const void* bv;         /* [nkv*hd] or NULL */
  const void* q_norm;     /* [hd] per-head q RMSNorm gain, shared by heads */
  const void* k_norm;     /* [hd] */
  const void* wo;         /* [H, nh*hd] */
  const void* ffn_norm;   /* [H] post-attention RMSNorm gain */
  const void* wg;         /* [I, H] gate */
  const void* wu;         /* [I, H] up */
  const void* wd;         /* [H, I] down */
} q3vl_raw_weights;

/* A packed layer: views into a buffer written by q3vl_pack_layer (device). */
typedef struct q3vl_layer {
  const void* w_qkv;   /* [nh*hd + 2*nkv*hd, H]: rows Wq;Wk;Wv, column k scaled by attn_norm[k] */
  const float* b_qkv;  /* [nh*hd + 2*nkv*hd] fp32, or NULL without bias */
  const float* q_norm; /* [hd] fp32 */
  const float* k_norm; /* [hd] fp32 */
  const void* w_o;     /* [H, nh*hd] */
  const void* w_gu;    /* [2I, H]: 256-row blocks of 128 gate rows then the 128 matching up
                          rows; column k scaled by ffn_norm[k] */
  const void* w_down;  /* [H, I] */
} q3vl_layer;

/* Byte size of one packed layer. Returns 0 for an invalid config. */
size_t q3vl_packed_layer_bytes(const q3vl_config* cfg);

/* Packs `raw` into `packed` (device, >= q3vl_packed_layer_bytes, 256-byte
 * aligned) and fills `out` with views into it. The input-norm gain is folded
 * into the columns of [Wq;Wk;Wv] and the FFN-norm gain into the gate/up
 * rows, so that RMSNorm(x) W^T = inv_rms(x) * (x (W diag g)^T) ([C]
 * `rms_norm_into`). One-time work; stream-ordered. */
int q3vl_pack_layer(const q3vl_config* cfg, const q3vl_raw_weights* raw, void* packed,
                    size_t packed_bytes, q3vl_layer* out, q3vl_stream stream);

/* Fills `out` with the views of an already packed buffer. */
int q3vl_layer_views(const q3vl_config* cfg, const void* packed, q3vl_layer* out);

/* ---------------------------------------------------------------------------
 * P0. MRoPE position ids ([P] `mrope_positions`, [C] `mrope_positions`).
 * token_types: device uint8 [S], 0 = text, 1 = image placeholder.
 * grids:       device int32 [n_grids][3] = (t, merged rows, merged cols) of
 *              each image or video in prompt order; t = frames (1 for a
 *              still image), all three >= 1.
 * pos:         device int32 [3][S] out, axis-major (t row, h row, w row).
 * info:        device int32 [2] out: info[0] = status (Q3VL_OK or
 *              Q3VL_EGRID), info[1] = next position (one past the largest
 *              position on any axis).
 * A text token takes (c, c, c) and advances c by 1. Grid g occupies
 * t * rows * cols placeholder tokens in (frame, row, col) order; token
 * (f, r, q) takes (c + f, c + r, c + q), and the grid advances c by
 * max(rows, cols) only ([P] `mrope_positions`). Grids are consumed whole and
 * in order. 1 <= S <= 2^30, 0 <= n_grids <= 4096; otherwise Q3VL_EINVAL.
 * Bit-exact integer work.
 * ------------------------------------------------------------------------- */
int q3vl_mrope_positions(const uint8_t* token_types, int64_t S, const int32_t* grids,
                         int32_t n_grids, int32_t* pos, int32_t* info, q3vl_stream stream);

/* ---------------------------------------------------------------------------
 * Whole-layer and whole-stack prefill.
 * ------------------------------------------------------------------------- */

/* Workspace bytes for q3vl_layer_prefill / q3vl_stack_prefill at length S
 * (0 for an invalid config). */
size_t q3vl_workspace_bytes(const q3vl_config* cfg, int64_t S);

/* One decoder layer, in place: x <- layer(x) ([C] `encode_with_images`,
 * loop body):
 *   xn = RMSNorm(x, attn_norm); q,k,v = xn W^T (+ b);
 *   q,k <- MRoPE(RMSNorm_head(q|k, q_norm|k_norm), pos);
 *   h = x + attention_causal_gqa(q, k, v) Wo^T;
 *   x' = h + (silu(hn Wg^T) * (hn Wu^T)) Wd^T, hn = RMSNorm(h, ffn_norm);
 *   x'[ds_rows[k]] += ds_slab[k] when ds_slab != NULL (DeepStack).
 * x:       device [S, H] in/out.
 * pos:     device int32 [3][S] (from q3vl_mrope_positions).
 * ds_slab: device [n_img, H] or NULL; ds_rows: device int32 [n_img], the
 *          image rows in span order (required iff ds_slab != NULL, n_img > 0;
 *          rows outside [0, S) or repeated are a device error Q3VL_ERANGE).
 * ws:      device workspace of >= q3vl_workspace_bytes(cfg, S) bytes,
 *          256-byte aligned. */
int q3vl_layer_prefill(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int64_t S,
                       const int32_t* pos, const void* ds_slab, const int32_t* ds_rows,
                       int32_t n_img, void* ws, size_t ws_bytes, q3vl_stream stream);

/* n_layers layers, DeepStack slab l added after layer l for l < n_ds, then
 * x <- RMSNorm(x, final_norm) when final_norm != NULL (otherwise the
 * unnormalised residual stream is returned, as the 32B prompt encoder does).
 * layers:    host array [n_layers] of packed layers.
 * ds_slabs:  host array [n_ds] of device [n_img, H] slabs, or NULL with
 *            n_ds = 0. With slabs, n_ds >= 3 and n_img > 0 ([H]); otherwise
 *            Q3VL_EDEEPSTACK. */
int q3vl_stack_prefill(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                       const void* final_norm, void* x, int64_t S, const int32_t* pos,
                       const void* const* ds_slabs, int32_t n_ds, const int32_t* ds_rows,
                       int32_t n_img, void* ws, size_t ws_bytes, q3vl_stream stream);

/* The same layer as q3vl_layer_prefill, with no workspace argument and no
 * allocation of any kind: for callers that cannot allocate device memory (a
 * plug-in inside a framework whose memory manager has reserved the GPU's
 * memory, a C caller with no device allocator, a path that must not pay
 * cudaMalloc's device-wide synchronisation). The pages have no counterpart;
 * it exists for such callers only. Scratch is a 64 MiB array inside the
 * library that every GPU loading it keeps until the process exits; a layer
 * whose q3vl_workspace_bytes(cfg, S) exceeds 64 MiB is refused with
 * Q3VL_EWORKSPACE (e.g. the 2B shape fits up to S = 1536 on a 148-SM GPU). The first call on
 * a device looks up the array's device address with that device current;
 * make that first call before any stream capture. The address is kept for
 * the life of the process: do not call this entry point again on a device
 * after cudaDeviceReset (or any other teardown of its primary context),
 * which reloads the library's device code at a new address. All calls share the one
 * array: calls that overlap on the GPU (other streams, other host threads)
 * race on it and must be serialised by the caller. Each call writes every
 * scratch region before reading it, so nothing carries over between calls. */
int q3vl_layer_prefill_noalloc(const q3vl_config* cfg, const q3vl_layer* layer, void* x,
                               int64_t S, const int32_t* pos, const void* ds_slab,
                               const int32_t* ds_rows, int32_t n_img, q3vl_stream stream);

/* ---------------------------------------------------------------------------
 * Step-level calls: each step of the layer on its own, for per-step
 * parity and timing. The layer call is exactly this sequence.
 * Ntot = nh*hd + 2*nkv*hd. The four GEMM steps (P3, P6, P8, P9) also take a
 * layer workspace `ws` (>= q3vl_workspace_bytes(cfg, S) bytes, 256-byte
 * aligned): only its stream-K region (fp32 partial tiles and flags for the
 * tiles whose K range is split across CTAs) is used.
 * ------------------------------------------------------------------------- */

/* P1. cos_sin[p][i] = (cos, sin)(pos[axis(i)][p] * theta^(-2i/hd)), i < hd/2,
 * fp32 [S][hd/2][2]. axis(i) = h for i = 1 (mod 3) below 3*section[1], w
 * for i = 2 (mod 3) below 3*section[2], t otherwise ([C] `norm_rope`). The
 * angle is formed in fp64. */
int q3vl_rope_table(const q3vl_config* cfg, const int32_t* pos, int64_t S, float* cos_sin,
                    q3vl_stream stream);

/* P2/P7. inv_rms[r] = 1 / sqrt(mean_j x[r][j]^2 + eps) over `width`
 * columns of x (device, cfg dtype, row stride = width). */
int q3vl_rms_rowstat(const q3vl_config* cfg, const void* x, int64_t S, int64_t width,
                     float* inv_rms, q3vl_stream stream);

/* P3+P4. qkv[r] = [q | k | v] of token r, [S, Ntot] in cfg dtype:
 * q,k,v = inv_rms[r] * (x W_qkv^T) + b, then each q and k head is
 * RMS-normalised with q_norm / k_norm and rotated by cos_sin ([S][64][2] as
 * q3vl_rope_table writes it; a bf16 call first copies it, slot-major, into
 * the workspace, so it must not overlap the workspace's first
 * S * 512 bytes). */
int q3vl_qkv_proj(const q3vl_config* cfg, const q3vl_layer* layer, const void* x, int64_t S,
                  const float* inv_rms, const float* cos_sin, void* qkv, void* ws,
                  size_t ws_bytes, q3vl_stream stream);

/* P5. o[r][h*hd + d] = causal GQA softmax attention of q head h over KV head
 * h / (nh/nkv), scale 1/sqrt(hd); qkv as written by q3vl_qkv_proj, o
 * [S, nh*hd] in cfg dtype. */
int q3vl_attention(const q3vl_config* cfg, const void* qkv, int64_t S, void* o,
                   q3vl_stream stream);

/* P6. h = x + o Wo^T, [S, H]. */
int q3vl_o_proj(const q3vl_config* cfg, const q3vl_layer* layer, const void* o, const void* x,
                int64_t S, void* h, void* ws, size_t ws_bytes, q3vl_stream stream);

/* P8. act = silu(g) * u with [g|u] = inv_rms2[r] * (h W_gu^T), [S, I]. */
int q3vl_gate_up(const q3vl_config* cfg, const q3vl_layer* layer, const void* h, int64_t S,
                 const float* inv_rms2, void* act, void* ws, size_t ws_bytes,
                 q3vl_stream stream);

/* P9. out = h + act Wd^T, plus slab row ds_map[r] on rows with ds_map[r] >= 0
 * (ds_slab and ds_map may be NULL). ds_map: device int32 [S]. out may
 * equal neither h nor act. */
int q3vl_down(const q3vl_config* cfg, const q3vl_layer* layer, const void* act, const void* h,
              int64_t S, const void* ds_slab, const int32_t* ds_map, void* out, void* ws,
              size_t ws_bytes, q3vl_stream stream);

/* DeepStack row map: ds_map[r] = k if ds_rows[k] == r, else -1 (device
 * int32 [S]). Out-of-range or repeated rows record Q3VL_ERANGE. */
int q3vl_deepstack_map(const int32_t* ds_rows, int32_t n_img, int64_t S, int32_t* ds_map,
                       q3vl_stream stream);

/* P10. x <- RMSNorm(x, gain) in place over rows of width H. */
int q3vl_final_norm(const q3vl_config* cfg, void* x, int64_t S, const void* gain,
                    q3vl_stream stream);

/* ---------------------------------------------------------------------------
 * KV cache and incremental decode (bf16 only; FP32 configs are refused with
 * Q3VL_EUNSUPPORTED).
 *
 * [H] "Why no KV cache yet": a generation loop may re-run the prefill over
 * prompt + tokens decoded so far and keep the last row; a KV cache gives the
 * same result without re-running the earlier rows. The calls below keep,
 * per layer, the K (after the per-head norm and MRoPE) and V rows of each
 * sequence, and decode one new token per sequence against them.
 * ------------------------------------------------------------------------- */

/* One layer's cache (device memory owned by the caller). Row r of sequence
 * slot s is at k + (s * cap + r) * nkv*hd elements (likewise v): K and V of
 * every KV head of one token, head-major, exactly as the prefill's QKV step
 * lays them out. */
typedef struct q3vl_kv_cache {
  void* k;        /* device bf16 [n_seq][cap][nkv*hd], 16-byte aligned */
  void* v;        /* device bf16 [n_seq][cap][nkv*hd], 16-byte aligned */
  int64_t cap;    /* rows per sequence slot, 1 <= cap <= 131072 */
  int32_t n_seq;  /* sequence slots, >= 1, with n_seq * cap < 2^31 */
} q3vl_kv_cache;

/* q3vl_layer_prefill / q3vl_stack_prefill that also write rows 0..S-1 of
 * sequence slot `seq` of each layer's cache (kv: host pointer to one cache
 * for the layer call, to an array [n_layers] for the stack call). Requires
 * S <= cap and 0 <= seq < n_seq (else Q3VL_ERANGE). Same workspace. */
int q3vl_layer_prefill_kv(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int64_t S,
                          const int32_t* pos, const void* ds_slab, const int32_t* ds_rows,
                          int32_t n_img, const q3vl_kv_cache* kv, int32_t seq, void* ws,
                          size_t ws_bytes, q3vl_stream stream);
int q3vl_stack_prefill_kv(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                          const void* final_norm, void* x, int64_t S, const int32_t* pos,
                          const void* const* ds_slabs, int32_t n_ds, const int32_t* ds_rows,
                          int32_t n_img, const q3vl_kv_cache* kv, int32_t seq, void* ws,
                          size_t ws_bytes, q3vl_stream stream);

/* Workspace bytes for the decode calls with batch B (1 <= B <= 256) against
 * caches of `cap` rows per slot (0 for invalid arguments). */
size_t q3vl_decode_workspace_bytes(const q3vl_config* cfg, int32_t B, int64_t cap);

/* One new token for each of B sequences through one layer, in place:
 * x[b] <- layer(x[b]) where token b attends to rows 0..len[b]-1 of cache
 * slot seq[b] and to itself, and its own K/V row is written at row len[b]
 * of that slot first (the same arithmetic as the prefill's row len[b]).
 * x:   device bf16 [B, H] in/out, 16-byte aligned.
 * pos: device int32 [3][B], the new tokens' (t, h, w) positions (a text
 *      token after a prompt: next position + i on every axis).
 * kv:  host pointer to this layer's cache.
 * seq: device int32 [B], distinct slots in [0, n_seq).
 * len: device int32 [B], rows already cached, 0 <= len[b] < cap. The call
 *      reads but does not advance it (see q3vl_decode_advance).
 * A seq or len out of range is recorded as the device error Q3VL_ERANGE and
 * that token's output row is left unspecified.
 * ws:  device workspace of >= q3vl_decode_workspace_bytes(cfg, B, cap)
 *      bytes, 256-byte aligned.
 * The call starts after all earlier work in `stream`; its attention reads the
 * cached rows 0..len[b]-1 while the projection before it still runs, so no
 * other stream may write those rows during the call. */
int q3vl_layer_decode(const q3vl_config* cfg, const q3vl_layer* layer, void* x, int32_t B,
                      const int32_t* pos, const q3vl_kv_cache* kv, const int32_t* seq,
                      const int32_t* len, void* ws, size_t ws_bytes, q3vl_stream stream);

/* n_layers layers of q3vl_layer_decode (kv: host array [n_layers]), then
 * x <- RMSNorm(x, final_norm) when final_norm != NULL. The new tokens are
 * text, so no DeepStack slab applies. */
int q3vl_stack_decode(const q3vl_config* cfg, int32_t n_layers, const q3vl_layer* layers,
                      const void* final_norm, void* x, int32_t B, const int32_t* pos,
                      const q3vl_kv_cache* kv, const int32_t* seq, const int32_t* len, void* ws,
                      size_t ws_bytes, q3vl_stream stream);

/* After a decode step of text tokens: len[b] += 1 and pos[a][b] += 1 on all
 * three axes (device int32 arrays [B] and [3][B]), so that a captured decode
 * step can be replayed for the next token. */
int q3vl_decode_advance(int32_t B, int32_t* pos, int32_t* len, q3vl_stream stream);

/* ---------------------------------------------------------------------------
 * The steps either side of the layers ([H] `forward_text_prefill_logits_last`
 * steps 1 and 4).
 * ------------------------------------------------------------------------- */

/* Token embedding gather with the soft-token splice: x[p] = table[tokens[p]]
 * for p < S, then x[soft_rows[k]] = soft[k] (the rows a vision tower's
 * embeddings replace; an injected range [s, e) is the rows s..e-1).
 * table:  device [vocab, H] in cfg dtype, 16-byte aligned.
 * tokens: device int32 [S]. An id outside [0, vocab) is the device error
 *         Q3VL_ERANGE, and that row is left zero.
 * soft, soft_rows: device [n_soft, H] (cfg dtype) and int32 [n_soft], or NULL
 *         with n_soft = 0. Rows outside [0, S) or repeated (overlapping
 *         injections) are the device error Q3VL_ERANGE ([H] validation).
 * x:      device [S, H] out.
 * ws:     device scratch of >= 4*S bytes, 256-byte aligned, when n_soft > 0
 *         (a row map); may be NULL otherwise. */
int q3vl_embed(const q3vl_config* cfg, const void* table, int64_t vocab, const int32_t* tokens,
               int64_t S, const void* soft, const int32_t* soft_rows, int32_t n_soft, void* x,
               void* ws, size_t ws_bytes, q3vl_stream stream);

/* Workspace bytes of q3vl_lm_head for B rows (0 for invalid arguments). */
size_t q3vl_lm_head_workspace_bytes(const q3vl_config* cfg, int32_t B);

/* Final norm and LM head: logits[b] = RMSNorm(x[b], final_norm) W^T in fp32
 * (bf16 configs only; the rows are normalised in fp32 and rounded to bf16
 * before the product).
 * x:          device bf16 [B, H], 1 <= B <= 256: e.g. the last row of a
 *             prefill, or the B decoded tokens.
 * final_norm: device bf16 [H] gain, or NULL for rows already normalised.
 * weight:     device bf16 [vocab, H], 16-byte aligned: the output weight, or
 *             the token embedding table when the embeddings are tied.
 * logits:     device fp32 [B, vocab] out.
 * ws:         >= q3vl_lm_head_workspace_bytes(cfg, B) bytes, 256-byte aligned. */
int q3vl_lm_head(const q3vl_config* cfg, const void* x, int32_t B, const void* final_norm,
                 const void* weight, int64_t vocab, float* logits, void* ws, size_t ws_bytes,
                 q3vl_stream stream);

/* ---------------------------------------------------------------------------
 * Diagnostics.
 * ------------------------------------------------------------------------- */

/* Synchronises `stream`, returns the current device's recorded error
 * (Q3VL_OK if none) in *code and an internal location tag in *where, and
 * clears the record. Returns Q3VL_ECUDA if the synchronisation failed. */
int q3vl_device_status(q3vl_stream stream, int32_t* code, int32_t* where);

/* Launches one tiny kernel that waits on an mbarrier nothing arrives at,
 * with a limit of timeout_us microseconds; the wait gives up, records
 * Q3VL_ETIMEOUT and the kernel returns. Exercises the time-limit path of
 * every device wait without faulting or hanging the GPU. */
int q3vl_selftest_wait_timeout(uint32_t timeout_us, q3vl_stream stream);

/* Stage timing: from now on, every q3vl_layer_prefill call on this thread
 * records events[i] (cudaEvent_t handles, created by the caller) on its
 * stream at the stage boundaries: 0 start, 1 after the cos/sin table (and
 * DeepStack map), 2 after the input RMS statistic, 3 after the QKV
 * projection (norm + MRoPE epilogue), 4 after attention, 5 after the
 * o-projection, 6 after the post-attention statistic, 7 after gate/up,
 * 8 after down. n_events must be 9, or 0 to stop recording. The same events
 * are re-recorded by each call, so pass a fresh set per call to keep them
 * all. q3vl_stack_prefill records none. */
int q3vl_set_stage_events(void* const* events, int32_t n_events);

/* Number of kernels this library has enqueued in this process. */
uint64_t q3vl_launch_count(void);

/* Message of the calling thread's last non-zero status. */
const char* q3vl_last_error(void);

/* Library version string. */
const char* q3vl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* Q3VL_H */
