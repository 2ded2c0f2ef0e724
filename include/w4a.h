/*
 * w4a -- int4 weight-only (AWQ-format) decode of an OLMo-3-32B-shaped dense
 * decoder on one NVIDIA B200 (sm_100a).  Public C ABI.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Returns an int status: W4A_OK (0) or a negative W4A_ERR_* code.  On error,
 *    w4a_last_error() returns a thread-local, human-readable message.  Nothing
 *    aborts, exits or throws across this boundary.
 *  - Pointers named as device pointers must be CUDA device memory aligned to 16
 *    bytes; pointers to W4A* descriptor structs and sizes are host memory.
 *  - Every GPU call is asynchronous and ordered on the caller's stream
 *    (`stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream).  No entry point synchronises except w4a_check().
 *  - All device memory is owned by the caller.  Workspaces are sized by the
 *    matching *_workspace_bytes() query and must be zero-filled once before
 *    their first use; the kernels leave them zeroed again on success.  After a
 *    W4A_ERR_TIMEOUT / W4A_ERR_KERNEL result a workspace must be re-zeroed.
 *  - Device-side failures (a bounded wait that ran out) are recorded in the
 *    workspace's error word; w4a_check() synchronises the stream and turns it
 *    into a status.  Kernels never trap.
 */
#ifndef W4A_H
#define W4A_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4A_MAX_LAYERS 128

#if defined(__GNUC__)
#define W4A_API __attribute__((visibility("default")))
#else
#define W4A_API
#endif

enum {
  W4A_OK = 0,
  W4A_ERR_ARG = -1,          /* null pointer or invalid enum */
  W4A_ERR_SHAPE = -2,        /* sizes the kernels do not support */
  W4A_ERR_ALIGN = -3,        /* pointer not 16-byte aligned */
  W4A_ERR_UNSUPPORTED = -4,  /* valid request the library does not implement */
  W4A_ERR_CUDA = -5,         /* a CUDA runtime call failed */
  W4A_ERR_WORKSPACE = -6,    /* workspace too small */
  W4A_ERR_KERNEL = -7,       /* device error word set (bad shape / position / fp16 overflow) */
  W4A_ERR_TIMEOUT = -8       /* a bounded device wait ran out */
};

enum { W4A_F32 = 0, W4A_BF16 = 1 };
enum { W4A_LAYOUT_CANONICAL = 0, W4A_LAYOUT_TILED = 1, W4A_LAYOUT_SYM32 = 2 };
enum { W4A_EPI_NONE = 0, W4A_EPI_SUMSQ = 1, W4A_EPI_SILU_MUL = 2 };

/* Model shape.  Source: ATLAS-OLMo-3-32B-Think-v4 model card, "Architecture
 * deep-dive" (64 layers, [SWA,SWA,SWA,full] x16, window 4,096, GQA 40/8,
 * head_dim 128, hidden 5,120, FFN 27,648 SwiGLU, post-norm + full-projection
 * QK-norm, RoPE theta 500,000 with YaRN x8 from 8,192, attention factor
 * ~1.208, vocab 100,278); archdb "Olmo-3-1125-32B" (RMSNorm eps 1e-6, YaRN on
 * full-attention layers only). */
typedef struct {
  int32_t d_model, n_layers, n_heads, n_kv_heads, head_dim, ffn, vocab, window;
  uint8_t full_layers[W4A_MAX_LAYERS]; /* 1 = full attention (YaRN), 0 = sliding window */
  double rope_theta;                   /* 500000 */
  double yarn_factor;                  /* 8 */
  int32_t yarn_orig_ctx;               /* 8192 */
  int32_t group;                       /* 128: asymmetric int4 (fp16 scale, int4 zero);
                                          32: the symmetric checkpoint format (bf16 scale) */
  double yarn_beta_fast, yarn_beta_slow; /* 32, 1 */
  double eps;                          /* 1e-6 */
  int32_t final_norm;                  /* 1: RMSNorm with gains before lm_head */
  int32_t reserved;
} W4AConfig;

/* One int4 matrix W [n, k] (n outputs, k inputs).  Source: ATLAS-OLMo-3-32B-
 * Think-v4 model card, "Quantization recipe" (column j in word j/8,
 * little-endian nibble).  Two formats:
 *  group 128, w = (q - z) * s, asymmetric (the AWQ-style g128 format):
 *   CANONICAL: qweight uint32 [n, k/8]; scales fp16 bits [k/128, n];
 *              qzeros uint32 [k/128, n/8] (eight rows per word, same nibble order).
 *  group 32, w = (nibble - 8) * s, symmetric (the model card's checkpoint:
 *  "symmetric (no zero-points), group size 32", bf16 scales, stored nibble
 *  q + 8), ingested as stored:
 *   SYM32:     qweight uint32 [n, k/8] (stored nibbles); scales bf16 bits
 *              [n, k/32] (one per output row and 32-input group); qzeros unused.
 *  TILED:     qweight points at the kernel layout written by w4a_tile() from
 *             either canonical form (group selects which); scales and qzeros
 *             are unused.  row_interleave = 1 means tiled rows alternate
 *             between canonical rows [0, n/2) and [n/2, n) (the fused gate/up
 *             matrix). */
typedef struct {
  int64_t n, k;
  int32_t group;
  int32_t layout;
  int32_t row_interleave;
  int32_t reserved;
  const void* qweight;
  const void* scales;
  const void* qzeros;
} W4ATensor;

/* Per-layer weights of the decoder (device pointers).  qkv rows are [Q; K; V]
 * (q_dim + 2 kv_dim rows), gate_up rows are [gate; up] and must be tiled with
 * row_interleave = 1.  Gains are fp32. */
typedef struct {
  const void* qkv;       /* tiled int4 [q_dim + 2 kv_dim, d] */
  const void* o;         /* tiled int4 [d, q_dim] */
  const void* gate_up;   /* tiled int4, interleaved [2 ffn, d] */
  const void* down;      /* tiled int4 [d, ffn] */
  const float* q_norm;   /* [q_dim]  RMSNorm over the whole Q projection */
  const float* k_norm;   /* [kv_dim] RMSNorm over the whole K projection */
  const float* post_attn_norm; /* [d] */
  const float* post_ffn_norm;  /* [d] */
} W4ALayerWeights;

typedef struct {
  const uint16_t* embed;        /* bf16 [vocab, d] */
  const void* lm_head;          /* bf16 tiled by w4a_tile_bf16() from [vocab, d] */
  const float* final_norm;      /* [d], or NULL when cfg.final_norm == 0 */
  const W4ALayerWeights* layers;/* HOST array [n_layers] of device pointers */
} W4AModelWeights;

/* KV cache: one caller-owned device allocation of w4a_kv_bytes() bytes.  Layer
 * l stores K then V, each [batch, n_kv_heads, slots_l, head_dim] bf16, with
 * slots_l = max_ctx on full layers and = window (a ring, slot = pos % window)
 * on sliding-window layers.  Rows are stored with their 16-byte chunks
 * permuted (chunk c of slot s at position c ^ (s & 7)); use w4a_kv_write /
 * w4a_kv_read to move logical rows in and out.  Zero it once before use. */
typedef struct {
  void* base;
  int32_t batch;
  int32_t max_ctx;   /* multiple of 16 */
} W4AKVCache;

typedef struct W4AModel W4AModel;

W4A_API const char* w4a_last_error(void);
W4A_API int w4a_version(void);

/* ---- int4 codec --------------------------------------------------------- */

/* Quantize W [n, k] (device, fp32 or bf16 per w_dtype) to the canonical
 * triple.  Round-to-nearest min/max asymmetric per (row, group) in IEEE fp32:
 * s = fp16(fl32(fl32(max - min) / 15)) (0 -> 2^-24, overflow -> 65504),
 * z = clamp(rint(-min / s), 0, 15), q = clamp(rint(w / s) + z, 0, 15).
 * Source: model card "Quantization recipe" (format); AWQ's calibrated scale
 * search is replaced by RTN since it needs calibration data.
 * n % 8 == 0, k % group == 0, group == 128. */
W4A_API int w4a_pack(const void* W, int w_dtype, int64_t n, int64_t k, int group,
             uint32_t* qweight, uint16_t* scales, uint32_t* qzeros, void* stream);

/* Exact dequantization to fp32 [n, k] (device), from any layout: (q - z) * s,
 * or (nibble - 8) * s for group 32.  Bit-exact: the product of a 5-bit
 * integer and an fp16 or bf16 value is exact in fp32. */
W4A_API int w4a_unpack(const W4ATensor* t, float* out, void* stream);

/* Size of the tiled layout of an n x k int4 matrix: group 128, 16 x 512 units
 * of 4,256 bytes (n % 16 == 0, k % 512 == 0); group 32, 16 x 256 units of
 * 2,304 bytes (k % 256 == 0). */
W4A_API int w4a_tiled_bytes(int64_t n, int64_t k, int group, size_t* bytes);

/* Rewrite a CANONICAL (group 128) or SYM32 (group 32) tensor into the kernel
 * layout: units of 16 rows (codes in mma-fragment order, then the scales; the
 * zeros for group 128), ordered row-block-major.  row_interleave as in
 * W4ATensor. */
W4A_API int w4a_tile(const W4ATensor* canonical, int row_interleave, void* tiled,
             size_t tiled_bytes, void* stream);

/* Size / tiling of a bf16 matrix [n, k] (the lm_head) into 16-row x 128-column
 * units of 4,096 bytes; rows are padded to a multiple of 16 with zeros. */
W4A_API int w4a_tiled_bf16_bytes(int64_t n, int64_t k, size_t* bytes);
W4A_API int w4a_tile_bf16(const uint16_t* W, int64_t n, int64_t k, void* tiled,
                  size_t tiled_bytes, void* stream);

/* ---- GEMV ------------------------------------------------------------- */

W4A_API int w4a_gemv_workspace_bytes(const W4ATensor* W, int batch, size_t* bytes);

/* out = W~ x for x bf16 [batch, k] (device), batch 1..16, W TILED.
 * fp32 accumulation; split-K pieces are combined in a fixed order, so results
 * are bit-reproducible run to run.  Epilogues:
 *  W4A_EPI_NONE     out fp32 [batch, n]
 *  W4A_EPI_SUMSQ    out fp32 [batch, n]; aux fp32 [n/16, batch] = sum of
 *                   out^2 over each 16-row block (RMSNorm partials)
 *  W4A_EPI_SILU_MUL W tiled with row_interleave = 1; out bf16 [batch, n/2] =
 *                   silu(gate) * up (SwiGLU; model card "Architecture deep-dive")
 * Source: model card "What ATLAS implements for the W4 path" (GEMV with
 * inline int4 dequant). */
W4A_API int w4a_gemv(const W4ATensor* W, const uint16_t* x, int batch, void* out, int epilogue,
             float* aux, void* ws, size_t ws_bytes, void* stream);

/* ---- GEMV without a caller workspace --------------------------------------
 * This entry point is the library's own addition; the pages have no
 * counterpart.  It computes exactly what w4a_gemv computes (same kernel, same
 * split, bit-identical results) but takes no workspace and allocates nothing:
 * its scratch is a fixed array of W4A_NOALLOC_SCRATCH_BYTES inside the
 * library, one per device, whose address is looked up once per device.
 *  - Returns W4A_ERR_WORKSPACE when the shape and batch need more scratch
 *    than that (w4a_gemv_workspace_bytes tells how much they need).
 *  - The scratch is shared by every call on a device: calls that overlap in
 *    time (two streams, two host threads) race on it and give undefined
 *    results; serialize them.
 *  - The array keeps the last call's contents; each call first clears the
 *    part that must start at zero (the control words: grid barrier counters
 *    and the device error word) on `stream`.
 *  - Device-side failures (a bounded wait that ran out) land in the array's
 *    error word like in a workspace: w4a_check(NULL, 0, stream) reads it for
 *    the current device.  Call it after a call and before the next one on
 *    that device, since the next call clears the word.
 * Arguments, layouts and the other errors are as for w4a_gemv. */
#define W4A_NOALLOC_SCRATCH_BYTES 4194304
W4A_API int w4a_gemv_noalloc(const W4ATensor* W, const uint16_t* x, int batch, void* out, int epilogue,
                     float* aux, void* stream);

/* ---- attention ----------------------------------------------------------- */

W4A_API int w4a_attn_workspace_bytes(int batch, int n_heads, int n_kv_heads, int head_dim, size_t* bytes);

/* GQA decode attention for one layer.  q: bf16 [batch, n_heads, head_dim],
 * already QK-normed and rotated.  k_cache / v_cache: that layer's K and V
 * regions ([batch, n_kv_heads, slots, head_dim], chunk-permuted, see
 * W4AKVCache) which already hold the token at pos[b] (device int32 [batch]).
 * window == 0: full attention over slots [0, pos]; window == slots: a ring,
 * attending the last `window` positions.  out: bf16 [batch, n_heads, head_dim]
 * = softmax(q K^T / sqrt(head_dim)) V, query head h reading KV head
 * h / (n_heads / n_kv_heads).  Source: model card "Architecture deep-dive"
 * (GQA 40/8, SWA 4,096) and "Why the 3:1 SWA layout matters for serving". */
W4A_API int w4a_attn_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                    int batch, int n_heads, int n_kv_heads, int head_dim, int slots,
                    const int32_t* pos, int window, uint16_t* out,
                    void* ws, size_t ws_bytes, void* stream);

/* QK-norm + rotation + KV append for one layer: q_raw fp32 [batch, q_dim],
 * k_raw/v_raw fp32 [batch, kv_dim] (device).  q_out bf16 [batch, n_heads,
 * head_dim] = rope(RMSNorm(q_raw) * q_gain); k = rope(RMSNorm(k_raw) * k_gain)
 * and v are written as bf16 to slot pos % slots (full: slot pos) of k_cache /
 * v_cache.  `full` selects YaRN frequencies and the attention factor. */
W4A_API int w4a_qk_prep(const W4AConfig* cfg, int full, const float* q_raw, const float* k_raw,
                const float* v_raw, const float* q_gain, const float* k_gain,
                const int32_t* pos, int batch, uint16_t* q_out,
                uint16_t* k_cache, uint16_t* v_cache, int slots, void* stream);

/* ---- KV cache ------------------------------------------------------------ */

W4A_API int w4a_kv_bytes(const W4AConfig* cfg, int batch, int max_ctx, size_t* bytes);
/* Byte offsets of layer l's K and V regions inside the cache, and its slots. */
W4A_API int w4a_kv_layer(const W4AConfig* cfg, int batch, int max_ctx, int layer,
                 size_t* k_offset, size_t* v_offset, int* slots);
/* Copy logical rows k_src/v_src bf16 [n_kv_heads, n, head_dim] (device) into
 * slots [slot0, slot0 + n) of sequence b of one layer region (k/v point at
 * the layer's K and V regions). */
W4A_API int w4a_kv_write(uint16_t* k, uint16_t* v, int batch, int n_kv_heads, int head_dim, int slots,
                 int b, int slot0, int n, const uint16_t* k_src, const uint16_t* v_src, void* stream);
/* Inverse of w4a_kv_write. */
W4A_API int w4a_kv_read(const uint16_t* k, const uint16_t* v, int batch, int n_kv_heads, int head_dim,
                int slots, int b, int slot0, int n, uint16_t* k_dst, uint16_t* v_dst, void* stream);

/* ---- model ----------------------------------------------------------------- */

/* Builds a host-side handle (no device allocation, no copy of weights: the
 * pointers are kept).  YaRN/RoPE frequency tables are computed here. */
W4A_API int w4a_model_create(const W4AConfig* cfg, const W4AModelWeights* weights, W4AModel** out);
W4A_API int w4a_model_destroy(W4AModel* model);

W4A_API int w4a_decode_workspace_bytes(const W4AModel* model, int batch, size_t* bytes);

/* One decode step for sequences [seq0, seq0 + batch) of the cache: token_ids
 * and pos are device int32 [batch]; the token's K and V are appended at its
 * slot.  logits: fp32 [batch, vocab] (device, required); next_token: int32
 * [batch] greedy argmax (ties to the lowest index) or NULL; hidden_dump: fp32
 * [n_layers + 1, batch, d] (embedding, then the residual after each layer) or
 * NULL.  Runs as one persistent kernel with grid-wide phase barriers.
 * Source: model card "Architecture deep-dive" (post-norm, QK-norm, RoPE/YaRN,
 * GQA, SWA stack, SwiGLU, bf16 lm_head). */
W4A_API int w4a_decode_step(W4AModel* model, const int32_t* token_ids, const W4AKVCache* kv,
                    int seq0, int batch, const int32_t* pos, float* logits,
                    int32_t* next_token, float* hidden_dump, void* ws, size_t ws_bytes,
                    void* stream);

/* Prefill T tokens (device int32 [T]) of sequence `seq` at positions
 * start_pos .. start_pos + T - 1: what T sequential decode steps compute
 * (their K / V written to the cache, the last token's logits), with the
 * prompt's tokens taken through each layer together (model card
 * "Limitations & roadmap": batched / tiled prefill, GEMV -> GEMM): the int4
 * projections as tcgen05 GEMMs on weights expanded to fp16, causal attention
 * with the sliding window as a flash-attention kernel, then the final norm
 * and the lm_head for the last token only.  Prompts of fewer than 9 tokens
 * run token by token.
 * last_logits: fp32 [vocab] of the last token, or NULL.  ws: device scratch
 * of w4a_prefill_workspace_bytes(model, T) bytes, zero-filled once before its
 * first use (its leading part is a decode workspace, whose error word
 * w4a_check reads).  Full-attention layers need start_pos + T <= max_ctx. */
W4A_API int w4a_prefill_workspace_bytes(const W4AModel* model, int T, size_t* bytes);
W4A_API int w4a_prefill(W4AModel* model, const int32_t* tokens, int T, const W4AKVCache* kv,
                int seq, int start_pos, float* last_logits, void* ws, size_t ws_bytes,
                void* stream);

/* ---- prompt-time building blocks -------------------------------------------
 * int4 GEMM for many tokens: out = x . W~^T for x fp16 [M, k] (row-major,
 * 16-byte aligned rows), W TILED.  The weights are first expanded to fp16
 * (q - z) * s (rounded to nearest) in the workspace, then multiplied on the
 * tcgen05 tensor cores with fp32 accumulation.  row_scale: fp32 [M] or NULL;
 * row m of the product is multiplied by row_scale[m] (an fp16 range scaling
 * of x undone).  Epilogues: W4A_EPI_NONE out fp32 [M, n]; W4A_EPI_SILU_MUL (W
 * tiled with row_interleave = 1) out fp16 [M, n / 2] = silu(gate) * up, an
 * fp16 overflow is reported by w4a_check as W4A_ERR_KERNEL.  ws: device
 * scratch of w4a_gemm_workspace_bytes() bytes, its first 256 bytes zeroed
 * once (error word).  Source: model card "Limitations & roadmap" (GEMV ->
 * GEMM for prefill). */
W4A_API int w4a_gemm_workspace_bytes(const W4ATensor* W, size_t* bytes);
W4A_API int w4a_gemm(const W4ATensor* W, const uint16_t* x, int M, const float* row_scale, void* out,
             int epilogue, void* ws, size_t ws_bytes, void* stream);

/* Causal GQA attention of T prompt tokens at positions start_pos .. start_pos
 * + T - 1.  q bf16 [T, n_heads, head_dim] (normed and rotated); the prompt's
 * own keys and values k_new / v_new bf16 [n_kv_heads, T, head_dim] in plain
 * order; the positions before the prompt from one layer's cache regions
 * k_cache / v_cache (see W4AKVCache) of a cache of `batch` sequences,
 * sequence `seq`, which is only read (a ring of `window` slots cannot hold
 * the windows of two consecutive prompt tokens, so the prompt's rows are
 * appended to it afterwards).  window == 0: full attention over positions
 * 0 .. p (slot = position, start_pos + T <= slots); window == slots (a
 * multiple of 64): the last `window` positions, slot = position % window.
 * out fp16 [T, n_heads, head_dim] = softmax(q K^T / sqrt(head_dim)) V per
 * query head h over KV head h / (n_heads / n_kv_heads).  ws: >= 256 device
 * bytes, zeroed once (error word).  Source: model card "Architecture
 * deep-dive" (GQA 40/8, SWA 4,096). */
W4A_API int w4a_attn_prefill(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int batch,
                     int seq, int n_heads, int n_kv_heads, int head_dim, int slots, int window,
                     int start_pos, int T, const uint16_t* k_new, const uint16_t* v_new, uint16_t* out,
                     void* ws, size_t ws_bytes, void* stream);

/* Profiling aid (off by default).  With a device buffer set, every later
 * w4a_decode_step / w4a_prefill launch writes, per phase p (5 per layer, then
 * lm_head and argmax) and CTA c, eight %globaltimer stamps (ns) as uint64 at
 * buf[(p * n_sms + c) * 8 + i]: i = 0 phase start, 1 phase descriptor ready,
 * 2 first input pass done (norm statistics / raw inputs loaded), 3 inputs
 * staged, 4 units done, 5 partial results combined, 6 arrived at the grid
 * barrier, 7 unused except in the launch's first phase, where it holds the
 * CTA's start (before the launch setup).  A stamp the phase does not reach
 * stays as it was.
 * Phases beyond bytes / (64 * n_sms) are not recorded.  buf = NULL turns
 * tracing off.  Process-wide setting. */
W4A_API int w4a_trace(void* buf, size_t bytes);

/* ---- sampling --------------------------------------------------------------
 * Temperature / top-p (nucleus) sampling of one token per row, the sampling
 * of the ATLAS-OLMo-3-32B-Think-v4 model card ("Benchmarks", "Prompting guide
 * for Think models": temperature 0.6, top-p 0.95), with the uniform draws
 * given so that results are reproducible: p = softmax(logits / temperature);
 * tokens ordered by logit, largest first, equal logits by the lower index;
 * the nucleus is the shortest prefix of that order whose mass reaches top_p;
 * the token is the first of the nucleus whose cumulative mass, divided by the
 * nucleus mass, exceeds u[row].
 *   logits  fp32 [batch, vocab] (device, finite)
 *   u       fp32 [batch] (device), each in [0, 1)
 *   tokens  int32 [batch] (device), written
 *   ws      device scratch of w4a_sample_workspace_bytes() bytes (no zeroing
 *           needed), 16-byte aligned
 * temperature > 0, 0 < top_p <= 1; W4A_ERR_ARG / _SHAPE / _ALIGN /
 * _WORKSPACE on bad arguments.  Masses are float64 sums in a fixed order. */
W4A_API int w4a_sample_workspace_bytes(int batch, int vocab, size_t* bytes);
W4A_API int w4a_sample(const float* logits, int batch, int vocab, float temperature, float top_p,
               const float* u, int32_t* tokens, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream` and report the device error word of a workspace:
 * W4A_OK, W4A_ERR_TIMEOUT (a bounded wait ran out) or W4A_ERR_KERNEL (a
 * device-side check failed: a position outside the cache, a bad shape).
 * ws == NULL reads the fixed scratch of w4a_gemv_noalloc on the current
 * device instead (ws_bytes is then ignored; W4A_ERR_ARG before the first
 * w4a_gemv_noalloc call on that device).
 * Debugging: the environment variable W4A_BARRIER_WAIT_CYCLES, when set to a
 * positive number of SM cycles at a launch, bounds that launch's waits for
 * other CTAs (default ~2 s); a wait that runs out yields W4A_ERR_TIMEOUT
 * here, and the workspace must be zeroed again before its next use. */
W4A_API int w4a_check(const void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* W4A_H */
