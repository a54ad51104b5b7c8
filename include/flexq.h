/*
 * flexq: group-wise 4-bit OPT-style decoding on one B200 (sm_100a).
 *
 * C ABI of libflexq.so.  The operations follow the FlexGen pages:
 *   [WT]  "FlexGen: High-Throughput Generative Inference of Large Language
 *         Models with a Single GPU" walk-through (qingweiji.github.io):
 *         section "P/D阶段计算" (prefill and decode equations), section
 *         "内存占用分析" (biases, LayerNorms, tied embedding, KV cache shape
 *         [b, s, a, h/a] and peak size), section "Throughput And Latency"
 *         (generation throughput b n / t), section "Search Space" (GPU batch,
 *         block = GPU batch x GPU batches, column-wise zig-zag traversal).
 *   [RPT] "FlexGen研究学术报告" (fmread.com), section 三(C): group-wise
 *         asymmetric 4-bit quantization of weights and KV cache, groups of 64
 *         contiguous elements, dequantized to FP16 before compute.
 *   [SRV] survey notes (gumorming.cn), "Transformer-Styles LLMs" eqs. (1)-(3)
 *         (multi-head attention) and the word + positional embedding.
 *
 * Conventions (all entry points):
 * - Memory: the caller allocates every buffer; the library never allocates
 *   or frees device memory.  Pointers named *_dev are device pointers, *_host
 *   host pointers.  fp16 tensors are passed as void* and are row-major.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Calls enqueue work and return without synchronising, unless a
 *   comment says otherwise.
 * - Errors: argument errors are detected on the host before any launch and
 *   return FLEXQ_ERR_INVALID (or FLEXQ_ERR_WORKSPACE for a short workspace);
 *   a failed launch returns FLEXQ_ERR_CUDA.  flexq_last_error() returns the
 *   calling thread's last message.  Kernels never trap: a device-side wait
 *   that runs out, or a token id out of range, sets a device error word that
 *   flexq_device_status() reports.
 * - Aliasing: outputs never alias inputs unless stated.
 * - Shapes: h % 128 == 0, ffn % 128 == 0, d = h / heads in {64, 128}; linear
 *   weights are stored [N_out][K_in] (y = x W^T + b) with K_in % 64 == 0.
 */
#ifndef FLEXQ_H
#define FLEXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLEXQ_OK = 0,
  FLEXQ_ERR_INVALID = 1,     /* bad argument (null pointer, shape, alignment) */
  FLEXQ_ERR_CUDA = 2,        /* a CUDA call or kernel launch failed */
  FLEXQ_ERR_WORKSPACE = 3,   /* workspace pointer null or too small */
  FLEXQ_ERR_TIMEOUT = 4,     /* a device-side bounded wait gave up */
  FLEXQ_ERR_UNSUPPORTED = 5, /* valid request the library does not handle */
  FLEXQ_ERR_DEVICE = 6       /* a kernel reported a bad device-side input */
} flexq_status;

/* Message of the calling thread's last failed call ("" if none). */
const char* flexq_last_error(void);

/* ABI version of this header (major * 100 + minor). */
int flexq_version(void);

/* Synchronises `stream`, then reads and clears the device error word:
 * FLEXQ_OK, FLEXQ_ERR_TIMEOUT (a bounded wait ran out) or FLEXQ_ERR_DEVICE
 * (e.g. a token id outside [0, vocab)). */
flexq_status flexq_device_status(void* stream);

/* Deadline, in nanoseconds of device time, of every bounded wait inside the
 * kernels (default 2e9; 0 restores the default).  A test knob: a tiny value
 * makes pipelined kernels give up and report FLEXQ_ERR_TIMEOUT. */
flexq_status flexq_set_wait_limit_ns(uint64_t ns);

/* Programmatic dependent launch of the GEMMs and the decode attention (on by
 * default): such a kernel may start while its predecessor in the stream is
 * still running; it streams weights at once and waits for the predecessor
 * before touching anything earlier kernels write, so results are unchanged.
 * Returns the previous setting; 0 turns the overlap off (for measurement). */
int flexq_set_launch_overlap(int on);

/* ------------------------------------------------------------------------ */
/* Seeded synthetic inputs (not part of the method: workload generation).     */
/* Element i of stream (seed, tensor_id) is splitmix64's output function      */
/* (Steele, Lea and Flood 2014) applied to key + 0x9E3779B97F4A7C15 * (i + 1),  */
/* key = mix(seed * 0x9E3779B97F4A7C15 + tensor_id).                          */
/* ------------------------------------------------------------------------ */

/* out_dev: n fp16.  Element i (of start .. start+n-1) is
 * fp16_rn(fp32(sum of the hash's four 16-bit fields - 131070) * c + mean)
 * with c = fp32(sqrt(3) / 65536 * sigma): ~N(mean, sigma^2) bounded at
 * 3.46 sigma. */
flexq_status flexq_synth_normal_f16(void* out_dev, size_t n, uint64_t seed, uint64_t tensor_id,
                                    size_t start, float sigma, float mean, void* stream);

/* out_dev: n int32 ids, ((hash >> 32) * vocab) >> 32, uniform on [0, vocab). */
flexq_status flexq_synth_tokens(int32_t* out_dev, size_t n, uint64_t seed, uint64_t tensor_id,
                                size_t start, int32_t vocab, void* stream);

/* ------------------------------------------------------------------------ */
/* Group-wise asymmetric 4-bit codec [RPT 三(C)].                              */
/* ------------------------------------------------------------------------ */

/* x_dev: n fp16 (n % 64 == 0, |x| <= 2^15, finite), groups = runs of 64
 * contiguous elements.  Outputs: codes_dev n/2 bytes (byte j = code[2j] |
 * code[2j+1] << 4), min_dev and scale_dev n/64 fp16 each.  Per group:
 * scale = fp16_rn((max - min) / 15), min = fp16(min) (-0 stored as +0),
 * code = clamp(rint((x - min) / scale), 0, 15) (0 when scale == 0), all in
 * fp32 round-to-nearest-even without fused multiply-add: bit-exact by
 * contract.  All pointers 16-byte aligned. */
flexq_status flexq_quantize(const void* x_dev, size_t n, uint8_t* codes_dev, void* min_dev,
                            void* scale_dev, void* stream);

/* Inverse: out_dev n fp16, x_hat = fp16_rn(fp32(code * scale) + min). */
flexq_status flexq_dequantize(const uint8_t* codes_dev, const void* min_dev,
                              const void* scale_dev, size_t n, void* out_dev, void* stream);

/* Bytes of a 4-bit weight [n_out][k_in] in the GEMM's tiled layout:
 * ceil(n_out / 128) * (k_in / 64) tiles of 4608 bytes, each tile = 128 rows x
 * 32 bytes of codes (nibble order within every 32-bit word: element e in
 * nibble (e >> 1) + 4 (e & 1)) followed by 128 (min, scale) fp16 pairs;
 * tiles ordered [row tile][k block]; rows past n_out are zero. */
size_t flexq_packed_weight_bytes(int n_out, int k_in);

/* Canonical codec output (codes [n_out][k_in/2], min/scale [n_out][k_in/64])
 * -> tiled layout (a pure permutation; bit-exact). */
flexq_status flexq_pack_weight_q4(const uint8_t* codes_dev, const void* min_dev,
                                  const void* scale_dev, int n_out, int k_in, void* packed_dev,
                                  void* stream);

/* fp16 W [n_out][k_in] -> tiled 4-bit layout in one pass (same codes as
 * flexq_quantize followed by flexq_pack_weight_q4). */
flexq_status flexq_quantize_weight_q4(const void* w_dev, int n_out, int k_in, void* packed_dev,
                                      void* stream);

/* ------------------------------------------------------------------------ */
/* Layer building blocks.                                                     */
/* ------------------------------------------------------------------------ */

/* Y[m][n] = epilogue(X[m][k] W^T): the linear layers of [WT] "P/D阶段计算".
 * x_dev fp16 [m][ldx] (ldx % 8 == 0, 16-byte aligned); w_dev: packed 4-bit
 * (w_bits = 4) or fp16 [n][k] (w_bits = 16, n may be any size).  epilogue
 * flags: 1 = + bias[n], 2 = GELU (erf form) after the bias, 4 = + residual
 * [m][ld_res] last, 8 = write fp32 (alone).  y_dev fp16 (or fp32) [m][ldy].
 * ws: fp32 partial output tiles when K is shared out across CTAs (small
 * grids) plus two counters per tile (contributors arrived, partials
 * published; zeroed on the stream by the call); size from
 * flexq_linear_workspace with the same force_splits (0 means none needed).
 * force_splits = 0 lets the library choose (whole tiles per SM when there are
 * many, equal shares of all k-blocks per SM when there are few); s > 1 cuts
 * every tile's K into s parts (tests); 1 forbids splitting K.  A split tile is
 * summed in a fixed contributor order, so results do not depend on timing. */
size_t flexq_linear_workspace(int m, int n, int k, int w_bits, int force_splits);
flexq_status flexq_linear(const void* x_dev, int ldx, const void* w_dev, int w_bits, int m, int n,
                          int k, const void* bias_dev, const void* residual_dev, int ld_res,
                          int epilogue, void* y_dev, int ldy, void* ws_dev, size_t ws_bytes,
                          int force_splits, void* stream);

/* flexq_linear for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is a library-service entry point.  A caller such
 * as a plug-in that a host framework hands only its input and output buffers
 * (the framework's pool owning the rest of device memory), or a loop that
 * must not pay for cudaMalloc/cudaFree, has no workspace to offer; here the
 * K-split partial sums live in an 8 MiB array compiled into the library
 * (reserved on a GPU from the library's first use there until exit).
 * Arguments and results as flexq_linear, without ws; the output is bit for
 * bit that of flexq_linear with the same force_splits.  Limit: the K-split
 * scratch the shape needs (flexq_linear_workspace with the same force_splits)
 * must fit in 8 MiB; larger requests return FLEXQ_ERR_INVALID without
 * launching.  The first call on a device looks up the array's address for
 * that device (kept once found, retried after a failure): make it before any
 * stream capture.  All calls share the array (each clears what it uses
 * first); calls that overlap on the GPU race on it, so serialise them.
 * Allocates nothing. */
flexq_status flexq_linear_static_scratch(const void* x_dev, int ldx, const void* w_dev, int w_bits,
                                         int m, int n, int k, const void* bias_dev,
                                         const void* residual_dev, int ld_res, int epilogue,
                                         void* y_dev, int ldy, int force_splits, void* stream);

/* LayerNorm of rows [rows][h] (biased variance, fp32 statistics). */
flexq_status flexq_layernorm(const void* x_dev, int ldx, const void* gamma_dev,
                             const void* beta_dev, void* y_dev, int ldy, int rows, int h,
                             float eps, void* stream);

/* ------------------------------------------------------------------------ */
/* Model description.                                                         */
/* ------------------------------------------------------------------------ */

typedef struct {
  int h;        /* hidden size, % 128 == 0 */
  int heads;    /* attention heads; d = h / heads in {64, 128} */
  int ffn;      /* MLP width (ih), % 128 == 0 */
  int w_bits;   /* 4 (packed tiled weights) or 16 (fp16 [N_out][K_in]) */
  int kv_bits;  /* 4 (group-wise codes) or 16 (fp16) */
  float ln_eps; /* LayerNorm epsilon (1e-5) */
  int attn_topk_permille; /* 0: dense decode attention; 1..1000: top-k sparse
                             decode attention keeping ceil(L * permille / 1000)
                             keys (100 = the pages' top 10 %); 4-bit KV only */
  int prefill_kv_cache;   /* 0: prefill attention uses the pass's own fp16 K/V;
                             1: it reads them back from the cache as stored
                             (4-bit: the dequantized codes, "FlexGen研究学术报告"
                             section 三(C): the cache is kept compressed and
                             dequantized before compute) */
} flexq_config;

/* One decoder layer's parameters (device pointers).  Linear weights [N_out]
 * [K_in]: w_qkv [3h][h] (rows: Q heads, then K heads, then V heads, head j
 * at rows j*d .. j*d+d-1), w_o [h][h], w_fc1 [ffn][h], w_fc2 [h][ffn];
 * packed per flexq_packed_weight_bytes when w_bits == 4.  Biases and
 * LayerNorm parameters fp16: b_qkv [3h], b_o [h], b_fc1 [ffn], b_fc2 [h],
 * ln*_g / ln*_b [h]. */
typedef struct {
  const void *w_qkv, *w_o, *w_fc1, *w_fc2;
  const void *b_qkv, *b_o, *b_fc1, *b_fc2;
  const void *ln1_g, *ln1_b, *ln2_g, *ln2_b;
} flexq_layer;

/* One layer's KV cache for b sequences, max_len slots each ([WT]
 * "内存占用分析": K and V of shape [b, s, a, h/a], stored here head-major).
 * kv_bits == 4: k = codes [b][heads][max_len][d/2] (canonical nibble order);
 * v = codes in 32-bit words [b][heads][L8/8][d] with L8 = max_len rounded up
 * to a multiple of 8, token-interleaved: nibble k (bits 4k..4k+3) of word
 * (block, e) is the code of token 8*block + k at dimension e; k_meta, v_meta
 * = (min, scale) fp16 pairs [b][heads][max_len][d/64].  kv_bits == 16: k, v =
 * fp16 [b][heads][max_len][d]; metas NULL.  A GPU batch of sequences i0.. is
 * the same layout with pointers advanced by i0 rows of heads * max_len slots
 * (heads * L8 for 4-bit V). */
typedef struct {
  void *k, *v, *k_meta, *v_meta;
  int b, max_len;
} flexq_kv;

/* Bytes of K (codes or values) + V + their metadata for one layer. */
size_t flexq_kv_bytes(const flexq_config* cfg, int b, int max_len);

/* Quantize-on-append, the decode update x_K <- Concat(x_K, t W_K) (and V)
 * of [WT] "P/D阶段计算", and the prefill's bulk write.  k_dev, v_dev: fp16
 * rows [b * ntok][ld] (row i*ntok + t, head j at columns j*d ..) written to
 * slots pos0 .. pos0+ntok-1.  In 4-bit mode each (sequence, head, token)
 * row is quantized exactly as flexq_quantize would quantize it. */
flexq_status flexq_kv_append(const flexq_config* cfg, const flexq_kv* kv, const void* k_dev,
                             const void* v_dev, int ld, int b, int pos0, int ntok, void* stream);

/* Decode attention: out[i][j*d ..] = softmax(q_ij K_ij^T / sqrt(d)) V_ij over
 * slots 0..len-1 of the cache (dequantized in 4-bit mode).  q_dev fp16
 * [b][ldq] (head j at columns j*d), out_dev fp16 [b][ldo].  In 4-bit mode the
 * dequantization is folded into the sums (scale * sum q*code + min * sum q),
 * which are formed with integer dot products: q as 15-bit fixed point per
 * head row and the softmax weights as 16-bit fixed point per 8-token block
 * and group (held to the layer tolerance by the parity tests). */
flexq_status flexq_attention_decode(const flexq_config* cfg, const flexq_kv* kv, const void* q_dev,
                                    int ldq, int b, int len, void* out_dev, int ldo, void* stream);

/* Top-k sparse decode attention over a 4-bit cache ("FlexGen研究学术报告"
 * section 三(C): only the top 10 % of the KV cache by attention value is
 * loaded).  Per (sequence, head): scores s_t = q k_hat_t / sqrt(d) over all
 * len slots, p = softmax(s) over all of them, T = the k slots with the
 * largest scores (a lower slot wins a tie), out = sum_{t in T} p_t v_hat_t
 * (full-softmax weights, not renormalised over T; k = len is dense
 * attention).  K is read in full; V and its (min, scale) only for the 8-token
 * blocks that hold a kept slot.  1 <= k <= len <= 16384.  idx_dev (may be
 * NULL): int32 [b][heads][k], the kept slots in ascending order.  Scores,
 * weights and sums are formed as in flexq_attention_decode. */
flexq_status flexq_attention_decode_topk(const flexq_config* cfg, const flexq_kv* kv, const void* q_dev, int ldq,
                                         int b, int len, int k, void* out_dev, int ldo, int32_t* idx_dev,
                                         void* stream);

/* Causal prefill attention on fp16 Q/K/V: qkv_dev [b*s][ldqkv] with Q, K, V
 * at column offsets 0, h, 2h; out_dev [b*s][ldo]. */
flexq_status flexq_attention_prefill(const flexq_config* cfg, const void* qkv_dev, int ldqkv,
                                     int b, int s, void* out_dev, int ldo, void* stream);

/* Causal prefill attention whose keys and values are read back from the
 * cache: q_dev fp16 [b*s][ldq] (Q of sequence i, token t at row i*s + t),
 * query t attends over cache slots pos0 .. pos0 + t (stored by
 * flexq_kv_append; 4-bit codes are dequantized as the codec does,
 * fp16(fp32(code * scale) + min)).  pos0 + s <= kv->max_len; in 4-bit mode
 * pos0 % 8 == 0.  out_dev fp16 [b*s][ldo]. */
flexq_status flexq_attention_prefill_cache(const flexq_config* cfg, const flexq_kv* kv, const void* q_dev,
                                           int ldq, int b, int s, int pos0, void* out_dev, int ldo,
                                           void* stream);

/* ------------------------------------------------------------------------ */
/* Layer steps ([WT] "P/D阶段计算", pre-LN OPT block).                          */
/*   u = LN1(x); [Q|K|V] = u W_qkv^T + b_qkv; o = attention;                   */
/*   x_out = o W_o^T + b_o + x; v = LN2(x_out);                                */
/*   y = GELU(v W_1^T + b_1) W_2^T + b_2 + x_out.                              */
/* ------------------------------------------------------------------------ */

/* Workspace bytes for a prefill over `rows` = b*s tokens (mode 0) or a decode
 * over `rows` = b sequences (mode 1). */
size_t flexq_layer_workspace(const flexq_config* cfg, int rows, int mode);

/* Prefill of one layer over b sequences of s tokens: x_dev, y_dev fp16
 * [b*s][h] (distinct).  Writes cache slots 0..s-1 (quantized in 4-bit
 * mode); attention uses the pass's own fp16 K/V, or with
 * cfg->prefill_kv_cache reads them back from those slots. */
flexq_status flexq_layer_prefill(const flexq_config* cfg, const flexq_layer* layer,
                                 const void* x_dev, void* y_dev, const flexq_kv* kv, int b, int s,
                                 void* ws_dev, size_t ws_bytes, void* stream);

/* Decode of one layer for the token at position pos of b sequences: t_dev,
 * y_dev fp16 [b][h] (distinct).  Appends this token's K/V to slot pos, then
 * attends over slots 0..pos read back from the cache.  For b <= 256 the
 * append needs no launch of its own: a 4-bit cache is appended by the
 * decode attention kernel (the warps of each (sequence, head) CTA quantize
 * the token's K/V rows, one warp per 64-element group, the same codes
 * flexq_kv_append gives those fp16 rows, before the CTA reads the cache;
 * when the attention splits each head's cache over several CTAs the append
 * is a launch of its own), an fp16 cache by the Q/K/V projection's
 * epilogue; LN2 runs inside the output projection (a
 * cooperative launch whose CTAs normalise the finished rows after a
 * grid-wide barrier); decode attention splits each head's cache over several
 * CTAs when b * heads CTAs would not fill the GPU. */
flexq_status flexq_layer_decode(const flexq_config* cfg, const flexq_layer* layer,
                                const void* t_dev, void* y_dev, const flexq_kv* kv, int b,
                                int pos, void* ws_dev, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* Generation over a block ([WT] "Search Space" and "Throughput And Latency"). */
/* ------------------------------------------------------------------------ */

typedef struct {
  flexq_config cfg;
  int layers;
  int vocab;
  int max_pos;                /* rows of pos_embed */
  const flexq_layer* layer;   /* host array [layers] of device-pointer sets */
  const flexq_kv* kv;         /* host array [layers]; each b x max_len >= s+n */
  const void* embed;          /* word embedding E [vocab][h], also the tied LM head
                                 ([WT] "内存占用分析"): fp16, or (embed_bits 4)
                                 group-wise 4-bit in the tiled layout of
                                 flexq_packed_weight_bytes(vocab, h), groups along
                                 h; the lookups then read E's dequantized rows
                                 fp16_rn(fp32(code * scale) + min) and the LM head
                                 is the dequant-fused GEMM */
  const void* pos_embed;      /* fp16 P [max_pos][h] */
  const void* lnf_g;          /* final LayerNorm, fp16 [h] */
  const void* lnf_b;
  int embed_bits;             /* 16 or 4: the format of embed */
} flexq_model;

typedef struct {
  float prefill_ms; /* device time of embedding + prefill + first token */
  float decode_ms;  /* device time of the n-1 decode steps */
} flexq_timing;

/* Workspace bytes for flexq_generate (and its two halves below). */
size_t flexq_generate_workspace(const flexq_model* model, int b, int s, int gpu_batch);

/* The prefill column of flexq_generate alone: embeds the prompts, runs every
 * layer over every GPU batch (filling cache slots 0..s-1) and writes token 1
 * to out_dev[i*n + 0]. */
flexq_status flexq_generate_prefill(const flexq_model* model, const int32_t* prompt_dev, int b, int s,
                                    int n, int gpu_batch, int32_t* out_dev, void* ws_dev,
                                    size_t ws_bytes, void* stream);

/* The n-1 decode columns of flexq_generate alone: column j reads token
 * out_dev[i*n + j-1] at position s+j-1, appends its K/V to slot s+j-1 of every
 * layer and writes out_dev[i*n + j].  Needs the caches a prefill over the same
 * b sequences left (slots 0..s-1); re-running it rewrites slots s..s+n-2.
 * With gpu_batch <= 256 each column is fused as in flexq_layer_decode, and
 * further: the embedding kernel applies layer 0's LN1, and every layer's FC2
 * kernel LayerNorms its output with the next layer's LN1 (the last layer's
 * with the final LayerNorm), so a layer is five kernels (QKV, attention with
 * the append, output projection + LN, FC1 + GELU, FC2 + LN).  The split-tile
 * counters in the workspace are zeroed once per call and every kernel leaves
 * them zero; a kernel that gives up a bounded wait (FLEXQ_ERR_TIMEOUT) may
 * leave them dirty, so results of the rest of that call are undefined. */
flexq_status flexq_generate_decode(const flexq_model* model, int b, int s, int n, int gpu_batch,
                                   int32_t* out_dev, void* ws_dev, size_t ws_bytes, void* stream);

/* Greedy generation for a block of b sequences (prompt length s, n output
 * tokens) processed as GPU batches of gpu_batch sequences (b % gpu_batch ==
 * 0).  Zig-zag order: for each token column, for each layer, for each GPU
 * batch; the prefill column emits token 1 from the last prompt position, each
 * of the n-1 decode columns emits one more (lowest index among equal
 * logits).  prompt_dev int32 [b][s], out_dev int32 [b][n].  With timing !=
 * NULL the call synchronises the stream and fills it. */
flexq_status flexq_generate(const flexq_model* model, const int32_t* prompt_dev, int b, int s,
                            int n, int gpu_batch, int32_t* out_dev, void* ws_dev, size_t ws_bytes,
                            flexq_timing* timing, void* stream);

/* ------------------------------------------------------------------------ */
/* Offloaded weights ([WT] "Search Space", "Cost Model"; [RPT] 三(A)/(B)).     */
/* ------------------------------------------------------------------------ */

/* Bytes of one device slot holding a layer's four weight matrices
 * (qkv, o, fc1, fc2 in that order, each 256-byte aligned). */
size_t flexq_offload_slot_bytes(const flexq_config* cfg);

/* flexq_generate with the layer weights resident in host memory: every
 * model->layer[i].w_qkv / w_o / w_fc1 / w_fc2 points into page-locked host
 * memory (checked; FLEXQ_ERR_INVALID otherwise), every other pointer of the
 * model is device memory.  Each column of the zig-zag block (the prefill,
 * then each decode step) walks the layers in order and runs every GPU batch
 * of the block on one layer before the next, so each layer's weights cross
 * the host link once per column: they are copied into one of two device
 * slots (slots_dev: 2 * flexq_offload_slot_bytes bytes, caller-owned) on
 * copy_stream (a stream other than `stream`) two layer steps ahead of the
 * compute on `stream`, overlapping the copy of the next layer with this
 * layer's compute.  Results equal flexq_generate's on the same weights.
 * The call returns once all work is enqueued (with timing, once it ends). */
flexq_status flexq_generate_offload(const flexq_model* model, void* slots_dev, size_t slots_bytes,
                                    void* copy_stream, const int32_t* prompt_dev, int b, int s, int n,
                                    int gpu_batch, int32_t* out_dev, void* ws_dev, size_t ws_bytes,
                                    flexq_timing* timing, void* stream);

typedef struct {
  double h2d_gbps;      /* host-to-device copy rate (GB/s), measured by the caller */
  double hbm_gbps;      /* device memory rate (GB/s) */
  double tensor_tflops; /* dense fp16 tensor rate (TFLOP/s) */
  double device_bytes;  /* device memory the generation may use */
} flexq_hw;

typedef struct {
  int gpu_batch;               /* sequences per GPU batch */
  int num_batches;             /* GPU batches per block: b = gpu_batch * num_batches */
  double decode_tokens_per_s;  /* modelled decode throughput of the choice */
  double column_io_s;          /* modelled weight-copy time of one decode column */
  double column_compute_s;     /* modelled compute time of one decode column */
  double device_bytes;         /* modelled device memory of the choice */
} flexq_offload_choice;

/* Cost model of the offloaded block schedule: per decode column and layer,
 * T = max(weight bytes / h2d, num_batches * t_batch) with t_batch the
 * roofline time of one GPU batch's layer step at the mean KV length s + n/2
 * (weights and KV at hbm_gbps, 2 * tokens * weights flops at tensor_tflops),
 * plus the LM head once per column; throughput = b / column time.  Device
 * memory = two weight slots, E, P, biases and LayerNorms, every layer's KV
 * cache for b sequences of s + n slots and flexq_generate_workspace.
 * Enumerates gpu_batch = 256, 240, .., 16 and num_batches = 1, 2, .. while
 * the memory fits and b <= max_block, and returns the highest modelled
 * throughput; a later candidate replaces the best only when it is more than
 * 0.1 % faster, so among near-equal choices the larger GPU batch (the more
 * efficient GEMMs) and then the smaller block win. */
flexq_status flexq_offload_plan(const flexq_model* model, int s, int n, const flexq_hw* hw, int max_block,
                                flexq_offload_choice* out);

/* ------------------------------------------------------------------------ */
/* Instrumentation (measurement only; not part of the method).                */
/* ------------------------------------------------------------------------ */

/* Number of kernels this library has launched in the process so far. */
uint64_t flexq_launch_count(void);

/* Kernel kinds reported by the profiler. */
typedef enum {
  FLEXQ_K_LAYERNORM = 0,
  FLEXQ_K_QKV = 1,
  FLEXQ_K_KV_APPEND = 2,
  FLEXQ_K_ATTN_PREFILL = 3,
  FLEXQ_K_ATTN_DECODE = 4,
  FLEXQ_K_OUT_PROJ = 5,
  FLEXQ_K_FC1 = 6,
  FLEXQ_K_FC2 = 7,
  FLEXQ_K_EMBED = 8,
  FLEXQ_K_LM_HEAD = 9,
  FLEXQ_K_ARGMAX = 10,
  FLEXQ_K_COUNT = 11
} flexq_kernel_kind;

/* Between start and stop, every kernel the layer steps and the generator
 * launch is bracketed by two CUDA events on its stream (adds a little time;
 * one host thread at a time).  stop synchronises `stream` and writes, per
 * kind, the summed device milliseconds and the number of bracketed calls
 * (an unfused linear layer's call also holds the memset of its split-tile
 * counters; a fused decode kernel counts under the kind of the kernel it
 * runs in: a 4-bit decode append under ATTN_DECODE (an fp16 one under QKV),
 * LN2 under OUT_PROJ, the next LN1 or the final LayerNorm under FC2, layer
 * 0's LN1 under EMBED). */
flexq_status flexq_profile_start(void);
flexq_status flexq_profile_stop(void* stream, float* total_ms /* [FLEXQ_K_COUNT] */,
                                int* calls /* [FLEXQ_K_COUNT] */);

#ifdef __cplusplus
}
#endif

#endif /* FLEXQ_H */
