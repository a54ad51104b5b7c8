// Internal launch interface between the C ABI (flexq.cu) and the kernels.
// Every launcher enqueues on `stream` and returns the launch status.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace flexq {

// Bytes of one packed 4-bit weight tile: 128 rows x 64 codes (4096 B) followed
// by 128 (min, scale) fp16 pairs (512 B).  Tiles are stored [n_tile][k_block].
constexpr int kTileRows = 128;
constexpr int kGroup = 64;
constexpr int kTileCodeBytes = kTileRows * kGroup / 2;
constexpr int kTileMetaBytes = kTileRows * 4;
constexpr int kTileBytes = kTileCodeBytes + kTileMetaBytes;

struct Runtime {
  uint64_t wait_limit_ns;  // deadline of every bounded device wait
  uint32_t* err;           // device error word
  int num_sms;
  int pdl;                 // launch GEMMs and decode attention with programmatic dependent launch
};

const Runtime& runtime();

// Counts one kernel launch of this library and returns the launch status.
cudaError_t launched();

// Launches `kernel` on `s`, with the programmatic stream-serialization
// attribute when runtime().pdl (the kernel must pdl_wait() before touching
// memory earlier kernels write), and counts it.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = runtime().pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
  if (e != cudaSuccess) return e;
  return launched();
}

// Sets the calling thread's message returned by flexq_last_error().
void set_last_error(const char* msg);

// synthetic inputs
cudaError_t launch_synth_normal(__half* out, size_t n, uint64_t key, size_t start, float scale,
                                float mean, cudaStream_t s);
cudaError_t launch_synth_tokens(int32_t* out, size_t n, uint64_t key, size_t start, int vocab,
                                cudaStream_t s);

// codec
cudaError_t launch_quantize(const __half* x, size_t n, uint8_t* codes, __half* mn, __half* sc,
                            cudaStream_t s);
cudaError_t launch_dequantize(const uint8_t* codes, const __half* mn, const __half* sc, size_t n,
                              __half* out, cudaStream_t s);
cudaError_t launch_pack_weight(const uint8_t* codes, const __half* mn, const __half* sc, int n_out,
                               int k_in, uint8_t* packed, cudaStream_t s);
cudaError_t launch_quantize_weight(const __half* w, int n_out, int k_in, uint8_t* packed,
                                   cudaStream_t s);

// Slots per (sequence, head) of the token-interleaved 4-bit V codes: max_len
// rounded up to whole blocks of 8 tokens.
__host__ __device__ inline int kv_pad_len(int max_len) { return (max_len + 7) & ~7; }

// KV cache append (quantize on append in 4-bit mode)
struct KvView {
  void* k;        // 4-bit: codes [b][a][L][d/2]; 16-bit: fp16 [b][a][L][d]
  void* v;
  void* k_meta;   // 4-bit: (min, scale) fp16 pairs [b][a][L][d/64]
  void* v_meta;
  int max_len;
};
cudaError_t launch_kv_append(const __half* k_src, const __half* v_src, int ld_src, int b, int ntok,
                             int heads, int d, int kv_bits, const KvView& kv, int pos0,
                             cudaStream_t s);

// LayerNorm over rows of width h (fp16 in/out, fp32 statistics)
cudaError_t launch_layernorm(const __half* x, int ldx, const __half* g, const __half* bta,
                             __half* y, int ldy, int rows, int h, float eps, cudaStream_t s);
// Bytes of the split-tile counters a linear layer of this shape uses (0 when
// it splits no tile), and of its partial tiles alone.
size_t linear_counter_bytes(int m, int n, int k, int w_bits, int force_splits);
size_t linear_partial_bytes(int m, int n, int k, int w_bits, int force_splits);

// GEMM: Y[m][n] = epilogue(X[m][k] . W[n][k]^T)
enum Epilogue : int {
  EPI_BIAS = 1,       // + bias[n]
  EPI_GELU = 2,       // GELU (exact erf form) after the bias
  EPI_RESIDUAL = 4,   // + residual[m][n] last
  EPI_F32_OUT = 8,    // write fp32 (no bias/act/residual allowed)
};
// Decode-step fusions of a linear layer (one token per sequence, m rows):
// KvFuse makes the QKV projection store its K and V columns straight into
// the fp16 cache slot `pos` of each of the m sequences instead of its output
// (a 4-bit cache is appended by the decode attention, see AppendRow);
// LnFuse makes the layer LayerNorm its finished rows [m][n] into `y` after a
// grid-wide barrier (the launch is cooperative; `sync` = two ints of device
// memory that are zero on entry and left zero).
struct KvFuse {
  __half* k;  // fp16 caches in the KvView layout of the m sequences
  __half* v;
  int h, heads, d, max_len, pos;
};
struct LnFuse {
  const __half* g;
  const __half* b;
  __half* y;
  int ldy;
  float eps;
  int* sync;
};
struct LinearArgs {
  const __half* x; int ldx;       // activations [m][k]
  const void* w; int w_bits;      // packed 4-bit tiles, or fp16 [n][k]
  int m, n, k;
  const __half* bias;
  const __half* residual; int ld_res;
  void* y; int ldy;
  int epi;
  int force_splits;               // 0 = automatic
  int force_tok_tile;             // 0 = automatic
  const KvFuse* kv;               // decode QKV: quantize K/V into the cache
  const LnFuse* ln;               // decode out-proj / FC2: LayerNorm of the output rows
  // Split-tile counters that are zero on entry (and left zero by the
  // kernel), linear_counter_bytes of them; ws then holds only the partial
  // tiles.  NULL: the counters follow the partials in ws and are zeroed on
  // the stream by the launch.
  int* counters;
};
// Largest m the fused decode variants take (one token tile).
constexpr int kFuseMaxRows = 256;
size_t linear_workspace_bytes(int m, int n, int k, int w_bits, int force_splits);
cudaError_t launch_linear(const LinearArgs& a, void* ws, size_t ws_bytes, cudaStream_t s);

// attention
// The decode token's fp16 K and V rows ([b][ld], head j at columns j*d),
// which the decode attention quantizes into cache slot `pos` before reading
// the cache (4-bit caches; pos < 0: nothing to append).
struct AppendRow {
  const __half* k;
  const __half* v;
  int ld;
  int pos;
};
constexpr AppendRow kNoAppend = {nullptr, nullptr, 0, -1};

// Decode attention.  With part/ctr: when b * heads CTAs cannot fill the
// GPU, each (sequence, head) is split over several CTAs
// along the cache, partial results go to `part`
// (attn_decode_partial_bytes) and the last split of each merges them;
// ctr = b * heads ints, zero on entry and left zero.
cudaError_t launch_attn_decode(const __half* q, int ldq, const KvView& kv, int b, int heads, int d,
                               int kv_bits, int len, __half* out, int ldo, float* part, int* ctr,
                               const AppendRow& app, cudaStream_t s);
int attn_decode_splits(int b, int heads, int len);
// Top-k sparse decode attention over a 4-bit cache: kk keys kept per
// (sequence, head); idx (optional) receives the kept slots [b][heads][kk] in
// ascending order.
cudaError_t launch_attn_topk(const __half* q, int ldq, const KvView& kv, int b, int heads, int d, int len, int kk,
                             __half* out, int ldo, int32_t* idx, const AppendRow& app, cudaStream_t s);
// ceil(len * permille / 1000), clamped to 1..len.
inline int topk_count(int len, int permille) {
  const long long k = (static_cast<long long>(len) * permille + 999) / 1000;
  return static_cast<int>(k < 1 ? 1 : (k > len ? len : k));
}
size_t attn_decode_partial_bytes(int b, int heads, int d);
cudaError_t launch_attn_prefill(const __half* qkv, int ldqkv, int b, int seq, int heads, int d,
                                __half* out, int ldo, cudaStream_t s);
// Causal prefill attention of `seq` queries per sequence (q rows i * seq + t,
// stride ldq) over cache slots pos0 .. pos0 + seq - 1 read back as stored.
cudaError_t launch_attn_prefill_cache(const __half* q, int ldq, const KvView& kv, int kv_bits, int pos0, int b,
                                      int seq, int heads, int d, __half* out, int ldo, cudaStream_t s);

// embedding and greedy choice
// E: fp16 [vocab][h] (embed_bits 16) or the 4-bit tiled layout (embed_bits 4).
cudaError_t launch_embed(const int32_t* tok, int ld_tok, int b, int ntok, const void* E, int embed_bits,
                         int vocab, const __half* P, int pos0, int h, __half* x, cudaStream_t s);
// Decode embedding of one token per sequence fused with the first layer's
// LN1: x = E[tok] + P[pos] (fp16) and u = LN(x) (gamma g, beta bta).
cudaError_t launch_embed_ln(const int32_t* tok, int ld_tok, int b, const void* E, int embed_bits, int vocab,
                            const __half* P, int pos, int h, __half* x, const __half* g,
                            const __half* bta, float eps, __half* u, cudaStream_t s);
cudaError_t launch_argmax(const float* logits, int rows, int vocab, int ld, int32_t* out,
                          int ld_out, cudaStream_t s);

}  // namespace flexq
