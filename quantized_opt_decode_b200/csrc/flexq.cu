// C ABI of libflexq: argument validation, workspace carving, and the
// composition of the kernels into the layer steps and the block generator.
// The operations and their sources are documented in include/flexq.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "flexq.h"
#include "kernels.h"

namespace flexq {

__device__ uint32_t g_device_error;

namespace {

thread_local std::string g_last_error;
uint64_t g_wait_limit_ns = 2000000000ull;
int g_pdl = 1;
constexpr int kMaxDevices = 64;
Runtime g_rt[kMaxDevices];
std::once_flag g_rt_once[kMaxDevices];
std::atomic<uint64_t> g_launches{0};

// Optional per-kernel timing: while on, every kernel of the layer steps and
// the generator is bracketed by two CUDA events on its stream (one host
// thread at a time).
struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  std::vector<std::pair<int, size_t>> marks;  // (kind, index of the start event)
};
Profiler g_prof;

struct ProfScope {
  int kind;
  cudaStream_t s;
  size_t idx = 0;
  bool on;
  ProfScope(int k, cudaStream_t st) : kind(k), s(st), on(g_prof.on) {
    if (!on) return;
    while (g_prof.pool.size() < g_prof.used + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) {
        on = false;
        return;
      }
      g_prof.pool.push_back(e);
    }
    idx = g_prof.used;
    g_prof.used += 2;
    cudaEventRecord(g_prof.pool[idx], s);
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(g_prof.pool[idx + 1], s);
    g_prof.marks.emplace_back(kind, idx);
  }
};

flexq_status fail(flexq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

flexq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FLEXQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define FQ_CHECK(cond, ...)                                \
  do {                                                     \
    if (!(cond)) return fail(FLEXQ_ERR_INVALID, __VA_ARGS__); \
  } while (0)

#define FQ_CUDA(expr, what)                      \
  do {                                           \
    cudaError_t e_ = (expr);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

#define FQ_TRY(expr)                  \
  do {                                \
    flexq_status st_ = (expr);        \
    if (st_ != FLEXQ_OK) return st_;  \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

flexq_status check_config(const flexq_config* c) {
  FQ_CHECK(c != nullptr, "config is NULL");
  FQ_CHECK(c->h > 0 && c->h % 128 == 0, "h must be a positive multiple of 128 (got %d)", c->h);
  FQ_CHECK(c->heads > 0 && c->h % c->heads == 0, "heads must divide h");
  const int d = c->h / c->heads;
  FQ_CHECK(d == 64 || d == 128, "head dim h/heads must be 64 or 128 (got %d)", d);
  FQ_CHECK(c->ffn > 0 && c->ffn % 128 == 0, "ffn must be a positive multiple of 128");
  FQ_CHECK(c->h <= 12288, "h above 12288 is not supported");
  FQ_CHECK(c->w_bits == 4 || c->w_bits == 16, "w_bits must be 4 or 16");
  FQ_CHECK(c->kv_bits == 4 || c->kv_bits == 16, "kv_bits must be 4 or 16");
  FQ_CHECK(c->ln_eps > 0.f, "ln_eps must be positive");
  FQ_CHECK(c->attn_topk_permille >= 0 && c->attn_topk_permille <= 1000, "attn_topk_permille must be in 0..1000");
  FQ_CHECK(c->attn_topk_permille == 0 || c->kv_bits == 4, "top-k sparse attention needs the 4-bit KV cache");
  FQ_CHECK(c->prefill_kv_cache == 0 || c->prefill_kv_cache == 1, "prefill_kv_cache must be 0 or 1");
  return FLEXQ_OK;
}

flexq_status check_kv(const flexq_config* c, const flexq_kv* kv, int b) {
  FQ_CHECK(kv != nullptr, "kv is NULL");
  FQ_CHECK(kv->k && kv->v, "kv->k / kv->v is NULL");
  FQ_CHECK(c->kv_bits == 16 || (kv->k_meta && kv->v_meta), "4-bit KV needs k_meta and v_meta");
  FQ_CHECK(kv->b >= b, "kv holds %d sequences, call needs %d", kv->b, b);
  FQ_CHECK(kv->max_len > 0, "kv->max_len must be positive");
  FQ_CHECK(aligned16(kv->k) && aligned16(kv->v), "KV buffers must be 16-byte aligned");
  FQ_CHECK(c->kv_bits == 16 || ((reinterpret_cast<uintptr_t>(kv->k_meta) & 3) == 0 &&
                                (reinterpret_cast<uintptr_t>(kv->v_meta) & 3) == 0),
           "KV metadata must be 4-byte aligned");
  return FLEXQ_OK;
}

flexq_status check_layer(const flexq_config* c, const flexq_layer* L) {
  FQ_CHECK(L != nullptr, "layer is NULL");
  FQ_CHECK(L->w_qkv && L->w_o && L->w_fc1 && L->w_fc2, "layer weight pointer is NULL");
  FQ_CHECK(L->b_qkv && L->b_o && L->b_fc1 && L->b_fc2, "layer bias pointer is NULL");
  FQ_CHECK(L->ln1_g && L->ln1_b && L->ln2_g && L->ln2_b, "layer LayerNorm pointer is NULL");
  FQ_CHECK(aligned16(L->ln1_g) && aligned16(L->ln1_b) && aligned16(L->ln2_g) && aligned16(L->ln2_b),
           "LayerNorm parameters must be 16-byte aligned");
  FQ_CHECK(aligned16(L->w_qkv) && aligned16(L->w_o) && aligned16(L->w_fc1) && aligned16(L->w_fc2),
           "weights must be 16-byte aligned");
  (void)c;
  return FLEXQ_OK;
}

KvView view_of(const flexq_config* c, const flexq_kv* kv, int seq0) {
  const int d = c->h / c->heads;
  const size_t slots = static_cast<size_t>(seq0) * c->heads * kv->max_len;
  KvView v{};
  v.max_len = kv->max_len;
  if (c->kv_bits == 4) {
    v.k = static_cast<uint8_t*>(kv->k) + slots * (d / 2);
    v.v = static_cast<uint8_t*>(kv->v) +
          static_cast<size_t>(seq0) * c->heads * kv_pad_len(kv->max_len) * (d / 2);
    v.k_meta = static_cast<uint8_t*>(kv->k_meta) + slots * (d / 64) * 4;
    v.v_meta = static_cast<uint8_t*>(kv->v_meta) + slots * (d / 64) * 4;
  } else {
    v.k = static_cast<uint8_t*>(kv->k) + slots * d * 2;
    v.v = static_cast<uint8_t*>(kv->v) + slots * d * 2;
  }
  return v;
}

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace layout of one layer step over M rows.  ctr is a region that is
// zeroed once per call and that the fused decode kernels leave zero: its
// first 256 bytes hold the grid-barrier words, then the split-tile counters.
struct LayerWs {
  __half *u, *qkv, *xo, *g, *o, *v;
  float* acc;
  size_t acc_bytes;
  float* attn_part;  // split decode attention partials
  int* ctr;          // zeroed region: grid-barrier words | tile counters | attention counters
  size_t ctr_bytes;
  int* tile_ctr;
  int* attn_ctr;
  size_t total;
};

constexpr size_t kSyncBytes = 256;

LayerWs layer_ws_layout(const flexq_config* c, int M, uint8_t* base) {
  LayerWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const size_t h = c->h, f = c->ffn;
  w.u = reinterpret_cast<__half*>(take(M * h * 2));
  w.qkv = reinterpret_cast<__half*>(take(M * 3 * h * 2));
  w.xo = reinterpret_cast<__half*>(take(M * h * 2));
  w.g = reinterpret_cast<__half*>(take(M * f * 2));
  w.o = reinterpret_cast<__half*>(take(M * h * 2));
  w.v = reinterpret_cast<__half*>(take(M * h * 2));
  const int shapes[4][2] = {{3 * c->h, c->h}, {c->h, c->h}, {c->ffn, c->h}, {c->h, c->ffn}};
  size_t acc = 0, ctr = 0;
  for (const auto& sh : shapes) {
    acc = std::max(acc, linear_workspace_bytes(M, sh[0], sh[1], c->w_bits, 0));
    ctr = std::max(ctr, linear_counter_bytes(M, sh[0], sh[1], c->w_bits, 0));
  }
  w.acc_bytes = acc;
  w.acc = reinterpret_cast<float*>(take(acc));
  const int d = c->h / c->heads;
  w.attn_part = reinterpret_cast<float*>(take(attn_decode_partial_bytes(M, c->heads, d)));
  const size_t attn_ctr = align_up(static_cast<size_t>(M) * c->heads * sizeof(int));
  w.ctr_bytes = kSyncBytes + align_up(ctr) + attn_ctr;
  w.ctr = reinterpret_cast<int*>(take(w.ctr_bytes));
  w.tile_ctr = w.ctr ? w.ctr + kSyncBytes / sizeof(int) : nullptr;
  w.attn_ctr = w.ctr ? w.tile_ctr + align_up(ctr) / sizeof(int) : nullptr;
  w.total = off;
  return w;
}

flexq_status zero_counters(const LayerWs& w, cudaStream_t s) {
  FQ_CUDA(cudaMemsetAsync(w.ctr, 0, w.ctr_bytes, s), "zero split-tile counters");
  return FLEXQ_OK;
}

flexq_status run_linear(const __half* x, int ldx, const void* w, int w_bits, int m, int n, int k,
                        const __half* bias, const __half* res, int ld_res, int epi, void* y, int ldy,
                        void* ws, size_t ws_bytes, cudaStream_t s, const char* what,
                        const KvFuse* kvf = nullptr, const LnFuse* lnf = nullptr, int* counters = nullptr) {
  LinearArgs a{};
  a.x = x;
  a.ldx = ldx;
  a.w = w;
  a.w_bits = w_bits;
  a.m = m;
  a.n = n;
  a.k = k;
  a.bias = bias;
  a.residual = res;
  a.ld_res = ld_res;
  a.y = y;
  a.ldy = ldy;
  a.epi = epi;
  a.kv = kvf;
  a.ln = lnf;
  a.counters = counters;
  FQ_CUDA(launch_linear(a, ws, ws_bytes, s), what);
  return FLEXQ_OK;
}

// Decode attention of a layer step: dense, or top-k sparse when the config
// asks for it; with app.pos >= 0 it first appends the token's K/V rows to a
// 4-bit cache.
cudaError_t decode_attention(const flexq_config* c, const __half* q, int ldq, const KvView& kvv, int b, int len,
                             __half* out, int ldo, float* part, int* ctr, const AppendRow& app, cudaStream_t s) {
  const int d = c->h / c->heads;
  if (c->attn_topk_permille > 0)
    return launch_attn_topk(q, ldq, kvv, b, c->heads, d, len, topk_count(len, c->attn_topk_permille), out, ldo,
                            nullptr, app, s);
  return launch_attn_decode(q, ldq, kvv, b, c->heads, d, c->kv_bits, len, out, ldo, part, ctr, app, s);
}

// The fused decode step takes at most one token tile of sequences.
bool decode_fusable(int b) { return b >= 1 && b <= kFuseMaxRows; }

// Decode step of one layer for b sequences, fused ([WT] "P/D阶段计算",
// decoding phase): u_in = LN1(t) computed by the caller (the previous
// layer's FC2 or the embedding); the QKV projection stores this token's K/V
// straight into an fp16 cache slot pos, or the decode attention quantizes
// them into a 4-bit cache slot pos before it reads slots 0..pos; the output
// projection adds the residual and LayerNorms its rows (LN2) after a grid
// barrier; FC1 + GELU; FC2 adds the residual and, when ln_next_g is set,
// LayerNorms its rows into u_out (the next layer's LN1 or the final LN).
// w.ctr must be zero (it is left zero).
flexq_status decode_fused(const flexq_config* c, const flexq_layer* L, const __half* t, const __half* u_in,
                          __half* y, __half* u_out, const void* ln_next_g, const void* ln_next_b,
                          const flexq_kv* kv, int seq0, int b, int pos, const LayerWs& w, cudaStream_t s) {
  const int h = c->h, f = c->ffn, d = h / c->heads;
  const KvView kvv = view_of(c, kv, seq0);
  int* tile_ctr = w.tile_ctr;
  KvFuse kf{};
  AppendRow app = kNoAppend;
  if (c->kv_bits == 16) {
    kf.k = static_cast<__half*>(kvv.k);
    kf.v = static_cast<__half*>(kvv.v);
    kf.h = h;
    kf.heads = c->heads;
    kf.d = d;
    kf.max_len = kvv.max_len;
    kf.pos = pos;
  } else {
    app.k = w.qkv + h;
    app.v = w.qkv + 2 * h;
    app.ld = 3 * h;
    app.pos = pos;
  }
  {
    ProfScope ps(FLEXQ_K_QKV, s);
    FQ_TRY(run_linear(u_in, h, L->w_qkv, c->w_bits, b, 3 * h, h, static_cast<const __half*>(L->b_qkv), nullptr, 0,
                      EPI_BIAS, w.qkv, 3 * h, w.acc, w.acc_bytes, s, "QKV projection",
                      c->kv_bits == 16 ? &kf : nullptr, nullptr, tile_ctr));
  }
  {
    ProfScope ps(FLEXQ_K_ATTN_DECODE, s);
    FQ_CUDA(decode_attention(c, w.qkv, 3 * h, kvv, b, pos + 1, w.o, h, w.attn_part, w.attn_ctr, app, s),
            "decode attention");
  }
  LnFuse ln2{};
  ln2.g = static_cast<const __half*>(L->ln2_g);
  ln2.b = static_cast<const __half*>(L->ln2_b);
  ln2.y = w.v;
  ln2.ldy = h;
  ln2.eps = c->ln_eps;
  ln2.sync = w.ctr;
  {
    ProfScope ps(FLEXQ_K_OUT_PROJ, s);
    FQ_TRY(run_linear(w.o, h, L->w_o, c->w_bits, b, h, h, static_cast<const __half*>(L->b_o), t, h,
                      EPI_BIAS | EPI_RESIDUAL, w.xo, h, w.acc, w.acc_bytes, s, "output projection with LN2",
                      nullptr, &ln2, tile_ctr));
  }
  {
    ProfScope ps(FLEXQ_K_FC1, s);
    FQ_TRY(run_linear(w.v, h, L->w_fc1, c->w_bits, b, f, h, static_cast<const __half*>(L->b_fc1), nullptr, 0,
                      EPI_BIAS | EPI_GELU, w.g, f, w.acc, w.acc_bytes, s, "FC1", nullptr, nullptr, tile_ctr));
  }
  LnFuse lnn{};
  lnn.g = static_cast<const __half*>(ln_next_g);
  lnn.b = static_cast<const __half*>(ln_next_b);
  lnn.y = u_out;
  lnn.ldy = h;
  lnn.eps = c->ln_eps;
  lnn.sync = w.ctr;
  {
    ProfScope ps(FLEXQ_K_FC2, s);
    FQ_TRY(run_linear(w.g, f, L->w_fc2, c->w_bits, b, h, f, static_cast<const __half*>(L->b_fc2), w.xo, h,
                      EPI_BIAS | EPI_RESIDUAL, y, h, w.acc, w.acc_bytes, s, "FC2",
                      nullptr, ln_next_g != nullptr ? &lnn : nullptr, tile_ctr));
  }
  return FLEXQ_OK;
}

// One layer step over M = b*ntok rows.  prefill: ntok = s, pos = 0.
flexq_status layer_step(const flexq_config* c, const flexq_layer* L, const __half* x, __half* y,
                        const flexq_kv* kv, int seq0, int b, int ntok, int pos, bool prefill,
                        const LayerWs& w, cudaStream_t s) {
  const int h = c->h, f = c->ffn, M = b * ntok, d = h / c->heads;
  const KvView kvv = view_of(c, kv, seq0);
  {
    ProfScope ps(FLEXQ_K_LAYERNORM, s);
    FQ_CUDA(launch_layernorm(x, h, static_cast<const __half*>(L->ln1_g), static_cast<const __half*>(L->ln1_b), w.u,
                             h, M, h, c->ln_eps, s),
            "LayerNorm 1");
  }
  {
    ProfScope ps(FLEXQ_K_QKV, s);
    FQ_TRY(run_linear(w.u, h, L->w_qkv, c->w_bits, M, 3 * h, h, static_cast<const __half*>(L->b_qkv), nullptr, 0,
                      EPI_BIAS, w.qkv, 3 * h, w.acc, w.acc_bytes, s, "QKV projection"));
  }
  {
    ProfScope ps(FLEXQ_K_KV_APPEND, s);
    FQ_CUDA(launch_kv_append(w.qkv + h, w.qkv + 2 * h, 3 * h, b, ntok, c->heads, d, c->kv_bits, kvv, pos, s),
            "KV append");
  }
  if (prefill && c->prefill_kv_cache) {
    ProfScope ps(FLEXQ_K_ATTN_PREFILL, s);
    FQ_CUDA(launch_attn_prefill_cache(w.qkv, 3 * h, kvv, c->kv_bits, pos, b, ntok, c->heads, d, w.u, h, s),
            "prefill attention (cache)");
  } else if (prefill) {
    ProfScope ps(FLEXQ_K_ATTN_PREFILL, s);
    FQ_CUDA(launch_attn_prefill(w.qkv, 3 * h, b, ntok, c->heads, d, w.u, h, s), "prefill attention");
  } else {
    ProfScope ps(FLEXQ_K_ATTN_DECODE, s);
    FQ_CUDA(decode_attention(c, w.qkv, 3 * h, kvv, b, pos + 1, w.u, h, nullptr, nullptr, kNoAppend, s),
            "decode attention");
  }
  {
    ProfScope ps(FLEXQ_K_OUT_PROJ, s);
    FQ_TRY(run_linear(w.u, h, L->w_o, c->w_bits, M, h, h, static_cast<const __half*>(L->b_o), x, h,
                      EPI_BIAS | EPI_RESIDUAL, w.xo, h, w.acc, w.acc_bytes, s, "output projection"));
  }
  {
    ProfScope ps(FLEXQ_K_LAYERNORM, s);
    FQ_CUDA(launch_layernorm(w.xo, h, static_cast<const __half*>(L->ln2_g), static_cast<const __half*>(L->ln2_b),
                             w.u, h, M, h, c->ln_eps, s),
            "LayerNorm 2");
  }
  {
    ProfScope ps(FLEXQ_K_FC1, s);
    FQ_TRY(run_linear(w.u, h, L->w_fc1, c->w_bits, M, f, h, static_cast<const __half*>(L->b_fc1), nullptr, 0,
                      EPI_BIAS | EPI_GELU, w.g, f, w.acc, w.acc_bytes, s, "FC1"));
  }
  {
    ProfScope ps(FLEXQ_K_FC2, s);
    FQ_TRY(run_linear(w.g, f, L->w_fc2, c->w_bits, M, h, f, static_cast<const __half*>(L->b_fc2), w.xo, h,
                      EPI_BIAS | EPI_RESIDUAL, y, h, w.acc, w.acc_bytes, s, "FC2"));
  }
  return FLEXQ_OK;
}

}  // namespace

const Runtime& runtime() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) dev = 0;
  std::call_once(g_rt_once[dev], [dev] {
    Runtime& r = g_rt[dev];
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    r.num_sms = sms;
    void* p = nullptr;
    cudaGetSymbolAddress(&p, g_device_error);
    r.err = static_cast<uint32_t*>(p);
  });
  g_rt[dev].wait_limit_ns = g_wait_limit_ns;
  g_rt[dev].pdl = g_pdl;
  return g_rt[dev];
}

uint32_t* device_error_word() { return runtime().err; }

void set_last_error(const char* msg) { g_last_error = msg; }

cudaError_t launched() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError();
}

}  // namespace flexq

using namespace flexq;

extern "C" {

const char* flexq_last_error(void) { return g_last_error.c_str(); }

int flexq_version(void) { return 102; }

flexq_status flexq_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns == 0 ? 2000000000ull : ns;
  return FLEXQ_OK;
}

int flexq_set_launch_overlap(int on) {
  const int old = g_pdl;
  g_pdl = on ? 1 : 0;
  return old;
}

flexq_status flexq_device_status(void* stream) {
  FQ_CUDA(cudaStreamSynchronize(as_stream(stream)), "stream synchronize");
  uint32_t* err = runtime().err;
  if (err == nullptr) return fail(FLEXQ_ERR_CUDA, "device error word unavailable");
  uint32_t v = 0;
  FQ_CUDA(cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost), "read device error word");
  if (v != 0) {
    const uint32_t zero = 0;
    FQ_CUDA(cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice), "clear device error word");
    if (v == DEV_BAD_ARGUMENT) return fail(FLEXQ_ERR_DEVICE, "a kernel rejected a device-side input");
    return fail(FLEXQ_ERR_TIMEOUT, "a bounded device wait gave up (code %u)", v);
  }
  return FLEXQ_OK;
}

// --- synthetic inputs -------------------------------------------------------
static uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

flexq_status flexq_synth_normal_f16(void* out_dev, size_t n, uint64_t seed, uint64_t tensor_id, size_t start,
                                    float sigma, float mean, void* stream) {
  FQ_CHECK(n == 0 || out_dev != nullptr, "out is NULL");
  const uint64_t key = mix64(seed * 0x9E3779B97F4A7C15ull + tensor_id);
  const float scale = static_cast<float>(sqrt(3.0) / 65536.0 * static_cast<double>(sigma));
  FQ_CUDA(launch_synth_normal(static_cast<__half*>(out_dev), n, key, start, scale, mean, as_stream(stream)),
          "synth normal");
  return FLEXQ_OK;
}

flexq_status flexq_synth_tokens(int32_t* out_dev, size_t n, uint64_t seed, uint64_t tensor_id, size_t start,
                                int32_t vocab, void* stream) {
  FQ_CHECK(n == 0 || out_dev != nullptr, "out is NULL");
  FQ_CHECK(vocab > 0, "vocab must be positive");
  const uint64_t key = mix64(seed * 0x9E3779B97F4A7C15ull + tensor_id);
  FQ_CUDA(launch_synth_tokens(out_dev, n, key, start, vocab, as_stream(stream)), "synth tokens");
  return FLEXQ_OK;
}

// --- codec ---------------------------------------------------------------------
flexq_status flexq_quantize(const void* x_dev, size_t n, uint8_t* codes_dev, void* min_dev, void* scale_dev,
                            void* stream) {
  FQ_CHECK(n % 64 == 0, "n must be a multiple of 64 (got %zu)", n);
  if (n == 0) return FLEXQ_OK;
  FQ_CHECK(x_dev && codes_dev && min_dev && scale_dev, "NULL pointer");
  FQ_CHECK(aligned16(x_dev) && aligned16(codes_dev), "x and codes must be 16-byte aligned");
  FQ_CUDA(launch_quantize(static_cast<const __half*>(x_dev), n, codes_dev, static_cast<__half*>(min_dev),
                          static_cast<__half*>(scale_dev), as_stream(stream)),
          "quantize");
  return FLEXQ_OK;
}

flexq_status flexq_dequantize(const uint8_t* codes_dev, const void* min_dev, const void* scale_dev, size_t n,
                              void* out_dev, void* stream) {
  FQ_CHECK(n % 64 == 0, "n must be a multiple of 64 (got %zu)", n);
  if (n == 0) return FLEXQ_OK;
  FQ_CHECK(codes_dev && min_dev && scale_dev && out_dev, "NULL pointer");
  FQ_CHECK(aligned16(codes_dev) && aligned16(out_dev), "codes and out must be 16-byte aligned");
  FQ_CUDA(launch_dequantize(codes_dev, static_cast<const __half*>(min_dev), static_cast<const __half*>(scale_dev),
                            n, static_cast<__half*>(out_dev), as_stream(stream)),
          "dequantize");
  return FLEXQ_OK;
}

size_t flexq_packed_weight_bytes(int n_out, int k_in) {
  if (n_out <= 0 || k_in <= 0 || k_in % 64) return 0;
  return static_cast<size_t>((n_out + kTileRows - 1) / kTileRows) * (k_in / 64) * kTileBytes;
}

flexq_status flexq_pack_weight_q4(const uint8_t* codes_dev, const void* min_dev, const void* scale_dev, int n_out,
                                  int k_in, void* packed_dev, void* stream) {
  FQ_CHECK(n_out > 0 && k_in > 0 && k_in % 64 == 0, "need n_out > 0 and k_in a positive multiple of 64");
  FQ_CHECK(codes_dev && min_dev && scale_dev && packed_dev, "NULL pointer");
  FQ_CHECK(aligned16(codes_dev) && aligned16(packed_dev), "codes and packed must be 16-byte aligned");
  FQ_CUDA(launch_pack_weight(codes_dev, static_cast<const __half*>(min_dev), static_cast<const __half*>(scale_dev),
                             n_out, k_in, static_cast<uint8_t*>(packed_dev), as_stream(stream)),
          "pack weight");
  return FLEXQ_OK;
}

flexq_status flexq_quantize_weight_q4(const void* w_dev, int n_out, int k_in, void* packed_dev, void* stream) {
  FQ_CHECK(n_out > 0 && k_in > 0 && k_in % 64 == 0, "need n_out > 0 and k_in a positive multiple of 64");
  FQ_CHECK(w_dev && packed_dev, "NULL pointer");
  FQ_CHECK(aligned16(w_dev) && aligned16(packed_dev), "w and packed must be 16-byte aligned");
  FQ_CUDA(launch_quantize_weight(static_cast<const __half*>(w_dev), n_out, k_in, static_cast<uint8_t*>(packed_dev),
                                 as_stream(stream)),
          "quantize weight");
  return FLEXQ_OK;
}

// --- building blocks -----------------------------------------------------------
size_t flexq_linear_workspace(int m, int n, int k, int w_bits, int force_splits) {
  if (m <= 0 || n <= 0 || k <= 0 || k % 64 || force_splits < 0) return 0;
  return linear_workspace_bytes(m, n, k, w_bits, force_splits);
}

flexq_status flexq_linear(const void* x_dev, int ldx, const void* w_dev, int w_bits, int m, int n, int k,
                          const void* bias_dev, const void* residual_dev, int ld_res, int epilogue, void* y_dev,
                          int ldy, void* ws_dev, size_t ws_bytes, int force_splits, void* stream) {
  FQ_CHECK(m >= 0 && n > 0 && k > 0 && k % 64 == 0, "need n > 0 and k a positive multiple of 64");
  FQ_CHECK(w_bits == 4 || w_bits == 16, "w_bits must be 4 or 16");
  if (m == 0) return FLEXQ_OK;
  FQ_CHECK(x_dev && w_dev && y_dev, "NULL pointer");
  FQ_CHECK(ldx >= k && ldx % 8 == 0 && aligned16(x_dev), "x needs ldx >= k, ldx %% 8 == 0, 16-byte alignment");
  FQ_CHECK(aligned16(w_dev), "w must be 16-byte aligned");
  FQ_CHECK(ldy >= n, "ldy must be >= n");
  FQ_CHECK(!(epilogue & EPI_BIAS) || bias_dev, "bias flag without bias");
  FQ_CHECK(!(epilogue & EPI_RESIDUAL) || (residual_dev && ld_res >= n), "residual flag without residual");
  FQ_CHECK(!(epilogue & EPI_F32_OUT) || epilogue == EPI_F32_OUT, "fp32 output takes no other epilogue");
  FQ_CHECK(force_splits >= 0 && force_splits <= k / 64, "force_splits out of range");
  const size_t need = linear_workspace_bytes(m, n, k, w_bits, force_splits);
  if (need > 0 && (ws_dev == nullptr || ws_bytes < need))
    return fail(FLEXQ_ERR_WORKSPACE, "linear needs %zu workspace bytes", need);
  LinearArgs a{};
  a.x = static_cast<const __half*>(x_dev);
  a.ldx = ldx;
  a.w = w_dev;
  a.w_bits = w_bits;
  a.m = m;
  a.n = n;
  a.k = k;
  a.bias = static_cast<const __half*>(bias_dev);
  a.residual = static_cast<const __half*>(residual_dev);
  a.ld_res = ld_res;
  a.y = y_dev;
  a.ldy = ldy;
  a.epi = epilogue;
  a.force_splits = force_splits;
  FQ_CUDA(launch_linear(a, ws_dev, ws_bytes, as_stream(stream)), "linear");
  return FLEXQ_OK;
}

flexq_status flexq_layernorm(const void* x_dev, int ldx, const void* gamma_dev, const void* beta_dev, void* y_dev,
                             int ldy, int rows, int h, float eps, void* stream) {
  FQ_CHECK(h > 0 && h % 8 == 0 && h <= 12288, "h must be a multiple of 8 up to 12288");
  FQ_CHECK(rows >= 0, "rows must be >= 0");
  if (rows == 0) return FLEXQ_OK;
  FQ_CHECK(x_dev && gamma_dev && beta_dev && y_dev, "NULL pointer");
  FQ_CHECK(ldx >= h && ldy >= h && ldx % 8 == 0 && ldy % 8 == 0, "row strides must be >= h and multiples of 8");
  FQ_CHECK(aligned16(x_dev) && aligned16(y_dev) && aligned16(gamma_dev) && aligned16(beta_dev),
           "pointers must be 16-byte aligned");
  FQ_CUDA(launch_layernorm(static_cast<const __half*>(x_dev), ldx, static_cast<const __half*>(gamma_dev),
                           static_cast<const __half*>(beta_dev), static_cast<__half*>(y_dev), ldy, rows, h, eps,
                           as_stream(stream)),
          "layernorm");
  return FLEXQ_OK;
}

size_t flexq_kv_bytes(const flexq_config* cfg, int b, int max_len) {
  if (check_config(cfg) != FLEXQ_OK || b <= 0 || max_len <= 0) return 0;
  const size_t elems = static_cast<size_t>(b) * max_len * cfg->h;  // per K or V
  if (cfg->kv_bits == 16) return 2 * elems * 2;
  const size_t v_elems = static_cast<size_t>(b) * kv_pad_len(max_len) * cfg->h;  // whole 8-token blocks
  return elems / 2 + v_elems / 2 + 2 * (elems / 64 * 4);
}

flexq_status flexq_kv_append(const flexq_config* cfg, const flexq_kv* kv, const void* k_dev, const void* v_dev,
                             int ld, int b, int pos0, int ntok, void* stream) {
  FQ_TRY(check_config(cfg));
  FQ_TRY(check_kv(cfg, kv, b));
  FQ_CHECK(b >= 0 && ntok >= 0, "b and ntok must be >= 0");
  FQ_CHECK(pos0 >= 0 && pos0 + ntok <= kv->max_len, "slots %d..%d outside max_len %d", pos0, pos0 + ntok - 1,
           kv->max_len);
  if (b == 0 || ntok == 0) return FLEXQ_OK;
  FQ_CHECK(k_dev && v_dev, "NULL pointer");
  FQ_CHECK(ld >= cfg->h && ld % 8 == 0 && aligned16(k_dev) && aligned16(v_dev),
           "K/V rows need ld >= h, ld %% 8 == 0 and 16-byte alignment");
  FQ_CUDA(launch_kv_append(static_cast<const __half*>(k_dev), static_cast<const __half*>(v_dev), ld, b, ntok,
                           cfg->heads, cfg->h / cfg->heads, cfg->kv_bits, view_of(cfg, kv, 0), pos0,
                           as_stream(stream)),
          "kv append");
  return FLEXQ_OK;
}

flexq_status flexq_attention_decode(const flexq_config* cfg, const flexq_kv* kv, const void* q_dev, int ldq, int b,
                                    int len, void* out_dev, int ldo, void* stream) {
  FQ_TRY(check_config(cfg));
  FQ_TRY(check_kv(cfg, kv, b));
  FQ_CHECK(len >= 1 && len <= kv->max_len, "len must be in 1..max_len");
  FQ_CHECK(len <= 16384, "len above 16384 is not supported");
  if (b == 0) return FLEXQ_OK;
  FQ_CHECK(q_dev && out_dev, "NULL pointer");
  FQ_CHECK(ldq >= cfg->h && ldo >= cfg->h && ldq % 8 == 0 && ldo % 8 == 0, "bad row strides");
  FQ_CUDA(launch_attn_decode(static_cast<const __half*>(q_dev), ldq, view_of(cfg, kv, 0), b, cfg->heads,
                             cfg->h / cfg->heads, cfg->kv_bits, len, static_cast<__half*>(out_dev), ldo, nullptr,
                             nullptr, kNoAppend, as_stream(stream)),
          "decode attention");
  return FLEXQ_OK;
}

flexq_status flexq_attention_decode_topk(const flexq_config* cfg, const flexq_kv* kv, const void* q_dev, int ldq,
                                         int b, int len, int k, void* out_dev, int ldo, int32_t* idx_dev,
                                         void* stream) {
  FQ_TRY(check_config(cfg));
  FQ_CHECK(cfg->kv_bits == 4, "top-k sparse attention reads the 4-bit cache");
  FQ_TRY(check_kv(cfg, kv, b));
  FQ_CHECK(len >= 1 && len <= kv->max_len && len <= 16384, "len must be in 1..min(max_len, 16384)");
  FQ_CHECK(k >= 1 && k <= len, "k must be in 1..len");
  if (b == 0) return FLEXQ_OK;
  FQ_CHECK(q_dev && out_dev, "NULL pointer");
  FQ_CHECK(ldq >= cfg->h && ldo >= cfg->h && ldq % 8 == 0 && ldo % 8 == 0, "bad row strides");
  FQ_CUDA(launch_attn_topk(static_cast<const __half*>(q_dev), ldq, view_of(cfg, kv, 0), b, cfg->heads,
                           cfg->h / cfg->heads, len, k, static_cast<__half*>(out_dev), ldo, idx_dev, kNoAppend,
                           as_stream(stream)),
          "top-k decode attention");
  return FLEXQ_OK;
}

flexq_status flexq_attention_prefill(const flexq_config* cfg, const void* qkv_dev, int ldqkv, int b, int s,
                                     void* out_dev, int ldo, void* stream) {
  FQ_TRY(check_config(cfg));
  FQ_CHECK(b >= 0 && s >= 0, "b and s must be >= 0");
  if (b == 0 || s == 0) return FLEXQ_OK;
  FQ_CHECK(qkv_dev && out_dev, "NULL pointer");
  FQ_CHECK(ldqkv >= 3 * cfg->h && ldqkv % 8 == 0 && ldo >= cfg->h && ldo % 8 == 0, "bad row strides");
  FQ_CHECK(aligned16(qkv_dev) && aligned16(out_dev), "pointers must be 16-byte aligned");
  FQ_CUDA(launch_attn_prefill(static_cast<const __half*>(qkv_dev), ldqkv, b, s, cfg->heads, cfg->h / cfg->heads,
                              static_cast<__half*>(out_dev), ldo, as_stream(stream)),
          "prefill attention");
  return FLEXQ_OK;
}

flexq_status flexq_attention_prefill_cache(const flexq_config* cfg, const flexq_kv* kv, const void* q_dev,
                                           int ldq, int b, int s, int pos0, void* out_dev, int ldo, void* stream) {
  FQ_TRY(check_config(cfg));
  FQ_CHECK(b >= 0 && s >= 0 && pos0 >= 0, "b, s and pos0 must be >= 0");
  if (b == 0 || s == 0) return FLEXQ_OK;
  FQ_TRY(check_kv(cfg, kv, b));
  FQ_CHECK(q_dev && out_dev, "NULL pointer");
  FQ_CHECK(pos0 + s <= kv->max_len, "slots %d..%d exceed the cache (%d)", pos0, pos0 + s - 1, kv->max_len);
  FQ_CHECK(cfg->kv_bits == 16 || pos0 % 8 == 0, "4-bit mode needs pos0 %% 8 == 0");
  FQ_CHECK(ldq >= cfg->h && ldq % 8 == 0 && ldo >= cfg->h && ldo % 8 == 0, "bad row strides");
  FQ_CHECK(aligned16(q_dev) && aligned16(out_dev), "pointers must be 16-byte aligned");
  FQ_CUDA(launch_attn_prefill_cache(static_cast<const __half*>(q_dev), ldq, view_of(cfg, kv, 0), cfg->kv_bits, pos0,
                                    b, s, cfg->heads, cfg->h / cfg->heads, static_cast<__half*>(out_dev), ldo,
                                    as_stream(stream)),
          "prefill attention (cache)");
  return FLEXQ_OK;
}

// --- layer steps ----------------------------------------------------------------
size_t flexq_layer_workspace(const flexq_config* cfg, int rows, int mode) {
  if (check_config(cfg) != FLEXQ_OK || rows <= 0 || (mode != 0 && mode != 1)) return 0;
  return layer_ws_layout(cfg, rows, nullptr).total;
}

static flexq_status layer_common(const flexq_config* cfg, const flexq_layer* layer, const void* x, void* y,
                                 const flexq_kv* kv, int b, int ntok, int pos, bool prefill, void* ws,
                                 size_t ws_bytes, void* stream) {
  FQ_TRY(check_config(cfg));
  FQ_TRY(check_layer(cfg, layer));
  FQ_TRY(check_kv(cfg, kv, b));
  FQ_CHECK(b >= 0, "b must be >= 0");
  if (b == 0) return FLEXQ_OK;
  FQ_CHECK(x && y, "NULL activation pointer");
  FQ_CHECK(x != y, "y may not alias x");
  FQ_CHECK(aligned16(x) && aligned16(y), "activations must be 16-byte aligned");
  const int M = b * ntok;
  const LayerWs probe = layer_ws_layout(cfg, M, nullptr);
  if (ws == nullptr || ws_bytes < probe.total)
    return fail(FLEXQ_ERR_WORKSPACE, "layer needs %zu workspace bytes, got %zu", probe.total, ws_bytes);
  FQ_CHECK(aligned16(ws), "workspace must be 16-byte aligned");
  const LayerWs w = layer_ws_layout(cfg, M, static_cast<uint8_t*>(ws));
  cudaStream_t st = as_stream(stream);
  if (prefill || !decode_fusable(b))
    return layer_step(cfg, layer, static_cast<const __half*>(x), static_cast<__half*>(y), kv, 0, b, ntok, pos,
                      prefill, w, st);
  FQ_TRY(zero_counters(w, st));
  {
    ProfScope ps(FLEXQ_K_LAYERNORM, st);
    FQ_CUDA(launch_layernorm(static_cast<const __half*>(x), cfg->h, static_cast<const __half*>(layer->ln1_g),
                             static_cast<const __half*>(layer->ln1_b), w.u, cfg->h, b, cfg->h, cfg->ln_eps, st),
            "LayerNorm 1");
  }
  return decode_fused(cfg, layer, static_cast<const __half*>(x), w.u, static_cast<__half*>(y), nullptr, nullptr,
                      nullptr, kv, 0, b, pos, w, st);
}

flexq_status flexq_layer_prefill(const flexq_config* cfg, const flexq_layer* layer, const void* x_dev, void* y_dev,
                                 const flexq_kv* kv, int b, int s, void* ws_dev, size_t ws_bytes, void* stream) {
  FQ_CHECK(kv != nullptr, "kv is NULL");
  FQ_CHECK(s >= 1 && s <= kv->max_len, "s must be in 1..max_len");
  return layer_common(cfg, layer, x_dev, y_dev, kv, b, s, 0, true, ws_dev, ws_bytes, stream);
}

flexq_status flexq_layer_decode(const flexq_config* cfg, const flexq_layer* layer, const void* t_dev, void* y_dev,
                                const flexq_kv* kv, int b, int pos, void* ws_dev, size_t ws_bytes, void* stream) {
  FQ_CHECK(kv != nullptr, "kv is NULL");
  FQ_CHECK(pos >= 0 && pos < kv->max_len, "pos must be in 0..max_len-1");
  FQ_CHECK(pos < 16384, "pos above 16383 is not supported");
  return layer_common(cfg, layer, t_dev, y_dev, kv, b, 1, pos, false, ws_dev, ws_bytes, stream);
}

// --- generation -----------------------------------------------------------------
namespace {
struct GenWs {
  __half *x, *y, *t, *t2, *tn;
  float* logits;
  uint8_t* layer;
  size_t layer_bytes;
  float* head_acc;
  size_t head_acc_bytes;
  size_t total;
};

GenWs gen_ws_layout(const flexq_model* m, int b, int s, int gbs, uint8_t* base) {
  GenWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const size_t h = m->cfg.h;
  w.x = reinterpret_cast<__half*>(take(static_cast<size_t>(b) * s * h * 2));
  w.y = reinterpret_cast<__half*>(take(static_cast<size_t>(b) * s * h * 2));
  w.t = reinterpret_cast<__half*>(take(static_cast<size_t>(b) * h * 2));
  w.t2 = reinterpret_cast<__half*>(take(static_cast<size_t>(b) * h * 2));
  w.tn = reinterpret_cast<__half*>(take(static_cast<size_t>(b) * h * 2));
  w.logits = reinterpret_cast<float*>(take(static_cast<size_t>(b) * m->vocab * 4));
  w.layer_bytes =
      std::max(layer_ws_layout(&m->cfg, gbs * s, nullptr).total, layer_ws_layout(&m->cfg, gbs, nullptr).total);
  w.layer = take(w.layer_bytes);
  w.head_acc_bytes = linear_workspace_bytes(b, m->vocab, m->cfg.h, m->embed_bits == 4 ? 4 : 16, 0);
  w.head_acc = reinterpret_cast<float*>(take(w.head_acc_bytes));
  w.total = off;
  return w;
}

flexq_status check_model(const flexq_model* m) {
  FQ_CHECK(m != nullptr, "model is NULL");
  FQ_TRY(check_config(&m->cfg));
  FQ_CHECK(m->layers > 0 && m->layer && m->kv, "model needs layers, layer and kv arrays");
  FQ_CHECK(m->vocab > 0 && m->max_pos > 0, "vocab and max_pos must be positive");
  FQ_CHECK(m->embed && m->pos_embed && m->lnf_g && m->lnf_b, "model embedding/final LN pointer is NULL");
  FQ_CHECK(m->embed_bits == 16 || m->embed_bits == 4, "embed_bits must be 16 or 4");
  FQ_CHECK(aligned16(m->embed) && aligned16(m->pos_embed) && aligned16(m->lnf_g) && aligned16(m->lnf_b),
           "embedding and final LayerNorm tensors must be 16-byte aligned");
  for (int i = 0; i < m->layers; ++i) FQ_TRY(check_layer(&m->cfg, &m->layer[i]));
  return FLEXQ_OK;
}

// Validates a generation request and carves its workspace.
flexq_status check_generation(const flexq_model* model, int b, int s, int n, int gpu_batch, const int32_t* out_dev,
                              void* ws_dev, size_t ws_bytes, GenWs* w) {
  FQ_TRY(check_model(model));
  FQ_CHECK(b > 0 && s > 0 && n > 0, "b, s and n must be positive");
  FQ_CHECK(gpu_batch > 0 && b % gpu_batch == 0, "gpu_batch must divide b");
  FQ_CHECK(out_dev != nullptr, "NULL out pointer");
  FQ_CHECK(s + n - 1 <= model->max_pos, "s + n - 1 positions exceed max_pos");
  for (int i = 0; i < model->layers; ++i) {
    FQ_TRY(check_kv(&model->cfg, &model->kv[i], b));
    FQ_CHECK(model->kv[i].max_len >= s + n - 1, "layer %d cache holds %d slots, need %d", i, model->kv[i].max_len,
             s + n - 1);
  }
  const GenWs probe = gen_ws_layout(model, b, s, gpu_batch, nullptr);
  if (ws_dev == nullptr || ws_bytes < probe.total)
    return fail(FLEXQ_ERR_WORKSPACE, "generate needs %zu workspace bytes, got %zu", probe.total, ws_bytes);
  FQ_CHECK(aligned16(ws_dev), "workspace must be 16-byte aligned");
  *w = gen_ws_layout(model, b, s, gpu_batch, static_cast<uint8_t*>(ws_dev));
  return FLEXQ_OK;
}

// Final LayerNorm (unless the rows arrive normalised in w.tn), tied LM head
// and greedy choice.
flexq_status lm_head(const flexq_model* m, const __half* x_last, int ldx, int b, const GenWs& w, int32_t* out,
                     int ld_out, cudaStream_t s, bool normalised = false) {
  const int h = m->cfg.h;
  if (!normalised) {
    ProfScope ps(FLEXQ_K_LAYERNORM, s);
    FQ_CUDA(launch_layernorm(x_last, ldx, static_cast<const __half*>(m->lnf_g),
                             static_cast<const __half*>(m->lnf_b), w.tn, h, b, h, m->cfg.ln_eps, s),
            "final LayerNorm");
  }
  {
    ProfScope ps(FLEXQ_K_LM_HEAD, s);
    FQ_TRY(run_linear(w.tn, h, m->embed, m->embed_bits, b, m->vocab, h, nullptr, nullptr, 0, EPI_F32_OUT, w.logits,
                      m->vocab,
                      w.head_acc, w.head_acc_bytes, s, "LM head"));
  }
  ProfScope ps(FLEXQ_K_ARGMAX, s);
  FQ_CUDA(launch_argmax(w.logits, b, m->vocab, m->vocab, out, ld_out, s), "argmax");
  return FLEXQ_OK;
}

// Where a column's layer weights come from.  Resident: the model's own
// device pointers.  Offloaded ([WT] "Search Space": the zig-zag block
// schedule loads a layer's weights once per column and reuses them for every
// GPU batch of the block; [RPT] 三(A)): the four weight matrices of every
// layer stay in page-locked host memory and are copied into one of two
// device slots on a copy stream two (column, layer) steps ahead of the
// compute stream, so the copy of the next layer overlaps this layer's
// compute; events order each slot's reuse.
struct LayerFeed {
  const flexq_model* m = nullptr;
  bool offload = false;
  uint8_t* slots = nullptr;
  size_t slot_bytes = 0;
  size_t off[4] = {};
  size_t bytes[4] = {};
  cudaStream_t copy = nullptr, compute = nullptr;
  cudaEvent_t copied[2] = {}, freed[2] = {};
  flexq_layer slot_layer[2] = {};
  long long step = 0, total = 0;  // (column, layer) steps taken / to take in this call

  explicit LayerFeed(const flexq_model* model) : m(model) {}
  LayerFeed(const LayerFeed&) = delete;
  ~LayerFeed() {
    for (int i = 0; i < 2; ++i) {
      if (copied[i]) cudaEventDestroy(copied[i]);
      if (freed[i]) cudaEventDestroy(freed[i]);
    }
  }

  flexq_status copy_step(long long g) {
    const int slot = static_cast<int>(g & 1);
    const flexq_layer& L = m->layer[g % m->layers];
    const void* src[4] = {L.w_qkv, L.w_o, L.w_fc1, L.w_fc2};
    FQ_CUDA(cudaStreamWaitEvent(copy, freed[slot], 0), "wait for a free weight slot");
    for (int i = 0; i < 4; ++i)
      FQ_CUDA(cudaMemcpyAsync(slots + slot * slot_bytes + off[i], src[i], bytes[i], cudaMemcpyHostToDevice, copy),
              "weight copy to the device");
    FQ_CUDA(cudaEventRecord(copied[slot], copy), "event record");
    return FLEXQ_OK;
  }

  flexq_status start(long long steps) {
    total = steps;
    step = 0;
    if (!offload) return FLEXQ_OK;
    for (int i = 0; i < 2; ++i) {
      FQ_CUDA(cudaEventCreateWithFlags(&copied[i], cudaEventDisableTiming), "event create");
      FQ_CUDA(cudaEventCreateWithFlags(&freed[i], cudaEventDisableTiming), "event create");
      // nothing has used the slot yet: its first copy need not wait
      FQ_CUDA(cudaEventRecord(freed[i], compute), "event record");
    }
    for (long long g = 0; g < std::min<long long>(2, total); ++g) FQ_TRY(copy_step(g));
    return FLEXQ_OK;
  }

  // The layer to run at this step (waits for its weights when offloaded).
  const flexq_layer* begin(int l, flexq_status* st) {
    *st = FLEXQ_OK;
    if (!offload) return &m->layer[l];
    const int slot = static_cast<int>(step & 1);
    const cudaError_t e = cudaStreamWaitEvent(compute, copied[slot], 0);
    if (e != cudaSuccess) {
      *st = cuda_fail(e, "wait for layer weights");
      return nullptr;
    }
    slot_layer[slot] = m->layer[l];
    uint8_t* base = slots + slot * slot_bytes;
    slot_layer[slot].w_qkv = base + off[0];
    slot_layer[slot].w_o = base + off[1];
    slot_layer[slot].w_fc1 = base + off[2];
    slot_layer[slot].w_fc2 = base + off[3];
    return &slot_layer[slot];
  }

  flexq_status end() {
    if (offload) {
      const int slot = static_cast<int>(step & 1);
      FQ_CUDA(cudaEventRecord(freed[slot], compute), "event record");
      if (step + 2 < total) FQ_TRY(copy_step(step + 2));
    }
    ++step;
    return FLEXQ_OK;
  }
};

// Bytes of one matrix as the layer stores it.
size_t weight_bytes(const flexq_config* c, int n_out, int k_in) {
  return c->w_bits == 4 ? flexq_packed_weight_bytes(n_out, k_in) : static_cast<size_t>(n_out) * k_in * 2;
}

// Offsets of a layer's four weight matrices in a device slot; returns the
// slot's size.
size_t slot_layout(const flexq_config* c, size_t off[4], size_t bytes[4]) {
  const size_t b[4] = {weight_bytes(c, 3 * c->h, c->h), weight_bytes(c, c->h, c->h), weight_bytes(c, c->ffn, c->h),
                       weight_bytes(c, c->h, c->ffn)};
  size_t o = 0;
  for (int i = 0; i < 4; ++i) {
    off[i] = o;
    bytes[i] = b[i];
    o += align_up(b[i]);
  }
  return o;
}

// Prefill column of the zig-zag block: every layer over every GPU batch,
// then the first token of each sequence.
flexq_status prefill_column(const flexq_model* model, const int32_t* prompt_dev, int b, int s, int n, int gpu_batch,
                            int32_t* out_dev, const GenWs& w, cudaStream_t st, LayerFeed& feed) {
  const flexq_config* c = &model->cfg;
  const int h = c->h, nb = b / gpu_batch;
  {
    ProfScope ps(FLEXQ_K_EMBED, st);
    FQ_CUDA(launch_embed(prompt_dev, s, b, s, model->embed, model->embed_bits, model->vocab,
                         static_cast<const __half*>(model->pos_embed), 0, h, w.x, st),
            "embedding");
  }
  __half *x = w.x, *y = w.y;
  const LayerWs lw = layer_ws_layout(c, gpu_batch * s, w.layer);
  for (int l = 0; l < model->layers; ++l) {
    flexq_status fs;
    const flexq_layer* L = feed.begin(l, &fs);
    FQ_TRY(fs);
    for (int k = 0; k < nb; ++k) {
      const size_t off = static_cast<size_t>(k) * gpu_batch * s * h;
      FQ_TRY(layer_step(c, L, x + off, y + off, &model->kv[l], k * gpu_batch, gpu_batch, s, 0, true, lw, st));
    }
    FQ_TRY(feed.end());
    std::swap(x, y);
  }
  return lm_head(model, x + static_cast<size_t>(s - 1) * h, s * h, b, w, out_dev, n, st);
}

// Decode columns j = 1 .. n-1: the token in out[:, j-1] at position s+j-1
// runs through every layer for every GPU batch and yields out[:, j].
flexq_status decode_columns(const flexq_model* model, int b, int s, int n, int gpu_batch, int32_t* out_dev,
                            const GenWs& w, cudaStream_t st, LayerFeed& feed) {
  const flexq_config* c = &model->cfg;
  const int h = c->h, nb = b / gpu_batch;
  const LayerWs lw = layer_ws_layout(c, gpu_batch, w.layer);
  if (decode_fusable(gpu_batch)) {
    // Fused columns: the embedding applies layer 0's LN1; each layer's FC2
    // LayerNorms its output with the next layer's LN1 (the last layer's with
    // the final LN) into w.tn, which the next QKV projection (or the LM
    // head) reads.  The counters are zeroed once for all columns.
    FQ_TRY(zero_counters(lw, st));
    for (int j = 1; j < n; ++j) {
      const int pos = s + j - 1;
      {
        ProfScope ps(FLEXQ_K_EMBED, st);
        FQ_CUDA(launch_embed_ln(out_dev + (j - 1), n, b, model->embed, model->embed_bits, model->vocab,
                                static_cast<const __half*>(model->pos_embed), pos, h, w.t,
                                static_cast<const __half*>(model->layer[0].ln1_g),
                                static_cast<const __half*>(model->layer[0].ln1_b), c->ln_eps, w.tn, st),
                "embedding with LN1");
      }
      __half *t = w.t, *t2 = w.t2;
      for (int l = 0; l < model->layers; ++l) {
        const bool last = l + 1 == model->layers;
        const void* g = last ? model->lnf_g : model->layer[l + 1].ln1_g;
        const void* bb = last ? model->lnf_b : model->layer[l + 1].ln1_b;
        flexq_status fs;
        const flexq_layer* L = feed.begin(l, &fs);
        FQ_TRY(fs);
        for (int k = 0; k < nb; ++k) {
          const size_t off = static_cast<size_t>(k) * gpu_batch * h;
          FQ_TRY(decode_fused(c, L, t + off, w.tn + off, t2 + off, w.tn + off, g, bb, &model->kv[l], k * gpu_batch,
                              gpu_batch, pos, lw, st));
        }
        FQ_TRY(feed.end());
        std::swap(t, t2);
      }
      FQ_TRY(lm_head(model, w.tn, h, b, w, out_dev + j, n, st, true));
    }
    return FLEXQ_OK;
  }
  for (int j = 1; j < n; ++j) {
    const int pos = s + j - 1;
    {
      ProfScope ps(FLEXQ_K_EMBED, st);
      FQ_CUDA(launch_embed(out_dev + (j - 1), n, b, 1, model->embed, model->embed_bits, model->vocab,
                           static_cast<const __half*>(model->pos_embed), pos, h, w.t, st),
              "embedding");
    }
    __half *t = w.t, *t2 = w.t2;
    for (int l = 0; l < model->layers; ++l) {
      flexq_status fs;
      const flexq_layer* L = feed.begin(l, &fs);
      FQ_TRY(fs);
      for (int k = 0; k < nb; ++k) {
        const size_t off = static_cast<size_t>(k) * gpu_batch * h;
        FQ_TRY(layer_step(c, L, t + off, t2 + off, &model->kv[l], k * gpu_batch, gpu_batch, 1, pos, false, lw, st));
      }
      FQ_TRY(feed.end());
      std::swap(t, t2);
    }
    FQ_TRY(lm_head(model, t, h, b, w, out_dev + j, n, st));
  }
  return FLEXQ_OK;
}
}  // namespace

size_t flexq_generate_workspace(const flexq_model* model, int b, int s, int gpu_batch) {
  if (model == nullptr || check_config(&model->cfg) != FLEXQ_OK || b <= 0 || s <= 0 || gpu_batch <= 0) return 0;
  return gen_ws_layout(model, b, s, gpu_batch, nullptr).total;
}

flexq_status flexq_generate_prefill(const flexq_model* model, const int32_t* prompt_dev, int b, int s, int n,
                                    int gpu_batch, int32_t* out_dev, void* ws_dev, size_t ws_bytes, void* stream) {
  GenWs w;
  FQ_TRY(check_generation(model, b, s, n, gpu_batch, out_dev, ws_dev, ws_bytes, &w));
  FQ_CHECK(prompt_dev != nullptr, "NULL prompt pointer");
  LayerFeed feed(model);
  FQ_TRY(feed.start(model->layers));
  return prefill_column(model, prompt_dev, b, s, n, gpu_batch, out_dev, w, as_stream(stream), feed);
}

flexq_status flexq_generate_decode(const flexq_model* model, int b, int s, int n, int gpu_batch, int32_t* out_dev,
                                   void* ws_dev, size_t ws_bytes, void* stream) {
  GenWs w;
  FQ_TRY(check_generation(model, b, s, n, gpu_batch, out_dev, ws_dev, ws_bytes, &w));
  LayerFeed feed(model);
  FQ_TRY(feed.start(static_cast<long long>(n - 1) * model->layers));
  return decode_columns(model, b, s, n, gpu_batch, out_dev, w, as_stream(stream), feed);
}

namespace {
// The whole generation (prefill column, n-1 decode columns) with the given
// layer feed; fills timing when asked.
flexq_status generate_all(const flexq_model* model, const int32_t* prompt_dev, int b, int s, int n, int gpu_batch,
                          int32_t* out_dev, const GenWs& w, flexq_timing* timing, cudaStream_t st, LayerFeed& feed) {
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
  if (timing) {
    for (auto& e : ev) FQ_CUDA(cudaEventCreate(&e), "event create");
    FQ_CUDA(cudaEventRecord(ev[0], st), "event record");
  }
  flexq_status rc = feed.start(static_cast<long long>(n) * model->layers);
  if (rc == FLEXQ_OK) rc = prefill_column(model, prompt_dev, b, s, n, gpu_batch, out_dev, w, st, feed);
  if (rc == FLEXQ_OK && timing) cudaEventRecord(ev[1], st);
  if (rc == FLEXQ_OK) rc = decode_columns(model, b, s, n, gpu_batch, out_dev, w, st, feed);
  if (timing) {
    if (rc == FLEXQ_OK) {
      cudaEventRecord(ev[2], st);
      cudaEventSynchronize(ev[2]);
      cudaEventElapsedTime(&timing->prefill_ms, ev[0], ev[1]);
      cudaEventElapsedTime(&timing->decode_ms, ev[1], ev[2]);
    }
    for (auto& e : ev)
      if (e) cudaEventDestroy(e);
  }
  return rc;
}
}  // namespace

flexq_status flexq_generate(const flexq_model* model, const int32_t* prompt_dev, int b, int s, int n, int gpu_batch,
                            int32_t* out_dev, void* ws_dev, size_t ws_bytes, flexq_timing* timing, void* stream) {
  GenWs w;
  FQ_TRY(check_generation(model, b, s, n, gpu_batch, out_dev, ws_dev, ws_bytes, &w));
  FQ_CHECK(prompt_dev != nullptr, "NULL prompt pointer");
  LayerFeed feed(model);
  return generate_all(model, prompt_dev, b, s, n, gpu_batch, out_dev, w, timing, as_stream(stream), feed);
}

// --- offloaded weights --------------------------------------------------------------
size_t flexq_offload_slot_bytes(const flexq_config* cfg) {
  if (check_config(cfg) != FLEXQ_OK) return 0;
  size_t off[4], bytes[4];
  return slot_layout(cfg, off, bytes);
}

flexq_status flexq_generate_offload(const flexq_model* model, void* slots_dev, size_t slots_bytes, void* copy_stream,
                                    const int32_t* prompt_dev, int b, int s, int n, int gpu_batch, int32_t* out_dev,
                                    void* ws_dev, size_t ws_bytes, flexq_timing* timing, void* stream) {
  GenWs w;
  FQ_TRY(check_generation(model, b, s, n, gpu_batch, out_dev, ws_dev, ws_bytes, &w));
  FQ_CHECK(prompt_dev != nullptr, "NULL prompt pointer");
  FQ_CHECK(copy_stream != stream, "the weight copies need a stream of their own");
  LayerFeed feed(model);
  feed.offload = true;
  feed.slot_bytes = slot_layout(&model->cfg, feed.off, feed.bytes);
  FQ_CHECK(slots_dev != nullptr && aligned16(slots_dev), "slots must be a 16-byte aligned device buffer");
  if (slots_bytes < 2 * feed.slot_bytes)
    return fail(FLEXQ_ERR_WORKSPACE, "offload needs %zu slot bytes, got %zu", 2 * feed.slot_bytes, slots_bytes);
  for (int i = 0; i < model->layers; ++i) {
    const flexq_layer& L = model->layer[i];
    for (const void* p : {L.w_qkv, L.w_o, L.w_fc1, L.w_fc2}) {
      cudaPointerAttributes attr{};
      const cudaError_t e = cudaPointerGetAttributes(&attr, p);
      if (e != cudaSuccess) cudaGetLastError();
      FQ_CHECK(e == cudaSuccess && attr.type == cudaMemoryTypeHost,
               "layer %d: offloaded weights must be page-locked host memory", i);
    }
  }
  feed.slots = static_cast<uint8_t*>(slots_dev);
  feed.copy = as_stream(copy_stream);
  feed.compute = as_stream(stream);
  return generate_all(model, prompt_dev, b, s, n, gpu_batch, out_dev, w, timing, feed.compute, feed);
}

flexq_status flexq_offload_plan(const flexq_model* model, int s, int n, const flexq_hw* hw, int max_block,
                                flexq_offload_choice* out) {
  FQ_CHECK(model != nullptr && hw != nullptr && out != nullptr, "NULL pointer");
  FQ_TRY(check_config(&model->cfg));
  FQ_CHECK(model->layers > 0 && model->vocab > 0, "model needs layers and a vocabulary");
  FQ_CHECK(s > 0 && n > 0 && max_block > 0, "s, n and max_block must be positive");
  FQ_CHECK(hw->h2d_gbps > 0 && hw->hbm_gbps > 0 && hw->tensor_tflops > 0 && hw->device_bytes > 0,
           "hardware rates and memory must be positive");
  const flexq_config* c = &model->cfg;
  const double h = c->h, ffn = c->ffn, L = model->layers;
  size_t off[4], bytes[4];
  const double slot = static_cast<double>(slot_layout(c, off, bytes));
  const double w_layer = static_cast<double>(bytes[0] + bytes[1] + bytes[2] + bytes[3]);
  const double flop_tok = 2.0 * (4.0 * h * h + 2.0 * h * ffn);  // 2 * (QKV + out + FC1 + FC2) per token
  const double kv_row = static_cast<double>(flexq_kv_bytes(c, 1, 1024)) / 1024.0 / 2.0;  // K or V bytes per slot
  const double lbar = s + n / 2.0;
  const double bw = hw->hbm_gbps * 1e9, tc = hw->tensor_tflops * 1e12, io_bw = hw->h2d_gbps * 1e9;
  const double e_bytes = model->embed_bits == 4 ? static_cast<double>(flexq_packed_weight_bytes(model->vocab, c->h))
                                                : static_cast<double>(model->vocab) * h * 2;
  const double fixed = 2.0 * slot + e_bytes + static_cast<double>(model->max_pos) * h * 2 + L * (16.0 * h + 2 * ffn);
  flexq_offload_choice best{};
  best.decode_tokens_per_s = -1.0;
  // larger GPU batches first: among choices within 0.1 % of each other the
  // model cannot tell apart, the larger batch runs the more efficient GEMMs
  for (int gbs = kFuseMaxRows; gbs >= 16; gbs -= 16) {
    for (int nb = 1; static_cast<long long>(gbs) * nb <= max_block; ++nb) {
      const int b = gbs * nb;
      const double mem = fixed + L * static_cast<double>(flexq_kv_bytes(c, b, s + n)) +
                         static_cast<double>(flexq_generate_workspace(model, b, s, gbs));
      if (mem > hw->device_bytes) break;  // a larger block only needs more
      const double batch = std::max(w_layer / bw, flop_tok * gbs / tc) + gbs * lbar * 2.0 * kv_row / bw;
      const double io = w_layer / io_bw, comp = nb * batch;
      const double head = std::max(e_bytes / bw, 2.0 * b * model->vocab * h / tc);
      const double column = L * std::max(io, comp) + head;
      const double tps = b / column;
      if (tps > best.decode_tokens_per_s * 1.001) {
        best.gpu_batch = gbs;
        best.num_batches = nb;
        best.decode_tokens_per_s = tps;
        best.column_io_s = L * io;
        best.column_compute_s = L * comp + head;
        best.device_bytes = mem;
      }
    }
  }
  FQ_CHECK(best.gpu_batch > 0, "no block of at least 16 sequences fits in %.3g device bytes", hw->device_bytes);
  *out = best;
  return FLEXQ_OK;
}

// --- instrumentation -------------------------------------------------------------
uint64_t flexq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

flexq_status flexq_profile_start(void) {
  g_prof.on = true;
  g_prof.used = 0;
  g_prof.marks.clear();
  return FLEXQ_OK;
}

flexq_status flexq_profile_stop(void* stream, float* total_ms, int* calls) {
  g_prof.on = false;
  FQ_CUDA(cudaStreamSynchronize(as_stream(stream)), "stream synchronize");
  for (int k = 0; k < FLEXQ_K_COUNT; ++k) {
    if (total_ms) total_ms[k] = 0.f;
    if (calls) calls[k] = 0;
  }
  for (const auto& m : g_prof.marks) {
    float ms = 0.f;
    FQ_CUDA(cudaEventElapsedTime(&ms, g_prof.pool[m.second], g_prof.pool[m.second + 1]), "event elapsed");
    if (total_ms) total_ms[m.first] += ms;
    if (calls) calls[m.first] += 1;
  }
  g_prof.marks.clear();
  g_prof.used = 0;
  return FLEXQ_OK;
}

}  // extern "C"
