// Host side of the C ABI declared in include/hymba.h: argument validation,
// workspace layout and the launch sequence of one hybrid-head layer
// (Hymba §2.1 Eq. 1-3; §2.2 local/global attention and cross-layer KV sharing;
// §2.3 meta tokens).  Nothing here computes the layer: every step is a kernel.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"

namespace hymba {

static thread_local char g_msg[512] = "";

static std::atomic<unsigned long long> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

void set_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

}  // namespace hymba

using namespace hymba;

// ---------------------------------------------------------------------------
// Optional per-step timing with CUDA events (hymba_profile_enable).
// ---------------------------------------------------------------------------
namespace {
struct ProfRecord {
  const char *name;
  cudaEvent_t start, stop;
  unsigned long long kernels;
};
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t next = 0;
  std::vector<ProfRecord> recs;
};
Profiler &prof() {
  static Profiler p;
  return p;
}
constexpr size_t kProfEvents = 8192;

class ProfScope {
 public:
  ProfScope(cudaStream_t s, const char *name) : s_(s) {
    Profiler &p = prof();
    if (!p.on) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
    std::lock_guard<std::mutex> g(p.mu);
    if (p.next + 2 > p.pool.size()) return;  // pool exhausted: stop recording until collected
    rec_.name = name;
    launches0_ = g_launches.load();
    rec_.start = p.pool[p.next++];
    rec_.stop = p.pool[p.next++];
    cudaEventRecord(rec_.start, s_);
    active_ = true;
  }
  ~ProfScope() {
    if (!active_) return;
    cudaEventRecord(rec_.stop, s_);
    rec_.kernels = g_launches.load() - launches0_;
    Profiler &p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    p.recs.push_back(rec_);
  }

 private:
  cudaStream_t s_;
  ProfRecord rec_{};
  unsigned long long launches0_ = 0;
  bool active_ = false;
};
}  // namespace

struct hymba_layer {
  hymba_layer_config cfg;
  hymba_layer_weights w;
  uint64_t id;
  const hymba_layer *producer;  // non-null for a K/V-sharing consumer
  uint64_t producer_id;
};

static std::atomic<uint64_t> g_next_id{1};

#define FAIL(code, ...)        \
  do {                         \
    set_error(__VA_ARGS__);    \
    return code;               \
  } while (0)

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static size_t esize(hymba_dtype d) { return d == HYMBA_BF16 ? 2 : 4; }
static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

static int qk_width(const hymba_layer_config &c) { return c.n_heads * c.head_dim_qk; }
static int k_width(const hymba_layer_config &c) { return c.n_kv_heads * c.head_dim_qk; }
static int v_width(const hymba_layer_config &c) { return c.n_kv_heads * c.head_dim_v; }
static int xdbl_width(const hymba_layer_config &c) { return c.dt_rank + 2 * c.d_state; }
static float score_scale(const hymba_layer_config &c) {
  return c.softmax_scale > 0.f ? c.softmax_scale : 1.0f / std::sqrt((float)c.head_dim_qk);
}

extern "C" {

const char *hymba_last_error(void) { return g_msg; }

const char *hymba_status_string(hymba_status s) {
  switch (s) {
    case HYMBA_OK: return "ok";
    case HYMBA_ERR_INVALID_ARG: return "invalid argument";
    case HYMBA_ERR_UNSUPPORTED: return "unsupported";
    case HYMBA_ERR_WORKSPACE: return "workspace too small";
    case HYMBA_ERR_NOT_BOUND: return "K/V sharing not bound";
    case HYMBA_ERR_CUDA: return "CUDA error";
    case HYMBA_ERR_TIMEOUT: return "device wait timed out";
    case HYMBA_ERR_DEVICE: return "no usable device";
  }
  return "unknown status";
}

const char *hymba_version(void) { return "hymba-b200 0.1 sm_100a"; }

hymba_status hymba_layer_create(const hymba_layer_config *cfg, const hymba_layer_weights *w,
                                hymba_layer **out) {
  g_msg[0] = 0;
  if (!cfg || !w || !out) FAIL(HYMBA_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  const hymba_layer_config &c = *cfg;
  if (c.dtype != HYMBA_F32 && c.dtype != HYMBA_BF16) FAIL(HYMBA_ERR_INVALID_ARG, "dtype %d", c.dtype);
  if (c.d_model <= 0 || c.n_heads <= 0 || c.n_kv_heads <= 0 || c.head_dim_qk <= 0 ||
      c.head_dim_v <= 0 || c.d_inner <= 0 || c.d_state <= 0 || c.d_conv <= 0 || c.dt_rank <= 0)
    FAIL(HYMBA_ERR_INVALID_ARG, "every dimension must be positive");
  if (c.n_heads % c.n_kv_heads) FAIL(HYMBA_ERR_INVALID_ARG, "n_heads %% n_kv_heads != 0");
  if (c.head_dim_v * c.n_heads != c.d_inner)
    FAIL(HYMBA_ERR_INVALID_ARG, "head_dim_v * n_heads must equal d_inner (Eq. 3 adds the branches)");
  if (c.n_meta < 0) FAIL(HYMBA_ERR_INVALID_ARG, "n_meta < 0");
  if (!c.is_global && c.window < 1) FAIL(HYMBA_ERR_INVALID_ARG, "window < 1 on a sliding-window layer");
  if (!(c.rms_eps >= 0.f) || !(c.softmax_scale >= 0.f)) FAIL(HYMBA_ERR_INVALID_ARG, "eps/scale < 0");
  if (c.d_state != 16) FAIL(HYMBA_ERR_UNSUPPORTED, "d_state must be 16");
  if (c.d_conv > 4) FAIL(HYMBA_ERR_UNSUPPORTED, "d_conv must be <= 4");
  if (c.dt_rank % 4) FAIL(HYMBA_ERR_UNSUPPORTED, "dt_rank must be a multiple of 4 (16-byte rows of W_dt)");
  if (xdbl_width(c) % 4) FAIL(HYMBA_ERR_UNSUPPORTED, "dt_rank + 2*d_state must be a multiple of 4");
  if (c.n_heads / c.n_kv_heads > 8) FAIL(HYMBA_ERR_UNSUPPORTED, "more than 8 query heads per kv head");
  if (c.head_dim_qk > 128) FAIL(HYMBA_ERR_UNSUPPORTED, "head_dim_qk > 128");
  if (c.dtype == HYMBA_BF16) {
    if (c.head_dim_qk != 64 || c.head_dim_v != 128)
      FAIL(HYMBA_ERR_UNSUPPORTED, "bf16 attention kernel needs head_dim_qk 64 and head_dim_v 128");
    if (c.d_model % 64 || c.d_inner % 64)
      FAIL(HYMBA_ERR_UNSUPPORTED, "bf16 path needs d_model and d_inner multiples of 64");
  } else {
    if (c.head_dim_v > 256) FAIL(HYMBA_ERR_UNSUPPORTED, "fp32 attention needs head_dim_v <= 256");
    if (c.d_model % 4 || c.d_inner % 32 || c.head_dim_qk % 4 || c.head_dim_v % 4)
      FAIL(HYMBA_ERR_UNSUPPORTED, "fp32 path needs d_model %% 4, d_inner %% 32, head dims %% 4 == 0");
  }
  const void *ptrs[] = {w->w_in, w->conv_w, w->conv_b, w->w_x, w->w_dt, w->b_dt,
                        w->a_log, w->d_skip, w->beta_attn, w->beta_ssm, w->w_out};
  for (const void *p : ptrs) {
    if (!p) FAIL(HYMBA_ERR_INVALID_ARG, "null weight pointer");
    if (!aligned16(p)) FAIL(HYMBA_ERR_INVALID_ARG, "weight pointer not 16-byte aligned");
  }
  hymba_layer *L = new hymba_layer;
  L->cfg = c;
  L->w = *w;
  L->id = g_next_id.fetch_add(1);
  L->producer = nullptr;
  L->producer_id = 0;
  *out = L;
  return HYMBA_OK;
}

void hymba_layer_destroy(hymba_layer *layer) { delete layer; }

int hymba_layer_is_consumer(const hymba_layer *layer) { return layer && layer->producer ? 1 : 0; }

hymba_status hymba_kv_share_bind(hymba_layer *consumer, const hymba_layer *producer) {
  g_msg[0] = 0;
  if (!consumer || !producer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  if (consumer == producer) FAIL(HYMBA_ERR_NOT_BOUND, "a layer cannot share its own K/V");
  if (producer->producer) FAIL(HYMBA_ERR_NOT_BOUND, "producer is itself a consumer");
  const hymba_layer_config &c = consumer->cfg, &p = producer->cfg;
  if (c.n_kv_heads != p.n_kv_heads || c.head_dim_qk != p.head_dim_qk ||
      c.head_dim_v != p.head_dim_v || c.n_meta != p.n_meta || c.is_global != p.is_global ||
      (!c.is_global && c.window != p.window) || c.dtype != p.dtype || c.n_heads != p.n_heads)
    FAIL(HYMBA_ERR_NOT_BOUND, "producer and consumer differ in heads, head dims, n_meta, window, "
                              "global flag or dtype");
  consumer->producer = producer;
  consumer->producer_id = producer->id;
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// prefill
// ---------------------------------------------------------------------------
static hymba_status prefill_layout(const hymba_layer *layer, int batch, int n_tokens,
                                   hymba_prefill_layout *o, size_t *scan_floats) {
  if (!layer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  if (batch < 1 || n_tokens < 0) FAIL(HYMBA_ERR_INVALID_ARG, "batch < 1 or n_tokens < 0");
  const hymba_layer_config &c = layer->cfg;
  const long long L = (long long)c.n_meta + n_tokens;
  if (L < 1) FAIL(HYMBA_ERR_INVALID_ARG, "a sequence needs at least one row");
  if (L > (1LL << 30)) FAIL(HYMBA_ERR_UNSUPPORTED, "sequence too long");
  const size_t M = (size_t)batch * L, es = esize(c.dtype), E = c.d_inner;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  o->q = take(M * qk_width(c) * es);
  o->x_ssm = take(M * E * es);
  o->z = take(M * E * es);
  o->u = take(M * E * es);
  o->xdbl = take(M * xdbl_width(c) * 4);
  o->delta = take(M * E * es);
  o->y_ssm = take(M * E * es);
  o->o_attn = take(M * E * es);
  o->fused = take(M * E * es);
  size_t sf = scan_workspace_floats(batch, (int)L, c.d_inner, c.d_state, nullptr);
  if (scan_floats) *scan_floats = sf;
  take(sf * 4);  // scan chunk states, after `fused`
  o->total = off;
  return HYMBA_OK;
}

hymba_status hymba_layer_prefill_layout(const hymba_layer *layer, int batch, int n_tokens,
                                        hymba_prefill_layout *out) {
  g_msg[0] = 0;
  if (!out) FAIL(HYMBA_ERR_INVALID_ARG, "null output");
  return prefill_layout(layer, batch, n_tokens, out, nullptr);
}

hymba_status hymba_layer_prefill_workspace(const hymba_layer *layer, int batch, int n_tokens,
                                           size_t *bytes) {
  g_msg[0] = 0;
  if (!bytes) FAIL(HYMBA_ERR_INVALID_ARG, "null output");
  hymba_prefill_layout lay;
  hymba_status st = prefill_layout(layer, batch, n_tokens, &lay, nullptr);
  if (st != HYMBA_OK) return st;
  *bytes = lay.total;
  return HYMBA_OK;
}

static EpiSeg seg(void *ptr, long long ld_row, int col0, int col1, int f32, size_t es,
                  long long ld_group = 0, int inner = 0) {
  EpiSeg s;
  s.ptr = ptr;
  s.ld_row = ld_row;
  s.col0 = col0;
  s.col1 = col1;
  s.inner = inner > 0 ? inner : (col1 - col0);
  s.ld_group = ld_group;
  s.f32 = f32;
  const size_t b = f32 ? 4 : es;
  s.vec_ok = aligned16(ptr) && ((ld_row * b) % 16 == 0) && ((ld_group * b) % 16 == 0) &&
             (s.inner % 8 == 0);
  s.vec32 = s.vec_ok && (reinterpret_cast<uintptr_t>(ptr) % 32 == 0) && ((ld_row * b) % 32 == 0) &&
            ((ld_group * b) % 32 == 0) && (s.inner % 16 == 0) && (col0 % 16 == 0);
  return s;
}

static hymba_status gemm(const GemmArgs &g, hymba_dtype dt, cudaStream_t s) {
  if (dt == HYMBA_BF16) return gemm_tc(g, s);
  return gemm_simt_f32(g, s);
}

// in_proj: one GEMM, columns routed to Q, (K, V), x_ssm, z.
static Epilogue in_proj_epilogue(const hymba_layer_config &c, bool consumer, void *q, long long ldq,
                                 void *k, void *v, long long ld_k_row, long long ld_v_row,
                                 long long k_group, long long v_group, void *xs, void *z,
                                 long long ld_e) {
  Epilogue e{};
  const size_t es = esize(c.dtype);
  const int f32 = c.dtype == HYMBA_F32;
  int col = 0, n = 0;
  e.seg[n++] = seg(q, ldq, col, col + qk_width(c), f32, es);
  col += qk_width(c);
  if (!consumer) {
    e.seg[n++] = seg(k, ld_k_row, col, col + k_width(c), f32, es, k_group, k_group ? c.head_dim_qk : 0);
    col += k_width(c);
    e.seg[n++] = seg(v, ld_v_row, col, col + v_width(c), f32, es, v_group, v_group ? c.head_dim_v : 0);
    col += v_width(c);
  }
  e.seg[n++] = seg(xs, ld_e, col, col + c.d_inner, f32, es);
  col += c.d_inner;
  e.seg[n++] = seg(z, ld_e, col, col + c.d_inner, f32, es);
  e.nseg = n;
  return e;
}

hymba_status hymba_layer_prefill(hymba_layer *layer, int batch, int n_tokens, const void *x, void *y,
                                 hymba_kv_seq *kv, hymba_kv_cache *kv_cache,
                                 hymba_ssm_cache *ssm_cache, void *workspace, size_t workspace_bytes,
                                 hymba_stream_t stream_) {
  g_msg[0] = 0;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  hymba_prefill_layout lay;
  size_t scan_floats = 0;
  hymba_status st = prefill_layout(layer, batch, n_tokens, &lay, &scan_floats);
  if (st != HYMBA_OK) return st;
  const hymba_layer_config &c = layer->cfg;
  const bool consumer = layer->producer != nullptr;
  const int L = c.n_meta + n_tokens;
  const long long M = (long long)batch * L;
  const size_t es = esize(c.dtype);
  const int E = c.d_inner;
  if (!x || !y || !aligned16(x) || !aligned16(y)) FAIL(HYMBA_ERR_INVALID_ARG, "x/y null or misaligned");
  if (!kv || !kv->k || !kv->v || !aligned16(kv->k) || !aligned16(kv->v))
    FAIL(HYMBA_ERR_INVALID_ARG, "kv buffers null or misaligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  if (workspace_bytes < lay.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, lay.total);
  if (consumer) {
    if (kv->owner != layer->producer_id || layer->producer->id != layer->producer_id)
      FAIL(HYMBA_ERR_NOT_BOUND, "kv was not written by this consumer's producer");
    if (kv->batch != batch || kv->rows != L)
      FAIL(HYMBA_ERR_NOT_BOUND, "producer K/V has batch %d rows %d, consumer needs %d x %d",
           kv->batch, kv->rows, batch, L);
    if (kv_cache) FAIL(HYMBA_ERR_INVALID_ARG, "a consumer does not write a decode K/V store");
  }
  if (kv_cache) {
    const long long need = c.is_global ? L : (long long)c.n_meta + c.window;
    if (!kv_cache->k || !kv_cache->v || !aligned16(kv_cache->k) || !aligned16(kv_cache->v))
      FAIL(HYMBA_ERR_INVALID_ARG, "kv_cache buffers null or misaligned");
    if (kv_cache->batch != batch || kv_cache->capacity < need)
      FAIL(HYMBA_ERR_INVALID_ARG, "kv_cache batch %d capacity %d; need batch %d capacity >= %lld",
           kv_cache->batch, kv_cache->capacity, batch, need);
  }
  if (ssm_cache && (!ssm_cache->h || !ssm_cache->conv || !aligned16(ssm_cache->h) ||
                    !aligned16(ssm_cache->conv)))
    FAIL(HYMBA_ERR_INVALID_ARG, "ssm_cache buffers null or misaligned");

  char *ws = reinterpret_cast<char *>(workspace);
  void *q = ws + lay.q, *xs = ws + lay.x_ssm, *z = ws + lay.z, *u = ws + lay.u;
  float *xdbl = reinterpret_cast<float *>(ws + lay.xdbl);
  void *delta = ws + lay.delta, *yssm = ws + lay.y_ssm, *o = ws + lay.o_attn, *f = ws + lay.fused;
  float *scan_ws = reinterpret_cast<float *>(ws + lay.fused + up256((size_t)M * E * es));

  // 1. input projection (§2.1 W_in_proj) -> Q, K, V, x_ssm, z
  {
    ProfScope prof_scope(stream, "in_proj");
    GemmArgs g{};
    g.A = x;
    g.lda = c.d_model;
    g.B = layer->w.w_in;
    g.ldb = c.d_model;
    g.M = (int)M;
    g.N = qk_width(c) + (consumer ? 0 : k_width(c) + v_width(c)) + 2 * E;
    g.K = c.d_model;
    g.elem = (int)es;
    g.ksplit = 1;
    g.epi = in_proj_epilogue(c, consumer, q, qk_width(c), kv->k, kv->v, k_width(c), v_width(c), 0, 0,
                             xs, z, E);
    if (M > 0x7fffffffLL) FAIL(HYMBA_ERR_UNSUPPORTED, "too many rows");
    if ((st = gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 2. causal conv + SiLU -> u (and the conv state)
  {
    ProfScope prof_scope(stream, "conv");
    ConvArgs a{};
    a.x = xs;
    a.ld_x = E;
    a.u = u;
    a.w = layer->w.conv_w;
    a.bias = layer->w.conv_b;
    a.conv_state = ssm_cache ? ssm_cache->conv : nullptr;
    a.B = batch;
    a.L = L;
    a.E = E;
    a.K = c.d_conv;
    if ((st = conv_silu(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 3. x_proj -> [delta_r, B, C] (fp32)
  {
    ProfScope prof_scope(stream, "x_proj");
    GemmArgs g{};
    g.A = u;
    g.lda = E;
    g.B = layer->w.w_x;
    g.ldb = E;
    g.M = (int)M;
    g.N = xdbl_width(c);
    g.K = E;
    g.elem = (int)es;
    g.ksplit = 1;
    g.epi.seg[0] = seg(xdbl, xdbl_width(c), 0, xdbl_width(c), 1, es);
    g.epi.nseg = 1;
    if ((st = gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 4. dt_proj + bias + softplus -> delta (tf32 on the tensor cores for the bf16 path)
  {
    ProfScope prof_scope(stream, "dt_proj");
    GemmArgs g{};
    g.A = xdbl;
    g.lda = xdbl_width(c);
    g.B = layer->w.w_dt;
    g.ldb = c.dt_rank;
    g.M = (int)M;
    g.N = E;
    g.K = c.dt_rank;
    g.elem = 4;
    g.ksplit = 1;
    g.epi.seg[0] = seg(delta, E, 0, E, c.dtype == HYMBA_F32, es);
    g.epi.nseg = 1;
    g.epi.bias = layer->w.b_dt;
    g.epi.act = 1;
    st = c.dtype == HYMBA_BF16 ? gemm_tc(g, stream) : gemm_simt_f32(g, stream);
    if (st != HYMBA_OK) return st;
  }
  // 5. selective scan + D skip + SiLU(z) gate -> y_ssm (and the final state)
  {
    ProfScope prof_scope(stream, "scan");
    ScanArgs a{};
    a.u = u;
    a.delta = delta;
    a.z = z;
    a.ld_z = E;
    a.bc = xdbl;
    a.ld_bc = xdbl_width(c);
    a.bc_col = c.dt_rank;
    a.a_log = layer->w.a_log;
    a.d_skip = layer->w.d_skip;
    a.y = yssm;
    a.h_out = ssm_cache ? ssm_cache->h : nullptr;
    a.h_in = nullptr;
    a.B = batch;
    a.L = L;
    a.E = E;
    a.N = c.d_state;
    a.chunk_ws = scan_ws;
    if ((st = selective_scan(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 6. attention heads over the own or the producer's K/V
  {
    ProfScope prof_scope(stream, "attention");
    AttnArgs a{};
    a.q = q;
    a.k = kv->k;
    a.v = kv->v;
    a.o = o;
    a.B = batch;
    a.L = L;
    a.H = c.n_heads;
    a.Hkv = c.n_kv_heads;
    a.dqk = c.head_dim_qk;
    a.dv = c.head_dim_v;
    a.n_meta = c.n_meta;
    a.window = c.window;
    a.is_global = c.is_global;
    a.scale = score_scale(c);
    if ((st = attention_prefill(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 7. norm, beta, mean (Eq. 3)
  {
    ProfScope prof_scope(stream, "fuse");
    FuseArgs a{};
    a.o = o;
    a.y = yssm;
    a.beta_attn = layer->w.beta_attn;
    a.beta_ssm = layer->w.beta_ssm;
    a.f = f;
    a.M = (int)M;
    a.E = E;
    a.eps = c.rms_eps;
    if ((st = fuse_branches(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 8. output projection
  {
    ProfScope prof_scope(stream, "out_proj");
    GemmArgs g{};
    g.A = f;
    g.lda = E;
    g.B = layer->w.w_out;
    g.ldb = E;
    g.M = (int)M;
    g.N = c.d_model;
    g.K = E;
    g.elem = (int)es;
    g.ksplit = 1;
    g.epi.seg[0] = seg(y, c.d_model, 0, c.d_model, c.dtype == HYMBA_F32, es);
    g.epi.nseg = 1;
    if ((st = gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 9. decode K/V store
  if (kv_cache) {
    ProfScope prof_scope(stream, "kv_emit");
    KvEmitArgs a{};
    a.k_seq = kv->k;
    a.v_seq = kv->v;
    a.k_cache = kv_cache->k;
    a.v_cache = kv_cache->v;
    a.B = batch;
    a.L = L;
    a.Hkv = c.n_kv_heads;
    a.dqk = c.head_dim_qk;
    a.dv = c.head_dim_v;
    a.cap = kv_cache->capacity;
    a.n_meta = c.n_meta;
    a.window = c.window;
    a.is_global = c.is_global;
    if ((st = kv_cache_emit(a, c.dtype, stream)) != HYMBA_OK) return st;
    kv_cache->owner = layer->id;
  }
  if (!consumer) {
    kv->owner = layer->id;
    kv->batch = batch;
    kv->rows = L;
  }
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------
struct DecodeLayout {
  size_t q, x_ssm, z, u, xdbl, y_ssm, o, f, y32, part, total;
};

static DecodeLayout decode_layout(const hymba_layer_config &c, int batch, long long pos) {
  DecodeLayout d{};
  const size_t es = esize(c.dtype), E = c.d_inner, B = batch;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  d.q = take(B * qk_width(c) * es);
  d.x_ssm = take(B * E * es);
  d.z = take(B * E * es);
  d.u = take(B * E * es);
  d.xdbl = take(B * xdbl_width(c) * 4);  // xdbl and y32 adjacent: zeroed in one range
  d.y32 = take(B * c.d_model * 4);
  d.y_ssm = take(B * E * es);
  d.o = take(B * E * es);
  d.f = take(B * E * es);
  d.part = take(decode_attn_workspace_floats(batch, c.n_heads, c.head_dim_v, pos, c.n_meta,
                                             c.window, c.is_global) * 4);
  d.total = off;
  return d;
}

hymba_status hymba_layer_decode_workspace(const hymba_layer *layer, int batch, int64_t max_pos,
                                          size_t *bytes) {
  g_msg[0] = 0;
  if (!layer || !bytes || batch < 1) FAIL(HYMBA_ERR_INVALID_ARG, "null argument or batch < 1");
  const hymba_layer_config &c = layer->cfg;
  if (max_pos < c.n_meta) FAIL(HYMBA_ERR_INVALID_ARG, "max_pos %lld is a meta position", (long long)max_pos);
  if (c.is_global && max_pos >= (1LL << 24)) FAIL(HYMBA_ERR_UNSUPPORTED, "max_pos beyond 2^24");
  // the workspace grows with the number of visible keys, which never falls as pos grows
  *bytes = decode_layout(c, batch, max_pos).total;
  return HYMBA_OK;
}

hymba_status hymba_layer_decode_step(hymba_layer *layer, int batch, int64_t pos, const void *x_t,
                                     void *y_t, hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                                     void *workspace, size_t workspace_bytes,
                                     hymba_stream_t stream_) {
  g_msg[0] = 0;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!layer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  const hymba_layer_config &c = layer->cfg;
  const bool consumer = layer->producer != nullptr;
  if (batch < 1) FAIL(HYMBA_ERR_INVALID_ARG, "batch < 1");
  if (pos < c.n_meta) FAIL(HYMBA_ERR_INVALID_ARG, "pos %lld is a meta position", (long long)pos);
  if (c.is_global && pos >= (1LL << 24)) FAIL(HYMBA_ERR_UNSUPPORTED, "pos beyond 2^24");
  if (!x_t || !y_t || !aligned16(x_t) || !aligned16(y_t)) FAIL(HYMBA_ERR_INVALID_ARG, "x_t/y_t null or misaligned");
  if (!kv_cache || !kv_cache->k || !kv_cache->v || !aligned16(kv_cache->k) || !aligned16(kv_cache->v))
    FAIL(HYMBA_ERR_INVALID_ARG, "kv_cache null or misaligned");
  if (!ssm_cache || !ssm_cache->h || !ssm_cache->conv || !aligned16(ssm_cache->h) ||
      !aligned16(ssm_cache->conv))
    FAIL(HYMBA_ERR_INVALID_ARG, "ssm_cache null or misaligned");
  if (kv_cache->batch != batch) FAIL(HYMBA_ERR_INVALID_ARG, "kv_cache batch %d != %d", kv_cache->batch, batch);
  const long long need = c.is_global ? pos + 1 : (long long)c.n_meta + c.window;
  if (kv_cache->capacity < need)
    FAIL(HYMBA_ERR_INVALID_ARG, "kv_cache capacity %d < %lld", kv_cache->capacity, need);
  if (consumer && kv_cache->owner != layer->producer_id)
    FAIL(HYMBA_ERR_NOT_BOUND, "kv_cache is not this consumer's producer's store");
  if (!consumer && kv_cache->owner != 0 && kv_cache->owner != layer->id)
    FAIL(HYMBA_ERR_NOT_BOUND, "kv_cache belongs to another layer");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  const DecodeLayout d = decode_layout(c, batch, pos);
  if (workspace_bytes < d.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, d.total);

  const size_t es = esize(c.dtype);
  const int E = c.d_inner;
  char *ws = reinterpret_cast<char *>(workspace);
  void *q = ws + d.q, *xs = ws + d.x_ssm, *z = ws + d.z, *u = ws + d.u;
  float *xdbl = reinterpret_cast<float *>(ws + d.xdbl);
  void *yssm = ws + d.y_ssm, *o = ws + d.o, *f = ws + d.f;
  float *y32 = reinterpret_cast<float *>(ws + d.y32);
  float *part = reinterpret_cast<float *>(ws + d.part);
  hymba_status st;
  const long long slot = (c.is_global || pos < c.n_meta) ? pos : c.n_meta + (pos - c.n_meta) % c.window;
  const long long cap = kv_cache->capacity;

  // 1. input projection; a K/V owner writes this token's K/V straight into its slot
  {
    ProfScope prof_scope(stream, "dec_in_proj");
    GemmArgs g{};
    g.A = x_t;
    g.lda = c.d_model;
    g.B = layer->w.w_in;
    g.ldb = c.d_model;
    g.M = batch;
    g.N = qk_width(c) + (consumer ? 0 : k_width(c) + v_width(c)) + 2 * E;
    g.K = c.d_model;
    g.elem = (int)es;
    g.ksplit = 1;
    char *kbase = reinterpret_cast<char *>(kv_cache->k) + (size_t)slot * c.head_dim_qk * es;
    char *vbase = reinterpret_cast<char *>(kv_cache->v) + (size_t)slot * c.head_dim_v * es;
    g.epi = in_proj_epilogue(c, consumer, q, qk_width(c), kbase, vbase,
                             (long long)c.n_kv_heads * cap * c.head_dim_qk,
                             (long long)c.n_kv_heads * cap * c.head_dim_v,
                             cap * c.head_dim_qk, cap * c.head_dim_v, xs, z, E);
    // the split-K accumulators of x_proj and out_proj (adjacent) start at zero
    g.epi.zero = xdbl;
    g.epi.zero_n = (long long)((d.y32 - d.xdbl) / 4) + (long long)batch * c.d_model;
    if ((st = gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 2-5. SSM branch: conv + x_proj, then dt_proj + softplus + one scan step + gate
  {
    ProfScope prof_scope(stream, "dec_ssm");
    DecodeSsmArgs a{};
    a.x = xs;
    a.ld_x = E;
    a.z = z;
    a.ld_z = E;
    a.conv_state = ssm_cache->conv;
    a.conv_w = layer->w.conv_w;
    a.conv_b = layer->w.conv_b;
    a.w_x = layer->w.w_x;
    a.xdbl = xdbl;
    a.u = u;
    a.w_dt = layer->w.w_dt;
    a.b_dt = layer->w.b_dt;
    a.a_log = layer->w.a_log;
    a.d_skip = layer->w.d_skip;
    a.h = ssm_cache->h;
    a.y = yssm;
    a.B = batch;
    a.E = E;
    a.K = c.d_conv;
    a.R = c.dt_rank;
    a.N = c.d_state;
    if ((st = decode_ssm(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 6. single-query attention over the store
  int fuse_nchunks = 0;
  long long fuse_per = 1;
  {
    ProfScope prof_scope(stream, "dec_attention");
    DecodeAttnArgs a{};
    a.q = q;
    a.k_cache = kv_cache->k;
    a.v_cache = kv_cache->v;
    a.o = o;
    a.partial = part;
    a.B = batch;
    a.H = c.n_heads;
    a.Hkv = c.n_kv_heads;
    a.dqk = c.head_dim_qk;
    a.dv = c.head_dim_v;
    a.cap = kv_cache->capacity;
    a.pos = pos;
    a.n_meta = c.n_meta;
    a.window = c.window;
    a.is_global = c.is_global;
    a.scale = score_scale(c);
    // bf16: the fuse below merges the attention's run partials itself
    a.fuse_later = c.dtype == HYMBA_BF16 && c.n_heads <= 32 && c.head_dim_v == 128 &&
                   (long long)c.n_heads * c.head_dim_v == E;
    if ((st = attention_decode(a, c.dtype, stream)) != HYMBA_OK) return st;
    fuse_nchunks = a.nchunks_out;
    fuse_per = a.per_out;
  }
  // 7. norm, beta, mean
  if (fuse_nchunks > 0) {
    ProfScope prof_scope(stream, "dec_fuse");
    FuseDecodeArgs a{};
    a.part = part;
    a.H = c.n_heads;
    a.Hkv = c.n_kv_heads;
    a.dv = c.head_dim_v;
    a.nchunks = fuse_nchunks;
    a.per = fuse_per;
    a.y = yssm;
    a.beta_attn = layer->w.beta_attn;
    a.beta_ssm = layer->w.beta_ssm;
    a.f = f;
    a.B = batch;
    a.eps = c.rms_eps;
    if ((st = fuse_decode(a, stream)) != HYMBA_OK) return st;
  } else {
    ProfScope prof_scope(stream, "dec_fuse");
    FuseArgs a{};
    a.o = o;
    a.y = yssm;
    a.beta_attn = layer->w.beta_attn;
    a.beta_ssm = layer->w.beta_ssm;
    a.f = f;
    a.M = batch;
    a.E = E;
    a.eps = c.rms_eps;
    if ((st = fuse_branches(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // 8. output projection, split over K into fp32, then to the storage dtype
  {
    ProfScope prof_scope(stream, "dec_out_proj");
    const int ksplit = 4;
    GemmArgs g{};
    g.A = f;
    g.lda = E;
    g.B = layer->w.w_out;
    g.ldb = E;
    g.M = batch;
    g.N = c.d_model;
    g.K = E;
    g.elem = (int)es;
    g.ksplit = ksplit;
    g.epi.seg[0] = seg(y32, c.d_model, 0, c.d_model, 1, es);
    g.epi.nseg = 1;
    g.epi.atomic = 1;
    if ((st = gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
    if ((st = convert_f32_to(y32, y_t, (long long)batch * c.d_model, c.dtype, stream)) != HYMBA_OK)
      return st;
  }
  if (!consumer) kv_cache->owner = layer->id;
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// status and diagnostics
// ---------------------------------------------------------------------------
hymba_status hymba_stream_status(hymba_stream_t stream) {
  g_msg[0] = 0;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) FAIL(HYMBA_ERR_CUDA, "%s", cudaGetErrorString(e));
  e = cudaGetLastError();
  if (e != cudaSuccess) FAIL(HYMBA_ERR_CUDA, "%s", cudaGetErrorString(e));
  const unsigned err = take_error_gemm() | take_error_attn();
  if (err & kErrTimeoutHost) FAIL(HYMBA_ERR_TIMEOUT, "a device-side wait timed out");
  return HYMBA_OK;
}

hymba_status hymba_profile_enable(int on) {
  g_msg[0] = 0;
  Profiler &p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (on && p.pool.empty()) {
    p.pool.resize(kProfEvents);
    for (auto &e : p.pool)
      if (cudaEventCreate(&e) != cudaSuccess) {
        p.pool.clear();
        FAIL(HYMBA_ERR_CUDA, "cudaEventCreate failed");
      }
  }
  p.on = on != 0;
  return HYMBA_OK;
}

hymba_status hymba_profile_collect(hymba_profile_entry *out, int max, int *n) {
  g_msg[0] = 0;
  if (!n || (max > 0 && !out)) FAIL(HYMBA_ERR_INVALID_ARG, "null output");
  Profiler &p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  struct Acc {
    int calls = 0;
    unsigned long long kernels = 0;
    double ms = 0;
  };
  std::map<std::string, Acc> acc;
  std::vector<std::string> order;
  for (const ProfRecord &r : p.recs) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) FAIL(HYMBA_ERR_CUDA, "event sync failed");
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.start, r.stop);
    if (!acc.count(r.name)) order.push_back(r.name);
    Acc &a = acc[r.name];
    a.calls += 1;
    a.kernels += r.kernels;
    a.ms += ms;
  }
  p.recs.clear();
  p.next = 0;
  int k = 0;
  for (const std::string &name : order) {
    if (k >= max) break;
    snprintf(out[k].name, sizeof(out[k].name), "%s", name.c_str());
    out[k].calls = acc[name].calls;
    out[k].kernels = (int)acc[name].kernels;
    out[k].total_ms = acc[name].ms;
    ++k;
  }
  *n = k;
  return HYMBA_OK;
}

hymba_status hymba_debug_mask_bitmap(int L, int n_meta, int window, int is_global, uint32_t *bits,
                                     uint8_t *tile_class, hymba_stream_t stream) {
  g_msg[0] = 0;
  if (L < 1 || n_meta < 0 || (!is_global && window < 1)) FAIL(HYMBA_ERR_INVALID_ARG, "bad mask shape");
  if (!bits) FAIL(HYMBA_ERR_INVALID_ARG, "null bits");
  return mask_bitmap(L, n_meta, window, is_global, bits, tile_class,
                     reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
