// Host side of the C ABI declared in include/hymba.h: argument validation,
// workspace layout and the launch sequence of one hybrid-head layer
// (Hymba §2.1 Eq. 1-3; §2.2 local/global attention and cross-layer KV sharing;
// §2.3 meta tokens).  Nothing here computes the layer: every step is a kernel.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
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

constexpr long long kDefaultWaitLimit = 1000000000LL;  // ~0.5 s at 2 GHz
constexpr long long kMinWaitLimit = 100000LL;
static std::atomic<long long> g_wait_limit{0};  // 0: not set through the ABI
static long long env_wait_limit() {
  static const long long v = [] {
    const char *e = getenv("HYMBA_WAIT_LIMIT");
    return e ? atoll(e) : 0LL;
  }();
  return v;
}
long long wait_limit_cycles() {
  long long v = g_wait_limit.load(std::memory_order_relaxed);
  if (v <= 0) v = env_wait_limit();
  if (v <= 0) v = kDefaultWaitLimit;
  return std::max(v, kMinWaitLimit);
}
static thread_local bool t_pdl = false;
bool pdl_enabled() { return t_pdl; }
PdlScope::PdlScope() : prev(t_pdl) { t_pdl = true; }
PdlScope::~PdlScope() { t_pdl = prev; }

static thread_local bool t_prio_set = false;
static thread_local int t_prio = 0;
bool launch_priority(int *prio) {
  if (t_prio_set) *prio = t_prio;
  return t_prio_set;
}
PrioScope::PrioScope(int prio) : prev_set(t_prio_set), prev(t_prio) {
  t_prio_set = true;
  t_prio = prio;
}
PrioScope::~PrioScope() {
  t_prio_set = prev_set;
  t_prio = prev;
}

static std::atomic<int> g_stall{0};
int take_debug_stall() {
  int v = g_stall.load();
  while (v > 0 && !g_stall.compare_exchange_weak(v, v - 1)) {
  }
  return v > 0 ? 1 : 0;
}

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

// Side stream of the concurrent prefill (branch_chunks >= 2) and its events: one fork
// event, then per chunk one after its dt_proj and one after its scan.
constexpr int kMaxBranchChunks = 8;
constexpr int kBranchEvents = 1 + 2 * kMaxBranchChunks;
struct BranchStreams {
  cudaStream_t side = nullptr;
  cudaEvent_t ev[kBranchEvents] = {};
  int prio_hi = 0;  // the greatest scheduling priority of the device (main chain)
  bool ready = false;
};

struct hymba_layer {
  hymba_layer_config cfg;
  hymba_layer_weights w;
  uint64_t id;
  const hymba_layer *producer;  // non-null for a K/V-sharing consumer
  uint64_t producer_id;
  BranchStreams br;
};

static void branch_release(BranchStreams &b) {
  for (cudaEvent_t &e : b.ev)
    if (e) {
      cudaEventDestroy(e);
      e = nullptr;
    }
  if (b.side) cudaStreamDestroy(b.side);
  b.side = nullptr;
  b.ready = false;
}
// Creates the side stream (lowest priority, non-blocking) and the events on the current
// device.  False (and nothing kept) when that fails, e.g. without a device.
static bool branch_create(BranchStreams &b) {
  if (b.ready) return true;
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
      cudaStreamCreateWithPriority(&b.side, cudaStreamNonBlocking, least) != cudaSuccess) {
    cudaGetLastError();
    b.side = nullptr;
    return false;
  }
  for (cudaEvent_t &e : b.ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      e = nullptr;
      branch_release(b);
      return false;
    }
  b.prio_hi = greatest;
  b.ready = true;
  return true;
}

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
  if (!(c.rope_base >= 0.f) || !std::isfinite(c.rope_base)) FAIL(HYMBA_ERR_INVALID_ARG, "rope_base < 0");
  if (c.rope_base > 0.f && (c.rope_base <= 1.f || (c.head_dim_qk & (c.head_dim_qk - 1)) || c.head_dim_qk < 2))
    FAIL(HYMBA_ERR_UNSUPPORTED, "rotary embedding needs a base > 1 and a power-of-two head_dim_qk");
  if (c.branch_chunks < 0 || c.branch_chunks > kMaxBranchChunks)
    FAIL(HYMBA_ERR_INVALID_ARG, "branch_chunks %d outside 0..%d", c.branch_chunks, kMaxBranchChunks);
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
  // the concurrent prefill's side stream, on the current device (retried at the first
  // prefill where no device was usable here)
  if (c.branch_chunks >= 2) branch_create(L->br);
  *out = L;
  return HYMBA_OK;
}

void hymba_layer_destroy(hymba_layer *layer) {
  if (!layer) return;
  branch_release(layer->br);
  delete layer;
}

int hymba_layer_is_consumer(const hymba_layer *layer) { return layer && layer->producer ? 1 : 0; }

hymba_status hymba_kv_share_bind(hymba_layer *consumer, const hymba_layer *producer) {
  g_msg[0] = 0;
  if (!consumer || !producer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  if (consumer == producer) FAIL(HYMBA_ERR_NOT_BOUND, "a layer cannot share its own K/V");
  if (producer->producer) FAIL(HYMBA_ERR_NOT_BOUND, "producer is itself a consumer");
  const hymba_layer_config &c = consumer->cfg, &p = producer->cfg;
  if (c.n_kv_heads != p.n_kv_heads || c.head_dim_qk != p.head_dim_qk ||
      c.head_dim_v != p.head_dim_v || c.n_meta != p.n_meta || c.is_global != p.is_global ||
      (!c.is_global && c.window != p.window) || c.dtype != p.dtype || c.n_heads != p.n_heads ||
      c.rope_base != p.rope_base)
    FAIL(HYMBA_ERR_NOT_BOUND, "producer and consumer differ in heads, head dims, n_meta, window, "
                              "global flag, dtype or rotary base");
  consumer->producer = producer;
  consumer->producer_id = producer->id;
  return HYMBA_OK;
}

// ---------------------------------------------------------------------------
// prefill
// ---------------------------------------------------------------------------
// Work counters of the persistent kernels in a prefill's workspace (one per launch).
constexpr int kSchedCounters = 64;

// Batch chunks of the concurrent prefill: *n chunks of *bc sequences (the last one may be
// shorter); n = 1 runs the serial order.
static void branch_split(const hymba_layer_config &c, int batch, int *n, int *bc) {
  const int want = c.branch_chunks >= 2 ? std::min(c.branch_chunks, batch) : 1;
  *bc = (batch + want - 1) / want;
  *n = (batch + *bc - 1) / *bc;
}

// Workspace of a prefill whose intermediates have `rows` rows per sequence: all L = m + n
// rows, or the n real rows when the meta rows come from a precomputed meta cache.
static hymba_status prefill_layout_rows(const hymba_layer *layer, int batch, long long rows,
                                        hymba_prefill_layout *o, size_t *scan_floats) {
  if (!layer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  if (batch < 1) FAIL(HYMBA_ERR_INVALID_ARG, "batch < 1");
  const hymba_layer_config &c = layer->cfg;
  if (rows < 1) FAIL(HYMBA_ERR_INVALID_ARG, "a sequence needs at least one row");
  if (rows + c.n_meta > (1LL << 30)) FAIL(HYMBA_ERR_UNSUPPORTED, "sequence too long");
  const size_t M = (size_t)batch * rows, es = esize(c.dtype), E = c.d_inner;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  o->q = take(M * qk_width(c) * es);
  o->x_ssm = take(M * E * es);
  o->gate = take(M * E * es);
  o->u = take(M * E * es);
  o->xdbl = take(M * xdbl_width(c) * 4);
  o->delta = take(M * E * es);
  o->y_ssm = take(M * E * es);
  o->o_attn = take(M * E * es);
  o->fused = take(M * E * es);
  // the scan's chunk states for the whole batch (a concurrent prefill's batch chunks scan
  // with the whole batch's time chunks, one after another, in the same region)
  size_t sf = scan_workspace_floats(batch, (int)rows, c.d_inner, c.d_state, nullptr);
  if (scan_floats) *scan_floats = sf;
  take(sf * 4);  // scan chunk states, after `fused`
  // rotary table of the positions 0..L-1 (none without a rotary embedding)
  o->rope = take(c.rope_base > 0.f ? (size_t)(rows + c.n_meta) * (c.head_dim_qk / 2) * 8 : 0);
  o->sched = take(kSchedCounters * sizeof(unsigned));
  o->total = off;
  return HYMBA_OK;
}

static hymba_status prefill_layout(const hymba_layer *layer, int batch, int n_tokens,
                                   hymba_prefill_layout *o, size_t *scan_floats) {
  if (!layer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  if (n_tokens < 0) FAIL(HYMBA_ERR_INVALID_ARG, "n_tokens < 0");
  return prefill_layout_rows(layer, batch, (long long)layer->cfg.n_meta + n_tokens, o, scan_floats);
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
  EpiSeg s{};
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
// The decode step's projections: a few activation rows against a whole weight matrix.
static bool gemm_decode_streams(const GemmArgs &g, hymba_dtype dt) { return dt == HYMBA_BF16 && g.M <= 256; }
static hymba_status gemm_decode(const GemmArgs &g, hymba_dtype dt, cudaStream_t s) {
  if (gemm_decode_streams(g, dt)) return gemm_ws(g, s);
  return gemm(g, dt, s);
}

// in_proj: one GEMM, columns routed to Q, (K, V), x_ssm and the gate SiLU(z).
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
  // the gate's SiLU is applied here, so the scan multiplies by a stored SiLU(z)
  e.seg[n] = seg(z, ld_e, col, col + c.d_inner, f32, es);
  e.seg[n++].act = 2;
  e.nseg = n;
  return e;
}

// The launch sequence of one prefill over `rows` rows per sequence whose first row is X~
// position q_off: the whole sequence (q_off = 0, rows = L), or its real rows after a
// precomputed meta cache (q_off = m, rows = n; the meta rows' K/V are then in kv already,
// and their SSM state and conv history come from `meta`).  Arguments validated.
struct PrefillRun {
  const void *x;  // [B, rows, d]
  void *y;        // [B, rows, d]
  int rows, q_off;
  const float *h0;    // broadcast initial SSM state [E, N] or null
  const void *conv0;  // broadcast conv history [K-1, E] or null
  bool meta;          // the meta-cache precompute: its steps are profiled under "meta_*" names
  const void *resid;  // [B, rows, d] added to the output by the output projection (block) or null
};
// Profiler step name of a prefill step (the meta-cache precompute has its own names).
static const char *step_name(const PrefillRun &r, int step) {
  static const char *const names[2][9] = {
      {"in_proj", "conv", "x_proj", "dt_proj", "scan", "attention", "fuse", "out_proj", "kv_emit"},
      {"meta_in_proj", "meta_conv", "meta_x_proj", "meta_dt_proj", "meta_scan", "meta_attention",
       "meta_fuse", "meta_out_proj", "meta_kv_emit"}};
  return names[r.meta ? 1 : 0][step];
}

// Byte pointer to element `elems` of a buffer of `es`-byte elements.
static void *elem_at(void *base, long long elems, size_t es) {
  return base ? reinterpret_cast<char *>(base) + elems * (long long)es : nullptr;
}
static const void *celem_at(const void *base, long long elems, size_t es) {
  return base ? reinterpret_cast<const char *>(base) + elems * (long long)es : nullptr;
}

static hymba_status prefill_run(hymba_layer *layer, int batch, const PrefillRun &r, hymba_kv_seq *kv,
                                hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache, void *workspace,
                                const hymba_prefill_layout &lay, cudaStream_t stream) {
  const hymba_layer_config &c = layer->cfg;
  const bool consumer = layer->producer != nullptr;
  const int L = r.q_off + r.rows;
  const long long M = (long long)batch * r.rows;
  const size_t es = esize(c.dtype);
  const int E = c.d_inner;
  const int XW = xdbl_width(c);
  hymba_status st;
  if (M > 0x7fffffffLL) FAIL(HYMBA_ERR_UNSUPPORTED, "too many rows");

  char *ws = reinterpret_cast<char *>(workspace);
  void *q = ws + lay.q, *xs = ws + lay.x_ssm, *z = ws + lay.gate, *u = ws + lay.u;
  float *xdbl = reinterpret_cast<float *>(ws + lay.xdbl);
  void *delta = ws + lay.delta, *yssm = ws + lay.y_ssm, *o = ws + lay.o_attn, *f = ws + lay.fused;
  float *scan_ws = reinterpret_cast<float *>(ws + lay.fused + up256((size_t)M * E * es));
  // work counters of this call's persistent GEMMs, one per launch
  unsigned *sched = reinterpret_cast<unsigned *>(ws + lay.sched);
  int next_ctr = 0;
  auto take_ctr = [&]() -> unsigned * { return next_ctr < kSchedCounters ? sched + next_ctr++ : nullptr; };
  if (cudaMemsetAsync(sched, 0, kSchedCounters * sizeof(unsigned), stream) != cudaSuccess)
    FAIL(HYMBA_ERR_CUDA, "cudaMemsetAsync(work counters): %s", cudaGetErrorString(cudaGetLastError()));

  // rotary table of positions 0..L-1 (§2.5 RoPE), shared by every sequence
  float2 *rope_tab = nullptr;
  if (c.rope_base > 0.f) {
    rope_tab = reinterpret_cast<float2 *>(ws + lay.rope);
    if ((st = rope_table(rope_tab, L, 0, c.head_dim_qk, c.rope_base, stream)) != HYMBA_OK) return st;
  }

  // The steps over the sequences b0 .. b0+nb-1 (rows m0 = b0 * rows .. of the intermediates).
  // 1. input projection (§2.1 W_in_proj) -> Q, K, V, x_ssm, SiLU(z); K and V go to their
  //    rows q_off.. of each sequence of the full-length K/V
  auto in_proj = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 0));
    const long long m0 = (long long)b0 * r.rows;
    GemmArgs g{};
    g.A = celem_at(r.x, m0 * c.d_model, es);
    g.lda = c.d_model;
    g.B = layer->w.w_in;
    g.ldb = c.d_model;
    g.M = (int)((long long)nb * r.rows);
    g.N = qk_width(c) + (consumer ? 0 : k_width(c) + v_width(c)) + 2 * E;
    g.K = c.d_model;
    g.elem = (int)es;
    g.epi = in_proj_epilogue(c, consumer, elem_at(q, m0 * qk_width(c), es), qk_width(c),
                             consumer ? nullptr : elem_at(kv->k, (long long)b0 * L * k_width(c), es),
                             consumer ? nullptr : elem_at(kv->v, (long long)b0 * L * v_width(c), es),
                             k_width(c), v_width(c), 0, 0, elem_at(xs, m0 * E, es), elem_at(z, m0 * E, es), E);
    if (!consumer && r.q_off > 0) {
      g.epi.seg[1].rmap = g.epi.seg[2].rmap = 1;
      g.epi.rmap_rows = r.rows;
      g.epi.rmap_stride = L;
      g.epi.rmap_off = r.q_off;
    }
    if (rope_tab) {
      // Q and K rotated in the epilogue, positions q_off.. of each sequence
      g.epi.rope_tab = rope_tab;
      g.epi.rope_rows = r.rows;
      g.epi.rope_off = r.q_off;
      g.epi.rope_hd = c.head_dim_qk;
      g.epi.seg[0].rope = 1;
      if (!consumer) g.epi.seg[1].rope = 1;
    }
    g.tile_ctr = take_ctr();
    return gemm(g, c.dtype, s);
  };
  // 2. causal conv + SiLU -> u (and the conv state)
  auto conv = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 1));
    const long long m0 = (long long)b0 * r.rows;
    ConvArgs a{};
    a.x = elem_at(xs, m0 * E, es);
    a.ld_x = E;
    a.u = elem_at(u, m0 * E, es);
    a.w = layer->w.conv_w;
    a.bias = layer->w.conv_b;
    a.conv_state = ssm_cache ? elem_at(ssm_cache->conv, (long long)b0 * (c.d_conv - 1) * E, es) : nullptr;
    a.hist = r.conv0;
    a.B = nb;
    a.L = r.rows;
    a.E = E;
    a.K = c.d_conv;
    return conv_silu(a, c.dtype, s);
  };
  // 3. x_proj -> [delta_r, B, C] (fp32)
  auto x_proj = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 2));
    const long long m0 = (long long)b0 * r.rows;
    GemmArgs g{};
    g.A = elem_at(u, m0 * E, es);
    g.lda = E;
    g.B = layer->w.w_x;
    g.ldb = E;
    g.M = (int)((long long)nb * r.rows);
    g.N = XW;
    g.K = E;
    g.elem = (int)es;
    g.epi.seg[0] = seg(xdbl + m0 * XW, XW, 0, XW, 1, es);
    g.epi.nseg = 1;
    g.tile_ctr = take_ctr();
    return gemm(g, c.dtype, s);
  };
  // 4. dt_proj + bias + softplus -> delta (tf32 on the tensor cores for the bf16 path)
  auto dt_proj = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 3));
    const long long m0 = (long long)b0 * r.rows;
    GemmArgs g{};
    g.A = xdbl + m0 * XW;
    g.lda = XW;
    g.B = layer->w.w_dt;
    g.ldb = c.dt_rank;
    g.M = (int)((long long)nb * r.rows);
    g.N = E;
    g.K = c.dt_rank;
    g.elem = 4;
    g.epi.seg[0] = seg(elem_at(delta, m0 * E, es), E, 0, E, c.dtype == HYMBA_F32, es);
    g.epi.nseg = 1;
    g.epi.bias = layer->w.b_dt;
    g.epi.act = 1;
    g.tile_ctr = take_ctr();
    return c.dtype == HYMBA_BF16 ? gemm_tc(g, s) : gemm_simt_f32(g, s);
  };
  // 5. selective scan + D skip, times the gate SiLU(z) -> y_ssm (and the final state)
  auto scan = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 4));
    const long long m0 = (long long)b0 * r.rows;
    ScanArgs a{};
    a.u = elem_at(u, m0 * E, es);
    a.delta = elem_at(delta, m0 * E, es);
    a.z = elem_at(z, m0 * E, es);
    a.ld_z = E;
    a.bc = xdbl + m0 * XW;
    a.ld_bc = XW;
    a.bc_col = c.dt_rank;
    a.a_log = layer->w.a_log;
    a.d_skip = layer->w.d_skip;
    a.y = elem_at(yssm, m0 * E, es);
    a.h_out = ssm_cache ? ssm_cache->h + (long long)b0 * E * c.d_state : nullptr;
    a.h_in = r.h0;
    a.h_in_bstride = 0;
    a.B = nb;
    a.L = r.rows;
    a.E = E;
    a.N = c.d_state;
    a.chunk_ws = scan_ws;
    a.time_chunks = scan_time_chunks(batch, r.rows, E);
    return selective_scan(a, c.dtype, s);
  };
  // 6. attention heads over the own or the producer's K/V
  auto attention = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 5));
    const long long m0 = (long long)b0 * r.rows;
    AttnArgs a{};
    a.q = elem_at(q, m0 * qk_width(c), es);
    a.k = elem_at(kv->k, (long long)b0 * L * k_width(c), es);
    a.v = elem_at(kv->v, (long long)b0 * L * v_width(c), es);
    a.o = elem_at(o, m0 * E, es);
    a.B = nb;
    a.L = L;
    a.q_off = r.q_off;
    a.Lq = r.rows;
    a.H = c.n_heads;
    a.Hkv = c.n_kv_heads;
    a.dqk = c.head_dim_qk;
    a.dv = c.head_dim_v;
    a.n_meta = c.n_meta;
    a.window = c.window;
    a.is_global = c.is_global;
    a.scale = score_scale(c);
    return attention_prefill(a, c.dtype, s);
  };
  // 7. norm, beta, mean (Eq. 3)
  auto fuse = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 6));
    const long long m0 = (long long)b0 * r.rows;
    FuseArgs a{};
    a.o = elem_at(o, m0 * E, es);
    a.y = elem_at(yssm, m0 * E, es);
    a.beta_attn = layer->w.beta_attn;
    a.beta_ssm = layer->w.beta_ssm;
    a.f = elem_at(f, m0 * E, es);
    a.M = (int)((long long)nb * r.rows);
    a.E = E;
    a.eps = c.rms_eps;
    return fuse_branches(a, c.dtype, s);
  };
  // 8. output projection (plus the residual in a block)
  auto out_proj = [&](int b0, int nb, cudaStream_t s) -> hymba_status {
    ProfScope prof_scope(s, step_name(r, 7));
    const long long m0 = (long long)b0 * r.rows;
    GemmArgs g{};
    g.A = elem_at(f, m0 * E, es);
    g.lda = E;
    g.B = layer->w.w_out;
    g.ldb = E;
    g.M = (int)((long long)nb * r.rows);
    g.N = c.d_model;
    g.K = E;
    g.elem = (int)es;
    g.epi.seg[0] = seg(elem_at(r.y, m0 * c.d_model, es), c.d_model, 0, c.d_model, c.dtype == HYMBA_F32, es);
    g.epi.seg[0].resid = celem_at(r.resid, m0 * c.d_model, es);
    g.epi.seg[0].ld_resid = c.d_model;
    g.epi.nseg = 1;
    g.stall = take_debug_stall();
    g.tile_ctr = take_ctr();
    return gemm(g, c.dtype, s);
  };

  int nch = 1, bc = batch;
  branch_split(c, batch, &nch, &bc);
  if (nch > 1 && !branch_create(layer->br)) {
    set_error("could not create the concurrent prefill's side stream: %s", cudaGetErrorString(cudaGetLastError()));
    return HYMBA_ERR_CUDA;
  }
  if (nch == 1) {
    // serial order on the caller's stream
    if ((st = in_proj(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = conv(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = x_proj(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = dt_proj(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = scan(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = attention(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = fuse(0, batch, stream)) != HYMBA_OK) return st;
    if ((st = out_proj(0, batch, stream)) != HYMBA_OK) return st;
  } else {
    // The two branches side by side: chunk k's scan (MUFU-bound, one small CTA per SM beside
    // a GEMM CTA) runs on the low-priority side stream while the caller's stream, at the
    // device's highest priority, runs chunk k's attention and chunk k+1's projections; the
    // last chunk's scan runs beside the first chunks' output projections.
    BranchStreams &br = layer->br;
    auto check = [](cudaError_t e, const char *what) -> hymba_status {
      if (e == cudaSuccess) return HYMBA_OK;
      set_error("%s failed: %s", what, cudaGetErrorString(e));
      return HYMBA_ERR_CUDA;
    };
    cudaEvent_t ev_fork = br.ev[0];
    if ((st = check(cudaEventRecord(ev_fork, stream), "cudaEventRecord")) != HYMBA_OK) return st;
    if ((st = check(cudaStreamWaitEvent(br.side, ev_fork, 0), "cudaStreamWaitEvent")) != HYMBA_OK) return st;
    // Per chunk: in_proj .. dt_proj, fork its scan, then its attention.  (Measured against
    // every chunk's in_proj first, and every chunk's attention after all projections:
    // 158.2 against 162.9 and 162.3 ms per headline step.)
    for (int k = 0; k < nch; ++k) {
      const int b0 = k * bc, nb = std::min(bc, batch - b0);
      cudaEvent_t ev_dt = br.ev[1 + 2 * k], ev_scan = br.ev[2 + 2 * k];
      {
        PrioScope hi(br.prio_hi);
        if ((st = in_proj(b0, nb, stream)) != HYMBA_OK) return st;
        if ((st = conv(b0, nb, stream)) != HYMBA_OK) return st;
        if ((st = x_proj(b0, nb, stream)) != HYMBA_OK) return st;
        if ((st = dt_proj(b0, nb, stream)) != HYMBA_OK) return st;
      }
      if ((st = check(cudaEventRecord(ev_dt, stream), "cudaEventRecord")) != HYMBA_OK) return st;
      if ((st = check(cudaStreamWaitEvent(br.side, ev_dt, 0), "cudaStreamWaitEvent")) != HYMBA_OK) return st;
      if ((st = scan(b0, nb, br.side)) != HYMBA_OK) return st;
      if ((st = check(cudaEventRecord(ev_scan, br.side), "cudaEventRecord")) != HYMBA_OK) return st;
      PrioScope hi(br.prio_hi);
      if ((st = attention(b0, nb, stream)) != HYMBA_OK) return st;
    }
    for (int k = 0; k < nch; ++k) {
      const int b0 = k * bc, nb = std::min(bc, batch - b0);
      if ((st = check(cudaStreamWaitEvent(stream, br.ev[2 + 2 * k], 0), "cudaStreamWaitEvent")) != HYMBA_OK)
        return st;
      PrioScope hi(br.prio_hi);
      if ((st = fuse(b0, nb, stream)) != HYMBA_OK) return st;
      if ((st = out_proj(b0, nb, stream)) != HYMBA_OK) return st;
    }
  }
  // 9. decode K/V store
  if (kv_cache) {
    ProfScope prof_scope(stream, step_name(r, 8));
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

// Checks shared by both prefill entry points: K/V of L rows per sequence (written by an
// owner, stamped by the producer for a consumer), the optional decode stores.
static hymba_status check_prefill_kv(const hymba_layer *layer, int batch, int L, const hymba_kv_seq *kv,
                                     const hymba_kv_cache *kv_cache, const hymba_ssm_cache *ssm_cache) {
  const hymba_layer_config &c = layer->cfg;
  const bool consumer = layer->producer != nullptr;
  if (!kv || !kv->k || !kv->v || !aligned16(kv->k) || !aligned16(kv->v))
    FAIL(HYMBA_ERR_INVALID_ARG, "kv buffers null or misaligned");
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
  return HYMBA_OK;
}

hymba_status hymba_layer_prefill(hymba_layer *layer, int batch, int n_tokens, const void *x, void *y,
                                 hymba_kv_seq *kv, hymba_kv_cache *kv_cache,
                                 hymba_ssm_cache *ssm_cache, void *workspace, size_t workspace_bytes,
                                 hymba_stream_t stream_) {
  g_msg[0] = 0;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  hymba_prefill_layout lay;
  hymba_status st = prefill_layout(layer, batch, n_tokens, &lay, nullptr);
  if (st != HYMBA_OK) return st;
  const int L = layer->cfg.n_meta + n_tokens;
  if (!x || !y || !aligned16(x) || !aligned16(y)) FAIL(HYMBA_ERR_INVALID_ARG, "x/y null or misaligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  if (workspace_bytes < lay.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, lay.total);
  if ((st = check_prefill_kv(layer, batch, L, kv, kv_cache, ssm_cache)) != HYMBA_OK) return st;
  PrefillRun r{};
  r.x = x;
  r.y = y;
  r.rows = L;
  r.q_off = 0;
  return prefill_run(layer, batch, r, kv, kv_cache, ssm_cache, workspace, lay, stream);
}

// ---------------------------------------------------------------------------
// meta-token cache (§2.3: the meta rows do not depend on the input, so their K/V, SSM
// state and conv history are computed once and every prefill starts from them)
// ---------------------------------------------------------------------------
hymba_status hymba_layer_meta_workspace(const hymba_layer *layer, size_t *bytes) {
  g_msg[0] = 0;
  if (!layer || !bytes) FAIL(HYMBA_ERR_INVALID_ARG, "null argument");
  if (layer->cfg.n_meta < 1) FAIL(HYMBA_ERR_INVALID_ARG, "the layer has no meta tokens");
  return hymba_layer_prefill_workspace(layer, 1, 0, bytes);
}

hymba_status hymba_layer_meta_precompute(hymba_layer *layer, const void *x_meta, hymba_meta_cache *meta,
                                         const hymba_meta_cache *producer_meta, void *workspace,
                                         size_t workspace_bytes, hymba_stream_t stream) {
  g_msg[0] = 0;
  if (!layer || !meta) FAIL(HYMBA_ERR_INVALID_ARG, "null argument");
  const hymba_layer_config &c = layer->cfg;
  const bool consumer = layer->producer != nullptr;
  if (c.n_meta < 1) FAIL(HYMBA_ERR_INVALID_ARG, "the layer has no meta tokens");
  if (!meta->y || !meta->h || !meta->conv || !aligned16(meta->y) || !aligned16(meta->h) ||
      !aligned16(meta->conv))
    FAIL(HYMBA_ERR_INVALID_ARG, "meta cache y/h/conv null or misaligned");
  hymba_kv_seq kv{};
  if (consumer) {
    if (!producer_meta || producer_meta->owner != layer->producer_id)
      FAIL(HYMBA_ERR_NOT_BOUND, "a consumer needs its producer's meta cache");
    kv.k = producer_meta->k;
    kv.v = producer_meta->v;
    kv.batch = 1;
    kv.rows = c.n_meta;
    kv.owner = producer_meta->owner;
  } else {
    if (producer_meta) FAIL(HYMBA_ERR_INVALID_ARG, "a layer that owns its K/V takes no producer cache");
    kv.k = meta->k;
    kv.v = meta->v;
  }
  hymba_ssm_cache ssm{meta->h, meta->conv};
  meta->owner = 0;
  hymba_prefill_layout lay;
  hymba_status st = prefill_layout(layer, 1, 0, &lay, nullptr);
  if (st != HYMBA_OK) return st;
  if (!x_meta || !aligned16(x_meta)) FAIL(HYMBA_ERR_INVALID_ARG, "x_meta null or misaligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  if (workspace_bytes < lay.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, lay.total);
  if ((st = check_prefill_kv(layer, 1, c.n_meta, &kv, nullptr, &ssm)) != HYMBA_OK) return st;
  PrefillRun r{};
  r.x = x_meta;
  r.y = meta->y;
  r.rows = c.n_meta;
  r.q_off = 0;
  r.meta = true;
  st = prefill_run(layer, 1, r, &kv, nullptr, &ssm, workspace, lay, reinterpret_cast<cudaStream_t>(stream));
  if (st != HYMBA_OK) return st;
  meta->owner = layer->id;
  return HYMBA_OK;
}

hymba_status hymba_layer_prefill_cached_workspace(const hymba_layer *layer, int batch, int n_tokens,
                                                  size_t *bytes) {
  g_msg[0] = 0;
  if (!bytes) FAIL(HYMBA_ERR_INVALID_ARG, "null output");
  if (n_tokens < 1) FAIL(HYMBA_ERR_INVALID_ARG, "n_tokens < 1");
  hymba_prefill_layout lay;
  hymba_status st = prefill_layout_rows(layer, batch, n_tokens, &lay, nullptr);
  if (st != HYMBA_OK) return st;
  *bytes = lay.total;
  return HYMBA_OK;
}

hymba_status hymba_layer_prefill_cached(hymba_layer *layer, int batch, int n_tokens, const void *x,
                                        void *y, const hymba_meta_cache *meta, hymba_kv_seq *kv,
                                        hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                                        void *workspace, size_t workspace_bytes, hymba_stream_t stream_) {
  g_msg[0] = 0;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!layer) FAIL(HYMBA_ERR_INVALID_ARG, "null layer");
  const hymba_layer_config &c = layer->cfg;
  const bool consumer = layer->producer != nullptr;
  if (n_tokens < 1) FAIL(HYMBA_ERR_INVALID_ARG, "n_tokens < 1");
  if (c.n_meta < 1) FAIL(HYMBA_ERR_INVALID_ARG, "the layer has no meta tokens");
  hymba_prefill_layout lay;
  hymba_status st = prefill_layout_rows(layer, batch, n_tokens, &lay, nullptr);
  if (st != HYMBA_OK) return st;
  const int L = c.n_meta + n_tokens;
  if (!x || !y || !aligned16(x) || !aligned16(y)) FAIL(HYMBA_ERR_INVALID_ARG, "x/y null or misaligned");
  if (!meta || meta->owner != layer->id) FAIL(HYMBA_ERR_NOT_BOUND, "meta cache not computed by this layer");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  if (workspace_bytes < lay.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, lay.total);
  if ((st = check_prefill_kv(layer, batch, L, kv, kv_cache, ssm_cache)) != HYMBA_OK) return st;
  if (!consumer) {
    // the meta rows' K/V into rows 0..m-1 of every sequence
    if (!meta->k || !meta->v || !aligned16(meta->k) || !aligned16(meta->v))
      FAIL(HYMBA_ERR_INVALID_ARG, "meta cache K/V null or misaligned");
    if ((k_width(c) * esize(c.dtype)) % 16 || (v_width(c) * esize(c.dtype)) % 16)
      FAIL(HYMBA_ERR_UNSUPPORTED, "K/V rows must be multiples of 16 bytes");
    ProfScope prof_scope(stream, "kv_meta");
    KvBroadcastArgs a{};
    a.k_meta = meta->k;
    a.v_meta = meta->v;
    a.k_seq = kv->k;
    a.v_seq = kv->v;
    a.B = batch;
    a.L = L;
    a.m = c.n_meta;
    a.kw = k_width(c);
    a.vw = v_width(c);
    if ((st = kv_broadcast_meta(a, c.dtype, stream)) != HYMBA_OK) return st;
  }
  PrefillRun r{};
  r.x = x;
  r.y = y;
  r.rows = n_tokens;
  r.q_off = c.n_meta;
  r.h0 = meta->h;
  r.conv0 = meta->conv;
  return prefill_run(layer, batch, r, kv, kv_cache, ssm_cache, workspace, lay, stream);
}

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------
struct DecodeLayout {
  size_t q, x_ssm, z, u, xacc, y_ssm, o, f, part, rope, total;
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
  d.xacc = take(B * xdbl_width(c) * 8 + B * 4);  // x_proj result as 64-bit fixed point, then [B] flags
  d.y_ssm = take(B * E * es);
  d.o = take(B * E * es);
  d.f = take(B * E * es);
  d.part = take(decode_attn_workspace_floats(batch, c.n_heads, c.head_dim_v, pos, c.n_meta,
                                             c.window, c.is_global) * 4);
  d.rope = take(c.rope_base > 0.f ? (size_t)(c.head_dim_qk / 2) * 8 : 0);
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

// The decode step of the mixer; `resid` (optional, [batch, d_model]) is added to its output
// by the output projection (the block's residual).
static hymba_status decode_run(hymba_layer *layer, int batch, int64_t pos, const void *x_t, void *y_t,
                               const void *resid, hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                               void *workspace, size_t workspace_bytes, cudaStream_t stream) {
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
  long long *xacc = reinterpret_cast<long long *>(ws + d.xacc);
  void *yssm = ws + d.y_ssm, *o = ws + d.o, *f = ws + d.f;
  float *part = reinterpret_cast<float *>(ws + d.part);
  hymba_status st;
  const long long slot = (c.is_global || pos < c.n_meta) ? pos : c.n_meta + (pos - c.n_meta) % c.window;
  const long long cap = kv_cache->capacity;
  // the step's kernels are launched programmatically: each starts while its predecessor ends
  PdlScope pdl;

  const long long xacc_n = (long long)batch * xdbl_width(c);
  unsigned *xbad = reinterpret_cast<unsigned *>(xacc + xacc_n);
  bool xacc_zeroed = false;
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
    char *kbase = reinterpret_cast<char *>(kv_cache->k) + (size_t)slot * c.head_dim_qk * es;
    char *vbase = reinterpret_cast<char *>(kv_cache->v) + (size_t)slot * c.head_dim_v * es;
    g.epi = in_proj_epilogue(c, consumer, q, qk_width(c), kbase, vbase,
                             (long long)c.n_kv_heads * cap * c.head_dim_qk,
                             (long long)c.n_kv_heads * cap * c.head_dim_v,
                             cap * c.head_dim_qk, cap * c.head_dim_v, xs, z, E);
    if (c.rope_base > 0.f) {
      // the new token's Q and K rotated by the angles of its position
      float2 *tab = reinterpret_cast<float2 *>(ws + d.rope);
      if ((st = rope_table(tab, 1, pos, c.head_dim_qk, c.rope_base, stream)) != HYMBA_OK) return st;
      g.epi.rope_tab = tab;
      g.epi.rope_rows = 1;
      g.epi.rope_off = 0;
      g.epi.rope_hd = c.head_dim_qk;
      g.epi.seg[0].rope = 1;
      if (!consumer) g.epi.seg[1].rope = 1;
    }
    if (gemm_decode_streams(g, c.dtype)) {  // its launch also zeroes the x_proj accumulator
      g.epi.zero = reinterpret_cast<float *>(xacc);
      g.epi.zero_n = 2 * xacc_n + batch;  // the 64-bit sums (pairs of zero words), then the flags
      xacc_zeroed = true;
    }
    if ((st = gemm_decode(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  // The two branches side by side when the handle has a side stream (branch_chunks >= 2):
  // the SSM branch there, at the highest priority (short launches), beside the attention.
  BranchStreams &br = layer->br;
  const bool side_by_side = c.branch_chunks >= 2 && br.ready;
  cudaStream_t ssm_stream = side_by_side ? br.side : stream;
  if (side_by_side) {
    if (cudaEventRecord(br.ev[0], stream) != cudaSuccess || cudaStreamWaitEvent(br.side, br.ev[0], 0) != cudaSuccess)
      FAIL(HYMBA_ERR_CUDA, "decode fork: %s", cudaGetErrorString(cudaGetLastError()));
  }
  // 2-5. SSM branch: conv + SiLU and x_proj (per-CTA shares added as fixed-point integers
  //      into an accumulator zeroed by the input projection's launch or a memset), then
  //      dt_proj + softplus + one scan step + gate
  {
    ProfScope prof_scope(ssm_stream, "dec_ssm");
    PrioScope prio(side_by_side ? br.prio_hi : 0);
    DecodeSsmArgs a{};
    a.x = xs;
    a.ld_x = E;
    a.z = z;
    a.ld_z = E;
    a.conv_state = ssm_cache->conv;
    a.conv_w = layer->w.conv_w;
    a.conv_b = layer->w.conv_b;
    a.xacc = xacc;
    a.xbad = xbad;
    a.w_x = layer->w.w_x;
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
    if (!xacc_zeroed &&
        cudaMemsetAsync(xacc, 0, (size_t)xacc_n * sizeof(long long) + (size_t)batch * 4, ssm_stream) != cudaSuccess)
      FAIL(HYMBA_ERR_CUDA, "cudaMemsetAsync(x_proj accumulator): %s", cudaGetErrorString(cudaGetLastError()));
    if ((st = decode_conv_xproj(a, c.dtype, ssm_stream)) != HYMBA_OK) return st;
    if ((st = decode_scan(a, c.dtype, ssm_stream)) != HYMBA_OK) return st;
  }
  if (side_by_side && cudaEventRecord(br.ev[1], br.side) != cudaSuccess)
    FAIL(HYMBA_ERR_CUDA, "decode join: %s", cudaGetErrorString(cudaGetLastError()));
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
  if (side_by_side && cudaStreamWaitEvent(stream, br.ev[1], 0) != cudaSuccess)
    FAIL(HYMBA_ERR_CUDA, "decode join: %s", cudaGetErrorString(cudaGetLastError()));
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
  // 8. output projection, straight into y_t
  {
    ProfScope prof_scope(stream, "dec_out_proj");
    GemmArgs g{};
    g.A = f;
    g.lda = E;
    g.B = layer->w.w_out;
    g.ldb = E;
    g.M = batch;
    g.N = c.d_model;
    g.K = E;
    g.elem = (int)es;
    g.epi.seg[0] = seg(y_t, c.d_model, 0, c.d_model, c.dtype == HYMBA_F32, es);
    g.epi.seg[0].resid = resid;
    g.epi.seg[0].ld_resid = c.d_model;
    g.epi.nseg = 1;
    if ((st = gemm_decode(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  if (!consumer) kv_cache->owner = layer->id;
  return HYMBA_OK;
}

hymba_status hymba_layer_decode_step(hymba_layer *layer, int batch, int64_t pos, const void *x_t,
                                     void *y_t, hymba_kv_cache *kv_cache, hymba_ssm_cache *ssm_cache,
                                     void *workspace, size_t workspace_bytes,
                                     hymba_stream_t stream) {
  g_msg[0] = 0;
  return decode_run(layer, batch, pos, x_t, y_t, nullptr, kv_cache, ssm_cache, workspace, workspace_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// the Hymba block: x + mixer(norm1(x)), then + MLP(norm2(.)) (Fig. 4 (b); Table 11)
// ---------------------------------------------------------------------------
static hymba_status check_block(const hymba_layer *layer, const hymba_block_weights *bw) {
  if (!layer || !bw) FAIL(HYMBA_ERR_INVALID_ARG, "null layer or block weights");
  const hymba_layer_config &c = layer->cfg;
  if (!bw->norm1 || !bw->norm2 || !bw->w_gate_up || !bw->w_down || !aligned16(bw->norm1) ||
      !aligned16(bw->norm2) || !aligned16(bw->w_gate_up) || !aligned16(bw->w_down))
    FAIL(HYMBA_ERR_INVALID_ARG, "block weights null or misaligned");
  if (bw->mlp_hidden < 8 || bw->mlp_hidden % 8) FAIL(HYMBA_ERR_UNSUPPORTED, "mlp_hidden must be a multiple of 8");
  const int V = c.dtype == HYMBA_BF16 ? 8 : 4;
  if (c.d_model % V || c.d_model / V > 256) FAIL(HYMBA_ERR_UNSUPPORTED, "d_model too wide for the block's norm");
  return HYMBA_OK;
}

// Block workspace: the mixer's own, then the normed rows [M, d] and the MLP's hidden rows [M, F].
struct BlockLayout {
  size_t mixer, xn, hid, total;
};
static BlockLayout block_layout(size_t mixer_bytes, const hymba_layer_config &c, long long M, int F) {
  BlockLayout b{};
  b.mixer = 0;
  b.xn = up256(mixer_bytes);
  b.hid = b.xn + up256((size_t)M * c.d_model * esize(c.dtype));
  b.total = b.hid + up256((size_t)M * F * esize(c.dtype));
  return b;
}

hymba_status hymba_block_prefill_workspace(const hymba_layer *layer, int mlp_hidden, int batch, int n_tokens,
                                           size_t *bytes) {
  g_msg[0] = 0;
  if (!bytes || mlp_hidden < 1) FAIL(HYMBA_ERR_INVALID_ARG, "null output or mlp_hidden < 1");
  hymba_prefill_layout lay;
  hymba_status st = prefill_layout(layer, batch, n_tokens, &lay, nullptr);
  if (st != HYMBA_OK) return st;
  const long long M = (long long)batch * (layer->cfg.n_meta + n_tokens);
  *bytes = block_layout(lay.total, layer->cfg, M, mlp_hidden).total;
  return HYMBA_OK;
}

// MLP of M rows: hid = SiLU(hn W_gate^T) * (hn W_up^T); y += hid W_down^T (y holds h).
static hymba_status block_mlp(const hymba_layer *layer, const hymba_block_weights *bw, long long M, const void *hn,
                              void *hid, void *y, bool decode, cudaStream_t stream) {
  const hymba_layer_config &c = layer->cfg;
  const size_t es = esize(c.dtype);
  const int F = bw->mlp_hidden;
  hymba_status st;
  {
    ProfScope prof_scope(stream, decode ? "dec_mlp_up" : "mlp_up");
    GemmArgs g{};
    g.A = hn;
    g.lda = c.d_model;
    g.B = bw->w_gate_up;
    g.ldb = c.d_model;
    g.M = (int)M;
    g.N = 2 * F;
    g.K = c.d_model;
    g.elem = (int)es;
    g.epi.seg[0] = seg(hid, F, 0, 2 * F, c.dtype == HYMBA_F32, es);
    g.epi.seg[0].act = 3;
    g.epi.nseg = 1;
    if ((st = decode ? gemm_decode(g, c.dtype, stream) : gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  {
    ProfScope prof_scope(stream, decode ? "dec_mlp_down" : "mlp_down");
    GemmArgs g{};
    g.A = hid;
    g.lda = F;
    g.B = bw->w_down;
    g.ldb = F;
    g.M = (int)M;
    g.N = c.d_model;
    g.K = F;
    g.elem = (int)es;
    g.epi.seg[0] = seg(y, c.d_model, 0, c.d_model, c.dtype == HYMBA_F32, es);
    g.epi.seg[0].resid = y;  // in place: each element is read, then written, by one thread
    g.epi.seg[0].ld_resid = c.d_model;
    g.epi.nseg = 1;
    if ((st = decode ? gemm_decode(g, c.dtype, stream) : gemm(g, c.dtype, stream)) != HYMBA_OK) return st;
  }
  return HYMBA_OK;
}

hymba_status hymba_block_prefill(hymba_layer *layer, const hymba_block_weights *bw, int batch, int n_tokens,
                                 const void *x, void *y, hymba_kv_seq *kv, hymba_kv_cache *kv_cache,
                                 hymba_ssm_cache *ssm_cache, void *workspace, size_t workspace_bytes,
                                 hymba_stream_t stream_) {
  g_msg[0] = 0;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  hymba_status st = check_block(layer, bw);
  if (st != HYMBA_OK) return st;
  hymba_prefill_layout lay;
  if ((st = prefill_layout(layer, batch, n_tokens, &lay, nullptr)) != HYMBA_OK) return st;
  const hymba_layer_config &c = layer->cfg;
  const int L = c.n_meta + n_tokens;
  const long long M = (long long)batch * L;
  const BlockLayout bl = block_layout(lay.total, c, M, bw->mlp_hidden);
  if (!x || !y || !aligned16(x) || !aligned16(y) || x == y) FAIL(HYMBA_ERR_INVALID_ARG, "x/y null, misaligned or the same");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  if (workspace_bytes < bl.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, bl.total);
  if ((st = check_prefill_kv(layer, batch, L, kv, kv_cache, ssm_cache)) != HYMBA_OK) return st;
  char *ws = reinterpret_cast<char *>(workspace);
  void *xn = ws + bl.xn, *hid = ws + bl.hid;
  {
    ProfScope prof_scope(stream, "norm1");
    if ((st = rms_norm_rows(x, bw->norm1, xn, M, c.d_model, c.rms_eps, c.dtype, stream)) != HYMBA_OK) return st;
  }
  PrefillRun r{};
  r.x = xn;
  r.y = y;
  r.rows = L;
  r.q_off = 0;
  r.resid = x;  // y = x + mixer(norm1(x))
  if ((st = prefill_run(layer, batch, r, kv, kv_cache, ssm_cache, workspace, lay, stream)) != HYMBA_OK) return st;
  {
    ProfScope prof_scope(stream, "norm2");
    if ((st = rms_norm_rows(y, bw->norm2, xn, M, c.d_model, c.rms_eps, c.dtype, stream)) != HYMBA_OK) return st;
  }
  return block_mlp(layer, bw, M, xn, hid, y, false, stream);
}

hymba_status hymba_block_decode_workspace(const hymba_layer *layer, int mlp_hidden, int batch, int64_t max_pos,
                                          size_t *bytes) {
  g_msg[0] = 0;
  size_t mixer = 0;
  hymba_status st = hymba_layer_decode_workspace(layer, batch, max_pos, &mixer);
  if (st != HYMBA_OK) return st;
  if (mlp_hidden < 1) FAIL(HYMBA_ERR_INVALID_ARG, "mlp_hidden < 1");
  *bytes = block_layout(mixer, layer->cfg, batch, mlp_hidden).total;
  return HYMBA_OK;
}

hymba_status hymba_block_decode_step(hymba_layer *layer, const hymba_block_weights *bw, int batch, int64_t pos,
                                     const void *x_t, void *y_t, hymba_kv_cache *kv_cache,
                                     hymba_ssm_cache *ssm_cache, void *workspace, size_t workspace_bytes,
                                     hymba_stream_t stream_) {
  g_msg[0] = 0;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  hymba_status st = check_block(layer, bw);
  if (st != HYMBA_OK) return st;
  const hymba_layer_config &c = layer->cfg;
  if (batch < 1 || pos < c.n_meta) FAIL(HYMBA_ERR_INVALID_ARG, "batch < 1 or pos is a meta position");
  const size_t mixer = decode_layout(c, batch, pos).total;
  const BlockLayout bl = block_layout(mixer, c, batch, bw->mlp_hidden);
  if (!x_t || !y_t || !aligned16(x_t) || !aligned16(y_t) || x_t == y_t)
    FAIL(HYMBA_ERR_INVALID_ARG, "x_t/y_t null, misaligned or the same");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    FAIL(HYMBA_ERR_INVALID_ARG, "workspace null or not 256-byte aligned");
  if (workspace_bytes < bl.total)
    FAIL(HYMBA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, bl.total);
  char *ws = reinterpret_cast<char *>(workspace);
  void *xn = ws + bl.xn, *hid = ws + bl.hid;
  {
    ProfScope prof_scope(stream, "dec_norm1");
    if ((st = rms_norm_rows(x_t, bw->norm1, xn, batch, c.d_model, c.rms_eps, c.dtype, stream)) != HYMBA_OK)
      return st;
  }
  if ((st = decode_run(layer, batch, pos, xn, y_t, x_t, kv_cache, ssm_cache, workspace, mixer, stream)) !=
      HYMBA_OK)
    return st;
  {
    ProfScope prof_scope(stream, "dec_norm2");
    if ((st = rms_norm_rows(y_t, bw->norm2, xn, batch, c.d_model, c.rms_eps, c.dtype, stream)) != HYMBA_OK)
      return st;
  }
  return block_mlp(layer, bw, batch, xn, hid, y_t, true, stream);
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

hymba_status hymba_set_wait_limit(int64_t cycles, int64_t *applied) {
  g_msg[0] = 0;
  if (cycles < 0) FAIL(HYMBA_ERR_INVALID_ARG, "negative wait limit");
  g_wait_limit.store(cycles);
  if (applied) *applied = wait_limit_cycles();
  return HYMBA_OK;
}

hymba_status hymba_debug_stall_next_prefill(int count) {
  g_msg[0] = 0;
  if (count < 0) FAIL(HYMBA_ERR_INVALID_ARG, "negative count");
  g_stall.store(count);
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

hymba_status hymba_debug_mask_bitmap(int L, int n_meta, int window, int is_global, int path,
                                     uint32_t *bits, uint8_t *tile_class, hymba_stream_t stream) {
  g_msg[0] = 0;
  if (L < 1 || n_meta < 0 || (!is_global && window < 1)) FAIL(HYMBA_ERR_INVALID_ARG, "bad mask shape");
  if (path != 0 && path != 1) FAIL(HYMBA_ERR_INVALID_ARG, "path must be 0 (tensor-core) or 1 (fp32)");
  if (!bits) FAIL(HYMBA_ERR_INVALID_ARG, "null bits");
  return mask_bitmap(L, n_meta, window, is_global, path, bits, tile_class,
                     reinterpret_cast<cudaStream_t>(stream));
}

hymba_status hymba_debug_decode_mask(int64_t pos, int n_meta, int window, int is_global,
                                     int capacity, uint32_t *bits, hymba_stream_t stream) {
  g_msg[0] = 0;
  if (n_meta < 0 || pos < n_meta || (!is_global && window < 1) || capacity < 1)
    FAIL(HYMBA_ERR_INVALID_ARG, "bad decode mask shape");
  const long long need = is_global ? pos + 1 : (long long)n_meta + window;
  if (capacity < need) FAIL(HYMBA_ERR_INVALID_ARG, "capacity %d < %lld slots read", capacity, need);
  if (!bits) FAIL(HYMBA_ERR_INVALID_ARG, "null bits");
  return decode_mask(pos, n_meta, window, is_global, capacity, bits,
                     reinterpret_cast<cudaStream_t>(stream));
}

hymba_status hymba_debug_exp2_poly(int degree, const float *x, float *y, int64_t n,
                                   hymba_stream_t stream) {
  g_msg[0] = 0;
  if (degree != 3 && degree != 5) FAIL(HYMBA_ERR_INVALID_ARG, "degree must be 3 or 5");
  if (n < 0 || (n > 0 && (!x || !y))) FAIL(HYMBA_ERR_INVALID_ARG, "null buffer or n < 0");
  return exp2_poly_eval(degree, x, y, n, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
