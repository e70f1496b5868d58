// Internal launcher interface between the C ABI host layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "hymba.h"

namespace hymba {

// One flag per device ordinal, set once a kernel's launch attributes have been configured
// on that device.  Atomic, so that first launches from several host threads at once are
// well defined: each may then set the (idempotent) attribute.  Ordinals past the table
// are never marked, so their attributes are set on every launch.
struct DeviceOnce {
  static constexpr int kMaxDevices = 256;
  std::atomic<bool> flag[kMaxDevices] = {};
  bool done(int dev) const {
    return dev >= 0 && dev < kMaxDevices && flag[dev].load(std::memory_order_acquire);
  }
  void mark(int dev) {
    if (dev >= 0 && dev < kMaxDevices) flag[dev].store(true, std::memory_order_release);
  }
};


// Programmatic dependent launch.  While a PdlScope is alive on the calling thread, the
// kernels launched through launch_kernel (and the weight-streaming GEMM) carry the
// programmatic-serialisation attribute, so that each may start its prologue while the
// kernel before it in the stream finishes; every such kernel calls pdl_wait() (see
// common.cuh) in every CTA before it touches memory that another kernel writes.
bool pdl_enabled();
struct PdlScope {
  bool prev;
  PdlScope();
  ~PdlScope();
  PdlScope(const PdlScope &) = delete;
  PdlScope &operator=(const PdlScope &) = delete;
};
// Launch priority.  While a PrioScope is alive on the calling thread, the kernels launched
// through launch_kernel (and the tensor-core GEMMs) carry that scheduling priority (lower
// numbers first), so that their pending CTAs take freed SM space before those of a
// lower-priority kernel running beside them.
bool launch_priority(int *prio);
struct PrioScope {
  bool prev_set;
  int prev;
  explicit PrioScope(int prio);
  ~PrioScope();
  PrioScope(const PrioScope &) = delete;
  PrioScope &operator=(const PrioScope &) = delete;
};
// The launch attributes of the calling thread's scopes, appended to attr[n..]; returns n.
inline unsigned launch_attrs(cudaLaunchAttribute *attr, unsigned n) {
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  int prio = 0;
  if (launch_priority(&prio)) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = prio;
    ++n;
  }
  return n;
}
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = launch_attrs(attr, 0);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Where a GEMM output column goes.  Column c in [col0, col1) of the product is
// written to  ptr + row*ld_row + ((c-col0)/inner)*ld_group + (c-col0)%inner
// (element offsets), as fp32 (f32 = 1) or bf16 (f32 = 0).
struct EpiSeg {
  void *ptr;
  long long ld_row;
  long long ld_group;
  int col0, col1;
  int inner;
  int f32;
  int vec_ok;  // 16-byte aligned rows/groups: 8-column vector stores allowed
  int vec32;   // 32-byte aligned rows/groups: whole-sector (256-bit) stores allowed
  int act;     // activation of this segment's columns (after the GEMM's own): 0 none, 2 SiLU,
               // 3 gated SiLU: product columns (2i, 2i+1) = (gate_i, up_i) give output column
               // i = SiLU(gate_i) * up_i (the segment's destination has half its columns)
  int rmap;    // 1: rows go through the epilogue's row remap
  int rope;    // 1: rotary position embedding of this segment's heads (pairs of columns)
  const void *resid;  // optional residual added to the result: same dtype as the destination,
  long long ld_resid; // [rows, col1 - col0] with row stride ld_resid (one group only)
};
// Epilogue features a GEMM instantiation carries (bit flags).
constexpr int kEpiRoute = 1;  // several segments, row remap, rotary embedding
constexpr int kEpiResid = 2;  // residual add
constexpr int kEpiGlu = 4;    // gated SiLU of column pairs
constexpr int kEpiSoftplus = 8;  // bias + softplus into one plain segment (dt_proj)

struct Epilogue {
  EpiSeg seg[5];
  int nseg;
  // Row remap of the segments with rmap set: product row r is stored at row
  // (r / rmap_rows) * rmap_stride + r % rmap_rows + rmap_off of that segment (rows of
  // sequences that sit after a prefix of rmap_off rows in a longer destination).
  int rmap_rows;
  long long rmap_stride;
  int rmap_off;
  // Rotary position embedding of the segments with rope set: product row r is at position
  // r % rope_rows + rope_off; column pair i of a head (head width rope_hd, a power of two)
  // is rotated by rope_tab[pos * rope_hd / 2 + i] = (cos, sin).
  const float2 *rope_tab;
  int rope_rows, rope_off, rope_hd;
  const float *bias;  // per product column (nullable)
  int act;            // 0 = identity, 1 = softplus
  float *zero;        // weight-streaming GEMM: zero_n floats set to 0 by the launch (after it
  long long zero_n;   // has waited for the preceding kernel); for the next kernel's accumulator
};

// out[m, n] = epi( sum_k A[m, k] * B[n, k] )  (A: [M, K], B: [N, K], row-major)
struct GemmArgs {
  const void *A;
  long long lda;
  const void *B;
  long long ldb;
  int M, N, K;
  int elem;    // 2: bf16 operands; 4: fp32 operands
  Epilogue epi;
  int stall;   // tensor-core path: the MMA warp waits for an arrival that never comes
  unsigned *tile_ctr;  // tensor-core path: a zeroed counter -> tiles handed out in the order
                       // CTAs ask for them (CTAs that start late take fewer); null -> each
                       // CTA takes every gridDim-th tile
};

// Tensor-core path (tcgen05 + TMA).  elem 2 -> kind::f16 (bf16), 4 -> kind::tf32.
hymba_status gemm_tc(const GemmArgs &g, cudaStream_t s);
// Weight-streaming tensor-core path for at most 256 activation rows (decode): clusters of
// CTAs split K, partials reduced through distributed shared memory.  bf16 only.
hymba_status gemm_ws(const GemmArgs &g, cudaStream_t s);
// fp32 CUDA-core path for the fp32 storage configuration.
hymba_status gemm_simt_f32(const GemmArgs &g, cudaStream_t s);

// ---- SSM branch -----------------------------------------------------------
struct ConvArgs {
  const void *x;      // [B, L, E] rows of x_ssm, row stride ld_x elements
  long long ld_x;
  void *u;            // [B, L, E] dense
  const float *w;     // [E, K]
  const float *bias;  // [E]
  void *conv_state;   // optional [B, K-1, E]: the last K-1 rows of x
  const void *hist;   // optional [K-1, E]: the rows before row 0 (the same for every
                      // sequence; zero rows when null)
  int B, L, E, K;
};
hymba_status conv_silu(const ConvArgs &a, hymba_dtype dt, cudaStream_t s);

struct ScanArgs {
  const void *u;       // [B, L, E]
  const void *delta;   // [B, L, E]
  const void *z;       // [B, L, E] the gate SiLU(z), row stride ld_z
  long long ld_z;
  const float *bc;     // [B*L, ld_bc] fp32; B at column bc_col, C at bc_col + N
  long long ld_bc;
  int bc_col;
  const float *a_log;  // [E, N]
  const float *d_skip; // [E]
  void *y;             // [B, L, E] gated output
  float *h_out;        // optional [B, E, N] final state
  const float *h_in;   // optional initial state: [E, N] per sequence, h_in_bstride floats
  long long h_in_bstride;  // apart (0: one state for every sequence); zero when null
  int B, L, E, N;
  float *chunk_ws;     // workspace for the chunked scan (see scan_workspace_floats)
  int time_chunks;     // time chunks of the scan (0: chosen from B, L, E); a batch split into
                       // parts passes the whole batch's count, so every part rounds alike
};
size_t scan_workspace_floats(int B, int L, int E, int N, int *chunks_out);
// The scan's time chunks for B sequences of L steps and E channels.
int scan_time_chunks(int B, int L, int E);
hymba_status selective_scan(const ScanArgs &a, hymba_dtype dt, cudaStream_t s);

// ---- fused norm / beta / mean -------------------------------------------
struct FuseArgs {
  const void *o;       // [M, E]
  const void *y;       // [M, E]
  const float *beta_attn, *beta_ssm;
  void *f;             // [M, E]
  int M, E;
  float eps;
};
hymba_status fuse_branches(const FuseArgs &a, hymba_dtype dt, cudaStream_t s);
// Decode: the attention output is merged from the run partials of the tensor-core
// decode attention (per (sequence, head): nchunks slots of (max, sum, O[dv]), the run
// starts at chunk 0 and at every chunk whose item index is a multiple of per), then
// fused with the SSM branch as fuse_branches does.
struct FuseDecodeArgs {
  const float *part;
  int H, Hkv, dv, nchunks;
  long long per;
  const void *y;       // [B, H*dv]
  const float *beta_attn, *beta_ssm;
  void *f;             // [B, H*dv]
  int B;
  float eps;
};
hymba_status fuse_decode(const FuseDecodeArgs &a, cudaStream_t s);

// y = x / rms(x) * w per row of d elements (the block's pre-norms).
hymba_status rms_norm_rows(const void *x, const float *w, void *y, long long M, int d, float eps, hymba_dtype dt,
                           cudaStream_t s);

// ---- attention -----------------------------------------------------------
// Queries are the positions q_off .. q_off + Lq - 1 of sequences of L = q_off + Lq rows,
// stored from row 0 of q and o; keys are all L positions.
struct AttnArgs {
  const void *q;   // [B, Lq, H*dqk]
  const void *k;   // [B, L, Hkv*dqk]
  const void *v;   // [B, L, Hkv*dv]
  void *o;         // [B, Lq, H*dv]
  int B, L, H, Hkv, dqk, dv;
  int q_off, Lq;
  int n_meta, window, is_global;
  float scale;
};
hymba_status attention_prefill(const AttnArgs &a, hymba_dtype dt, cudaStream_t s);

// Copies one sequence's first m rows of K and V (the meta rows) into every sequence.
struct KvBroadcastArgs {
  const void *k_meta, *v_meta;  // [m, Hkv*dqk], [m, Hkv*dv]
  void *k_seq, *v_seq;          // [B, L, Hkv*dqk], [B, L, Hkv*dv]
  int B, L, m, kw, vw;          // kw, vw: row widths in elements
};
hymba_status kv_broadcast_meta(const KvBroadcastArgs &a, hymba_dtype dt, cudaStream_t s);

struct KvEmitArgs {
  const void *k_seq, *v_seq;  // [B, L, Hkv*d]
  void *k_cache, *v_cache;    // [B, Hkv, cap, d]
  int B, L, Hkv, dqk, dv, cap;
  int n_meta, window, is_global;
};
hymba_status kv_cache_emit(const KvEmitArgs &a, hymba_dtype dt, cudaStream_t s);

struct DecodeAttnArgs {
  const void *q;             // [B, H*dqk]
  const void *k_cache, *v_cache;  // [B, Hkv, cap, d]
  void *o;                   // [B, H*dv]
  float *partial;            // workspace
  int B, H, Hkv, dqk, dv, cap;
  long long pos;
  int n_meta, window, is_global;
  float scale;
  int fuse_later;            // bf16 tensor-core path: leave the run partials for fuse_decode
  // out (fuse_later): where the run partials of (sequence, head) start, see fuse_decode
  int nchunks_out;
  long long per_out;
};
size_t decode_attn_workspace_floats(int B, int H, int dv, long long pos, int n_meta, int window,
                                    int is_global);
// a.nchunks_out > 0 on return: the partials were left for fuse_decode (no output written)
hymba_status attention_decode(DecodeAttnArgs &a, hymba_dtype dt, cudaStream_t s);


// ---- decode SSM branch: conv + SiLU; x_proj (a GEMM); dt_proj + softplus + scan step + gate ----
struct DecodeSsmArgs {
  const void *x;       // [B, E] x_ssm of the new token, row stride ld_x
  long long ld_x;
  const void *z;       // [B, E] the gate SiLU(z), row stride ld_z
  long long ld_z;
  void *conv_state;    // [B, K-1, E] in/out
  const float *conv_w, *conv_b;  // [E, K], [E]
  long long *xacc;     // [B, R + 2N] delta_r, B, C of the new token as fixed-point integers
                       // (value * 2^32), zeroed beforehand, summed by the conv kernel's
                       // integer atomic adds (the same bits whatever the order)
  unsigned *xbad;      // [B] zeroed beforehand: set where a share was not finite or
                       // |share| >= 2^31 (that row's delta_r, B, C are then NaN)
  const void *w_x;     // [R + 2N, E] x_proj weights (dtype)
  void *u;             // [B, E] conv + SiLU output
  const float *w_dt, *b_dt;      // [E, R], [E]
  const float *a_log, *d_skip;   // [E, N], [E]
  float *h;            // [B, E, N] fp32 state, updated in place
  void *y;             // [B, E] gated output
  int B, E, K, R, N;
};
// u = SiLU(conv(window, x) + b), the conv window advanced in place, and x_proj:
// xacc += u W_x^T per channel block, in fixed point (xacc zeroed beforehand).
hymba_status decode_conv_xproj(const DecodeSsmArgs &a, hymba_dtype dt, cudaStream_t s);
// delta = softplus(delta_r W_dt^T + b_dt), one recurrence step, y = (C.h + D u) * gate.
hymba_status decode_scan(const DecodeSsmArgs &a, hymba_dtype dt, cudaStream_t s);

hymba_status mask_bitmap(int L, int n_meta, int window, int is_global, int path, uint32_t *bits,
                         uint8_t *tile_class, cudaStream_t s);
// The decode kernels' slot predicate for the query at `pos`, one bit per slot.
hymba_status decode_mask(long long pos, int n_meta, int window, int is_global, int capacity,
                         uint32_t *bits, cudaStream_t s);
// Rotary table: tab[p * hd/2 + i] = (cos, sin)((pos0 + p) * base^(-2i/hd)), p < npos.
hymba_status rope_table(float2 *tab, int npos, long long pos0, int hd, float base, cudaStream_t s);
// exp2 of n floats by the polynomial the attention softmax uses (degree 3 or 5).
hymba_status exp2_poly_eval(int degree, const float *x, float *y, long long n, cudaStream_t s);


// Cycle limit the kernels' bounded waits are launched with: HYMBA_WAIT_LIMIT from the
// environment, else hymba_set_wait_limit()'s value, else 1e9; never below 1e5.
long long wait_limit_cycles();
// One-shot diagnostic: 1 if the next prefill's output projection is to stall (consumed).
int take_debug_stall();

// Device error word bit for a bounded wait that gave up.
constexpr unsigned kErrTimeoutHost = 1u;
// Device error words of every translation unit: read and clear.
unsigned take_error_gemm();
unsigned take_error_attn();

// Counts kernel launches of this library (for the optional profiler).
void note_launch(int n = 1);

// Thread-local reason for the last failure.
void set_error(const char *fmt, ...);

}  // namespace hymba
